// Instantiations of the tensor-core decode kernel for int8 keys (one translation
// unit per key width, so that the instantiations compile in parallel).

#include "decode_mma_impl.cuh"

namespace tq {
namespace mmadec {
cudaError_t launch_k8(const Args& a, int vb, int nt, bool qjl, bool rec, int grid, size_t smem, cudaStream_t s) {
    return launch_k<INT8_BITS>(a, vb, nt, qjl, rec, grid, smem, s);
}
}  // namespace mmadec
}  // namespace tq
