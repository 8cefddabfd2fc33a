// Instantiations of the tensor-core decode kernel for 2-bit keys (one translation
// unit per key width, so that the instantiations compile in parallel).

#include "decode_mma_impl.cuh"

namespace tq {
namespace mmadec {
cudaError_t launch_k2(const Args& a, int vb, int nt, bool qjl, bool rec, int grid, size_t smem, cudaStream_t s) {
    return launch_k<2>(a, vb, nt, qjl, rec, grid, smem, s);
}
}  // namespace mmadec
}  // namespace tq
