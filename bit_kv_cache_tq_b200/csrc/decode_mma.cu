// Host side of the tensor-core decode kernel (decode_mma_impl.cuh): which
// configurations it takes, the kernel arguments, the shared-memory plan and
// the launch.  The kernel's instantiations are spread over decode_mma_k*.cu,
// one file per key width, so that they compile in parallel.

#include "decode_mma_impl.cuh"

namespace tq {
namespace mmadec {
// one per key width (decode_mma_k2.cu, _k3.cu, _k4.cu, _k8.cu)
cudaError_t launch_k2(const Args& a, int vb, int nt, bool qjl, bool rec, int grid, size_t smem, cudaStream_t s);
cudaError_t launch_k3(const Args& a, int vb, int nt, bool qjl, bool rec, int grid, size_t smem, cudaStream_t s);
cudaError_t launch_k4(const Args& a, int vb, int nt, bool qjl, bool rec, int grid, size_t smem, cudaStream_t s);
cudaError_t launch_k8(const Args& a, int vb, int nt, bool qjl, bool rec, int grid, size_t smem, cudaStream_t s);
}  // namespace mmadec

bool decode_mma_supported(const tq_params& p) {
    // turbo keys (any bits, optional sketch) or int8 keys (no sketch); turbo
    // values, or int8 values beside int8 keys
    const bool keys = p.k_mode == TQ_MODE_TURBO ? p.qjl_dims <= 64 : (p.k_mode == TQ_MODE_INT8 && p.qjl_dims == 0);
    const bool values = p.v_mode == TQ_MODE_TURBO || (p.v_mode == TQ_MODE_INT8 && p.k_mode == TQ_MODE_INT8);
    return p.head_dim == 128 && keys && values && p.num_q_heads / p.num_kv_heads <= 16;
}

static uint16_t half_bits(double v) {
    const __half h = __float2half_rn(static_cast<float>(v));
    return *reinterpret_cast<const uint16_t*>(&h);
}

cudaError_t launch_decode_mma(const tq_params& p, const tq_codebook* kcb, const tq_codebook* vcb, const tq_cache& c,
                              const void* q, int q_dtype, const int32_t* seq_lens, int max_len, float* out,
                              const DecodePlan& plan, char* ws, uint32_t* err, int num_sms, cudaStream_t stream,
                              const void* k_new, const void* v_new, int new_dtype, const PageMap* pm,
                              uint32_t* skip_mask) {
    using namespace mmadec;
    const bool k_int8 = p.k_mode == TQ_MODE_INT8, v_int8 = p.v_mode == TQ_MODE_INT8;
    Args a{};
    a.append = k_new != nullptr;
    a.early = (p.flags & TQ_PARAM_PREFETCH_EARLY) ? 1 : 0;
    a.k_new = k_new;
    a.v_new = v_new;
    a.new_dtype = new_dtype;
    a.new_bytes = new_dtype == TQ_F32 ? 4 : 2;
    {
        // int8 keys: no boundaries, centroids or table entries
        const int hk = k_int8 ? 1 : 1 << (p.k_bits - 1), hv = v_int8 ? 1 : 1 << (p.v_bits - 1);
        for (int k = 0; k < 8; ++k) {
            a.kbound[k] = k < hk - 1 ? static_cast<float>(kcb->boundaries[hk + k]) : INFINITY;
            a.vbound[k] = k < hv - 1 ? static_cast<float>(vcb->boundaries[hv + k]) : INFINITY;
        }
        for (int j = 0; j < 16; ++j)
            a.kc32[j] = (!k_int8 && j < (1 << p.k_bits)) ? static_cast<float>(kcb->centroids[j]) : 0.f;
    }
    a.k_codes = c.k_codes;
    a.v_codes = c.v_codes;
    a.k_norms = c.k_norms;
    a.v_norms = c.v_norms;
    a.k_qjl = c.k_qjl;
    a.k_gamma = c.k_gamma;
    a.sketch = c.qjl_matrix;
    a.q = q;
    a.q_dtype = q_dtype;
    a.q_bytes = q_dtype == TQ_F32 ? 4 : 2;
    a.seq_lens = seq_lens;
    a.ws_ml = reinterpret_cast<float2*>(ws + plan.off_ml);
    a.ws_acc = reinterpret_cast<float*>(ws + plan.off_acc);
    a.counters = reinterpret_cast<uint32_t*>(ws + plan.off_counters);
    a.out = out;
    a.err = err;
    a.batch = c.batch;
    a.hq = p.num_q_heads;
    a.hkv = p.num_kv_heads;
    a.group = p.num_q_heads / p.num_kv_heads;
    a.capacity = c.capacity;
    a.n_split = plan.n_split;
    a.split_len = plan.split_len;
    a.max_len = max_len;
    a.units = c.batch * p.num_kv_heads;
    a.n_items = a.units * plan.n_split;
    a.m = p.qjl_dims;
    const float sm = p.sm_scale > 0.0f ? p.sm_scale : 1.0f / std::sqrt(128.0f);
    a.sm_scale_log2 = sm * LOG2E;
    a.tau = p.sparse_v_threshold;
    a.skip_mask = a.tau > 0.0f ? skip_mask : nullptr;
    a.mask_words = (max_len + 31) / 32;
    const double sd = std::sqrt(128.0);
    // int8 keys enter the products as exact integers (the scale rides in the norm)
    const double ak = k_int8 ? 1.0 : kcb->fp16_scale > 0.0 ? kcb->fp16_scale : sd;
    const double av = v_int8 ? 1.0 : vcb->fp16_scale > 0.0 ? vcb->fp16_scale : sd;
    a.inv_alpha_k = static_cast<float>(1.0 / ak);
    a.inv_alpha_v = static_cast<float>(1.0 / av);
    for (int j = 0; j < 16; ++j) {
        a.kcent[j] = (!k_int8 && j < (1 << p.k_bits)) ? half_bits(kcb->centroids[j] * ak) : 0;
        a.vcent[j] = (!v_int8 && j < (1 << p.v_bits)) ? half_bits(vcb->centroids[j] * av) : 0;
    }
    a.staged_norms = (c.capacity % 8) == 0;  // a paged pool's capacity is its block size, a multiple of 16
    if (pm) {
        a.table = pm->table;
        a.max_blocks = pm->max_blocks;
        a.block_size = pm->block_size;
        a.num_blocks = pm->num_blocks;
        a.batch = pm->batch;
        a.capacity = pm->max_blocks * pm->block_size;
        a.units = a.batch * p.num_kv_heads;
        a.n_items = a.units * plan.n_split;
        a.early = 0;  // the table itself may come from the previous kernel
    }
    uint32_t words[8];
    rotation_sign_bits(p.seed, 128, words);
    for (int i = 0; i < 4; ++i) a.signs[i] = words[i];
    int reserved = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        static_cast<uint32_t>(reserved) != WINDOW)
        return cudaErrorNotSupported;
    const int nt = a.group <= 8 ? 1 : 2;
    const int kb = k_int8 ? INT8_BITS : p.k_bits, vb = v_int8 ? INT8_BITS : p.v_bits;
    // as many stages as fit in 227 KB next to the tables and the merge buffers
    const Layout fixed = layout(kb, vb, nt, 0, p.qjl_dims, a.group, a.q_bytes, a.append ? a.new_bytes : 0, a.n_split);
    int stages = static_cast<int>((232448u - fixed.total) / fixed.stage_bytes);
    if (stages > 8) stages = 8;
    // fewer than two stages (an all-int8 layer with 16-head groups of fp32
    // queries: its 92 KB stages and query slots do not fit twice): the caller
    // takes the general kernels
    if (stages < 2) return cudaErrorNotSupported;
    a.stages = stages;
    const size_t smem =
        layout(kb, vb, nt, stages, p.qjl_dims, a.group, a.q_bytes, a.append ? a.new_bytes : 0, a.n_split).total;
    int grid = num_sms;
    if (grid > a.n_items) grid = a.n_items;
    const bool qjl = p.qjl_dims > 0;
    const bool rec = a.skip_mask != nullptr;
    switch (kb) {
        case INT8_BITS: return launch_k8(a, vb, nt, qjl, rec, grid, smem, stream);
        case 2: return launch_k2(a, vb, nt, qjl, rec, grid, smem, stream);
        case 3: return launch_k3(a, vb, nt, qjl, rec, grid, smem, stream);
        default: return launch_k4(a, vb, nt, qjl, rec, grid, smem, stream);
    }
}

}  // namespace tq
