// Decode attention straight from the compressed cache (sm_100a), and its
// C entry point.
//
// Pages (by title):
//   [google]  "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！",
//             sections "再看速度" (attention from 4-bit TurboQuant keys) and
//             "第二步：QJL —— 1 bit 清理殘差"
//   [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命", section
//             "Sparse V：速度加成"
//   [tqai]    "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术",
//             section "TurboQuant的核心创新"
//
// Structure (flash-decoding): kernel 1 runs one thread block per (token
// split, kv head, sequence).  It rotates the G = Hq/Hkv queries of the kv
// head once (q~ = H diag(s) q / sqrt(d)), streams the split's packed keys and
// values, scores s_i = sm_scale * ||k_i|| * <q~, c[code_i]> (+ the QJL term
// gamma_i sqrt(pi/2)/m <S q~, 2z_i - 1>), keeps an online softmax, and sums
// p_i ||v_i|| c[code_i] in the rotated domain.  It writes (m, l, acc[d]) per
// query head.  Kernel 2 merges the splits by log-sum-exp and applies the one
// inverse rotation.  INT8 sides work in the original domain.
//
// This is the general path: every mode, bit width, head size and group size.

#include <cuda_runtime.h>

#include <cmath>

#include "device_common.cuh"
#include "internal.h"

namespace tq {

struct DecodeSide {
    const uint8_t* codes;
    const uint16_t* norms;
    int mode, bits, vbytes;
    float centroids[16];
};

struct DecodeArgs {
    DecodeSide k, v;
    const uint8_t* k_qjl;
    const uint16_t* k_gamma;
    const float* sketch;
    int m;
    const void* q;
    int q_dtype;
    const int32_t* seq_lens;
    int max_len;
    float2* ws_ml;    // [batch][hq][n_split]
    float* ws_acc;    // [batch][hq][n_split][d]
    float* out;       // [batch][hq][d]
    uint32_t* err;
    int batch, hq, hkv, group, capacity, n_split, split_len;
    float sm_scale, tau;
    uint32_t* skip_mask;  // Sparse V: [batch][hq][mask_words] bits of dropped positions, or null
    int mask_words;
    uint32_t signs[8];
};

constexpr int kDecodeWarps = 4;

// Values of the lane's V consecutive coordinates [lane*V, lane*V + V) of a
// stored vector.
template <int V>
__device__ __forceinline__ void load_lane_values(const DecodeSide& s, size_t slot, int lane, float (&out)[V]) {
    const uint8_t* row = s.codes + slot * static_cast<size_t>(s.vbytes);
    if (s.mode == TQ_MODE_INT8) {
#pragma unroll
        for (int e = 0; e < V; ++e) out[e] = static_cast<float>(static_cast<int8_t>(row[lane * V + e]));
        return;
    }
    const uint32_t bits = stream_bits(reinterpret_cast<const uint32_t*>(row), s.vbytes / 4, s.bits * lane * V,
                                      s.bits * V);
    const uint32_t mask = (1u << s.bits) - 1u;
#pragma unroll
    for (int e = 0; e < V; ++e) out[e] = s.centroids[(bits >> (s.bits * e)) & mask];
}

template <int D, int GMAX>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_split_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int V = D / 32;
    extern __shared__ float smem[];
    float* q_s = smem;                          // [GMAX][D]
    float* sq_s = q_s + GMAX * D;               // [GMAX][D]   S q~ (QJL)
    float* acc_s = sq_s + GMAX * D;             // [warps][GMAX][D]
    float* ml_s = acc_s + kDecodeWarps * GMAX * D;  // [warps][GMAX][2]

    const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int G = a.group;
    int len = a.seq_lens[b];
    if (len < 1 || len > a.capacity || len > a.max_len) {
        if (a.err && split == 0 && kv == 0 && threadIdx.x == 0) atomicOr(a.err, TQ_DEVERR_SEQLEN);
        len = 0;
    }
    const int s0 = split * a.split_len;
    const int s1 = min(len, s0 + a.split_len);
    const size_t slot_base = (static_cast<size_t>(b) * a.hkv + kv) * a.capacity;
    if (s0 >= s1) {
        if (threadIdx.x < G) {
            const size_t o = (static_cast<size_t>(b) * a.hq + kv * G + threadIdx.x) * a.n_split + split;
            a.ws_ml[o] = make_float2(-INFINITY, 0.0f);
        }
        return;
    }

    // queries of this kv head, rotated when K is stored rotated
    const bool k_rot = a.k.mode == TQ_MODE_TURBO;
    for (int h = warp; h < G; h += kDecodeWarps) {
        float x[V];
        const size_t qoff = (static_cast<size_t>(b) * a.hq + kv * G + h) * D + lane * V;
#pragma unroll
        for (int e = 0; e < V; ++e) x[e] = load_scalar(a.q, qoff + e, a.q_dtype);
        if (k_rot) {
#pragma unroll
            for (int e = 0; e < V; ++e) x[e] = flip_sign(x[e], sign_bit(a.signs, lane * V + e));
            fwht_registers(x);
            fwht_lanes<V, 32>(x, lane);
#pragma unroll
            for (int e = 0; e < V; ++e) x[e] *= rsqrtf(static_cast<float>(D));
        }
#pragma unroll
        for (int e = 0; e < V; ++e) q_s[h * D + lane * V + e] = x[e];
    }
    __syncthreads();
    if (a.m > 0) {
        for (int idx = threadIdx.x; idx < G * a.m; idx += blockDim.x) {
            const int h = idx / a.m, r = idx % a.m;
            const float* srow = a.sketch + static_cast<size_t>(r) * D;
            float acc = 0.0f;
            for (int i = 0; i < D; ++i) acc = fmaf(__ldg(srow + i), q_s[h * D + i], acc);
            sq_s[h * D + r] = acc;
        }
        __syncthreads();
    }

    const float qjl_coef = a.m > 0 ? sqrtf(0.5f * 3.14159265358979f) / a.m : 0.0f;
    float m_run[GMAX], l_run[GMAX], acc[GMAX][V];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.0f;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[h][e] = 0.0f;
    }

    for (int t = s0 + warp; t < s1; t += kDecodeWarps) {
        const size_t slot = slot_base + t;
        float kv_vals[V];
        load_lane_values<V>(a.k, slot, lane, kv_vals);
        const float k_norm = half_bits_to_float(a.k.norms[slot]);
        float part[GMAX];
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            part[h] = 0.0f;
            if (h < G) {
#pragma unroll
                for (int e = 0; e < V; ++e) part[h] = fmaf(q_s[h * D + lane * V + e], kv_vals[e], part[h]);
            }
        }
        if (a.m > 0) {
            const uint32_t* z = reinterpret_cast<const uint32_t*>(a.k_qjl + slot * static_cast<size_t>(a.m / 8));
            const float w = half_bits_to_float(a.k_gamma[slot]) * qjl_coef;
            for (int r = lane; r < a.m; r += 32) {
                const float sgn = (z[r >> 5] >> (r & 31)) & 1u ? w : -w;
#pragma unroll
                for (int h = 0; h < GMAX; ++h)
                    if (h < G) part[h] = fmaf(sgn, sq_s[h * D + r], part[h]);
            }
        }
#pragma unroll
        for (int h = 0; h < GMAX; ++h) part[h] = group_sum<32>(part[h]);
        load_lane_values<V>(a.v, slot, lane, kv_vals);
        const float v_norm = half_bits_to_float(a.v.norms[slot]);
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h >= G) continue;
            const float s = a.sm_scale * k_norm * part[h];
            const float m_new = fmaxf(m_run[h], s);
            const float corr = __expf(m_run[h] - m_new);
            const float p = __expf(s - m_new);
            l_run[h] = fmaf(l_run[h], corr, p);
            m_run[h] = m_new;
            // Sparse V: p / l_run is an upper bound on the exact weight
            const bool skip = a.tau > 0.0f && p < a.tau * l_run[h];
            if (skip && a.skip_mask && lane == 0)
                atomicOr(a.skip_mask + (static_cast<size_t>(b) * a.hq + kv * G + h) * a.mask_words + (t >> 5),
                         1u << (t & 31));
            const float pv = skip ? 0.0f : p * v_norm;
#pragma unroll
            for (int e = 0; e < V; ++e) acc[h][e] = fmaf(acc[h][e], corr, pv * kv_vals[e]);
        }
    }

    // merge the warps of the block
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
        if (h >= G) continue;
#pragma unroll
        for (int e = 0; e < V; ++e) acc_s[(warp * GMAX + h) * D + lane * V + e] = acc[h][e];
        if (lane == 0) {
            ml_s[(warp * GMAX + h) * 2] = m_run[h];
            ml_s[(warp * GMAX + h) * 2 + 1] = l_run[h];
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, c = idx % D;
        float mx = -INFINITY;
        for (int w = 0; w < kDecodeWarps; ++w) mx = fmaxf(mx, ml_s[(w * GMAX + h) * 2]);
        float l = 0.0f, s = 0.0f;
        for (int w = 0; w < kDecodeWarps; ++w) {
            const float mw = ml_s[(w * GMAX + h) * 2];
            if (mw == -INFINITY) continue;
            const float f = __expf(mw - mx);
            l = fmaf(ml_s[(w * GMAX + h) * 2 + 1], f, l);
            s = fmaf(acc_s[(w * GMAX + h) * D + c], f, s);
        }
        const size_t o = (static_cast<size_t>(b) * a.hq + kv * G + h) * a.n_split + split;
        a.ws_acc[o * D + c] = s;
        if (c == 0) a.ws_ml[o] = make_float2(mx, l);
    }
}

template <int D>
__global__ void __launch_bounds__(32) decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int V = D / 32;
    const int hq = blockIdx.x, b = blockIdx.y, lane = threadIdx.x;
    const size_t base = (static_cast<size_t>(b) * a.hq + hq) * a.n_split;
    float mx = -INFINITY;
    for (int s = lane; s < a.n_split; s += 32) {
        const float2 ml = a.ws_ml[base + s];
        if (ml.y > 0.0f) mx = fmaxf(mx, ml.x);
    }
    mx = group_max<32>(mx);
    float l = 0.0f, o[V];
#pragma unroll
    for (int e = 0; e < V; ++e) o[e] = 0.0f;
    if (mx > -INFINITY) {
        for (int s = 0; s < a.n_split; ++s) {
            const float2 ml = a.ws_ml[base + s];
            if (!(ml.y > 0.0f)) continue;
            const float f = __expf(ml.x - mx);
            l = fmaf(ml.y, f, l);
            const float* src = a.ws_acc + (base + s) * D + lane * V;
#pragma unroll
            for (int e = 0; e < V; ++e) o[e] = fmaf(src[e], f, o[e]);
        }
    }
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
    for (int e = 0; e < V; ++e) o[e] *= inv;
    if (a.v.mode == TQ_MODE_TURBO) {
        fwht_registers(o);
        fwht_lanes<V, 32>(o, lane);
#pragma unroll
        for (int e = 0; e < V; ++e) o[e] = flip_sign(o[e] * rsqrtf(static_cast<float>(D)), sign_bit(a.signs, lane * V + e));
    }
    float* dst = a.out + (static_cast<size_t>(b) * a.hq + hq) * D + lane * V;
#pragma unroll
    for (int e = 0; e < V; ++e) dst[e] = o[e];
}

static void fill_decode_side(DecodeSide& s, int mode, int bits, int d, const tq_codebook* cb, const uint8_t* codes,
                             const uint16_t* norms) {
    s.codes = codes;
    s.norms = norms;
    s.mode = mode;
    s.bits = mode == TQ_MODE_INT8 ? 8 : bits;
    s.vbytes = vector_bytes(mode, bits, d);
    for (int j = 0; j < 16; ++j) s.centroids[j] = 0.0f;
    if (mode == TQ_MODE_TURBO)
        for (int j = 0; j < (1 << bits); ++j) s.centroids[j] = static_cast<float>(cb->centroids[j]);
}

template <int D, int GMAX>
static cudaError_t launch_decode_general(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(float) * (2 * GMAX * D + kDecodeWarps * GMAX * D + kDecodeWarps * GMAX * 2);
    if (smem > 48 * 1024) {  // opt in per call: the attribute belongs to the current device
        cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, GMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    decode_split_kernel<D, GMAX><<<dim3(a.n_split, a.hkv, a.batch), kDecodeWarps * 32, smem, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<D><<<dim3(a.hq, a.batch), 32, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_decode_dim(const DecodeArgs& a, cudaStream_t stream) {
    if (a.group <= 4) return launch_decode_general<D, 4>(a, stream);
    if (a.group <= 8) return launch_decode_general<D, 8>(a, stream);
    return launch_decode_general<D, 16>(a, stream);
}

// k_new / v_new non-null: append mode (one new token per sequence at seq_len - 1).
// pm non-null: c is the pool of a paged cache.
cudaError_t launch_decode_mma(const tq_params& p, const tq_codebook* kcb, const tq_codebook* vcb, const tq_cache& c,
                              const void* q, int q_dtype, const int32_t* seq_lens, int max_len, float* out,
                              const DecodePlan& plan, char* ws, uint32_t* err, int num_sms, cudaStream_t stream,
                              const void* k_new = nullptr, const void* v_new = nullptr, int new_dtype = 0,
                              const PageMap* pm = nullptr, uint32_t* skip_mask = nullptr);

}  // namespace tq

namespace tq {
// Decode attention; with k_new / v_new set, the step's new token of every
// sequence is first written at position seq_len - 1 (append mode).  With a
// block table, `cache` is the pool of a paged cache (tensor-core path only).
static tq_status decode_impl(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                             const void* d_q, tq_dtype q_dtype, const tq_cache* cache, const int32_t* d_seq_lens,
                             int32_t max_seq_len, float* d_out, void* d_workspace, size_t workspace_bytes,
                             uint32_t* d_skip_mask, uint32_t* d_error, void* stream, const void* k_new,
                             const void* v_new, tq_dtype kv_dtype, const tq_block_table* table = nullptr) {
    tq_status st = validate_params(params);
    if (st != TQ_OK) return st;
    const tq_params& p = *params;
    PageMap pages;
    const PageMap* pm = nullptr;
    if (table) {
        if ((st = validate_pages(p, cache, table, &pages)) != TQ_OK) return st;
        pm = &pages;
    } else if ((st = validate_cache(p, cache)) != TQ_OK) {
        return st;
    }
    const int batch = pm ? pm->batch : cache->batch;
    if (!d_q || !d_seq_lens || !d_out || !d_workspace || max_seq_len < 1) return TQ_ERR_INVALID_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16 && q_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
    if (!aligned16(d_q) || !aligned16(d_out) || !aligned16(d_workspace)) return TQ_ERR_ALIGNMENT;
    if (d_skip_mask && (reinterpret_cast<uintptr_t>(d_skip_mask) & 3u)) return TQ_ERR_ALIGNMENT;
    if (p.k_mode == TQ_MODE_TURBO && (st = validate_codebook(kcb, p.head_dim, p.k_bits)) != TQ_OK) return st;
    if (p.v_mode == TQ_MODE_TURBO && (st = validate_codebook(vcb, p.head_dim, p.v_bits)) != TQ_OK) return st;
    const bool append = k_new != nullptr;
    if (append) {
        if (!v_new) return TQ_ERR_INVALID_ARG;
        if (kv_dtype != TQ_F32 && kv_dtype != TQ_BF16 && kv_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
        if (!aligned16(k_new) || !aligned16(v_new)) return TQ_ERR_ALIGNMENT;
    }
    const int sms = num_sms_current();
    if (sms <= 0) return TQ_ERR_CUDA;
    const DecodePlan plan = plan_decode(p, batch, max_seq_len, sms, workspace_bytes, !decode_mma_supported(p));
    if (workspace_bytes < plan.bytes) return TQ_ERR_CAPACITY;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (decode_mma_supported(p)) {
        const cudaError_t e = launch_decode_mma(p, kcb, vcb, *cache, d_q, q_dtype, d_seq_lens, max_seq_len, d_out, plan,
                                                static_cast<char*>(d_workspace), d_error, sms, s, k_new, v_new,
                                                kv_dtype, pm, d_skip_mask);
        if (e != cudaErrorNotSupported) return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
        // otherwise (shared memory too small for two stages, or a device whose
        // shared-memory window differs) take the general path
    }
    if (pm) return TQ_ERR_UNSUPPORTED;  // the general kernels read contiguous caches only
    if (append) {  // two launches: append, then attend
        st = quantize_append_impl(params, kcb, vcb, k_new, v_new, kv_dtype, 1, d_seq_lens, true, cache, d_error,
                                  stream);
        if (st != TQ_OK) return st;
    }
    DecodeArgs a{};
    fill_decode_side(a.k, p.k_mode, p.k_bits, p.head_dim, kcb, cache->k_codes, cache->k_norms);
    fill_decode_side(a.v, p.v_mode, p.v_bits, p.head_dim, vcb, cache->v_codes, cache->v_norms);
    a.k_qjl = cache->k_qjl;
    a.k_gamma = cache->k_gamma;
    a.sketch = cache->qjl_matrix;
    a.m = p.qjl_dims;
    a.q = d_q;
    a.q_dtype = q_dtype;
    a.seq_lens = d_seq_lens;
    a.max_len = max_seq_len;
    char* ws = static_cast<char*>(d_workspace);
    a.ws_ml = reinterpret_cast<float2*>(ws + plan.off_ml);
    a.ws_acc = reinterpret_cast<float*>(ws + plan.off_acc);
    a.out = d_out;
    a.err = d_error;
    a.batch = cache->batch;
    a.hq = p.num_q_heads;
    a.hkv = p.num_kv_heads;
    a.group = p.num_q_heads / p.num_kv_heads;
    a.capacity = cache->capacity;
    a.n_split = plan.n_split;
    a.split_len = plan.split_len;
    a.sm_scale = p.sm_scale > 0.0f ? p.sm_scale : 1.0f / std::sqrt(static_cast<float>(p.head_dim));
    a.tau = p.sparse_v_threshold;
    a.skip_mask = a.tau > 0.0f ? d_skip_mask : nullptr;
    a.mask_words = (max_seq_len + 31) / 32;
    rotation_sign_bits(p.seed, p.head_dim, a.signs);
    cudaError_t e;
    switch (p.head_dim) {
        case 64: e = launch_decode_dim<64>(a, s); break;
        case 128: e = launch_decode_dim<128>(a, s); break;
        default: e = launch_decode_dim<256>(a, s); break;
    }
    return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
}  // namespace tq

extern "C" tq_status tq_decode_attention(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                         const void* d_q, tq_dtype q_dtype, const tq_cache* cache,
                                         const int32_t* d_seq_lens, int32_t max_seq_len, float* d_out,
                                         void* d_workspace, size_t workspace_bytes, uint32_t* d_skip_mask,
                                         uint32_t* d_error, void* stream) {
    return tq::decode_impl(params, kcb, vcb, d_q, q_dtype, cache, d_seq_lens, max_seq_len, d_out, d_workspace,
                           workspace_bytes, d_skip_mask, d_error, stream, nullptr, nullptr, TQ_BF16);
}

extern "C" tq_status tq_decode_attention_paged(const tq_params* params, const tq_codebook* kcb,
                                               const tq_codebook* vcb, const void* d_q, tq_dtype q_dtype,
                                               const tq_cache* pool, const tq_block_table* table,
                                               const int32_t* d_seq_lens, int32_t max_seq_len, float* d_out,
                                               void* d_workspace, size_t workspace_bytes, uint32_t* d_skip_mask,
                                               uint32_t* d_error, void* stream) {
    if (!table) return TQ_ERR_INVALID_ARG;
    return tq::decode_impl(params, kcb, vcb, d_q, q_dtype, pool, d_seq_lens, max_seq_len, d_out, d_workspace,
                           workspace_bytes, d_skip_mask, d_error, stream, nullptr, nullptr, TQ_BF16, table);
}

extern "C" tq_status tq_append_decode_attention_paged(const tq_params* params, const tq_codebook* kcb,
                                                      const tq_codebook* vcb, const void* k_new, const void* v_new,
                                                      tq_dtype kv_dtype, const void* d_q, tq_dtype q_dtype,
                                                      const tq_cache* pool, const tq_block_table* table,
                                                      const int32_t* d_seq_lens, int32_t max_seq_len, float* d_out,
                                                      void* d_workspace, size_t workspace_bytes,
                                                      uint32_t* d_skip_mask, uint32_t* d_error, void* stream) {
    if (!k_new || !v_new || !table) return TQ_ERR_INVALID_ARG;
    return tq::decode_impl(params, kcb, vcb, d_q, q_dtype, pool, d_seq_lens, max_seq_len, d_out, d_workspace,
                           workspace_bytes, d_skip_mask, d_error, stream, k_new, v_new, kv_dtype, table);
}

extern "C" tq_status tq_append_decode_attention(const tq_params* params, const tq_codebook* kcb,
                                                const tq_codebook* vcb, const void* k_new, const void* v_new,
                                                tq_dtype kv_dtype, const void* d_q, tq_dtype q_dtype,
                                                const tq_cache* cache, const int32_t* d_seq_lens,
                                                int32_t max_seq_len, float* d_out, void* d_workspace,
                                                size_t workspace_bytes, uint32_t* d_skip_mask, uint32_t* d_error,
                                                void* stream) {
    if (!k_new || !v_new) return TQ_ERR_INVALID_ARG;
    return tq::decode_impl(params, kcb, vcb, d_q, q_dtype, cache, d_seq_lens, max_seq_len, d_out, d_workspace,
                           workspace_bytes, d_skip_mask, d_error, stream, k_new, v_new, kv_dtype);
}

// ---------------------------------------------------------------------------
// Decode attention with library-owned scratch.  Some callers cannot allocate
// device memory at the point of the call: an allocator hook that must not
// recurse into allocation, a runtime whose memory pool is fixed before
// serving starts, or code that runs while another component holds the
// allocator.  For them the split partials and counters live in one fixed
// device array of this library, so a call allocates nothing.  The array is
// shared by every call on a device and keeps the last call's partials; calls
// that overlap on the device race on it.

namespace tq {
namespace {

__device__ __align__(256) unsigned char g_static_scratch[TQ_DECODE_STATIC_SCRATCH_BYTES];

// Address of the current device's scratch array, looked up on every call (a
// host query that allocates nothing; nothing cached survives a device reset),
// and a zero fill of the counter words a call over `units` (sequence, kv
// head) pairs uses, queued on `stream` ahead of the call's kernels.  Every
// call therefore starts from zeroed counters, whatever the previous call on
// the array left behind (one that ended with TQ_DEVERR_TIMEOUT included).
cudaError_t static_scratch(void** out, long long units, cudaStream_t stream) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess) return e;
    const size_t counter_bytes = static_cast<size_t>(units + kGlobalCounters) * sizeof(uint32_t);
    e = cudaMemsetAsync(ptr, 0, counter_bytes, stream);
    if (e != cudaSuccess) return e;
    *out = ptr;
    return cudaSuccess;
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_decode_attention_static(const tq_params* params, const tq_codebook* kcb,
                                                const tq_codebook* vcb, const void* d_q, tq_dtype q_dtype,
                                                const tq_cache* cache, const int32_t* d_seq_lens,
                                                int32_t max_seq_len, float* d_out, uint32_t* d_error, void* stream) {
    using namespace tq;
    tq_status st = validate_params(params);
    if (st != TQ_OK) return st;
    if ((st = validate_cache(*params, cache)) != TQ_OK) return st;
    if (max_seq_len < 1) return TQ_ERR_INVALID_ARG;
    // Reject calls whose partials cannot fit before touching the device.
    const int sms = num_sms_current();
    if (sms <= 0) return TQ_ERR_CUDA;
    if (plan_decode(*params, cache->batch, max_seq_len, sms, TQ_DECODE_STATIC_SCRATCH_BYTES,
                    !decode_mma_supported(*params)).bytes >
        TQ_DECODE_STATIC_SCRATCH_BYTES)
        return TQ_ERR_CAPACITY;
    void* scratch = nullptr;
    const long long units = static_cast<long long>(cache->batch) * params->num_kv_heads;
    if (static_scratch(&scratch, units, static_cast<cudaStream_t>(stream)) != cudaSuccess) return TQ_ERR_CUDA;
    return tq_decode_attention(params, kcb, vcb, d_q, q_dtype, cache, d_seq_lens, max_seq_len, d_out, scratch,
                               TQ_DECODE_STATIC_SCRATCH_BYTES, nullptr, d_error, stream);
}

// Fill the counter region of the static array (the words a static call's
// own zero fill covers, for any batch) with the byte `value`, on `stream`;
// nothing is allocated.  0 is a full reset; other values stand for whatever
// an interrupted call could leave there.
extern "C" tq_status tq_decode_static_fill(uint8_t value, void* stream) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, tq::g_static_scratch) != cudaSuccess) return TQ_ERR_CUDA;
    const size_t bytes = tq::counter_region_bytes(TQ_DECODE_STATIC_SCRATCH_BYTES);
    return cudaMemsetAsync(ptr, value, bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TQ_OK
                                                                                              : TQ_ERR_CUDA;
}
