// Chunked prefill attention from the compressed cache on the 5th-generation
// tensor cores (sm_100a, tcgen05 with tensor-memory accumulators).
//
// Pages (by title):
//   [google]  "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！", table
//             "M5 Max 128GB 上的實測" (prefill speed with TurboQuant caches)
//   [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命", table "性能表现"
//   [tqai]    "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术", section
//             "TurboQuant的核心创新" (the encoding being read)
//
// What is computed: a chunk of C new tokens of every sequence is first
// appended to the cache (the quantise kernel), then query j of sequence b
// attends causally to cache positions 0 .. start_b + j, exactly as a decode
// step over start_b + j + 1 tokens would:
//   s_i = sm_scale ||k_i|| <q~, c[code_i]>,  p = softmax(s),
//   out = R^-1( sum_i p_i ||v_i|| c[code_i] ).
//
// How: one thread block per (sequence, kv head, 128 query rows), a row being
// one (query token, head of the GQA group).  The rotated query rows, scaled
// to a largest magnitude of 1, enter as two fp16 terms (the rounded value
// and its remainder, two MMAs into the same accumulator), so the scores keep
// about 22 bits of the query.  Per 64-key tile the block
// dequantises the packed codes into fp16 tiles in shared memory, laid out as
// the tensor cores read them (K-major, 128-byte swizzle): K~ [64 keys x 128
// channels] and V~^T [128 channels x 64 keys], centroids only (the norms
// scale the scores and the softmax weights instead).  One thread issues
// S = Q~ K~^T (M = 128, N = 64, K = 128) into tensor memory; each thread then
// owns one query row: it reads its scores from tensor memory, applies the key
// norms, the causal limit and the online softmax, and writes its weights
// p_i ||v_i|| (fp16) back as the A operand of O_tile = P V~ (M = 128, N = 128,
// K = 64), whose tensor-memory result it adds to its fp32 row accumulator.
// The end divides by the softmax sum and applies the inverse rotation.  The
// keys' fp16 centroids carry the codebook's fp16 scale (as in the decode
// kernels), removed from the scores and the output.
//
// Every mbarrier wait is bounded (about a second; TQ_DEVERR_TIMEOUT, the
// block stops issuing work and still frees its tensor memory).

#include <cuda_runtime.h>

#include <cmath>

#include "device_common.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace tq {
namespace prefill {

constexpr int D = 128;
constexpr int BM = 128;                  // query rows per block
constexpr int BK = 64;                   // keys per tile
constexpr int NTHREADS = 128;            // one thread per query row
constexpr uint32_t TMEM_COLS = 256;      // S at column 0 (64 columns), O at column 128 (128 columns)
constexpr uint32_t TMEM_S = 0, TMEM_O = 128;
constexpr long long WAIT_LIMIT = 2000000000ll;  // clock cycles (~1 s)

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_Q = 0;                     // fp16 [128 rows][128 ch], 2 column blocks of 16 KB
constexpr uint32_t SM_QLO = SM_Q + BM * D * 2;   // fp16 remainder q~ - fp16(q~), same layout
constexpr uint32_t SM_K = SM_QLO + BM * D * 2;   // fp16 [64 keys][128 ch], 2 column blocks of 8 KB
constexpr uint32_t SM_VT = SM_K + BK * D * 2;    // fp16 [128 ch][64 keys], 1 column block
constexpr uint32_t SM_P = SM_VT + D * BK * 2;    // fp16 [128 rows][64 keys], 1 column block
constexpr uint32_t SM_KC = SM_P + BM * BK * 2;   // packed key codes of the tile [64][16 kb]
constexpr uint32_t SM_VC = SM_KC + BK * 64;      // packed value codes of the tile [64][16 vb]
constexpr uint32_t SM_KN = SM_VC + BK * 64;      // float key norms [64]
constexpr uint32_t SM_VN = SM_KN + BK * 4;       // float value norms [64]
constexpr uint32_t SM_CENT = SM_VN + BK * 4;     // fp16 key centroids [16], value centroids [16]
constexpr uint32_t SM_BAR = SM_CENT + 64;        // mbarrier
constexpr uint32_t SM_TMEM = SM_BAR + 8;         // tensor-memory address
constexpr uint32_t SM_FLAG = SM_TMEM + 4;        // abort flag
constexpr uint32_t SM_BYTES = SM_FLAG + 4;
constexpr uint32_t SM_ALLOC = SM_BYTES + 1024;   // room to align the base

struct Args {
    const uint8_t* k_codes;
    const uint8_t* v_codes;
    const uint16_t* k_norms;
    const uint16_t* v_norms;
    const void* q;           // [batch][n_new][hq][d]
    const int32_t* positions;
    float* out;              // [batch][n_new][hq][d]
    uint32_t* err;
    int q_dtype, batch, hq, hkv, group, capacity, n_new, tok_per_tile, kb, vb;
    float score_scale;       // sm_scale * log2(e) / alpha_k
    float inv_alpha_v;
    uint32_t signs[4];
    uint16_t kcent[16];      // fp16 bits of alpha_k * key centroid
    uint16_t vcent[16];
};

// Unnormalised Walsh-Hadamard butterflies over the 128 values a thread holds
// (Sylvester order).
__device__ __forceinline__ void fwht128(float (&x)[D]) {
#pragma unroll
    for (int h = 1; h < D; h <<= 1)
#pragma unroll
        for (int i = 0; i < D; ++i)
            if ((i & h) == 0) {
                const float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
}

__device__ __forceinline__ uint32_t pack2(uint16_t lo, uint16_t hi) { return lo | (static_cast<uint32_t>(hi) << 16); }

// code `i` of a packed row (LSB-first bitstream of `bits`-bit codes) held in
// shared memory as 32-bit words
__device__ __forceinline__ uint32_t code_at(const uint32_t* row, int i, int bits) {
    const int bit = bits * i;
    const uint32_t lo = row[bit >> 5];
    const int sh = bit & 31;
    uint32_t v = lo >> sh;
    if (sh + bits > 32) v |= row[(bit >> 5) + 1] << (32 - sh);
    return v & ((1u << bits) - 1u);
}

__global__ void __launch_bounds__(NTHREADS, 1) prefill_kernel(const __grid_constant__ Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int qt = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
    const int G = a.group, TT = a.tok_per_tile;
    const int tok0 = qt * TT;
    const uint32_t bar = sbase + SM_BAR;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_FLAG);

    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (tid < 32) {
        reinterpret_cast<uint16_t*>(smem + SM_CENT)[tid] = tid < 16 ? a.kcent[tid] : a.vcent[tid - 16];
    }
    if (warp == 0) {
        tc::tmem_alloc(sbase + SM_TMEM, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SM_TMEM);
    const uint16_t* kcent = reinterpret_cast<const uint16_t*>(smem + SM_CENT);
    const uint16_t* vcent = kcent + 16;

    // the chunk's first cache slot; an out-of-range start gives zeros
    const int start = a.positions[b];
    const bool bad = start < 0 || start > a.capacity - a.n_new;
    if (bad && qt == 0 && kv == 0 && tid == 0 && a.err) atomicOr(a.err, TQ_DEVERR_POSITION);
    const int ntok = bad ? 0 : min(TT, a.n_new - tok0);  // query tokens of this block

    // ---- this thread's query row: token tok0 + r / G, head kv * G + r % G
    const int r = tid;
    const int rt = r / G, rh = r % G;
    const bool row_ok = rt < ntok && rt * G + rh < BM;
    float qscale = 0.f;  // largest |q~| of the row: the fp16 terms hold q~ / qscale
    {
        float x[D];
        if (row_ok) {
            const size_t qoff = ((static_cast<size_t>(b) * a.n_new + tok0 + rt) * a.hq + kv * G + rh) * D;
#pragma unroll
            for (int c = 0; c < D; c += 4) {
                float v4[4];
                load4(a.q, qoff + c, a.q_dtype, v4);
#pragma unroll
                for (int e = 0; e < 4; ++e) x[c + e] = flip_sign(v4[e], (a.signs[(c + e) >> 5] >> ((c + e) & 31)) & 1u);
            }
            fwht128(x);
        } else {
#pragma unroll
            for (int c = 0; c < D; ++c) x[c] = 0.f;
        }
        float amax = 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) amax = fmaxf(amax, fabsf(x[c]));
        const float inv_sqrt_d = 0.08838834764831845f;
        qscale = amax * inv_sqrt_d;
        const float rs = amax > 0.f ? 1.f / amax : 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 8) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float u0 = x[c + 2 * e] * rs, u1 = x[c + 2 * e + 1] * rs;
                const __half h0 = __float2half_rn(u0), h1 = __float2half_rn(u1);
                hw[e] = pack2(__half_as_ushort(h0), __half_as_ushort(h1));
                lw[e] = pack2(__half_as_ushort(__float2half_rn(u0 - __half2float(h0))),
                              __half_as_ushort(__float2half_rn(u1 - __half2float(h1))));
            }
            *reinterpret_cast<uint4*>(smem + SM_Q + tc::sw128_offset(r, c, BM)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(smem + SM_QLO + tc::sw128_offset(r, c, BM)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
    }
    const float row_scale = qscale * a.score_scale;  // scores: S * ||k|| * row_scale (log2 units)
    const int qpos = start + tok0 + rt;                       // this row's own position: the causal limit
    const int kend = ntok > 0 ? start + tok0 + ntok : 0;      // keys [0, kend) are needed by some row
    const int ntiles = (kend + BK - 1) / BK;
    const int kbytes = 16 * a.kb, vbytes = 16 * a.vb;         // packed row sizes
    const size_t unit_row = (static_cast<size_t>(b) * a.hkv + kv) * a.capacity;

    float o[D];
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] = 0.f;
    float m = -INFINITY, l = 0.f;
    uint32_t phase = 0;
    const uint32_t idesc_s = tc::idesc_f16(BM, BK), idesc_o = tc::idesc_f16(BM, D);
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

    for (int tile = 0; tile < ntiles; ++tile) {
        const int key0 = tile * BK;
        const int nk = min(BK, kend - key0);  // keys of this tile below kend (all within the cache)
        // ---- stage the tile's packed codes and norms (coalesced 16-byte loads)
        {
            const uint4* ksrc = reinterpret_cast<const uint4*>(a.k_codes + (unit_row + key0) * kbytes);
            const uint4* vsrc = reinterpret_cast<const uint4*>(a.v_codes + (unit_row + key0) * vbytes);
            uint4* kdst = reinterpret_cast<uint4*>(smem + SM_KC);
            uint4* vdst = reinterpret_cast<uint4*>(smem + SM_VC);
            const int kwords = nk * kbytes / 16, vwords = nk * vbytes / 16;
            for (int i = tid; i < kwords; i += NTHREADS) kdst[i] = ksrc[i];
            for (int i = tid; i < vwords; i += NTHREADS) vdst[i] = vsrc[i];
            if (tid < BK) {
                float* kn = reinterpret_cast<float*>(smem + SM_KN);
                float* vn = reinterpret_cast<float*>(smem + SM_VN);
                kn[tid] = tid < nk ? half_bits_to_float(a.k_norms[unit_row + key0 + tid]) : 0.f;
                vn[tid] = tid < nk ? half_bits_to_float(a.v_norms[unit_row + key0 + tid]) : 0.f;
            }
        }
        __syncthreads();
        // ---- dequantise: K~ [64 keys][128 ch] and V~^T [128 ch][64 keys]
        for (int it = tid; it < BK * (D / 8); it += NTHREADS) {
            const int key = it / (D / 8), cg = it % (D / 8);  // 8 channels 8 cg .. 8 cg + 7
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (key < nk) {
                const uint32_t* row = reinterpret_cast<const uint32_t*>(smem + SM_KC + key * kbytes);
                uint16_t h[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) h[e] = kcent[code_at(row, 8 * cg + e, a.kb)];
                w = make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
            }
            *reinterpret_cast<uint4*>(smem + SM_K + tc::sw128_offset(key, 8 * cg, BK)) = w;
        }
        for (int it = tid; it < D * (BK / 8); it += NTHREADS) {
            const int ch = it % D, kg = it / D;  // channel ch of keys 8 kg .. 8 kg + 7
            uint16_t h[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int key = 8 * kg + e;
                h[e] = 0;
                if (key < nk) {
                    const uint32_t* row = reinterpret_cast<const uint32_t*>(smem + SM_VC + key * vbytes);
                    h[e] = vcent[code_at(row, ch, a.vb)];
                }
            }
            const uint4 w = make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
            *reinterpret_cast<uint4*>(smem + SM_VT + tc::sw128_offset(ch, 8 * kg, D)) = w;
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        // ---- S = (Q~hi + Q~lo) K~^T
        if (tid == 0 && !*abort_flag) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t blk = ks >> 2, within = (ks & 3) * 32;
                const uint64_t bd = tc::sw128_desc(sbase + SM_K + blk * (BK * 128) + within);
                tc::mma_f16(tmem + TMEM_S, tc::sw128_desc(sbase + SM_Q + blk * (BM * 128) + within), bd, idesc_s,
                            ks > 0);
                tc::mma_f16(tmem + TMEM_S, tc::sw128_desc(sbase + SM_QLO + blk * (BM * 128) + within), bd, idesc_s,
                            true);
            }
            tc::commit(bar);
        }
        if (!*abort_flag && !ptx::mbar_wait_bounded(bar, phase & 1, WAIT_LIMIT)) {
            if (a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
        ++phase;
        tc::fence_after_sync();
        // ---- online softmax of this row over the tile: one pass over the
        // scores in tensor memory for the maximum, a second one for the
        // weights (rereading tensor memory is cheaper than holding 64 scores)
        {
            float sv[32];
            const float* kn = reinterpret_cast<const float*>(smem + SM_KN);
            const float* vn = reinterpret_cast<const float*>(smem + SM_VN);
            float mt = -INFINITY;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::ld_32cols(tmem + lane_base + TMEM_S + 32 * half, sv);
                tc::ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int key = key0 + 32 * half + j;
                    if (row_ok && key <= qpos) mt = fmaxf(mt, sv[j] * kn[32 * half + j] * row_scale);
                }
            }
            const float mn = fmaxf(m, mt);
            const float corr = (m == -INFINITY) ? 0.f : ptx::ex2(m - mn);
            float ls = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::ld_32cols(tmem + lane_base + TMEM_S + 32 * half, sv);
                tc::ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int key = key0 + 32 * half + j;
                    const float e = (row_ok && key <= qpos) ? ptx::ex2(sv[j] * kn[32 * half + j] * row_scale - mn)
                                                            : 0.f;
                    ls += e;
                    sv[j] = e * vn[32 * half + j];
                }
#pragma unroll
                for (int c = 0; c < 32; c += 8) {
                    uint4 w;
                    w.x = pack2(__half_as_ushort(__float2half_rn(sv[c])), __half_as_ushort(__float2half_rn(sv[c + 1])));
                    w.y = pack2(__half_as_ushort(__float2half_rn(sv[c + 2])), __half_as_ushort(__float2half_rn(sv[c + 3])));
                    w.z = pack2(__half_as_ushort(__float2half_rn(sv[c + 4])), __half_as_ushort(__float2half_rn(sv[c + 5])));
                    w.w = pack2(__half_as_ushort(__float2half_rn(sv[c + 6])), __half_as_ushort(__float2half_rn(sv[c + 7])));
                    *reinterpret_cast<uint4*>(smem + SM_P + tc::sw128_offset(r, 32 * half + c, BM)) = w;
                }
            }
            l = l * corr + ls;
            m = mn;
#pragma unroll
            for (int c = 0; c < D; ++c) o[c] *= corr;
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        // ---- O_tile = P V~
        if (tid == 0 && !*abort_flag) {
#pragma unroll
            for (int ks = 0; ks < BK / 16; ++ks) {
                const uint64_t ad = tc::sw128_desc(sbase + SM_P + ks * 32);
                const uint64_t bd = tc::sw128_desc(sbase + SM_VT + ks * 32);
                tc::mma_f16(tmem + TMEM_O, ad, bd, idesc_o, ks > 0);
            }
            tc::commit(bar);
        }
        if (!*abort_flag && !ptx::mbar_wait_bounded(bar, phase & 1, WAIT_LIMIT)) {
            if (a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
        ++phase;
        tc::fence_after_sync();
        {
            float ov[32];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                tc::ld_32cols(tmem + lane_base + TMEM_O + 32 * q4, ov);
                tc::ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) o[32 * q4 + j] += ov[j];
            }
        }
        // every thread's tensor-memory reads and shared-memory uses of this
        // tile are done before the next tile's operands and MMAs
        tc::fence_before_sync();
        if (__syncthreads_or(*abort_flag)) break;
        tc::fence_after_sync();
    }

    // ---- epilogue: normalise, undo the value scale, inverse rotation
    if (row_ok) {
        const float inv = l > 0.f ? a.inv_alpha_v / l : 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) o[c] *= inv;
        fwht128(o);
        const float inv_sqrt_d = 0.08838834764831845f;
        float* dst = a.out + ((static_cast<size_t>(b) * a.n_new + tok0 + rt) * a.hq + kv * G + rh) * D;
#pragma unroll
        for (int c = 0; c < D; c += 4) {
            float4 v;
            v.x = flip_sign(o[c] * inv_sqrt_d, (a.signs[c >> 5] >> (c & 31)) & 1u);
            v.y = flip_sign(o[c + 1] * inv_sqrt_d, (a.signs[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u);
            v.z = flip_sign(o[c + 2] * inv_sqrt_d, (a.signs[(c + 2) >> 5] >> ((c + 2) & 31)) & 1u);
            v.w = flip_sign(o[c + 3] * inv_sqrt_d, (a.signs[(c + 3) >> 5] >> ((c + 3) & 31)) & 1u);
            *reinterpret_cast<float4*>(dst + c) = v;
        }
    } else if (bad && rt < min(TT, a.n_new - tok0) && rt * G + rh < BM) {
        // out-of-range start: zeros for every row of the block
        float* dst = a.out + ((static_cast<size_t>(b) * a.n_new + tok0 + rt) * a.hq + kv * G + rh) * D;
        for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace prefill

bool prefill_supported(const tq_params& p) {
    return p.head_dim == 128 && p.k_mode == TQ_MODE_TURBO && p.v_mode == TQ_MODE_TURBO && p.qjl_dims == 0 &&
           p.num_q_heads / p.num_kv_heads <= 16;
}

}  // namespace tq

extern "C" tq_status tq_prefill_attention(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                          const void* k_new, const void* v_new, tq_dtype kv_dtype, const void* d_q,
                                          tq_dtype q_dtype, int32_t n_new, const int32_t* d_positions,
                                          const tq_cache* cache, float* d_out, uint32_t* d_error, void* stream) {
    using namespace tq;
    tq_status st = validate_params(params);
    if (st != TQ_OK) return st;
    const tq_params& p = *params;
    if ((st = validate_cache(p, cache)) != TQ_OK) return st;
    if (!prefill_supported(p)) return TQ_ERR_UNSUPPORTED;
    if (!d_q || !d_out || !d_positions || n_new < 1) return TQ_ERR_INVALID_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16 && q_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
    if (!aligned16(d_q) || !aligned16(d_out)) return TQ_ERR_ALIGNMENT;
    if (n_new > cache->capacity) return TQ_ERR_CAPACITY;
    if ((st = validate_codebook(kcb, p.head_dim, p.k_bits)) != TQ_OK) return st;
    if ((st = validate_codebook(vcb, p.head_dim, p.v_bits)) != TQ_OK) return st;
    // append the chunk (positions[b] .. positions[b] + n_new - 1), then attend
    st = quantize_append_impl(params, kcb, vcb, k_new, v_new, kv_dtype, n_new, d_positions, false, cache, d_error,
                              stream);
    if (st != TQ_OK) return st;

    prefill::Args a{};
    a.k_codes = cache->k_codes;
    a.v_codes = cache->v_codes;
    a.k_norms = cache->k_norms;
    a.v_norms = cache->v_norms;
    a.q = d_q;
    a.q_dtype = q_dtype;
    a.positions = d_positions;
    a.out = d_out;
    a.err = d_error;
    a.batch = cache->batch;
    a.hq = p.num_q_heads;
    a.hkv = p.num_kv_heads;
    a.group = p.num_q_heads / p.num_kv_heads;
    a.capacity = cache->capacity;
    a.n_new = n_new;
    a.tok_per_tile = prefill::BM / a.group;
    a.kb = p.k_bits;
    a.vb = p.v_bits;
    const double ak = kcb->fp16_scale > 0.0 ? kcb->fp16_scale : std::sqrt(128.0);
    const double av = vcb->fp16_scale > 0.0 ? vcb->fp16_scale : std::sqrt(128.0);
    const float sm = p.sm_scale > 0.0f ? p.sm_scale : 1.0f / std::sqrt(128.0f);
    a.score_scale = static_cast<float>(sm * 1.4426950408889634 / ak);
    a.inv_alpha_v = static_cast<float>(1.0 / av);
    for (int j = 0; j < 16; ++j) {
        const __half hk = __float2half_rn(j < (1 << p.k_bits) ? static_cast<float>(kcb->centroids[j] * ak) : 0.f);
        const __half hv = __float2half_rn(j < (1 << p.v_bits) ? static_cast<float>(vcb->centroids[j] * av) : 0.f);
        a.kcent[j] = __half_as_ushort(hk);
        a.vcent[j] = __half_as_ushort(hv);
    }
    uint32_t words[8];
    rotation_sign_bits(p.seed, 128, words);
    for (int i = 0; i < 4; ++i) a.signs[i] = words[i];
    const dim3 grid((n_new + a.tok_per_tile - 1) / a.tok_per_tile, p.num_kv_heads, cache->batch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaFuncSetAttribute(prefill::prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(prefill::SM_ALLOC));
    if (e != cudaSuccess) return TQ_ERR_CUDA;
    prefill::prefill_kernel<<<grid, prefill::NTHREADS, prefill::SM_ALLOC, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
