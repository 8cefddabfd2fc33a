// Quantise-append and dequantise kernels (sm_100a) and their C entry points.
//
// Pages (by title):
//   [tqai]    "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术",
//             section "TurboQuant的核心创新：极坐标量化与随机旋转"
//   [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命", sections
//             "核心技术", "压缩格式对比", "三个反直觉的关键发现"
//   [fwht]    "TurboQuant：用Rust核心与FWHT预处理实现LLM推理的4-bit KV缓存量化",
//             section "2. 快速Walsh-Hadamard变换（FWHT）预处理"
//   [google]  "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！",
//             section "第二步：QJL —— 1 bit 清理殘差"
//
// Work layout: a head vector of d coordinates is held by d/32 lanes, 32
// coordinates each.  The vector is read as 16-byte chunks of 8 elements;
// lane j of the vector's lane group holds chunks j, j + d/32, j + 2d/32,
// j + 3d/32, so every load instruction of a warp covers whole 32-byte
// sectors.  The Walsh-Hadamard transform then runs 5 butterfly stages in
// registers and log2(d/32) stages across lanes (warp shuffles).

#include <cuda_runtime.h>

#include <chrono>
#include <cmath>
#include <cstring>
#include <algorithm>
#include <thread>

#include "device_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace tq {

struct QuantSide {
    const void* src;        // [batch][n_new][Hkv][d]
    uint8_t* codes;         // [batch][Hkv][capacity][vbytes]
    uint16_t* norms;        // [batch][Hkv][capacity]
    uint8_t* qjl;           // [batch][Hkv][capacity][m/8] or null
    uint16_t* gamma;        // [batch][Hkv][capacity] or null
    const float* sketch;    // [m][d] or null
    int mode, bits, vbytes, m;
    float centroids[16];
    float pos_boundaries[8];  // boundaries above zero, ascending (2^(bits-1) - 1 of them)
    // Code grid (turbo mode; grid_inv_w = 0 when the table cannot hold the
    // codebook): the rotated unit coordinate y is cut into cells of width w
    // (no wider than the narrowest code cell, so a grid cell holds at most one
    // boundary), cell c = round(y / w) covering [(c - 0.5) w, (c + 0.5) w).
    // Entry c & 127 is the fp32 bit pattern of the boundary inside the cell,
    // in cells, with its 4 low mantissa bits replaced by the number of
    // boundaries below the cell (the boundary moves by at most 15 ulps); a
    // cell without a boundary holds +inf's pattern, a NaN once those bits are
    // set, so it never compares below y.  The code of y is the count plus
    // (y / w > the boundary).  |y| <= 1 keeps c within +-63.
    float grid_inv_w;
    uint32_t grid[128];
};

struct QuantArgs {
    QuantSide side[2];  // 0 = K, 1 = V
    const int32_t* positions;  // per sequence: first slot written, or (pos_from_lens) the length after the append
    uint32_t* err;
    int batch, n_new, hkv, capacity, pos_from_lens;  // capacity: tokens a sequence may hold
    uint32_t total;                     // batch * n_new * hkv vectors (< 2^32)
    uint64_t hkv_magic, n_new_magic;    // quotient multipliers: see div_magic
    // paged cache (table non-null): token t of sequence b is in block
    // table[b * max_blocks + t / block_size] of the pool
    const int32_t* table;
    int max_blocks, block_size, num_blocks;
    uint32_t signs[8];
};

template <int BITS>
__device__ __forceinline__ void store_chunk_codes(uint8_t* row, int chunk, uint32_t packed) {
    if constexpr (BITS == 4) {
        *reinterpret_cast<uint32_t*>(row + 4 * chunk) = packed;
    } else if constexpr (BITS == 2) {
        *reinterpret_cast<uint16_t*>(row + 2 * chunk) = static_cast<uint16_t>(packed);
    } else {
        row[3 * chunk] = static_cast<uint8_t>(packed);
        row[3 * chunk + 1] = static_cast<uint8_t>(packed >> 8);
        row[3 * chunk + 2] = static_cast<uint8_t>(packed >> 16);
    }
}

// Code of the rotated coordinate x = y * sqrt(d) * ||x|| against the
// boundaries scaled the same way (ts[k] = t_k sqrt(d) ||x||, ascending): the
// count of boundaries below y, found with a binary search over the positive
// half (the table is odd-symmetric, its middle boundary is 0).  Deciding on x
// against scaled boundaries instead of on y = x / (sqrt(d) ||x||) moves a
// decision only when y is within a few ulp of a boundary.
template <int BITS>
__device__ __forceinline__ uint32_t code_scaled(float x, const float (&ts)[7]) {
    constexpr int half = 1 << (BITS - 1);
    const float a = fabsf(x);
    int m;
    if constexpr (BITS == 4) {
        const bool p2 = a > ts[3];
        const bool p1 = a > (p2 ? ts[5] : ts[1]);
        const float w = p1 ? (p2 ? ts[6] : ts[2]) : (p2 ? ts[4] : ts[0]);
        m = 4 * p2 + 2 * p1 + (a > w);
    } else if constexpr (BITS == 3) {
        const bool p1 = a > ts[1];
        m = 2 * p1 + (a > (p1 ? ts[2] : ts[0]));
    } else {
        m = a > ts[0];
    }
    return x > 0.0f ? static_cast<uint32_t>(half + m) : static_cast<uint32_t>(half - 1 - m);
}

// n / d for n < 2^32 as the high word of n * M, M = ceil(2^64 / d) (exact:
// the product overshoots n / d by less than n / 2^64 < 1 / d); M = 0 stands
// for d = 1.
__device__ __forceinline__ uint32_t div_magic(uint32_t n, uint64_t m) {
    return m == 0 ? n : static_cast<uint32_t>(__umul64hi(static_cast<uint64_t>(n), m));
}

// Walsh-Hadamard butterflies over a lane's 32 values, the stages of span 2
// and more as packed fp32 pairs (the same additions, in the same order).
__device__ __forceinline__ void fwht32_pairs(float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const float a = v[i], b = v[i + 1];
        v[i] = a + b;
        v[i + 1] = a - b;
    }
#pragma unroll
    for (int h = 2; h < 32; h <<= 1)
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            if (!(i & h)) {
                const float2 a = make_float2(v[i], v[i + 1]), b = make_float2(v[i + h], v[i + h + 1]);
                const float2 s = ptx::fadd2(a, b), d = ptx::fsub2(a, b);
                v[i] = s.x;
                v[i + 1] = s.y;
                v[i + h] = d.x;
                v[i + h + 1] = d.y;
            }
}

// fwht_lanes with the fused multiply-adds in packed pairs.
template <int SPAN>
__device__ __forceinline__ void fwht_lanes_pairs(float (&v)[32], int sub) {
#pragma unroll
    for (int m = 1; m < SPAN; m <<= 1) {
        const float sg = (sub & m) ? -1.0f : 1.0f;  // upper lane: p - v, lower lane: v + p
        const float2 sg2 = make_float2(sg, sg);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const float2 p = make_float2(__shfl_xor_sync(kFullMask, v[i], m), __shfl_xor_sync(kFullMask, v[i + 1], m));
            const float2 r = ptx::ffma2(make_float2(v[i], v[i + 1]), sg2, p);
            v[i] = r.x;
            v[i + 1] = r.y;
        }
    }
}

// Turbo encode through the code grid (shared copy `grid`); x holds the
// lane's 32 coordinates with the rotation signs already applied.
template <int D, int BITS>
__device__ __forceinline__ void turbo_encode_grid(const QuantSide& s, const uint32_t* grid, float (&x)[32], int sub,
                                                  size_t slot, bool valid) {
    constexpr int LPV = D / 32;
    float sumsq = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) sumsq = fmaf(x[j], x[j], sumsq);
    fwht32_pairs(x);
    fwht_lanes_pairs<LPV>(x, sub);
    sumsq = group_sum<LPV>(sumsq);
    const float n = sqrtf(sumsq);
    const float scale = sqrtf(static_cast<float>(D)) * n;  // y_i = x_i / scale
    const float inv = n > 0.0f ? s.grid_inv_w / scale : 0.0f;  // grid cells per unit of x
    uint32_t packed[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t acc = 0;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
            const float g = x[8 * k + e] * inv;
            // round(g) in the low mantissa bits of g + 1.5 * 2^23 (|g| < 64)
            const uint32_t cell = grid[__float_as_uint(g + 12582912.0f) & 127u];
            const uint32_t code = (cell & 15u) + (g > __uint_as_float(cell) ? 1u : 0u);
            acc = acc * (1u << BITS) + code;
        }
        packed[k] = acc;
    }
    if (valid) {
        uint8_t* row = s.codes + slot * static_cast<size_t>(s.vbytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) store_chunk_codes<BITS>(row, sub + LPV * k, packed[k]);
        if (sub == 0) s.norms[slot] = float_to_half_bits(n);
    }
    if (s.m > 0) {  // QJL residual sketch (keys only)
        const float rinv = n > 0.0f ? 1.0f / scale : 0.0f;
        float g2 = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t code = (packed[i >> 3] >> (BITS * (i & 7))) & ((1u << BITS) - 1u);
            x[i] = x[i] * rinv - s.centroids[code];  // residual r_i = y_i - c[code_i]
            g2 = fmaf(x[i], x[i], g2);
        }
        g2 = group_sum<LPV>(g2);
        uint32_t word = 0;
        for (int r = 0; r < s.m; ++r) {
            const float* row = s.sketch + static_cast<size_t>(r) * D;
            float acc = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 a = __ldg(reinterpret_cast<const float4*>(row + 8 * (sub + LPV * k)));
                const float4 b = __ldg(reinterpret_cast<const float4*>(row + 8 * (sub + LPV * k) + 4));
                acc = fmaf(a.x, x[8 * k + 0], acc); acc = fmaf(a.y, x[8 * k + 1], acc);
                acc = fmaf(a.z, x[8 * k + 2], acc); acc = fmaf(a.w, x[8 * k + 3], acc);
                acc = fmaf(b.x, x[8 * k + 4], acc); acc = fmaf(b.y, x[8 * k + 5], acc);
                acc = fmaf(b.z, x[8 * k + 6], acc); acc = fmaf(b.w, x[8 * k + 7], acc);
            }
            acc = group_sum<LPV>(acc);
            word |= static_cast<uint32_t>(acc >= 0.0f) << (r & 31);
            if ((r & 31) == 31) {
                if (valid && sub == 0)
                    reinterpret_cast<uint32_t*>(s.qjl + slot * static_cast<size_t>(s.m / 8))[r >> 5] = word;
                word = 0;
            }
        }
        if (valid && sub == 0) s.gamma[slot] = float_to_half_bits(sqrtf(g2));
    }
}

// Rotation signs of this lane's 32 coordinates 8 (sub + LPV k) + e, as bit
// 8 k + e of one word (built once per thread).
template <int D>
__device__ __forceinline__ uint32_t lane_sign_mask(const uint32_t* signs, int sub) {
    constexpr int LPV = D / 32;
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int i0 = 8 * (sub + LPV * k);
        m |= ((signs[i0 >> 5] >> (i0 & 31)) & 0xFFu) << (8 * k);
    }
    return m;
}

template <int D, int BITS>
__device__ __forceinline__ void turbo_encode(const QuantSide& s, float (&x)[32], int sub, size_t slot, bool valid,
                                             uint32_t smask) {
    constexpr int LPV = D / 32;
    float sumsq = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        sumsq = fmaf(x[j], x[j], sumsq);
        x[j] = __uint_as_float(__float_as_uint(x[j]) ^ ((smask << (31 - j)) & 0x80000000u));
    }
    fwht_registers(x);
    fwht_lanes<32, LPV>(x, sub);
    sumsq = group_sum<LPV>(sumsq);
    const float n = sqrtf(sumsq);
    const float scale = sqrtf(static_cast<float>(D)) * n;  // y_i = x_i / scale
    float ts[7];
#pragma unroll
    for (int k = 0; k < 7; ++k) ts[k] = s.pos_boundaries[k] * scale;
    uint32_t codes[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) codes[i] = code_scaled<BITS>(x[i], ts);
    if (valid) {
        uint8_t* row = s.codes + slot * static_cast<size_t>(s.vbytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t packed = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) packed |= codes[8 * k + e] << (BITS * e);
            store_chunk_codes<BITS>(row, sub + LPV * k, packed);
        }
        if (sub == 0) s.norms[slot] = float_to_half_bits(n);
    }
    if (s.m > 0) {  // QJL residual sketch (keys only)
        const float inv = n > 0.0f ? 1.0f / scale : 0.0f;
        float g2 = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            x[i] = x[i] * inv - s.centroids[codes[i]];  // residual r_i = y_i - c[code_i]
            g2 = fmaf(x[i], x[i], g2);
        }
        g2 = group_sum<LPV>(g2);
        uint32_t word = 0;
        for (int r = 0; r < s.m; ++r) {
            const float* row = s.sketch + static_cast<size_t>(r) * D;
            float acc = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 a = __ldg(reinterpret_cast<const float4*>(row + 8 * (sub + LPV * k)));
                const float4 b = __ldg(reinterpret_cast<const float4*>(row + 8 * (sub + LPV * k) + 4));
                acc = fmaf(a.x, x[8 * k + 0], acc); acc = fmaf(a.y, x[8 * k + 1], acc);
                acc = fmaf(a.z, x[8 * k + 2], acc); acc = fmaf(a.w, x[8 * k + 3], acc);
                acc = fmaf(b.x, x[8 * k + 4], acc); acc = fmaf(b.y, x[8 * k + 5], acc);
                acc = fmaf(b.z, x[8 * k + 6], acc); acc = fmaf(b.w, x[8 * k + 7], acc);
            }
            acc = group_sum<LPV>(acc);
            word |= static_cast<uint32_t>(acc >= 0.0f) << (r & 31);
            if ((r & 31) == 31) {
                if (valid && sub == 0)
                    reinterpret_cast<uint32_t*>(s.qjl + slot * static_cast<size_t>(s.m / 8))[r >> 5] = word;
                word = 0;
            }
        }
        if (valid && sub == 0) s.gamma[slot] = float_to_half_bits(sqrtf(g2));
    }
}

template <int D>
__device__ __forceinline__ void int8_encode(const QuantSide& s, const float (&x)[32], int sub, size_t slot,
                                            bool valid) {
    constexpr int LPV = D / 32;
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = group_max<LPV>(amax);
    const __half scale16 = __float2half_rn(__fdiv_rn(amax, 127.0f));
    const float scale = __half2float(scale16);
    const float recip = (scale > 0.0f && scale < INFINITY) ? __frcp_rn(scale) : 0.0f;
    if (!valid) return;
    uint8_t* row = s.codes + slot * static_cast<size_t>(D);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float q = fminf(fmaxf(rintf(__fmul_rn(x[8 * k + e], recip)), -127.0f), 127.0f);
            const uint32_t byte = static_cast<uint32_t>(static_cast<int32_t>(q)) & 0xffu;
            if (e < 4) lo |= byte << (8 * e);
            else hi |= byte << (8 * (e - 4));
        }
        *reinterpret_cast<uint2*>(row + 8 * (sub + LPV * k)) = make_uint2(lo, hi);
    }
    if (sub == 0) s.norms[slot] = __half_as_ushort(scale16);
}

// One side (K = 0, V = 1: blockIdx.y) of the quantise-append kernel; the side
// is a template argument so that its fields are static parameter reads.
template <int D, int DTYPE, int SIDE>
__device__ __forceinline__ void quantize_side(const QuantArgs& a, uint32_t* sgrid) {
    constexpr int LPV = D / 32;  // lanes per vector
    constexpr int VPW = 32 / LPV;  // vectors per warp pass
    const QuantSide& s = a.side[SIDE];
    const bool grid_path = s.mode == TQ_MODE_TURBO && s.grid_inv_w > 0.0f;
    if (grid_path && threadIdx.x < 128) sgrid[threadIdx.x] = s.grid[threadIdx.x];
    __syncthreads();
    ptx::wait_prerequisites();   // inputs and cache may come from the previous kernel
    // the next kernel may start launching; as this comes after the wait, every
    // kernel before this one has finished by then, so before its own wait the
    // next kernel can read anything but what this one writes
    ptx::launch_dependents();
    const int lane = threadIdx.x & 31, sub = lane % LPV, grp = lane / LPV;
    const uint32_t smask = lane_sign_mask<D>(a.signs, sub);
    // bf16 inputs: the rotation signs of word i of chunk k (coordinates
    // 8 k + 2 i and 8 k + 2 i + 1) at bits 15 and 31, applied to the raw words
    uint32_t sw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        sw[i] = (((smask >> (2 * i)) & 1u) << 15) | (((smask >> (2 * i + 1)) & 1u) << 31);
    const long long nwarps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
    for (long long base = (static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32) * VPW;
         base < a.total; base += nwarps * VPW) {
        const uint32_t v = static_cast<uint32_t>(base) + grp;
        bool valid = v < a.total;
        size_t slot = 0;
        if (valid) {
            const uint32_t bt = div_magic(v, a.hkv_magic);
            const int h = static_cast<int>(v - bt * static_cast<uint32_t>(a.hkv));
            const uint32_t b32 = div_magic(bt, a.n_new_magic);
            const int t = static_cast<int>(bt - b32 * static_cast<uint32_t>(a.n_new));
            const int b = static_cast<int>(b32);
            const int pos = a.positions[b] - (a.pos_from_lens ? a.n_new : 0);
            if (pos < 0 || pos > a.capacity - a.n_new) {
                if (a.err && t == 0 && h == 0 && sub == 0 && blockIdx.y == 0) atomicOr(a.err, TQ_DEVERR_POSITION);
                valid = false;
            } else if (a.table) {
                const int tok = pos + t;
                const int blk = __ldg(a.table + static_cast<size_t>(b) * a.max_blocks + tok / a.block_size);
                if (blk < 0 || blk >= a.num_blocks) {
                    if (a.err && sub == 0 && blockIdx.y == 0) atomicOr(a.err, TQ_DEVERR_PAGE);
                    valid = false;
                } else {
                    slot = (static_cast<size_t>(blk) * a.hkv + h) * a.block_size + tok % a.block_size;
                }
            } else {
                slot = (static_cast<size_t>(b) * a.hkv + h) * a.capacity + pos + t;
            }
        }
        float x[32];
        if (DTYPE == 1 && grid_path) {
            // raw bf16 words with the rotation signs flipped in place
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint4 w = make_uint4(0u, 0u, 0u, 0u);
                if (v < a.total)
                    w = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(s.src) +
                                                              static_cast<size_t>(v) * D + 8 * (sub + LPV * k)));
                const uint32_t ws[4] = {w.x ^ sw[4 * k], w.y ^ sw[4 * k + 1], w.z ^ sw[4 * k + 2], w.w ^ sw[4 * k + 3]};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    x[8 * k + 2 * i] = __uint_as_float(ws[i] << 16);
                    x[8 * k + 2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
                }
            }
        } else {
            if (v < a.total) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    load8_stream<DTYPE>(s.src, static_cast<size_t>(v) * D + 8 * (sub + LPV * k), &x[8 * k]);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = 0.0f;
            }
            if (grid_path) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    x[j] = __uint_as_float(__float_as_uint(x[j]) ^ ((smask << (31 - j)) & 0x80000000u));
            }
        }
        if (s.mode == TQ_MODE_INT8) {
            int8_encode<D>(s, x, sub, slot, valid);
        } else if (grid_path) {
            if (s.bits == 4) turbo_encode_grid<D, 4>(s, sgrid, x, sub, slot, valid);
            else if (s.bits == 3) turbo_encode_grid<D, 3>(s, sgrid, x, sub, slot, valid);
            else turbo_encode_grid<D, 2>(s, sgrid, x, sub, slot, valid);
        } else if (s.bits == 4) {
            turbo_encode<D, 4>(s, x, sub, slot, valid, smask);
        } else if (s.bits == 3) {
            turbo_encode<D, 3>(s, x, sub, slot, valid, smask);
        } else {
            turbo_encode<D, 2>(s, x, sub, slot, valid, smask);
        }
    }
}

template <int D, int DTYPE>
__global__ void __launch_bounds__(256, 3) quantize_append_kernel(const __grid_constant__ QuantArgs a) {
    __shared__ uint32_t sgrid[128];
    if (blockIdx.y == 0) quantize_side<D, DTYPE, 0>(a, sgrid);
    else quantize_side<D, DTYPE, 1>(a, sgrid);
}

// ------------------------------------------------------------- dequantise
struct DequantArgs {
    QuantSide side[2];
    float* out[2];
    int b, start, count, hkv, capacity;
    uint32_t signs[8];
};

template <int D>
__global__ void __launch_bounds__(256) dequantize_kernel(const __grid_constant__ DequantArgs a) {
    constexpr int LPV = D / 32;
    constexpr int VPW = 32 / LPV;
    const QuantSide& s = a.side[blockIdx.y];
    float* out = a.out[blockIdx.y];
    if (!out) return;  // (the whole block: one side per block)
    // the centroids in shared memory: a per-thread index into the kernel
    // parameters would be served one address at a time
    __shared__ float scen[16];
    if (threadIdx.x < 16) scen[threadIdx.x] = s.centroids[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31, sub = lane % LPV, grp = lane / LPV;
    const long long total = static_cast<long long>(a.count) * a.hkv;
    const long long nwarps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
    for (long long base = (static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32) * VPW;
         base < total; base += nwarps * VPW) {
        const long long v = base + grp;
        const bool valid = v < total;
        const int h = valid ? static_cast<int>(v % a.hkv) : 0;
        const int t = valid ? static_cast<int>(v / a.hkv) : 0;
        const size_t slot = (static_cast<size_t>(a.b) * a.hkv + h) * a.capacity + a.start + t;
        float x[32];
        if (s.mode == TQ_MODE_INT8) {
            const float scale = valid ? half_bits_to_float(s.norms[slot]) : 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint2 w = valid ? *reinterpret_cast<const uint2*>(s.codes + slot * D + 8 * (sub + LPV * k))
                                      : make_uint2(0, 0);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t word = e < 4 ? w.x : w.y;
                    const int8_t q = static_cast<int8_t>((word >> (8 * (e & 3))) & 0xffu);
                    x[8 * k + e] = scale * static_cast<float>(q);
                }
            }
        } else {
            const uint32_t* words = reinterpret_cast<const uint32_t*>(s.codes + slot * static_cast<size_t>(s.vbytes));
            const int nwords = s.vbytes / 4;
            const uint32_t mask = (1u << s.bits) - 1u;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t chunk = valid ? stream_bits(words, nwords, 8 * s.bits * (sub + LPV * k), 8 * s.bits) : 0u;
#pragma unroll
                for (int e = 0; e < 8; ++e) x[8 * k + e] = scen[(chunk >> (s.bits * e)) & mask];
            }
            if (s.m > 0 && valid) {
                const float coef = half_bits_to_float(s.gamma[slot]) * sqrtf(0.5f * 3.14159265358979f) / s.m;
                const uint32_t* z = reinterpret_cast<const uint32_t*>(s.qjl + slot * static_cast<size_t>(s.m / 8));
                for (int r = 0; r < s.m; ++r) {
                    const float w = (z[r >> 5] >> (r & 31)) & 1u ? coef : -coef;
                    const float* row = s.sketch + static_cast<size_t>(r) * D;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[8 * k + e] = fmaf(w, __ldg(row + 8 * (sub + LPV * k) + e), x[8 * k + e]);
                }
            }
            fwht_registers(x);
            fwht_lanes<32, LPV>(x, sub);
            const float scale = (valid ? half_bits_to_float(s.norms[slot]) : 0.0f) / sqrtf(static_cast<float>(D));
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = 8 * (sub + LPV * k) + e;
                    x[8 * k + e] = flip_sign(x[8 * k + e] * scale, sign_bit(a.signs, i));
                }
        }
        if (valid) {
            float* dst = out + static_cast<size_t>(v) * D;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float4* p = reinterpret_cast<float4*>(dst + 8 * (sub + LPV * k));
                p[0] = make_float4(x[8 * k + 0], x[8 * k + 1], x[8 * k + 2], x[8 * k + 3]);
                p[1] = make_float4(x[8 * k + 4], x[8 * k + 5], x[8 * k + 6], x[8 * k + 7]);
            }
        }
    }
}

// ---------------------------------------------------------------- launchers
static void fill_side(QuantSide& s, int mode, int bits, int d, const tq_codebook* cb) {
    s.mode = mode;
    s.bits = mode == TQ_MODE_INT8 ? 8 : bits;
    s.vbytes = vector_bytes(mode, bits, d);
    for (int j = 0; j < 16; ++j) s.centroids[j] = 0.0f;
    for (int j = 0; j < 8; ++j) s.pos_boundaries[j] = INFINITY;
    s.grid_inv_w = 0.0f;
    if (mode == TQ_MODE_TURBO) {
        const int n = 1 << bits, half = n / 2;
        for (int j = 0; j < n; ++j) s.centroids[j] = static_cast<float>(cb->centroids[j]);
        for (int k = 0; k < half - 1; ++k) s.pos_boundaries[k] = static_cast<float>(cb->boundaries[half + k]);
        // the code grid: cells no wider than the narrowest code cell; used
        // only when |y| <= 1 stays within 62.5 cells of zero (else the binary
        // search below serves)
        double w = INFINITY;
        for (int j = 0; j + 1 < n - 1; ++j) w = std::min(w, cb->boundaries[j + 1] - cb->boundaries[j]);
        if (n == 2) w = 1.0;  // (not a width the codebooks produce: one boundary, at zero)
        w *= 1.0 - 1e-6;
        bool ok = 1.0 / w < 62.5;
        for (int idx = 0; ok && idx < 128; ++idx) {
            const int c = idx < 64 ? idx : idx - 128;
            const double lo = (c - 0.5) * w, hi = (c + 0.5) * w;
            uint32_t below = 0;
            int inside = -1;
            for (int j = 0; j < n - 1; ++j) {
                const double t = cb->boundaries[j];
                if (t < lo) ++below;
                else if (t < hi) {
                    if (inside >= 0) ok = false;  // two boundaries in a cell
                    inside = j;
                }
            }
            const float bnd = inside >= 0 ? static_cast<float>(cb->boundaries[inside] / w) : INFINITY;
            uint32_t bits32;
            std::memcpy(&bits32, &bnd, 4);
            s.grid[idx] = (bits32 & ~15u) | below;
        }
        if (ok) s.grid_inv_w = static_cast<float>(1.0 / w);
    }
}

// ceil(2^64 / d) for the quotients of div_magic; 0 for d = 1.
static uint64_t quotient_magic(uint32_t d) { return d <= 1 ? 0 : UINT64_MAX / d + 1; }

int num_sms_current() {  // SM count of the current device, 0 if unknown
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

template <int D, int DTYPE>
static cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t stream) {
    constexpr int VPW = 32 / (D / 32);
    const long long total = a.total;
    const long long warps_needed = (total + VPW - 1) / VPW;
    const int sms = num_sms_current();
    long long blocks = (warps_needed + 7) / 8;
    const long long cap = static_cast<long long>(sms > 0 ? sms : 148) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 2);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_append_kernel<D, DTYPE>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_quantize_dtype(const QuantArgs& a, int dtype, cudaStream_t stream) {
    switch (dtype) {
        case TQ_F32: return launch_quantize<D, 0>(a, stream);
        case TQ_BF16: return launch_quantize<D, 1>(a, stream);
        default: return launch_quantize<D, 2>(a, stream);
    }
}

}  // namespace tq

// =================================================================== C ABI
extern "C" {

tq_status tq_quantize_append(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                             const void* k_new, const void* v_new, tq_dtype dtype, int32_t n_new,
                             const int32_t* d_positions, const tq_cache* cache, uint32_t* d_error,
                             void* stream) {
    return tq::quantize_append_impl(params, kcb, vcb, k_new, v_new, dtype, n_new, d_positions, false, cache, d_error,
                                    stream);
}

tq_status tq_quantize_append_paged(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                   const void* k_new, const void* v_new, tq_dtype dtype, int32_t n_new,
                                   const int32_t* d_positions, const tq_cache* pool, const tq_block_table* table,
                                   uint32_t* d_error, void* stream) {
    if (!params) return TQ_ERR_INVALID_ARG;
    tq::PageMap pm;
    const tq_status st = tq::validate_pages(*params, pool, table, &pm);
    if (st != TQ_OK) return st;
    return tq::quantize_append_impl(params, kcb, vcb, k_new, v_new, dtype, n_new, d_positions, false, pool, d_error,
                                    stream, &pm);
}

}  // extern "C"

tq_status tq::quantize_append_impl(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                   const void* k_new, const void* v_new, int dtype, int32_t n_new,
                                   const int32_t* d_positions, bool pos_from_lens, const tq_cache* cache,
                                   uint32_t* d_error, void* stream, const PageMap* pm) {
    using namespace tq;
    tq_status st = validate_params(params);
    if (st != TQ_OK) return st;
    const tq_params& p = *params;
    if ((st = validate_cache(p, cache)) != TQ_OK) return st;
    if (!k_new || !v_new || !d_positions || n_new < 1) return TQ_ERR_INVALID_ARG;
    if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new)) return TQ_ERR_ALIGNMENT;
    const int capacity = pm ? pm->max_blocks * pm->block_size : cache->capacity;  // tokens per sequence
    if (n_new > capacity) return TQ_ERR_CAPACITY;
    if (p.k_mode == TQ_MODE_TURBO && (st = validate_codebook(kcb, p.head_dim, p.k_bits)) != TQ_OK) return st;
    if (p.v_mode == TQ_MODE_TURBO && (st = validate_codebook(vcb, p.head_dim, p.v_bits)) != TQ_OK) return st;
    QuantArgs a{};
    fill_side(a.side[0], p.k_mode, p.k_bits, p.head_dim, kcb);
    fill_side(a.side[1], p.v_mode, p.v_bits, p.head_dim, vcb);
    a.side[0].src = k_new;
    a.side[0].codes = cache->k_codes;
    a.side[0].norms = cache->k_norms;
    a.side[0].qjl = cache->k_qjl;
    a.side[0].gamma = cache->k_gamma;
    a.side[0].sketch = cache->qjl_matrix;
    a.side[0].m = p.qjl_dims;
    a.side[1].src = v_new;
    a.side[1].codes = cache->v_codes;
    a.side[1].norms = cache->v_norms;
    a.side[1].m = 0;
    a.positions = d_positions;
    a.pos_from_lens = pos_from_lens ? 1 : 0;
    a.err = d_error;
    a.batch = pm ? pm->batch : cache->batch;
    a.n_new = n_new;
    a.hkv = p.num_kv_heads;
    {
        const long long total = static_cast<long long>(a.batch) * n_new * p.num_kv_heads;
        if (total >= (1ll << 32)) return TQ_ERR_INVALID_ARG;
        a.total = static_cast<uint32_t>(total);
        a.hkv_magic = quotient_magic(static_cast<uint32_t>(p.num_kv_heads));
        a.n_new_magic = quotient_magic(static_cast<uint32_t>(n_new));
    }
    a.capacity = capacity;
    if (pm) {
        a.table = pm->table;
        a.max_blocks = pm->max_blocks;
        a.block_size = pm->block_size;
        a.num_blocks = pm->num_blocks;
    }
    rotation_sign_bits(p.seed, p.head_dim, a.signs);
    cudaError_t e;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (p.head_dim) {
        case 64: e = launch_quantize_dtype<64>(a, dtype, s); break;
        case 128: e = launch_quantize_dtype<128>(a, dtype, s); break;
        default: e = launch_quantize_dtype<256>(a, dtype, s); break;
    }
    return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

extern "C" {

tq_status tq_dequantize(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                        const tq_cache* cache, int32_t b, int32_t start, int32_t count, float* d_k_out,
                        float* d_v_out, void* stream) {
    using namespace tq;
    tq_status st = validate_params(params);
    if (st != TQ_OK) return st;
    const tq_params& p = *params;
    if ((st = validate_cache(p, cache)) != TQ_OK) return st;
    if (b < 0 || b >= cache->batch || start < 0 || count < 1 || start > cache->capacity - count)
        return TQ_ERR_INVALID_ARG;
    if (!d_k_out && !d_v_out) return TQ_ERR_INVALID_ARG;
    if ((d_k_out && !aligned16(d_k_out)) || (d_v_out && !aligned16(d_v_out))) return TQ_ERR_ALIGNMENT;
    if (p.k_mode == TQ_MODE_TURBO && (st = validate_codebook(kcb, p.head_dim, p.k_bits)) != TQ_OK) return st;
    if (p.v_mode == TQ_MODE_TURBO && (st = validate_codebook(vcb, p.head_dim, p.v_bits)) != TQ_OK) return st;
    DequantArgs a{};
    fill_side(a.side[0], p.k_mode, p.k_bits, p.head_dim, kcb);
    fill_side(a.side[1], p.v_mode, p.v_bits, p.head_dim, vcb);
    a.side[0].codes = cache->k_codes;
    a.side[0].norms = cache->k_norms;
    a.side[0].qjl = cache->k_qjl;
    a.side[0].gamma = cache->k_gamma;
    a.side[0].sketch = cache->qjl_matrix;
    a.side[0].m = p.qjl_dims;
    a.side[1].codes = cache->v_codes;
    a.side[1].norms = cache->v_norms;
    a.out[0] = d_k_out;
    a.out[1] = d_v_out;
    a.b = b;
    a.start = start;
    a.count = count;
    a.hkv = p.num_kv_heads;
    a.capacity = cache->capacity;
    rotation_sign_bits(p.seed, p.head_dim, a.signs);
    const int lpv = p.head_dim / 32;
    const long long warps = (static_cast<long long>(count) * p.num_kv_heads * lpv + 31) / 32;
    long long blocks = (warps + 7) / 8;
    if (blocks > 148 * 8) blocks = 148 * 8;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 grid(static_cast<unsigned>(blocks), 2);
    switch (p.head_dim) {
        case 64: dequantize_kernel<64><<<grid, 256, 0, s>>>(a); break;
        case 128: dequantize_kernel<128><<<grid, 256, 0, s>>>(a); break;
        default: dequantize_kernel<256><<<grid, 256, 0, s>>>(a); break;
    }
    return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_read_device_error(const uint32_t* d_error, uint32_t* out, void* stream, int32_t timeout_ms) {
    if (!d_error || !out || timeout_ms < 0) return TQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return TQ_ERR_CUDA;
    if (cudaEventRecord(ev, s) != cudaSuccess) {
        cudaEventDestroy(ev);
        return TQ_ERR_CUDA;
    }
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);
    cudaError_t q;
    while ((q = cudaEventQuery(ev)) == cudaErrorNotReady) {
        if (std::chrono::steady_clock::now() > deadline) {
            cudaEventDestroy(ev);
            return TQ_ERR_TIMEOUT;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
    cudaEventDestroy(ev);
    if (q != cudaSuccess) return TQ_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, d_error, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return TQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return TQ_ERR_CUDA;
    *out = word;
    return word ? TQ_ERR_DEVICE : TQ_OK;
}

}  // extern "C"
