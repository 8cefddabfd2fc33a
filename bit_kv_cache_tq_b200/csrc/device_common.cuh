// Device helpers shared by the TurboQuant kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace tq {

constexpr unsigned kFullMask = 0xffffffffu;

// Flip the sign of x when bit is 1 (multiplication by a rotation sign).
__device__ __forceinline__ float flip_sign(float x, uint32_t bit) {
    return __uint_as_float(__float_as_uint(x) ^ (bit << 31));
}

__device__ __forceinline__ uint32_t sign_bit(const uint32_t* words, int i) { return (words[i >> 5] >> (i & 31)) & 1u; }

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ uint16_t float_to_half_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }

// Eight consecutive input elements (16-byte aligned for 16-bit types, 32 for
// fp32) as floats, read with streaming (evict-first) loads.
template <int DTYPE>
__device__ __forceinline__ void load8_stream(const void* base, size_t elem_off, float out[8]) {
    if constexpr (DTYPE == 0) {  // fp32
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_off);
        const float4 a = __ldcs(p), b = __ldcs(p + 1);
        out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
        out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
    } else {
        const uint4 w = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem_off));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (DTYPE == 1) {  // bf16: the upper half of an fp32
                out[2 * i] = __uint_as_float(ws[i] << 16);
                out[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
            } else {  // fp16
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
                out[2 * i] = f.x;
                out[2 * i + 1] = f.y;
            }
        }
    }
}

// Four consecutive elements (16-byte aligned for fp32, 8-byte otherwise) in
// any of the three dtypes, as fp32.
__device__ __forceinline__ void load4(const void* base, size_t off, int dtype, float (&out)[4]) {
    if (dtype == 0) {
        const float4 v = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
        return;
    }
    const uint2 w = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + off);
    if (dtype == 1) {  // bf16: the upper half of an fp32
        out[0] = __uint_as_float(w.x << 16);
        out[1] = __uint_as_float(w.x & 0xffff0000u);
        out[2] = __uint_as_float(w.y << 16);
        out[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
        out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
    }
}

// One scalar of a query in any of the three dtypes.
__device__ __forceinline__ float load_scalar(const void* base, size_t off, int dtype) {
    if (dtype == 0) return static_cast<const float*>(base)[off];
    const uint16_t h = static_cast<const uint16_t*>(base)[off];
    if (dtype == 1) return __uint_as_float(static_cast<uint32_t>(h) << 16);
    return half_bits_to_float(h);
}

// Unnormalised Walsh-Hadamard butterflies over all index bits of a register
// array (Sylvester order: (a, b) -> (a + b, a - b) for the pair that differs
// in one bit, lower index first).
template <int N>
__device__ __forceinline__ void fwht_registers(float (&v)[N]) {
#pragma unroll
    for (int h = 1; h < N; h <<= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            if (!(i & h)) {
                const float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
        }
    }
}

// Butterflies across lanes: lanes l and l ^ m (for every m = 1, 2, .. < SPAN)
// hold coordinates that differ in one bit; `sub` is the lane's index in its
// SPAN-lane group.  The lower lane keeps a + b, the upper one a - b.
template <int N, int SPAN>
__device__ __forceinline__ void fwht_lanes(float (&v)[N], int sub) {
#pragma unroll
    for (int m = 1; m < SPAN; m <<= 1) {
        const float sg = (sub & m) ? -1.0f : 1.0f;  // upper lane: p - v, lower lane: v + p (one rounding)
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const float p = __shfl_xor_sync(kFullMask, v[i], m);
            v[i] = fmaf(v[i], sg, p);
        }
    }
}

template <int SPAN>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int m = 1; m < SPAN; m <<= 1) x += __shfl_xor_sync(kFullMask, x, m);
    return x;
}

template <int SPAN>
__device__ __forceinline__ float group_max(float x) {
#pragma unroll
    for (int m = 1; m < SPAN; m <<= 1) x = fmaxf(x, __shfl_xor_sync(kFullMask, x, m));
    return x;
}

// Code of a rotated unit coordinate y: the number of boundaries below it.
// With an odd-symmetric table the middle boundary is 0, so the count is
// 2^(b-1) + #{t_k > 0 : |y| > t_k} for y > 0 and 2^(b-1) - 1 - #{...} otherwise
// (an exact tie |y| == t_k on the negative side lands one cell high, inside
// the boundary window the codes are compared with).
template <int BITS>
__device__ __forceinline__ uint32_t code_of(float y, const float* tpos) {
    constexpr int half = 1 << (BITS - 1);
    const float a = fabsf(y);
    int m = 0;
#pragma unroll
    for (int k = 0; k < half - 1; ++k) m += a > tpos[k];
    return y > 0.0f ? static_cast<uint32_t>(half + m) : static_cast<uint32_t>(half - 1 - m);
}

// `nbits` (<= 32) bits of a packed little-endian bitstream starting at bit
// `bitoff`; `words` is the stream as 32-bit words and `nwords` its length
// (never read past).
__device__ __forceinline__ uint32_t stream_bits(const uint32_t* words, int nwords, int bitoff, int nbits) {
    const int w = bitoff >> 5, sh = bitoff & 31;
    uint64_t lo = words[w];
    if (sh + nbits > 32 && w + 1 < nwords) lo |= static_cast<uint64_t>(words[w + 1]) << 32;
    const uint64_t mask = nbits >= 32 ? 0xffffffffull : ((1ull << nbits) - 1);
    return static_cast<uint32_t>((lo >> sh) & mask);
}

}  // namespace tq
