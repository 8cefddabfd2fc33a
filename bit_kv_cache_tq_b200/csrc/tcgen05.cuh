// Hand-written inline-PTX wrappers for the 5th-generation tensor cores of
// sm_100a (tcgen05): tensor-memory allocation, MMA with A in tensor memory
// and B from a shared-memory descriptor into tensor memory, completion
// through an mbarrier, and loads from and stores to tensor memory.  Only the
// forms the prefill kernel uses.
#pragma once

#include <cstdint>

namespace tq {
namespace tc {

// Allocate `ncols` (a power of two >= 32) tensor-memory columns for this CTA;
// the address is written to shared memory at `dst`.  One full warp executes it.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
// Free the columns allocated at `taddr` (the same warp, the same count).
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// True in one lane of the (converged) warp.  MMAs go out fastest when the
// whole warp runs the issuing loop and the elected lane issues: issued from a
// lone thread of a diverged warp, each costs over a hundred cycles more.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{\n\t.reg .pred P1;\n\telect.sync _|P1, %1;\n\tselp.b32 %0, 1, 0, P1;\n\t}"
                 : "+r"(pred)
                 : "r"(0xffffffffu));
    return pred != 0;
}

// Order tensor-core operations against thread synchronisation.
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Make this thread's ordinary shared-memory writes visible to the tensor
// cores (the async proxy) before they read the operands.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }


// D[tmem] (+)= A[tmem] * B[smem]^T, fp16 inputs, fp32 accumulation; `accum`
// false overwrites D.  One thread issues it.  A is read from tensor memory at
// `a_tmem` (M = 128: row m in lane m; fp16 element k of the row in column
// k / 2, even k in the low half, so a 16-element K step spans 8 columns).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           bool accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(static_cast<uint32_t>(accum))
        : "memory");
}

// Arrive once on the mbarrier when every tensor-core operation this thread
// issued so far has completed.
__device__ __forceinline__ void commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane (warp w of
// a warpgroup reads lanes 32 w .. 32 w + 31; `taddr` carries the lane base in
// bits 16 and up).  Wait with ld_wait before using the values.
__device__ __forceinline__ void ld_32cols(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Raw 32-bit words to 8 or 16 consecutive columns of this thread's lane (the
// lane layout of ld_32cols); wait with st_wait before the tensor cores read
// them.
__device__ __forceinline__ void st_8cols(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
__device__ __forceinline__ void st_16cols_u(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
// 16 consecutive fp32 columns (the lane layout of ld_32cols).
__device__ __forceinline__ void ld_16cols(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void st_16cols(uint32_t taddr, const float (&v)[16]) {
    uint32_t r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(v[i]);
    st_16cols_u(taddr, r);
}
__device__ __forceinline__ void st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzled canonical layout: rows of 64 fp16 (128 bytes), eight rows to a
// 1024-byte swizzle atom (16-byte chunk c of row r stored at chunk c ^ (r % 8)),
// atoms of consecutive row groups 1024 bytes apart.  `addr` is the shared
// address of the first element of the K-slice (the atom base, plus 32 bytes
// per 16-element step within the row); atoms are 1024-byte aligned.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFFu);  // start address, 16-byte units
    d |= static_cast<uint64_t>(1) << 16;                        // leading byte offset (unused when swizzled)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;                // stride byte offset: next 8-row group
    d |= static_cast<uint64_t>(1) << 46;                        // descriptor version of sm_100
    d |= static_cast<uint64_t>(2) << 61;                        // 128-byte swizzle
    return d;
}

// Descriptor of an MN-major operand in the same 128-byte swizzled atoms:
// rows along K (one per K index, 128 bytes = 64 MN elements), eight rows to a
// 1024-byte atom; atoms of consecutive 8-row K groups `k_stride` bytes apart,
// atoms of consecutive 64-element MN blocks `mn_stride` bytes apart.  A tile
// stored [K rows][MN] in the K-major formula of sw128_offset (rows = K) is
// this layout with k_stride = 1024 and mn_stride = rows * 128.
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t addr, uint32_t mn_stride, uint32_t k_stride) {
    uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((mn_stride >> 4) & 0x3FFFu) << 16;  // leading byte offset: next MN block
    d |= static_cast<uint64_t>((k_stride >> 4) & 0x3FFFu) << 32;   // stride byte offset: next K group
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor of kind::f16: fp16 A and B, both K-major, fp32 D,
// shape M x N (M = 64 or 128, N a multiple of 8 up to 256 for M = 64, of 16
// for M = 128).
__host__ __device__ constexpr uint32_t idesc_f16(int m, int n) {
    return (1u << 4)                                      // D format: fp32
           | (0u << 7) | (0u << 10)                       // A, B format: fp16
           | (static_cast<uint32_t>(n >> 3) << 17)        // N / 8
           | (static_cast<uint32_t>(m >> 4) << 24);       // M / 16
}
// The same with B MN-major.
__host__ __device__ constexpr uint32_t idesc_f16_bmn(int m, int n) { return idesc_f16(m, n) | (1u << 16); }

// Byte offset of fp16 element (r, k) in a K-major 128-byte-swizzled tile of
// `rows` rows: K is cut into 64-element column blocks of rows x 128 bytes.
__host__ __device__ constexpr uint32_t sw128_offset(int r, int k, int rows) {
    return static_cast<uint32_t>((k >> 6) * rows * 128 + (r >> 3) * 1024 + (r & 7) * 128 +
                                 ((((k & 63) >> 3) ^ (r & 7)) << 4) + ((k & 7) << 1));
}

}  // namespace tc
}  // namespace tq
