// Chunked prefill attention from the compressed cache on the 5th-generation
// tensor cores (sm_100a, tcgen05 with tensor-memory operands and
// accumulators).
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
// How: the work comes in units of (sequence, kv head, 128 query rows), a row
// being one (query token, head of the GQA group), each unit a run of 64-key
// tiles.  One thread block per SM takes an equal share of the sequence of
// all units' tiles (so a unit can be cut between blocks: each piece's rows
// go to the workspace as (O, m, l), and a second kernel merges them by
// log-sum-exp); a block runs its share as
// segments (unit, tile range) in warp-specialised roles that overlap every
// stage of a tile with the tensor cores' work on others.  (With more units
// than the schedule holds, each block takes one whole unit.)
// Shared memory carries only what the tensor cores must read from it (the
// dequantised key and value tiles); the queries, the scores, the weights and
// the output accumulator live in tensor memory:
//  * a producer warp bulk-copies each tile's packed codes and norms (1-D
//    TMA copies, no multicast) into a ring of four stages;
//  * eight dequantising warps turn a stage into fp16 operand tiles in shared
//    memory, laid out as the tensor cores read them (K-major, 128-byte
//    swizzle), double-buffered, through tables that map a field of two codes
//    to a pair of fp16 centroids (one copy of each table per lane, so that the
//    lookups of a warp never share a bank): K~ [64 keys x 128 channels], the
//    centroids (the key norms multiply the fp32 scores instead: an fp16
//    product per element would add a rounding error that the exponential
//    amplifies with the score), and V~ [64 keys x 128 channels], the
//    centroids times the value norms, in the same per-key layout, which the
//    P V~ product reads as an MN-major operand; the tile's key norms go to a
//    small ring the softmax reads;
//  * one warp issues the tcgen05 MMAs (an elected lane), both with A in
//    tensor memory:
//    S = (Q~hi + Q~lo) K~^T (M = 128, N = 64, K = 128, into one of two score
//    buffers) for tile j + 1 before O += P V~ (M = 128, N = 128, K = 64,
//    accumulated across tiles) for tile j, and signals completions through
//    tcgen05.commit on mbarriers;
//  * four softmax warps own one query row per thread (the tensor-memory lane
//    of the row): they rotate the queries and store them as two fp16 terms
//    (rows scaled to a largest magnitude of 1, so the scores keep about 22
//    bits), then per tile read their scores, apply the causal limit and the
//    online softmax with a lazy reference (the accumulator is rescaled only
//    when a score passes the reference by more than 2^8), and store the fp16
//    weights (at most 2^8) as the A operand of P V~.  The end divides by the
//    softmax sum and applies the inverse rotation.
// Two idle warps complete the producer and MMA warps' warpgroup, so that the
// block's registers can be moved between warpgroups (setmaxnreg): the
// softmax warps run at 160 registers, the dequantising warps at 128, the
// producer, MMA and idle warps at 96.  The attention kernel and the merge
// kernel start as programmatic dependents of the kernel before them on the
// stream.
// The keys' and values' fp16 centroids carry the codebook's fp16 scale (as in
// the decode kernels; the values' also a factor 2^-4 that keeps centroid x
// norm inside the fp16 range), removed from the scores and the output.
//
// Every mbarrier wait is bounded (about a second, then TQ_DEVERR_TIMEOUT; the
// block stops issuing work, waits for its copies and MMAs, and frees its
// tensor memory).

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
constexpr int NS = 4;                    // code stages
constexpr int SOFTMAX_WARPS = 4, DEQ_WARPS = 8;
constexpr int DEQ0 = SOFTMAX_WARPS * 32;           // first dequantising thread
constexpr int PRODUCER = DEQ0 + DEQ_WARPS * 32;    // first thread of the producer warp
constexpr int MMA_WARP = PRODUCER / 32 + 1;        // MMA issuer warp (also allocates tensor memory)
// Two idle warps complete the producer and MMA warps' warpgroup, so that the
// block's registers can be moved between warpgroups (setmaxnreg works on
// whole warpgroups): launched at 128 registers a thread (16 warps x 32 x 128
// = the SM's 64 K), the softmax warpgroup takes 160 and the producer's gives
// up to 96 (per sub-partition, one warp of each: +32 and -32).
constexpr int NTHREADS = 16 * 32;
constexpr int REGS_SOFTMAX = 160, REGS_LIGHT = 96;
static_assert(MMA_WARP < NTHREADS / 32 && MMA_WARP / 4 == PRODUCER / 128 && PRODUCER / 128 == NTHREADS / 128 - 1,
              "the producer and MMA warps share the last warpgroup");
static_assert(SOFTMAX_WARPS == 4 && 4 * REGS_SOFTMAX + 8 * 128 + 4 * REGS_LIGHT == 16 * 128,
              "the register split adds up to the launch's");
// tensor-memory columns (32-bit; fp16 operands take two elements a column)
constexpr uint32_t TM_QHI = 0;           // Q~ / qscale, fp16 [128 rows][128 ch]
constexpr uint32_t TM_QLO = 64;          // its fp16 remainder
constexpr uint32_t TM_S = 128;           // 2 x fp32 scores [128 rows][64 keys]
constexpr uint32_t TM_P = 256;           // 2 x fp16 weights [128 rows][64 keys]
constexpr uint32_t TM_O = 320;           // fp32 accumulator [128 rows][128 ch]
constexpr uint32_t TMEM_COLS = 512;
constexpr long long WAIT_LIMIT = 2000000000ll;  // clock cycles (~1 s)
constexpr float VFOLD = 1.0f / 16.0f;           // value centroids x norms enter V~ scaled by 2^-4
constexpr float LAZY = 8.0f;                    // log2 headroom before the reference moves

// shared-memory map (offsets from a 1024-byte aligned base); the code tables'
// sizes depend on the widths
constexpr uint32_t SM_K = 0;                       // 2 x fp16 [64 keys][128 ch] (2 column blocks of 8 KB each)
constexpr uint32_t SM_VT = SM_K + 2 * BK * D * 2;  // 2 x fp16 V~ [64 keys][128 ch], the layout of K~
constexpr uint32_t STAGE_BYTES = BK * 64 + BK * 64 + BK * 2 + BK * 2;  // K codes, V codes, K norms, V norms
constexpr uint32_t ST_KC = 0, ST_VC = BK * 64, ST_KN = 2 * BK * 64, ST_VN = 2 * BK * 64 + BK * 2;
constexpr uint32_t SM_STAGE = SM_VT + 2 * D * BK * 2;
constexpr uint32_t SM_KNR = SM_STAGE + NS * STAGE_BYTES;   // fp32 key norms of the last four tiles [4][64]
constexpr uint32_t SM_CENT = SM_KNR + 4 * BK * 4;          // fp16 key centroids [16], value centroids [16]
constexpr uint32_t SM_BAR = SM_CENT + 64;
// mbarriers (8 bytes each)
constexpr int B_FULL = 0, B_EMPTY = NS, B_KFULL = 2 * NS, B_KEMPTY = B_KFULL + 2, B_VFULL = B_KEMPTY + 2,
              B_VEMPTY = B_VFULL + 2, B_SFULL = B_VEMPTY + 2, B_SEMPTY = B_SFULL + 2, B_PFULL = B_SEMPTY + 2,
              B_PEMPTY = B_PFULL + 2, B_QREADY = B_PEMPTY + 2, B_FINAL = B_QREADY + 1, NBARS = B_FINAL + 1;
// (B_PEMPTY[j % 2] also tells that every P V up to tile j is in the accumulator:
// commits complete in order.  Waiting on it rather than on one shared
// barrier keeps every wait within one phase of the barrier's state.)
constexpr uint32_t SM_TMEM = SM_BAR + NBARS * 8;   // tensor-memory address
constexpr uint32_t SM_FLAG = SM_TMEM + 4;          // abort flag
constexpr uint32_t SM_SEG = (SM_FLAG + 4 + 15) & ~15u;     // uint32 [4]: the block's g0, g1, g1x, C (spread mode)
constexpr uint32_t SM_USTART = SM_SEG + 16;                // int: the block's first unit
// uint32 [NTHREADS]: per-thread tile sums in the prologue, then each thread's
// segment iterator (kept here, not in a register, through the tile loops)
constexpr uint32_t SM_SCAN = SM_SEG + 32;
constexpr int SCHED_MAX = 4096;                            // most units the shared schedule holds
constexpr uint32_t SM_SCHED = SM_SCAN + NTHREADS * 4;      // uint32 [units + 1]: tiles before each unit
constexpr uint32_t SM_KLUT = (SM_SCHED + (SCHED_MAX + 1) * 4 + 127) & ~127u;  // key code table, one copy per lane
// A code table maps a field of two codes (2 BITS bits) to their fp16
// centroids, packed, with 32 copies interleaved word by word: entry e of lane
// l is word 32 e + l, so a warp's lookups fall in 32 distinct banks.
__host__ __device__ constexpr uint32_t lut_bytes(int bits) { return 32u * 4u * (1u << (2 * bits)); }
// The key table of 4-bit codes has 256-byte rows instead (entry e of lane l
// at byte 256 e + 4 l, the upper half of each row unused), so that a lookup
// address is one byte permute of the code word (code byte in bits 8-15, the
// lane's offset below) and the load's immediate offset holds the table's
// shared-window address: dynamic shared memory begins at window address
// SMEM_WINDOW (the host checks the reserved size), where the kernel's
// 1024-byte alignment leaves it.
constexpr uint32_t SMEM_WINDOW = 1024;
__host__ __device__ constexpr bool wide_klut(int kb) { return kb == 4; }
__host__ __device__ constexpr uint32_t klut_bytes(int kb) { return wide_klut(kb) ? 65536u : lut_bytes(kb); }
__host__ __device__ constexpr uint32_t sm_vlut(int kb) { return SM_KLUT + klut_bytes(kb); }
__host__ __device__ constexpr uint32_t sm_alloc(int kb, int vb) { return sm_vlut(kb) + lut_bytes(vb) + 1024; }
static_assert(sm_alloc(4, 4) <= 227u * 1024u, "the largest code tables must fit a block's shared memory");

struct Args {
    const uint8_t* k_codes;
    const uint8_t* v_codes;
    const uint16_t* k_norms;
    const uint16_t* v_norms;
    const void* q;           // [batch][n_new][hq][d]
    const int32_t* positions;
    float* out;              // [batch][n_new][hq][d]
    uint32_t* err;
    int q_dtype, batch, hq, hkv, group, capacity, n_new, tok_per_tile;
    int staged_norms;        // capacity % 8 == 0: norms ride in the bulk copies
    int qtiles, units;       // query blocks per (sequence, kv head); units = batch * hkv * qtiles
    int spread;              // 1: the blocks share the (unit, key tile) sequence evenly (see the kernel)
    uint32_t* sched;         // [units + 1] the tile schedule, written by block 0 for the merge kernel
    float* parts;            // [2 * blocks][BM][D + 2] partial outputs of cut units
    float score_scale;       // sm_scale * log2(e) / alpha_k
    float out_scale;         // 1 / (alpha_v * VFOLD)
    uint32_t signs[4];
    uint16_t kcent[16];      // fp16 bits of alpha_k * key centroid
    uint16_t vcent[16];      // fp16 bits of alpha_v * VFOLD * value centroid
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

// One query row (D values of dtype 0 fp32, 1 bf16 or 2 fp16, 16-byte
// aligned) into x: the dtype is chosen once and eight 16-byte loads are in
// flight at a time (loads of four values with the dtype tested at each
// came one after another, an L2 round trip apiece).
__device__ __forceinline__ void load_row(const void* base, size_t off, int dtype, float (&x)[D]) {
    if (dtype == 0) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
#pragma unroll
        for (int h = 0; h < D / 32; ++h) {
            float4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = p[8 * h + i];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = 32 * h + 4 * i;
                x[c] = v[i].x;
                x[c + 1] = v[i].y;
                x[c + 2] = v[i].z;
                x[c + 3] = v[i].w;
            }
        }
        return;
    }
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off);
#pragma unroll
    for (int h = 0; h < D / 64; ++h) {
        uint4 w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = p[8 * h + i];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
            const int c = 64 * h + 8 * i;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (dtype == 1) {  // bf16: the upper half of an fp32
                    x[c + 2 * k] = __uint_as_float(u[k] << 16);
                    x[c + 2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
                } else {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
                    x[c + 2 * k] = f.x;
                    x[c + 2 * k + 1] = f.y;
                }
            }
        }
    }
}

__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// One unit of work: 128 query rows (TT tokens x G heads) of one (sequence,
// kv head); units are numbered (b, kv, qt), qt fastest.
struct Unit {
    int qt, kv, b, tok0, ntok, start, kend, ntiles;
    bool bad;  // the sequence's chunk position is out of range: no tiles, zero rows
};

__device__ __forceinline__ Unit unit_of(const Args& a, int u) {
    Unit x;
    x.qt = u % a.qtiles;
    const int bk = u / a.qtiles;
    x.kv = bk % a.hkv;
    x.b = bk / a.hkv;
    x.tok0 = x.qt * a.tok_per_tile;
    x.start = a.positions[x.b];
    x.bad = x.start < 0 || x.start > a.capacity - a.n_new;
    x.ntok = x.bad ? 0 : min(a.tok_per_tile, a.n_new - x.tok0);
    x.kend = x.ntok > 0 ? x.start + x.tok0 + x.ntok : 0;  // keys [0, kend) are needed by some row
    x.ntiles = (x.kend + BK - 1) / BK;
    return x;
}

// A 32-bit store to a shared-window address.
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// This block's key tiles [j0, j1) of unit u (one the block visits).
__device__ __forceinline__ void segment_bounds(const Args& a, const uint8_t* smem, int u, int& j0, int& j1) {
    if (!a.spread) {
        j0 = 0;
        j1 = unit_of(a, u).ntiles;
        return;
    }
    const volatile uint32_t* seg = reinterpret_cast<const volatile uint32_t*>(smem + SM_SEG);
    const volatile uint32_t* P = reinterpret_cast<const volatile uint32_t*>(smem + SM_SCHED);
    const uint32_t pu = P[u], pn = P[u + 1], g0 = seg[0], g1 = seg[1];
    j0 = static_cast<int>((pu > g0 ? pu : g0) - pu);
    j1 = static_cast<int>((pn < g1 ? pn : g1) - pu);
}

// The block's share of the work as segments (unit, key tiles [j0, j1)),
// one per call.  The iterator (the first unit not yet visited) is the
// shared word at `slot`, so that it takes no register through the tile
// loops; segment_unit(slot) is the unit of the segment last returned.
// Spread mode: the units' tiles form one sequence (P[u] tiles before unit
// u); with C = min(blocks, total) sharing, block c takes tiles
// [c total / C, (c + 1) total / C) of it, so a unit can be cut between
// blocks; a unit without tiles goes to the block whose range holds its
// start (the last block for those at the very end).  Otherwise block c is
// unit c, whole.
__device__ __forceinline__ bool next_segment(const Args& a, const uint8_t* smem, uint32_t slot, int& j0, int& j1) {
    const int it = static_cast<int>(ptx::lds32(slot));
    if (it >= a.units || (!a.spread && it != static_cast<int>(blockIdx.x))) return false;
    // (a unit starting at or past the range's end, g1x, belongs to a later block)
    if (a.spread && reinterpret_cast<const volatile uint32_t*>(smem + SM_SCHED)[it] >=
                        reinterpret_cast<const volatile uint32_t*>(smem + SM_SEG)[2])
        return false;
    segment_bounds(a, smem, it, j0, j1);
    sts32(slot, static_cast<uint32_t>(it + 1));
    return true;
}

// The unit of the segment that next_segment returned last.
__device__ __forceinline__ int segment_unit(uint32_t slot) { return static_cast<int>(ptx::lds32(slot)) - 1; }

// Whether unit u, which has tiles in this block, has some in another block too.
__device__ __forceinline__ bool unit_is_cut(const Args& a, const uint8_t* smem, int u) {
    if (!a.spread) return false;
    const volatile uint32_t* seg = reinterpret_cast<const volatile uint32_t*>(smem + SM_SEG);
    const volatile uint32_t* P = reinterpret_cast<const volatile uint32_t*>(smem + SM_SCHED);
    return P[u] < seg[0] || P[u + 1] > seg[1];
}

// The block whose range holds global tile g (spread mode, g < total).
__device__ __forceinline__ int block_of(uint32_t g, uint32_t total, uint32_t nblocks) {
    return static_cast<int>(((static_cast<uint64_t>(g) + 1) * nblocks - 1) / total);
}

// A block holds at most two pieces of cut units: the head of the unit its
// range starts (the first block of that unit: slot 2c + 1) and a piece of a
// unit begun earlier (slot 2c).  A slot is [BM][D] fp32 O rows, then the
// rows' m and l.
constexpr size_t PART_FLOATS = static_cast<size_t>(BM) * (D + 2);
__device__ __forceinline__ int part_slot(int block, int first_block) { return 2 * block + (block == first_block); }

// The code table of BITS-bit codes: field e (code e & m, then code e >> BITS)
// -> fp16 centroid pair, for every lane.
// (ROW: words per entry, 32, or 64 for the 256-byte rows)
template <int BITS, int ROW = 32>
__device__ void build_lut(uint32_t* lut, const uint16_t* cent, int t, int nthreads) {
    constexpr int n = 32 << (2 * BITS), m = (1 << BITS) - 1;
    for (int i = t; i < n; i += nthreads) {
        const int e = i >> 5;
        lut[e * ROW + (i & 31)] = pack2(cent[e & m], cent[e >> BITS]);
    }
}

// One fp16 operand tile (64 keys x 128 channels, K-major, 128-byte swizzle)
// from a stage's packed codes (rows of 16 BITS bytes, LSB-first): this
// thread's share is channel group cg = dt % 16 (8 channels) of keys
// dt / 16 + 16 i.  All shared addresses are 32-bit shared-window addresses;
// `lut` is this lane's column of the code table.  The loads of the four
// groups go out together, then the lookups, then the stores.  SCALE: times
// the key's fp16 norm (from the stage, or from `gnorms` when the stage holds
// none).  Keys at or past nk are written as zeros.
template <int BITS, bool SCALE, bool WIDE = false>
__device__ __forceinline__ void dequant_tile(uint32_t tile, uint32_t codes, uint32_t lut, uint32_t snorms,
                                             const uint16_t* gnorms, bool staged, int dt, int nk) {
    static_assert(!WIDE || BITS == 4, "the 256-byte-row table holds 4-bit code pairs");
    constexpr int RB = 16 * BITS, W = 2 * BITS, IT = BK * (D / 8) / (DEQ_WARPS * 32);
    constexpr uint32_t M = (1u << W) - 1;
    const int cg = dt & 15, k0 = dt >> 4;
    uint32_t c8[IT];
#pragma unroll
    for (int i = 0; i < IT; ++i) {
        const uint32_t row = codes + (k0 + 16 * i) * RB;
        if constexpr (BITS == 4) {
            c8[i] = ptx::lds32(row + 4 * cg);
        } else if constexpr (BITS == 2) {
            c8[i] = ptx::lds32(row + 4 * (cg >> 1)) >> (16 * (cg & 1));
        } else {  // 24 bits from bit 24 cg: may straddle two words
            const int bit = 24 * cg, w = bit >> 5, sh = bit & 31;
            const uint32_t lo = ptx::lds32(row + 4 * w), hi = ptx::lds32(row + 4 * min(w + 1, RB / 4 - 1));
            c8[i] = sh <= 8 ? lo >> sh : __funnelshift_r(lo, hi, sh);
        }
    }
    uint32_t n2[IT];
    if constexpr (SCALE) {
#pragma unroll
        for (int i = 0; i < IT; ++i) {
            const int key = k0 + 16 * i;
            const uint16_t nb = staged ? ptx::lds16(snorms + 2 * key) : (key < nk ? gnorms[key] : uint16_t(0));
            n2[i] = nb | (static_cast<uint32_t>(nb) << 16);
        }
    }
    uint4 v[IT];
    if constexpr (WIDE) {
        // byte permute: bits 0-7 the lane's offset, bits 8-15 code byte j
        const uint32_t l4 = 4u * static_cast<uint32_t>(dt & 31);
        constexpr uint32_t T = SMEM_WINDOW + SM_KLUT;
#pragma unroll
        for (int i = 0; i < IT; ++i) {
            v[i].x = ptx::lds32_imm<T>(__byte_perm(c8[i], l4, 0x7604));
            v[i].y = ptx::lds32_imm<T>(__byte_perm(c8[i], l4, 0x7614));
            v[i].z = ptx::lds32_imm<T>(__byte_perm(c8[i], l4, 0x7624));
            v[i].w = ptx::lds32_imm<T>(__byte_perm(c8[i], l4, 0x7634));
        }
    } else {
#pragma unroll
        for (int i = 0; i < IT; ++i) {
            v[i].x = ptx::lds32(lut + 128u * (c8[i] & M));
            v[i].y = ptx::lds32(lut + 128u * ((c8[i] >> W) & M));
            v[i].z = ptx::lds32(lut + 128u * ((c8[i] >> (2 * W)) & M));
            v[i].w = ptx::lds32(lut + 128u * ((c8[i] >> (3 * W)) & M));
        }
    }
    if constexpr (SCALE) {
#pragma unroll
        for (int i = 0; i < IT; ++i) {
            const __half2 f = *reinterpret_cast<const __half2*>(&n2[i]);
            __half2* h = reinterpret_cast<__half2*>(&v[i]);
#pragma unroll
            for (int e = 0; e < 4; ++e) h[e] = __hmul2(h[e], f);
        }
    }
    if (nk < BK) {  // the last, partial tile only
#pragma unroll
        for (int i = 0; i < IT; ++i)
            if (k0 + 16 * i >= nk) v[i] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < IT; ++i) ptx::sts128(tile + tc::sw128_offset(k0 + 16 * i, 8 * cg, BK), v[i]);
}

template <int KB, int VB>
__global__ void __launch_bounds__(NTHREADS, 1) prefill_kernel(const __grid_constant__ Args a) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, reached by pointer arithmetic on the shared
    // array (a round trip through an integer would hide the address space and
    // turn every access below into a generic load or store)
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = ptx::smem_addr(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Launched as a programmatic dependent of the append kernel, which lets it
    // start only after every earlier kernel has finished: everything but the
    // chunk's own slots (codes and norms of positions[b] ..) is final here, and
    // the producer waits for the append before it copies a tile holding any
    // of them.  The merge kernel may start launching now (it waits for this
    // one to finish).
    ptx::launch_dependents();
    const uint32_t bars = sbase + SM_BAR;
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_FLAG);
    auto fail = [&]() {
        if (!*abort_flag && a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
        *abort_flag = 1;
    };
    // bounded wait on phase `parity` of mbarrier i; false (and the abort flag set) when it runs out
    auto wait = [&](int i, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (!ptx::mbar_wait_bounded_lean(bar(i), parity, WAIT_LIMIT)) {
            fail();
            return false;
        }
        return true;
    };
    const int G = a.group, TT = a.tok_per_tile;

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            ptx::mbar_init(bar(B_FULL + i), 1);
            ptx::mbar_init(bar(B_EMPTY + i), DEQ_WARPS);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(B_KFULL + i), DEQ_WARPS);
            ptx::mbar_init(bar(B_KEMPTY + i), 1);
            ptx::mbar_init(bar(B_VFULL + i), DEQ_WARPS);
            ptx::mbar_init(bar(B_VEMPTY + i), 1);
            ptx::mbar_init(bar(B_SFULL + i), 1);
            ptx::mbar_init(bar(B_SEMPTY + i), SOFTMAX_WARPS);
            ptx::mbar_init(bar(B_PFULL + i), SOFTMAX_WARPS);
            ptx::mbar_init(bar(B_PEMPTY + i), 1);
        }
        ptx::mbar_init(bar(B_QREADY), SOFTMAX_WARPS);
        ptx::mbar_init(bar(B_FINAL), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (tid < 32) reinterpret_cast<uint16_t*>(smem + SM_CENT)[tid] = tid < 16 ? a.kcent[tid] : a.vcent[tid - 16];
    if (warp == MMA_WARP) {
        tc::tmem_alloc(sbase + SM_TMEM, TMEM_COLS);
        tc::tmem_relinquish();
    }
    // ---- the schedule (spread mode): P[u] = tiles of the units before u,
    // from per-thread sums over contiguous runs of units and a scan of those
    uint32_t* P = reinterpret_cast<uint32_t*>(smem + SM_SCHED);
    uint32_t* scan = reinterpret_cast<uint32_t*>(smem + SM_SCAN);
    const int U = a.units;
    const int per = (U + NTHREADS - 1) / NTHREADS, u0 = tid * per, u1 = min(U, u0 + per);
    if (a.spread) {
        uint32_t sum = 0;
        for (int u = u0; u < u1; ++u) sum += static_cast<uint32_t>(unit_of(a, u).ntiles);
        scan[tid] = sum;
    }
    __syncthreads();
    if (a.spread && warp == 0) {  // exclusive scan of the NTHREADS sums
        constexpr int PER_LANE = NTHREADS / 32;
        uint32_t v[PER_LANE], t = 0;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            v[i] = scan[lane * PER_LANE + i];
            t += v[i];
        }
        uint32_t incl = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        uint32_t run = incl - t;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            scan[lane * PER_LANE + i] = run;
            run += v[i];
        }
    }
    __syncthreads();
    if (a.spread) {
        // (every block computes the same schedule; block 0 also leaves it in
        // the workspace for the merge kernel)
        const bool keep = blockIdx.x == 0;
        uint32_t run = scan[tid];
        for (int u = u0; u < u1; ++u) {
            P[u] = run;
            if (keep) a.sched[u] = run;
            run += static_cast<uint32_t>(unit_of(a, u).ntiles);
        }
        if (u1 == U && u0 < u1) {
            P[U] = run;
            if (keep) a.sched[U] = run;
        }
        if (U == 0 && tid == 0) {
            P[0] = 0;
            if (keep) a.sched[0] = 0;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SM_TMEM);
    constexpr int kbytes = 16 * KB, vbytes = 16 * VB;  // packed row sizes

    // this block's range of the tile sequence, and its first unit
    if (tid == 0) {
        const int cb = static_cast<int>(blockIdx.x);
        int ustart = cb;
        if (a.spread) {
            // (the host spreads only while the tile total fits 31 bits)
            const uint32_t total = P[U];
            // no more sharing blocks than tiles: each one's range then holds at
            // least one tile, so a cut unit's pieces are in every block from its
            // first to its last; the blocks past C take nothing
            const uint32_t C = gridDim.x > total ? (total > 0 ? total : 1u) : gridDim.x;
            uint32_t* seg = reinterpret_cast<uint32_t*>(smem + SM_SEG);
            const uint32_t c = static_cast<uint32_t>(cb);
            const uint32_t g0 = static_cast<uint32_t>(static_cast<uint64_t>(c) * total / C);
            const uint32_t g1 = static_cast<uint32_t>(static_cast<uint64_t>(c + 1) * total / C);
            seg[0] = g0;
            seg[1] = g1;
            seg[2] = c == C - 1 ? total + 1 : g1;
            seg[3] = C;
            if (c >= C) {
                ustart = U;
            } else {
                int lo = 0, hi = U;  // first u with P[u + 1] > g0 or P[u] >= g0
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (P[mid + 1] > g0 || P[mid] >= g0) hi = mid;
                    else lo = mid + 1;
                }
                ustart = lo;
            }
        }
        *reinterpret_cast<int*>(smem + SM_USTART) = ustart;
    }
    __syncthreads();
    // each thread's segment iterator (its prologue scan word is free now)
    const uint32_t slot = sbase + SM_SCAN + 4u * static_cast<uint32_t>(tid);
    sts32(slot, static_cast<uint32_t>(*reinterpret_cast<volatile int*>(smem + SM_USTART)));

    // The register split (setmaxnreg works on whole warpgroups, each at one
    // instruction): the last warpgroup (producer, MMA issuer, two idle warps)
    // gives up registers, then the softmax warpgroup takes them; every role's
    // code follows its own warpgroup's instruction, so the compiler allocates
    // it within that warpgroup's count.  (The increase is covered by the
    // decrease, so it cannot wait for ever.)
    if (warp >= NTHREADS / 32 - 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_LIGHT));
        if (warp == PRODUCER / 32) {
            // ---------------------------------------------------------- producer
            // the whole warp waits; one elected lane issues the copies
            const bool leader = tc::elect_one();
            int gi = 0;  // tiles issued so far (the ring position)
            int j0, j1;
            while (next_segment(a, smem, slot, j0, j1)) {
                const Unit x = unit_of(a, segment_unit(slot));
                // ring tile g holds the unit's keys from g BK - koff (koff = (gi - j0) BK);
                // knew: the chunk's first slot in those coordinates
                const int koff = (gi - j0) * BK, kend = x.kend + koff, knew = x.start + koff;
                const long long row0 =
                    static_cast<long long>((static_cast<size_t>(x.b) * a.hkv + x.kv) * a.capacity) - koff;
                for (const int gend = gi + (j1 - j0); gi < gend; ++gi) {
                    const int s = gi % NS;
                    // (the ring is four tiles deep: the producer can poll slowly and
                    // leave the issue slots of its sub-partition to the working warps)
                    if (gi >= NS) {
                        if (*abort_flag) goto produced;
                        if (!ptx::mbar_wait_bounded_sleep(bar(B_EMPTY + s), ((gi - NS) / NS) & 1, WAIT_LIMIT, 256)) {
                            fail();
                            goto produced;
                        }
                    }
                    if (leader) {
                        const int key0 = gi * BK, nk = min(BK, kend - key0);
                        if (key0 + nk > knew) ptx::wait_prerequisites();  // the tile holds appended slots
                        const size_t row = static_cast<size_t>(row0 + key0);
                        const uint32_t dst = sbase + SM_STAGE + s * STAGE_BYTES;
                        const int n8 = (nk + 7) & ~7;  // norms move in 16-byte pieces (8 keys)
                        const uint32_t bytes = nk * (kbytes + vbytes) + (a.staged_norms ? n8 * 4 : 0);
                        ptx::mbar_arrive_expect_tx(bar(B_FULL + s), bytes);
                        ptx::bulk_copy_g2s(dst + ST_KC, a.k_codes + row * kbytes, nk * kbytes, bar(B_FULL + s));
                        ptx::bulk_copy_g2s(dst + ST_VC, a.v_codes + row * vbytes, nk * vbytes, bar(B_FULL + s));
                        if (a.staged_norms) {
                            // capacity and the unit's key offset are multiples of 8: the
                            // rounded range stays inside the cache
                            ptx::bulk_copy_g2s(dst + ST_KN, a.k_norms + row, n8 * 2, bar(B_FULL + s));
                            ptx::bulk_copy_g2s(dst + ST_VN, a.v_norms + row, n8 * 2, bar(B_FULL + s));
                        }
                    }
                    __syncwarp();
                }
            }
        produced:
            // every copy issued must land before the block may exit
            for (int k = max(0, gi - NS); k < gi; ++k)
                ptx::mbar_wait_bounded(bar(B_FULL + k % NS), (k / NS) & 1, WAIT_LIMIT);
        } else if (warp == MMA_WARP) {
            // ------------------------------------------------------- MMA issuer
            // the whole warp waits; one elected lane issues the MMAs and commits
            const bool leader = tc::elect_one();
            const uint32_t idesc_s = tc::idesc_f16(BM, BK), idesc_o = tc::idesc_f16_bmn(BM, D);
            // descriptors are linear in the start address: the K slices and
            // buffers are fixed offsets (in 16-byte units) from these
            const uint64_t kdesc0 = tc::sw128_desc(sbase + SM_K);
            const uint64_t vdesc0 = tc::sw128_mn_desc(sbase + SM_VT, BK * 128, 1024);
            auto issue_s = [&](int gi) -> bool {
                const int bf = gi & 1;
                if (!wait(B_KFULL + bf, (gi >> 1) & 1)) return false;
                if (gi >= 2 && !wait(B_SEMPTY + bf, ((gi - 2) >> 1) & 1)) return false;
                tc::fence_after_sync();
                if (leader) {
                    const uint64_t kd = kdesc0 + static_cast<uint64_t>(bf * (BK * D * 2) >> 4);
                    const uint32_t sd = tmem + TM_S + BK * bf;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        // 16 channels per step: 32 bytes within a 64-channel block
                        const uint64_t bd = kd + static_cast<uint64_t>(((ks >> 2) * (BK * 128) + (ks & 3) * 32) >> 4);
                        tc::mma_f16_ts(sd, tmem + TM_QHI + 8 * ks, bd, idesc_s, ks > 0);
                        tc::mma_f16_ts(sd, tmem + TM_QLO + 8 * ks, bd, idesc_s, true);
                    }
                    tc::commit(bar(B_SFULL + bf));
                    tc::commit(bar(B_KEMPTY + bf));
                }
                __syncwarp();
                return true;
            };
            // first: the segment's first tile (the accumulator starts afresh)
            auto issue_pv = [&](int gi, bool first) -> bool {
                const int bf = gi & 1;
                if (!wait(B_PFULL + bf, (gi >> 1) & 1)) return false;
                if (!wait(B_VFULL + bf, (gi >> 1) & 1)) return false;
                tc::fence_after_sync();
                if (leader) {
                    const uint64_t vd = vdesc0 + static_cast<uint64_t>(bf * (BK * D * 2) >> 4);
                    const uint32_t pa = tmem + TM_P + (BK / 2) * bf;
                    // V~ [64 keys][128 ch]: 16 keys per step = two 1024-byte K groups;
                    // the two 64-channel blocks lie 64 rows x 128 bytes apart
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks)
                        tc::mma_f16_ts(tmem + TM_O, pa + 8 * ks, vd + static_cast<uint64_t>(ks * 2048 >> 4), idesc_o,
                                       !first || ks > 0);
                    tc::commit(bar(B_PEMPTY + bf));
                    tc::commit(bar(B_VEMPTY + bf));
                }
                __syncwarp();
                return true;
            };
            int gi = 0, qs = 0;  // tiles issued, segments with tiles begun (the QREADY phase)
            int j0, j1;
            while (next_segment(a, smem, slot, j0, j1)) {
                if (j1 <= j0) continue;  // no tiles: the softmax writes the unit's zero rows alone
                // the segment's queries are in tensor memory (which also tells
                // that the previous segment's output has been read)
                if (!wait(B_QREADY, qs & 1)) break;
                ++qs;
                if (!issue_s(gi)) break;
                const int gfirst = gi;
                for (const int gend = gi + (j1 - j0); gi < gend; ++gi) {
                    if (gi + 1 < gend && !issue_s(gi + 1)) goto issued;
                    if (!issue_pv(gi, gi == gfirst)) goto issued;
                }
            }
        issued:
            // every tensor-core operation issued completes before the block
            // frees its tensor memory (bounded, also after an abort)
            if (leader) {
                tc::commit(bar(B_FINAL));
                ptx::mbar_wait_bounded(bar(B_FINAL), 0, WAIT_LIMIT);
            }
            __syncwarp();
        }
    } else if (warp < SOFTMAX_WARPS) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
        // ---------------------------------------------------------- softmax
        const int r = tid;
        const int rt = r / G, rh = r % G;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float inv_sqrt_d = 0.08838834764831845f;
        int gi = 0;  // tiles done (the ring position)
        int j0, j1;
        // rows of a unit that exist in the output (all of them but the padding
        // of a last, partial query block), and this thread's
        auto out_row = [&](const Unit& x) -> float* {
            const bool row_out = rt < min(TT, a.n_new - x.tok0) && rt * G + rh < BM;
            return row_out ? a.out + ((static_cast<size_t>(x.b) * a.n_new + x.tok0 + rt) * a.hq + x.kv * G + rh) * D
                           : nullptr;
        };
        while (next_segment(a, smem, slot, j0, j1)) {
            // (what the tile loop needs is worked out again after the query's
            // preparation, which holds a 128-value row: a value kept through
            // it would be spilled, and reloaded at every tile)
            float qscale = 0.f;  // largest |q~| of the row: the fp16 terms hold q~ / qscale
            {
                const Unit x = unit_of(a, segment_unit(slot));
                const bool row_ok = rt < x.ntok && rt * G + rh < BM;
                if (j1 <= j0) {
                    // no tiles: a sequence whose chunk position was refused (zero rows)
                    if (x.bad && x.qt == 0 && x.kv == 0 && tid == 0 && a.err) atomicOr(a.err, TQ_DEVERR_POSITION);
                    float* dst = out_row(x);
                    if (dst) {
#pragma unroll
                        for (int c = 0; c < D; c += 4)
                            *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    continue;
                }
                float xq[D];
                if (row_ok) {
                    const size_t qoff =
                        ((static_cast<size_t>(x.b) * a.n_new + x.tok0 + rt) * a.hq + x.kv * G + rh) * D;
#pragma unroll
                    load_row(a.q, qoff, a.q_dtype, xq);
#pragma unroll
                    for (int c = 0; c < D; ++c) xq[c] = flip_sign(xq[c], (a.signs[c >> 5] >> (c & 31)) & 1u);
                    fwht128(xq);
                } else {
#pragma unroll
                    for (int c = 0; c < D; ++c) xq[c] = 0.f;
                }
                float amax = 0.f;
#pragma unroll
                for (int c = 0; c < D; ++c) amax = fmaxf(amax, fabsf(xq[c]));
                qscale = amax * inv_sqrt_d;
                const float rsq = amax > 0.f ? 1.f / amax : 0.f;
#pragma unroll
                for (int c = 0; c < D; c += 16) {
                    uint32_t hw[8], lw[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float v0 = xq[c + 2 * e] * rsq, v1 = xq[c + 2 * e + 1] * rsq;
                        const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
                        hw[e] = pack2(__half_as_ushort(h0), __half_as_ushort(h1));
                        lw[e] = half2_bits(v0 - __half2float(h0), v1 - __half2float(h1));
                    }
                    tc::st_8cols(tmem + lane_base + TM_QHI + c / 2, hw);
                    tc::st_8cols(tmem + lane_base + TM_QLO + c / 2, lw);
                }
            }
            tc::st_wait();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(B_QREADY));
            // scores in log2 units: S kn rs; a zero query row keeps rs > 0 so that a
            // masked (-inf) score stays -inf
            const float rs = fmaxf(qscale * a.score_scale, 1e-30f);
            const Unit x = unit_of(a, segment_unit(slot));
            const bool row_ok = rt < x.ntok && rt * G + rh < BM;
            segment_bounds(a, smem, segment_unit(slot), j0, j1);
            // the unit's first query position, in ring coordinates (ring tile g
            // holds the unit's keys from g BK - (gi - j0) BK): keys past
            // dlim + rt are past the row's own position
            const int dlim = x.start + x.tok0 + (gi - j0) * BK;
            float mref = -INFINITY, l = 0.f;
            for (const int gend = gi + (j1 - j0); gi < gend; ++gi) {
                const int bf = gi & 1, key0 = gi * BK;  // (ring coordinates)
                if (!wait(B_SFULL + bf, (gi >> 1) & 1)) goto softmax_done;
                tc::fence_after_sync();
                float sc[BK];
                {
                    float (&sc0)[32] = *reinterpret_cast<float (*)[32]>(&sc[0]);
                    float (&sc1)[32] = *reinterpret_cast<float (*)[32]>(&sc[32]);
                    tc::ld_32cols(tmem + lane_base + TM_S + BK * bf, sc0);
                    tc::ld_32cols(tmem + lane_base + TM_S + BK * bf + 32, sc1);
                }
                tc::ld_wait();
                const float4* kn4 = reinterpret_cast<const float4*>(smem + SM_KNR + (gi & 3) * BK * 4);
#pragma unroll
                for (int i = 0; i < BK; i += 4) {
                    const float4 k4 = kn4[i / 4];
                    const float2 a01 = ptx::fmul2(make_float2(sc[i], sc[i + 1]), make_float2(k4.x, k4.y));
                    const float2 a23 = ptx::fmul2(make_float2(sc[i + 2], sc[i + 3]), make_float2(k4.z, k4.w));
                    sc[i] = a01.x;
                    sc[i + 1] = a01.y;
                    sc[i + 2] = a23.x;
                    sc[i + 3] = a23.y;
                }
                if (key0 + BK - 1 > dlim) {
                    // a tile on the diagonal: keys past the row's own position drop
                    // out (rows outside the chunk are never stored; every key of an
                    // earlier tile is visible to every row of the unit)
                    const int qlim = dlim + rt;
#pragma unroll
                    for (int i = 0; i < BK; ++i)
                        if (!row_ok || key0 + i > qlim) sc[i] = -INFINITY;
                }
                float m4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float m = sc[16 * q];
#pragma unroll
                    for (int i = 1; i < 15; i += 2) m = ptx::fmax3(m, sc[16 * q + i], sc[16 * q + i + 1]);
                    m4[q] = fmaxf(m, sc[16 * q + 15]);
                }
                const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * rs;
                // lazy reference: moves (and the accumulator is rescaled) only when a
                // score passes it by more than 2^LAZY; the weights stay below 2^LAZY
                const bool need = mt > mref + LAZY;
                if (__any_sync(0xffffffffu, need)) {
                    const float mnew = need ? mt : mref;
                    const float c = (need && mref > -INFINITY) ? ptx::ex2(mref - mnew) : 1.f;
                    if (__any_sync(0xffffffffu, mref > -INFINITY)) {
                        // not the segment's first tile (where every reference is
                        // still -inf and the accumulator holds nothing): every P V
                        // of the segment's earlier tiles is in the accumulator
                        if (!wait(B_PEMPTY + ((gi - 1) & 1), ((gi - 1) >> 1) & 1)) goto softmax_done;
                        tc::fence_after_sync();
#pragma unroll 1
                        for (int q8 = 0; q8 < 8; ++q8) {
                            float ov[16];
                            tc::ld_16cols(tmem + lane_base + TM_O + 16 * q8, ov);
                            tc::ld_wait();
#pragma unroll
                            for (int i = 0; i < 16; ++i) ov[i] *= c;
                            tc::st_16cols(tmem + lane_base + TM_O + 16 * q8, ov);
                        }
                    }
                    l *= c;
                    mref = mnew;
                }
                // weights of the tile, fp16, as the A operand of P V~ (stored in
                // two halves of 32 keys)
                if (gi >= 2 && !wait(B_PEMPTY + bf, ((gi - 2) >> 1) & 1)) goto softmax_done;
                const bool live = mref > -INFINITY;
                const float2 rs2 = make_float2(rs, rs), nm2 = make_float2(-mref, -mref);
                float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pw[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float2 t0 = ptx::ffma2(make_float2(sc[32 * h + i], sc[32 * h + i + 1]), rs2, nm2);
                        const float2 t1 = ptx::ffma2(make_float2(sc[32 * h + i + 2], sc[32 * h + i + 3]), rs2, nm2);
                        const float2 p0 = make_float2(ptx::ex2(t0.x), ptx::ex2(t0.y));
                        const float2 p1 = make_float2(ptx::ex2(t1.x), ptx::ex2(t1.y));
                        acc0 = ptx::fadd2(acc0, p0);
                        acc1 = ptx::fadd2(acc1, p1);
                        pw[i / 2] = half2_bits(p0.x, p0.y);
                        pw[i / 2 + 1] = half2_bits(p1.x, p1.y);
                    }
                    if (!live) {  // no visible key yet (a row past the chunk): no weight
#pragma unroll
                        for (int i = 0; i < 16; ++i) pw[i] = 0u;
                    }
                    tc::st_16cols_u(tmem + lane_base + TM_P + (BK / 2) * bf + 16 * h, pw);
                }
                if (live) l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
                tc::st_wait();
                tc::fence_before_sync();
                __syncwarp();
                // the weights are stored and the score buffer, the tile's norms and
                // any accumulator rescale are done with
                if (lane == 0) {
                    ptx::mbar_arrive(bar(B_SEMPTY + bf));
                    ptx::mbar_arrive(bar(B_PFULL + bf));
                }
            }
            // ---- the segment's end: wait for its last P V, read the accumulator
            const bool done = wait(B_PEMPTY + ((gi - 1) & 1), ((gi - 1) >> 1) & 1);
            tc::fence_after_sync();
            float o[D];
            if (done) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float ov[32];
                    tc::ld_32cols(tmem + lane_base + TM_O + 32 * q4, ov);
                    tc::ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[32 * q4 + i] = ov[i];
                }
            } else {
#pragma unroll
                for (int c = 0; c < D; ++c) o[c] = 0.f;
            }
            tc::fence_before_sync();
            if (!done) goto softmax_done;
            bool write = true;
            const int u = segment_unit(slot);
            if (unit_is_cut(a, smem, u)) {
                // a unit cut between blocks: this piece's (O, m, l) rows go to
                // the workspace; the merge kernel that follows on the stream
                // combines the pieces and writes the unit's output
                const volatile uint32_t* seg = reinterpret_cast<const volatile uint32_t*>(smem + SM_SEG);
                const volatile uint32_t* sched = reinterpret_cast<const volatile uint32_t*>(smem + SM_SCHED);
                const uint32_t total = sched[a.units], C = seg[3];
                const int cb = static_cast<int>(blockIdx.x), ca = block_of(sched[u], total, C);
                float* mine = a.parts + static_cast<size_t>(part_slot(cb, ca)) * PART_FLOATS;
#pragma unroll
                for (int c = 0; c < D; c += 4)
                    *reinterpret_cast<float4*>(mine + r * D + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
                mine[BM * D + r] = mref;
                mine[BM * D + BM + r] = l;
                write = false;
            }
            // ---- the unit's output: normalise, inverse rotation
            float* dst = out_row(unit_of(a, u));
            if (write && dst) {
                const float inv = (row_ok && l > 0.f && !*abort_flag) ? a.out_scale / l : 0.f;
#pragma unroll
                for (int c = 0; c < D; ++c) o[c] *= inv;
                fwht128(o);
#pragma unroll
                for (int c = 0; c < D; c += 4) {
                    float4 v;
                    v.x = flip_sign(o[c] * inv_sqrt_d, (a.signs[c >> 5] >> (c & 31)) & 1u);
                    v.y = flip_sign(o[c + 1] * inv_sqrt_d, (a.signs[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u);
                    v.z = flip_sign(o[c + 2] * inv_sqrt_d, (a.signs[(c + 2) >> 5] >> ((c + 2) & 31)) & 1u);
                    v.w = flip_sign(o[c + 3] * inv_sqrt_d, (a.signs[(c + 3) >> 5] >> ((c + 3) & 31)) & 1u);
                    *reinterpret_cast<float4*>(dst + c) = v;
                }
            }
        }
    softmax_done:;
    } else {
        // ------------------------------------------------------ dequantisers
        const int dt = tid - DEQ0;  // 0 .. 32 DEQ_WARPS - 1
        const uint16_t* kcent = reinterpret_cast<const uint16_t*>(smem + SM_CENT);
        const uint16_t* vcent = kcent + 16;
        uint32_t* klut = reinterpret_cast<uint32_t*>(smem + SM_KLUT);
        uint32_t* vlut = reinterpret_cast<uint32_t*>(smem + sm_vlut(KB));
        build_lut<KB, wide_klut(KB) ? 64 : 32>(klut, kcent, dt, DEQ_WARPS * 32);
        build_lut<VB>(vlut, vcent, dt, DEQ_WARPS * 32);
        ptx::named_barrier(1, DEQ_WARPS * 32);
        const uint32_t klane = sbase + SM_KLUT + 4 * lane, vlane = sbase + sm_vlut(KB) + 4 * lane;
        int gi = 0;
        int j0, j1;
        while (next_segment(a, smem, slot, j0, j1)) {
            const Unit x = unit_of(a, segment_unit(slot));
            // ring tile g holds the unit's keys from g BK - koff (as the producer's)
            const int koff = (gi - j0) * BK, kend = x.kend + koff;
            const long long row0 =
                static_cast<long long>((static_cast<size_t>(x.b) * a.hkv + x.kv) * a.capacity) - koff;
            for (const int gend = gi + (j1 - j0); gi < gend; ++gi) {
                const int s = gi % NS, bf = gi & 1;
                if (!wait(B_FULL + s, (gi / NS) & 1)) goto dequantised;
                const uint8_t* st = smem + SM_STAGE + s * STAGE_BYTES;
                const uint32_t sst = sbase + SM_STAGE + s * STAGE_BYTES;
                const int key0 = gi * BK, nk = min(BK, kend - key0);
                const size_t row = static_cast<size_t>(row0 + key0);
                const uint16_t* skn = reinterpret_cast<const uint16_t*>(st + ST_KN);
                // K~[bf]: 64 keys x 16 groups of 8 channels, centroids; the tile's
                // key norms go to the softmax's ring (its tile gi - 4 is done: this
                // tile's K~ buffer was free only after S(gi - 2), which needed the
                // softmax to be through tile gi - 4)
                if (gi >= 2 && !wait(B_KEMPTY + bf, ((gi - 2) >> 1) & 1)) goto dequantised;
                if (dt < BK)
                    reinterpret_cast<float*>(smem + SM_KNR)[(gi & 3) * BK + dt] =
                        dt < nk ? half_bits_to_float(a.staged_norms ? skn[dt] : a.k_norms[row + dt]) : 0.f;
                dequant_tile<KB, false, wide_klut(KB)>(sbase + SM_K + bf * (BK * D * 2), sst + ST_KC, klane, 0u,
                                                       nullptr, true, dt, nk);
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(B_KFULL + bf));
                // V~[bf]: the same per-key layout, centroids x norms
                if (gi >= 2 && !wait(B_VEMPTY + bf, ((gi - 2) >> 1) & 1)) goto dequantised;
                dequant_tile<VB, true>(sbase + SM_VT + bf * (BK * D * 2), sst + ST_VC, vlane, sst + ST_VN,
                                       a.v_norms + row, a.staged_norms != 0, dt, nk);
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(bar(B_VFULL + bf));
                    ptx::mbar_arrive(bar(B_EMPTY + s));  // the stage's codes and norms are used
                }
            }
        }
    dequantised:;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ merge
// The output rows of the units cut between blocks, after the attention
// kernel on the same stream.  Block (u, y) takes rows [32 y, 32 y + 32) of
// unit u (nothing when the unit lies in one block, whose attention block
// wrote it); eight threads per row, sixteen channels each.  Piece p of the
// unit holds unnormalised rows O_p with their reference m_p (log2 units)
// and sum l_p; the output is
//   sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p,  M = max_p m_p,
// then the inverse rotation with the butterflies of fwht128 in the same
// order (strides 1 .. 8 within a thread, 16 .. 64 across its row's lanes).
// (For few units, prefill_merge_rows_kernel below.)
constexpr int MERGE_ROWS = 32, MERGE_THREADS = MERGE_ROWS * 8, MERGE_BATCH = 8;

__global__ void __launch_bounds__(MERGE_THREADS) prefill_merge_kernel(const __grid_constant__ Args a, int nblocks) {
    ptx::wait_prerequisites();  // launched as a programmatic dependent of the attention kernel
    const uint32_t total = a.sched[a.units];
    const int u = static_cast<int>(blockIdx.x);
    const uint32_t pu = a.sched[u], pn = a.sched[u + 1];
    if (total == 0 || pn <= pu) return;  // (a unit without tiles has zero rows, written by the attention kernel)
    const uint32_t C = static_cast<uint32_t>(nblocks) > total ? total : static_cast<uint32_t>(nblocks);
    const int ca = block_of(pu, total, C), cz = block_of(pn - 1, total, C);
    if (ca == cz) return;
    const int tid = static_cast<int>(threadIdx.x), sub = tid & 7;
    const int r = static_cast<int>(blockIdx.y) * MERGE_ROWS + (tid >> 3);
    const Unit x = unit_of(a, u);
    const int G = a.group, rt = r / G, rh = r % G;
    const bool row_ok = rt < x.ntok && rt * G + rh < BM;
    const bool row_out = rt < min(a.tok_per_tile, a.n_new - x.tok0) && rt * G + rh < BM;
    auto piece = [&](int c2) { return a.parts + static_cast<size_t>(part_slot(c2, ca)) * PART_FLOATS; };

    float M = -INFINITY;
    for (int c0 = ca; c0 <= cz; c0 += MERGE_BATCH) {
        float mv[MERGE_BATCH];
#pragma unroll
        for (int k = 0; k < MERGE_BATCH; ++k) mv[k] = c0 + k <= cz ? __ldcg(piece(c0 + k) + BM * D + r) : -INFINITY;
#pragma unroll
        for (int k = 0; k < MERGE_BATCH; ++k) M = fmaxf(M, mv[k]);
    }
    float acc[16], L = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    for (int c0 = ca; c0 <= cz; c0 += MERGE_BATCH) {
        float4 v[MERGE_BATCH][4];
        float mk[MERGE_BATCH], lk[MERGE_BATCH];
#pragma unroll
        for (int k = 0; k < MERGE_BATCH; ++k) {
            const bool in = c0 + k <= cz;
            const float* sp = piece(in ? c0 + k : ca);
            const float4* row = reinterpret_cast<const float4*>(sp + r * D + 16 * sub);
#pragma unroll
            for (int q = 0; q < 4; ++q) v[k][q] = in ? __ldcg(row + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            mk[k] = in ? __ldcg(sp + BM * D + r) : -INFINITY;
            lk[k] = in ? __ldcg(sp + BM * D + BM + r) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < MERGE_BATCH; ++k) {
            const float w = (mk[k] > -INFINITY && M > -INFINITY) ? ptx::ex2(mk[k] - M) : 0.f;
            L = fmaf(lk[k], w, L);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[4 * q] = fmaf(v[k][q].x, w, acc[4 * q]);
                acc[4 * q + 1] = fmaf(v[k][q].y, w, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(v[k][q].z, w, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(v[k][q].w, w, acc[4 * q + 3]);
            }
        }
    }
    const float inv = (row_ok && L > 0.f) ? a.out_scale / L : 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] *= inv;
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((i & h) == 0) {
                const float e0 = acc[i], e1 = acc[i + h];
                acc[i] = e0 + e1;
                acc[i + h] = e0 - e1;
            }
    // (every lane of the warp takes part: the four rows of a warp are all
    // computed, padding rows included, and only the stores are skipped)
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
        const bool upper = (sub & m) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, acc[i], m);
            acc[i] = upper ? o - acc[i] : acc[i] + o;
        }
    }
    if (row_out) {
        const float inv_sqrt_d = 0.08838834764831845f;
        float* dst = a.out + ((static_cast<size_t>(x.b) * a.n_new + x.tok0 + rt) * a.hq + x.kv * G + rh) * D;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = 16 * sub + 4 * q;
            float4 v;
            v.x = flip_sign(acc[4 * q] * inv_sqrt_d, (a.signs[c >> 5] >> (c & 31)) & 1u);
            v.y = flip_sign(acc[4 * q + 1] * inv_sqrt_d, (a.signs[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u);
            v.z = flip_sign(acc[4 * q + 2] * inv_sqrt_d, (a.signs[(c + 2) >> 5] >> ((c + 2) & 31)) & 1u);
            v.w = flip_sign(acc[4 * q + 3] * inv_sqrt_d, (a.signs[(c + 3) >> 5] >> ((c + 3) & 31)) & 1u);
            *reinterpret_cast<float4*>(dst + c) = v;
        }
    }
}

// The same merge for calls with few units, whose pieces are many (three or
// more per unit): block (u, y) takes rows [8 y, 8 y + 8) of unit u, one warp
// per row, four channels a lane.  Piece p of the unit
// holds unnormalised rows O_p with their reference m_p (log2 units) and sum
// l_p; the output is
//   sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p,  M = max_p m_p,
// then the inverse rotation with the butterflies of fwht128 in the same
// order (strides 1 and 2 within a lane, 4 .. 64 across the row's lanes).
// The pieces' (m, l) come in one lane-parallel round trip, their rows
// RMERGE_BATCH at a time.
constexpr int RMERGE_ROWS = 8, RMERGE_THREADS = RMERGE_ROWS * 32, RMERGE_BATCH = 16;
constexpr long long RMERGE_MAX_UNITS = 48;  // at least three pieces a unit on 148 SMs

__global__ void __launch_bounds__(RMERGE_THREADS)
    prefill_merge_rows_kernel(const __grid_constant__ Args a, int nblocks) {
    ptx::wait_prerequisites();  // launched as a programmatic dependent of the attention kernel
    const uint32_t total = a.sched[a.units];
    const int u = static_cast<int>(blockIdx.x);
    const uint32_t pu = a.sched[u], pn = a.sched[u + 1];
    if (total == 0 || pn <= pu) return;  // (a unit without tiles has zero rows, written by the attention kernel)
    const uint32_t C = static_cast<uint32_t>(nblocks) > total ? total : static_cast<uint32_t>(nblocks);
    const int ca = block_of(pu, total, C), cz = block_of(pn - 1, total, C);
    if (ca == cz) return;
    const int lane = static_cast<int>(threadIdx.x) & 31;
    const int r = static_cast<int>(blockIdx.y) * RMERGE_ROWS + (static_cast<int>(threadIdx.x) >> 5);
    const Unit x = unit_of(a, u);
    const int G = a.group, rt = r / G, rh = r % G;
    const bool row_ok = rt < x.ntok && rt * G + rh < BM;
    const bool row_out = rt < min(a.tok_per_tile, a.n_new - x.tok0) && rt * G + rh < BM;
    auto piece = [&](int c2) { return a.parts + static_cast<size_t>(part_slot(c2, ca)) * PART_FLOATS; };
    const int np = cz - ca + 1;

    // (m, l) of pieces lane, lane + 32, ...: the maximum, then each piece's
    // weight 2^(m - M) kept by the lane that loaded it
    float M = -INFINITY;
    for (int j = lane; j < np; j += 32) M = fmaxf(M, __ldcg(piece(ca + j) + BM * D + r));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < np; j0 += 32) {
        float w = 0.f;  // the weight of piece j0 + lane
        if (j0 + lane < np) {
            const float* sp = piece(ca + j0 + lane);
            const float mk = __ldcg(sp + BM * D + r), lk = __ldcg(sp + BM * D + BM + r);
            w = (mk > -INFINITY && M > -INFINITY) ? ptx::ex2(mk - M) : 0.f;
            L = fmaf(lk, w, L);
        }
        const int nj = min(32, np - j0);
        for (int b = 0; b < nj; b += RMERGE_BATCH) {
            float4 v[RMERGE_BATCH];
#pragma unroll
            for (int k = 0; k < RMERGE_BATCH; ++k)
                v[k] = b + k < nj ? __ldcg(reinterpret_cast<const float4*>(piece(ca + j0 + b + k) + r * D) + lane)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < RMERGE_BATCH; ++k) {
                const float wk = __shfl_sync(0xffffffffu, w, (b + k) & 31);
                if (b + k < nj) {
                    acc.x = fmaf(v[k].x, wk, acc.x);
                    acc.y = fmaf(v[k].y, wk, acc.y);
                    acc.z = fmaf(v[k].z, wk, acc.z);
                    acc.w = fmaf(v[k].w, wk, acc.w);
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    const float inv = (row_ok && L > 0.f) ? a.out_scale / L : 0.f;
    float e[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
    // strides 1 and 2 within the lane, then 4 .. 64 across lanes (bits 0 .. 4
    // of the lane); every lane of the warp takes part (one row per warp)
#pragma unroll
    for (int h = 1; h < 4; h <<= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if ((i & h) == 0) {
                const float e0 = e[i], e1 = e[i + h];
                e[i] = e0 + e1;
                e[i + h] = e0 - e1;
            }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, e[i], m);
            e[i] = upper ? o - e[i] : e[i] + o;
        }
    }
    if (row_out) {
        const float inv_sqrt_d = 0.08838834764831845f;
        float* dst = a.out + ((static_cast<size_t>(x.b) * a.n_new + x.tok0 + rt) * a.hq + x.kv * G + rh) * D;
        const int c = 4 * lane;
        float4 v;
        v.x = flip_sign(e[0] * inv_sqrt_d, (a.signs[c >> 5] >> (c & 31)) & 1u);
        v.y = flip_sign(e[1] * inv_sqrt_d, (a.signs[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u);
        v.z = flip_sign(e[2] * inv_sqrt_d, (a.signs[(c + 2) >> 5] >> ((c + 2) & 31)) & 1u);
        v.w = flip_sign(e[3] * inv_sqrt_d, (a.signs[(c + 3) >> 5] >> ((c + 3) & 31)) & 1u);
        *reinterpret_cast<float4*>(dst + c) = v;
    }
}

// A launch that may start before the previous kernel on the stream finishes
// (programmatic stream serialisation): the kernel waits for it with
// griddepcontrol.wait where it first needs that kernel's results.
template <typename... P, typename... T>
static cudaError_t launch_dependent(void (*kernel)(P...), dim3 grid, dim3 block, uint32_t smem_bytes, cudaStream_t s,
                                    T&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<T&&>(args)...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int KB, int VB>
static cudaError_t launch_typed(const Args& a, dim3 grid, cudaStream_t s) {
    constexpr uint32_t bytes = sm_alloc(KB, VB);
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<KB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(bytes));
    if (e != cudaSuccess) return e;
    return launch_dependent(prefill_kernel<KB, VB>, grid, dim3(NTHREADS), bytes, s, a);
}

template <int KB>
static cudaError_t launch_k(int vb, const Args& a, dim3 grid, cudaStream_t s) {
    switch (vb) {
        case 2: return launch_typed<KB, 2>(a, grid, s);
        case 3: return launch_typed<KB, 3>(a, grid, s);
        default: return launch_typed<KB, 4>(a, grid, s);
    }
}

static cudaError_t launch_kb(int kb, int vb, const Args& a, dim3 grid, cudaStream_t s) {
    switch (kb) {
        case 2: return launch_k<2>(vb, a, grid, s);
        case 3: return launch_k<3>(vb, a, grid, s);
        default: return launch_k<4>(vb, a, grid, s);
    }
}

}  // namespace prefill

bool prefill_supported(const tq_params& p) {
    return p.head_dim == 128 && p.k_mode == TQ_MODE_TURBO && p.v_mode == TQ_MODE_TURBO && p.qjl_dims == 0 &&
           p.num_q_heads / p.num_kv_heads <= 16;
}

namespace prefill {

// Work layout of a call: units, whether the blocks share the tile sequence
// (spread) and, if so, how many blocks and the workspace: the schedule
// (units + 1 words), then two partial-output slots per block.
struct Plan {
    long long units;
    int spread, blocks;
    size_t sched_bytes, bytes;
};

static Plan plan(const tq_params& p, int batch, int n_new, int sms) {
    Plan pl{};
    const int tt = BM / (p.num_q_heads / p.num_kv_heads);
    pl.units = static_cast<long long>(batch) * p.num_kv_heads * ((n_new + tt - 1) / tt);
    pl.spread = pl.units <= SCHED_MAX && sms > 0;
    pl.blocks = pl.spread ? sms : static_cast<int>(pl.units);
    if (pl.spread) {
        pl.sched_bytes = (static_cast<size_t>(pl.units + 1) * 4 + 255) / 256 * 256;
        pl.bytes = pl.sched_bytes + static_cast<size_t>(2 * pl.blocks) * PART_FLOATS * sizeof(float);
    }
    return pl;
}

}  // namespace prefill
}  // namespace tq

extern "C" tq_status tq_prefill_workspace_bytes(const tq_params* params, int32_t batch, int32_t n_new,
                                                size_t* bytes) {
    using namespace tq;
    tq_status st = validate_params(params);
    if (st != TQ_OK) return st;
    if (!bytes || batch < 1 || n_new < 1) return TQ_ERR_INVALID_ARG;
    if (!prefill_supported(*params)) return TQ_ERR_UNSUPPORTED;
    const int sms = num_sms_current();
    if (sms <= 0) return TQ_ERR_CUDA;
    *bytes = prefill::plan(*params, batch, n_new, sms).bytes;
    return TQ_OK;
}

extern "C" tq_status tq_prefill_attention(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                          const void* k_new, const void* v_new, tq_dtype kv_dtype, const void* d_q,
                                          tq_dtype q_dtype, int32_t n_new, const int32_t* d_positions,
                                          const tq_cache* cache, float* d_out, void* d_workspace,
                                          size_t workspace_bytes, uint32_t* d_error, void* stream) {
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
    const int sms = num_sms_current();
    if (sms <= 0) return TQ_ERR_CUDA;
    if (prefill::wide_klut(p.k_bits)) {
        // the 4-bit key table's lookups carry its shared-window address
        int reserved = 0, dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
            return TQ_ERR_CUDA;
        if (static_cast<uint32_t>(reserved) != prefill::SMEM_WINDOW) return TQ_ERR_UNSUPPORTED;
    }
    prefill::Plan pl = prefill::plan(p, cache->batch, n_new, sms);
    if (pl.spread && pl.units * ((cache->capacity + prefill::BK - 1) / prefill::BK) >= (1LL << 31)) {
        // the shared tile sequence is counted in 32 bits: a cache long enough
        // to overflow it takes whole units per block instead
        pl.spread = 0;
        pl.blocks = static_cast<int>(pl.units);
        pl.bytes = 0;
    }
    if (pl.bytes > 0) {
        if (!d_workspace) return TQ_ERR_INVALID_ARG;
        if (workspace_bytes < pl.bytes) return TQ_ERR_CAPACITY;
        if (!aligned16(d_workspace)) return TQ_ERR_ALIGNMENT;
    }
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
    a.staged_norms = (cache->capacity % 8) == 0;
    const double ak = kcb->fp16_scale > 0.0 ? kcb->fp16_scale : std::sqrt(128.0);
    const double av = vcb->fp16_scale > 0.0 ? vcb->fp16_scale : std::sqrt(128.0);
    const float sm = p.sm_scale > 0.0f ? p.sm_scale : 1.0f / std::sqrt(128.0f);
    a.score_scale = static_cast<float>(sm * 1.4426950408889634 / ak);
    a.out_scale = static_cast<float>(1.0 / (av * prefill::VFOLD));
    for (int j = 0; j < 16; ++j) {
        const __half hk = __float2half_rn(j < (1 << p.k_bits) ? static_cast<float>(kcb->centroids[j] * ak) : 0.f);
        const __half hv =
            __float2half_rn(j < (1 << p.v_bits) ? static_cast<float>(vcb->centroids[j] * av * prefill::VFOLD) : 0.f);
        a.kcent[j] = __half_as_ushort(hk);
        a.vcent[j] = __half_as_ushort(hv);
    }
    uint32_t words[8];
    rotation_sign_bits(p.seed, 128, words);
    for (int i = 0; i < 4; ++i) a.signs[i] = words[i];
    a.qtiles = (n_new + a.tok_per_tile - 1) / a.tok_per_tile;
    a.units = static_cast<int>(pl.units);
    a.spread = pl.spread;
    a.sched = pl.spread ? static_cast<uint32_t*>(d_workspace) : nullptr;
    a.parts = pl.spread ? reinterpret_cast<float*>(static_cast<char*>(d_workspace) + pl.sched_bytes) : nullptr;
    const dim3 grid(static_cast<unsigned>(pl.blocks));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = prefill::launch_kb(p.k_bits, p.v_bits, a, grid, s);
    if (e == cudaSuccess && pl.spread) {
        // the rows of the units cut between blocks
        // (with few units each is cut into many pieces: a warp per row loads
        // them with more parallelism; with many, pieces are few and the
        // smaller grid of eight threads a row costs less)
        if (pl.units <= prefill::RMERGE_MAX_UNITS) {
            const dim3 mgrid(static_cast<unsigned>(pl.units), prefill::BM / prefill::RMERGE_ROWS);
            e = prefill::launch_dependent(prefill::prefill_merge_rows_kernel, mgrid, dim3(prefill::RMERGE_THREADS), 0u,
                                          s, a, pl.blocks);
        } else {
            const dim3 mgrid(static_cast<unsigned>(pl.units), prefill::BM / prefill::MERGE_ROWS);
            e = prefill::launch_dependent(prefill::prefill_merge_kernel, mgrid, dim3(prefill::MERGE_THREADS), 0u, s, a,
                                          pl.blocks);
        }
    }
    return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
