// Decode attention from the compressed cache on the tensor cores (sm_100a),
// head dimension 128, GQA groups of up to 16: TURBO keys (optionally with the
// QJL sketch) or int8 keys, TURBO values or (beside int8 keys) int8 values;
// contiguous or paged (block-table) caches.
//
// Pages (by title):
//   [google]  "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！",
//             sections "再看速度" and "第二步：QJL —— 1 bit 清理殘差"
//   [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命", sections "Sparse V：速度加成",
//             "三个反直觉的关键发现" (int8 boundary layers, int8 keys with 2-bit
//             values) and "二、inferrs：TurboQuant 轻量推理服务器" (PagedAttention)
//   [tqai]    "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术", section
//             "TurboQuant的核心创新"
//
// What is computed is the same as decode_split_kernel in decode.cu:
//   s_i = sm_scale ||k_i|| (<q~, c[code_i]> + gamma_i sqrt(pi/2)/m <S q~, 2z_i - 1>),
//   softmax over the sequence, acc = sum_i p_i ||v_i|| c[code_i] in the rotated
//   domain, and one inverse rotation of acc / sum_i p_i.  An int8 side uses
//   its scale for the norm and its bytes for the centroids, in the original
//   domain (unrotated query for int8 keys; no inverse rotation for int8 values).
//
// How (one persistent thread block per SM):
//  * Work items are (sequence, kv head, token split).  A producer thread takes
//    items (the block's first one statically, the rest from a global atomic
//    counter, so ragged batches balance; splits past a sequence's end are
//    skipped).  For each item it writes a header (range, length, flags) into
//    the next of two query slots and bulk-copies the item's queries behind it
//    (plus, in append mode, the step's new key and value rows), then streams
//    the packed K and V codes, norms and QJL words of 352-token chunks into a
//    ring of shared-memory stages with 1-D bulk async copies (TMA engine, no
//    multicast), completion tracked by mbarriers.  The block's first chunk and
//    queries are requested before the sequence lengths are read.
//  * Eleven consumer warps each take two 16-token tiles of every chunk (tiles
//    CW apart, so a short last chunk spreads over many warps); each warp waits
//    for a stage on its own, with no block barrier per chunk.
//  * The dequantised tiles of a GQA group form real dense products, so both
//    contractions run on the tensor cores with warp-level m16n8k16 fp16 MMA
//    (fp32 accumulate):  S^T[16 tok x 8 heads] = K~[16 x 128] Q~^T and
//    O^T[128 x 8 heads] += V~^T[128 x 16 tok] P^T.  The query enters as two
//    fp16 terms (hi + lo), so the scores keep about 22 bits of it.  The A
//    operands are built in registers straight from the codes through a
//    per-lane replicated shared-memory table: one byte of 4-bit key codes
//    gives a pair of fp16 centroids, one byte of 2-bit value codes (two
//    tokens, two channels) gives two pairs.
//    Since sum_c q~_c c[code_c] does not depend on the order of c, channels are
//    assigned to fragment slots so that each lane's 16-byte load of a key row
//    feeds its fragments directly (the query uses the same order); tokens of a
//    tile are permuted the same way on both sides (tau) so that neither the
//    key rows nor the value words a warp reads have bank conflicts.
//  * The score fragment becomes the second MMA's operand through one movmatrix
//    transpose per 8x8 block.  The softmax rescales lazily: the running max
//    used for exp2 only moves (with a warp-wide reduction) when a score exceeds
//    it by more than 2^8, decided by one warp vote per chunk.
//  * Split results are merged by the last block to finish a (sequence, kv
//    head), found with one acquire-release atomic per split (no spin-wait);
//    it also applies the inverse rotation and writes the output.
//  Every wait on an mbarrier is bounded (about a second); a wait that runs out
//  sets TQ_DEVERR_TIMEOUT and later waits are skipped; the consumer warps take
//  the same abort decision at the item boundaries (a barrier with an OR
//  reduction), and the block leaves after draining its copies.

#pragma once

#include <cuda_runtime.h>

#include <cmath>

#include "device_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace tq {
namespace mmadec {

constexpr int D = 128;
constexpr int CW = 11;                       // consumer warps (3 warps per scheduler with the producer)
constexpr int TPW = 2;                       // 16-token tiles per warp and chunk
constexpr int NUM_THREADS = (CW + 1) * 32;   // + one producer warp
constexpr int NUM_CONSUMERS = CW * 32;
constexpr int CHUNK = CW * TPW * 16;         // tokens per stage
constexpr uint32_t LUT_BYTES = 65536;        // 256 entries x 256 B
// Shared-window address of the dynamic shared memory (the per-block reserved
// shared memory precedes it); the host checks it before choosing this kernel,
// and table lookups carry it as an immediate offset.
constexpr uint32_t WINDOW = 1024;
constexpr uint32_t QHDR = 32;                 // item header at the front of a query slot
// The warps' partials are combined this many query heads at a time, so the
// combine buffer stays at 22.5 KB for any GQA group (8 or 16 heads would
// otherwise crowd out the second stage).
constexpr int MERGE_HEADS = 4;
// A warp's partial of one head in the combine buffer: eight 16-channel blocks
// of 20 floats (4 of padding), so the eight lane groups g writing channels
// 16 g + 2 i at once hit eight distinct banks (a 128-float row would put every
// other g on the same bank); blocks stay 16-byte aligned for float4 reads.
constexpr int MBLK = 20;
constexpr int MSTRIDE = 8 * MBLK;
__device__ __forceinline__ int mslot(int c) { return (c >> 4) * MBLK + (c & 15); }
// Row strides (halves) of the fp16 query and sketch buffers: 2 words past a
// multiple of 32 banks, so the 8-byte fragment loads of a half-warp (lane
// groups g = 0..3 at rows g, columns 16 t) hit 32 distinct banks.
constexpr int QH_STRIDE = D + 4;
constexpr int SQ_STRIDE = 64 + 4;
// the appended token's patch area: packed key row (up to 128 B: int8 keys),
// packed value row, key norm, value norm, gamma, sketch words, then the
// encoders' scratch (code bytes of each side, the key residual)
constexpr uint32_t AP_K = 0, AP_V = 128, AP_KN = 256, AP_VN = 258, AP_GAM = 260, AP_Z = 264, AP_KC = 288,
                   AP_VC = 416, AP_R = 544;
constexpr uint32_t APP_BYTES = AP_R + 4 * D;
// a side in int8 mode (one byte per channel, fp16 scale in the norm slot):
// the kernel's KB / VB template parameters take this value.  Int8 values come
// only with int8 keys (an all-int8 layer), which need no centroid tables.
constexpr int INT8_BITS = 8;
__host__ __device__ constexpr bool uses_tables(int kb, int vb) { return !(kb == INT8_BITS && vb == INT8_BITS); }
constexpr long long WAIT_LIMIT = 2000000000ll;  // clock cycles (~1 s)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LAZY = 8.0f;                 // log2 headroom before the running max moves
constexpr float VRANGE = 64.0f;              // bound on ||v|| * vscale

// item header flags (query slot): EMPTY / END / APPEND / SKIP (no work: only the
// drain); bits DRAIN_SHIFT and up count the stages the consumers release unread
// after the item's chunks (speculative stages past the sequence's end)
constexpr int F_EMPTY = 4, F_END = 8, F_APPEND = 16, F_SKIP = 64, DRAIN_SHIFT = 8;
// global counters after the per-(sequence, kv head) split counters
constexpr int C_ITEM = 0, C_DONE = 1;

struct Args {
    const uint8_t* k_codes;
    const uint8_t* v_codes;
    const uint16_t* k_norms;
    const uint16_t* v_norms;
    const uint8_t* k_qjl;
    const uint16_t* k_gamma;
    const float* sketch;
    const void* q;
    const int32_t* seq_lens;
    float2* ws_ml;
    float* ws_acc;
    uint32_t* counters;  // [units] split counters, then [2] global counters
    float* out;
    uint32_t* err;
    int q_dtype, q_bytes, batch, hq, hkv, group, capacity, n_split, split_len, max_len, n_items, units, stages, m;
    float sm_scale_log2;  // sm_scale * log2(e)
    float tau;
    uint32_t* skip_mask;  // Sparse V: [batch][hq][mask_words] bits of dropped positions, or null
    int mask_words;
    float inv_alpha_k, inv_alpha_v;  // 1 / (centroid scale applied before fp16 rounding)
    int staged_norms;     // capacity % 8 == 0: norms and QJL words ride in the stages
    uint32_t signs[4];
    uint16_t kcent[16];  // fp16 bits of alpha_k * key centroid
    uint16_t vcent[16];  // fp16 bits of alpha_v * value centroid
    // append mode: one new token per sequence, written at position seq_len - 1
    int append, new_dtype, new_bytes;
    int early;           // TQ_PARAM_PREFETCH_EARLY: the first chunk may be read before the previous kernel ends
    const void* k_new;   // [batch][1][Hkv][d]
    const void* v_new;
    // paged cache (table non-null): token t of (sequence b, kv head h) is row
    // (table[b * max_blocks + t / block_size] * hkv + h) * block_size + t % block_size;
    // `capacity` is then max_blocks * block_size
    const int32_t* table;
    int max_blocks, block_size, num_blocks;
    float kbound[8];     // positive decision boundaries, ascending (unused ones +inf)
    float vbound[8];
    float kc32[16];      // fp32 key centroids (QJL residual)
};

// Shared-memory map (byte offsets from the dynamic base).  A stage is
// [header | K codes | V codes | K norms | V norms | QJL words | gammas].
struct Layout {
    uint32_t ring, stage_bytes, k_off, v_off, kn_off, vn_off, z_off, gam_off;
    uint32_t qslot, qrows, qring, qh, qlo, sq, app, fac, merge, ml, bars, flags, total;
};

__host__ __device__ inline uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }

// g: query heads per kv head; q_bytes, new_bytes: element sizes of the
// queries and of the appended rows (0: no append); n_split: splits per
// (sequence, kv head).
__host__ __device__ inline Layout layout(int kb, int vb, int nt, int stages, int m, int g, int q_bytes, int new_bytes,
                                         int n_split) {
    Layout L{};
    L.ring = uses_tables(kb, vb) ? LUT_BYTES : 0;
    L.k_off = 16;
    L.v_off = L.k_off + CHUNK * 16 * kb;
    L.kn_off = L.v_off + CHUNK * 16 * vb;
    L.vn_off = L.kn_off + CHUNK * 2;
    L.z_off = L.vn_off + CHUNK * 2;
    L.gam_off = L.z_off + CHUNK * (m / 8);
    L.stage_bytes = L.gam_off + (m > 0 ? CHUNK * 2 : 0);
    // query slot: header, the item's g query rows, the appended key and value rows
    L.qrows = QHDR + align16(g * D * q_bytes);
    L.qslot = align16(L.qrows + 2 * D * new_bytes);
    L.qring = L.ring + stages * L.stage_bytes;        // 2 query slots
    L.qh = L.qring + 2 * L.qslot;                      // fp16 [8 nt][QH_STRIDE], rounded q~
    L.qlo = L.qh + 8 * nt * QH_STRIDE * 2;             // fp16 [8 nt][QH_STRIDE], q~ minus the rounded part
    L.sq = L.qlo + 8 * nt * QH_STRIDE * 2;             // fp16 [8 nt][SQ_STRIDE]
    L.app = align16(L.sq + 8 * nt * SQ_STRIDE * 2);    // appended token: packed rows, norms, scratch
    L.fac = L.app + APP_BYTES;                         // float F1[16], F2[16]
    L.merge = L.fac + 32 * 4;
    // merge area, reused: per-warp partials of up to MERGE_HEADS heads at a
    // time [CW][MERGE_HEADS][MSTRIDE]; the final merge's [g][128] outputs and
    // [CW][n_split] weights; the prologue's [8 nt][128] sketch staging; the
    // table build's 768 compact words
    uint32_t merge = CW * (g < MERGE_HEADS ? g : MERGE_HEADS) * MSTRIDE * 4;
    const uint32_t fin = (g * D + CW * n_split) * 4;
    if (fin > merge) merge = fin;
    if (8u * nt * D * 4 > merge) merge = 8 * nt * D * 4;
    if (768u * 4 > merge) merge = 768 * 4;
    L.ml = L.merge + align16(merge);                   // float2 [CW][16]
    L.bars = L.ml + CW * 16 * 8;                       // u64 full[8], empty[8], qfull[2], qempty[2], q0
    L.flags = L.bars + 21 * 8;                         // int abort, last
    L.total = L.flags + 16;
    return L;
}

// Physical token (within a 16-token tile) of logical MMA row r: even rows
// 2i -> i, odd rows 2i+1 -> 4 + (i ^ 1), plus 8 for rows 8..15.  The value
// words a lane reads (rows 2t, 2t+1, 2t+8, 2t+9: tokens t, 4 + (t ^ 1), 8 + t,
// 12 + (t ^ 1)) fall in four distinct bank groups, and the two key rows a
// quarter-warp reads (rows 2q, 2q+1) lie an odd number of 64-byte rows apart,
// so neither read has bank conflicts.
__device__ __forceinline__ int tau_row(int r) {
    const int i = (r & 7) >> 1;
    return (r & 8) + ((r & 1) ? 4 + (i ^ 1) : i);
}

struct Item {
    int unit, split, b, kv, s0, s1, len;
    bool bad;  // seq_len out of range: the sequence is treated as empty
};

// Splits of a unit that hold tokens (at least 1, so an empty sequence still
// gets its zero output): the merge waits for exactly these; the others are
// skipped without any work.
__device__ __forceinline__ int live_splits(const Args& a, int len) {
    const int n = (len + a.split_len - 1) / a.split_len;
    return n > 1 ? n : 1;
}

__device__ __forceinline__ Item item_of(const Args& a, int item) {
    Item it;
    it.unit = item / a.n_split;
    it.split = item % a.n_split;
    it.b = it.unit / a.hkv;
    it.kv = it.unit % a.hkv;
    int len = a.seq_lens[it.b];
    it.bad = len < 1 || len > a.capacity || len > a.max_len;
    if (it.bad) len = 0;
    it.s0 = it.split * a.split_len;
    it.s1 = min(len, it.s0 + a.split_len);
    it.len = len;
    return it;
}

// ------------------------------------------------------------------ producer
template <int KB, int VB, bool QJL>
__device__ void producer(const Args& a, uint8_t* smem, const Layout& L) {
    const uint32_t base = ptx::smem_addr(smem);
    const uint32_t full0 = base + L.bars, empty0 = full0 + 64, qfull0 = full0 + 128, qempty0 = full0 + 144;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flags);
    constexpr int VBK = 16 * KB, VBV = 16 * VB;
    const int zb = QJL ? a.m / 8 : 0;
    const int G = a.group;
    int seq = 0, qseq = 0;
    bool ok = true;
    auto fail = [&]() {
        if (!*abort_flag && a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
        *abort_flag = 1;
        ok = false;
    };
    // claim a free stage slot (bounded wait); false on abort
    auto claim = [&](uint32_t& full, uint8_t*& st) -> bool {
        const int slot = seq % a.stages, use = seq / a.stages;
        if (use > 0 && !ptx::mbar_wait_bounded_sleep(empty0 + 8 * slot, (use - 1) & 1, WAIT_LIMIT, 100)) {
            fail();
            return false;
        }
        // Every block asks for its first stage at the same moment; the other
        // stages follow once it has landed, so first bytes do not queue behind
        // the whole grid's prefetch.  (With the early prefetch the blocks start
        // at staggered times, while the previous kernel drains: no such wait.)
        if (seq == 1 && !a.early && !ptx::mbar_wait_bounded(full0, 0, WAIT_LIMIT)) {
            fail();
            return false;
        }
        if (*abort_flag) {
            ok = false;
            return false;
        }
        full = full0 + 8 * slot;
        st = smem + L.ring + slot * L.stage_bytes;
        return true;
    };
    // Every item starts with a header in the next query slot (the queries and,
    // for a sequence's last split in append mode, the new key and value rows
    // follow it), so consumers can prepare the item while its chunks fly.
    // Empty items take a query slot but no stage.
    auto claim_q = [&](uint8_t*& slot, uint32_t& qfull) -> bool {
        const int qs = qseq & 1;
        if (qseq >= 2 && !ptx::mbar_wait_bounded_sleep(qempty0 + 8 * qs, ((qseq - 2) >> 1) & 1, WAIT_LIMIT, 100)) {
            fail();
            return false;
        }
        if (*abort_flag) {
            ok = false;
            return false;
        }
        slot = smem + L.qring + qs * L.qslot;
        qfull = qfull0 + 8 * qs;
        ++qseq;
        return true;
    };
    // issue the copies of chunk [t0, t0 + n) of a unit into the next stage;
    // `needed`: every token of the range lies below the sequence's length
    auto issue_chunk = [&](int unit, int t0, int n, bool needed) -> bool {
        uint32_t full;
        uint8_t* st;
        if (!claim(full, st)) return false;
        const uint32_t dst = ptx::smem_addr(st);
        const size_t row = static_cast<size_t>(unit) * a.capacity + t0;
        if (a.table) {
            // paged: one copy per block and array.  Block sizes are multiples of
            // 16 and t0 a multiple of 8, so every piece but the chunk's last
            // covers a multiple of 8 tokens, and rounding the last up to 8 stays
            // inside its block (norms then stay 16-byte sized).  A block outside
            // the pool is not read.
            // The chunk's table entries (at most MAXB: blocks hold >= 16
            // tokens) are loaded together, so their latencies overlap.
            constexpr int MAXB = CHUNK / 16 + 1;
            const int b = unit / a.hkv, kv = unit % a.hkv, bs = a.block_size;
            const int end = t0 + ((n + 7) & ~7);
            const int j0 = t0 / bs, nb = (end - 1) / bs - j0 + 1;
            const int32_t* trow = a.table + static_cast<size_t>(b) * a.max_blocks + j0;
            int blk[MAXB];
#pragma unroll
            for (int j = 0; j < MAXB; ++j) blk[j] = j < nb ? __ldg(trow + j) : -1;
            const uint32_t per = VBK + VBV + 4 + (QJL ? zb + 2 : 0);
            uint32_t bytes = 0;
            bool bad = false;
            // (the loops below stay rolled: unrolled, their copies bloat the
            // kernel's code and slow every configuration)
#pragma unroll 1
            for (int j = 0; j < nb; ++j) {
                const int ts = max(t0, (j0 + j) * bs), te = min(end, (j0 + j + 1) * bs);
                if (blk[j] >= 0 && blk[j] < a.num_blocks) bytes += (te - ts) * per;
                else bad = true;
            }
            if (bad && needed && a.err) atomicOr(a.err, TQ_DEVERR_PAGE);
            ptx::mbar_arrive_expect_tx(full, bytes);
#pragma unroll 1
            for (int j = 0; j < nb; ++j) {
                if (blk[j] >= 0 && blk[j] < a.num_blocks) {
                    const int ts = max(t0, (j0 + j) * bs), cnt = min(end, (j0 + j + 1) * bs) - ts;
                    const size_t r = (static_cast<size_t>(blk[j]) * a.hkv + kv) * bs + ts % bs;
                    const uint32_t o = ts - t0;
                    ptx::bulk_copy_g2s(dst + L.k_off + o * VBK, a.k_codes + r * VBK, cnt * VBK, full);
                    ptx::bulk_copy_g2s(dst + L.v_off + o * VBV, a.v_codes + r * VBV, cnt * VBV, full);
                    ptx::bulk_copy_g2s(dst + L.kn_off + o * 2, a.k_norms + r, cnt * 2, full);
                    ptx::bulk_copy_g2s(dst + L.vn_off + o * 2, a.v_norms + r, cnt * 2, full);
                    if constexpr (QJL) {
                        ptx::bulk_copy_g2s(dst + L.z_off + o * zb, a.k_qjl + r * zb, cnt * zb, full);
                        ptx::bulk_copy_g2s(dst + L.gam_off + o * 2, a.k_gamma + r, cnt * 2, full);
                    }
                }
            }
        } else if (a.staged_norms) {
            // capacity and t0 are multiples of 8, so rounding n up to 8 tokens
            // stays inside the cache and keeps every 2-byte array 16-byte sized
            const int n8 = (n + 7) & ~7;
            ptx::mbar_arrive_expect_tx(full, n8 * (VBK + VBV + 4 + (QJL ? zb + 2 : 0)));
            ptx::bulk_copy_g2s(dst + L.k_off, a.k_codes + row * VBK, n8 * VBK, full);
            ptx::bulk_copy_g2s(dst + L.v_off, a.v_codes + row * VBV, n8 * VBV, full);
            ptx::bulk_copy_g2s(dst + L.kn_off, a.k_norms + row, n8 * 2, full);
            ptx::bulk_copy_g2s(dst + L.vn_off, a.v_norms + row, n8 * 2, full);
            if constexpr (QJL) {
                ptx::bulk_copy_g2s(dst + L.z_off, a.k_qjl + row * zb, n8 * zb, full);
                ptx::bulk_copy_g2s(dst + L.gam_off, a.k_gamma + row, n8 * 2, full);
            }
        } else {
            ptx::mbar_arrive_expect_tx(full, n * (VBK + VBV));
            ptx::bulk_copy_g2s(dst + L.k_off, a.k_codes + row * VBK, n * VBK, full);
            ptx::bulk_copy_g2s(dst + L.v_off, a.v_codes + row * VBV, n * VBV, full);
        }
        ++seq;
        return true;
    };
    const uint32_t qbytes = G * D * a.q_bytes;
    // The block's first item is static: its queries and first chunk (as many
    // tokens as the cache could hold there) are requested before the sequence
    // length is read, so the first bytes arrive a DRAM round trip sooner.  If
    // the item turns out empty, its header tells the consumers to drain that
    // stage; if shorter, they only read its valid part.
    // With TQ_PARAM_PREFETCH_EARLY the first chunk is even requested before
    // the previous kernel on the stream has finished (the caller promises it
    // does not write this cache; in append mode the step's own new token is
    // patched in from its staged rows), so it streams in while the previous
    // layer's blocks drain.  Queries, lengths and everything else wait.
    int i = blockIdx.x;
    bool first = true, q0_issued = false;
    int nspec = 0;  // stages of the first item requested before its length was known
    const bool have_first = i < a.n_items;
    const int unit0 = i / a.n_split, split0 = i % a.n_split;
    const int s00 = split0 * a.split_len;
    // the first item's tokens as far as the cache reaches (a split may start
    // past the cache's end when max_seq_len exceeds the capacity: nothing to
    // fetch speculatively there)
    const int spec_end = min(a.capacity, s00 + a.split_len);
    // The length is read first thing after the wait; bring its line into L2
    // now (L2 is coherent with any write of the previous kernel), so that read
    // does not queue behind the grid's first copies in DRAM.
    if (have_first) ptx::prefetch_l2(a.seq_lens + unit0 / a.hkv);
    // With the early prefetch, as many of the first item's chunks as the
    // stages hold stream in before the previous kernel ends.
    if (have_first && a.early)
        for (int t = s00; t < spec_end && nspec < a.stages && !*abort_flag; t += CHUNK) {
            if (!issue_chunk(unit0, t, min(CHUNK, spec_end - t), false)) break;
            ++nspec;
        }
    ptx::wait_prerequisites();
    if (have_first && !*abort_flag) {
        const int b = unit0 / a.hkv, kv = unit0 % a.hkv;
        const uint32_t q0 = full0 + 160;  // its own barrier: consumers rotate before the header lands
        ptx::mbar_arrive_expect_tx(q0, qbytes);
        ptx::bulk_copy_g2s(ptx::smem_addr(smem + L.qring) + QHDR,
                           static_cast<const uint8_t*>(a.q) + (static_cast<size_t>(b) * a.hq + kv * G) * D * a.q_bytes,
                           qbytes, q0);
        q0_issued = true;
        if (!a.early && s00 < spec_end && issue_chunk(unit0, s00, min(CHUNK, spec_end - s00), false)) nspec = 1;
    }
    while (ok) {
        if (i >= a.n_items) break;
        const Item w = item_of(a, i);
        if (w.bad && a.err && w.split == 0 && w.kv == 0) atomicOr(a.err, TQ_DEVERR_SEQLEN);
        // a dead split holds no token and the merge does not wait for it: skip
        // it, unless it is the block's first item (its queries and speculative
        // chunk already fill query slot 0 and a stage; the header then tells
        // the consumers to release them and do nothing else)
        const bool dead = w.split >= live_splits(a, w.len);
        if (dead && !first) {
            i = static_cast<int>(gridDim.x + atomicAdd(a.counters + a.units + C_ITEM, 1u));
            continue;
        }
        const bool empty = w.s0 >= w.s1;
        const bool app = a.append && !empty && w.s1 == w.len;
        if (first && nspec > 0 && a.table && !empty) {
            // the speculative chunks were fetched before the length was known:
            // report an unmapped block among their valid tokens now
            const int32_t* trow = a.table + static_cast<size_t>(w.b) * a.max_blocks;
            const int e = min(w.s1, w.s0 + nspec * CHUNK);
            for (int t = w.s0; t < e; t += a.block_size - t % a.block_size) {
                const int blk = __ldg(trow + t / a.block_size);
                if (blk < 0 || blk >= a.num_blocks) {
                    if (a.err) atomicOr(a.err, TQ_DEVERR_PAGE);
                    break;
                }
            }
        }
        uint8_t* qslot;
        uint32_t qfull;
        if (!claim_q(qslot, qfull)) break;
        // chunks the consumers take for this item; speculative stages past
        // them are released unread
        const int nchunks = empty ? 0 : (w.s1 - w.s0 + CHUNK - 1) / CHUNK;
        const int ndrain = first && nspec > nchunks ? nspec - nchunks : 0;
        int4* hdr = reinterpret_cast<int4*>(qslot);
        hdr[0] = make_int4(i, w.s0, w.s1, w.len);
        hdr[1] = make_int4((empty ? F_EMPTY : 0) | (app ? F_APPEND : 0) | (dead ? F_SKIP : 0) | (ndrain << DRAIN_SHIFT),
                           w.unit, w.b, w.kv);
        const uint32_t rbytes = D * a.new_bytes;
        const uint32_t extra = app ? 2 * rbytes : 0u;  // append rows
        if (first) {  // queries already requested; add the append rows, then arrive
            if (app) ptx::mbar_expect_tx(qfull, extra);
        } else if (!empty) {
            ptx::mbar_expect_tx(qfull, qbytes + extra);
            ptx::bulk_copy_g2s(ptx::smem_addr(qslot) + QHDR,
                               static_cast<const uint8_t*>(a.q) +
                                   (static_cast<size_t>(w.b) * a.hq + w.kv * G) * D * a.q_bytes,
                               qbytes, qfull);
        }
        if (app) {
            const size_t row = (static_cast<size_t>(w.b) * a.hkv + w.kv) * rbytes;
            const uint32_t rdst = ptx::smem_addr(qslot) + L.qrows;
            ptx::bulk_copy_g2s(rdst, static_cast<const uint8_t*>(a.k_new) + row, rbytes, qfull);
            ptx::bulk_copy_g2s(rdst + rbytes, static_cast<const uint8_t*>(a.v_new) + row, rbytes, qfull);
        }
        ptx::mbar_arrive(qfull);  // header written, every copy of the slot accounted for
        int t0 = w.s0;
        if (first) t0 += nspec * CHUNK;  // the speculative stages hold the first chunks
        for (; t0 < w.s1; t0 += CHUNK)
            if (!issue_chunk(w.unit, t0, min(CHUNK, w.s1 - t0), true)) break;
        first = false;
        if (!ok) break;
        i = static_cast<int>(gridDim.x + atomicAdd(a.counters + a.units + C_ITEM, 1u));
    }
    if (ok) {  // end-of-work sentinel, in the next query slot
        uint8_t* qslot;
        uint32_t qfull;
        if (claim_q(qslot, qfull)) {
            reinterpret_cast<int4*>(qslot)[1] = make_int4(F_END, 0, 0, 0);
            ptx::mbar_arrive_expect_tx(qfull, 0);
        }
    }
    // every copy issued must have landed before the block may exit
    for (int j = max(0, seq - a.stages); j < seq; ++j)
        ptx::mbar_wait_bounded(full0 + 8 * (j % a.stages), (j / a.stages) & 1, WAIT_LIMIT);
    for (int j = max(0, qseq - 2); j < qseq; ++j) ptx::mbar_wait_bounded(qfull0 + 8 * (j & 1), (j >> 1) & 1, WAIT_LIMIT);
    if (q0_issued) ptx::mbar_wait_bounded(full0 + 160, 0, WAIT_LIMIT);
}

// ----------------------------------------------------------------- consumers
// Key fragment register for channel pair (4j + 2h, 4j + 2h + 1) of the lane's
// 32-channel segment (KB words, little-endian bitstream): table address.
template <int KB>
__device__ __forceinline__ uint32_t key_lut_addr(const uint32_t (&seg)[4], int j, int h, uint32_t laneoff) {
    const int bit = KB * (4 * j + 2 * h);
    if constexpr (KB == 4) {
        const uint32_t w = seg[bit >> 5];
        const int byte = (bit & 31) >> 3;
        // byte -> bits 8..15, lane offset (lane*4 < 256) -> bits 0..7
        return __byte_perm(w, laneoff, 0x6504 | (byte << 4));
    } else {
        const int wi = bit >> 5, sh = bit & 31;
        uint32_t v = seg[wi] >> sh;
        if (sh + 2 * KB > 32) v |= seg[wi + 1] << (32 - sh);
        return ((v & ((1u << (2 * KB)) - 1u)) << 8) | laneoff;
    }
}

// Four int8 bytes of one word as two fp16 pairs (bytes 0, 1 and bytes 2, 3),
// exactly: b ^ 0x80 = b + 128 becomes the mantissa of 1024 + (b + 128), and
// subtracting 1152 leaves b.
__device__ __forceinline__ void int8_pairs(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t pl = __byte_perm(u, 0x64646464u, 0x5140);  // channels 0, 1
    const uint32_t ph = __byte_perm(u, 0x64646464u, 0x7362);  // channels 2, 3
    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
    const __half2 l2 = __hsub2(*reinterpret_cast<const __half2*>(&pl), bias);
    const __half2 h2 = __hsub2(*reinterpret_cast<const __half2*>(&ph), bias);
    lo = *reinterpret_cast<const uint32_t*>(&l2);
    hi = *reinterpret_cast<const uint32_t*>(&h2);
}

// Value fragments A[m-tile i][reg] of one 16-token tile for lane group g.
template <int VB>
__device__ __forceinline__ void value_fragments(uint32_t vst, uint32_t base, int g, int t, uint32_t laneoff,
                                                uint32_t (&A)[8][4]) {
    constexpr int VBV = 16 * VB;
    if constexpr (VB == INT8_BITS) {
        // channels 16 g .. 16 g + 15 (16 bytes) of physical tokens t, 4 + (t ^ 1),
        // 8 + t, 12 + (t ^ 1) (logical k = 2t, 2t+1, 2t+8, 2t+9); row g of m-tile
        // i is channel 16 g + 2 i, row g + 8 channel 16 g + 2 i + 1
        const uint4 xa = ptx::lds128(vst + t * VBV + 16 * g);
        const uint4 xb = ptx::lds128(vst + (4 + (t ^ 1)) * VBV + 16 * g);
        const uint4 xc = ptx::lds128(vst + (8 + t) * VBV + 16 * g);
        const uint4 xd = ptx::lds128(vst + (12 + (t ^ 1)) * VBV + 16 * g);
        const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w}, wb[4] = {xb.x, xb.y, xb.z, xb.w};
        const uint32_t wc[4] = {xc.x, xc.y, xc.z, xc.w}, wd[4] = {xd.x, xd.y, xd.z, xd.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int w = i >> 1;
            const uint32_t sel = (i & 1) ? 0x7362u : 0x5140u;  // bytes 2p, 2p + 1 of both words, interleaved
            const uint32_t ab = __byte_perm(wa[w], wb[w], sel);
            const uint32_t cd = __byte_perm(wc[w], wd[w], sel);
            int8_pairs(ab, A[i][0], A[i][1]);
            int8_pairs(cd, A[i][2], A[i][3]);
        }
    } else if constexpr (VB == 2) {
        // word g of physical tokens t, 4 + (t ^ 1), 8 + t, 12 + (t ^ 1)
        // (logical k = 2t, 2t+1, 2t+8, 2t+9)
        const uint32_t w0 = ptx::lds32(vst + t * VBV + 4 * g);
        const uint32_t w1 = ptx::lds32(vst + (4 + (t ^ 1)) * VBV + 4 * g);
        const uint32_t w2 = ptx::lds32(vst + (8 + t) * VBV + 4 * g);
        const uint32_t w3 = ptx::lds32(vst + (12 + (t ^ 1)) * VBV + 4 * g);
        // Nibble n of a word holds channels 16g+2n (bits 0-1) and 16g+2n+1
        // (bits 2-3), i.e. rows g and g+8 of m-tile n.  Interleaving the nibbles
        // of the two tokens gives bytes (token a nibble | token b nibble << 4);
        // each byte indexes the 64-bit table entry {(c[a0], c[b0]), (c[a1], c[b1])}
        // = the row-g and row-(g+8) registers of that m-tile.
        const uint32_t voff = 128u | ((laneoff & 60u) << 1);  // half-warp replica (lane & 15) * 8
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t wa = half ? w2 : w0, wb = half ? w3 : w1;
            const uint32_t even = (wa & 0x0F0F0F0Fu) | ((wb << 4) & 0xF0F0F0F0u);  // nibbles 0, 2, 4, 6
            const uint32_t odd = ((wa >> 4) & 0x0F0F0F0Fu) | (wb & 0xF0F0F0F0u);   // nibbles 1, 3, 5, 7
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint2 re = ptx::lds64_imm<WINDOW>(__byte_perm(even, voff, 0x6504 | (k << 4)));
                const uint2 ro = ptx::lds64_imm<WINDOW>(__byte_perm(odd, voff, 0x6504 | (k << 4)));
                A[2 * k][2 * half] = re.x;
                A[2 * k][2 * half + 1] = re.y;
                A[2 * k + 1][2 * half] = ro.x;
                A[2 * k + 1][2 * half + 1] = ro.y;
            }
        }
    } else {
        // 16 * VB bits per lane group and token (2*VB bytes at byte 2*VB*g),
        // realigned to two words; code pairs read through the value table
        uint32_t seg[4][2];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            const int tok = 4 * k4 + ((k4 & 1) ? (t ^ 1) : t);  // tau of logical k = 2t, 2t+1, 2t+8, 2t+9
            const uint32_t byte_off = 2 * VB * g;
            const uint32_t wbase = byte_off >> 2, wsh = (byte_off & 3) * 8;
            const uint32_t lo = ptx::lds32(vst + tok * VBV + 4 * wbase);
            const uint32_t hi = (4 * wbase + 4 < VBV) ? ptx::lds32(vst + tok * VBV + 4 * wbase + 4) : 0u;
            const uint32_t hi2 = (4 * wbase + 8 < VBV) ? ptx::lds32(vst + tok * VBV + 4 * wbase + 8) : 0u;
            seg[k4][0] = __funnelshift_r(lo, hi, wsh);
            seg[k4][1] = __funnelshift_r(hi, hi2, wsh);
        }
        constexpr uint32_t vm = (1u << VB) - 1u;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                const int bit = VB * (2 * i + f);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t* sx = seg[2 * half];
                    const uint32_t* sy = seg[2 * half + 1];
                    const uint32_t cx = bit >= 32 ? (sx[1] >> (bit - 32)) & vm
                                                  : (bit + VB <= 32 ? (sx[0] >> bit) & vm
                                                                    : __funnelshift_r(sx[0], sx[1], bit) & vm);
                    const uint32_t cy = bit >= 32 ? (sy[1] >> (bit - 32)) & vm
                                                  : (bit + VB <= 32 ? (sy[0] >> bit) & vm
                                                                    : __funnelshift_r(sy[0], sy[1], bit) & vm);
                    A[i][2 * half + f] = ptx::lds32_imm<WINDOW>(((cx | (cy << VB)) << 8) | 128u | laneoff);
                }
            }
    }
}

template <int NT>
struct SoftState {
    float m[NT][2];  // exp2 reference of heads 2t, 2t+1 (uniform over the lane group)
    float l[NT][2];  // this lane's partial sum of exp2(s - m)
    float acc[NT][8][4];
    float vscale;    // power of two keeping p * ||v|| inside fp16 range; 0 = not set

    __device__ void reset() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[nt][i][0] = acc[nt][i][1] = acc[nt][i][2] = acc[nt][i][3] = 0.f;
        }
        vscale = 0.f;
    }
};

template <int KB, int VB, int NT, bool QJL, bool REC>
struct Consumer {
    const Args& a;
    uint8_t* smem;
    const Layout& L;
    int tid, warp, lane, g, t;
    uint32_t base, laneoff, sgn4;

    __device__ Consumer(const Args& a_, uint8_t* s_, const Layout& L_) : a(a_), smem(s_), L(L_) {
        tid = threadIdx.x;
        warp = tid >> 5;
        lane = tid & 31;
        g = lane >> 2;
        t = lane & 3;
        base = ptx::smem_addr(smem);
        laneoff = lane * 4;
        // rotation signs of coordinates 4 lane .. 4 lane + 3 (word lane / 8),
        // read with constant indices: a per-lane index into the parameters
        // would serialise
        const int wsel = lane >> 3;
        const uint32_t sw = wsel == 0 ? a.signs[0] : wsel == 1 ? a.signs[1] : wsel == 2 ? a.signs[2] : a.signs[3];
        sgn4 = (sw >> (4 * (lane & 7))) & 0xFu;
    }

    __device__ bool aborted() const { return *reinterpret_cast<volatile int*>(smem + L.flags) != 0; }

    // Sparse V's record: which positions of a tile the gate dropped from the V
    // sum.  drop[nt][e] is lane (g, t)'s decision for row g (e < 2) or g + 8
    // (e >= 2) and head nt * 8 + 2 t + (e & 1); lane h gathers head h's 16 bits
    // (row r is token tau(r) of the tile) and ORs them into that head's row of
    // the caller's mask (two tiles share a 32-bit word).
    __device__ void record_drops(const Item& w, int tile_start, const bool (&drop)[NT][4]) {
        uint32_t bal[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) bal[nt][e] = __ballot_sync(kFullMask, drop[nt][e]);
        const int h = lane;
        if (h >= a.group || h >= NT * 8) return;
        const int col = h & 7, tt = col >> 1;
        uint32_t lo_b = 0, hi_b = 0;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            if (nt == (h >> 3)) {
                lo_b = (col & 1) ? bal[nt][1] : bal[nt][0];
                hi_b = (col & 1) ? bal[nt][3] : bal[nt][2];
            }
        uint32_t field = 0;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            field |= ((lo_b >> (4 * r + tt)) & 1u) << tau_row(r);
            field |= ((hi_b >> (4 * r + tt)) & 1u) << tau_row(r + 8);
        }
        if (field) {
            uint32_t* row = a.skip_mask + (static_cast<size_t>(w.b) * a.hq + w.kv * a.group + h) * a.mask_words;
            atomicOr(row + (tile_start >> 5), field << (tile_start & 16));
        }
    }
    __device__ void set_abort() {
        if (!aborted() && a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
        *reinterpret_cast<volatile int*>(smem + L.flags) = 1;
    }

    // Rotated queries of the item (fp16 hi + lo pair, scaled to max |q~| = 1) and the scale
    // factors of the scores; false on abort.
    // The appended token of the item's sequence (append mode): warp 0 encodes
    // the new key, warp 1 the new value, from the rows staged beside the
    // queries, exactly as the quantise-append kernel does (norm, rotation,
    // codes, packing, and for keys the QJL sign sketch of the residual).  The
    // result goes to the cache slot and to the patch area, from which the
    // stage holding the token is updated before it is consumed.
    // (codes == nullptr: fill the patch area only, write nothing to the cache)
    template <int BITS, bool SKETCH>
    __device__ void encode_new(const uint8_t* src, uint8_t* codes, uint16_t* norms, const float* bounds, size_t slot,
                               uint8_t* prow, uint16_t* pnorm, uint8_t* cbytes, float* rbuf) {
        if constexpr (BITS == INT8_BITS)
            encode_int8(src, codes, norms, slot, prow, pnorm);
        else
            encode_turbo<BITS, SKETCH>(src, codes, norms, bounds, slot, prow, pnorm, cbytes, rbuf);
    }

    // int8 row (the quantise kernel's arithmetic): fp16 scale = absmax / 127,
    // bytes rint(x / scale) clamped to +-127, one per channel in natural order
    __device__ void encode_int8(const uint8_t* src, uint8_t* codes, uint16_t* norms, size_t slot, uint8_t* prow,
                                uint16_t* pnorm) {
        float x[4];
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] = load_scalar(src, lane * 4 + e, a.new_dtype);
            amax = fmaxf(amax, fabsf(x[e]));
        }
        amax = group_max<32>(amax);
        const __half scale16 = __float2half_rn(__fdiv_rn(amax, 127.0f));
        const float scale = __half2float(scale16);
        const float recip = (scale > 0.0f && scale < INFINITY) ? __frcp_rn(scale) : 0.0f;
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float q = fminf(fmaxf(rintf(__fmul_rn(x[e], recip)), -127.0f), 127.0f);
            word |= (static_cast<uint32_t>(static_cast<int32_t>(q)) & 0xffu) << (8 * e);
        }
        if (codes) reinterpret_cast<uint32_t*>(codes + slot * D)[lane] = word;
        reinterpret_cast<uint32_t*>(prow)[lane] = word;
        if (lane == 0) {
            if (codes) norms[slot] = __half_as_ushort(scale16);
            *pnorm = __half_as_ushort(scale16);
        }
    }

    template <int BITS, bool SKETCH>
    __device__ void encode_turbo(const uint8_t* src, uint8_t* codes, uint16_t* norms, const float* bounds, size_t slot,
                                 uint8_t* prow, uint16_t* pnorm, uint8_t* cbytes, float* rbuf) {
        float x[4];
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] = load_scalar(src, lane * 4 + e, a.new_dtype);
            ss = fmaf(x[e], x[e], ss);
            x[e] = flip_sign(x[e], (sgn4 >> e) & 1u);
        }
        fwht_registers(x);
        fwht_lanes<4, 32>(x, lane);
        ss = group_sum<32>(ss);
        const float n = sqrtf(ss);
        const float inv = n > 0.0f ? 1.0f / (sqrtf(static_cast<float>(D)) * n) : 0.0f;
        uint32_t code[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] *= inv;  // rotated unit-vector coordinate
            code[e] = code_of<BITS>(x[e], bounds);
            cbytes[lane * 4 + e] = static_cast<uint8_t>(code[e]);
        }
        __syncwarp();
        if (lane < 4 * BITS) {  // word `lane` of the LSB-first bitstream
            const int c0 = (32 * lane) / BITS, c1 = (32 * lane + 31) / BITS;
            uint32_t word = 0;
            for (int c = c0; c <= c1; ++c) {
                const int sh = c * BITS - 32 * lane;
                const uint32_t v = cbytes[c];
                word |= sh >= 0 ? (v << sh) : (v >> -sh);
            }
            if (codes) reinterpret_cast<uint32_t*>(codes + slot * (16 * BITS))[lane] = word;
            reinterpret_cast<uint32_t*>(prow)[lane] = word;
        }
        if (lane == 0) {
            const uint16_t n16 = float_to_half_bits(n);
            if (codes) norms[slot] = n16;
            *pnorm = n16;
        }
        if constexpr (SKETCH) {
            float g2 = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float r = x[e] - a.kc32[code[e]];
                g2 = fmaf(r, r, g2);
                rbuf[lane * 4 + e] = r;
            }
            g2 = group_sum<32>(g2);
            __syncwarp();
            float acc0 = 0.f, acc1 = 0.f;
            if (lane < a.m) {
                const float* srow = a.sketch + static_cast<size_t>(lane) * D;
                for (int c = 0; c < D; ++c) acc0 = fmaf(__ldg(srow + c), rbuf[c], acc0);
            }
            if (lane + 32 < a.m) {
                const float* srow = a.sketch + static_cast<size_t>(lane + 32) * D;
                for (int c = 0; c < D; ++c) acc1 = fmaf(__ldg(srow + c), rbuf[c], acc1);
            }
            const uint32_t z0 = __ballot_sync(kFullMask, lane < a.m && acc0 >= 0.f);
            const uint32_t z1 = __ballot_sync(kFullMask, lane + 32 < a.m && acc1 >= 0.f);
            uint8_t* pz = smem + L.app + AP_Z;
            uint32_t* qjl = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.k_qjl) + slot * (a.m / 8));
            if (lane == 0) {
                const uint16_t g16 = float_to_half_bits(sqrtf(g2));
                if (codes) const_cast<uint16_t*>(a.k_gamma)[slot] = g16;
                *reinterpret_cast<uint16_t*>(smem + L.app + AP_GAM) = g16;
                if (codes) qjl[0] = z0;
                reinterpret_cast<uint32_t*>(pz)[0] = z0;
                if (a.m > 32) {
                    if (codes) qjl[1] = z1;
                    reinterpret_cast<uint32_t*>(pz)[1] = z1;
                }
            }
        }
    }

    // Copy the appended token from the patch area into the stage that holds it
    // (chunk-local index p); warps 0 (key side) and 1 (value side).
    __device__ void patch_stage(uint8_t* st, int p) {
        const uint8_t* ap = smem + L.app;
        if (warp == 0) {
            if (lane < 4 * KB)
                reinterpret_cast<uint32_t*>(st + L.k_off + p * (16 * KB))[lane] = reinterpret_cast<const uint32_t*>(ap + AP_K)[lane];
            if (a.staged_norms && lane == 0) {
                reinterpret_cast<uint16_t*>(st + L.kn_off)[p] = *reinterpret_cast<const uint16_t*>(ap + AP_KN);
                if constexpr (QJL) {
                    reinterpret_cast<uint16_t*>(st + L.gam_off)[p] = *reinterpret_cast<const uint16_t*>(ap + AP_GAM);
                    const int zb = a.m / 8;
                    for (int i = 0; i < zb / 4; ++i)
                        reinterpret_cast<uint32_t*>(st + L.z_off + p * zb)[i] = reinterpret_cast<const uint32_t*>(ap + AP_Z)[i];
                }
            }
        } else if (warp == 1) {
            if (lane < 4 * VB)
                reinterpret_cast<uint32_t*>(st + L.v_off + p * (16 * VB))[lane] =
                    reinterpret_cast<const uint32_t*>(ap + AP_V)[lane];
            if (a.staged_norms && lane == 0)
                reinterpret_cast<uint16_t*>(st + L.vn_off)[p] = *reinterpret_cast<const uint16_t*>(ap + AP_VN);
        }
        // the stage is refilled later by the copy engine: order these writes first
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }

    // The item's queries are in query slot `qseq` (already waited for).
    // Rotate the queries in query slot `qseq` into the fp16 fragment buffers
    // and the score factors (no barrier; the prologue's barrier publishes them).
    __device__ void rotate(int qseq) {
        const int G = a.group;
        const uint8_t* qsrc = smem + L.qring + (qseq & 1) * L.qslot + QHDR;
        __half* qh = reinterpret_cast<__half*>(smem + L.qh);
        __half* ql = reinterpret_cast<__half*>(smem + L.qlo);
        __half* sq = reinterpret_cast<__half*>(smem + L.sq);
        float* fac = reinterpret_cast<float*>(smem + L.fac);
        float* merge = reinterpret_cast<float*>(smem + L.merge);
        const float inv_sqrt_d = 0.08838834764831845f;
        for (int h = warp; h < NT * 8; h += CW) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (h < G) {
                load4(qsrc, h * D + lane * 4, a.q_dtype, x);
                if constexpr (KB != INT8_BITS) {  // int8 keys live in the original domain
#pragma unroll
                    for (int e = 0; e < 4; ++e) x[e] = flip_sign(x[e], (sgn4 >> e) & 1u);
                    fwht_registers(x);
                    fwht_lanes<4, 32>(x, lane);
#pragma unroll
                    for (int e = 0; e < 4; ++e) x[e] *= inv_sqrt_d;
                }
            }
            float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
            amax = group_max<32>(amax);
            const float qmax = amax > 0.f ? amax : 1.f;
            const float rq = 1.0f / qmax;  // F1 undoes the scale (to one fp32 ulp)
            // two fp16 terms: the scores keep about 22 bits of q~
            uint32_t hw[2], lw[2];
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const float u0 = x[2 * e2] * rq, u1 = x[2 * e2 + 1] * rq;
                const __half2 hi = __floats2half2_rn(u0, u1);
                const float2 hf = __half22float2(hi);
                const __half2 lo = __floats2half2_rn(u0 - hf.x, u1 - hf.y);
                hw[e2] = *reinterpret_cast<const uint32_t*>(&hi);
                lw[e2] = *reinterpret_cast<const uint32_t*>(&lo);
            }
            *reinterpret_cast<uint2*>(qh + h * QH_STRIDE + lane * 4) = make_uint2(hw[0], hw[1]);
            *reinterpret_cast<uint2*>(ql + h * QH_STRIDE + lane * 4) = make_uint2(lw[0], lw[1]);
            float smax = 1.f;
            if constexpr (QJL) {
                // S q~ for sketch rows lane and lane + 32 (m <= 64); q~ staged in
                // the merge buffer, which is free until the item's end
                float* qf = merge + h * D;
#pragma unroll
                for (int e = 0; e < 4; ++e) qf[lane * 4 + e] = x[e];
                __syncwarp();
                float sv[2] = {0.f, 0.f};
                if (h < G) {
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int r = lane + 32 * rr;
                        if (r < a.m) {
                            const float* srow = a.sketch + static_cast<size_t>(r) * D;
                            float acc = 0.f;
                            for (int c = 0; c < D; ++c) acc = fmaf(__ldg(srow + c), qf[c], acc);
                            sv[rr] = acc;
                        }
                    }
                }
                const float sm = group_max<32>(fmaxf(fabsf(sv[0]), fabsf(sv[1])));
                smax = sm > 0.f ? sm : 1.f;
                sq[h * SQ_STRIDE + lane] = __float2half_rn(sv[0] / smax);
                sq[h * SQ_STRIDE + lane + 32] = __float2half_rn(sv[1] / smax);
            }
            if (lane == 0) {
                fac[h] = h < G ? a.sm_scale_log2 * qmax * a.inv_alpha_k : 0.f;
                fac[16 + h] = (QJL && h < G) ? a.sm_scale_log2 * 1.2533141373155003f / a.m * smax : 0.f;
            }
        }
    }

    // Item start: the queries (rotated here unless `rotated`), the appended
    // token's encoding (append mode), then every warp's query fragments.
    __device__ void prologue(int qseq, bool rotated, const Item& w, bool app, uint32_t (&bq)[NT][8][4],
                             uint32_t (&bz)[NT][4][2], float (&f1)[NT][2], float (&f2)[NT][2]) {
        if (!rotated) rotate(qseq);
        __half* qh = reinterpret_cast<__half*>(smem + L.qh);
        __half* ql = reinterpret_cast<__half*>(smem + L.qlo);
        __half* sq = reinterpret_cast<__half*>(smem + L.sq);
        float* fac = reinterpret_cast<float*>(smem + L.fac);
        if (app && warp < 2) {
            // the new token's cache row; a paged cache whose block is outside
            // the pool gets no write (the token still joins this attention)
            size_t slot = static_cast<size_t>(w.unit) * a.capacity + (w.len - 1);
            bool store = true;
            if (a.table) {
                const int tok = w.len - 1;
                const int blk = __ldg(a.table + static_cast<size_t>(w.b) * a.max_blocks + tok / a.block_size);
                store = blk >= 0 && blk < a.num_blocks;
                slot = store ? (static_cast<size_t>(blk) * a.hkv + w.kv) * a.block_size + tok % a.block_size : 0;
                if (!store && warp == 0 && lane == 0 && a.err) atomicOr(a.err, TQ_DEVERR_PAGE);
            }
            const uint8_t* rows = smem + L.qring + (qseq & 1) * L.qslot + L.qrows;
            uint8_t* ap = smem + L.app;
            if (warp == 0)
                encode_new<KB, QJL>(rows, store ? const_cast<uint8_t*>(a.k_codes) : nullptr,
                                    const_cast<uint16_t*>(a.k_norms), a.kbound, slot, ap + AP_K,
                                    reinterpret_cast<uint16_t*>(ap + AP_KN), ap + AP_KC,
                                    reinterpret_cast<float*>(ap + AP_R));
            else
                encode_new<VB, false>(rows + D * a.new_bytes, store ? const_cast<uint8_t*>(a.v_codes) : nullptr,
                                      const_cast<uint16_t*>(a.v_norms), a.vbound, slot, ap + AP_V,
                                      reinterpret_cast<uint16_t*>(ap + AP_VN), ap + AP_VC,
                                      reinterpret_cast<float*>(ap + AP_R));
        }
        ptx::named_barrier(1, NUM_CONSUMERS);  // every warp is done with the query slot
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const __half* qrow = qh + (nt * 8 + g) * QH_STRIDE + 32 * t;
            const __half* lrow = ql + (nt * 8 + g) * QH_STRIDE + 32 * t;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint2 hv = *reinterpret_cast<const uint2*>(qrow + 4 * j);
                const uint2 lv = *reinterpret_cast<const uint2*>(lrow + 4 * j);
                bq[nt][j][0] = hv.x;
                bq[nt][j][1] = hv.y;
                bq[nt][j][2] = lv.x;
                bq[nt][j][3] = lv.y;
            }
            if constexpr (QJL) {
                const __half* srow = sq + (nt * 8 + g) * SQ_STRIDE + 16 * t;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    bz[nt][j][0] = *reinterpret_cast<const uint32_t*>(srow + 4 * j);
                    bz[nt][j][1] = *reinterpret_cast<const uint32_t*>(srow + 4 * j + 2);
                }
            }
            f1[nt][0] = fac[nt * 8 + 2 * t];
            f1[nt][1] = fac[nt * 8 + 2 * t + 1];
            f2[nt][0] = fac[16 + nt * 8 + 2 * t];
            f2[nt][1] = fac[16 + nt * 8 + 2 * t + 1];
        }
    }

    // One chunk: this warp's TPW tiles.  MASK: the chunk may end before CHUNK
    // tokens.  Each phase handles all of the warp's tiles in one branch-free
    // stretch (the tiles are independent, so their load, lookup and MMA chains
    // interleave); tokens past the item's end are computed on whatever the
    // stage holds (finite table values) and masked afterwards.
    template <bool MASK>
    __device__ void chunk_il(const Item& w, const uint8_t* st, int t0, const uint32_t (&bq)[NT][8][4],
                          const uint32_t (&bz)[NT][4][2], const float (&f1)[NT][2], const float (&f2)[NT][2],
                          SoftState<NT>& S) {
        constexpr int VBK = 16 * KB, VBV = 16 * VB;
        // this warp's tiles are k * CW + warp (k < TPW): a short last chunk
        // spreads over many warps instead of keeping two tiles on a few
        const int lb = 16 * warp;  // first chunk-local token of this warp's first tile
        constexpr int TS = 16 * CW;  // token distance between a warp's tiles
        if (MASK && t0 + lb >= w.s1) return;  // nothing of this warp's tiles is valid
        const uint32_t sbase = ptx::smem_addr(st);
        const int ra = tau_row(g), rb = tau_row(g + 8);
        const int zw = a.m / 16;
        const bool zt = 16 * t < a.m;
        const size_t unit_row = static_cast<size_t>(w.unit) * a.capacity;
        // chunk-local tokens of rows g, g + 8 of each tile, and their validity
        int la[TPW], lbb[TPW];
        bool va[TPW], vb[TPW];
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            la[k] = lb + TS * k + ra;
            lbb[k] = lb + TS * k + rb;
            va[k] = !MASK || t0 + la[k] < w.s1;
            vb[k] = !MASK || t0 + lbb[k] < w.s1;
        }
        // ---- norms (and QJL words and gammas) of every tile
        float kna[TPW], knb[TPW], vn[TPW][2], ga[TPW], gb[TPW];
        uint32_t za[TPW], zb2[TPW];
        if (a.staged_norms) {
            const __half* skn = reinterpret_cast<const __half*>(st + L.kn_off);
            const __half* svn = reinterpret_cast<const __half*>(st + L.vn_off);
#pragma unroll
            for (int k = 0; k < TPW; ++k) {
                kna[k] = __half2float(skn[la[k]]);
                knb[k] = __half2float(skn[lbb[k]]);
                vn[k][0] = va[k] ? __half2float(svn[la[k]]) : 0.f;
                vn[k][1] = vb[k] ? __half2float(svn[lbb[k]]) : 0.f;
                ga[k] = gb[k] = 0.f;
                za[k] = zb2[k] = 0u;
                if constexpr (QJL) {
                    const uint16_t* sz = reinterpret_cast<const uint16_t*>(st + L.z_off);
                    const __half* sg = reinterpret_cast<const __half*>(st + L.gam_off);
                    za[k] = zt ? sz[la[k] * zw + t] : 0u;
                    zb2[k] = zt ? sz[lbb[k] * zw + t] : 0u;
                    ga[k] = __half2float(sg[la[k]]);
                    gb[k] = __half2float(sg[lbb[k]]);
                }
            }
        } else {
#pragma unroll
            for (int k = 0; k < TPW; ++k) {
                const size_t ra_g = unit_row + t0 + la[k], rb_g = unit_row + t0 + lbb[k];
                kna[k] = va[k] ? half_bits_to_float(a.k_norms[ra_g]) : 0.f;
                knb[k] = vb[k] ? half_bits_to_float(a.k_norms[rb_g]) : 0.f;
                vn[k][0] = va[k] ? half_bits_to_float(a.v_norms[ra_g]) : 0.f;
                vn[k][1] = vb[k] ? half_bits_to_float(a.v_norms[rb_g]) : 0.f;
                ga[k] = gb[k] = 0.f;
                za[k] = zb2[k] = 0u;
                if constexpr (QJL) {
                    const uint16_t* zr = reinterpret_cast<const uint16_t*>(a.k_qjl);
                    za[k] = (va[k] && zt) ? zr[ra_g * zw + t] : 0u;
                    zb2[k] = (vb[k] && zt) ? zr[rb_g * zw + t] : 0u;
                    ga[k] = va[k] ? half_bits_to_float(a.k_gamma[ra_g]) : 0.f;
                    gb[k] = vb[k] ? half_bits_to_float(a.k_gamma[rb_g]) : 0.f;
                }
            }
        }
        // ---- keys: the lane's 4*KB bytes of rows tau(g) and tau(g+8) of every tile
        uint32_t sa[TPW][4], sb[TPW][4];
        uint32_t ka[TPW][8], kb8[TPW][8];  // int8 keys: channels 32 t .. 32 t + 31 of rows tau(g), tau(g + 8)
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            const uint32_t kst = sbase + L.k_off + (lb + TS * k) * VBK;
            if constexpr (KB == INT8_BITS) {
                // 128-byte rows all start at bank 0: lanes of odd g read their
                // second 16 bytes first, so a quarter-warp (g = 2q, 2q + 1) hits
                // 32 distinct banks
                const uint32_t sw = (g & 1) * 16;
                const uint4 x0 = ptx::lds128(kst + ra * VBK + 32 * t + sw);
                const uint4 x1 = ptx::lds128(kst + ra * VBK + 32 * t + (sw ^ 16));
                const uint4 y0 = ptx::lds128(kst + rb * VBK + 32 * t + sw);
                const uint4 y1 = ptx::lds128(kst + rb * VBK + 32 * t + (sw ^ 16));
                const bool odd = g & 1;
                ka[k][0] = odd ? x1.x : x0.x; ka[k][1] = odd ? x1.y : x0.y; ka[k][2] = odd ? x1.z : x0.z; ka[k][3] = odd ? x1.w : x0.w;
                ka[k][4] = odd ? x0.x : x1.x; ka[k][5] = odd ? x0.y : x1.y; ka[k][6] = odd ? x0.z : x1.z; ka[k][7] = odd ? x0.w : x1.w;
                kb8[k][0] = odd ? y1.x : y0.x; kb8[k][1] = odd ? y1.y : y0.y; kb8[k][2] = odd ? y1.z : y0.z; kb8[k][3] = odd ? y1.w : y0.w;
                kb8[k][4] = odd ? y0.x : y1.x; kb8[k][5] = odd ? y0.y : y1.y; kb8[k][6] = odd ? y0.z : y1.z; kb8[k][7] = odd ? y0.w : y1.w;
            } else if constexpr (KB == 4) {
                const uint4 x = ptx::lds128(kst + ra * VBK + 16 * t);
                const uint4 y = ptx::lds128(kst + rb * VBK + 16 * t);
                sa[k][0] = x.x; sa[k][1] = x.y; sa[k][2] = x.z; sa[k][3] = x.w;
                sb[k][0] = y.x; sb[k][1] = y.y; sb[k][2] = y.z; sb[k][3] = y.w;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) sa[k][q] = sb[k][q] = 0u;
#pragma unroll
                for (int q = 0; q < KB; ++q) {
                    sa[k][q] = ptx::lds32(kst + ra * VBK + 4 * KB * t + 4 * q);
                    sb[k][q] = ptx::lds32(kst + rb * VBK + 4 * KB * t + 4 * q);
                }
            }
        }
        // ---- scores: hi and lo query parts accumulate in separate chains
        float cs[TPW][NT][4], cl[TPW][NT][4], cz[TPW][NT][4];
#pragma unroll
        for (int k = 0; k < TPW; ++k)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) cs[k][nt][e] = cl[k][nt][e] = cz[k][nt][e] = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int k = 0; k < TPW; ++k) {
                uint32_t a0, a1, a2, a3;
                if constexpr (KB == INT8_BITS) {
                    int8_pairs(ka[k][j], a0, a2);
                    int8_pairs(kb8[k][j], a1, a3);
                } else {
                    a0 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sa[k], j, 0, laneoff));
                    a1 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sb[k], j, 0, laneoff));
                    a2 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sa[k], j, 1, laneoff));
                    a3 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sb[k], j, 1, laneoff));
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    ptx::mma_16816(cs[k][nt], a0, a1, a2, a3, bq[nt][j][0], bq[nt][j][1]);
                    ptx::mma_16816(cl[k][nt], a0, a1, a2, a3, bq[nt][j][2], bq[nt][j][3]);
                }
            }
        if constexpr (QJL) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int k = 0; k < TPW; ++k) {
                    // +-1 pairs from sign bits (bit set -> +1)
                    const uint32_t xa = za[k] >> (4 * j), xb = zb2[k] >> (4 * j);
                    const uint32_t a0 = 0xBC00BC00u ^ ((xa & 1u) << 15) ^ ((xa & 2u) << 30);
                    const uint32_t a2 = 0xBC00BC00u ^ ((xa & 4u) << 13) ^ ((xa & 8u) << 28);
                    const uint32_t a1 = 0xBC00BC00u ^ ((xb & 1u) << 15) ^ ((xb & 2u) << 30);
                    const uint32_t a3 = 0xBC00BC00u ^ ((xb & 4u) << 13) ^ ((xb & 8u) << 28);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) ptx::mma_16816(cz[k][nt], a0, a1, a2, a3, bz[nt][j][0], bz[nt][j][1]);
                }
        }
        float s[TPW][NT][4];
#pragma unroll
        for (int k = 0; k < TPW; ++k)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v = (cs[k][nt][e] + cl[k][nt][e]) * f1[nt][e & 1];
                    if constexpr (QJL) v = fmaf((e < 2 ? ga[k] : gb[k]) * cz[k][nt][e], f2[nt][e & 1], v);
                    v *= e < 2 ? kna[k] : knb[k];
                    if (MASK) v = (e < 2 ? va[k] : vb[k]) ? v : -INFINITY;
                    s[k][nt][e] = v;
                }

        // ---- softmax: the reference max moves only when a score exceeds it by 2^LAZY
        bool need = false;
        float lm[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            lm[nt][0] = lm[nt][1] = -INFINITY;
#pragma unroll
            for (int k = 0; k < TPW; ++k) {
                lm[nt][0] = fmaxf(lm[nt][0], fmaxf(s[k][nt][0], s[k][nt][2]));
                lm[nt][1] = fmaxf(lm[nt][1], fmaxf(s[k][nt][1], s[k][nt][3]));
            }
            need |= lm[nt][0] > S.m[nt][0] + LAZY || lm[nt][1] > S.m[nt][1] + LAZY;
        }
        float vmax = 0.f;
#pragma unroll
        for (int k = 0; k < TPW; ++k) vmax = fmaxf(vmax, fmaxf(vn[k][0], vn[k][1]));
        need |= (S.vscale == 0.f && vmax > 0.f) || vmax * S.vscale > VRANGE;
        if (__any_sync(kFullMask, need)) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    lm[nt][0] = fmaxf(lm[nt][0], __shfl_xor_sync(kFullMask, lm[nt][0], o));
                    lm[nt][1] = fmaxf(lm[nt][1], __shfl_xor_sync(kFullMask, lm[nt][1], o));
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float mn = fmaxf(S.m[nt][h], lm[nt][h]);
                    if (mn > S.m[nt][h]) {
                        const float c = ptx::ex2(S.m[nt][h] - mn);
                        S.l[nt][h] *= c;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            S.acc[nt][i][h] *= c;
                            S.acc[nt][i][h + 2] *= c;
                        }
                        S.m[nt][h] = mn;
                    }
                }
            }
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(kFullMask, vmax, o));
            if (vmax > 0.f && (S.vscale == 0.f || vmax * S.vscale > VRANGE)) {
                const float target = exp2f(-ceilf(log2f(vmax)));  // vmax * target in (0.5, 1]
                if (S.vscale > 0.f) {
                    const float f = target / S.vscale;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 8; ++i)
#pragma unroll
                            for (int e = 0; e < 4; ++e) S.acc[nt][i][e] *= f;
                }
                S.vscale = target;
            }
        }

        // ---- weights of every tile (Sparse V drops provably small ones)
        float pv[TPW][NT][4];
        bool any_v = false;
#pragma unroll
        for (int k = 0; k < TPW; ++k)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) pv[k][nt][e] = ptx::ex2(s[k][nt][e] - S.m[nt][e & 1]);
                S.l[nt][0] += pv[k][nt][0] + pv[k][nt][2];
                S.l[nt][1] += pv[k][nt][1] + pv[k][nt][3];
            }
        if (a.tau > 0.f) {
            // Sparse V: the exact denominator relative to the reference is at
            // least 1 (the reference is a seen score) and at least this lane's
            // partial sum, so p / max(1, l) bounds the exact weight
            bool drop[TPW][NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float th0 = a.tau * fmaxf(1.f, S.l[nt][0]), th1 = a.tau * fmaxf(1.f, S.l[nt][1]);
#pragma unroll
                for (int k = 0; k < TPW; ++k) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        drop[k][nt][e] = pv[k][nt][e] < ((e & 1) ? th1 : th0) && (e < 2 ? va[k] : vb[k]);
                        if (drop[k][nt][e]) pv[k][nt][e] = 0.f;
                    }
                    any_v |= (pv[k][nt][0] + pv[k][nt][1] + pv[k][nt][2] + pv[k][nt][3]) > 0.f;
                }
            }
            if (a.skip_mask) {
#pragma unroll
                for (int k = 0; k < TPW; ++k)
                    if (!MASK || t0 + lb + TS * k < w.s1) record_drops(w, t0 + lb + TS * k, drop[k]);
            }
            // no weight of this warp's tiles left: their value products add nothing
            if (!__any_sync(kFullMask, any_v)) return;
        }
        // ---- values: both tiles' products in one stretch (a tile past the
        // item's end has zero weights and adds nothing)
        uint32_t bv[TPW][NT][2];
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            const float wa = vn[k][0] * S.vscale, wb = vn[k][1] * S.vscale;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                bv[k][nt][0] = ptx::movmatrix_trans(ptx::pack_half2(pv[k][nt][0] * wa, pv[k][nt][1] * wa));
                bv[k][nt][1] = ptx::movmatrix_trans(ptx::pack_half2(pv[k][nt][2] * wb, pv[k][nt][3] * wb));
            }
        }
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            uint32_t A[8][4];
            value_fragments<VB>(sbase + L.v_off + (lb + TS * k) * VBV, base, g, t, laneoff, A);
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    ptx::mma_16816(S.acc[nt][i], A[i][0], A[i][1], A[i][2], A[i][3], bv[k][nt][0], bv[k][nt][1]);
        }
    }

    // One chunk, tile after tile: the form for the register-heavy
    // configurations (16-head groups, the QJL sketch), where holding both
    // tiles' scores at once would spill.  MASK: the chunk may end before CHUNK
    // tokens.
    template <bool MASK>
    __device__ void chunk_seq(const Item& w, const uint8_t* st, int t0, const uint32_t (&bq)[NT][8][4],
                          const uint32_t (&bz)[NT][4][2], const float (&f1)[NT][2], const float (&f2)[NT][2],
                          SoftState<NT>& S) {
        constexpr int VBK = 16 * KB, VBV = 16 * VB;
        // this warp's tiles are k * CW + warp (k < TPW): a short last chunk
        // spreads over many warps instead of keeping two tiles on a few
        const int lb = 16 * warp;  // first chunk-local token of this warp's first tile
        constexpr int TS = 16 * CW;  // token distance between a warp's tiles
        if (MASK && t0 + lb >= w.s1) return;  // nothing of this warp's tiles is valid
        const uint32_t sbase = ptx::smem_addr(st);
        const int ra = tau_row(g), rb = tau_row(g + 8);
        const int zw = a.m / 16;
        const bool zt = 16 * t < a.m;
        const size_t unit_row = static_cast<size_t>(w.unit) * a.capacity;
        float s[TPW][NT][4];
        float vn[TPW][2];
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            if (MASK && t0 + lb + TS * k >= w.s1) {  // tile past the item's end (warp-uniform)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[k][nt][e] = -INFINITY;
                vn[k][0] = vn[k][1] = 0.f;
                continue;
            }
            const int la = lb + TS * k + ra, lbb = lb + TS * k + rb;  // chunk-local tokens of rows g, g+8
            const bool va = !MASK || t0 + la < w.s1, vb = !MASK || t0 + lbb < w.s1;
            float kna, knb, ga = 0.f, gb = 0.f;
            uint32_t za = 0, zb2 = 0;
            if (a.staged_norms) {
                const __half* skn = reinterpret_cast<const __half*>(st + L.kn_off);
                const __half* svn = reinterpret_cast<const __half*>(st + L.vn_off);
                kna = __half2float(skn[la]);
                knb = __half2float(skn[lbb]);
                vn[k][0] = va ? __half2float(svn[la]) : 0.f;
                vn[k][1] = vb ? __half2float(svn[lbb]) : 0.f;
                if constexpr (QJL) {
                    const uint16_t* sz = reinterpret_cast<const uint16_t*>(st + L.z_off);
                    const __half* sg = reinterpret_cast<const __half*>(st + L.gam_off);
                    za = zt ? sz[la * zw + t] : 0u;
                    zb2 = zt ? sz[lbb * zw + t] : 0u;
                    ga = __half2float(sg[la]);
                    gb = __half2float(sg[lbb]);
                }
            } else {
                kna = va ? half_bits_to_float(a.k_norms[unit_row + t0 + la]) : 0.f;
                knb = vb ? half_bits_to_float(a.k_norms[unit_row + t0 + lbb]) : 0.f;
                vn[k][0] = va ? half_bits_to_float(a.v_norms[unit_row + t0 + la]) : 0.f;
                vn[k][1] = vb ? half_bits_to_float(a.v_norms[unit_row + t0 + lbb]) : 0.f;
                if constexpr (QJL) {
                    const uint16_t* zr = reinterpret_cast<const uint16_t*>(a.k_qjl);
                    za = (va && zt) ? zr[(unit_row + t0 + la) * zw + t] : 0u;
                    zb2 = (vb && zt) ? zr[(unit_row + t0 + lbb) * zw + t] : 0u;
                    ga = va ? half_bits_to_float(a.k_gamma[unit_row + t0 + la]) : 0.f;
                    gb = vb ? half_bits_to_float(a.k_gamma[unit_row + t0 + lbb]) : 0.f;
                }
            }
            // ---- keys: the lane's 4*KB bytes of rows tau(g) and tau(g+8)
            const uint32_t kst = sbase + L.k_off + (lb + TS * k) * VBK;
            uint32_t sa[4] = {0, 0, 0, 0}, sb[4] = {0, 0, 0, 0};
            uint32_t ka[8], kb8[8];  // int8 keys: channels 32 t .. 32 t + 31 of rows tau(g), tau(g + 8)
            if constexpr (KB == INT8_BITS) {
                // 128-byte rows all start at bank 0: lanes of odd g read their
                // second 16 bytes first, so a quarter-warp (g = 2q, 2q + 1) hits
                // 32 distinct banks
                const uint32_t sw = (g & 1) * 16;
                const uint4 x0 = ptx::lds128(kst + ra * VBK + 32 * t + sw);
                const uint4 x1 = ptx::lds128(kst + ra * VBK + 32 * t + (sw ^ 16));
                const uint4 y0 = ptx::lds128(kst + rb * VBK + 32 * t + sw);
                const uint4 y1 = ptx::lds128(kst + rb * VBK + 32 * t + (sw ^ 16));
                const bool odd = g & 1;
                ka[0] = odd ? x1.x : x0.x; ka[1] = odd ? x1.y : x0.y; ka[2] = odd ? x1.z : x0.z; ka[3] = odd ? x1.w : x0.w;
                ka[4] = odd ? x0.x : x1.x; ka[5] = odd ? x0.y : x1.y; ka[6] = odd ? x0.z : x1.z; ka[7] = odd ? x0.w : x1.w;
                kb8[0] = odd ? y1.x : y0.x; kb8[1] = odd ? y1.y : y0.y; kb8[2] = odd ? y1.z : y0.z; kb8[3] = odd ? y1.w : y0.w;
                kb8[4] = odd ? y0.x : y1.x; kb8[5] = odd ? y0.y : y1.y; kb8[6] = odd ? y0.z : y1.z; kb8[7] = odd ? y0.w : y1.w;
            } else if constexpr (KB == 4) {
                const uint4 x = ptx::lds128(kst + ra * VBK + 16 * t);
                const uint4 y = ptx::lds128(kst + rb * VBK + 16 * t);
                sa[0] = x.x; sa[1] = x.y; sa[2] = x.z; sa[3] = x.w;
                sb[0] = y.x; sb[1] = y.y; sb[2] = y.z; sb[3] = y.w;
            } else {
#pragma unroll
                for (int q = 0; q < KB; ++q) {
                    sa[q] = ptx::lds32(kst + ra * VBK + 4 * KB * t + 4 * q);
                    sb[q] = ptx::lds32(kst + rb * VBK + 4 * KB * t + 4 * q);
                }
            }
            // hi and lo query parts accumulate in separate chains
            float cs[NT][4], cl[NT][4], cz[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) cs[nt][e] = cl[nt][e] = cz[nt][e] = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t a0, a1, a2, a3;
                if constexpr (KB == INT8_BITS) {
                    int8_pairs(ka[j], a0, a2);
                    int8_pairs(kb8[j], a1, a3);
                } else {
                    a0 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sa, j, 0, laneoff));
                    a1 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sb, j, 0, laneoff));
                    a2 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sa, j, 1, laneoff));
                    a3 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sb, j, 1, laneoff));
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    ptx::mma_16816(cs[nt], a0, a1, a2, a3, bq[nt][j][0], bq[nt][j][1]);
                    ptx::mma_16816(cl[nt], a0, a1, a2, a3, bq[nt][j][2], bq[nt][j][3]);
                }
            }
            if constexpr (QJL) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // +-1 pairs from sign bits (bit set -> +1)
                    const uint32_t xa = za >> (4 * j), xb = zb2 >> (4 * j);
                    const uint32_t a0 = 0xBC00BC00u ^ ((xa & 1u) << 15) ^ ((xa & 2u) << 30);
                    const uint32_t a2 = 0xBC00BC00u ^ ((xa & 4u) << 13) ^ ((xa & 8u) << 28);
                    const uint32_t a1 = 0xBC00BC00u ^ ((xb & 1u) << 15) ^ ((xb & 2u) << 30);
                    const uint32_t a3 = 0xBC00BC00u ^ ((xb & 4u) << 13) ^ ((xb & 8u) << 28);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) ptx::mma_16816(cz[nt], a0, a1, a2, a3, bz[nt][j][0], bz[nt][j][1]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v = (cs[nt][e] + cl[nt][e]) * f1[nt][e & 1];
                    if constexpr (QJL) v = fmaf((e < 2 ? ga : gb) * cz[nt][e], f2[nt][e & 1], v);
                    v *= e < 2 ? kna : knb;
                    if (MASK) v = (e < 2 ? va : vb) ? v : -INFINITY;
                    s[k][nt][e] = v;
                }
        }

        // ---- softmax: the reference max moves only when a score exceeds it by 2^LAZY
        bool need = false;
        float lm[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            lm[nt][0] = lm[nt][1] = -INFINITY;
#pragma unroll
            for (int k = 0; k < TPW; ++k) {
                lm[nt][0] = fmaxf(lm[nt][0], fmaxf(s[k][nt][0], s[k][nt][2]));
                lm[nt][1] = fmaxf(lm[nt][1], fmaxf(s[k][nt][1], s[k][nt][3]));
            }
            need |= lm[nt][0] > S.m[nt][0] + LAZY || lm[nt][1] > S.m[nt][1] + LAZY;
        }
        float vmax = 0.f;
#pragma unroll
        for (int k = 0; k < TPW; ++k) vmax = fmaxf(vmax, fmaxf(vn[k][0], vn[k][1]));
        need |= (S.vscale == 0.f && vmax > 0.f) || vmax * S.vscale > VRANGE;
        if (__any_sync(kFullMask, need)) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    lm[nt][0] = fmaxf(lm[nt][0], __shfl_xor_sync(kFullMask, lm[nt][0], o));
                    lm[nt][1] = fmaxf(lm[nt][1], __shfl_xor_sync(kFullMask, lm[nt][1], o));
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float mn = fmaxf(S.m[nt][h], lm[nt][h]);
                    if (mn > S.m[nt][h]) {
                        const float c = ptx::ex2(S.m[nt][h] - mn);
                        S.l[nt][h] *= c;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            S.acc[nt][i][h] *= c;
                            S.acc[nt][i][h + 2] *= c;
                        }
                        S.m[nt][h] = mn;
                    }
                }
            }
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(kFullMask, vmax, o));
            if (vmax > 0.f && (S.vscale == 0.f || vmax * S.vscale > VRANGE)) {
                const float target = exp2f(-ceilf(log2f(vmax)));  // vmax * target in (0.5, 1]
                if (S.vscale > 0.f) {
                    const float f = target / S.vscale;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 8; ++i)
#pragma unroll
                            for (int e = 0; e < 4; ++e) S.acc[nt][i][e] *= f;
                }
                S.vscale = target;
            }
        }

        // ---- values, tile by tile
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            if (MASK && t0 + lb + TS * k >= w.s1) break;  // warp-uniform
            float pv[NT][4];
            bool any_v = false;
            bool drop[NT][4];
            // rows g and g + 8 hold tokens of the sequence (the last chunk may end early)
            const bool rva = !MASK || t0 + lb + TS * k + ra < w.s1, rvb = !MASK || t0 + lb + TS * k + rb < w.s1;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) pv[nt][e] = ptx::ex2(s[k][nt][e] - S.m[nt][e & 1]);
                S.l[nt][0] += pv[nt][0] + pv[nt][2];
                S.l[nt][1] += pv[nt][1] + pv[nt][3];
                if (a.tau > 0.f) {
                    // Sparse V: the exact denominator relative to the reference is at
                    // least 1 (the reference is a seen score) and at least this lane's
                    // partial sum, so p / max(1, l) bounds the exact weight
                    const float th0 = a.tau * fmaxf(1.f, S.l[nt][0]), th1 = a.tau * fmaxf(1.f, S.l[nt][1]);
                    if constexpr (REC) {  // the caller asked which positions were dropped
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            drop[nt][e] = pv[nt][e] < ((e & 1) ? th1 : th0) && (e < 2 ? rva : rvb);
                    }
                    if (pv[nt][0] < th0) pv[nt][0] = 0.f;
                    if (pv[nt][2] < th0) pv[nt][2] = 0.f;
                    if (pv[nt][1] < th1) pv[nt][1] = 0.f;
                    if (pv[nt][3] < th1) pv[nt][3] = 0.f;
                    any_v |= (pv[nt][0] + pv[nt][1] + pv[nt][2] + pv[nt][3]) > 0.f;
                }
            }
            if constexpr (REC)
                if (a.tau > 0.f) record_drops(w, t0 + lb + TS * k, drop);
            if (a.tau > 0.f && !__any_sync(kFullMask, any_v)) continue;
            if (S.vscale == 0.f) continue;  // every value norm so far is zero
            const float wa = vn[k][0] * S.vscale, wb = vn[k][1] * S.vscale;
            uint32_t bv[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                bv[nt][0] = ptx::movmatrix_trans(ptx::pack_half2(pv[nt][0] * wa, pv[nt][1] * wa));
                bv[nt][1] = ptx::movmatrix_trans(ptx::pack_half2(pv[nt][2] * wb, pv[nt][3] * wb));
            }
            uint32_t A[8][4];
            value_fragments<VB>(sbase + L.v_off + (lb + TS * k) * VBV, base, g, t, laneoff, A);
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    ptx::mma_16816(S.acc[nt][i], A[i][0], A[i][1], A[i][2], A[i][3], bv[nt][0], bv[nt][1]);
        }
    }

    template <bool MASK>
    __device__ void chunk(const Item& w, const uint8_t* st, int t0, const uint32_t (&bq)[NT][8][4],
                          const uint32_t (&bz)[NT][4][2], const float (&f1)[NT][2], const float (&f2)[NT][2],
                          SoftState<NT>& S) {
        if constexpr (NT == 1 && !QJL) chunk_il<MASK>(w, st, t0, bq, bz, f1, f2, S);
        else chunk_seq<MASK>(w, st, t0, bq, bz, f1, f2, S);
    }

    __device__ float group_sum_g(float x) const {  // sum over the 8 lanes sharing t
        x += __shfl_xor_sync(kFullMask, x, 4);
        x += __shfl_xor_sync(kFullMask, x, 8);
        x += __shfl_xor_sync(kFullMask, x, 16);
        return x;
    }

    // End of an item: merge the warps, publish the split's partial, and merge
    // all splits when this is the last one of its (sequence, kv head).
    __device__ void epilogue(const Item& w, SoftState<NT>& S) {
        const int G = a.group;
        float* merge = reinterpret_cast<float*>(smem + L.merge);
        float2* ml = reinterpret_cast<float2*>(smem + L.ml);
        int* last_flag = reinterpret_cast<int*>(smem + L.flags + 4);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float l = group_sum_g(S.l[nt][h]);
                if (g == 0) ml[warp * 16 + nt * 8 + 2 * t + h] = make_float2(S.m[nt][h], l);
            }
        const float unscale = S.vscale > 0.f ? 1.0f / S.vscale : 0.f;
        const size_t pbase = (static_cast<size_t>(w.unit) * a.n_split + w.split) * G;
        const int GM = G < MERGE_HEADS ? G : MERGE_HEADS;  // heads per combine pass
        for (int hb = 0; hb < G; hb += GM) {
            if (hb > 0) ptx::named_barrier(1, NUM_CONSUMERS);  // the previous pass has read the buffer
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int h0 = nt * 8 + 2 * t;  // heads h0, h0 + 1 of this lane's columns (same pass)
                    if (h0 < hb || h0 >= hb + GM) continue;
                    float* mw = merge + (warp * GM + h0 - hb) * MSTRIDE;
                    const int c_lo = mslot(16 * g + 2 * i), c_hi = c_lo + 1;
                    if (h0 < G) {
                        mw[c_lo] = S.acc[nt][i][0] * unscale;
                        mw[c_hi] = S.acc[nt][i][2] * unscale;
                    }
                    if (h0 + 1 < G) {
                        mw[MSTRIDE + c_lo] = S.acc[nt][i][1] * unscale;
                        mw[MSTRIDE + c_hi] = S.acc[nt][i][3] * unscale;
                    }
                }
            ptx::named_barrier(1, NUM_CONSUMERS);
            // every output column is one weighted sum over the warps, with the
            // weights 2^(m_w - M) of its head (each thread forms them; the
            // thread of a head's first column also writes the split's (M, L))
            const float4* m4 = reinterpret_cast<const float4*>(merge);
            float4* dst4 = reinterpret_cast<float4*>(a.ws_acc + pbase * D);
            const int np = G - hb < GM ? G - hb : GM;  // heads of this pass (the last may hold fewer)
            for (int idx = tid; idx < np * (D / 4); idx += NUM_CONSUMERS) {
                const int hl = idx / (D / 4), h = hb + hl, c4 = idx % (D / 4);
                float mx = -INFINITY;
#pragma unroll
                for (int ww = 0; ww < CW; ++ww)
                    if (ml[ww * 16 + h].y > 0.f) mx = fmaxf(mx, ml[ww * 16 + h].x);
                float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
                float l = 0.f;
#pragma unroll
                for (int ww = 0; ww < CW; ++ww) {
                    const float2 mlw = ml[ww * 16 + h];
                    const float f = (mlw.y > 0.f && mx > -INFINITY) ? ptx::ex2(mlw.x - mx) : 0.f;
                    l = fmaf(mlw.y, f, l);
                    const float4 v = m4[(ww * GM + hl) * (MSTRIDE / 4) + (c4 >> 2) * (MBLK / 4) + (c4 & 3)];
                    acc4.x = fmaf(v.x, f, acc4.x);
                    acc4.y = fmaf(v.y, f, acc4.y);
                    acc4.z = fmaf(v.z, f, acc4.z);
                    acc4.w = fmaf(v.w, f, acc4.w);
                }
                const float iv = a.inv_alpha_v;  // undo the centroid scale
                dst4[h * (D / 4) + c4] = make_float4(acc4.x * iv, acc4.y * iv, acc4.z * iv, acc4.w * iv);
                if (c4 == 0) a.ws_ml[pbase + h] = make_float2(mx, l);
            }
        }
        // publish the partial: the barrier orders every thread's writes before
        // thread 0's release, and its acquire orders the merge's reads after
        // the other blocks' partials
        ptx::named_barrier(1, NUM_CONSUMERS);
        const int nlive = live_splits(a, w.len);  // the splits the merge waits for
        if (tid == 0) *last_flag = ptx::atom_add_acq_rel_gpu(a.counters + w.unit, 1u) ==
                                   static_cast<uint32_t>(nlive - 1);
        ptx::named_barrier(1, NUM_CONSUMERS);
        if (*last_flag) {
            // Merge the splits: two warps per head, each lane two channels.
            // With at most 32 live splits (the usual case) every load, the
            // partial rows and one (m, l) pair per lane, is issued before any
            // is used, so the merge costs one round trip to L2; the weights
            // 2^(m_s - M) are formed per lane and broadcast by shuffles.  Longer
            // lists take batches.  Either way the weighted sum runs in split
            // order, so the result does not depend on timing.
            float* o_s = merge;  // [G][D]
            const size_t ubase = static_cast<size_t>(w.unit) * a.n_split * G;
            const float2* src2 = reinterpret_cast<const float2*>(a.ws_acc + ubase * D);
            // splits per batch of loads (at most one per lane for the weights); the
            // register-heavy configurations take smaller batches
            constexpr int PB = (NT == 1 && !QJL) ? 32 : 8;
            for (int u = warp; u < 2 * G; u += CW) {
                const int h = u >> 1, c2 = (u & 1) * 32 + lane;  // float2 column
                float2 acc = make_float2(0.f, 0.f);
                float l = 0.f;
                if (nlive <= PB) {
                    float2 v[PB];
#pragma unroll
                    for (int j = 0; j < PB; ++j)
                        v[j] = j < nlive ? __ldcg(src2 + (j * G + h) * (D / 2) + c2) : make_float2(0.f, 0.f);
                    const float2 m2 = lane < nlive ? __ldcg(a.ws_ml + ubase + lane * G + h) : make_float2(-INFINITY, 0.f);
                    const float mx = group_max<32>(m2.y > 0.f ? m2.x : -INFINITY);
                    const float wgt = (m2.y > 0.f && mx > -INFINITY) ? ptx::ex2(m2.x - mx) : 0.f;
                    l = group_sum<32>(m2.y * wgt);
#pragma unroll
                    for (int j = 0; j < PB; ++j) {
                        const float wj = __shfl_sync(kFullMask, wgt, j);
                        if (j < nlive) {
                            acc.x = fmaf(v[j].x, wj, acc.x);
                            acc.y = fmaf(v[j].y, wj, acc.y);
                        }
                    }
                } else {
                    float* wts = merge + G * D + warp * a.n_split;
                    float mx = -INFINITY;
                    for (int sp = lane; sp < nlive; sp += 32) {
                        const float2 m2 = __ldcg(a.ws_ml + ubase + sp * G + h);
                        if (m2.y > 0.f) mx = fmaxf(mx, m2.x);
                    }
                    mx = group_max<32>(mx);
                    for (int sp = lane; sp < nlive; sp += 32) {
                        const float2 m2 = __ldcg(a.ws_ml + ubase + sp * G + h);
                        const float wgt = (m2.y > 0.f && mx > -INFINITY) ? ptx::ex2(m2.x - mx) : 0.f;
                        wts[sp] = wgt;
                        l = fmaf(m2.y, wgt, l);
                    }
                    l = group_sum<32>(l);
                    __syncwarp();
                    for (int s0 = 0; s0 < nlive; s0 += PB) {
                        float2 v[PB];
#pragma unroll
                        for (int j = 0; j < PB; ++j)
                            v[j] = s0 + j < nlive ? __ldcg(src2 + ((s0 + j) * G + h) * (D / 2) + c2)
                                                  : make_float2(0.f, 0.f);
#pragma unroll
                        for (int j = 0; j < PB; ++j) {
                            const float wgt = s0 + j < nlive ? wts[s0 + j] : 0.f;
                            acc.x = fmaf(v[j].x, wgt, acc.x);
                            acc.y = fmaf(v[j].y, wgt, acc.y);
                        }
                    }
                    __syncwarp();  // the weights row is rewritten by this warp's next unit
                }
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                *reinterpret_cast<float2*>(o_s + h * D + 2 * c2) = make_float2(acc.x * inv_l, acc.y * inv_l);
            }
            ptx::named_barrier(1, NUM_CONSUMERS);
            const float inv_sqrt_d = 0.08838834764831845f;
            for (int h = warp; h < G; h += CW) {
                float x[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) x[e] = o_s[h * D + lane * 4 + e];
                float* dst = a.out + (static_cast<size_t>(w.b) * a.hq + w.kv * G + h) * D + lane * 4;
                if constexpr (VB == INT8_BITS) {  // int8 values: already in the original domain
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = x[e];
                } else {
                    fwht_registers(x);
                    fwht_lanes<4, 32>(x, lane);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = flip_sign(x[e] * inv_sqrt_d, (sgn4 >> e) & 1u);
                }
            }
            if (tid == 0) a.counters[w.unit] = 0;
        }
        ptx::named_barrier(1, NUM_CONSUMERS);
    }

    __device__ void run() {
        const uint32_t full0 = base + L.bars, empty0 = full0 + 64, qfull0 = full0 + 128, qempty0 = full0 + 144;
        uint32_t bq[NT][8][4];
        uint32_t bz[NT][4][2];
        float f1[NT][2], f2[NT][2];
        SoftState<NT> S;
        int seq = 0, qseq = 0;
        bool done_ok = false, first_rotated = false;
        // The block's first item: its queries were requested before anything
        // else and complete on their own barrier, so they are rotated before
        // the item's header (which waits for the sequence length) arrives.
        if (static_cast<int>(blockIdx.x) < a.n_items) {
            if (!ptx::mbar_wait_bounded(base + L.bars + 160, 0, WAIT_LIMIT)) set_abort();
            if (!aborted()) {
                rotate(0);
                first_rotated = true;
            }
        }
        while (true) {
            // next item: its header (and queries) in query slot qseq
            if (!ptx::mbar_wait_bounded(qfull0 + 8 * (qseq & 1), (qseq >> 1) & 1, WAIT_LIMIT)) set_abort();
            // every consumer warp takes the same decision (the producer may set
            // the flag at any moment, so each thread's own read could differ)
            if (ptx::named_barrier_or(1, NUM_CONSUMERS, aborted())) break;
            const int4* qh = reinterpret_cast<const int4*>(smem + L.qring + (qseq & 1) * L.qslot);
            const int4 h0 = qh[0], h1 = qh[1];
            if (h1.x & F_END) {
                done_ok = true;
                break;
            }
            Item w;
            w.split = h0.x % a.n_split;
            w.s0 = h0.y;
            w.s1 = h0.z;
            w.len = h0.w;
            w.unit = h1.y;
            w.b = h1.z;
            w.kv = h1.w;
            w.bad = false;
            const bool empty = h1.x & F_EMPTY, app = h1.x & F_APPEND;
            S.reset();
            if (!empty) prologue(qseq, qseq == 0 && first_rotated, w, app, bq, bz, f1, f2);  // ends the slot's use
            else ptx::named_barrier(1, NUM_CONSUMERS);           // every warp has read the header
            if (tid == 0) ptx::mbar_arrive(qempty0 + 8 * (qseq & 1));  // query slot free
            ++qseq;
            // Warps wait for each stage on their own.  A wait that runs out sets
            // the abort flag and later waits are skipped, but every warp still
            // walks the item's stages and meets the others at the item's named
            // barriers (the patch below, the epilogue), so none is left behind.
            for (int t0 = w.s0; t0 < w.s1; t0 += CHUNK) {
                const int slot = seq % a.stages, use = seq / a.stages;
                if (!aborted() && !ptx::mbar_wait_bounded(full0 + 8 * slot, use & 1, WAIT_LIMIT)) set_abort();
                const bool ok = !aborted();
                const uint8_t* st = smem + L.ring + slot * L.stage_bytes;
                const bool last = t0 + CHUNK >= w.s1;
                if (app && last) {  // the stage holding the appended token
                    if (ok) patch_stage(const_cast<uint8_t*>(st), w.len - 1 - t0);
                    ptx::named_barrier(1, NUM_CONSUMERS);
                }
                if (ok) {
                    if (last) chunk<true>(w, st, t0, bq, bz, f1, f2, S);
                    else chunk<false>(w, st, t0, bq, bz, f1, f2, S);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(empty0 + 8 * slot);
                ++seq;
            }
            // stages requested before the item's length was known and not
            // needed after all: wait for their copies, release them unread
            for (int dr = h1.x >> DRAIN_SHIFT; dr > 0; --dr) {
                const int slot = seq % a.stages, use = seq / a.stages;
                if (!aborted() && !ptx::mbar_wait_bounded(full0 + 8 * slot, use & 1, WAIT_LIMIT)) set_abort();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(empty0 + 8 * slot);
                ++seq;
            }
            if (!(h1.x & F_SKIP)) epilogue(w, S);
            if (ptx::named_barrier_or(1, NUM_CONSUMERS, aborted())) break;
        }
        if (done_ok && tid == 0) {
            // the last block to finish re-arms the global counters for the next call
            __threadfence();
            if (atomicAdd(a.counters + a.units + C_DONE, 1u) == gridDim.x - 1) {
                a.counters[a.units + C_ITEM] = 0;
                a.counters[a.units + C_DONE] = 0;
            }
        }
    }
};

template <int KB, int VB, int NT, bool QJL, bool REC>
__global__ void __launch_bounds__(NUM_THREADS, 1) decode_mma_kernel(const __grid_constant__ Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const Layout L = layout(KB, VB, NT, a.stages, QJL ? a.m : 0, a.group, a.q_bytes, a.append ? a.new_bytes : 0,
                            a.n_split);
    ptx::launch_dependents();  // the next kernel may start launching; it waits for this one to finish
    if (threadIdx.x == NUM_CONSUMERS) {
        const uint32_t bars = ptx::smem_addr(smem + L.bars);
        for (int s = 0; s < a.stages; ++s) {
            ptx::mbar_init(bars + 8 * s, 1);
            ptx::mbar_init(bars + 64 + 8 * s, CW);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(bars + 128 + 8 * s, 1);
            ptx::mbar_init(bars + 144 + 8 * s, 1);
        }
        {
            ptx::mbar_init(bars + 160, 1);  // the first item's queries
        }
        *reinterpret_cast<int*>(smem + L.flags) = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();  // mbarriers initialised
    if (threadIdx.x >= NUM_CONSUMERS) {
        if (threadIdx.x == NUM_CONSUMERS) {
            producer<KB, VB, QJL>(a, smem, L);  // waits for the previous kernel itself
        }
        return;
    }
    // Per-lane replicated centroid-pair tables, built while the first copies
    // fly: row e (256 bytes) holds the key pair for code byte e in its first
    // 32 words and the value pair(s) in the last 32.  Step 1: thread e forms
    // row e's words once (from centroids staged in shared memory: a per-thread
    // index into the kernel parameters would serialise).  Step 2: the
    // threads replicate them in address order, 16 bytes per store (a warp
    // covers 512 contiguous bytes), with independent reads.
    if constexpr (uses_tables(KB, VB)) {
        __half* cen = reinterpret_cast<__half*>(smem + L.app);  // [16] key, [16] value
        uint32_t* compact = reinterpret_cast<uint32_t*>(smem + L.merge);  // [256] key, [256][2] value
        if (threadIdx.x == 0) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                cen[j] = __ushort_as_half(a.kcent[j]);
                cen[16 + j] = __ushort_as_half(a.vcent[j]);
            }
        }
        ptx::named_barrier(1, NUM_CONSUMERS);
        if (threadIdx.x < 256) {
            const int e = threadIdx.x;
            const __half* kc = cen;
            const __half* vc = cen + 16;
            constexpr int KM = KB == INT8_BITS ? 0 : (1 << KB) - 1;  // int8 keys use no table
            const __half2 k2 = __halves2half2(kc[e & KM], kc[(e >> (KB & 7)) & KM]);
            __half2 v0, v1;
            if constexpr (VB >= 3) {
                constexpr int VM = VB == INT8_BITS ? 0 : (1 << VB) - 1;
                v0 = v1 = __halves2half2(vc[e & VM], vc[(e >> (VB & 7)) & VM]);
            } else {
                // byte e = (token a: two 2-bit codes) | (token b: two codes) << 4; the
                // first word holds channel 1 of (a, b), the second channel 2
                v0 = __halves2half2(vc[e & 3], vc[(e >> 4) & 3]);
                v1 = __halves2half2(vc[(e >> 2) & 3], vc[(e >> 6) & 3]);
            }
            compact[e] = *reinterpret_cast<const uint32_t*>(&k2);
            compact[256 + 2 * e] = *reinterpret_cast<const uint32_t*>(&v0);
            compact[256 + 2 * e + 1] = *reinterpret_cast<const uint32_t*>(&v1);
        }
        ptx::named_barrier(1, NUM_CONSUMERS);
        uint4* lut4 = reinterpret_cast<uint4*>(smem);
        static_assert(NUM_CONSUMERS % 16 == 0, "each thread writes one 16-byte column of the rows");
        const int part = threadIdx.x & 15;  // the same 16-byte column of every row this thread writes
        constexpr int REP = (256 * 16 + NUM_CONSUMERS - 1) / NUM_CONSUMERS;
#pragma unroll
        for (int k = 0; k < REP; ++k) {
            const int c = threadIdx.x + NUM_CONSUMERS * k;
            if (c >= 256 * 16) break;
            const int e = c >> 4;
            uint4 v;
            if (part < 8) {
                const uint32_t w = compact[e];
                v = make_uint4(w, w, w, w);
            } else {
                const uint2 w = *reinterpret_cast<const uint2*>(compact + 256 + 2 * e);
                v = make_uint4(w.x, w.y, w.x, w.y);
            }
            lut4[c] = v;
        }
    }
    if (ptx::smem_addr(smem) != WINDOW) {  // the host checked the reserved size; never expected
        if (threadIdx.x == 0) {
            if (a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
            *reinterpret_cast<volatile int*>(smem + L.flags) = 1;
        }
    }
    ptx::wait_prerequisites();
    ptx::named_barrier(1, NUM_CONSUMERS);  // tables complete
    Consumer<KB, VB, NT, QJL, REC> c(a, smem, L);
    c.run();
}

template <int KB, int VB, int NT, bool QJL, bool REC = false>
static cudaError_t launch_typed(const Args& a, int grid, size_t smem, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<KB, VB, NT, QJL, REC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_mma_kernel<KB, VB, NT, QJL, REC>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The tile-by-tile chunk (QJL sketch, 16-head groups) records Sparse V's
// dropped positions only in its own instantiation (rec): inlined into the
// ordinary one, the recording code slowed its hot loop.  The two-tile chunk
// records them at no cost and has one instantiation.
template <int KB, int VB>
static cudaError_t launch_kv(const Args& a, int nt, bool qjl, bool rec, int grid, size_t smem, cudaStream_t s) {
    if constexpr (KB == INT8_BITS) {  // no sketch on int8 keys
        if (qjl) return cudaErrorNotSupported;
        if (nt == 1) return launch_typed<KB, VB, 1, false>(a, grid, smem, s);
        return rec ? launch_typed<KB, VB, 2, false, true>(a, grid, smem, s) : launch_typed<KB, VB, 2, false>(a, grid, smem, s);
    } else {
        if (nt == 1) {
            if (!qjl) return launch_typed<KB, VB, 1, false>(a, grid, smem, s);
            return rec ? launch_typed<KB, VB, 1, true, true>(a, grid, smem, s) : launch_typed<KB, VB, 1, true>(a, grid, smem, s);
        }
        if (qjl)
            return rec ? launch_typed<KB, VB, 2, true, true>(a, grid, smem, s) : launch_typed<KB, VB, 2, true>(a, grid, smem, s);
        return rec ? launch_typed<KB, VB, 2, false, true>(a, grid, smem, s) : launch_typed<KB, VB, 2, false>(a, grid, smem, s);
    }
}

template <int KB>
static cudaError_t launch_k(const Args& a, int vb, int nt, bool qjl, bool rec, int grid, size_t smem,
                            cudaStream_t s) {
    switch (vb) {
        case INT8_BITS:
            if constexpr (KB == INT8_BITS) return launch_kv<KB, INT8_BITS>(a, nt, qjl, rec, grid, smem, s);
            return cudaErrorNotSupported;
        case 2: return launch_kv<KB, 2>(a, nt, qjl, rec, grid, smem, s);
        case 3: return launch_kv<KB, 3>(a, nt, qjl, rec, grid, smem, s);
        default: return launch_kv<KB, 4>(a, nt, qjl, rec, grid, smem, s);
    }
}

}  // namespace mmadec

}  // namespace tq
