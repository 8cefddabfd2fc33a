// Decode attention from the compressed cache on the tensor cores (sm_100a),
// head dimension 128, TURBO keys and values, GQA groups of up to 16.
//
// Pages (by title):
//   [google]  "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！",
//             sections "再看速度" and "第二步：QJL —— 1 bit 清理殘差"
//   [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命", section "Sparse V：速度加成"
//   [tqai]    "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术", section
//             "TurboQuant的核心创新"
//
// What is computed is the same as decode_split_kernel in decode.cu:
//   s_i = sm_scale ||k_i|| (<q~, c[code_i]> + gamma_i sqrt(pi/2)/m <S q~, 2z_i - 1>),
//   softmax over the sequence, acc = sum_i p_i ||v_i|| c[code_i] in the rotated
//   domain, and one inverse rotation of acc / sum_i p_i.
//
// How (one persistent thread block per SM):
//  * Work items are (sequence, kv head, token split).  A producer warp takes
//    items from a global atomic counter (so ragged batches balance), and for
//    each one streams the packed K and V codes (plus norms, QJL words and the
//    queries) of 256-token chunks into a ring of shared-memory stages with 1-D
//    bulk async copies (TMA engine, no multicast).  Each stage starts with a
//    header naming its item and token range; completion is tracked by
//    mbarriers.  Eight consumer warps take two 16-token tiles of every chunk.
//  * The dequantised tiles of a GQA group form real dense products, so both
//    contractions run on the tensor cores with warp-level m16n8k16 fp16 MMA
//    (fp32 accumulate):  S^T[16 tok x 8 heads] = K~[16 x 128] Q~^T and
//    O^T[128 x 8 heads] += V~^T[128 x 16 tok] P^T.  The A operands are built
//    in registers straight from the codes: a 256-entry, per-lane replicated
//    shared-memory table maps one byte of 4-bit key codes to a pair of fp16
//    centroids, and a register byte-permute table maps 2-bit value codes.
//    Since sum_c q~_c c[code_c] does not depend on the order of c, channels are
//    assigned to fragment slots so that each lane's 16-byte load of a key row
//    feeds its fragments directly (the query uses the same order); tokens of a
//    tile are permuted the same way on both sides (tau) so that the value
//    words each lane needs are bank-conflict free.
//  * The score fragment becomes the second MMA's operand through one movmatrix
//    transpose per 8x8 block.  The softmax rescales lazily: the running max
//    used for exp2 only moves (with a warp-wide reduction) when a score exceeds
//    it by more than 2^8, decided by one warp vote per chunk.
//  * Split results are merged by the last block to finish a (sequence, kv
//    head), found with an atomic counter (no spin-wait); it also applies the
//    inverse rotation and writes the output.
//  Every wait on an mbarrier is bounded (about a second); a wait that runs out
//  sets TQ_DEVERR_TIMEOUT, all consumer warps agree on it at the next named
//  barrier, and the block leaves after draining its copies.

#include <cuda_runtime.h>

#include <cmath>

#include "device_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace tq {
namespace mmadec {

constexpr int D = 128;
constexpr int CW = 8;                        // consumer warps
constexpr int TPW = 2;                       // 16-token tiles per warp and chunk
constexpr int NUM_THREADS = (CW + 1) * 32;   // + one producer warp
constexpr int NUM_CONSUMERS = CW * 32;
constexpr int CHUNK = CW * TPW * 16;         // tokens per stage
constexpr uint32_t LUT_BYTES = 65536;        // 256 entries x 256 B
// Shared-window address of the dynamic shared memory (the per-block reserved
// shared memory precedes it); the host checks it before choosing this kernel,
// and table lookups carry it as an immediate offset.
constexpr uint32_t WINDOW = 1024;
constexpr uint32_t Q_BYTES = 16 * D * 4;     // one item's queries, up to 16 heads in fp32
constexpr uint32_t NEW_ROW = D * 4;           // one appended key or value row, up to fp32
constexpr uint32_t QSLOT_BYTES = Q_BYTES + 2 * NEW_ROW;  // queries, then the new key and value rows
constexpr uint32_t APP_BYTES = 1024;          // the appended token's codes and scratch
constexpr long long WAIT_LIMIT = 2000000000ll;  // clock cycles (~1 s)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LAZY = 8.0f;                 // log2 headroom before the running max moves
constexpr float VRANGE = 64.0f;              // bound on ||v|| * vscale

// stage header flags
constexpr int F_FIRST = 1, F_LAST = 2, F_EMPTY = 4, F_END = 8;
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
    float inv_alpha_k, inv_alpha_v;  // 1 / (centroid scale applied before fp16 rounding)
    int staged_norms;     // capacity % 8 == 0: norms and QJL words ride in the stages
    uint32_t signs[4];
    uint16_t kcent[16];  // fp16 bits of alpha_k * key centroid
    uint16_t vcent[16];  // fp16 bits of alpha_v * value centroid
    // append mode: one new token per sequence, written at position seq_len - 1
    int append, new_dtype, new_bytes;
    const void* k_new;   // [batch][1][Hkv][d]
    const void* v_new;
    float kbound[8];     // positive decision boundaries, ascending (unused ones +inf)
    float vbound[8];
    float kc32[16];      // fp32 key centroids (QJL residual)
};

// Shared-memory map (byte offsets from the dynamic base).  A stage is
// [header | K codes | V codes | K norms | V norms | QJL words | gammas].
struct Layout {
    uint32_t ring, stage_bytes, k_off, v_off, kn_off, vn_off, z_off, gam_off;
    uint32_t qring, qh, qlo, sq, app, fac, merge, ml, bars, flags, total;
};

__host__ __device__ inline Layout layout(int kb, int vb, int nt, int stages, int m) {
    Layout L{};
    L.ring = LUT_BYTES;
    L.k_off = 16;
    L.v_off = L.k_off + CHUNK * 16 * kb;
    L.kn_off = L.v_off + CHUNK * 16 * vb;
    L.vn_off = L.kn_off + CHUNK * 2;
    L.z_off = L.vn_off + CHUNK * 2;
    L.gam_off = L.z_off + CHUNK * (m / 8);
    L.stage_bytes = L.gam_off + (m > 0 ? CHUNK * 2 : 0);
    L.qring = L.ring + stages * L.stage_bytes;        // 2 query slots
    L.qh = L.qring + 2 * QSLOT_BYTES;                  // fp16 [16][128], rounded q~
    L.qlo = L.qh + 16 * D * 2;                         // fp16 [16][128], q~ minus the rounded part
    L.sq = L.qlo + 16 * D * 2;                         // fp16 [16][64]
    L.app = L.sq + 16 * 64 * 2;                        // appended token: packed rows, norms, scratch
    L.fac = L.app + APP_BYTES;                         // float F1[16], F2[16]
    L.merge = L.fac + 32 * 4;                          // float [CW][8*nt][128]
    L.ml = L.merge + CW * 8 * nt * D * 4;              // float2 [CW][16]
    L.bars = L.ml + CW * 16 * 8;                       // u64 full[8], empty[8], qfull[2], qempty[2]
    L.flags = L.bars + 20 * 8;                         // int abort, last
    L.total = L.flags + 16;
    return L;
}

// Physical token (within a 16-token tile) of logical MMA row r.
__device__ __forceinline__ int tau_row(int r) { return (r & 8) + (r & 1) * 4 + ((r & 7) >> 1); }

struct Item {
    int unit, split, b, kv, s0, s1, len;
    bool bad;  // seq_len out of range: the sequence is treated as empty
};

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
        if (use > 0 && !ptx::mbar_wait_bounded(empty0 + 8 * slot, (use - 1) & 1, WAIT_LIMIT)) {
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
    int i = blockIdx.x;  // the first item of every block is static; later ones come from the counter
    while (ok) {
        if (i >= a.n_items) break;
        const Item w = item_of(a, i);
        const bool empty = w.s0 >= w.s1;
        if (!empty) {  // the item's queries, into the next query slot
            const int qs = qseq & 1;
            if (qseq >= 2 && !ptx::mbar_wait_bounded(qempty0 + 8 * qs, ((qseq - 2) >> 1) & 1, WAIT_LIMIT)) {
                fail();
                break;
            }
            const uint32_t qbytes = G * D * a.q_bytes;
            // the item holding a sequence's last token also brings the token's new key and value
            const bool app = a.append && w.s1 == w.len;
            const uint32_t rbytes = D * a.new_bytes;
            ptx::mbar_arrive_expect_tx(qfull0 + 8 * qs, qbytes + (app ? 2 * rbytes : 0u));
            ptx::bulk_copy_g2s(base + L.qring + qs * QSLOT_BYTES,
                               static_cast<const uint8_t*>(a.q) +
                                   (static_cast<size_t>(w.b) * a.hq + w.kv * G) * D * a.q_bytes,
                               qbytes, qfull0 + 8 * qs);
            if (app) {
                const size_t row = (static_cast<size_t>(w.b) * a.hkv + w.kv) * rbytes;
                ptx::bulk_copy_g2s(base + L.qring + qs * QSLOT_BYTES + Q_BYTES,
                                   static_cast<const uint8_t*>(a.k_new) + row, rbytes, qfull0 + 8 * qs);
                ptx::bulk_copy_g2s(base + L.qring + qs * QSLOT_BYTES + Q_BYTES + NEW_ROW,
                                   static_cast<const uint8_t*>(a.v_new) + row, rbytes, qfull0 + 8 * qs);
            }
            ++qseq;
        }
        int t0 = w.s0;
        do {
            uint32_t full;
            uint8_t* st;
            if (!claim(full, st)) break;
            const int n = empty ? 0 : min(CHUNK, w.s1 - t0);
            const int flags = (t0 == w.s0 ? F_FIRST : 0) | ((empty || t0 + CHUNK >= w.s1) ? F_LAST : 0) |
                              (empty ? F_EMPTY : 0);
            *reinterpret_cast<int4*>(st) = make_int4(i, t0, n, flags);
            const uint32_t dst = ptx::smem_addr(st);
            const size_t row = static_cast<size_t>(w.unit) * a.capacity + t0;
            if (n == 0) {
                ptx::mbar_arrive_expect_tx(full, 0);
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
            t0 += CHUNK;
        } while (!empty && t0 < w.s1);
        i = static_cast<int>(gridDim.x + atomicAdd(a.counters + a.units + C_ITEM, 1u));
    }
    if (ok) {  // end-of-work sentinel
        uint32_t full;
        uint8_t* st;
        if (claim(full, st)) {
            *reinterpret_cast<int4*>(st) = make_int4(-1, 0, 0, F_END);
            ptx::mbar_arrive_expect_tx(full, 0);
            ++seq;
        }
    }
    // every copy issued must have landed before the block may exit
    for (int j = max(0, seq - a.stages); j < seq; ++j)
        ptx::mbar_wait_bounded(full0 + 8 * (j % a.stages), (j / a.stages) & 1, WAIT_LIMIT);
    for (int j = max(0, qseq - 2); j < qseq; ++j) ptx::mbar_wait_bounded(qfull0 + 8 * (j & 1), (j >> 1) & 1, WAIT_LIMIT);
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

// Value fragments A[m-tile i][reg] of one 16-token tile for lane group g.
template <int VB>
__device__ __forceinline__ void value_fragments(uint32_t vst, uint32_t base, int g, int t, uint32_t laneoff,
                                                uint32_t (&A)[8][4]) {
    constexpr int VBV = 16 * VB;
    if constexpr (VB == 2) {
        // word g of physical tokens t, 4+t, 8+t, 12+t (logical k = 2t, 2t+1, 2t+8, 2t+9)
        const uint32_t w0 = ptx::lds32(vst + t * VBV + 4 * g);
        const uint32_t w1 = ptx::lds32(vst + (4 + t) * VBV + 4 * g);
        const uint32_t w2 = ptx::lds32(vst + (8 + t) * VBV + 4 * g);
        const uint32_t w3 = ptx::lds32(vst + (12 + t) * VBV + 4 * g);
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
            const int tok = 4 * k4 + t;
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

template <int KB, int VB, int NT, bool QJL>
struct Consumer {
    const Args& a;
    uint8_t* smem;
    const Layout& L;
    int tid, warp, lane, g, t;
    uint32_t base, laneoff;

    __device__ Consumer(const Args& a_, uint8_t* s_, const Layout& L_) : a(a_), smem(s_), L(L_) {
        tid = threadIdx.x;
        warp = tid >> 5;
        lane = tid & 31;
        g = lane >> 2;
        t = lane & 3;
        base = ptx::smem_addr(smem);
        laneoff = lane * 4;
    }

    __device__ bool aborted() const { return *reinterpret_cast<volatile int*>(smem + L.flags) != 0; }
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
    template <int BITS, bool SKETCH>
    __device__ void encode_new(const uint8_t* src, uint8_t* codes, uint16_t* norms, const float* bounds, size_t slot,
                               uint8_t* prow, uint16_t* pnorm, uint8_t* cbytes, float* rbuf) {
        float x[4];
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] = load_scalar(src, lane * 4 + e, a.new_dtype);
            ss = fmaf(x[e], x[e], ss);
            x[e] = flip_sign(x[e], sign_bit(a.signs, lane * 4 + e));
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
            reinterpret_cast<uint32_t*>(codes + slot * (16 * BITS))[lane] = word;
            reinterpret_cast<uint32_t*>(prow)[lane] = word;
        }
        if (lane == 0) {
            const uint16_t n16 = float_to_half_bits(n);
            norms[slot] = n16;
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
            uint8_t* pz = smem + L.app + 136;
            uint32_t* qjl = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.k_qjl) + slot * (a.m / 8));
            if (lane == 0) {
                const uint16_t g16 = float_to_half_bits(sqrtf(g2));
                const_cast<uint16_t*>(a.k_gamma)[slot] = g16;
                *reinterpret_cast<uint16_t*>(smem + L.app + 132) = g16;
                qjl[0] = z0;
                reinterpret_cast<uint32_t*>(pz)[0] = z0;
                if (a.m > 32) {
                    qjl[1] = z1;
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
                reinterpret_cast<uint32_t*>(st + L.k_off + p * (16 * KB))[lane] = reinterpret_cast<const uint32_t*>(ap)[lane];
            if (a.staged_norms && lane == 0) {
                reinterpret_cast<uint16_t*>(st + L.kn_off)[p] = *reinterpret_cast<const uint16_t*>(ap + 128);
                if constexpr (QJL) {
                    reinterpret_cast<uint16_t*>(st + L.gam_off)[p] = *reinterpret_cast<const uint16_t*>(ap + 132);
                    const int zb = a.m / 8;
                    for (int i = 0; i < zb / 4; ++i)
                        reinterpret_cast<uint32_t*>(st + L.z_off + p * zb)[i] = reinterpret_cast<const uint32_t*>(ap + 136)[i];
                }
            }
        } else if (warp == 1) {
            if (lane < 4 * VB)
                reinterpret_cast<uint32_t*>(st + L.v_off + p * (16 * VB))[lane] =
                    reinterpret_cast<const uint32_t*>(ap + 64)[lane];
            if (a.staged_norms && lane == 0)
                reinterpret_cast<uint16_t*>(st + L.vn_off)[p] = *reinterpret_cast<const uint16_t*>(ap + 130);
        }
        // the stage is refilled later by the copy engine: order these writes first
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }

    __device__ bool prologue(int qseq, const Item& w, bool app, uint32_t (&bq)[NT][8][4], uint32_t (&bz)[NT][4][2],
                             float (&f1)[NT][2], float (&f2)[NT][2]) {
        const uint32_t qfull = base + L.bars + 128 + 8 * (qseq & 1);
        if (!ptx::mbar_wait_bounded(qfull, (qseq >> 1) & 1, WAIT_LIMIT)) set_abort();
        ptx::named_barrier(1, NUM_CONSUMERS);
        if (aborted()) return false;
        const int G = a.group;
        const uint8_t* qsrc = smem + L.qring + (qseq & 1) * QSLOT_BYTES;
        __half* qh = reinterpret_cast<__half*>(smem + L.qh);
        __half* ql = reinterpret_cast<__half*>(smem + L.qlo);
        __half* sq = reinterpret_cast<__half*>(smem + L.sq);
        float* fac = reinterpret_cast<float*>(smem + L.fac);
        float* merge = reinterpret_cast<float*>(smem + L.merge);
        const float inv_sqrt_d = 0.08838834764831845f;
        for (int h = warp; h < NT * 8; h += CW) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (h < G) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    x[e] = flip_sign(load_scalar(qsrc, h * D + lane * 4 + e, a.q_dtype), sign_bit(a.signs, lane * 4 + e));
                fwht_registers(x);
                fwht_lanes<4, 32>(x, lane);
#pragma unroll
                for (int e = 0; e < 4; ++e) x[e] *= inv_sqrt_d;
            }
            float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
            amax = group_max<32>(amax);
            const float qmax = amax > 0.f ? amax : 1.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                // two fp16 terms: the scores keep about 22 bits of q~
                const float u = x[e] / qmax;
                const __half hi = __float2half_rn(u);
                qh[h * D + lane * 4 + e] = hi;
                ql[h * D + lane * 4 + e] = __float2half_rn(u - __half2float(hi));
            }
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
                sq[h * 64 + lane] = __float2half_rn(sv[0] / smax);
                sq[h * 64 + lane + 32] = __float2half_rn(sv[1] / smax);
            }
            if (lane == 0) {
                fac[h] = h < G ? a.sm_scale_log2 * qmax * a.inv_alpha_k : 0.f;
                fac[16 + h] = (QJL && h < G) ? a.sm_scale_log2 * 1.2533141373155003f / a.m * smax : 0.f;
            }
        }
        if (app && warp < 2) {
            const size_t slot = static_cast<size_t>(w.unit) * a.capacity + (w.len - 1);
            const uint8_t* rows = smem + L.qring + (qseq & 1) * QSLOT_BYTES + Q_BYTES;
            uint8_t* ap = smem + L.app;
            if (warp == 0)
                encode_new<KB, QJL>(rows, const_cast<uint8_t*>(a.k_codes), const_cast<uint16_t*>(a.k_norms), a.kbound,
                                    slot, ap, reinterpret_cast<uint16_t*>(ap + 128), ap + 256,
                                    reinterpret_cast<float*>(ap + 512));
            else
                encode_new<VB, false>(rows + NEW_ROW, const_cast<uint8_t*>(a.v_codes), const_cast<uint16_t*>(a.v_norms),
                                      a.vbound, slot, ap + 64, reinterpret_cast<uint16_t*>(ap + 130), ap + 384,
                                      reinterpret_cast<float*>(ap + 512));
        }
        ptx::named_barrier(1, NUM_CONSUMERS);
        if (tid == 0) ptx::mbar_arrive(base + L.bars + 144 + 8 * (qseq & 1));  // query slot free
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const __half* qrow = qh + (nt * 8 + g) * D + 32 * t;
            const __half* lrow = ql + (nt * 8 + g) * D + 32 * t;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                bq[nt][j][0] = *reinterpret_cast<const uint32_t*>(qrow + 4 * j);
                bq[nt][j][1] = *reinterpret_cast<const uint32_t*>(qrow + 4 * j + 2);
                bq[nt][j][2] = *reinterpret_cast<const uint32_t*>(lrow + 4 * j);
                bq[nt][j][3] = *reinterpret_cast<const uint32_t*>(lrow + 4 * j + 2);
            }
            if constexpr (QJL) {
                const __half* srow = sq + (nt * 8 + g) * 64 + 16 * t;
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
        return true;
    }

    // One chunk: this warp's two tiles.  MASK: the chunk may end before CHUNK tokens.
    template <bool MASK>
    __device__ void chunk(const Item& w, const uint8_t* st, int t0, const uint32_t (&bq)[NT][8][4],
                          const uint32_t (&bz)[NT][4][2], const float (&f1)[NT][2], const float (&f2)[NT][2],
                          SoftState<NT>& S) {
        constexpr int VBK = 16 * KB, VBV = 16 * VB;
        const int lb = 32 * warp;  // first chunk-local token of this warp
        if (MASK && t0 + lb >= w.s1) return;  // nothing of this warp's range is valid
        const uint32_t sbase = ptx::smem_addr(st);
        const int ra = tau_row(g), rb = tau_row(g + 8);
        const int zw = a.m / 16;
        const bool zt = 16 * t < a.m;
        const size_t unit_row = static_cast<size_t>(w.unit) * a.capacity;
        float s[TPW][NT][4];
        float vn[TPW][2];
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            const int la = lb + 16 * k + ra, lbb = lb + 16 * k + rb;  // chunk-local tokens of rows g, g+8
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
            const uint32_t kst = sbase + L.k_off + (lb + 16 * k) * VBK;
            uint32_t sa[4] = {0, 0, 0, 0}, sb[4] = {0, 0, 0, 0};
            if constexpr (KB == 4) {
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
                const uint32_t a0 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sa, j, 0, laneoff));
                const uint32_t a1 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sb, j, 0, laneoff));
                const uint32_t a2 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sa, j, 1, laneoff));
                const uint32_t a3 = ptx::lds32_imm<WINDOW>(key_lut_addr<KB>(sb, j, 1, laneoff));
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
            if (MASK && t0 + lb + 16 * k >= w.s1) break;  // warp-uniform
            float pv[NT][4];
            bool any_v = false;
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
                    if (pv[nt][0] < th0) pv[nt][0] = 0.f;
                    if (pv[nt][2] < th0) pv[nt][2] = 0.f;
                    if (pv[nt][1] < th1) pv[nt][1] = 0.f;
                    if (pv[nt][3] < th1) pv[nt][3] = 0.f;
                    any_v |= (pv[nt][0] + pv[nt][1] + pv[nt][2] + pv[nt][3]) > 0.f;
                }
            }
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
            value_fragments<VB>(sbase + L.v_off + (lb + 16 * k) * VBV, base, g, t, laneoff, A);
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    ptx::mma_16816(S.acc[nt][i], A[i][0], A[i][1], A[i][2], A[i][3], bv[nt][0], bv[nt][1]);
        }
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
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float* mw = merge + (warp * 8 * NT + nt * 8) * D;
                const int c_lo = 16 * g + 2 * i, c_hi = c_lo + 1;
                mw[(2 * t) * D + c_lo] = S.acc[nt][i][0] * unscale;
                mw[(2 * t + 1) * D + c_lo] = S.acc[nt][i][1] * unscale;
                mw[(2 * t) * D + c_hi] = S.acc[nt][i][2] * unscale;
                mw[(2 * t + 1) * D + c_hi] = S.acc[nt][i][3] * unscale;
            }
        ptx::named_barrier(1, NUM_CONSUMERS);
        const size_t pbase = (static_cast<size_t>(w.unit) * a.n_split + w.split) * G;
        for (int idx = tid; idx < G * D; idx += NUM_CONSUMERS) {
            const int h = idx / D, c = idx % D;
            float mx = -INFINITY;
#pragma unroll
            for (int ww = 0; ww < CW; ++ww)
                if (ml[ww * 16 + h].y > 0.f) mx = fmaxf(mx, ml[ww * 16 + h].x);
            float l = 0.f, s = 0.f;
            if (mx > -INFINITY) {
#pragma unroll
                for (int ww = 0; ww < CW; ++ww) {
                    const float2 v = ml[ww * 16 + h];
                    if (!(v.y > 0.f)) continue;
                    const float f = ptx::ex2(v.x - mx);
                    l = fmaf(v.y, f, l);
                    s = fmaf(merge[(ww * 8 * NT + h) * D + c], f, s);
                }
            }
            a.ws_acc[(pbase + h) * D + c] = s * a.inv_alpha_v;  // undo the centroid scale
            if (c == 0) a.ws_ml[pbase + h] = make_float2(mx, l);
        }
        __threadfence();
        ptx::named_barrier(1, NUM_CONSUMERS);
        if (tid == 0) *last_flag = atomicAdd(a.counters + w.unit, 1u) == static_cast<uint32_t>(a.n_split - 1);
        ptx::named_barrier(1, NUM_CONSUMERS);
        if (*last_flag) {
            __threadfence();
            // Merge the splits: one warp per head, lane = float4 column.  The
            // first batch of partial rows is requested before the split weights
            // 2^(m_s - M) / L are reduced, so both reads overlap; the weighted sum
            // runs in split order, so the result does not depend on timing.
            float* o_s = merge;           // [G][D]
            float* wts = merge + 16 * D;  // [n_split][G]
            const size_t ubase = static_cast<size_t>(w.unit) * a.n_split * G;
            const float4* src4 = reinterpret_cast<const float4*>(a.ws_acc + ubase * D);
            constexpr int PB = 16;  // splits per batch of loads
            for (int h = warp; h < G; h += CW) {
                float4 v[PB];
#pragma unroll
                for (int j = 0; j < PB; ++j)
                    v[j] = j < a.n_split ? __ldcg(src4 + (j * G + h) * (D / 4) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
                float mx = -INFINITY;
                for (int sp = lane; sp < a.n_split; sp += 32) {
                    const float2 m2 = __ldcg(a.ws_ml + ubase + sp * G + h);
                    if (m2.y > 0.f) mx = fmaxf(mx, m2.x);
                }
                mx = group_max<32>(mx);
                float l = 0.f;
                for (int sp = lane; sp < a.n_split; sp += 32) {
                    const float2 m2 = __ldcg(a.ws_ml + ubase + sp * G + h);
                    const float wgt = (m2.y > 0.f && mx > -INFINITY) ? ptx::ex2(m2.x - mx) : 0.f;
                    wts[sp * G + h] = wgt;
                    l = fmaf(m2.y, wgt, l);
                }
                l = group_sum<32>(l);
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                __syncwarp();
                float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int s0 = 0; s0 < a.n_split; s0 += PB) {
                    if (s0 > 0) {
#pragma unroll
                        for (int j = 0; j < PB; ++j)
                            v[j] = s0 + j < a.n_split ? __ldcg(src4 + ((s0 + j) * G + h) * (D / 4) + lane)
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int j = 0; j < PB; ++j) {
                        const float wgt = s0 + j < a.n_split ? wts[(s0 + j) * G + h] : 0.f;
                        acc4.x = fmaf(v[j].x, wgt, acc4.x);
                        acc4.y = fmaf(v[j].y, wgt, acc4.y);
                        acc4.z = fmaf(v[j].z, wgt, acc4.z);
                        acc4.w = fmaf(v[j].w, wgt, acc4.w);
                    }
                }
                *reinterpret_cast<float4*>(o_s + h * D + 4 * lane) =
                    make_float4(acc4.x * inv_l, acc4.y * inv_l, acc4.z * inv_l, acc4.w * inv_l);
            }
            ptx::named_barrier(1, NUM_CONSUMERS);
            const float inv_sqrt_d = 0.08838834764831845f;
            for (int h = warp; h < G; h += CW) {
                float x[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) x[e] = o_s[h * D + lane * 4 + e];
                fwht_registers(x);
                fwht_lanes<4, 32>(x, lane);
                float* dst = a.out + (static_cast<size_t>(w.b) * a.hq + w.kv * G + h) * D + lane * 4;
#pragma unroll
                for (int e = 0; e < 4; ++e) dst[e] = flip_sign(x[e] * inv_sqrt_d, sign_bit(a.signs, lane * 4 + e));
            }
            if (tid == 0) a.counters[w.unit] = 0;
        }
        ptx::named_barrier(1, NUM_CONSUMERS);
    }

    __device__ void run() {
        const uint32_t full0 = base + L.bars, empty0 = full0 + 64;
        uint32_t bq[NT][8][4];
        uint32_t bz[NT][4][2];
        float f1[NT][2], f2[NT][2];
        SoftState<NT> S;
        S.reset();
        Item w{};
        int seq = 0, qseq = 0;
        bool done_ok = false, app = false;
        while (true) {
            const int slot = seq % a.stages, use = seq / a.stages;
            if (!ptx::mbar_wait_bounded(full0 + 8 * slot, use & 1, WAIT_LIMIT)) set_abort();
            ptx::named_barrier(1, NUM_CONSUMERS);  // every consumer warp sees the same abort state
            if (aborted()) break;
            const uint8_t* st = smem + L.ring + slot * L.stage_bytes;
            const int4 hdr = *reinterpret_cast<const int4*>(st);
            if (hdr.w & F_END) {
                done_ok = true;
                break;
            }
            const bool empty = hdr.w & F_EMPTY;
            if (hdr.w & F_FIRST) {
                w = item_of(a, hdr.x);
                if (w.bad && a.err && w.split == 0 && w.kv == 0 && tid == 0) atomicOr(a.err, TQ_DEVERR_SEQLEN);
                S.reset();
                app = a.append && !empty && w.s1 == w.len;
                if (!empty) {
                    if (!prologue(qseq, w, app, bq, bz, f1, f2)) break;
                    ++qseq;
                }
            }
            if (app && (hdr.w & F_LAST)) {  // the stage holding the appended token
                patch_stage(const_cast<uint8_t*>(st), w.len - 1 - hdr.y);
                ptx::named_barrier(1, NUM_CONSUMERS);
            }
            if (!empty) {
                if (hdr.w & F_LAST) chunk<true>(w, st, hdr.y, bq, bz, f1, f2, S);
                else chunk<false>(w, st, hdr.y, bq, bz, f1, f2, S);
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty0 + 8 * slot);
            if (hdr.w & F_LAST) epilogue(w, S);
            ++seq;
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

template <int KB, int VB, int NT, bool QJL>
__global__ void __launch_bounds__(NUM_THREADS, 1) decode_mma_kernel(const __grid_constant__ Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const Layout L = layout(KB, VB, NT, a.stages, QJL ? a.m : 0);
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
        *reinterpret_cast<int*>(smem + L.flags) = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();  // mbarriers initialised
    if (threadIdx.x >= NUM_CONSUMERS) {
        if (threadIdx.x == NUM_CONSUMERS) {
            ptx::wait_prerequisites();  // the cache and queries may come from the previous kernel
            producer<KB, VB, QJL>(a, smem, L);
        }
        return;
    }
    // per-lane replicated centroid-pair tables, built while the first copies fly:
    // key pairs in bytes [0,128) of each 256-byte entry, value pairs (3- and
    // 4-bit values) in [128, 256)
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
    const __half* kc = reinterpret_cast<const __half*>(a.kcent);
    const __half* vc = reinterpret_cast<const __half*>(a.vcent);
    constexpr int nk = 1 << (2 * KB), nv = VB >= 3 ? 1 << (2 * VB) : 256;
    for (int idx = threadIdx.x; idx < (nk + nv) * 32; idx += NUM_CONSUMERS) {
        const int e = idx >> 5, r = idx & 31;
        if (e < nk) {
            const __half2 v = __halves2half2(kc[e & ((1 << KB) - 1)], kc[e >> KB]);
            lut[e * 64 + r] = *reinterpret_cast<const uint32_t*>(&v);
        } else if (VB >= 3) {
            const int ev = e - nk;
            const __half2 v = __halves2half2(vc[ev & ((1 << VB) - 1)], vc[ev >> VB]);
            lut[ev * 64 + 32 + r] = *reinterpret_cast<const uint32_t*>(&v);
        } else {
            // byte ev = (token a: two 2-bit codes) | (token b: two codes) << 4;
            // word 2*replica: first channel (a, b), word 2*replica + 1: second channel
            const int ev = e - nk, rep = r >> 1;
            const int ca = (r & 1) ? (ev >> 2) & 3 : ev & 3;
            const int cb = (r & 1) ? (ev >> 6) & 3 : (ev >> 4) & 3;
            const __half2 v = __halves2half2(vc[ca], vc[cb]);
            lut[ev * 64 + 32 + 2 * rep + (r & 1)] = *reinterpret_cast<const uint32_t*>(&v);
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
    Consumer<KB, VB, NT, QJL> c(a, smem, L);
    c.run();
}

template <int KB, int VB, int NT, bool QJL>
static cudaError_t launch_typed(const Args& a, int grid, size_t smem, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<KB, VB, NT, QJL>,
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
    e = cudaLaunchKernelEx(&cfg, decode_mma_kernel<KB, VB, NT, QJL>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int KB, int VB>
static cudaError_t launch_kv(const Args& a, int nt, bool qjl, int grid, size_t smem, cudaStream_t s) {
    if (nt == 1) return qjl ? launch_typed<KB, VB, 1, true>(a, grid, smem, s) : launch_typed<KB, VB, 1, false>(a, grid, smem, s);
    return qjl ? launch_typed<KB, VB, 2, true>(a, grid, smem, s) : launch_typed<KB, VB, 2, false>(a, grid, smem, s);
}

template <int KB>
static cudaError_t launch_k(const Args& a, int vb, int nt, bool qjl, int grid, size_t smem, cudaStream_t s) {
    switch (vb) {
        case 2: return launch_kv<KB, 2>(a, nt, qjl, grid, smem, s);
        case 3: return launch_kv<KB, 3>(a, nt, qjl, grid, smem, s);
        default: return launch_kv<KB, 4>(a, nt, qjl, grid, smem, s);
    }
}

}  // namespace mmadec

bool decode_mma_supported(const tq_params& p) {
    return p.head_dim == 128 && p.k_mode == TQ_MODE_TURBO && p.v_mode == TQ_MODE_TURBO &&
           p.num_q_heads / p.num_kv_heads <= 16 && p.qjl_dims <= 64;
}

static uint16_t half_bits(double v) {
    const __half h = __float2half_rn(static_cast<float>(v));
    return *reinterpret_cast<const uint16_t*>(&h);
}

cudaError_t launch_decode_mma(const tq_params& p, const tq_codebook* kcb, const tq_codebook* vcb, const tq_cache& c,
                              const void* q, int q_dtype, const int32_t* seq_lens, int max_len, float* out,
                              const DecodePlan& plan, char* ws, uint32_t* err, int num_sms, cudaStream_t stream,
                              const void* k_new, const void* v_new, int new_dtype) {
    using namespace mmadec;
    Args a{};
    a.append = k_new != nullptr;
    a.k_new = k_new;
    a.v_new = v_new;
    a.new_dtype = new_dtype;
    a.new_bytes = new_dtype == TQ_F32 ? 4 : 2;
    {
        const int hk = 1 << (p.k_bits - 1), hv = 1 << (p.v_bits - 1);
        for (int k = 0; k < 8; ++k) {
            a.kbound[k] = k < hk - 1 ? static_cast<float>(kcb->boundaries[hk + k]) : INFINITY;
            a.vbound[k] = k < hv - 1 ? static_cast<float>(vcb->boundaries[hv + k]) : INFINITY;
        }
        for (int j = 0; j < 16; ++j) a.kc32[j] = j < (1 << p.k_bits) ? static_cast<float>(kcb->centroids[j]) : 0.f;
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
    const double sd = std::sqrt(128.0);
    const double ak = kcb->fp16_scale > 0.0 ? kcb->fp16_scale : sd;
    const double av = vcb->fp16_scale > 0.0 ? vcb->fp16_scale : sd;
    a.inv_alpha_k = static_cast<float>(1.0 / ak);
    a.inv_alpha_v = static_cast<float>(1.0 / av);
    for (int j = 0; j < 16; ++j) {
        a.kcent[j] = j < (1 << p.k_bits) ? half_bits(kcb->centroids[j] * ak) : 0;
        a.vcent[j] = j < (1 << p.v_bits) ? half_bits(vcb->centroids[j] * av) : 0;
    }
    a.staged_norms = (c.capacity % 8) == 0;
    uint32_t words[8];
    rotation_sign_bits(p.seed, 128, words);
    for (int i = 0; i < 4; ++i) a.signs[i] = words[i];
    int reserved = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        static_cast<uint32_t>(reserved) != WINDOW)
        return cudaErrorNotSupported;
    const int nt = a.group <= 8 ? 1 : 2;
    const int kb = p.k_bits, vb = p.v_bits;
    // as many stages as fit in 227 KB next to the tables and the merge buffers
    const Layout fixed = layout(kb, vb, nt, 0, p.qjl_dims);
    int stages = static_cast<int>((232448u - fixed.total) / fixed.stage_bytes);
    if (stages > 8) stages = 8;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    a.stages = stages;
    const size_t smem = layout(kb, vb, nt, stages, p.qjl_dims).total;
    int grid = num_sms;
    if (grid > a.n_items) grid = a.n_items;
    const bool qjl = p.qjl_dims > 0;
    switch (kb) {
        case 2: return launch_k<2>(a, vb, nt, qjl, grid, smem, stream);
        case 3: return launch_k<3>(a, vb, nt, qjl, grid, smem, stream);
        default: return launch_k<4>(a, vb, nt, qjl, grid, smem, stream);
    }
}

}  // namespace tq
