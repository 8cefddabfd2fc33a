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
//   online softmax, acc = sum_i p_i ||v_i|| c[code_i] (rotated domain), then a
//   log-sum-exp merge of the token splits and one inverse rotation.
//
// How (one persistent thread block per SM):
//  * a producer warp streams the packed K and V codes of 128-token chunks into
//    a ring of shared-memory stages with 1-D bulk async copies (TMA engine, no
//    multicast), completion tracked by mbarriers; eight consumer warps take one
//    16-token tile of every chunk;
//  * the dequantised tiles of a GQA group form real dense products, so both
//    contractions run on the tensor cores with warp-level m16n8k16 fp16 MMA
//    (fp32 accumulate):  S^T[16 tok x 8 heads] = K~[16 x 128] Q~^T and
//    O^T[128 x 8 heads] += V~^T[128 x 16 tok] P^T.  The A operands are built
//    in registers straight from the codes: a 256-entry (per-lane replicated)
//    shared-memory table maps one byte of 4-bit key codes to the fp16 pair of
//    centroids, and a register byte-permute table maps 2-bit value codes.
//    Because sum_c q~_c c[code_c] does not depend on the order of c, channels
//    are assigned to fragment slots so that each lane's 16-byte load of a key
//    row feeds its fragments directly (the query uses the same order).  Tokens
//    of a tile are permuted the same way on both sides (tau below) so that the
//    value words each lane needs are bank-conflict free.
//  * the score fragment is turned into the second MMA's operand with one
//    movmatrix transpose per 8x8 block; no shared-memory round trip.
//  * split results are merged by the last block to finish a (sequence, kv
//    head), found with an atomic counter (no spin-wait), which also applies the
//    inverse rotation and writes the output.
//  Every wait on an mbarrier is bounded (about a second); a wait that runs out
//  sets TQ_DEVERR_TIMEOUT and the block leaves after draining its copies.

#include <cuda_runtime.h>

#include <cmath>

#include "device_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace tq {
namespace mmadec {

constexpr int D = 128;
constexpr int CW = 8;                        // consumer warps
constexpr int NUM_THREADS = (CW + 1) * 32;   // + one producer warp
constexpr int NUM_CONSUMERS = CW * 32;
constexpr int CHUNK = CW * 16;               // tokens per stage
constexpr uint32_t LUT_BYTES = 65536;        // 256 entries x 256 B
constexpr long long WAIT_LIMIT = 2000000000ll;  // clock cycles (~1 s)
constexpr float LOG2E = 1.4426950408889634f;

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
    uint32_t* counters;
    float* out;
    uint32_t* err;
    int q_dtype, batch, hq, hkv, group, capacity, n_split, split_len, max_len, n_items, stages, m;
    float sm_scale_log2;  // sm_scale * log2(e)
    float tau;
    float inv_alpha_k, inv_alpha_v;  // 1 / (centroid scale applied before fp16 rounding)
    int staged_norms;     // capacity % 8 == 0: norms (and QJL words) ride in the TMA stages
    uint32_t signs[4];
    uint16_t kcent[16];  // fp16 bits of alpha_k * key centroid
    uint16_t vcent[16];  // fp16 bits of alpha_v * value centroid
};

// Shared-memory map (offsets in bytes from the dynamic base).
struct Layout {
    uint32_t ring, stage_bytes, kbytes_stage, vbytes_stage, kn_off, vn_off, z_off, gam_off;
    uint32_t qh, sq, fac, merge, ml, bars, flags, total;
};

// One stage: [K codes | V codes | K norms | V norms | QJL words | gammas] for
// CHUNK tokens, every part 16-byte aligned.
__host__ __device__ inline Layout layout(int kb, int vb, int nt, int stages, int m) {
    Layout L{};
    const uint32_t vbk = 16 * kb, vbv = 16 * vb;
    L.ring = LUT_BYTES;
    L.kbytes_stage = CHUNK * vbk;
    L.vbytes_stage = CHUNK * vbv;
    L.kn_off = L.kbytes_stage + L.vbytes_stage;
    L.vn_off = L.kn_off + CHUNK * 2;
    L.z_off = L.vn_off + CHUNK * 2;
    L.gam_off = L.z_off + CHUNK * (m / 8);
    L.stage_bytes = L.gam_off + (m > 0 ? CHUNK * 2 : 0);
    L.qh = L.ring + stages * L.stage_bytes;          // fp16 [16][128]
    L.sq = L.qh + 16 * D * 2;                          // fp16 [16][64]
    L.fac = L.sq + 16 * 64 * 2;                        // float F1[16], F2[16]
    L.merge = L.fac + 32 * 4;                          // float [CW][8*nt][128]
    L.ml = L.merge + CW * 8 * nt * D * 4;              // float2 [CW][16]
    L.bars = L.ml + CW * 16 * 8;                       // u64 full[8], empty[8]
    L.flags = L.bars + 16 * 8;                         // int abort, last
    L.total = L.flags + 16;
    return L;
}

// Physical token (within a 16-token tile) of logical MMA row r.
__device__ __forceinline__ int tau_row(int r) { return (r & 8) + (r & 1) * 4 + ((r & 7) >> 1); }

struct Item {
    int unit, split, b, kv, s0, s1;
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
    return it;
}

// ------------------------------------------------------------------ producer
template <int KB, int VB, bool QJL>
__device__ void producer(const Args& a, uint8_t* smem, const Layout& L) {
    const uint32_t base = ptx::smem_addr(smem);
    const uint32_t full0 = base + L.bars, empty0 = full0 + 64;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flags);
    constexpr int VBK = 16 * KB, VBV = 16 * VB;
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < a.n_items && ok; item += gridDim.x) {
        const Item w = item_of(a, item);
        for (int t0 = w.s0; t0 < w.s1; t0 += CHUNK) {
            const int slot = it % a.stages, use = it / a.stages;
            if (use > 0 && !ptx::mbar_wait_bounded(empty0 + 8 * slot, (use - 1) & 1, WAIT_LIMIT)) {
                if (a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
                *abort_flag = 1;
                ok = false;
                break;
            }
            if (*abort_flag) {
                ok = false;
                break;
            }
            int n = min(CHUNK, w.s1 - t0);
            const size_t row = static_cast<size_t>(w.unit) * a.capacity + t0;
            const uint32_t full = full0 + 8 * slot;
            const uint32_t dst = base + L.ring + slot * L.stage_bytes;
            if (a.staged_norms) {
                // capacity and t0 are multiples of 8, so rounding n up to 8 tokens
                // stays inside the cache and keeps every 2-byte array 16-byte sized
                n = (n + 7) & ~7;
                const int zb = QJL ? a.m / 8 : 0;
                ptx::mbar_arrive_expect_tx(full, n * (VBK + VBV + 4 + (QJL ? zb + 2 : 0)));
                ptx::bulk_copy_g2s(dst, a.k_codes + row * VBK, n * VBK, full);
                ptx::bulk_copy_g2s(dst + L.kbytes_stage, a.v_codes + row * VBV, n * VBV, full);
                ptx::bulk_copy_g2s(dst + L.kn_off, a.k_norms + row, n * 2, full);
                ptx::bulk_copy_g2s(dst + L.vn_off, a.v_norms + row, n * 2, full);
                if constexpr (QJL) {
                    ptx::bulk_copy_g2s(dst + L.z_off, a.k_qjl + row * zb, n * zb, full);
                    ptx::bulk_copy_g2s(dst + L.gam_off, a.k_gamma + row, n * 2, full);
                }
            } else {
                ptx::mbar_arrive_expect_tx(full, n * (VBK + VBV));
                ptx::bulk_copy_g2s(dst, a.k_codes + row * VBK, n * VBK, full);
                ptx::bulk_copy_g2s(dst + L.kbytes_stage, a.v_codes + row * VBV, n * VBV, full);
            }
            ++it;
        }
    }
    // every copy issued must have landed before the block may exit
    for (int j = max(0, it - a.stages); j < it; ++j)
        ptx::mbar_wait_bounded(full0 + 8 * (j % a.stages), (j / a.stages) & 1, WAIT_LIMIT);
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

template <int KB, int VB, int NT, bool QJL>
__device__ void consumer(const Args& a, uint8_t* smem, const Layout& L) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const uint32_t base = ptx::smem_addr(smem);
    const uint32_t full0 = base + L.bars, empty0 = full0 + 64;
    const uint32_t laneoff = lane * 4;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flags);
    __half* qh = reinterpret_cast<__half*>(smem + L.qh);
    __half* sq = reinterpret_cast<__half*>(smem + L.sq);
    float* fac = reinterpret_cast<float*>(smem + L.fac);
    float* merge = reinterpret_cast<float*>(smem + L.merge);
    float2* ml = reinterpret_cast<float2*>(smem + L.ml);
    int* last_flag = reinterpret_cast<int*>(smem + L.flags + 4);
    constexpr int VBK = 16 * KB, VBV = 16 * VB;
    const int G = a.group;
    const float inv_sqrt_d = 0.08838834764831845f;

    // value centroid pairs for the 2-bit byte-permute table
    const uint32_t vl0 = a.vcent[0] | (static_cast<uint32_t>(a.vcent[1]) << 16);
    const uint32_t vl1 = a.vcent[2] | (static_cast<uint32_t>(a.vcent[3]) << 16);

    int it = 0;
    for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
        const Item w = item_of(a, item);
        if (w.bad && a.err && w.split == 0 && w.kv == 0 && tid == 0) atomicOr(a.err, TQ_DEVERR_SEQLEN);

        // ---- rotated queries of the kv head (fp16, scaled to max |q~| = 1)
        for (int h = warp; h < NT * 8; h += CW) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (h < G) {
                const size_t off = (static_cast<size_t>(w.b) * a.hq + w.kv * G + h) * D + lane * 4;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    x[e] = flip_sign(load_scalar(a.q, off + e, a.q_dtype), sign_bit(a.signs, lane * 4 + e));
                fwht_registers(x);
                fwht_lanes<4, 32>(x, lane);
#pragma unroll
                for (int e = 0; e < 4; ++e) x[e] *= inv_sqrt_d;
            }
            float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
            amax = group_max<32>(amax);
            const float qmax = amax > 0.f ? amax : 1.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) qh[h * D + lane * 4 + e] = __float2half_rn(x[e] / qmax);
            float smax = 1.f;
            if constexpr (QJL) {
                // S q~ for sketch rows lane and lane + 32 (m <= 64); q~ staged in
                // the merge buffer, which is free until the end of the item
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
                float sm = group_max<32>(fmaxf(fabsf(sv[0]), fabsf(sv[1])));
                smax = sm > 0.f ? sm : 1.f;
                sq[h * 64 + lane] = __float2half_rn(sv[0] / smax);
                sq[h * 64 + lane + 32] = __float2half_rn(sv[1] / smax);
            }
            if (lane == 0) {
                fac[h] = h < G ? a.sm_scale_log2 * qmax * a.inv_alpha_k : 0.f;
                fac[16 + h] = (QJL && h < G) ? a.sm_scale_log2 * 1.2533141373155003f / a.m * smax : 0.f;
            }
        }
        ptx::named_barrier(1, NUM_CONSUMERS);

        // ---- per-lane operand fragments of the queries
        uint32_t bq[NT][8][2];
        uint32_t bz[NT][4][2];
        float f1[NT][2], f2[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const __half* qrow = qh + (nt * 8 + g) * D + 32 * t;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                bq[nt][j][0] = *reinterpret_cast<const uint32_t*>(qrow + 4 * j);
                bq[nt][j][1] = *reinterpret_cast<const uint32_t*>(qrow + 4 * j + 2);
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

        // ---- stream the split
        float m_run[NT][2], l_run[NT][2], acc[NT][8][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m_run[nt][0] = m_run[nt][1] = -INFINITY;
            l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[nt][i][0] = acc[nt][i][1] = acc[nt][i][2] = acc[nt][i][3] = 0.f;
        }
        float vscale = 0.f;  // power of two keeping p*||v|| inside fp16 range; 0 = not set yet
        const int ra = tau_row(g), rb = tau_row(g + 8);
        const size_t unit_row = static_cast<size_t>(w.unit) * a.capacity;
        for (int t0 = w.s0; t0 < w.s1; t0 += CHUNK) {
            const int slot = it % a.stages, use = it / a.stages;
            const int tile0 = t0 + 16 * warp;
            const int tok_a = tile0 + ra, tok_b = tile0 + rb;
            const bool va = tok_a < w.s1, vb = tok_b < w.s1;
            const bool zt = 16 * t < a.m;  // lanes past the sketch size carry no QJL bits
            const int zw = a.m / 16;       // 16-bit QJL words per token
            float kna = 0.f, knb = 0.f, vna = 0.f, vnb = 0.f, ga = 0.f, gb = 0.f;
            uint32_t za = 0, zb = 0;
            if (!a.staged_norms) {  // straight from global memory, issued before the wait
                kna = va ? half_bits_to_float(a.k_norms[unit_row + tok_a]) : 0.f;
                knb = vb ? half_bits_to_float(a.k_norms[unit_row + tok_b]) : 0.f;
                vna = va ? half_bits_to_float(a.v_norms[unit_row + tok_a]) : 0.f;
                vnb = vb ? half_bits_to_float(a.v_norms[unit_row + tok_b]) : 0.f;
                if constexpr (QJL) {
                    const uint16_t* zr = reinterpret_cast<const uint16_t*>(a.k_qjl);
                    za = (va && zt) ? zr[(unit_row + tok_a) * zw + t] : 0u;
                    zb = (vb && zt) ? zr[(unit_row + tok_b) * zw + t] : 0u;
                    ga = va ? half_bits_to_float(a.k_gamma[unit_row + tok_a]) : 0.f;
                    gb = vb ? half_bits_to_float(a.k_gamma[unit_row + tok_b]) : 0.f;
                }
            }
            if (*abort_flag || !ptx::mbar_wait_bounded(full0 + 8 * slot, use & 1, WAIT_LIMIT)) {
                if (!*abort_flag && a.err) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
                *abort_flag = 1;
                break;  // every consumer warp still reaches the barrier below
            }
            if (a.staged_norms) {
                const uint8_t* st = smem + L.ring + slot * L.stage_bytes;
                const int la = 16 * warp + ra, lb = 16 * warp + rb;
                const __half* skn = reinterpret_cast<const __half*>(st + L.kn_off);
                const __half* svn = reinterpret_cast<const __half*>(st + L.vn_off);
                kna = va ? __half2float(skn[la]) : 0.f;
                knb = vb ? __half2float(skn[lb]) : 0.f;
                vna = va ? __half2float(svn[la]) : 0.f;
                vnb = vb ? __half2float(svn[lb]) : 0.f;
                if constexpr (QJL) {
                    const uint16_t* sz = reinterpret_cast<const uint16_t*>(st + L.z_off);
                    const __half* sg = reinterpret_cast<const __half*>(st + L.gam_off);
                    za = (va && zt) ? sz[la * zw + t] : 0u;
                    zb = (vb && zt) ? sz[lb * zw + t] : 0u;
                    ga = va ? __half2float(sg[la]) : 0.f;
                    gb = vb ? __half2float(sg[lb]) : 0.f;
                }
            }
            if (tile0 < w.s1) {
                const uint32_t kst = base + L.ring + slot * L.stage_bytes + (16 * warp) * VBK;
                const uint32_t vst = base + L.ring + slot * L.stage_bytes + L.kbytes_stage + (16 * warp) * VBV;
                // ---- keys: 16 bytes (KB words) of rows tau(g) and tau(g+8)
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
                float cs[NT][4], cs2[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) cs[nt][e] = cs2[nt][e] = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t a0 = ptx::lds32(base + key_lut_addr<KB>(sa, j, 0, laneoff));
                    const uint32_t a1 = ptx::lds32(base + key_lut_addr<KB>(sb, j, 0, laneoff));
                    const uint32_t a2 = ptx::lds32(base + key_lut_addr<KB>(sa, j, 1, laneoff));
                    const uint32_t a3 = ptx::lds32(base + key_lut_addr<KB>(sb, j, 1, laneoff));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (j & 1) ptx::mma_16816(cs2[nt], a0, a1, a2, a3, bq[nt][j][0], bq[nt][j][1]);
                        else ptx::mma_16816(cs[nt], a0, a1, a2, a3, bq[nt][j][0], bq[nt][j][1]);
                    }
                }
                float cz[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) cz[nt][0] = cz[nt][1] = cz[nt][2] = cz[nt][3] = 0.f;
                if constexpr (QJL) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // +-1 pairs from sign bits (bit set -> +1)
                        const uint32_t xa = za >> (4 * j), xb = zb >> (4 * j);
                        const uint32_t a0 = 0xBC00BC00u ^ ((xa & 1u) << 15) ^ ((xa & 2u) << 30);
                        const uint32_t a2 = 0xBC00BC00u ^ ((xa & 4u) << 13) ^ ((xa & 8u) << 28);
                        const uint32_t a1 = 0xBC00BC00u ^ ((xb & 1u) << 15) ^ ((xb & 2u) << 30);
                        const uint32_t a3 = 0xBC00BC00u ^ ((xb & 4u) << 13) ^ ((xb & 8u) << 28);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) ptx::mma_16816(cz[nt], a0, a1, a2, a3, bz[nt][j][0], bz[nt][j][1]);
                    }
                }
                // ---- scores (log2 domain), online softmax
                float s[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float kn = e < 2 ? kna : knb;
                        const float gm = e < 2 ? ga : gb;
                        float v = (cs[nt][e] + cs2[nt][e]) * f1[nt][e & 1];
                        if constexpr (QJL) v = fmaf(gm * cz[nt][e], f2[nt][e & 1], v);
                        s[nt][e] = (e < 2 ? va : vb) ? v * kn : -INFINITY;
                    }
                }
                float pv[NT][4];
                bool any_v = false;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float mx0 = fmaxf(s[nt][0], s[nt][2]), mx1 = fmaxf(s[nt][1], s[nt][3]);
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, o));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, o));
                    }
                    const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
                    const float c0 = ptx::ex2(m_run[nt][0] - mn0), c1 = ptx::ex2(m_run[nt][1] - mn1);
                    m_run[nt][0] = mn0;
                    m_run[nt][1] = mn1;
                    const float p0 = ptx::ex2(s[nt][0] - mn0), p1 = ptx::ex2(s[nt][1] - mn1);
                    const float p2 = ptx::ex2(s[nt][2] - mn0), p3 = ptx::ex2(s[nt][3] - mn1);
                    l_run[nt][0] = fmaf(l_run[nt][0], c0, p0 + p2);
                    l_run[nt][1] = fmaf(l_run[nt][1], c1, p1 + p3);
                    if (c0 != 1.f || c1 != 1.f) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            acc[nt][i][0] *= c0;
                            acc[nt][i][2] *= c0;
                            acc[nt][i][1] *= c1;
                            acc[nt][i][3] *= c1;
                        }
                    }
                    pv[nt][0] = p0;
                    pv[nt][1] = p1;
                    pv[nt][2] = p2;
                    pv[nt][3] = p3;
                    if (a.tau > 0.f) {
                        // Sparse V: the exact denominator (relative to m_run) is at least
                        // 1 (the token that set the running max) and at least this lane's
                        // partial sum, so p / max(1, l) bounds the exact weight from above
                        const float t0v = a.tau * fmaxf(1.f, l_run[nt][0]);
                        const float t1v = a.tau * fmaxf(1.f, l_run[nt][1]);
                        if (p0 < t0v) pv[nt][0] = 0.f;
                        if (p2 < t0v) pv[nt][2] = 0.f;
                        if (p1 < t1v) pv[nt][1] = 0.f;
                        if (p3 < t1v) pv[nt][3] = 0.f;
                    }
                    any_v |= (pv[nt][0] + pv[nt][1] + pv[nt][2] + pv[nt][3]) > 0.f;
                }
                // keep p * ||v|| * vscale inside fp16 range (power-of-two rescale)
                float vmax = fmaxf(vna, vnb);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(kFullMask, vmax, o));
                if (vscale == 0.f) {
                    vscale = vmax > 0.f ? exp2f(8.0f - ceilf(log2f(vmax))) : 0.f;
                } else if (vmax * vscale > 16384.f) {
                    const float shrink = exp2f(8.0f - ceilf(log2f(vmax * vscale)));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 8; ++i)
#pragma unroll
                            for (int e = 0; e < 4; ++e) acc[nt][i][e] *= shrink;
                    vscale *= shrink;
                }
                if (__any_sync(kFullMask, any_v) && vscale > 0.f) {
                    const float wa = vna * vscale, wb = vnb * vscale;
                    uint32_t bv[NT][2];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        bv[nt][0] = ptx::movmatrix_trans(ptx::pack_half2(pv[nt][0] * wa, pv[nt][1] * wa));
                        bv[nt][1] = ptx::movmatrix_trans(ptx::pack_half2(pv[nt][2] * wb, pv[nt][3] * wb));
                    }
                    // ---- values: word(s) of lane group g from physical tokens t, 4+t, 8+t, 12+t
                    uint32_t A[8][4];
                    if constexpr (VB == 2) {
                        const uint32_t w0 = ptx::lds32(vst + (t) * VBV + 4 * g);
                        const uint32_t w1 = ptx::lds32(vst + (4 + t) * VBV + 4 * g);
                        const uint32_t w2 = ptx::lds32(vst + (8 + t) * VBV + 4 * g);
                        const uint32_t w3 = ptx::lds32(vst + (12 + t) * VBV + 4 * g);
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const uint32_t wa0 = half ? w2 : w0, wb0 = half ? w3 : w1;
                            const uint32_t P = __byte_perm(wa0, wb0, 0x5140), Q = __byte_perm(wa0, wb0, 0x7362);
#pragma unroll
                            for (int src = 0; src < 2; ++src) {
                                const uint32_t x = src ? Q : P;
#pragma unroll
                                for (int sh = 0; sh < 8; sh += 2) {
                                    const uint32_t sel = ((x >> sh) & 0x03030303u) * 0x22u + 0x10101010u;
                                    const int f = (sh >> 1) & 1, hb = sh >> 2;
                                    A[2 * (2 * src) + hb][2 * half + f] = __byte_perm(vl0, vl1, sel);
                                    A[2 * (2 * src + 1) + hb][2 * half + f] = __byte_perm(vl0, vl1, sel >> 16);
                                }
                            }
                        }
                    } else {
                        // 16 * VB bits per lane group and token (2*VB bytes at byte 2*VB*g),
                        // realigned to two words; codes read through the value table
                        uint32_t seg[4][2];
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int tok = 4 * k4 + t;  // physical tokens t, 4+t, 8+t, 12+t
                            const uint32_t byte_off = 2 * VB * g;  // 16*VB bits = 2*VB bytes per group
                            const uint32_t wbase = byte_off >> 2, wsh = (byte_off & 3) * 8;
                            const uint32_t lo = ptx::lds32(vst + tok * VBV + 4 * wbase);
                            const uint32_t hi = (4 * wbase + 4 < VBV) ? ptx::lds32(vst + tok * VBV + 4 * wbase + 4) : 0u;
                            const uint32_t hi2 = (4 * wbase + 8 < VBV) ? ptx::lds32(vst + tok * VBV + 4 * wbase + 8) : 0u;
                            seg[k4][0] = __funnelshift_r(lo, hi, wsh);
                            seg[k4][1] = __funnelshift_r(hi, hi2, wsh);
                        }
                        constexpr uint32_t vm = (1u << VB) - 1u;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
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
                                    const uint32_t idx = cx | (cy << VB);
                                    A[i][2 * half + f] = ptx::lds32(base + ((idx << 8) | 128u | laneoff));
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            ptx::mma_16816(acc[nt][i], A[i][0], A[i][1], A[i][2], A[i][3], bv[nt][0], bv[nt][1]);
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty0 + 8 * slot);
            ++it;
        }
        // ---- merge the eight warps of the block
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float l = l_run[nt][h];
                l += __shfl_xor_sync(kFullMask, l, 4);
                l += __shfl_xor_sync(kFullMask, l, 8);
                l += __shfl_xor_sync(kFullMask, l, 16);
                if (g == 0) ml[warp * 16 + nt * 8 + 2 * t + h] = make_float2(m_run[nt][h], l);
            }
        const float unscale = vscale > 0.f ? 1.0f / vscale : 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float* mw = merge + (warp * 8 * NT + nt * 8) * D;
                const int c_lo = 16 * g + 2 * i, c_hi = c_lo + 1;
                mw[(2 * t) * D + c_lo] = acc[nt][i][0] * unscale;
                mw[(2 * t + 1) * D + c_lo] = acc[nt][i][1] * unscale;
                mw[(2 * t) * D + c_hi] = acc[nt][i][2] * unscale;
                mw[(2 * t + 1) * D + c_hi] = acc[nt][i][3] * unscale;
            }
        ptx::named_barrier(1, NUM_CONSUMERS);
        if (*abort_flag) return;  // read after the barrier: every consumer leaves together
        const size_t pbase = (static_cast<size_t>(w.unit) * a.n_split + w.split) * G;
        for (int idx = tid; idx < G * D; idx += NUM_CONSUMERS) {
            const int h = idx / D, c = idx % D;
            float mx = -INFINITY;
#pragma unroll
            for (int ww = 0; ww < CW; ++ww) mx = fmaxf(mx, ml[ww * 16 + h].x);
            float l = 0.f, s = 0.f;
            if (mx > -INFINITY) {
#pragma unroll
                for (int ww = 0; ww < CW; ++ww) {
                    const float2 v = ml[ww * 16 + h];
                    if (v.x == -INFINITY) continue;
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
            // ---- last block of this (sequence, kv head): merge the splits.
            // Split weights 2^(m_s - M) / L per (split, head) go to shared memory
            // first (one warp per head), then every output channel is a weighted
            // sum of coalesced partial rows.
            float* o_s = merge;             // [G][D]
            float* wts = merge + 16 * D;    // [n_split][G]
            const size_t ubase = static_cast<size_t>(w.unit) * a.n_split * G;
            for (int h = warp; h < G; h += CW) {
                float mx = -INFINITY;
                for (int sp = lane; sp < a.n_split; sp += 32) {
                    const float2 v = __ldcg(a.ws_ml + ubase + sp * G + h);
                    if (v.y > 0.f) mx = fmaxf(mx, v.x);
                }
                mx = group_max<32>(mx);
                float l = 0.f;
                for (int sp = lane; sp < a.n_split; sp += 32) {
                    const float2 v = __ldcg(a.ws_ml + ubase + sp * G + h);
                    const float wgt = (v.y > 0.f && mx > -INFINITY) ? ptx::ex2(v.x - mx) : 0.f;
                    wts[sp * G + h] = wgt;
                    l = fmaf(v.y, wgt, l);
                }
                l = group_sum<32>(l);
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                __syncwarp();
                for (int sp = lane; sp < a.n_split; sp += 32) wts[sp * G + h] *= inv_l;
            }
            ptx::named_barrier(1, NUM_CONSUMERS);
            for (int idx = tid; idx < G * D; idx += NUM_CONSUMERS) {
                const int h = idx / D, c = idx % D;
                const float* src = a.ws_acc + (ubase + h) * D + c;
                float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
                int sp = 0;
                for (; sp + 4 <= a.n_split; sp += 4) {
                    s0 = fmaf(__ldcg(src + static_cast<size_t>(sp) * G * D), wts[sp * G + h], s0);
                    s1 = fmaf(__ldcg(src + static_cast<size_t>(sp + 1) * G * D), wts[(sp + 1) * G + h], s1);
                    s2 = fmaf(__ldcg(src + static_cast<size_t>(sp + 2) * G * D), wts[(sp + 2) * G + h], s2);
                    s3 = fmaf(__ldcg(src + static_cast<size_t>(sp + 3) * G * D), wts[(sp + 3) * G + h], s3);
                }
                for (; sp < a.n_split; ++sp) s0 = fmaf(__ldcg(src + static_cast<size_t>(sp) * G * D), wts[sp * G + h], s0);
                o_s[h * D + c] = (s0 + s1) + (s2 + s3);
            }
            ptx::named_barrier(1, NUM_CONSUMERS);
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
}

template <int KB, int VB, int NT, bool QJL>
__global__ void __launch_bounds__(NUM_THREADS, 1) decode_mma_kernel(const __grid_constant__ Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const Layout L = layout(KB, VB, NT, a.stages, QJL ? a.m : 0);
    // per-lane replicated centroid-pair tables: key pairs in bytes [0,128) of
    // each 256-byte entry, value pairs (3- and 4-bit values) in [128, 256)
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
    const __half* kc = reinterpret_cast<const __half*>(a.kcent);
    const __half* vc = reinterpret_cast<const __half*>(a.vcent);
    constexpr int nk = 1 << (2 * KB), nv = VB >= 3 ? 1 << (2 * VB) : 0;
    for (int idx = threadIdx.x; idx < (nk + nv) * 32; idx += NUM_THREADS) {
        const int e = idx >> 5, r = idx & 31;
        if (e < nk) {
            const __half2 v = __halves2half2(kc[e & ((1 << KB) - 1)], kc[e >> KB]);
            lut[e * 64 + r] = *reinterpret_cast<const uint32_t*>(&v);
        } else {
            const int ev = e - nk;
            const __half2 v = __halves2half2(vc[ev & ((1 << VB) - 1)], vc[ev >> VB]);
            lut[ev * 64 + 32 + r] = *reinterpret_cast<const uint32_t*>(&v);
        }
    }
    if (threadIdx.x == 0) {
        const uint32_t bars = ptx::smem_addr(smem + L.bars);
        for (int s = 0; s < a.stages; ++s) {
            ptx::mbar_init(bars + 8 * s, 1);
            ptx::mbar_init(bars + 64 + 8 * s, CW);
        }
        *reinterpret_cast<int*>(smem + L.flags) = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x >= NUM_CONSUMERS) {
        if (threadIdx.x == NUM_CONSUMERS) producer<KB, VB, QJL>(a, smem, L);
    } else {
        consumer<KB, VB, NT, QJL>(a, smem, L);
    }
}

template <int KB, int VB, int NT, bool QJL>
static cudaError_t launch_typed(const Args& a, int grid, size_t smem, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<KB, VB, NT, QJL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    decode_mma_kernel<KB, VB, NT, QJL><<<grid, NUM_THREADS, smem, stream>>>(a);
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
                              const DecodePlan& plan, char* ws, uint32_t* err, int num_sms, cudaStream_t stream) {
    using namespace mmadec;
    Args a{};
    a.k_codes = c.k_codes;
    a.v_codes = c.v_codes;
    a.k_norms = c.k_norms;
    a.v_norms = c.v_norms;
    a.k_qjl = c.k_qjl;
    a.k_gamma = c.k_gamma;
    a.sketch = c.qjl_matrix;
    a.q = q;
    a.q_dtype = q_dtype;
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
    a.n_items = c.batch * p.num_kv_heads * plan.n_split;
    a.m = p.qjl_dims;
    const float sm = p.sm_scale > 0.0f ? p.sm_scale : 1.0f / std::sqrt(128.0f);
    a.sm_scale_log2 = sm * LOG2E;
    a.tau = p.sparse_v_threshold;
    uint32_t words[8];
    rotation_sign_bits(p.seed, 128, words);
    for (int i = 0; i < 4; ++i) a.signs[i] = words[i];
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
    const int nt = a.group <= 8 ? 1 : 2;
    const int kb = p.k_bits, vb = p.v_bits;
    // as many stages as fit in 227 KB next to the table and the merge buffers
    const Layout fixed = layout(kb, vb, nt, 0, p.qjl_dims);
    const uint32_t stage = fixed.stage_bytes;
    int stages = static_cast<int>((232448u - fixed.total) / stage);
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
