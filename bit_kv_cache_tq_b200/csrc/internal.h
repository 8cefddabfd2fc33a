// Internal declarations shared by the host code and the kernel launchers.
#pragma once

#include <cstddef>
#include <cstdint>

#include "tq.h"

namespace tq {

// Decode split plan: the token axis of every (sequence, kv head) is cut into
// n_split ranges of split_len tokens (the last one may be shorter or empty).
// Workspace layout: the counter region comes first and its size depends only
// on the workspace size, so counters sit at the same addresses whatever the
// batch and lengths of a call; partial results follow it.
struct DecodePlan {
    int n_split = 1;
    int split_len = 0;
    size_t off_counters = 0;  // uint32 per (b, kv head): splits finished; then kGlobalCounters
    size_t off_ml = 0;        // float2 (m, l) per (b, hq, split)
    size_t off_acc = 0;       // float acc[d] per (b, hq, split)
    size_t bytes = 0;         // end of the partials
};

// Thread blocks aimed at per SM when choosing the split count.
constexpr int kBlocksPerSm = 2;
// Smallest token range worth a separate split.
constexpr int kMinSplitTokens = 256;
// Most splits per (sequence, kv head); bounds the merge scratch in shared memory.
constexpr int kMaxSplits = 384;
// Work-distribution counters after the per-(sequence, kv head) ones.
constexpr int kGlobalCounters = 2;
// Token granularity of split boundaries.
constexpr int kSplitAlign = 64;
// Fewest partial bytes one (sequence, kv head) takes: one split of one query
// head, (m, l) and acc[d] with d >= 64, is 8 + 4 d >= 264 bytes.  A workspace
// of W bytes therefore never serves more than W / kMinUnitBytes of them.
constexpr size_t kMinUnitBytes = 256;

// A paged cache seen by the kernels: table == nullptr means a contiguous
// cache.  Token t of sequence b, kv head h is row
// (table[b * max_blocks + t / block_size] * Hkv + h) * block_size + t % block_size.
struct PageMap {
    const int32_t* table = nullptr;
    int batch = 0, max_blocks = 0, block_size = 0, num_blocks = 0;
};

tq_status validate_params(const tq_params* p);
tq_status validate_codebook(const tq_codebook* cb, int head_dim, int bits);
tq_status validate_cache(const tq_params& p, const tq_cache* c);
// A pool and block table (block size a multiple of 16); fills *pm.
tq_status validate_pages(const tq_params& p, const tq_cache* pool, const tq_block_table* table, PageMap* pm);
bool aligned16(const void* ptr);
// Bytes of one stored vector: d*bits/8 (TURBO) or d (INT8).
int vector_bytes(int mode, int bits, int head_dim);
// Bytes of the counter region at the front of a workspace of this size.
size_t counter_region_bytes(size_t workspace_bytes);
// general_kernel: the plan is for the general split kernel (not the
// tensor-core decode kernel).
DecodePlan plan_decode(const tq_params& p, int batch, int max_seq_len, int num_sms, size_t workspace_bytes,
                       bool general_kernel);
// Tensor-core decode path (decode_mma.cu): d = 128; TURBO or INT8 K; TURBO V,
// or INT8 V beside INT8 K.
bool decode_mma_supported(const tq_params& p);
// SM count of the current CUDA device (0 when it cannot be queried).
int num_sms_current();
// Centroid scale in [8, 16) minimising the largest relative fp16 rounding error.
double best_fp16_scale(const double* c, int n);
// tq_quantize_append; with pos_from_lens, d_positions holds each sequence's
// length after the append and the new tokens go to its last n_new slots.
// pm: a paged cache (cache is then the pool), or nullptr.
tq_status quantize_append_impl(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                               const void* k_new, const void* v_new, int dtype, int32_t n_new,
                               const int32_t* d_positions, bool pos_from_lens, const tq_cache* cache,
                               uint32_t* d_error, void* stream, const PageMap* pm = nullptr);
// Rotation signs as a bit mask: bit i set <=> s_i = -1.
void rotation_sign_bits(uint64_t seed, int head_dim, uint32_t words[8]);

}  // namespace tq
