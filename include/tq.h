/*
 * tq.h — C ABI of the TurboQuant KV-cache library for NVIDIA B200 (sm_100a).
 *
 * The library compresses attention keys and values online and computes
 * decode attention straight from the compressed cache.  Every entry point
 * takes plain pointers and sizes; device pointers are CUDA device memory
 * owned by the caller, host pointers are ordinary process memory.  The
 * library allocates no device memory and keeps no global state: all caches,
 * inputs, outputs and workspaces are provided by the caller.
 *
 * Pages the operations follow (cited by title and section):
 *   [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命"
 *   [tqai]    "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术"
 *   [fwht]    "TurboQuant：用Rust核心与FWHT预处理实现LLM推理的4-bit KV缓存量化"
 *   [google]  "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！"
 *
 * Conventions
 * -----------
 * - Every function returns a tq_status.  Arguments are validated on the host
 *   before anything is launched; an invalid call launches nothing and
 *   returns TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_ALIGNMENT or
 *   TQ_ERR_CAPACITY.  No C++ exception crosses the ABI.
 * - Device work is enqueued asynchronously on `stream` (a cudaStream_t
 *   passed as void*; NULL means the legacy default stream).  A failed launch
 *   returns TQ_ERR_CUDA.
 * - Conditions only the device can see (an append position or sequence
 *   length out of range) are never trapped: the kernel skips the offending
 *   work and ORs a TQ_DEVERR_* bit into the caller's `d_error` word (device
 *   uint32, may be NULL to disable reporting).  Read it with
 *   tq_read_device_error.
 * - Functions are reentrant and thread-safe; calls on different streams may
 *   run concurrently as long as they do not write the same cache slots.
 * - fp16 values are IEEE binary16 bit patterns stored as uint16_t.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_ABI_VERSION 5

typedef enum tq_status {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, inconsistent params      */
    TQ_ERR_UNSUPPORTED = 2,  /* valid in principle but not built (e.g. d = 512)   */
    TQ_ERR_CAPACITY = 3,     /* workspace or cache too small for the request      */
    TQ_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed              */
    TQ_ERR_TIMEOUT = 5,      /* a bounded host wait ran out                       */
    TQ_ERR_DEVICE = 6,       /* the device error word is non-zero                 */
    TQ_ERR_ALIGNMENT = 7     /* a pointer is not 16-byte aligned                  */
} tq_status;

/* Storage mode of one side (K or V) of a cache. */
typedef enum tq_mode {
    TQ_MODE_TURBO = 0,  /* rotation + fp16 norm + Lloyd-Max b-bit codes         */
    TQ_MODE_INT8 = 1    /* per-vector absmax int8 ("q8_0"-style boundary layers) */
} tq_mode;

/* Element type of raw K/V inputs and queries. */
typedef enum tq_dtype { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* Bits ORed into the caller's device error word. */
#define TQ_DEVERR_POSITION 0x1u /* append: positions[b] < 0 or > capacity - n_new  */
#define TQ_DEVERR_SEQLEN 0x2u   /* decode: seq_lens[b] < 1, > capacity or > max_seq_len */
#define TQ_DEVERR_TIMEOUT 0x4u  /* decode: a bounded wait inside a kernel ran out (about 1 s);
                                   the output is not valid and the workspace must be zeroed again */
#define TQ_DEVERR_PAGE 0x8u     /* paged cache: a block-table entry a kernel needed lies outside
                                   the pool; that access was skipped */

/*
 * Lloyd-Max codebook for one (head_dim, bits) pair.  [tqai] section
 * "TurboQuant的核心创新：极坐标量化与随机旋转": after the rotation each
 * coordinate of the unit direction follows the density
 *     f_d(x) = C_d (1 - x^2)^((d-3)/2),  |x| <= 1,
 * and the optimal scalar quantiser for it is computed once, from the
 * density alone.  centroids[0 .. 2^bits-1] ascend; boundaries[j] is the
 * midpoint of centroids j and j+1.  Plain data, owned by the caller.
 */
typedef struct tq_codebook {
    int32_t head_dim;
    int32_t bits;
    double centroids[16];
    double boundaries[15];
    /* Scale the tensor-core kernels apply to the centroids before rounding
     * them to fp16 (their operand type); tq_codebook_init picks the value in
     * [8, 16) that minimises the largest relative rounding error of the table.
     * A representation detail, not part of the method: 0 selects sqrt(d). */
    double fp16_scale;
} tq_codebook;

/*
 * Cache configuration.  One tq_params describes one attention layer.
 *   head_dim            d; 64, 128 or 256.
 *   num_q_heads         Hq; a multiple of num_kv_heads.  Query head h reads
 *                       kv head h / (Hq / Hkv) (contiguous GQA groups); the
 *                       group size Hq / Hkv must be at most 16.
 *   num_kv_heads        Hkv >= 1.
 *   k_mode, v_mode      tq_mode of each side.  Asymmetric K/V bit widths:
 *                       [inferrs] "三个反直觉的关键发现", [tqai] "配置策略与质量权衡".
 *   k_bits, v_bits      2, 3 or 4 for TQ_MODE_TURBO; ignored for INT8.
 *   qjl_dims            m, the QJL sketch size for K ([google] "第二步：QJL"):
 *                       0 disables it; otherwise a multiple of 32 not above d,
 *                       and only with k_mode == TQ_MODE_TURBO.
 *   seed                selects the rotation signs and the QJL matrix
 *                       (tq_rotation_signs, tq_qjl_matrix).  Keys, values and
 *                       queries of one layer share the rotation.
 *   sm_scale            softmax scale; 0 selects 1/sqrt(d).
 *   sparse_v_threshold  Sparse V ([inferrs] "Sparse V：速度加成"): 0 disables;
 *                       otherwise positions whose softmax weight is provably
 *                       below it may be left out of the V sum (see
 *                       tq_decode_attention).
 *   flags               TQ_PARAM_* bits; 0 for none.
 *
 * TQ_PARAM_PREFETCH_EARLY: the caller promises that the kernel launched just
 * before a decode call on the same stream does not write this layer's cache
 * (nor does anything else still running).  Decode kernels are launched as
 * programmatic dependents of that kernel; with this flag they start streaming
 * the cache before it has finished (queries, new rows, lengths and every
 * write still wait for it), which hides most of their start-up behind the
 * previous layer's tail.  Without the flag nothing is read early.
 */
#define TQ_PARAM_PREFETCH_EARLY 0x1u

typedef struct tq_params {
    int32_t head_dim;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t k_mode;
    int32_t v_mode;
    int32_t k_bits;
    int32_t v_bits;
    int32_t qjl_dims;
    uint64_t seed;
    float sm_scale;
    float sparse_v_threshold;
    uint32_t flags;
    uint32_t reserved;  /* 0 */
} tq_params;

/*
 * Device-resident compressed cache of one layer (all pointers are device
 * memory owned by the caller, each 16-byte aligned).  Layout is
 * structure-of-arrays, per (batch entry, kv head), token-contiguous:
 *   k_codes   [batch][Hkv][capacity][kb]   kb = d*k_bits/8 bytes (TURBO) or d (INT8)
 *   k_norms   [batch][Hkv][capacity]       fp16 norm (TURBO) or fp16 scale (INT8)
 *   k_qjl     [batch][Hkv][capacity][m/8]  QJL sign bits (NULL when qjl_dims == 0)
 *   k_gamma   [batch][Hkv][capacity]       fp16 residual norm (NULL when qjl_dims == 0)
 *   v_codes, v_norms                       as for K
 *   qjl_matrix [m][d] fp32, row-major      the sketch S (NULL when qjl_dims == 0)
 * A capacity that is a multiple of 8 lets the decode kernels move the
 * norms, QJL words and gammas with the codes in their bulk copies; with any
 * other capacity they read them from global memory in the inner loop.
 * Codes of one vector are one LSB-first bitstream: code i occupies bits
 * [b*i, b*i+b), bit k of the stream is bit k%8 of byte k/8, so 3-bit codes
 * cross byte boundaries ([inferrs] "压缩格式对比", turbo2/3/4).  INT8 codes
 * are the d signed bytes of the vector.
 */
typedef struct tq_cache {
    int32_t batch;
    int32_t capacity;
    uint8_t* k_codes;
    uint16_t* k_norms;
    uint8_t* k_qjl;
    uint16_t* k_gamma;
    uint8_t* v_codes;
    uint16_t* v_norms;
    const float* qjl_matrix;
} tq_cache;

/* Human-readable name of a status. Never NULL. */
const char* tq_status_string(tq_status status);

/* TQ_ABI_VERSION of the loaded library. */
int32_t tq_abi_version(void);

/*
 * Host only.  Solve the Lloyd-Max conditions for f_d at `bits` bits
 * (1 <= bits <= 4, 3 <= head_dim <= 4096) in fp64 and write the table to
 * *out (caller-owned).  Deterministic: the result depends only on
 * (head_dim, bits).  [tqai] "TurboQuant的核心创新" (precomputed,
 * data-independent codebook).
 */
tq_status tq_codebook_init(int32_t head_dim, int32_t bits, tq_codebook* out);

/*
 * Host only.  The rotation of a layer is y = H diag(s) x / sqrt(d) with H
 * the Sylvester-order Walsh-Hadamard matrix ([inferrs] "核心技术", [fwht]
 * "2. 快速Walsh-Hadamard变换（FWHT）预处理").  Writes s (+1.0 / -1.0) for
 * `seed` into out[0 .. head_dim-1] (caller-owned host array).  s_i is -1
 * when bit 63 of the i-th SplitMix64 output from state `seed` is set.
 */
tq_status tq_rotation_signs(uint64_t seed, int32_t head_dim, float* out);

/*
 * Host only.  Writes the QJL sketch S (m x head_dim, row-major, iid N(0,1)
 * rounded to fp32) for `seed` into out (caller-owned host array of
 * m*head_dim floats).  The caller copies it to device memory and sets
 * tq_cache.qjl_matrix.  Entries come from Box-Muller pairs on the
 * SplitMix64 stream with state seed ^ 0x5155414E544A4C00.
 */
tq_status tq_qjl_matrix(uint64_t seed, int32_t m, int32_t head_dim, float* out);

/*
 * Host only.  Byte sizes of the six cache arrays, in tq_cache order
 * (k_codes, k_norms, k_qjl, k_gamma, v_codes, v_norms), for `batch` entries
 * of `capacity` tokens.  Unused arrays report 0.
 */
tq_status tq_cache_bytes(const tq_params* params, int32_t batch, int32_t capacity, size_t sizes_out[6]);

/*
 * Host only.  Bytes of device workspace tq_decode_attention needs for
 * `batch` sequences of at most `max_seq_len` tokens on any device.  The
 * workspace must be zero-filled once before its first use; every call that
 * completes leaves it ready for the next one, whatever its batch and lengths,
 * provided every call on it passes the same workspace_bytes (the size fixes
 * where its counters live).
 */
tq_status tq_decode_workspace_bytes(const tq_params* params, int32_t batch, int32_t max_seq_len,
                                    size_t* bytes_out);

/*
 * Quantise n_new new tokens per sequence and append them to the cache.
 * [tqai] "TurboQuant的核心创新" (rotation, fp16 norm, Lloyd-Max codes),
 * [google] "第二步：QJL" (1-bit residual sketch on K, when qjl_dims > 0),
 * [inferrs] "三个反直觉的关键发现" item 3 (INT8 boundary layers).
 *   k_new, v_new   device, [batch][n_new][Hkv][d] in `dtype`, 16-byte aligned.
 *   n_new          >= 1.
 *   d_positions    device int32 [batch]: sequence b's tokens go to cache
 *                  slots positions[b] .. positions[b]+n_new-1.
 *   kcb, vcb       codebooks matching (d, k_bits) and (d, v_bits); ignored
 *                  (may be NULL) for an INT8 side.
 * TURBO: norm n = ||x|| (fp32) stored as fp16 (round to nearest even);
 * direction y = R(x)/n; code_i = number of boundaries below y_i; with QJL,
 * r = y - c[code], gamma = ||r|| as fp16, sign bits of S r (1 when >= 0).
 * INT8: scale = fp16(absmax/127), q_i = rint(x_i * fp32(1/scale)) clamped
 * to [-127, 127].  A sequence whose position is out of range is skipped and
 * sets TQ_DEVERR_POSITION.
 */
tq_status tq_quantize_append(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                             const void* k_new, const void* v_new, tq_dtype dtype, int32_t n_new,
                             const int32_t* d_positions, const tq_cache* cache, uint32_t* d_error,
                             void* stream);

/*
 * Reconstruct cache slots [start, start+count) of sequence b as fp32:
 *   d_k_out, d_v_out  device, [count][Hkv][d] fp32 (either may be NULL).
 * TURBO: x_hat = n16 * R^-1(c[code] + gamma16 sqrt(pi/2)/m S^T(2z-1)) (the
 * QJL term only for K with qjl_dims > 0).  INT8: x_hat = scale16 * q.
 */
tq_status tq_dequantize(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                        const tq_cache* cache, int32_t b, int32_t start, int32_t count, float* d_k_out,
                        float* d_v_out, void* stream);

/*
 * One decode-attention step read straight from the compressed cache.
 * [google] "再看速度" (attention from 4-bit TurboQuant keys), [inferrs]
 * "Sparse V：速度加成".  For every batch entry b and query head h, with kv
 * head h / (Hq/Hkv) and L = seq_lens[b]:
 *     s_i = sm_scale * <q, k_hat_i>,  p = softmax(s_0 .. s_{L-1}),
 *     out = sum_i p_i v_hat_i
 * where k_hat, v_hat are the reconstructions tq_dequantize defines.  The
 * kernels never form k_hat: the query is rotated once, scores are
 * n_k * <R q, c[code]> (+ the QJL term), the V sum runs in the rotated
 * domain and one inverse rotation ends it.  The token axis is split across
 * thread blocks and the partial results are merged by log-sum-exp.
 *   d_q            device, [batch][Hq][d] in q_dtype.
 *   d_seq_lens     device int32 [batch], each in [1, min(capacity, max_seq_len)].
 *   max_seq_len    host upper bound on seq_lens (sizes the token split).
 *   d_out          device, [batch][Hq][d] fp32.
 *   d_workspace    device scratch of at least tq_decode_workspace_bytes
 *                  bytes (16-byte aligned), zero-filled before its first use
 *                  (its front holds per-(sequence, kv head) split counters
 *                  that each call returns to zero).  Calls sharing a
 *                  workspace pass the same workspace_bytes and must not
 *                  overlap on the device.
 * Sparse V (sparse_v_threshold = tau > 0): position i is dropped from the V
 * sum of head h only when exp(s_i - m)/l < tau for running softmax
 * statistics m, l over a subset of the positions that includes i; since
 * the full denominator is at least l e^m, every dropped position has exact
 * weight p_i < tau.  Dropped positions stay in the denominator.  Which
 * positions are dropped depends on the launch configuration.
 *   d_skip_mask    device uint32 [batch][Hq][(max_seq_len + 31) / 32], 4-byte
 *                  aligned, zero-filled by the caller, or NULL.  With tau > 0
 *                  the kernels set bit i % 32 of word i / 32 of row (b, h)
 *                  for every position i the gate dropped from head h's V sum
 *                  ([inferrs] "Sparse V：速度加成": the skipped low-weight V
 *                  positions); nothing else is written.  Ignored when tau = 0.
 * An out-of-range seq_len sets TQ_DEVERR_SEQLEN and yields zeros for b.
 */
tq_status tq_decode_attention(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                              const void* d_q, tq_dtype q_dtype, const tq_cache* cache,
                              const int32_t* d_seq_lens, int32_t max_seq_len, float* d_out,
                              void* d_workspace, size_t workspace_bytes, uint32_t* d_skip_mask,
                              uint32_t* d_error, void* stream);

/*
 * One decode step of a layer in one call: append the step's new token of
 * every sequence to the cache, then tq_decode_attention over the cache that
 * includes it ([tqai] "TurboQuant的核心创新" for the encoding, [google]
 * "再看速度" for the attention; the pages run the two one after the other).
 *   k_new, v_new  device, [batch][1][Hkv][d] in kv_dtype, 16-byte aligned.
 *   d_seq_lens    lengths AFTER the append: sequence b's new token goes to
 *                 slot seq_lens[b] - 1 and attention covers seq_lens[b]
 *                 tokens.
 *   Other arguments as for tq_decode_attention (same workspace and skip-mask
 *   rules).
 * The new token is encoded exactly as tq_quantize_append encodes it (the
 * cache afterwards holds what tq_quantize_append would have written, up to
 * codes within the boundary window).  On the tensor-core path (d = 128;
 * turbo or int8 K; turbo V, or int8 V beside int8 K; up to 16 query heads
 * per kv head, except 16 fp32 queries per kv head on an all-int8 layer) this
 * is one kernel: the block that owns a sequence's
 * last token split encodes the token while the cache streams in.  Other
 * configurations run tq_quantize_append's kernel and then the attention
 * kernels.  A seq_len outside [1, capacity] skips that sequence's append and
 * sets TQ_DEVERR_SEQLEN (or TQ_DEVERR_POSITION on the two-kernel path).
 */
tq_status tq_append_decode_attention(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                     const void* k_new, const void* v_new, tq_dtype kv_dtype, const void* d_q,
                                     tq_dtype q_dtype, const tq_cache* cache, const int32_t* d_seq_lens,
                                     int32_t max_seq_len, float* d_out, void* d_workspace, size_t workspace_bytes,
                                     uint32_t* d_skip_mask, uint32_t* d_error, void* stream);

/*
 * Chunked prefill from the compressed cache ([google] table "M5 Max 128GB
 * 上的實測" and [inferrs] table "性能表现" measure prefill over TurboQuant
 * caches): append n_new tokens of every sequence to the cache exactly as
 * tq_quantize_append does (slots positions[b] .. positions[b] + n_new - 1),
 * then attend causally with their queries: query j of sequence b attends to
 * cache positions 0 .. positions[b] + j (itself included), the result of a
 * decode step over positions[b] + j + 1 tokens.
 *   k_new, v_new  device, [batch][n_new][Hkv][d] in kv_dtype, 16-byte aligned.
 *   d_q           device, [batch][n_new][Hq][d] in q_dtype.
 *   d_positions   device int32 [batch]: the chunk's first slot per sequence.
 *   d_out         device, [batch][n_new][Hq][d] fp32.
 * Supported: d = 128, TURBO keys and values (2, 3 or 4 bits), no QJL
 * sketch, at most 16 query heads per kv head; other configurations return
 * TQ_ERR_UNSUPPORTED before any launch, as do 4-bit keys on a device whose
 * reserved shared memory per block is not 1 KB (the key table's lookups
 * carry its shared-window address; B200 reserves 1 KB).  The products Q K~^T and P V~ run on
 * the tcgen05 tensor cores (fp16 operands, fp32 accumulation in tensor
 * memory), 128 query rows (tokens x heads of a kv head's group) per block.
 * A position out of range sets TQ_DEVERR_POSITION; that sequence gets no
 * append and zero outputs.  Kernels on `stream`: the append, the attention,
 * then (when units are split, below) the merge.
 *   d_workspace, workspace_bytes  device scratch of at least
 *                 tq_prefill_workspace_bytes(params, cache->batch, n_new)
 *                 bytes (on the current device), 16-byte aligned; its
 *                 contents need no initial value and mean nothing after the
 *                 call.  Calls that overlap on one workspace race.  When that
 *                 size is 0 the workspace may be NULL.
 * Work distribution: the units of 128 query rows (the (sequence, kv head)
 * pairs times the chunk's query blocks) are spread over one block per SM,
 * each block taking an equal share of the units' key tiles, so a unit's
 * tiles may be split between blocks; each piece of a split unit leaves its
 * unnormalised rows with their softmax maximum and sum in the workspace,
 * and the merge kernel combines them (log-sum-exp) into the unit's output.
 * With more than 4096 units, or when units x ceil(capacity / 64) reaches
 * 2^31 (the tile sequence is counted in 32 bits), each block takes one
 * whole unit, the workspace is not used and no merge runs.  After
 * TQ_DEVERR_TIMEOUT the outputs are not valid.  TQ_ERR_CAPACITY when
 * workspace_bytes is too small.
 */
tq_status tq_prefill_attention(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                               const void* k_new, const void* v_new, tq_dtype kv_dtype, const void* d_q,
                               tq_dtype q_dtype, int32_t n_new, const int32_t* d_positions, const tq_cache* cache,
                               float* d_out, void* d_workspace, size_t workspace_bytes, uint32_t* d_error,
                               void* stream);

/*
 * Bytes of prefill workspace for `batch` sequences and chunks of n_new
 * tokens on the current device (its SM count decides): the tile schedule
 * (one word per unit, plus one) and two partial outputs of 128 rows per
 * block; 0 when the call does not need one.  TQ_ERR_UNSUPPORTED for configurations tq_prefill_attention
 * does not take.
 */
tq_status tq_prefill_workspace_bytes(const tq_params* params, int32_t batch, int32_t n_new, size_t* bytes);

/*
 * Paged cache.  [inferrs] manages its compressed cache with PagedAttention
 * ("二、inferrs：TurboQuant 轻量推理服务器"); the pages give no page format,
 * so this one follows the usual block-table scheme.  The pool is a tq_cache whose
 * `batch` counts physical blocks and whose `capacity` is the block size in
 * tokens, a multiple of 16: every array keeps the layout above,
 * [block][Hkv][block_size][...].  Token t of sequence b lives in block
 * d_table[b * max_blocks + t / block_size], row t % block_size.
 *   d_table     device int32 [batch][max_blocks]; entries of the blocks
 *               below a sequence's length (and those an append writes)
 *               must lie in [0, pool.batch).  A kernel that meets an entry
 *               outside the pool skips the access and sets TQ_DEVERR_PAGE
 *               (the decode may read entries past a sequence's length and
 *               ignores the ones outside the pool).
 *   batch       sequences.
 *   max_blocks  entries per sequence: a sequence holds at most
 *               max_blocks * block_size tokens.
 */
typedef struct tq_block_table {
    const int32_t* d_table;
    int32_t batch;
    int32_t max_blocks;
} tq_block_table;

/*
 * tq_quantize_append on a paged cache: positions count tokens of each
 * sequence (0 .. max_blocks * block_size - n_new) as before, and every token
 * goes to the block the table names.
 */
tq_status tq_quantize_append_paged(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                   const void* k_new, const void* v_new, tq_dtype dtype, int32_t n_new,
                                   const int32_t* d_positions, const tq_cache* pool, const tq_block_table* table,
                                   uint32_t* d_error, void* stream);

/*
 * tq_decode_attention and tq_append_decode_attention on a paged cache.  The
 * workspace is sized by tq_decode_workspace_bytes(params, table->batch,
 * max_seq_len).  Only the tensor-core path reads a paged cache (d = 128 and
 * the modes it takes, see tq_append_decode_attention); other configurations
 * return TQ_ERR_UNSUPPORTED.  The kernel copies each chunk of a sequence
 * block by block, so blocks of 64 or more tokens keep the copies large.
 * TQ_PARAM_PREFETCH_EARLY is ignored here.
 */
tq_status tq_decode_attention_paged(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                    const void* d_q, tq_dtype q_dtype, const tq_cache* pool,
                                    const tq_block_table* table, const int32_t* d_seq_lens, int32_t max_seq_len,
                                    float* d_out, void* d_workspace, size_t workspace_bytes,
                                    uint32_t* d_skip_mask, uint32_t* d_error, void* stream);
tq_status tq_append_decode_attention_paged(const tq_params* params, const tq_codebook* kcb,
                                           const tq_codebook* vcb, const void* k_new, const void* v_new,
                                           tq_dtype kv_dtype, const void* d_q, tq_dtype q_dtype,
                                           const tq_cache* pool, const tq_block_table* table,
                                           const int32_t* d_seq_lens, int32_t max_seq_len, float* d_out,
                                           void* d_workspace, size_t workspace_bytes, uint32_t* d_skip_mask,
                                           uint32_t* d_error, void* stream);

/* Bytes of the library's own decode scratch on each device. */
#define TQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)16 << 20)

/*
 * tq_decode_attention without a caller workspace; the pages have no
 * counterpart (the method says nothing about where scratch lives).  It is
 * for callers that must not allocate device memory when they decode: the
 * split partials and counters go to one fixed 16 MiB device array of the
 * library (TQ_DECODE_STATIC_SCRATCH_BYTES per device), and the call
 * allocates nothing.  Arguments as for tq_decode_attention.
 *   - Returns TQ_ERR_CAPACITY, before any device work, when the call needs
 *     more scratch than the array holds (the launch plan for batch and
 *     max_seq_len on the current device decides; a workspace bound from
 *     tq_decode_workspace_bytes at or below the limit always fits).
 *   - Every call looks up the array's address (a host query that allocates
 *     nothing) and queues, on `stream` ahead of its kernels, a zero fill of
 *     the counter words it uses ((batch * Hkv + 2) * 4 bytes at the front of
 *     the array).  Only those words must be zero when a call starts, so a
 *     call that ended with TQ_DEVERR_TIMEOUT leaves nothing behind that
 *     harms the next one.
 *   - The array is shared by all calls on the device and keeps the last
 *     call's partials.  Calls that overlap on the device (other streams,
 *     other threads) race on it: serialise them.
 */
tq_status tq_decode_attention_static(const tq_params* params, const tq_codebook* kcb, const tq_codebook* vcb,
                                     const void* d_q, tq_dtype q_dtype, const tq_cache* cache,
                                     const int32_t* d_seq_lens, int32_t max_seq_len, float* d_out,
                                     uint32_t* d_error, void* stream);

/*
 * Fill the counter region at the front of the static array (every counter
 * word any tq_decode_attention_static call can use) with the byte `value`,
 * queued on `stream`; allocates nothing.  0 resets the counters outright (for
 * a caller that wants the array in a known state, e.g. after an error); any
 * other value leaves them as an interrupted call could, which the next static
 * call's own zero fill repairs.  Returns TQ_ERR_CUDA if the fill cannot be
 * queued.  Races with static calls in flight on other streams.
 */
tq_status tq_decode_static_fill(uint8_t value, void* stream);

/*
 * Copy the device error word to *out after the work queued on `stream` so
 * far, waiting at most timeout_ms milliseconds (polling, never blocking
 * indefinitely).  Returns TQ_ERR_TIMEOUT when the wait runs out,
 * TQ_ERR_DEVICE when the word is non-zero (still written to *out), TQ_OK
 * otherwise.
 */
tq_status tq_read_device_error(const uint32_t* d_error, uint32_t* out, void* stream, int32_t timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
