// Host-side part of the TurboQuant library: codebooks, the random numbers of
// the method, sizes, validation and status strings.  No CUDA calls here.
//
// Pages (by title): [tqai] "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术",
// [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命",
// [google] "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！".

#include <cmath>
#include <cstring>

#include "internal.h"

namespace tq {

// ---------------------------------------------------------------- codebook
//
// [tqai] section "TurboQuant的核心创新": the rotated unit-vector coordinate X
// has density f_d(x) = C_d (1-x^2)^((d-3)/2); equivalently (1+X)/2 follows
// Beta(a, a) with a = (d-1)/2.  Its CDF is therefore the regularised
// incomplete beta function I_{(1+x)/2}(a, a), evaluated here by the
// continued fraction of DLMF 8.17.22 with the modified Lentz method
// (Lentz 1976; Thompson & Barnett 1986).  The centroid numerator has the
// closed form C_d [(1-u^2)^a - (1-v^2)^a] / (d-1) over a cell (u, v).

namespace {

double log_beta(double a, double b) { return std::lgamma(a) + std::lgamma(b) - std::lgamma(a + b); }

// Continued-fraction part of I_z(a, b); converges fast for z < (a+1)/(a+b+2).
double beta_continued_fraction(double a, double b, double z) {
    const double tiny = 1e-300;
    double c = 1.0;
    double dd = 1.0 - (a + b) * z / (a + 1.0);
    if (std::fabs(dd) < tiny) dd = tiny;
    dd = 1.0 / dd;
    double h = dd;
    for (int k = 1; k <= 20000; ++k) {
        const double k2 = 2.0 * k;
        // even term d_{2k} = k (b - k) z / ((a + 2k - 1)(a + 2k))
        double num = k * (b - k) * z / ((a + k2 - 1.0) * (a + k2));
        dd = 1.0 + num * dd;
        if (std::fabs(dd) < tiny) dd = tiny;
        c = 1.0 + num / c;
        if (std::fabs(c) < tiny) c = tiny;
        dd = 1.0 / dd;
        h *= dd * c;
        // odd term d_{2k+1} = -(a + k)(a + b + k) z / ((a + 2k)(a + 2k + 1))
        num = -(a + k) * (a + b + k) * z / ((a + k2) * (a + k2 + 1.0));
        dd = 1.0 + num * dd;
        if (std::fabs(dd) < tiny) dd = tiny;
        c = 1.0 + num / c;
        if (std::fabs(c) < tiny) c = tiny;
        dd = 1.0 / dd;
        const double delta = dd * c;
        h *= delta;
        if (std::fabs(delta - 1.0) < 1e-16) break;
    }
    return h;
}

// I_z(a, a) for 0 <= z <= 1/2 (the lower half, where the fraction converges).
double incomplete_beta_symmetric_lower(double a, double z) {
    if (z <= 0.0) return 0.0;
    const double front = std::exp(a * std::log(z) + a * std::log1p(-z) - log_beta(a, a)) / a;
    return front * beta_continued_fraction(a, a, z);
}

// P(X < x) for x <= 0.
double lower_tail(double a, double x) { return incomplete_beta_symmetric_lower(a, 0.5 * (1.0 + x)); }

// P(u < X < v), every term evaluated as a small tail so nothing cancels.
double cell_probability(double a, double u, double v) {
    if (v <= 0.0) return lower_tail(a, v) - lower_tail(a, u);
    if (u >= 0.0) return lower_tail(a, -u) - lower_tail(a, -v);
    return 1.0 - lower_tail(a, u) - lower_tail(a, -v);
}

double cell_first_moment(int d, double u, double v) {
    const double a = 0.5 * (d - 1);
    const double cd = std::exp(std::lgamma(0.5 * d) - std::lgamma(0.5 * (d - 1))) / std::sqrt(M_PI);
    const double pu = std::fabs(u) < 1.0 ? std::exp(a * std::log1p(-u * u)) : 0.0;
    const double pv = std::fabs(v) < 1.0 ? std::exp(a * std::log1p(-v * v)) : 0.0;
    return cd * (pu - pv) / (d - 1);
}

}  // namespace

static void lloyd_max(int d, int bits, double* c_out, double* t_out) {
    const int n = 1 << bits;
    const double a = 0.5 * (d - 1);
    const double span = std::fmin(1.0, 3.0 / std::sqrt(static_cast<double>(d)));
    double c[16], next[16], edges[17];
    for (int j = 0; j < n; ++j) c[j] = -span + (2 * j + 1) * span / n;
    // Stop at a relative move of 1e-15, or once the moves have stopped
    // shrinking for 100 sweeps below 1e-13 (the rounding floor of the tail
    // probabilities is reached before 1e-15 for some (d, bits)).
    double best = INFINITY;
    int since_best = 0;
    for (int it = 0; it < 200000; ++it) {
        edges[0] = -1.0;
        edges[n] = 1.0;
        for (int j = 1; j < n; ++j) edges[j] = 0.5 * (c[j - 1] + c[j]);
        double moved = 0.0, biggest = 0.0;
        for (int j = 0; j < n; ++j) {
            next[j] = cell_first_moment(d, edges[j], edges[j + 1]) / cell_probability(a, edges[j], edges[j + 1]);
            moved = std::fmax(moved, std::fabs(next[j] - c[j]));
            biggest = std::fmax(biggest, std::fabs(next[j]));
        }
        std::memcpy(c, next, sizeof(double) * n);
        if (moved <= 1e-15 * biggest) break;
        if (moved < best) {
            best = moved;
            since_best = 0;
        } else if (++since_best >= 100 && moved <= 1e-13 * biggest) {
            break;
        }
    }
    // the density is even, so the optimal table is exactly odd-symmetric
    for (int j = 0; j < n / 2; ++j) {
        const double m = 0.5 * (c[n - 1 - j] - c[j]);
        c[j] = -m;
        c[n - 1 - j] = m;
    }
    for (int j = 0; j < n; ++j) c_out[j] = c[j];
    for (int j = 0; j + 1 < n; ++j) t_out[j] = 0.5 * (c[j] + c[j + 1]);
}

// The tensor-core kernels hold alpha * c_j as fp16.  The rounding error of a
// table entry is systematic (every code using it errs the same way), so alpha
// is chosen on a fine grid of [8, 16) to make the largest relative rounding
// error of the table small; relative error is invariant under powers of two,
// so one octave covers every scale.
static float round_to_half(float x) {  // IEEE binary16 round-to-nearest-even, normal range
    int e;
    const float m = std::frexp(x, &e);  // x = m 2^e, |m| in [0.5, 1)
    return std::ldexp(std::nearbyint(std::ldexp(m, 11)), e - 11);
}

double best_fp16_scale(const double* c, int n) {
    double best_err = INFINITY, best = 8.0;
    for (int k = 0; k < 8192; ++k) {
        const double alpha = 8.0 + 8.0 * k / 8192.0;
        double worst = 0.0;
        for (int j = 0; j < n; ++j) {
            const double v = alpha * c[j];
            if (v == 0.0) continue;
            const double r = round_to_half(static_cast<float>(v));
            worst = std::fmax(worst, std::fabs(r - v) / std::fabs(v));
        }
        if (worst < best_err) {
            best_err = worst;
            best = alpha;
        }
    }
    return best;
}

// ------------------------------------------------------------ random numbers
//
// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): state += golden gamma, then
// the published xor-shift/multiply finaliser.
static uint64_t splitmix64_next(uint64_t& state) {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

void rotation_sign_bits(uint64_t seed, int head_dim, uint32_t words[8]) {
    for (int i = 0; i < 8; ++i) words[i] = 0;
    uint64_t s = seed;
    for (int i = 0; i < head_dim && i < 256; ++i) {
        if (splitmix64_next(s) >> 63) words[i >> 5] |= 1u << (i & 31);
    }
}

// ------------------------------------------------------------------ sizes
bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

int vector_bytes(int mode, int bits, int head_dim) {
    return mode == TQ_MODE_INT8 ? head_dim : head_dim * bits / 8;
}

static bool supported_dim(int d) { return d == 64 || d == 128 || d == 256; }

tq_status validate_params(const tq_params* p) {
    if (!p) return TQ_ERR_INVALID_ARG;
    if (p->head_dim <= 0 || (p->head_dim & (p->head_dim - 1))) return TQ_ERR_INVALID_ARG;
    if (!supported_dim(p->head_dim)) return TQ_ERR_UNSUPPORTED;
    if (p->num_kv_heads < 1 || p->num_q_heads < p->num_kv_heads) return TQ_ERR_INVALID_ARG;
    if (p->num_q_heads % p->num_kv_heads) return TQ_ERR_INVALID_ARG;
    if (p->num_q_heads / p->num_kv_heads > 16) return TQ_ERR_UNSUPPORTED;
    const int modes[2] = {p->k_mode, p->v_mode};
    const int bits[2] = {p->k_bits, p->v_bits};
    for (int s = 0; s < 2; ++s) {
        if (modes[s] != TQ_MODE_TURBO && modes[s] != TQ_MODE_INT8) return TQ_ERR_INVALID_ARG;
        if (modes[s] == TQ_MODE_TURBO && (bits[s] < 2 || bits[s] > 4)) return TQ_ERR_INVALID_ARG;
    }
    if (p->qjl_dims < 0 || p->qjl_dims % 32 || p->qjl_dims > p->head_dim) return TQ_ERR_INVALID_ARG;
    if (p->qjl_dims > 0 && p->k_mode != TQ_MODE_TURBO) return TQ_ERR_INVALID_ARG;
    if (!(std::isfinite(p->sm_scale) && p->sm_scale >= 0.0f)) return TQ_ERR_INVALID_ARG;
    if (!(std::isfinite(p->sparse_v_threshold) && p->sparse_v_threshold >= 0.0f && p->sparse_v_threshold < 1.0f))
        return TQ_ERR_INVALID_ARG;
    if ((p->flags & ~TQ_PARAM_PREFETCH_EARLY) != 0 || p->reserved != 0) return TQ_ERR_INVALID_ARG;
    return TQ_OK;
}

tq_status validate_codebook(const tq_codebook* cb, int head_dim, int bits) {
    if (!cb) return TQ_ERR_INVALID_ARG;
    if (cb->head_dim != head_dim || cb->bits != bits) return TQ_ERR_INVALID_ARG;
    const int n = 1 << bits;
    for (int j = 0; j < n; ++j) {
        if (!std::isfinite(cb->centroids[j])) return TQ_ERR_INVALID_ARG;
        if (j && !(cb->centroids[j] > cb->centroids[j - 1])) return TQ_ERR_INVALID_ARG;
        // the kernels rely on the odd symmetry of the table
        if (cb->centroids[j] != -cb->centroids[n - 1 - j]) return TQ_ERR_INVALID_ARG;
    }
    for (int j = 0; j + 1 < n; ++j) {
        if (!(cb->boundaries[j] > cb->centroids[j] && cb->boundaries[j] < cb->centroids[j + 1]))
            return TQ_ERR_INVALID_ARG;
        if (cb->boundaries[j] != -cb->boundaries[n - 2 - j]) return TQ_ERR_INVALID_ARG;
    }
    return TQ_OK;
}

tq_status validate_cache(const tq_params& p, const tq_cache* c) {
    if (!c) return TQ_ERR_INVALID_ARG;
    if (c->batch < 1 || c->capacity < 1) return TQ_ERR_INVALID_ARG;
    if (!c->k_codes || !c->k_norms || !c->v_codes || !c->v_norms) return TQ_ERR_INVALID_ARG;
    if (!aligned16(c->k_codes) || !aligned16(c->k_norms) || !aligned16(c->v_codes) || !aligned16(c->v_norms))
        return TQ_ERR_ALIGNMENT;
    if (p.qjl_dims > 0) {
        if (!c->k_qjl || !c->k_gamma || !c->qjl_matrix) return TQ_ERR_INVALID_ARG;
        if (!aligned16(c->k_qjl) || !aligned16(c->k_gamma) || !aligned16(c->qjl_matrix)) return TQ_ERR_ALIGNMENT;
    }
    return TQ_OK;
}

tq_status validate_pages(const tq_params& p, const tq_cache* pool, const tq_block_table* table, PageMap* pm) {
    tq_status st = validate_cache(p, pool);
    if (st != TQ_OK) return st;
    if (!table || !table->d_table || table->batch < 1 || table->max_blocks < 1) return TQ_ERR_INVALID_ARG;
    // blocks of whole 16-token tiles keep every per-block copy 16-byte sized
    if (pool->capacity % 16 != 0) return TQ_ERR_INVALID_ARG;
    if (static_cast<long long>(table->max_blocks) * pool->capacity > INT32_MAX) return TQ_ERR_INVALID_ARG;
    pm->table = table->d_table;
    pm->batch = table->batch;
    pm->max_blocks = table->max_blocks;
    pm->block_size = pool->capacity;
    pm->num_blocks = pool->batch;
    return TQ_OK;
}

static long long gcd_ll(long long a, long long b) {
    while (b) {
        const long long r = a % b;
        a = b;
        b = r;
    }
    return a;
}

size_t counter_region_bytes(size_t workspace_bytes) {
    const size_t words = workspace_bytes / kMinUnitBytes + kGlobalCounters;
    return (words * sizeof(uint32_t) + 255) / 256 * 256;
}

// Partials (m, l) then acc, after the counter region.
static void place_partials(DecodePlan& plan, size_t slots, int head_dim, size_t counters) {
    plan.off_counters = 0;
    plan.off_ml = counters;
    plan.off_acc = plan.off_ml + (slots * 2 * sizeof(float) + 255) / 256 * 256;
    plan.bytes = plan.off_acc + slots * head_dim * sizeof(float);
}

DecodePlan plan_decode(const tq_params& p, int batch, int max_seq_len, int num_sms, size_t workspace_bytes,
                       bool general_kernel) {
    // Split count.  Few long sequences: one wave of equal items, one per SM,
    // when that keeps at least 85% of the SMs busy (every item then carries
    // one prologue and one merge); otherwise a multiple of the SM count where
    // possible.  Many sequences (a batch, possibly ragged): about two items
    // per SM, which the kernel's dynamic scheduling balances (splits past a
    // sequence's end cost nothing).  Splits are never
    // shorter than kMinSplitTokens nor more than kMaxSplits.
    DecodePlan plan;
    const long long units = static_cast<long long>(batch) * p.num_kv_heads;
    long long most = (max_seq_len + kMinSplitTokens - 1) / kMinSplitTokens;
    if (most > kMaxSplits) most = kMaxSplits;
    long long n;
    const long long one_wave = num_sms / units;
    if (units * 4 >= num_sms) {
        n = (2ll * num_sms + units - 1) / units;
    } else if (one_wave >= 1 && one_wave * units * 100 >= 85ll * num_sms) {
        n = one_wave;
    } else {
        const long long want = (static_cast<long long>(num_sms) * kBlocksPerSm + units - 1) / units;
        const long long step = num_sms / gcd_ll(units, num_sms);
        n = (want + step - 1) / step * step;
        if (n > most) n = want;
    }
    // The general split kernel (four warps a block, no persistent
    // scheduling) hides its load latency only with many blocks: it takes the
    // finest split the workspace bound allows.
    if (general_kernel) n = most;
    if (n > most) n = most;
    if (n < 1) n = 1;
    long long len = (max_seq_len + n - 1) / n;
    len = (len + kSplitAlign - 1) / kSplitAlign * kSplitAlign;
    n = (max_seq_len + len - 1) / len;
    plan.n_split = static_cast<int>(n);
    plan.split_len = static_cast<int>(len);
    const size_t slots = static_cast<size_t>(batch) * p.num_q_heads * plan.n_split;
    place_partials(plan, slots, p.head_dim, counter_region_bytes(workspace_bytes));
    return plan;
}

// Workspace bound valid for every device: the split count never exceeds
// ceil(max_seq_len / kMinSplitTokens).  The counter region grows with the
// workspace, so the size is the least fixed point of
// bytes = counter_region_bytes(bytes) + partials.
static size_t workspace_bound(const tq_params& p, int batch, int max_seq_len) {
    long long most = (max_seq_len + kMinSplitTokens - 1) / kMinSplitTokens;
    if (most > kMaxSplits) most = kMaxSplits;
    const size_t slots = static_cast<size_t>(batch) * p.num_q_heads * most;
    DecodePlan plan;
    place_partials(plan, slots, p.head_dim, 0);
    const size_t partials = plan.bytes;
    size_t bytes = partials;
    for (;;) {
        const size_t next = partials + counter_region_bytes(bytes);
        if (next == bytes) return bytes;
        bytes = next;
    }
}

}  // namespace tq

// =================================================================== C ABI
extern "C" {

const char* tq_status_string(tq_status status) {
    switch (status) {
        case TQ_OK: return "ok";
        case TQ_ERR_INVALID_ARG: return "invalid argument";
        case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
        case TQ_ERR_CAPACITY: return "workspace or cache too small";
        case TQ_ERR_CUDA: return "CUDA error";
        case TQ_ERR_TIMEOUT: return "timed out";
        case TQ_ERR_DEVICE: return "device-side check failed";
        case TQ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    }
    return "unknown status";
}

int32_t tq_abi_version(void) { return TQ_ABI_VERSION; }

tq_status tq_codebook_init(int32_t head_dim, int32_t bits, tq_codebook* out) {
    if (!out || bits < 1 || bits > 4 || head_dim < 3 || head_dim > 4096) return TQ_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof(*out));
    out->head_dim = head_dim;
    out->bits = bits;
    tq::lloyd_max(head_dim, bits, out->centroids, out->boundaries);
    out->fp16_scale = tq::best_fp16_scale(out->centroids, 1 << bits);
    return TQ_OK;
}

tq_status tq_rotation_signs(uint64_t seed, int32_t head_dim, float* out) {
    if (!out || head_dim < 1 || head_dim > 4096) return TQ_ERR_INVALID_ARG;
    uint64_t s = seed;
    for (int i = 0; i < head_dim; ++i) out[i] = (tq::splitmix64_next(s) >> 63) ? -1.0f : 1.0f;
    return TQ_OK;
}

tq_status tq_qjl_matrix(uint64_t seed, int32_t m, int32_t head_dim, float* out) {
    if (!out || m < 1 || head_dim < 1 || static_cast<long long>(m) * head_dim > (1ll << 26)) return TQ_ERR_INVALID_ARG;
    uint64_t s = seed ^ 0x5155414E544A4C00ull;
    const long long n = static_cast<long long>(m) * head_dim;
    for (long long k = 0; k < n; k += 2) {
        const double u1 = static_cast<double>(tq::splitmix64_next(s) >> 11) * 0x1.0p-53;
        const double u2 = static_cast<double>(tq::splitmix64_next(s) >> 11) * 0x1.0p-53;
        const double r = std::sqrt(-2.0 * std::log(1.0 - u1));
        out[k] = static_cast<float>(r * std::cos(2.0 * M_PI * u2));
        if (k + 1 < n) out[k + 1] = static_cast<float>(r * std::sin(2.0 * M_PI * u2));
    }
    return TQ_OK;
}

tq_status tq_cache_bytes(const tq_params* params, int32_t batch, int32_t capacity, size_t sizes_out[6]) {
    tq_status st = tq::validate_params(params);
    if (st != TQ_OK) return st;
    if (!sizes_out || batch < 1 || capacity < 1) return TQ_ERR_INVALID_ARG;
    const size_t slots = static_cast<size_t>(batch) * params->num_kv_heads * capacity;
    sizes_out[0] = slots * tq::vector_bytes(params->k_mode, params->k_bits, params->head_dim);
    sizes_out[1] = slots * sizeof(uint16_t);
    sizes_out[2] = params->qjl_dims ? slots * (params->qjl_dims / 8) : 0;
    sizes_out[3] = params->qjl_dims ? slots * sizeof(uint16_t) : 0;
    sizes_out[4] = slots * tq::vector_bytes(params->v_mode, params->v_bits, params->head_dim);
    sizes_out[5] = slots * sizeof(uint16_t);
    return TQ_OK;
}

tq_status tq_decode_workspace_bytes(const tq_params* params, int32_t batch, int32_t max_seq_len,
                                    size_t* bytes_out) {
    tq_status st = tq::validate_params(params);
    if (st != TQ_OK) return st;
    if (!bytes_out || batch < 1 || max_seq_len < 1) return TQ_ERR_INVALID_ARG;
    *bytes_out = tq::workspace_bound(*params, batch, max_seq_len);
    return TQ_OK;
}

}  // extern "C"
