// api.cu — the extern "C" boundary of libinkling: argument validation, TMA
// descriptor encoding, launches on the caller's stream.  No allocation, no
// synchronisation, no state besides the per-thread error message.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace inkling {
cudaError_t launch_sconv_kv(const inkling_sconv_params &p, cudaStream_t stream,
                            bool zero_hist = false);
cudaError_t launch_attn_prefill(const inkling_prefill_params &p, const CUtensorMap *maps,
                                cudaStream_t stream);
cudaError_t launch_sconv_out(const inkling_sconv_out_params &p, cudaStream_t stream);
cudaError_t launch_sconv_out_sharded(const inkling_sconv_out_sharded_params &p,
                                     cudaStream_t stream);
cudaError_t launch_attn_decode_mq(const inkling_decode_params &p, int splits, int s_whole,
                                  void *workspace, const CUtensorMap &tm_q,
                                  const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                                  cudaStream_t stream);
cudaError_t launch_attn_prefill_paged(const inkling_prefill_paged_params &p, const CUtensorMap &tm_q,
                                      const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                                      cudaStream_t stream, int dense_T, int sms);
cudaError_t launch_attn_prefill_pair(const inkling_prefill_params &p, const CUtensorMap *maps,
                                     cudaStream_t stream);
cudaError_t launch_attn_decode(const inkling_decode_params &p, int splits, int s_whole,
                               void *workspace, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                               cudaStream_t stream);
cudaError_t decode_static_scratch(void **ptr, size_t *bytes);
cudaError_t launch_wait_timeout_probe(int32_t *status, uint32_t limit_us, cudaStream_t stream);
}  // namespace inkling

using namespace inkling;

namespace {

thread_local char g_err[512] = "";

inkling_status fail(inkling_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

inkling_status cuda_fail(cudaError_t e, const char *what) {
    return fail(INKLING_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    });
    return fn;
}

// bf16 tensor map, 128-byte swizzle, rank <= 4; dims/strides in elements/bytes
inkling_status make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                        const cuuint64_t *strides_bytes, const cuuint32_t *box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(INKLING_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base),
                    dims, strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(INKLING_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return INKLING_OK;
}

// sm_100 check for the current device (cached per device)
inkling_status check_device(int *num_sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    static int major[64], sms[64];
    if (dev < 0 || dev >= 64) return fail(INKLING_ERR_UNSUPPORTED, "device index %d", dev);
    if (major[dev] == 0) {
        int mj = 0, n = 0;
        e = cudaDeviceGetAttribute(&mj, cudaDevAttrComputeCapabilityMajor, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        sms[dev] = n;
        major[dev] = mj;
    }
    if (major[dev] != 10)
        return fail(INKLING_ERR_UNSUPPORTED, "libinkling is built for sm_100a (B200); device %d has "
                                             "compute capability %d.x", dev, major[dev]);
    if (num_sms) *num_sms = sms[dev];
    return INKLING_OK;
}

// sequences x query tokens: the rows of split partials
static int32_t decode_rows(const inkling_decode_params &p) {
    return p.num_seqs * (p.q_len > 1 ? p.q_len : 1);
}

// Split count for num_splits = 0.  Both decode kernels run two blocks per SM
// (`slots` = 2 x SMs).  When the (sequence, kv head) units alone fill the
// slots the key range is not split (no partials, no combine pass).  A short
// key range (at most 4096 keys per split) takes one wave: as many splits as
// fit in the slots, at least ~512 keys (8 chunks) each.  A long one starts at
// about 8 blocks per SM and, within twice that, takes the count whose last
// wave is fullest.  Measured on B200 (KV GB/s):
//   window 4096, 1 token:  8 seqs  4 splits 3839, 8 splits ~3000;
//                         16 seqs  2 splits 4774, 4: 4554, 8: 4150;
//                         32 seqs  1 split  5745, 2: 5458;
//   window 4096, 9 tokens: 8 seqs  4 splits 2882, 8: 2539;
//                         16 seqs  2 splits 3735, 8: 2940;  32 seqs 1 split 4574;
//   1M tokens, 1 token:  batch 8 37 splits (8 full waves) 6716 vs 19: 6081;
//                        batch 1 148 splits 6309 vs 222: 6262.
int decode_splits(const inkling_decode_params &p, int num_sms) {
    if (p.num_splits > 0) return p.num_splits;
    const long units = (long)p.num_seqs * p.num_kv_heads;
    const long slots = 2L * num_sms;
    if (units >= slots) return 1;
    const long max_keys = (long)p.max_blocks * 128;
    const long keys = p.window > 0 ? (p.window < max_keys ? p.window : max_keys) : max_keys;
    const long chunks = (keys + 63) / 64 + 1;
    long cap = chunks / 8;
    if (cap < 1) cap = 1;
    if (cap > 1024) cap = 1024;
    const long one_wave = slots / units;
    if (keys <= 4096L * one_wave) return (int)(one_wave < cap ? one_wave : cap);
    long s0 = (4 * slots + units - 1) / units;
    if (s0 > cap) s0 = cap;
    long best = s0;
    double best_fill = 0.0;
    for (long c = s0; c <= 2 * s0 && c <= cap; ++c) {
        const long blocks = units * c;
        const long waves = (blocks + slots - 1) / slots;
        const double fill = (double)blocks / (double)(waves * slots);
        if (fill > best_fill + 1e-9) {
            best_fill = fill;
            best = c;
        }
    }
    return (int)best;
}

// How a decode call runs: sequences [0, s_whole) unsplit, the others in
// `splits` key-range pieces (s_whole == num_seqs: no partials).
struct DecodePlan {
    int splits, s_whole;
};

// For num_splits = 0, when the (sequence, kv head) units fill the slots: the
// sequences that fill whole waves run unsplit and the rest, which would leave
// most of a last wave idle, in c pieces (2..8, at least ~512 keys each) whose
// partials the combine merges.  Cost model, in units of one whole unit's
// time, fitted to B200 measurements: a wave of pieces costs 1/c + 0.1 (a
// piece's setup, pipeline fill and partials), the combine 0.05; the plan is
// taken when it is 10% under the unsplit last wave (1).  Measured against the
// unsplit plan (window 4096, KV TB/s):
//   1 token:   40 sequences 4.34 -> 5.70 (8 pieces), 48: 5.20 -> 5.91 (3),
//              80: 5.43 -> 6.22 (6), 128: 6.20 -> 6.38 (2);
//   9 tokens:  40 sequences 3.15 -> 4.70 (8), 48: 3.76 -> 4.82 (3),
//              80: 4.23 -> 4.97 (6), 128: 4.94 -> 5.09 (2);
//   64 sequences stay unsplit (9 tokens in 4 pieces measured 4.71 vs 4.87).
static DecodePlan decode_plan(const inkling_decode_params &p, int num_sms) {
    const int sp = decode_splits(p, num_sms);
    DecodePlan plan{sp, sp == 1 ? p.num_seqs : 0};
    const long slots = 2L * num_sms;
    const long units = (long)p.num_seqs * p.num_kv_heads;
    if (p.num_splits > 0 || sp != 1 || units < slots) return plan;
    const int s_whole = (int)(((units / slots) * slots) / p.num_kv_heads);
    const long rest = units - (long)s_whole * p.num_kv_heads;
    if (rest <= 0 || s_whole >= p.num_seqs) return plan;
    const long max_keys = (long)p.max_blocks * 128;
    const long keys = p.window > 0 ? (p.window < max_keys ? p.window : max_keys) : max_keys;
    const long cap = ((keys + 63) / 64 + 1) / 8;
    double best = 0.9;  // the remainder's last wave, unsplit, costs 1
    int best_c = 1;
    for (int c = 2; c <= 8 && c <= cap; ++c) {
        const long waves = (rest * c + slots - 1) / slots;
        const double t = (double)waves * (1.0 / c + 0.1) + 0.05;
        if (t < best) {
            best = t;
            best_c = c;
        }
    }
    if (best_c > 1) plan = DecodePlan{best_c, s_whole};
    return plan;
}

// bytes of partials a plan needs (0: none)
static size_t plan_workspace(const inkling_decode_params &p, const DecodePlan &plan) {
    if (plan.splits <= 1 || plan.s_whole >= p.num_seqs) return 0;
    const int32_t rows = (p.num_seqs - plan.s_whole) * (p.q_len > 1 ? p.q_len : 1);
    return inkling_attn_decode_workspace_bytes(rows, p.num_q_heads, plan.splits);
}

inkling_status validate_decode(const inkling_decode_params *p) {
    if (!p) return fail(INKLING_ERR_INVALID, "params is NULL");
    if (p->num_seqs < 0 || p->num_q_heads < 1 || p->num_kv_heads < 1)
        return fail(INKLING_ERR_INVALID, "num_seqs must be >= 0 and head counts >= 1");
    if (p->head_dim != INKLING_HEAD_DIM)
        return fail(INKLING_ERR_UNSUPPORTED, "head_dim %d (only 128 is implemented)", p->head_dim);
    if (p->num_q_heads % p->num_kv_heads)
        return fail(INKLING_ERR_INVALID, "num_q_heads %% num_kv_heads != 0");
    if (p->num_q_heads / p->num_kv_heads > 8)
        return fail(INKLING_ERR_UNSUPPORTED, "decode supports at most 8 query heads per kv head");
    if (p->max_blocks < 1 || p->num_blocks < 1)
        return fail(INKLING_ERR_INVALID, "max_blocks and num_blocks must be >= 1");
    if ((long)p->max_blocks * 128 > (1L << 30))
        return fail(INKLING_ERR_UNSUPPORTED, "max_blocks * 128 exceeds 2^30 tokens");
    if ((long)p->num_blocks * p->num_kv_heads * 128 >= (1L << 31))
        return fail(INKLING_ERR_UNSUPPORTED, "cache pool rows exceed 2^31");
    if (p->window < 0 || p->d_max < 0) return fail(INKLING_ERR_INVALID, "window and d_max must be >= 0");
    if (p->num_splits < 0 || p->num_splits > 1024)
        return fail(INKLING_ERR_INVALID, "num_splits must be in [0, 1024]");
    if (p->q_len < 0) return fail(INKLING_ERR_INVALID, "q_len must be >= 0");
    if (p->q_len > 1 && (p->num_q_heads / p->num_kv_heads) * p->q_len > 80)
        return fail(INKLING_ERR_UNSUPPORTED,
                    "multi-token decode supports (query heads per kv head) * q_len <= 80");
    if ((long)p->num_seqs * (p->q_len > 1 ? p->q_len : 1) * p->num_q_heads >= (1L << 31))
        return fail(INKLING_ERR_UNSUPPORTED, "num_seqs * q_len * num_q_heads exceeds 2^31");
    if (p->num_seqs == 0) return INKLING_OK;
    if (!p->q || !p->k_cache || !p->v_cache || !p->block_table || !p->seq_lens || !p->bias || !p->out)
        return fail(INKLING_ERR_INVALID, "a required pointer is NULL");
    if (!aligned16(p->q) || !aligned16(p->k_cache) || !aligned16(p->v_cache) || !aligned16(p->out))
        return fail(INKLING_ERR_INVALID, "q, caches and out must be 16-byte aligned");
    if (((uintptr_t)p->bias & 3u) != 0) return fail(INKLING_ERR_INVALID, "bias must be 4-byte aligned");
    return INKLING_OK;
}

// Tensor maps of the paged prefill kernel: q [rows, Hq, 128] seen as (d,
// head, row), one box = 128 rows x 64 d of one head; the caches as (d, rows),
// one box = one 128-token (block, kv head) x 64 d.
inkling_status paged_maps(const void *q, long rows, int Hq, const void *k_cache,
                          const void *v_cache, long num_blocks, int Hkv, CUtensorMap *tm_q,
                          CUtensorMap *tm_k, CUtensorMap *tm_v) {
    inkling_status st;
    {
        cuuint64_t dims[3] = {128, (cuuint64_t)Hq, (cuuint64_t)rows};
        cuuint64_t str[2] = {256, (cuuint64_t)Hq * 256};
        cuuint32_t box[3] = {64, 1, 128};
        if ((st = make_map(tm_q, q, 3, dims, str, box)) != INKLING_OK) return st;
    }
    const cuuint64_t crows = (cuuint64_t)num_blocks * Hkv * 128;
    cuuint64_t dims[2] = {128, crows};
    cuuint64_t str[1] = {256};
    cuuint32_t box[2] = {64, 128};
    if ((st = make_map(tm_k, k_cache, 2, dims, str, box)) != INKLING_OK) return st;
    return make_map(tm_v, v_cache, 2, dims, str, box);
}

// The two-pass dense prefill: blocks per sequence of the scratch cache, its
// bytes, and whether the sizes fit the paged kernel's and the append's limits.
long scratch_blocks_per_seq(const inkling_prefill_params *p) { return (p->seq_len + 127) / 128; }

size_t scratch_bytes(const inkling_prefill_params *p) {
    return 2ull * (size_t)p->batch * (size_t)scratch_blocks_per_seq(p) * (size_t)p->num_kv_heads *
           128 * 128 * 2;
}

bool two_pass_fits(const inkling_prefill_params *p) {
    const long pool = p->k_cache ? (long)p->num_blocks : (long)p->batch * scratch_blocks_per_seq(p);
    return p->seq_len <= (1 << 20) && pool * p->num_kv_heads * 128 < (1L << 31) &&
           (long)p->batch * p->seq_len * p->num_q_heads < (1L << 31) &&
           (long)p->batch * scratch_blocks_per_seq(p) <= 0x7fffffffL;
}

bool wants_two_pass(const inkling_prefill_params *p) {
    return p->path == INKLING_PREFILL_TWO_PASS ||
           (p->path == INKLING_PREFILL_AUTO && p->seq_len >= INKLING_PREFILL_TWO_PASS_MIN_T &&
            (long)p->batch * p->seq_len >= INKLING_PREFILL_TWO_PASS_MIN_TOKENS);
}

// Pass 1: the sconv of all T raw keys/values of every sequence, zero history,
// into the paged layout (the caller's cache through its block table, else the
// scratch with sequence b on blocks b*nb ...), the state written when given.
// Pass 2: the paged prefill kernel with every sequence one chunk of T rows.
inkling_status prefill_two_pass(const inkling_prefill_params *p, cudaStream_t stream, int sms) {
    const bool cache = p->k_cache != nullptr;
    const int nb = (int)scratch_blocks_per_seq(p);
    void *kc = cache ? p->k_cache : p->workspace;
    void *vc = cache ? p->v_cache : (void *)((char *)p->workspace + scratch_bytes(p) / 2);
    const int32_t *table = cache ? p->block_table : nullptr;
    const int max_blocks = cache ? p->max_blocks : nb;
    const int num_blocks = cache ? p->num_blocks : p->batch * nb;

    inkling_sconv_params sp = {};
    sp.k_new = p->k_raw;
    sp.v_new = p->v_raw;
    sp.w_k = p->w_k;
    sp.w_v = p->w_v;
    sp.k_state = p->k_state;
    sp.v_state = p->v_state;
    sp.k_cache = kc;
    sp.v_cache = vc;
    sp.block_table = table;
    sp.seq_lens = nullptr;
    sp.status = p->status;
    sp.num_seqs = p->batch;
    sp.n_new = p->seq_len;
    sp.num_kv_heads = p->num_kv_heads;
    sp.head_dim = INKLING_HEAD_DIM;
    sp.max_blocks = max_blocks;
    sp.num_blocks = num_blocks;

    inkling_prefill_paged_params pp = {};
    pp.q = p->q;
    pp.cu_q = nullptr;
    pp.k_cache = kc;
    pp.v_cache = vc;
    pp.block_table = table;
    pp.seq_lens = nullptr;
    pp.bias = p->bias;
    pp.out = p->out;
    pp.lse = p->lse;
    pp.status = p->status;
    pp.num_seqs = p->batch;
    pp.total_q = p->batch * p->seq_len;
    pp.max_q = p->seq_len;
    pp.num_q_heads = p->num_q_heads;
    pp.num_kv_heads = p->num_kv_heads;
    pp.head_dim = INKLING_HEAD_DIM;
    pp.max_blocks = max_blocks;
    pp.num_blocks = num_blocks;
    pp.window = p->window;
    pp.d_max = p->d_max;

    CUtensorMap tm_q, tm_k, tm_v;
    inkling_status st = paged_maps(p->q, (long)p->batch * p->seq_len, p->num_q_heads, kc, vc,
                                   num_blocks, p->num_kv_heads, &tm_q, &tm_k, &tm_v);
    if (st != INKLING_OK) return st;
    cudaError_t e = launch_sconv_kv(sp, stream, /*zero_hist=*/true);
    if (e != cudaSuccess) return cuda_fail(e, "attn_prefill (two-pass) sconv launch");
    e = launch_attn_prefill_paged(pp, tm_q, tm_k, tm_v, stream, p->seq_len, sms);
    if (e != cudaSuccess) return cuda_fail(e, "attn_prefill (two-pass) paged launch");
    return INKLING_OK;
}

}  // namespace

extern "C" {

const char *inkling_last_error(void) { return g_err; }

int inkling_version(void) { return 100; }

inkling_status inkling_selftest_wait_timeout(int32_t *status, uint32_t limit_us,
                                             inkling_stream_t stream) {
    g_err[0] = 0;
    if (!status) return fail(INKLING_ERR_INVALID, "status is NULL");
    if (limit_us == 0 || limit_us > 10000000u)
        return fail(INKLING_ERR_INVALID, "limit_us must be in [1, 10^7]");
    inkling_status st = check_device(nullptr);
    if (st != INKLING_OK) return st;
    cudaError_t e = launch_wait_timeout_probe(status, limit_us, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait timeout probe launch");
    return INKLING_OK;
}

inkling_status inkling_sconv_kv(const inkling_sconv_params *p, inkling_stream_t stream) {
    g_err[0] = 0;
    if (!p) return fail(INKLING_ERR_INVALID, "params is NULL");
    if (p->num_seqs < 0 || p->num_kv_heads < 1)
        return fail(INKLING_ERR_INVALID, "num_seqs must be >= 0, num_kv_heads >= 1");
    if (p->head_dim != INKLING_HEAD_DIM)
        return fail(INKLING_ERR_UNSUPPORTED, "head_dim %d (only 128 is implemented)", p->head_dim);
    if (p->n_new < 1 || p->n_new > (1 << 20))
        return fail(INKLING_ERR_INVALID, "n_new must be in [1, 2^20]");
    if ((long)p->num_seqs * p->n_new * p->num_kv_heads * 16 * 2 >= (1L << 40))
        return fail(INKLING_ERR_UNSUPPORTED, "too many tokens in one append");
    if (p->max_blocks < 1 || p->num_blocks < 1)
        return fail(INKLING_ERR_INVALID, "max_blocks and num_blocks must be >= 1");
    if ((long)p->max_blocks * 128 > (1L << 30))
        return fail(INKLING_ERR_UNSUPPORTED, "max_blocks * 128 exceeds 2^30 tokens");
    if (p->num_seqs == 0) return INKLING_OK;
    if (!p->k_new || !p->v_new || !p->w_k || !p->w_v || !p->k_state || !p->v_state || !p->k_cache ||
        !p->v_cache || !p->block_table || !p->seq_lens)
        return fail(INKLING_ERR_INVALID, "a required pointer is NULL");
    if (!aligned16(p->k_new) || !aligned16(p->v_new) || !aligned16(p->w_k) || !aligned16(p->w_v) ||
        !aligned16(p->k_state) || !aligned16(p->v_state) || !aligned16(p->k_cache) ||
        !aligned16(p->v_cache))
        return fail(INKLING_ERR_INVALID, "tensors must be 16-byte aligned");
    inkling_status st = check_device(nullptr);
    if (st != INKLING_OK) return st;
    cudaError_t e = launch_sconv_kv(*p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "sconv_kv launch");
    return INKLING_OK;
}

inkling_status inkling_attn_prefill(const inkling_prefill_params *p, inkling_stream_t stream) {
    g_err[0] = 0;
    if (!p) return fail(INKLING_ERR_INVALID, "params is NULL");
    if (p->batch < 0 || p->seq_len < 0 || p->num_q_heads < 1 || p->num_kv_heads < 1)
        return fail(INKLING_ERR_INVALID, "batch, seq_len must be >= 0 and head counts >= 1");
    if (p->head_dim != INKLING_HEAD_DIM)
        return fail(INKLING_ERR_UNSUPPORTED, "head_dim %d (only 128 is implemented)", p->head_dim);
    if (p->num_q_heads % p->num_kv_heads)
        return fail(INKLING_ERR_INVALID, "num_q_heads %% num_kv_heads != 0");
    if (p->window < 0 || p->d_max < 0) return fail(INKLING_ERR_INVALID, "window and d_max must be >= 0");
    if (p->seq_len > (1 << 30)) return fail(INKLING_ERR_UNSUPPORTED, "seq_len above 2^30");
    const long blocks = (long)p->batch * p->num_q_heads * ((p->seq_len + 255) / 256);
    if (blocks > 0x7fffffffL) return fail(INKLING_ERR_UNSUPPORTED, "grid too large");
    if (blocks == 0) return INKLING_OK;
    if (!p->q || !p->k_raw || !p->v_raw || !p->w_k || !p->w_v || !p->bias || !p->out)
        return fail(INKLING_ERR_INVALID, "a required pointer is NULL");
    if (!aligned16(p->q) || !aligned16(p->k_raw) || !aligned16(p->v_raw) || !aligned16(p->w_k) ||
        !aligned16(p->w_v) || !aligned16(p->out))
        return fail(INKLING_ERR_INVALID, "q, k_raw, v_raw, taps and out must be 16-byte aligned");
    if (p->k_cache || p->v_cache || p->block_table) {
        if (!p->k_cache || !p->v_cache || !p->block_table)
            return fail(INKLING_ERR_INVALID, "k_cache, v_cache and block_table go together");
        if (!aligned16(p->k_cache) || !aligned16(p->v_cache))
            return fail(INKLING_ERR_INVALID, "caches must be 16-byte aligned");
        if (p->max_blocks < 1 || p->num_blocks < 1)
            return fail(INKLING_ERR_INVALID, "max_blocks and num_blocks must be >= 1");
        if ((long)p->max_blocks * 128 < p->seq_len)
            return fail(INKLING_ERR_INVALID, "max_blocks * 128 < seq_len");
        if ((long)p->num_blocks * p->num_kv_heads * 128 >= (1L << 31))
            return fail(INKLING_ERR_UNSUPPORTED, "cache pool rows exceed 2^31");
    }
    if ((p->k_state != nullptr) != (p->v_state != nullptr))
        return fail(INKLING_ERR_INVALID, "k_state and v_state go together");
    if (p->k_state && (!aligned16(p->k_state) || !aligned16(p->v_state)))
        return fail(INKLING_ERR_INVALID, "states must be 16-byte aligned");
    if (p->path < INKLING_PREFILL_AUTO || p->path > INKLING_PREFILL_TWO_PASS)
        return fail(INKLING_ERR_INVALID, "path must be INKLING_PREFILL_AUTO, _FUSED or _TWO_PASS");
    if (p->workspace && !aligned16(p->workspace))
        return fail(INKLING_ERR_INVALID, "workspace must be 16-byte aligned");
    bool two_pass = false;
    if (wants_two_pass(p)) {
        const bool room = p->k_cache || (p->workspace && p->workspace_bytes >= scratch_bytes(p));
        if (p->path == INKLING_PREFILL_TWO_PASS) {
            if (!two_pass_fits(p))
                return fail(INKLING_ERR_UNSUPPORTED,
                            "two-pass prefill: T above 2^20, or cache rows / B*T*Hq above 2^31");
            if (!room)
                return fail(INKLING_ERR_INVALID,
                            "two-pass prefill without a cache needs a workspace of %zu bytes",
                            scratch_bytes(p));
        }
        two_pass = room && two_pass_fits(p);
    }
    int sms = 0;
    inkling_status st = check_device(&sms);
    if (st != INKLING_OK) return st;
    if (two_pass) return prefill_two_pass(p, (cudaStream_t)stream, sms);

    const cuuint64_t T = (cuuint64_t)p->seq_len, B = (cuuint64_t)p->batch;
    const cuuint64_t Hq = (cuuint64_t)p->num_q_heads, Hkv = (cuuint64_t)p->num_kv_heads;
    // GQA groups of even size run on CTA pairs (2-SM MMAs sharing every
    // key/value tile); odd groups on single CTAs
    const bool pair = ((p->num_q_heads / p->num_kv_heads) % 2) == 0;
    CUtensorMap maps[6];
    {
        // q and out [B, T, Hq, 128] seen as (d, T, Hq, B)
        cuuint64_t dims[4] = {128, T, Hq, B};
        cuuint64_t str[3] = {Hq * 256, 256, T * Hq * 256};
        cuuint32_t box[4] = {64, 128, 1, 1};
        if ((st = make_map(&maps[0], p->q, 4, dims, str, box)) != INKLING_OK) return st;
        if ((st = make_map(&maps[5], p->out, 4, dims, str, box)) != INKLING_OK) return st;
    }
    const void *kv[2] = {p->k_raw, p->v_raw};
    for (int w = 0; w < 2; ++w) {
        // raw keys / values [B, T, Hkv, 128] seen as (d, T, Hkv, B): a tile box
        // (128 rows, or 64 key rows for a CTA pair) and an 8-row history box
        cuuint64_t dims[4] = {128, T, Hkv, B};
        cuuint64_t str[3] = {Hkv * 256, 256, T * Hkv * 256};
        cuuint32_t box_t[4] = {64, (cuuint32_t)((pair && w == 0) ? 64 : 128), 1, 1};
        cuuint32_t box_h[4] = {64, 8, 1, 1};
        if ((st = make_map(&maps[1 + 2 * w], kv[w], 4, dims, str, box_t)) != INKLING_OK) return st;
        if ((st = make_map(&maps[2 + 2 * w], kv[w], 4, dims, str, box_h)) != INKLING_OK) return st;
    }
    if (pair) {
        cudaError_t e = launch_attn_prefill_pair(*p, maps, (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_fail(e, "attn_prefill (CTA pairs) launch");
        return INKLING_OK;
    }
    cudaError_t e = launch_attn_prefill(*p, maps, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "attn_prefill launch");
    return INKLING_OK;
}

inkling_status inkling_sconv_out(const inkling_sconv_out_params *p, inkling_stream_t stream) {
    g_err[0] = 0;
    if (!p) return fail(INKLING_ERR_INVALID, "params is NULL");
    if (p->batch < 0 || p->seq_len < 0) return fail(INKLING_ERR_INVALID, "batch and seq_len must be >= 0");
    if (p->channels < 8 || p->channels % 8)
        return fail(INKLING_ERR_INVALID, "channels must be a positive multiple of 8");
    if ((long)p->batch * p->seq_len * p->channels >= (1L << 40))
        return fail(INKLING_ERR_UNSUPPORTED, "tensor too large");
    if (p->batch == 0) return INKLING_OK;
    if (!p->x || !p->w || !p->y) return fail(INKLING_ERR_INVALID, "x, w and y must not be NULL");
    if (!aligned16(p->x) || !aligned16(p->y) || !aligned16(p->w) ||
        (p->state && !aligned16(p->state)))
        return fail(INKLING_ERR_INVALID, "x, w, y and state must be 16-byte aligned");
    const size_t xb = (size_t)p->batch * p->seq_len * p->channels * 2;
    const char *x0 = (const char *)p->x, *y0 = (const char *)p->y;
    if (xb && x0 < y0 + xb && y0 < x0 + xb) return fail(INKLING_ERR_INVALID, "x and y overlap");
    inkling_status st = check_device(nullptr);
    if (st != INKLING_OK) return st;
    cudaError_t e = launch_sconv_out(*p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "sconv_out launch");
    return INKLING_OK;
}

inkling_status inkling_sconv_out_sharded(const inkling_sconv_out_sharded_params *p,
                                         inkling_stream_t stream) {
    g_err[0] = 0;
    if (!p) return fail(INKLING_ERR_INVALID, "params is NULL");
    if (p->n_ranks < 1 || p->n_ranks > INKLING_SHARD_MAX_RANKS)
        return fail(INKLING_ERR_INVALID, "n_ranks must be in [1, %d]", INKLING_SHARD_MAX_RANKS);
    if (p->rank < 0 || p->rank >= p->n_ranks)
        return fail(INKLING_ERR_INVALID, "rank must be in [0, n_ranks)");
    if (p->batch < 0 || p->seq_len < 0) return fail(INKLING_ERR_INVALID, "batch and seq_len must be >= 0");
    if (p->channels < 8 * p->n_ranks || p->channels % (8 * p->n_ranks))
        return fail(INKLING_ERR_INVALID, "channels must be a positive multiple of 8 * n_ranks");
    if ((long)p->batch * p->seq_len * p->channels >= (1L << 40))
        return fail(INKLING_ERR_UNSUPPORTED, "tensor too large");
    if (p->batch == 0 || p->seq_len == 0) return INKLING_OK;
    if (!p->x_parts || !p->y_parts || !p->w)
        return fail(INKLING_ERR_INVALID, "x_parts, y_parts and w must not be NULL");
    if (!aligned16(p->w) || (p->state && !aligned16(p->state)))
        return fail(INKLING_ERR_INVALID, "w and state must be 16-byte aligned");
    const size_t nb = (size_t)p->batch * p->seq_len * p->channels * 2;
    for (int r = 0; r < p->n_ranks; ++r) {
        if (!p->x_parts[r] || !p->y_parts[r])
            return fail(INKLING_ERR_INVALID, "x_parts[%d] / y_parts[%d] is NULL", r, r);
        if (!aligned16(p->x_parts[r]) || !aligned16(p->y_parts[r]))
            return fail(INKLING_ERR_INVALID, "x_parts and y_parts must be 16-byte aligned");
    }
    for (int r = 0; r < p->n_ranks; ++r)
        for (int q = 0; q < p->n_ranks; ++q) {
            const char *x0 = (const char *)p->x_parts[r], *y0 = (const char *)p->y_parts[q];
            if (x0 < y0 + nb && y0 < x0 + nb)
                return fail(INKLING_ERR_INVALID, "x_parts[%d] overlaps y_parts[%d]", r, q);
        }
    inkling_status st = check_device(nullptr);
    if (st != INKLING_OK) return st;
    cudaError_t e = launch_sconv_out_sharded(*p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "sconv_out_sharded launch");
    return INKLING_OK;
}

inkling_status inkling_attn_prefill_paged(const inkling_prefill_paged_params *p,
                                          inkling_stream_t stream) {
    g_err[0] = 0;
    if (!p) return fail(INKLING_ERR_INVALID, "params is NULL");
    if (p->num_seqs < 0 || p->total_q < 0 || p->max_q < 0 || p->num_q_heads < 1 ||
        p->num_kv_heads < 1)
        return fail(INKLING_ERR_INVALID, "sizes must be >= 0 and head counts >= 1");
    if (p->head_dim != INKLING_HEAD_DIM)
        return fail(INKLING_ERR_UNSUPPORTED, "head_dim %d (only 128 is implemented)", p->head_dim);
    if (p->num_q_heads % p->num_kv_heads)
        return fail(INKLING_ERR_INVALID, "num_q_heads %% num_kv_heads != 0");
    if (p->max_blocks < 1 || p->num_blocks < 1)
        return fail(INKLING_ERR_INVALID, "max_blocks and num_blocks must be >= 1");
    if ((long)p->max_blocks * 128 > (1L << 30))
        return fail(INKLING_ERR_UNSUPPORTED, "max_blocks * 128 exceeds 2^30 tokens");
    if ((long)p->num_blocks * p->num_kv_heads * 128 >= (1L << 31))
        return fail(INKLING_ERR_UNSUPPORTED, "cache pool rows exceed 2^31");
    if ((long)p->total_q * p->num_q_heads >= (1L << 31))
        return fail(INKLING_ERR_UNSUPPORTED, "total_q * num_q_heads exceeds 2^31");
    if (p->window < 0 || p->d_max < 0) return fail(INKLING_ERR_INVALID, "window and d_max must be >= 0");
    if (p->num_seqs == 0 || p->total_q == 0 || p->max_q == 0) return INKLING_OK;
    if ((long)p->num_seqs * p->num_q_heads * ((p->max_q + 255) / 256) >= (1L << 31))
        return fail(INKLING_ERR_UNSUPPORTED, "grid too large");
    if (!p->q || !p->cu_q || !p->k_cache || !p->v_cache || !p->block_table || !p->seq_lens ||
        !p->bias || !p->out)
        return fail(INKLING_ERR_INVALID, "a required pointer is NULL");
    if (!aligned16(p->q) || !aligned16(p->k_cache) || !aligned16(p->v_cache) || !aligned16(p->out))
        return fail(INKLING_ERR_INVALID, "q, caches and out must be 16-byte aligned");
    if (((uintptr_t)p->bias & 3u) != 0) return fail(INKLING_ERR_INVALID, "bias must be 4-byte aligned");
    int sms = 0;
    inkling_status st = check_device(&sms);
    if (st != INKLING_OK) return st;
    CUtensorMap tm_q, tm_k, tm_v;
    if ((st = paged_maps(p->q, p->total_q, p->num_q_heads, p->k_cache, p->v_cache, p->num_blocks,
                         p->num_kv_heads, &tm_q, &tm_k, &tm_v)) != INKLING_OK)
        return st;
    cudaError_t e = launch_attn_prefill_paged(*p, tm_q, tm_k, tm_v, (cudaStream_t)stream, 0, sms);
    if (e != cudaSuccess) return cuda_fail(e, "attn_prefill_paged launch");
    return INKLING_OK;
}

size_t inkling_attn_prefill_workspace_bytes(const inkling_prefill_params *p) {
    if (!p || p->batch <= 0 || p->seq_len <= 0 || p->num_kv_heads < 1 || p->num_q_heads < 1 ||
        p->k_cache || !wants_two_pass(p))
        return 0;
    if (p->path == INKLING_PREFILL_AUTO && !two_pass_fits(p)) return 0;
    return scratch_bytes(p);
}

size_t inkling_attn_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_splits) {
    if (num_seqs < 0 || num_q_heads < 1 || num_splits < 1 || num_splits > 1024) return 0;
    if (num_splits == 1) return 16;  // no partials; any non-NULL pointer will do
    return (size_t)num_seqs * num_q_heads * num_splits * (128 + 2) * sizeof(float);
}

int32_t inkling_attn_decode_num_splits(const inkling_decode_params *p) {
    if (validate_decode(p) != INKLING_OK) return 0;
    int sms = 0;
    if (check_device(&sms) != INKLING_OK) return 0;
    return decode_plan(*p, sms).splits;
}

static inkling_status decode_with(const inkling_decode_params *p, const DecodePlan &plan,
                                  void *workspace, size_t workspace_bytes, inkling_stream_t stream);

inkling_status inkling_attn_decode(const inkling_decode_params *p, void *workspace,
                                   size_t workspace_bytes, inkling_stream_t stream) {
    g_err[0] = 0;
    inkling_status st = validate_decode(p);
    if (st != INKLING_OK) return st;
    if (p->num_seqs == 0) return INKLING_OK;
    int sms = 0;
    if ((st = check_device(&sms)) != INKLING_OK) return st;
    DecodePlan plan = decode_plan(*p, sms);
    // a split plan chosen automatically over a workspace too small for it
    // (sized for one split) runs unsplit instead
    if (p->num_splits == 0 && plan.s_whole > 0 && plan.s_whole < p->num_seqs &&
        (!workspace || workspace_bytes < plan_workspace(*p, plan)))
        plan = DecodePlan{1, p->num_seqs};
    return decode_with(p, plan, workspace, workspace_bytes, stream);
}

inkling_status inkling_attn_decode_static(const inkling_decode_params *p, inkling_stream_t stream) {
    g_err[0] = 0;
    inkling_status st = validate_decode(p);
    if (st != INKLING_OK) return st;
    if (p->num_seqs == 0) return INKLING_OK;
    int sms = 0;
    if ((st = check_device(&sms)) != INKLING_OK) return st;
    void *scratch = nullptr;
    size_t cap = 0;
    cudaError_t e = decode_static_scratch(&scratch, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the decode scratch");
    DecodePlan plan = decode_plan(*p, sms);
    if (plan.s_whole > 0 && plan.s_whole < p->num_seqs) {
        // whole + pieces: run it when its partials fit, else unsplit
        if (plan_workspace(*p, plan) > cap) plan = DecodePlan{1, p->num_seqs};
        return decode_with(p, plan, scratch, cap, stream);
    }
    int splits = plan.splits;
    const int32_t rows = decode_rows(*p);
    if (inkling_attn_decode_workspace_bytes(rows, p->num_q_heads, splits) > cap) {
        if (p->num_splits > 0)
            return fail(INKLING_ERR_INVALID,
                        "num_splits %d needs %zu bytes of partials; the static scratch holds %zu "
                        "(use fewer splits, or inkling_attn_decode with a workspace)",
                        splits, inkling_attn_decode_workspace_bytes(rows, p->num_q_heads, splits),
                        cap);
        // automatic split count: the largest that fits (1 needs no scratch)
        while (splits > 1 && inkling_attn_decode_workspace_bytes(rows, p->num_q_heads, splits) > cap)
            --splits;
    }
    return decode_with(p, DecodePlan{splits, splits == 1 ? p->num_seqs : 0}, scratch, cap, stream);
}

static inkling_status decode_with(const inkling_decode_params *p, const DecodePlan &plan,
                                  void *workspace, size_t workspace_bytes, inkling_stream_t stream) {
    inkling_status st;
    const int splits = plan.splits;
    // one thread block per (sequence, kv head, split): the grid must fit a
    // signed 32-bit count
    if ((long)p->num_seqs * p->num_kv_heads * splits >= (1L << 31))
        return fail(INKLING_ERR_UNSUPPORTED, "num_seqs * num_kv_heads * splits (%d) exceeds 2^31",
                    splits);
    if (splits > 1) {
        // the combine pass runs one thread block per output row
        if ((long)decode_rows(*p) * p->num_q_heads >= (1L << 31))
            return fail(INKLING_ERR_UNSUPPORTED, "%ld output rows to combine exceed 2^31",
                        (long)decode_rows(*p) * p->num_q_heads);
        const size_t need = plan_workspace(*p, plan);
        if (!workspace || workspace_bytes < need)
            return fail(INKLING_ERR_INVALID, "workspace of %zu bytes given, %zu needed for %d splits",
                        workspace_bytes, need, splits);
        if (!aligned16(workspace)) return fail(INKLING_ERR_INVALID, "workspace must be 16-byte aligned");
    }
    CUtensorMap tm_k, tm_v;
    const cuuint64_t rows = (cuuint64_t)p->num_blocks * p->num_kv_heads * 128;
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t str[1] = {256};
    if (p->q_len > 1) {
        // multi-token decode: half a block (64 tokens) per key/value box, and
        // the G x q_len query rows of a kv head in one 3-D box of
        // q viewed as (d, head, sequence x token)
        const int G = p->num_q_heads / p->num_kv_heads;
        cuuint32_t box[2] = {64, 64};
        if ((st = make_map(&tm_k, p->k_cache, 2, dims, str, box)) != INKLING_OK) return st;
        if ((st = make_map(&tm_v, p->v_cache, 2, dims, str, box)) != INKLING_OK) return st;
        CUtensorMap tm_q;
        const cuuint64_t Hq = (cuuint64_t)p->num_q_heads;
        cuuint64_t qd[3] = {128, Hq, (cuuint64_t)p->num_seqs * p->q_len};
        cuuint64_t qs[2] = {256, Hq * 256};
        cuuint32_t qb[3] = {64, (cuuint32_t)G, (cuuint32_t)p->q_len};
        if ((st = make_map(&tm_q, p->q, 3, qd, qs, qb)) != INKLING_OK) return st;
        cudaError_t e = launch_attn_decode_mq(*p, splits, plan.s_whole, workspace, tm_q, tm_k,
                                              tm_v, (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_fail(e, "attn_decode (multi-token) launch");
        return INKLING_OK;
    }
    cuuint32_t box[2] = {64, 64};
    if ((st = make_map(&tm_k, p->k_cache, 2, dims, str, box)) != INKLING_OK) return st;
    if ((st = make_map(&tm_v, p->v_cache, 2, dims, str, box)) != INKLING_OK) return st;
    cudaError_t e = launch_attn_decode(*p, splits, plan.s_whole, workspace, tm_k, tm_v,
                                       (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "attn_decode launch");
    return INKLING_OK;
}

}  // extern "C"
