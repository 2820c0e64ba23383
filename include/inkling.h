/*
 * inkling.h — C ABI of the Inkling decoder attention layer for NVIDIA B200
 * (sm_100a).
 *
 * The layer (vLLM Recipes page "thinkingmachines/Inkling", section Overview,
 * bullets "Attention" and "Short convolution"):
 *   1. a causal, depthwise, window-4 short convolution (sconv) over the key
 *      and value channels:  y[t,c] = sum_{k=0..3} w[c,k] * x[t-k,c], tap 0 =
 *      current token, rounded once to bf16 (round to nearest even);
 *   2. grouped-query attention at head size 128 in which RoPE is replaced by
 *      a learned relative-position term added to the pre-softmax logits:
 *        s[i,j] = (q_i . k_j) / sqrt(128) + bias[h, min(i-j, D_max)]
 *      with query head h reading kv head h / (Hq/Hkv);
 *   3. a sliding-window mask (j allowed iff 0 <= i-j < window) or full causal
 *      mask (window = 0); the pages split the 66 layers into 55 sliding-window
 *      and 11 full-attention ones.
 * The sconv state is kept like the KV cache of a sliding-window layer (same
 * Overview bullet); the paged KV cache uses 128-token blocks (the
 * `--block-size 128` launch option in section Client Usage of the same page).
 *
 * Conventions shared by every entry point
 *  - bf16 tensors are passed as `const void*` / `void*` (IEEE bfloat16 bits);
 *    layouts are row-major, last index contiguous.
 *  - Every pointer named "device" must point to device memory of the current
 *    CUDA device and be 16-byte aligned.  The caller owns all memory; the
 *    library allocates nothing and keeps no state except a per-thread error
 *    message (and the scratch array of inkling_attn_decode_static).
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *    never synchronise.  Kernel faults surface at the caller's next
 *    synchronisation, as with any CUDA launch.
 *  - On invalid arguments a call returns INKLING_ERR_INVALID (or
 *    INKLING_ERR_UNSUPPORTED for shapes outside what the kernels implement)
 *    and launches nothing; inkling_last_error() describes why.  A failed
 *    launch returns INKLING_ERR_CUDA.  No C++ exception crosses this ABI.
 *  - `status` (optional, nullable, device int32): kernels OR error bits into it
 *    (INKLING_STATUS_* below) instead of trapping; the caller zeroes it and
 *    reads it after synchronising.
 *  - Failures found on the device cannot be return codes: the calls return
 *    before their kernels run.  A kernel that meets one reports it through
 *    `status`, and every output row it could not compute (a bounded wait that
 *    gave up, a decode sequence length outside [1, max_blocks*128]) is
 *    written as NaN, in `out` and `lse` alike, so a caller that passes
 *    status = NULL still cannot mistake it for a result.  A block-table
 *    entry outside [0, num_blocks) is reported only through `status`: a
 *    kernel reads block 0 in its place (the rows are finite but wrong) and
 *    skips a write to it.
 *  - Paged caches: the attention kernels read whole 128-token blocks and give
 *    the slots past a sequence's length zero weight (0 * x).  Those slots
 *    must therefore hold finite values (a pool cleared once, or values these
 *    calls wrote before); NaN or Inf bits there would reach the output.  The
 *    scratch blocks of the two-pass prefill are zeroed past each end.
 */
#ifndef INKLING_H
#define INKLING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *inkling_stream_t; /* same type as cudaStream_t */

typedef enum {
    INKLING_OK = 0,
    INKLING_ERR_INVALID = 1,     /* bad pointer / shape / size; nothing launched */
    INKLING_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim != 128) */
    INKLING_ERR_CUDA = 3         /* a CUDA runtime / driver call failed */
} inkling_status;

/* bits a kernel may OR into the optional device status word */
#define INKLING_STATUS_TIMEOUT 1      /* a bounded wait inside a kernel gave up */
#define INKLING_STATUS_BAD_BLOCK 2    /* a block-table entry was outside [0, num_blocks) */
#define INKLING_STATUS_BAD_LENGTH 4   /* a sequence length was outside [1, max_blocks*128] */

/* Head dimension and paged-cache block size the kernels are built for. */
#define INKLING_HEAD_DIM 128
#define INKLING_BLOCK_SIZE 128

/* Message for the last failed call on this host thread ("" if none). */
const char *inkling_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int inkling_version(void);

/* Self-test of failure detection (the pages have no counterpart).  Every wait
 * inside the kernels is bounded: when a wait runs out, the kernel ORs
 * INKLING_STATUS_TIMEOUT into the status word and returns instead of hanging,
 * and the CUDA context stays usable.  This call launches one block that waits,
 * with a limit of limit_us microseconds (1 .. 10^7), on a barrier that nothing
 * will ever arrive on, so the caller can check that path end to end.  status:
 * device int32, zeroed by the caller. */
inkling_status inkling_selftest_wait_timeout(int32_t *status, uint32_t limit_us,
                                             inkling_stream_t stream);

/* --------------------------------------------------------------------------
 * inkling_sconv_kv — decode-side sconv append (Overview, "Short convolution":
 * the sconv on keys and values, with its state kept as a sliding-window
 * cache).
 *
 * For every sequence s and each of its n_new new tokens (positions
 * L-n_new .. L-1, L = seq_lens[s]) the raw key and value are convolved with
 * the 3 previous raw tokens (from the rolling state, then from the earlier
 * new tokens), rounded to bf16 and written to their slot of the paged cache:
 * block block_table[s, pos/128], slot pos%128.  The state then holds the last
 * 3 raw tokens.  Arithmetic: fp32, taps applied oldest first
 * (w3*x[t-3] + w2*x[t-2] + w1*x[t-1] + w0*x[t], fused multiply-adds), one
 * bf16 rounding.
 * -------------------------------------------------------------------------- */
typedef struct {
    const void *k_new;           /* device [S, n_new, Hkv, d] bf16 raw keys */
    const void *v_new;           /* device [S, n_new, Hkv, d] bf16 raw values */
    const float *w_k;            /* device [Hkv*d, 4] fp32 key taps (tap 0 = current) */
    const float *w_v;            /* device [Hkv*d, 4] fp32 value taps */
    void *k_state;               /* device [S, 3, Hkv*d] bf16 raw key history, oldest first; updated */
    void *v_state;               /* device [S, 3, Hkv*d] bf16 raw value history; updated */
    void *k_cache;               /* device [num_blocks, Hkv, 128, d] bf16; new slots written */
    void *v_cache;               /* device [num_blocks, Hkv, 128, d] bf16 */
    const int32_t *block_table;  /* device [S, max_blocks] */
    const int32_t *seq_lens;     /* device [S], lengths after the append, >= n_new */
    int32_t *status;             /* device int32 or NULL */
    int32_t num_seqs;            /* S >= 0 (0 = nothing to do) */
    int32_t n_new;               /* new tokens per sequence, 1..2^20 (a decode step or a prefill chunk) */
    int32_t num_kv_heads;        /* Hkv >= 1 */
    int32_t head_dim;            /* d, must be 128 */
    int32_t max_blocks;          /* columns of block_table */
    int32_t num_blocks;          /* blocks in the cache pool */
} inkling_sconv_params;

inkling_status inkling_sconv_kv(const inkling_sconv_params *p, inkling_stream_t stream);

/* --------------------------------------------------------------------------
 * inkling_attn_prefill — prefill attention over a whole prompt, the sconv of
 * its keys and values included (Overview, "Attention" and "Short
 * convolution"; the relative term is the FA4 "sheared-bias" kernel named in
 * section Performance).
 *
 * Every query row i of every sequence attends to keys j of the same sequence
 * with 0 <= i-j (< window when window > 0).  Keys and values are the sconv of
 * k_raw / v_raw with zero history before t = 0, rounded to bf16, exactly as
 * inkling_sconv_kv would write them.  Logits use scale 1/sqrt(128) on q.k and
 * add bias[h, min(i-j, d_max)] unscaled; softmax and accumulation are fp32,
 * probabilities enter the P.V product as bf16, the output is rounded to bf16.
 *
 * Optional cache fill in the same pass (the sconv state is managed like the
 * KV cache of a sliding-window layer, Overview, "Short convolution"): when
 * k_cache, v_cache and block_table are given, the post-sconv keys and values
 * of tokens 0..T-1 of sequence b are also written to the paged cache, token t
 * at slot t%128 of block block_table[b, t/128], bit for bit what
 * inkling_sconv_kv writes when it appends the T tokens to an empty sequence.
 * Slots at positions >= T are not touched.  When k_state and v_state are also
 * given, they receive the new sconv state: the raw rows T-3..T-1 (zero where
 * negative), oldest first, so that inkling_sconv_kv continues the sequence.
 * A block id outside [0, num_blocks) sets INKLING_STATUS_BAD_BLOCK in *status
 * and that tile is not written.  With B = 0 or T = 0 nothing is written.
 *
 * Execution path (`path`).  Both paths give the same bits: the same tensor-core
 * accumulation order and softmax code over the same post-sconv keys and
 * values (the sconv arithmetic is shared with inkling_sconv_kv).
 *  - INKLING_PREFILL_FUSED: one kernel; the sconv is applied to each raw
 *    key/value tile in shared memory on its way to the tensor cores (and
 *    written to the cache from there when one is given).  Every thread block
 *    whose window covers a key tile converts it again.
 *  - INKLING_PREFILL_TWO_PASS: two kernels.  First the sconv of every key and
 *    value, written once in the paged layout [block, Hkv, 128, d]: into the
 *    caller's cache through block_table when one is given (the call is then
 *    inkling_sconv_kv appending T tokens to empty sequences, with the state
 *    written as above), else into `workspace`, where sequence b owns blocks
 *    b*ceil(T/128) ...  Then the paged prefill kernel of
 *    inkling_attn_prefill_paged over those blocks, every sequence one chunk
 *    of T rows.  With a cache, a bad block id also spoils the attention rows
 *    that read that block (block 0 is read in its place).  Needs
 *    num_blocks*Hkv*128 < 2^31 and B*T*Hq < 2^31 (the workspace blocks
 *    count when there is no cache); without a cache, workspace_bytes must be
 *    at least inkling_attn_prefill_workspace_bytes(p).
 *  - INKLING_PREFILL_AUTO: the two-pass path when B*T >= INKLING_PREFILL_TWO_PASS_MIN_TOKENS
 *    and T >= INKLING_PREFILL_TWO_PASS_MIN_T, and it is possible (a cache, or a
 *    large enough workspace, and the size limits above), else the fused one.
 *    On B200 the two-pass path is 9-23% faster there (the conversion is done
 *    once per token rather than once per covering block, for ~1.6% extra HBM
 *    traffic), and the fused one is faster on smaller calls (one launch
 *    instead of two, and its CTA pairs share each tile).
 * -------------------------------------------------------------------------- */
#define INKLING_PREFILL_AUTO 0
#define INKLING_PREFILL_FUSED 1
#define INKLING_PREFILL_TWO_PASS 2
#define INKLING_PREFILL_TWO_PASS_MIN_TOKENS 2048
#define INKLING_PREFILL_TWO_PASS_MIN_T 512

typedef struct {
    const void *q;        /* device [B, T, Hq, d] bf16 */
    const void *k_raw;    /* device [B, T, Hkv, d] bf16, before sconv */
    const void *v_raw;    /* device [B, T, Hkv, d] bf16, before sconv */
    const float *w_k;     /* device [Hkv*d, 4] fp32 */
    const float *w_v;     /* device [Hkv*d, 4] fp32 */
    const float *bias;    /* device [Hq, d_max+1] fp32 relative-position table */
    void *out;            /* device [B, T, Hq, d] bf16 */
    float *lse;           /* device [B, Hq, T] fp32 natural-log row logsumexp, or NULL */
    int32_t *status;      /* device int32 or NULL */
    int32_t batch;        /* B >= 0 */
    int32_t seq_len;      /* T >= 0 */
    int32_t num_q_heads;  /* Hq, a multiple of Hkv */
    int32_t num_kv_heads; /* Hkv >= 1 */
    int32_t head_dim;     /* d, must be 128 */
    int32_t window;       /* 0 = full causal, else keys with i-j < window */
    int32_t d_max;        /* bias table has d_max+1 entries per head, d_max >= 0 */
    /* optional cache fill (all NULL = none; k_cache, v_cache and block_table together) */
    void *k_cache;              /* device [num_blocks, Hkv, 128, d] bf16, or NULL */
    void *v_cache;              /* device [num_blocks, Hkv, 128, d] bf16, or NULL */
    const int32_t *block_table; /* device [B, max_blocks] int32, or NULL */
    int32_t max_blocks;         /* columns of block_table, max_blocks*128 >= T */
    int32_t num_blocks;         /* blocks in the cache pool */
    void *k_state;              /* device [B, 3, Hkv*d] bf16 out, or NULL (with v_state) */
    void *v_state;              /* device [B, 3, Hkv*d] bf16 out, or NULL (with k_state) */
    /* execution path and scratch */
    int32_t path;               /* INKLING_PREFILL_AUTO / _FUSED / _TWO_PASS */
    void *workspace;            /* device scratch of the two-pass path without a cache, or NULL */
    size_t workspace_bytes;     /* bytes at workspace */
} inkling_prefill_params;

inkling_status inkling_attn_prefill(const inkling_prefill_params *p, inkling_stream_t stream);

/* Bytes of workspace inkling_attn_prefill(p) uses: 2 * B * ceil(T/128) * Hkv
 * * 128 * 128 * 2 (post-sconv keys and values in the paged layout) when p's
 * path is TWO_PASS, or AUTO with B*T >= INKLING_PREFILL_TWO_PASS_MIN_TOKENS
 * and T >= INKLING_PREFILL_TWO_PASS_MIN_T, with no cache given; 0 when the
 * call needs none (the fused path, a cache given, B or T zero) or p is NULL.
 * Only the sizes, path and cache pointer of p are read. */
size_t inkling_attn_prefill_workspace_bytes(const inkling_prefill_params *p);

/* --------------------------------------------------------------------------
 * inkling_sconv_out — the window-4 short convolution on the attention output
 * (vLLM Recipes "thinkingmachines/Inkling", Overview, "Short convolution":
 * four sconv modules per layer, on keys, values, output and MoE output).
 *
 * y[b,t,c] = sum_{k=0..3} w[c,k] * x[b,t-k,c] for the C channels of the
 * attention output (C = Hq*128, before the output projection).  The 3 raw
 * rows before t = 0 come from state (oldest first), or are zero when state is
 * NULL.  A non-NULL state is then updated in place to the last 3 raw rows of
 * (old state, x), so a decode step or a prefill chunk continues where the
 * previous one stopped.
 *
 * Arithmetic: fp32, taps applied oldest first with fused multiply-adds, one
 * bf16 rounding (as inkling_sconv_kv).  x and y must not overlap.
 * -------------------------------------------------------------------------- */
typedef struct {
    const void *x;       /* device [B, T, C] bf16 */
    const float *w;      /* device [C, 4] fp32 taps (tap 0 = current token) */
    void *state;         /* device [B, 3, C] bf16 raw history, or NULL (zero history) */
    void *y;             /* device [B, T, C] bf16 */
    int32_t batch;       /* B >= 0 */
    int32_t seq_len;     /* T >= 0 */
    int32_t channels;    /* C, a positive multiple of 8 */
} inkling_sconv_out_params;

inkling_status inkling_sconv_out(const inkling_sconv_out_params *p, inkling_stream_t stream);

/* --------------------------------------------------------------------------
 * inkling_sconv_out_sharded — the output sconv sharded over channels across
 * n_ranks tensor-parallel ranks, fused with its reduce-scatter and
 * all-gather (vLLM Recipes "thinkingmachines/Inkling": Overview, "Short
 * convolution", which shards the sconv across the channel dimension with a
 * reduce-scatter / all-gather so that its cache and compute are not
 * replicated on every rank; Performance, "sconv-aware TP sharding", where
 * each rank stores only its channel shard of the sconv cache).
 *
 * Each rank holds a partial sum x_r [B, T, C] of the sconv's input (the
 * output of a row-parallel projection).  The call made on rank `rank`
 * computes the channels c in [rank*Cs, (rank+1)*Cs), Cs = C / n_ranks:
 *   s[b,t,c] = bf16( x_0[b,t,c] + x_1[b,t,c] + ... )   (fp32, rank order)
 *   y[b,t,c] = sum_{k=0..3} w[c,k] * s[b,t-k,c]        (as inkling_sconv_out)
 * and stores y[:, :, shard] into the output buffer of EVERY rank, so that
 * after all ranks' calls each y_r holds the full y.  The 3 rows of s before
 * t = 0 come from `state`, this rank's shard [B, 3, Cs] of the sconv state
 * (or zero when NULL), which is then updated in place to the last 3 rows of
 * (old state, s).
 *
 * Pointers: x_parts and y_parts are HOST arrays of n_ranks device pointers.
 * Every one of them must be readable / writable from the current device:
 * this GPU's own memory, or a peer's memory mapped into this process (CUDA
 * IPC, symmetric memory, or peer access).  The kernel reads and writes them
 * with plain 16-byte loads and stores (no TMA, no multicast).  The arrays
 * themselves are copied at the call and may be freed after it returns.
 * Ordering is the caller's: every x_r must be complete before any rank's call
 * starts, and a rank may read its y only after every rank's call has ended
 * (e.g. a cross-rank barrier before and after).  No x_r may overlap any y_r.
 * Errors: n_ranks outside [1, INKLING_SHARD_MAX_RANKS], rank outside
 * [0, n_ranks), C not a positive multiple of 8 * n_ranks, or a NULL pointer:
 * INKLING_ERR_INVALID, nothing launched.
 * -------------------------------------------------------------------------- */
#define INKLING_SHARD_MAX_RANKS 8

typedef struct {
    const void *const *x_parts; /* host [n_ranks]: device [B, T, C] bf16 partial sums */
    void *const *y_parts;       /* host [n_ranks]: device [B, T, C] bf16 outputs */
    const float *w;             /* device [C, 4] fp32 taps of all channels (tap 0 = current) */
    void *state;                /* device [B, 3, C/n_ranks] bf16 state shard, or NULL */
    int32_t n_ranks;            /* 1 .. INKLING_SHARD_MAX_RANKS */
    int32_t rank;               /* the channel shard this call computes, 0 .. n_ranks-1 */
    int32_t batch;              /* B >= 0 */
    int32_t seq_len;            /* T >= 0 */
    int32_t channels;           /* C, a positive multiple of 8 * n_ranks */
} inkling_sconv_out_sharded_params;

inkling_status inkling_sconv_out_sharded(const inkling_sconv_out_sharded_params *p,
                                         inkling_stream_t stream);

/* --------------------------------------------------------------------------
 * inkling_attn_prefill_paged — chunked prefill over the paged cache.
 *
 * A chunk of new tokens per sequence (variable lengths, rows packed): the
 * chunk's queries attend to the whole sequence so far through the paged cache
 * of post-sconv keys and values (vLLM Recipes "thinkingmachines/Inkling",
 * Overview: "Attention", and "Short convolution", whose cache is managed like
 * a sliding-window layer's KV cache; Client Usage: 128-token blocks).
 *
 * Call order for one chunk:
 *  1. inkling_sconv_kv with n_new = the chunk length.  It convolves the
 *     chunk's raw keys and values, continuing from the rolling 3-token state,
 *     and writes them into the cache.
 *  2. This call.
 *
 * Sequence s has n_s = cu_q[s+1] - cu_q[s] new tokens and length
 * L_s = seq_lens[s] after them.  Its query r (packed row cu_q[s] + r) sits at
 * position L_s - n_s + r and sees keys j <= that position, inside the window,
 * with the bias at distance position - j.  The rows equal rows
 * L_s - n_s .. L_s - 1 of inkling_attn_prefill on the whole sequence.
 *
 * Sequences with n_s = 0 produce nothing.
 *  - n_s > max_q, n_s < 0 or L_s < n_s: INKLING_STATUS_BAD_LENGTH.  Rows
 *    past max_q are not written.
 *  - A block id outside [0, num_blocks): INKLING_STATUS_BAD_BLOCK (block 0
 *    is read instead).
 * -------------------------------------------------------------------------- */
typedef struct {
    const void *q;               /* device [total_q, Hq, d] bf16, rows of all sequences packed */
    const int32_t *cu_q;         /* device [S+1] nondecreasing row offsets, cu_q[0] = 0 */
    const void *k_cache;         /* device [num_blocks, Hkv, 128, d] bf16, post-sconv */
    const void *v_cache;         /* device [num_blocks, Hkv, 128, d] bf16, post-sconv */
    const int32_t *block_table;  /* device [S, max_blocks] */
    const int32_t *seq_lens;     /* device [S] lengths including the new tokens */
    const float *bias;           /* device [Hq, d_max+1] fp32 */
    void *out;                   /* device [total_q, Hq, d] bf16 */
    float *lse;                  /* device [total_q, Hq] fp32 natural-log row logsumexp, or NULL */
    int32_t *status;             /* device int32 or NULL */
    int32_t num_seqs;            /* S >= 0 */
    int32_t total_q;             /* rows of q / out (= cu_q[S]) */
    int32_t max_q;               /* >= every n_s (sizes the grid) */
    int32_t num_q_heads;         /* Hq, a multiple of Hkv */
    int32_t num_kv_heads;        /* Hkv >= 1 */
    int32_t head_dim;            /* d, must be 128 */
    int32_t max_blocks;          /* columns of block_table */
    int32_t num_blocks;          /* blocks in the pool */
    int32_t window;              /* 0 = full causal, else keys with i-j < window */
    int32_t d_max;               /* >= 0 */
} inkling_prefill_paged_params;

inkling_status inkling_attn_prefill_paged(const inkling_prefill_paged_params *p,
                                          inkling_stream_t stream);

/* --------------------------------------------------------------------------
 * inkling_attn_decode — decode over the paged cache, split-KV.
 *
 * For sequence s with length L = seq_lens[s], the query q[s] sits at position
 * L-1 and attends to positions max(0, L-window) .. L-1 (0 .. L-1 when
 * window = 0), read through block_table, with the same logits as prefill.
 *
 * Multi-token decode (q_len >= 2): the draft tokens of speculative decoding /
 * multi-token prediction (vLLM Recipes "thinkingmachines/Inkling", Overview,
 * MTP bullet: 8 chained MTP heads, up to 9 tokens per forward step).  The
 * q_len newest tokens of each sequence, already appended to the cache, are
 * all queries: q [S, q_len, Hq, d]; query qi sits at position
 * i = L - q_len + qi and sees keys j <= i (and i - j < window), with the bias
 * at distance i - j, so the draft tokens are causal among themselves.
 * out [S, q_len, Hq, d], lse [S, q_len, Hq].  Needs seq_lens[s] >= q_len
 * (else INKLING_STATUS_BAD_LENGTH) and G * q_len <= 80.
 * The key range of every sequence is cut into num_splits parts that run on
 * separate thread blocks; their partial (max, sum, unnormalised output)
 * triples go to the caller's workspace and a second kernel merges them.
 * -------------------------------------------------------------------------- */
typedef struct {
    const void *q;               /* device [S, Hq, d] bf16 ([S, q_len, Hq, d] if q_len >= 2) */
    const void *k_cache;         /* device [num_blocks, Hkv, 128, d] bf16, post-sconv */
    const void *v_cache;         /* device [num_blocks, Hkv, 128, d] bf16, post-sconv */
    const int32_t *block_table;  /* device [S, max_blocks] */
    const int32_t *seq_lens;     /* device [S], each in [1, max_blocks*128] */
    const float *bias;           /* device [Hq, d_max+1] fp32 */
    void *out;                   /* device [S, Hq, d] bf16 ([S, q_len, Hq, d] if q_len >= 2) */
    float *lse;                  /* device [S, Hq] fp32 ([S, q_len, Hq]) or NULL */
    int32_t *status;             /* device int32 or NULL */
    int32_t num_seqs;            /* S >= 0 */
    int32_t num_q_heads;         /* Hq = G * Hkv with 1 <= G <= 8 */
    int32_t num_kv_heads;        /* Hkv >= 1 */
    int32_t head_dim;            /* d, must be 128 */
    int32_t max_blocks;          /* columns of block_table */
    int32_t num_blocks;          /* blocks in the pool */
    int32_t window;              /* 0 = full */
    int32_t d_max;               /* >= 0 */
    int32_t num_splits;          /* 0 = choose from the SM count, else 1..1024 */
    int32_t q_len;               /* query tokens per sequence: 0 or 1 = one, 2..10 = multi-token */
} inkling_decode_params;

/* Workspace bytes inkling_attn_decode needs for num_splits splits (pass the
 * value the call will use, or the result of inkling_attn_decode_num_splits).
 * For multi-token decode pass num_seqs * q_len as num_seqs.
 * Returns 0 for invalid arguments. */
size_t inkling_attn_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                           int32_t num_splits);

/* The split count to size the workspace for (resolves num_splits = 0);
 * returns 0 for invalid parameters.  With num_splits = 0 it is the count the
 * call uses: for every sequence, or, when the (sequence, kv head) units fill
 * the SMs, for the sequences past those that fill whole waves (those run
 * unsplit).  A call with num_splits = 0 whose workspace is smaller than that
 * count needs runs every sequence unsplit instead. */
int32_t inkling_attn_decode_num_splits(const inkling_decode_params *p);

/* workspace: device, >= inkling_attn_decode_workspace_bytes(...) bytes, 16-byte
 * aligned, contents need no initialisation; not used when the split count is 1. */
inkling_status inkling_attn_decode(const inkling_decode_params *p, void *workspace,
                                   size_t workspace_bytes, inkling_stream_t stream);

/* --------------------------------------------------------------------------
 * inkling_attn_decode_static — inkling_attn_decode with no caller workspace.
 *
 * The pages have no counterpart to this call.  It serves callers that can
 * hand the library only their inputs and outputs and cannot obtain device
 * memory for a workspace: code running under an allocator that owns the whole
 * device and forbids other allocations, or a latency-critical decode loop in
 * which an allocation (which may synchronise the device) is not acceptable.
 *
 * Same arguments and results as inkling_attn_decode.  The split partials go
 * to an 8 MiB array that the library holds in device memory on every GPU
 * that loads it, until the process exits; no allocation routine is called.
 *  - The first call on a device asks the runtime for that array's address on
 *    the current device; make that first call before any stream capture.
 *    The address is kept with the id of the CUDA context it belongs to and is
 *    asked for again when another context is current (after cudaDeviceReset,
 *    or under a context the caller created), so such a call is again a
 *    first call.
 *  - With num_splits = 0 the split count is lowered, if needed, until the
 *    partials fit (one split needs none).  An explicit num_splits whose
 *    partials exceed 8 MiB returns INKLING_ERR_INVALID and launches nothing.
 *  - All calls share the array and it keeps the last call's contents.  Every
 *    partial a call reads is written earlier by the same call (a split that
 *    cannot compute its rows writes a NaN partial, never leaves the slot
 *    alone), so nothing needs clearing, but calls that overlap on the GPU
 *    (e.g. on two streams at once, on one device) race with each other:
 *    serialise them.
 * -------------------------------------------------------------------------- */
inkling_status inkling_attn_decode_static(const inkling_decode_params *p, inkling_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* INKLING_H */
