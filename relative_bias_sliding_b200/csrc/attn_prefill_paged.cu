// attn_prefill_paged.cu — chunked prefill over the paged cache: the query rows
// of a chunk of new tokens per sequence (variable lengths, packed) attend to
// the whole sequence so far, read from the paged cache of post-sconv keys and
// values (vLLM Recipes "thinkingmachines/Inkling", Overview: "Attention" and
// "Short convolution" — the sconv cache is managed like the KV cache of a
// sliding-window layer; Client Usage: 128-token blocks).  The chunk's keys and
// values go into the cache first, with inkling_sconv_kv (n_new = chunk
// length), which continues the sconv from the rolling 3-token state; this
// kernel then computes rows L-n .. L-1 of the prefill of a sequence of length
// L, exactly what a prefill of the whole sequence gives for those rows.
//
// Same numerics and softmax as attn_prefill.cu (shared softmax role).  One
// thread block = one (sequence, query head, 256-row block of the chunk): two
// 128-row query tiles; TMEM S0 | S1 | O0 | O1.  A 128-token cache block is
// exactly one key tile, loaded by TMA straight into the MMA operand layout
// (two 64-column halves, 128-byte swizzle), so there is no sconv stage.
//
// Warp roles (16 warps): 0-7 softmax of the two query tiles, 12 TMA producer
// (queries once, then the key and value block of every key tile through the
// block table), 13 TMEM allocator and MMA issuer, 8-11 and 14-15 idle.
// Key/value stages: 2.  Rows of the last query tile past the chunk end are
// computed but not stored.
//
// The same kernel is the second pass of the two-pass dense prefill
// (inkling_attn_prefill): there every sequence is one chunk of T rows over an
// empty history, so cu_q and seq_lens are NULL (sequence s has rows s*T ..
// s*T+T-1 and length T), the block table is the caller's cache table or NULL
// for the scratch cache (sequence s owns blocks s*max_blocks ... in order),
// and the row log-sum-exp goes to the dense [B, Hq, T] layout.
#include "prefill_common.cuh"

namespace inkling {

constexpr uint32_t PG_Q = 0;             // 2 query tiles x 32 KB
constexpr uint32_t PG_K = 65536;         // 2 stages x 32 KB
constexpr uint32_t PG_V = 131072;        // 2 stages x 32 KB
constexpr uint32_t PG_BIAS = 196608;     // 2 softmax groups x 2 buffers x 4 copies x 264 fp32
constexpr uint32_t PG_BAR = PG_BIAS + kBiasBytes;
constexpr int kPagedSmem = PG_BAR + 512 + 1024;

enum {
    G_QFULL = 0,
    G_KFULL = 1,   // +stage
    G_VFULL = 3,
    G_KEMPTY = 5,
    G_VEMPTY = 7,
    G_SFULL = 9,   // +tile
    G_PFULL = 11,
    G_ODONE = 13,
    G_DRAIN = 15,
    G_COUNT = 16
};

struct PagedArgs {
    PrefillArgs pa;  // bias, d_max, window, status, Hq, Hkv (the softmax role's view)
    const int32_t *cu_q, *block_table, *seq_lens;  // cu_q / seq_lens NULL: dense rows
    uint16_t *out;
    float *lse;
    int S, max_blocks, num_blocks, nqb;
    int dense_T;  // rows (and length) of every sequence when cu_q is NULL
};

// Epilogue of a chunk row: 16-byte global stores of the rows inside the chunk.
struct RowStoreEpilogue {
    uint16_t *out;
    float *lse;
    long row0;       // packed row index of tile row 0
    int rows_valid;  // tile rows inside the chunk
    int Hq, h;
    int dense_T;     // 0: lse [rows, Hq]; else lse [B, Hq, T] with T = dense_T
    INK_DEV long lse_at(int u) const {
        const long r = row0 + u;
        if (!dense_T) return r * Hq + h;
        const long b = r / dense_T;
        return (b * Hq + h) * dense_T + (r - b * dense_T);
    }
    INK_DEV void operator()(bool have_o, int u, int, float l, float m_ref, uint32_t o_col,
                            volatile int *) const {
        const bool store = u < rows_valid;
        uint16_t *dst = out + ((row0 + u) * Hq + h) * 128;
        if (!have_o) {
            // a bounded wait gave up: the row reads NaN (the status word says why)
            if (store) {
                const uint32_t nb = 0x7fc07fc0u;
#pragma unroll
                for (int c = 0; c < 16; ++c) *(uint4 *)(dst + c * 8) = make_uint4(nb, nb, nb, nb);
                if (lse) lse[lse_at(u)] = __int_as_float(0x7fc00000);
            }
            return;  // warp-uniform: emit_row's TMEM loads need the whole warp
        }
        emit_row(o_col, l, [&](int c, uint4 v) {
            if (store) *(uint4 *)(dst + c * 8) = v;
        });
        if (lse && store) lse[lse_at(u)] = (l > 0.f) ? m_ref + __logf(l) : -INFINITY;
    }
};

__global__ void __launch_bounds__(512, 1)
attn_prefill_paged_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const PagedArgs g) {
    const PrefillArgs &a = g.pa;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- work item: CTAs run grouped by (sequence, kv head), so the CTAs
    // resident at one time read the same cache blocks (they stay in L2); inside
    // a group the later (longer) query blocks come first.
    const int G = a.Hq / a.Hkv;
    const int per_group = g.nqb * G;
    const int grp = (int)(blockIdx.x / per_group), rem = (int)(blockIdx.x % per_group);
    const int s = grp / a.Hkv;
    const int kvh = grp % a.Hkv;
    const int qb = g.nqb - 1 - rem / G;
    const int h = kvh * G + rem % G;
    const bool dense = g.cu_q == nullptr;
    const int q_begin = dense ? s * g.dense_T : g.cu_q[s];
    const int n = dense ? g.dense_T : g.cu_q[s + 1] - q_begin;  // query rows of this sequence
    const int L = g.seq_lens ? g.seq_lens[s] : g.dense_T;
    const int base = L - n;                 // position of the first new token
    if (n < 0 || base < 0 || L > g.max_blocks * 128) {
        if (threadIdx.x == 0 && qb == 0 && h == 0) report_status(a.status, INKLING_STATUS_BAD_LENGTH);
        return;
    }
    if (threadIdx.x == 0 && qb == g.nqb - 1 && h == 0 && n > g.nqb * kQRows)
        report_status(a.status, INKLING_STATUS_BAD_LENGTH);  // rows past max_q are not computed
    if (qb * kQRows >= n) return;  // the whole block: nothing of this sequence here

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bar = (uint64_t *)(smem + PG_BAR);
    uint32_t *tmem_slot = (uint32_t *)(bar + G_COUNT);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    int r0[2], lo[2], hi[2];
    bool ok[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        r0[t] = qb * kQRows + t * 128;  // chunk row of tile row 0
        ok[t] = r0[t] < n;
        const int last = base + min(r0[t] + 127, n - 1);
        hi[t] = last >> 7;
        lo[t] = (a.window > 0) ? (max(0, base + r0[t] - a.window + 1) >> 7) : 0;
    }
    const int ulo = lo[0];
    const int uhi = ok[1] ? hi[1] : hi[0];

    // ---- setup
    if (threadIdx.x == 0) {
        for (int i = 0; i < G_COUNT; ++i)
            mbar_init(&bar[i], (i == G_PFULL || i == G_PFULL + 1) ? 128 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 13) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp < 8) {
        // ================================================== softmax (2 WGs) ==
        setmaxnreg_inc184();
        const int t = warp >> 2;
        if (ok[t])
            softmax_role(a, (float *)(smem + PG_BIAS) + t * 2 * kBiasBuf, &bar[G_SFULL],
                         &bar[G_ODONE], abort_flag, tbase, t, h, base + r0[t], L, lo[t], hi[t],
                         3 + t, 0, 0u, [&](int tt) { mbar_arrive(&bar[G_PFULL + tt]); },
                         RowStoreEpilogue{g.out, g.lse, (long)q_begin + r0[t], n - r0[t], a.Hq, h,
                                          dense ? g.dense_T : 0});
    } else if (warp < 12) {
        setmaxnreg_dec80();
    } else {
        setmaxnreg_dec64();
        if (warp == 12 && lane == 0) {
            // ============================================== TMA producer ==
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(&bar[G_QFULL], 65536);
            for (int t = 0; t < 2; ++t)
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_3d(smem + PG_Q + t * 32768 + hf * 16384, &tm_q, &bar[G_QFULL],
                                hf * 64, h, q_begin + r0[t]);
            int kis = 0, vis = 0;  // key / value tile loads issued
            for (int nt = ulo; nt <= uhi; ++nt) {
                const int it = nt - ulo, st = it & 1;
                const uint32_t ph = ((it >> 1) & 1) ^ 1;
                int blk = g.block_table ? g.block_table[(long)s * g.max_blocks + nt]
                                        : s * g.max_blocks + nt;
                if (blk < 0 || blk >= g.num_blocks) {
                    report_status(a.status, INKLING_STATUS_BAD_BLOCK);
                    blk = 0;  // keep the pipeline running on a valid block
                }
                const int row = (blk * a.Hkv + kvh) * 128;
                if (!mbar_wait(&bar[G_KEMPTY + st], ph, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&bar[G_KFULL + st], 32768);
                tma_load_2d(smem + PG_K + st * 32768, &tm_k, &bar[G_KFULL + st], 0, row);
                tma_load_2d(smem + PG_K + st * 32768 + 16384, &tm_k, &bar[G_KFULL + st], 64, row);
                ++kis;
                if (!mbar_wait(&bar[G_VEMPTY + st], ph, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&bar[G_VFULL + st], 32768);
                tma_load_2d(smem + PG_V + st * 32768, &tm_v, &bar[G_VFULL + st], 0, row);
                tma_load_2d(smem + PG_V + st * 32768 + 16384, &tm_v, &bar[G_VFULL + st], 64, row);
                ++vis;
            }
            // drain: every load issued has landed before the block may exit
            mbar_wait(&bar[G_QFULL], 0, nullptr, a.status);
            for (int k = max(0, kis - 2); k < kis; ++k)
                mbar_wait(&bar[G_KFULL + (k & 1)], (k >> 1) & 1, nullptr, a.status);
            for (int k = max(0, vis - 2); k < vis; ++k)
                mbar_wait(&bar[G_VFULL + (k & 1)], (k >> 1) & 1, nullptr, a.status);
        } else if (warp == 13 && lane == 0) {
            // ================================================ MMA issuer ==
            const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_pv = idesc_bf16(128, 128, 0, 1);
            auto in_range = [&](int t, int nt) { return ok[t] && nt >= lo[t] && nt <= hi[t]; };
            auto issue_qk = [&](int t, int st) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint64_t ad = sw128_desc(sb + PG_Q + t * 32768 + koff, 16, 1024);
                    const uint64_t bd = sw128_desc(sb + PG_K + st * 32768 + koff, 16, 1024);
                    umma_ss(tbase + t * 128, ad, bd, id_qk, ks > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](int t, int st, bool acc) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t bd = sw128_desc(sb + PG_V + st * 32768 + ks * 2048, 16384, 1024);
                    umma_ts(tbase + 256 + t * 128, tbase + t * 128 + ks * 8, bd, id_pv,
                            (acc || ks > 0) ? 1u : 0u);
                }
            };
            bool alive = mbar_wait(&bar[G_QFULL], 0, abort_flag, a.status);
            if (alive) alive = mbar_wait(&bar[G_KFULL], 0, abort_flag, a.status);
            if (alive) {
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (in_range(t, ulo)) {
                        issue_qk(t, 0);
                        tc_commit(&bar[G_SFULL + t]);
                    }
                tc_commit(&bar[G_KEMPTY]);
                int it = 0;
                for (int nt = ulo; nt <= uhi && alive; ++nt, ++it) {
                    const int st = it & 1, st1 = (it + 1) & 1;
                    const uint32_t ph1 = ((it + 1) >> 1) & 1;
                    if (!mbar_wait(&bar[G_VFULL + st], (it >> 1) & 1, abort_flag, a.status)) break;
                    const bool has_next = nt < uhi;
                    // the next key tile, checked before waiting for P (it was
                    // requested two tiles ago): the wait then stays off the
                    // P -> P.V -> QK^T -> S chain
                    bool got_next = has_next && mbar_wait(&bar[G_KFULL + st1], ph1, abort_flag,
                                                          a.status);
                    if (has_next && !got_next) break;
                    tc_fence_after();
                    for (int t = 0; t < 2 && alive; ++t) {
                        if (in_range(t, nt)) {
                            if (!mbar_wait(&bar[G_PFULL + t], (nt - lo[t]) & 1, abort_flag,
                                           a.status)) {
                                alive = false;
                                break;
                            }
                            tc_fence_after();
                            issue_pv(t, st, nt > lo[t]);
                        }
                        if (has_next && in_range(t, nt + 1)) {
                            if (!got_next) {
                                if (!mbar_wait(&bar[G_KFULL + st1], ph1, abort_flag, a.status)) {
                                    alive = false;
                                    break;
                                }
                                tc_fence_after();
                                got_next = true;
                            }
                            issue_qk(t, st1);
                            tc_commit(&bar[G_SFULL + t]);
                        }
                    }
                    if (!alive) break;
                    if (has_next) {
                        if (!got_next && !mbar_wait(&bar[G_KFULL + st1], ph1, abort_flag, a.status))
                            break;
                        tc_commit(&bar[G_KEMPTY + st1]);
                    }
                    tc_commit(&bar[G_VEMPTY + st]);
                    for (int t = 0; t < 2; ++t)
                        if (ok[t] && nt == hi[t]) tc_commit(&bar[G_ODONE + t]);
                }
            }
            // every MMA issued has completed before TMEM is released
            tc_commit(&bar[G_DRAIN]);
            mbar_wait(&bar[G_DRAIN], 0, nullptr, a.status);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

cudaError_t launch_attn_prefill_paged(const inkling_prefill_paged_params &p, const CUtensorMap &tm_q,
                                      const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                                      cudaStream_t stream, int dense_T) {
    PagedArgs g = {};
    g.pa.bias = p.bias;
    g.pa.status = p.status;
    g.pa.Hq = p.num_q_heads;
    g.pa.Hkv = p.num_kv_heads;
    g.pa.window = p.window;
    g.pa.d_max = p.d_max;
    g.cu_q = p.cu_q;
    g.block_table = p.block_table;
    g.seq_lens = p.seq_lens;
    g.out = (uint16_t *)p.out;
    g.lse = p.lse;
    g.S = p.num_seqs;
    g.max_blocks = p.max_blocks;
    g.num_blocks = p.num_blocks;
    g.nqb = (p.max_q + kQRows - 1) / kQRows;
    g.dense_T = dense_T;
    const long grid = (long)g.S * p.num_q_heads * g.nqb;
    if (grid == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_paged_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPagedSmem);
    if (e != cudaSuccess) return e;
    attn_prefill_paged_kernel<<<(unsigned)grid, 512, kPagedSmem, stream>>>(tm_q, tm_k, tm_v, g);
    return cudaGetLastError();
}

}  // namespace inkling
