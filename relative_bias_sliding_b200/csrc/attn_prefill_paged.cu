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
// work item = one (sequence, query head, 256-row block of the chunk): two
// 128-row query tiles; TMEM S0 | S1 | O0 | O1.  Sliding-window calls run a
// persistent grid, one CTA per SM walking the items; full-attention calls run
// one item per CTA (see the kernel and its launcher).  A 128-token cache block is
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
    G_QEMPTY = 16,  // the item's last QK^T has read the query tiles
    G_COUNT = 17
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

// One work item = (sequence, query head, 256-row query block): its geometry,
// computed the same way by every role.  Items are numbered grouped by
// (sequence, kv head), so the items in flight at one time read the same cache
// blocks (they stay in L2); inside a group the later (longer) query blocks
// come first.
struct PagedItem {
    int s, kvh, qb, h, q_begin, n, L, base, ulo, uhi;
    int r0[2], lo[2], hi[2];
    bool ok[2];
    bool bad;   // a length outside what the arguments allow (BAD_LENGTH)
    bool live;  // false: nothing to compute (rows past the chunk, or a bad length)
};

INK_DEV void paged_item(const PagedArgs &g, int idx, PagedItem &it) {
    const PrefillArgs &a = g.pa;
    const int G = a.Hq / a.Hkv;
    const int per_group = g.nqb * G;
    const int grp = idx / per_group, rem = idx % per_group;
    it.s = grp / a.Hkv;
    it.kvh = grp % a.Hkv;
    it.qb = g.nqb - 1 - rem / G;
    it.h = it.kvh * G + rem % G;
    const bool dense = g.cu_q == nullptr;
    it.q_begin = dense ? it.s * g.dense_T : g.cu_q[it.s];
    it.n = dense ? g.dense_T : g.cu_q[it.s + 1] - it.q_begin;  // query rows of this sequence
    it.L = g.seq_lens ? g.seq_lens[it.s] : g.dense_T;
    it.base = it.L - it.n;  // position of the first new token
    it.bad = it.n < 0 || it.base < 0 || it.L > g.max_blocks * 128;
    it.live = !it.bad && it.qb * kQRows < it.n;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        it.r0[t] = it.qb * kQRows + t * 128;  // chunk row of tile row 0
        it.ok[t] = it.r0[t] < it.n;
        const int last = it.base + min(it.r0[t] + 127, it.n - 1);
        it.hi[t] = last >> 7;
        it.lo[t] = (a.window > 0) ? (max(0, it.base + it.r0[t] - a.window + 1) >> 7) : 0;
    }
    it.ulo = it.lo[0];
    it.uhi = it.ok[1] ? it.hi[1] : it.hi[0];
}

// Persistent grid (sliding-window calls): one CTA per SM walks the items in a
// snake order (below); full-attention calls run one item per CTA.
// Barrier phases run on across items (counters of items, key/value tiles and
// P tiles), so the producer loads the next item's queries and first key tile,
// and the MMA issuer its first QK^T, while the softmax groups still write the
// previous item's rows.  The next item's first P.V overwrites O only after
// its first P signal, which the softmax group gives after the previous
// epilogue has read O from TMEM; the queries are reloaded only after the
// previous item's last QK^T has completed (Q_EMPTY).
template <bool kPersist>
__global__ void __launch_bounds__(512, 1)
attn_prefill_paged_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const PagedArgs g) {
    const PrefillArgs &a = g.pa;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long total = (long)g.S * a.Hq * g.nqb;
    // Persistent (kPersist): round r of the walk takes item r*P + c, or
    // r*P + P-1-c on odd rounds (a snake): the items of a group come heaviest
    // first, so a plain stride would give the low CTAs the heavy end of every
    // group.  Otherwise one item per CTA (rounds = 1, item = blockIdx.x).
    const int rounds = kPersist ? (int)((total + gridDim.x - 1) / gridDim.x) : 1;
    auto snake_item = [&](int r) {
        return kPersist ? (int)(r * gridDim.x + ((r & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x))
                        : (int)blockIdx.x;
    };

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bar = (uint64_t *)(smem + PG_BAR);
    uint32_t *tmem_slot = (uint32_t *)(bar + G_COUNT);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    // ---- setup (once per CTA)
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
        if constexpr (kPersist)
            setmaxnreg_inc192();
        else
            setmaxnreg_inc200();
        const int t = warp >> 2;
        int k_base = 0;        // key tiles this group has processed (S_FULL, bias parities)
        uint32_t items = 0;    // items this group has finished (O_DONE parity)
        for (int r = 0; r < rounds; ++r) {
            const int idx = snake_item(r);
            if (idx >= total) continue;
            PagedItem it;
            paged_item(g, idx, it);
            if (threadIdx.x == 0 && it.h == 0) {
                if (it.bad && it.qb == 0) report_status(a.status, INKLING_STATUS_BAD_LENGTH);
                if (!it.bad && it.qb == g.nqb - 1 && it.n > g.nqb * kQRows)
                    report_status(a.status, INKLING_STATUS_BAD_LENGTH);  // rows past max_q are not computed
            }
            // this group's query tile, with constant indices (no local memory)
            const bool okt = t ? it.ok[1] : it.ok[0];
            if (!it.live || !okt) continue;
            const int r0 = t ? it.r0[1] : it.r0[0];
            const int lo = t ? it.lo[1] : it.lo[0], hi = t ? it.hi[1] : it.hi[0];
            softmax_role(a, (float *)(smem + PG_BIAS) + t * 2 * kBiasBuf, &bar[G_SFULL],
                         &bar[G_ODONE], abort_flag, tbase, t, it.h, it.base + r0, it.L, lo, hi,
                         3 + t, k_base, items & 1u,
                         [&](int tt) { mbar_arrive(&bar[G_PFULL + tt]); },
                         RowStoreEpilogue{g.out, g.lse, (long)it.q_begin + r0, it.n - r0,
                                          a.Hq, it.h, g.cu_q == nullptr ? g.dense_T : 0});
            k_base += hi - lo + 1;
            ++items;
        }
    } else if (warp < 12) {
        setmaxnreg_dec24();
    } else {
        if constexpr (kPersist)
            setmaxnreg_dec104();
        else
            setmaxnreg_dec88();
        if (warp == 12 && lane == 0) {
            // ============================================== TMA producer ==
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            long kv = 0;             // key/value tiles started (stage = kv & 1)
            long kis = 0, vis = 0;   // key / value tile loads issued
            int items = 0;           // items whose queries were loaded
            bool alive = true;
            for (int r = 0; r < rounds && alive; ++r) {
                const int idx = snake_item(r);
                if (idx >= total) continue;
                PagedItem it;
                paged_item(g, idx, it);
                if (!it.live) continue;
                // the previous item's QK^T have read their queries
                if (items > 0 && !mbar_wait(&bar[G_QEMPTY], (items - 1) & 1, abort_flag, a.status))
                    break;
                mbar_arrive_expect_tx(&bar[G_QFULL], 65536);
                for (int t = 0; t < 2; ++t)
                    for (int hf = 0; hf < 2; ++hf)
                        tma_load_3d(smem + PG_Q + t * 32768 + hf * 16384, &tm_q, &bar[G_QFULL],
                                    hf * 64, it.h, it.q_begin + it.r0[t]);
                ++items;
                for (int nt = it.ulo; nt <= it.uhi; ++nt, ++kv) {
                    const int st = (int)(kv & 1);
                    const uint32_t ph = (uint32_t)(((kv >> 1) & 1) ^ 1);
                    int blk = g.block_table ? g.block_table[(long)it.s * g.max_blocks + nt]
                                            : it.s * g.max_blocks + nt;
                    if (blk < 0 || blk >= g.num_blocks) {
                        report_status(a.status, INKLING_STATUS_BAD_BLOCK);
                        blk = 0;  // keep the pipeline running on a valid block
                    }
                    const int row = (blk * a.Hkv + it.kvh) * 128;
                    if (!mbar_wait(&bar[G_KEMPTY + st], ph, abort_flag, a.status)) {
                        alive = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar[G_KFULL + st], 32768);
                    tma_load_2d(smem + PG_K + st * 32768, &tm_k, &bar[G_KFULL + st], 0, row);
                    tma_load_2d(smem + PG_K + st * 32768 + 16384, &tm_k, &bar[G_KFULL + st], 64, row);
                    ++kis;
                    if (!mbar_wait(&bar[G_VEMPTY + st], ph, abort_flag, a.status)) {
                        alive = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar[G_VFULL + st], 32768);
                    tma_load_2d(smem + PG_V + st * 32768, &tm_v, &bar[G_VFULL + st], 0, row);
                    tma_load_2d(smem + PG_V + st * 32768 + 16384, &tm_v, &bar[G_VFULL + st], 64, row);
                    ++vis;
                }
            }
            // drain: every load issued has landed before the block may exit (the
            // earlier ones were consumed before their buffers were reused)
            if (items > 0) mbar_wait(&bar[G_QFULL], (items - 1) & 1, nullptr, a.status);
            for (long k = max(0L, kis - 2); k < kis; ++k)
                mbar_wait(&bar[G_KFULL + (k & 1)], (uint32_t)((k >> 1) & 1), nullptr, a.status);
            for (long k = max(0L, vis - 2); k < vis; ++k)
                mbar_wait(&bar[G_VFULL + (k & 1)], (uint32_t)((k >> 1) & 1), nullptr, a.status);
        } else if (warp == 13 && lane == 0) {
            // ================================================ MMA issuer ==
            const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_pv = idesc_bf16(128, 128, 0, 1);
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
            long kv = 0;                 // key/value tiles consumed
            uint32_t ptile[2] = {0, 0};  // P tiles consumed per query tile (P_FULL parity)
            int items = 0;
            bool alive = true;
            for (int r = 0; r < rounds && alive; ++r) {
                const int idx = snake_item(r);
                if (idx >= total) continue;
                PagedItem it;
                paged_item(g, idx, it);
                if (!it.live) continue;
                auto in_range = [&](int t, int nt) {
                    return it.ok[t] && nt >= it.lo[t] && nt <= it.hi[t];
                };
                if (!mbar_wait(&bar[G_QFULL], items & 1, abort_flag, a.status) ||
                    !mbar_wait(&bar[G_KFULL + (kv & 1)], (uint32_t)((kv >> 1) & 1), abort_flag,
                               a.status)) {
                    alive = false;
                    break;
                }
                ++items;
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (in_range(t, it.ulo)) {
                        issue_qk(t, (int)(kv & 1));
                        tc_commit(&bar[G_SFULL + t]);
                    }
                if (it.ulo == it.uhi) tc_commit(&bar[G_QEMPTY]);
                tc_commit(&bar[G_KEMPTY + (kv & 1)]);
                for (int nt = it.ulo; nt <= it.uhi; ++nt, ++kv) {
                    const int st = (int)(kv & 1), st1 = (int)((kv + 1) & 1);
                    const uint32_t ph1 = (uint32_t)(((kv + 1) >> 1) & 1);
                    if (!mbar_wait(&bar[G_VFULL + st], (uint32_t)((kv >> 1) & 1), abort_flag,
                                   a.status)) {
                        alive = false;
                        break;
                    }
                    const bool has_next = nt < it.uhi;
                    // the next key tile, checked before waiting for P (it was
                    // requested two tiles ago): the wait then stays off the
                    // P -> P.V -> QK^T -> S chain
                    bool got_next = has_next && mbar_wait(&bar[G_KFULL + st1], ph1, abort_flag,
                                                          a.status);
                    if (has_next && !got_next) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    for (int t = 0; t < 2 && alive; ++t) {
                        if (in_range(t, nt)) {
                            if (!mbar_wait(&bar[G_PFULL + t], ptile[t] & 1u, abort_flag,
                                           a.status)) {
                                alive = false;
                                break;
                            }
                            ++ptile[t];
                            tc_fence_after();
                            issue_pv(t, st, nt > it.lo[t]);
                        }
                        if (has_next && in_range(t, nt + 1)) {
                            issue_qk(t, st1);
                            tc_commit(&bar[G_SFULL + t]);
                        }
                    }
                    if (!alive) break;
                    if (has_next) {
                        if (nt + 1 == it.uhi) tc_commit(&bar[G_QEMPTY]);
                        tc_commit(&bar[G_KEMPTY + st1]);
                    }
                    tc_commit(&bar[G_VEMPTY + st]);
                    for (int t = 0; t < 2; ++t)
                        if (it.ok[t] && nt == it.hi[t]) tc_commit(&bar[G_ODONE + t]);
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
                                      cudaStream_t stream, int dense_T, int sms) {
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
    const long items = (long)g.S * p.num_q_heads * g.nqb;
    if (items == 0) return cudaSuccess;
    // Sliding-window calls walk the items on a persistent grid: the window
    // bounds every item's key range, so the items cost about the same and a
    // static walk stays balanced while it hides each item's start under the
    // previous item's end.  Full-attention items grow with the query position;
    // there one item per CTA lets the hardware scheduler balance them.
    const bool persist = p.window > 0;
    const long grid = persist ? (items < sms ? items : sms) : items;
    auto kernel = persist ? attn_prefill_paged_kernel<true> : attn_prefill_paged_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kPagedSmem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)grid, 512, kPagedSmem, stream>>>(tm_q, tm_k, tm_v, g);
    return cudaGetLastError();
}

}  // namespace inkling
