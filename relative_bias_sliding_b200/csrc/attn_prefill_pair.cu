// attn_prefill_pair.cu — the prefill of attn_prefill.cu run on CTA pairs with
// 2-SM tensor-core MMAs (tcgen05 cta_group::2), for GQA groups of even size.
//
// Same layer and numerics (vLLM Recipes "thinkingmachines/Inkling", Overview:
// "Attention" and "Short convolution").  A 2-CTA cluster takes query heads of
// one kv group over the same query rows (4 heads x 128 rows when the group
// size is a multiple of 4, else 2 heads x 256 rows), so both CTAs walk the
// same key/value tiles.  Each MMA is M = 256 (128 query rows from each CTA's shared
// memory, accumulators in each CTA's own tensor memory) and reads the B
// operand half from each CTA:
//   QK^T: N = 128 keys; CTA r holds keys 64r..64r+63 of the tile (all of d);
//   P.V:  N = 128 head dims; CTA r holds d columns 64r..64r+63 (all keys).
// So each SM loads and convolves only half of every key tile and half of every
// value tile (the sconv is depthwise, so splitting values by channel needs no
// exchange; a key half takes its 3 history rows straight from global memory),
// and the tensor core's shared-memory reads of K and V are halved too.
//
// Roles per CTA are those of attn_prefill.cu.  The even CTA's warp 13 issues
// all MMAs.  The odd CTA's threads report to the even CTA's mbarriers:
// converted halves (K/V ready), their P tiles (per warp) and their Q load.
// Commits are multicast to the same barrier offset in both CTAs, so each CTA's
// softmax and producer wait on local barriers.  Key/value stages: 4.  No TMA
// load uses multicast.
#include "prefill_common.cuh"

namespace inkling {

constexpr int kPS = 4;                          // key/value pipeline stages
constexpr uint32_t PQ = 0;                      // 2 query tiles x 32 KB
constexpr uint32_t PK = 65536;                  // kPS x 16 KB: this CTA's 64 keys x 128 d
constexpr uint32_t PV = PK + kPS * 16384;       // kPS x 16 KB: 128 keys x this CTA's 64 d
constexpr uint32_t PKH = PV + kPS * 16384;      // kPS x 2 KB: 8 history rows x 2 halves
constexpr uint32_t PVH = PKH + kPS * 2048;      // kPS x 1 KB: 8 history rows x this CTA's half
constexpr uint32_t PBIAS = PVH + kPS * 1024;    // bias diagonals of the 2 query tiles
constexpr uint32_t PBAR = PBIAS + kBiasBytes;   // mbarriers, tmem base, flags
constexpr int kPairSmem = PBAR + 512 + 1024;

enum {
    Q_FULL = 0,
    Q_PEER = 1,   // even CTA: the odd CTA's query tiles have landed
    K_RAW = 2,    // +stage
    V_RAW = K_RAW + kPS,
    K_READY = V_RAW + kPS,  // even CTA: both halves converted (64 + 64 arrivals)
    V_READY = K_READY + kPS,
    K_EMPTY = V_READY + kPS,
    V_EMPTY = K_EMPTY + kPS,
    S_FULL = V_EMPTY + kPS,  // +query tile
    P_FULL = S_FULL + 2,  // even CTA: 4 warps of each CTA
    O_DONE = P_FULL + 2,
    DRAIN = O_DONE + 2,
    NBAR = DRAIN + 1
};
static_assert(kPairSmem <= 232448, "shared memory per block");

// kFill: also write the post-sconv keys/values to the paged cache and the new
// sconv state (a separate instantiation, so the plain prefill keeps its
// registers).
template <bool kFill>
__global__ void __launch_bounds__(512, 1)
attn_prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k64,
                         const __grid_constant__ CUtensorMap tm_kh,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_vh,
                    const __grid_constant__ CUtensorMap tm_out, const PrefillArgs a,
                    const FillArgs f) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bar = (uint64_t *)(smem + PBAR);
    uint32_t *tmem_slot = (uint32_t *)(bar + NBAR);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 issues the MMAs

    // ---- work item.  When the GQA group size is a multiple of 4, a cluster
    // takes 4 heads of one kv group over the same 128 query rows: CTA r holds
    // heads 4q+2r and 4q+2r+1 as its two query tiles, so both tiles walk the
    // same key range.  Otherwise it takes 2 heads (one per CTA) over 256 rows,
    // two 128-row tiles per CTA whose key ranges differ by one tile at each end.
    // Clusters run grouped by (sequence, kv head), so the clusters resident at
    // one time read the same keys/values (they stay in L2); inside a group the
    // heaviest query blocks come first.
    const int G = a.Hq / a.Hkv;
    const bool quad = (G & 3) == 0;
    const int per_qb = quad ? G / 4 : G / 2;  // clusters per (kv head, query block)
    const int per_group = a.nqb * per_qb;
    const int cid = (int)(blockIdx.x >> 1);
    const int grp = cid / per_group, rem = cid % per_group;
    const int b = grp / a.Hkv;
    const int kvh = grp % a.Hkv;
    const int qb = a.nqb - 1 - rem / per_qb;
    const int hsel = rem % per_qb;
    int hd[2], r0[2], lo[2], hi[2];
    bool ok[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        hd[t] = quad ? kvh * G + 4 * hsel + 2 * (int)rank + t : kvh * G + 2 * hsel + (int)rank;
        r0[t] = quad ? qb * 128 : qb * 256 + t * 128;
        ok[t] = r0[t] < a.T;
        const int rmax = min(r0[t] + 127, a.T - 1);
        hi[t] = rmax >> 7;
        lo[t] = (a.window > 0) ? (max(0, r0[t] - a.window + 1) >> 7) : 0;
    }
    const int ulo = lo[0];
    const int uhi = ok[1] ? hi[1] : hi[0];

    // tile loads into this CTA's shared memory, completing on its own barriers
    const int krow = 64 * (int)rank;
    auto load_k = [&](int n, int st) {
        mbar_arrive_expect_tx(&bar[K_RAW + st], 16384 + 2048);
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(smem + PK + st * 16384 + hf * 8192, &tm_k64, &bar[K_RAW + st], hf * 64,
                        n * 128 + krow, kvh, b);
            tma_load_4d(smem + PKH + st * 2048 + hf * 1024, &tm_kh, &bar[K_RAW + st], hf * 64,
                        n * 128 + krow - 8, kvh, b);
        }
    };
    auto load_v = [&](int n, int st) {
        mbar_arrive_expect_tx(&bar[V_RAW + st], 16384 + 1024);
        tma_load_4d(smem + PV + st * 16384, &tm_v, &bar[V_RAW + st], 64 * (int)rank, n * 128, kvh,
                    b);
        tma_load_4d(smem + PVH + st * 1024, &tm_vh, &bar[V_RAW + st], 64 * (int)rank,
                    n * 128 - 8, kvh, b);
    };
    const int preload = min(kPS, uhi - ulo + 1);  // key/value tiles loaded during setup

    // ---- setup: barriers and the paired tensor-memory allocation must exist in
    // both CTAs before either CTA signals the other.  The query tiles and the
    // first kPS key/value tiles only involve this CTA's barriers, so the thread
    // that initialises them starts those loads at once, under the allocation
    // and the cluster barrier.
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) {
            uint32_t cnt = 1;
            if (i >= K_READY && i < K_EMPTY) cnt = 128;
            if (i == P_FULL || i == P_FULL + 1) cnt = 8;
            mbar_init(&bar[i], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bar[Q_FULL], 65536);
        for (int t = 0; t < 2; ++t)
            for (int hf = 0; hf < 2; ++hf)
                tma_load_4d(smem + PQ + t * 32768 + hf * 16384, &tm_q, &bar[Q_FULL], hf * 64,
                            r0[t], hd[t], b);
        for (int i = 0; i < preload; ++i) {
            load_k(ulo + i, i);
            load_v(ulo + i, i);
        }
    }
    if (warp == 13) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp < 8) {
        // ================================================== softmax (2 WGs) ==
        if (kFill)
            setmaxnreg_inc168();
        else
            setmaxnreg_inc184();
        const int t = warp >> 2;
        if (ok[t])
            softmax_role(a, (float *)(smem + PBIAS) + t * 2 * kBiasBuf, &bar[S_FULL], &bar[O_DONE],
                         abort_flag, tbase, t, hd[t], r0[t], a.T, lo[t], hi[t], 3 + t, 0, 0u,
                         [&](int tt) {
                             __syncwarp();
                             if (lane == 0) mbar_arrive_cta_relaxed(&bar[P_FULL + tt], 0);
                         },
                         TmaStoreEpilogue{a, smem + PQ + t * 32768, &tm_out, b, hd[t], r0[t], 3 + t});
    } else if (warp < 12) {
        // ==================== sconv of this CTA's halves: warps 8-9 keys, 10-11 values ==
        if (kFill)
            setmaxnreg_dec96();
        else
            setmaxnreg_dec80();
        const bool is_v = warp >= 10;
        const int v = threadIdx.x - (is_v ? 320 : 256);
        const int bar_id = is_v ? 2 : 1;
        // keys: 64 rows x 16 columns, thread = column v%16, rows 16(v/16)..+16;
        // values: 128 rows x 8 columns (this CTA's 64 channels), column v%8, rows 16(v/8)..+16
        const int col = is_v ? (v & 7) : (v & 15);
        const int row0 = is_v ? 16 * (v >> 3) : 16 * (v >> 4);
        const int ch0 = is_v ? (64 * (int)rank + 8 * col) : 8 * col;
        f32x2 w[4][4];
        load_taps(w, (is_v ? a.w_v : a.w_k) + ((long)kvh * 128 + ch0) * 4);
        uint64_t *raw_full = &bar[is_v ? V_RAW : K_RAW];
        uint64_t *ready = &bar[is_v ? V_READY : K_READY];
        const uint32_t tiles = sb + (is_v ? PV : PK);
        const uint32_t hists = sb + (is_v ? PVH : PKH);
        const uint32_t hist_stage = is_v ? 1024 : 2048;
        // with a cache to fill, the first cluster of the (sequence, kv head)
        // for this query block writes the key tiles it owns: quad ? qb : 2qb
        // up to its last tile (each CTA its converted half)
        const bool writer = kFill && hsel == 0 && f.k_cache != nullptr;
        bool dead = false;
        int it = 0;
        for (int n = ulo; n <= uhi; ++n, ++it) {
            const int st = it % kPS;
            if (!dead) dead = !mbar_wait(&raw_full[st], (it / kPS) & 1, abort_flag, a.status);
            if (dead) {
                named_bar_sync(bar_id, 64);  // keep the group's barrier count matched
                continue;
            }
            sconv_rows(tiles + st * 16384, hists + st * hist_stage, 8192, w, col, row0, 16, bar_id,
                       64);
            if (kFill && writer && n >= (quad ? qb : 2 * qb)) {
                const int krow = is_v ? 0 : 64 * (int)rank;  // token row of this CTA's tile row 0
                uint16_t *gdst = cache_rows(f, a, is_v ? f.v_cache : f.k_cache, b, kvh, n, krow, ch0);
                if (gdst) store_rows(tiles + st * 16384, 8192, col, row0, 16, gdst, a.T - n * 128 - krow);
            }
            fence_proxy_async_smem();
            mbar_arrive_cta(&ready[st], 0);
        }
    } else {
        if (kFill)
            setmaxnreg_dec80();
        else
            setmaxnreg_dec64();
        if (kFill && warp == 14 && rank == 0 && hsel == 0 && f.k_state &&
            uhi == (a.T - 1) >> 7) {
            // the new sconv state, by the block that owns the last key tile
            write_sconv_state(f, a, b, kvh, lane);
        } else if (warp == 12 && lane == 0) {
            // ============================================== TMA producer ==
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k64);
            tma_prefetch_desc(&tm_kh);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_vh);
            // the query tiles and the first kPS key/value tiles went out during setup
            if (rank == 1 && mbar_wait(&bar[Q_FULL], 0, abort_flag, a.status))
                mbar_arrive_cta(&bar[Q_PEER], 0);
            int kis = preload, vis = preload;  // key / value tile loads issued
            for (int n = ulo + preload; n <= uhi; ++n) {
                const int it = n - ulo, st = it % kPS;
                const uint32_t ph = ((it / kPS) & 1) ^ 1;
                if (!mbar_wait(&bar[K_EMPTY + st], ph, abort_flag, a.status)) break;
                load_k(n, st);
                ++kis;
                if (!mbar_wait(&bar[V_EMPTY + st], ph, abort_flag, a.status)) break;
                load_v(n, st);
                ++vis;
            }
            // drain: every load issued has landed before the block may exit
            mbar_wait(&bar[Q_FULL], 0, nullptr, a.status);
            for (int k = max(0, kis - kPS); k < kis; ++k)
                mbar_wait(&bar[K_RAW + k % kPS], (k / kPS) & 1, nullptr, a.status);
            for (int k = max(0, vis - kPS); k < vis; ++k)
                mbar_wait(&bar[V_RAW + k % kPS], (k / kPS) & 1, nullptr, a.status);
        } else if (warp == 13 && lane == 0 && rank == 0) {
            // ======================================= MMA issuer (even CTA) ==
            const uint32_t id_qk = idesc_bf16(256, 128, 0, 0);
            const uint32_t id_pv = idesc_bf16(256, 128, 0, 1);
            // descriptors at the same shared-memory offsets in both CTAs; a
            // k-step advances the start-address field (16-byte units)
            const uint64_t dq0 = sw128_desc(sb + PQ, 16, 1024);
            const uint64_t dk0 = sw128_desc(sb + PK, 16, 1024);
            const uint64_t dv0 = sw128_desc(sb + PV, 8192, 1024);
            auto in_range = [&](int t, int n) { return ok[t] && n >= lo[t] && n <= hi[t]; };
            auto issue_qk = [&](int t, int st) {
                const uint64_t ad = dq0 + (uint64_t)(t * 2048);
                const uint64_t bd = dk0 + (uint64_t)(st * 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ss_pair(tbase + t * 128, ad + (uint64_t)((ks >> 2) * 1024 + (ks & 3) * 2),
                                 bd + (uint64_t)((ks >> 2) * 512 + (ks & 3) * 2), id_qk,
                                 ks > 0 ? 1u : 0u);
            };
            auto issue_pv = [&](int t, int st, bool acc) {
                const uint64_t bd = dv0 + (uint64_t)(st * 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ts_pair(tbase + 256 + t * 128, tbase + t * 128 + ks * 8,
                                 bd + (uint64_t)(ks * 128), id_pv, (acc || ks > 0) ? 1u : 0u);
            };
            bool alive = mbar_wait(&bar[Q_FULL], 0, abort_flag, a.status) &&
                         mbar_wait_cluster(&bar[Q_PEER], 0, abort_flag, a.status) &&
                         mbar_wait_cluster(&bar[K_READY], 0, abort_flag, a.status);
            if (alive) {
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (in_range(t, ulo)) {
                        issue_qk(t, 0);
                        tc_commit_pair(&bar[S_FULL + t], 3);
                    }
                tc_commit_pair(&bar[K_EMPTY], 3);
                int it = 0;
                for (int n = ulo; n <= uhi && alive; ++n, ++it) {
                    const int st = it % kPS, st1 = (it + 1) % kPS;
                    const uint32_t ph1 = ((it + 1) / kPS) & 1;
                    if (!mbar_wait_cluster(&bar[V_READY + st], (it / kPS) & 1, abort_flag, a.status))
                        break;
                    const bool has_next = n < uhi;
                    // the next tile's converted keys, checked before waiting for
                    // P (they are normally ready long before): the wait then stays
                    // off the P -> P.V -> QK^T -> S chain
                    bool got_next = has_next && mbar_wait_cluster(&bar[K_READY + st1], ph1, abort_flag,
                                                                  a.status);
                    if (has_next && !got_next) break;
                    tc_fence_after();
                    for (int t = 0; t < 2 && alive; ++t) {
                        if (in_range(t, n)) {
                            if (!mbar_wait_cluster(&bar[P_FULL + t], (n - lo[t]) & 1, abort_flag,
                                                   a.status)) {
                                alive = false;
                                break;
                            }
                            tc_fence_after();
                            issue_pv(t, st, n > lo[t]);
                        }
                        if (has_next && in_range(t, n + 1)) {
                            if (!got_next) {
                                if (!mbar_wait_cluster(&bar[K_READY + st1], ph1, abort_flag,
                                                       a.status)) {
                                    alive = false;
                                    break;
                                }
                                tc_fence_after();
                                got_next = true;
                            }
                            issue_qk(t, st1);
                            tc_commit_pair(&bar[S_FULL + t], 3);
                        }
                    }
                    if (!alive) break;
                    if (has_next) {
                        if (!got_next &&
                            !mbar_wait_cluster(&bar[K_READY + st1], ph1, abort_flag, a.status))
                            break;
                        tc_commit_pair(&bar[K_EMPTY + st1], 3);
                    }
                    tc_commit_pair(&bar[V_EMPTY + st], 3);
                    for (int t = 0; t < 2; ++t)
                        if (ok[t] && n == hi[t]) tc_commit_pair(&bar[O_DONE + t], 3);
                }
            }
            // every MMA issued has completed before tensor memory is released
            tc_commit_pair(&bar[DRAIN], 1);
            mbar_wait(&bar[DRAIN], 0, nullptr, a.status);
        }
    }
    // both CTAs are done with each other's shared and tensor memory before
    // either frees its tensor memory or exits
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc_pair(tbase, 512);
    }
}

cudaError_t launch_attn_prefill_pair(const inkling_prefill_params &p, const CUtensorMap *maps,
                                     cudaStream_t stream) {
    PrefillArgs a = {};
    a.w_k = p.w_k;
    a.w_v = p.w_v;
    a.bias = p.bias;
    a.out = (uint16_t *)p.out;
    a.lse = p.lse;
    a.status = p.status;
    a.B = p.batch;
    a.T = p.seq_len;
    a.Hq = p.num_q_heads;
    a.Hkv = p.num_kv_heads;
    a.window = p.window;
    a.d_max = p.d_max;
    FillArgs f = {};
    f.k_cache = (uint16_t *)p.k_cache;
    f.v_cache = (uint16_t *)p.v_cache;
    f.block_table = p.block_table;
    f.max_blocks = p.max_blocks;
    f.num_blocks = p.num_blocks;
    f.k_state = (uint16_t *)p.k_state;
    f.v_state = (uint16_t *)p.v_state;
    f.k_raw = (const uint16_t *)p.k_raw;
    f.v_raw = (const uint16_t *)p.v_raw;
    const int G = a.Hq / a.Hkv;
    const bool quad = (G & 3) == 0;  // 4 heads x 128 rows per cluster, else 2 heads x 256 rows
    a.nqb = quad ? (p.seq_len + 127) / 128 : (p.seq_len + 255) / 256;
    const long clusters = (long)a.B * a.Hkv * (quad ? G / 4 : G / 2) * a.nqb;
    if (clusters == 0) return cudaSuccess;
    const bool fill = f.k_cache != nullptr || f.k_state != nullptr;
    auto kernel = fill ? attn_prefill_pair_kernel<true> : attn_prefill_pair_kernel<false>;
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    cfg.blockDim = dim3(512, 1, 1);
    cfg.dynamicSmemBytes = kPairSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5],
                           a, f);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace inkling
