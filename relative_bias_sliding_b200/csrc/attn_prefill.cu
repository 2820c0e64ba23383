// attn_prefill.cu — prefill attention of the Inkling decoder layer on tcgen05
// tensor cores, with the key/value short convolution fused into the tile load
// (vLLM Recipes "thinkingmachines/Inkling", Overview: "Attention" — GQA at head
// size 128, learned relative-position term added to the pre-softmax logits,
// sliding-window or full layers; "Short convolution" — window-4 sconv on keys
// and values; Performance names an FA4 "sheared-bias" kernel as prior art).
//
// One thread block = one (batch, query head, 256-row query block), i.e. two
// 128-row query tiles that share every key/value tile.  Tensor memory (512
// columns) holds S0 | S1 | O0 | O1, 128 fp32 columns each; P (bf16) is written
// over the first 64 columns of its S and fed to the P.V MMA from TMEM.
//
// Warp roles (16 warps):
//   0-3   softmax of query tile 0 (thread = one query row = one TMEM lane)
//   4-7   softmax of query tile 1
//   8-9   sconv of the key tile, 10-11 sconv of the value tile (in place)
//   12    TMA producer (Q once; raw K, raw V and their 3-row history per tile)
//   13    TMEM allocator and single-thread tcgen05.mma issuer
//   14-15 idle
// Pipelines: 2 stages of raw->converted K and V tiles; S/P/O handshakes per
// query tile.  The MMA issue order QK(t0) QK(t1) | PV(t0) QK'(t0) PV(t1)
// QK'(t1) | ... lets the tensor core work on one tile while the other tile's
// softmax runs.  Key tiles wholly outside the causal band or the window are
// never loaded; masking is applied only where a tile straddles an edge.
// The online softmax keeps a reference maximum per row and rescales O only
// when a row maximum grows by more than 8 (log2 units), which is exact up to
// rounding because numerator and denominator share the same reference.
#include "prefill_common.cuh"

namespace inkling {

constexpr uint32_t SM_Q = 0;            // 2 tiles x 32 KB
constexpr uint32_t SM_K = 65536;        // 2 stages x 32 KB
constexpr uint32_t SM_V = 131072;       // 2 stages x 32 KB
constexpr uint32_t SM_KH = 196608;      // 2 stages x 2 KB (8 history rows x 2 halves)
constexpr uint32_t SM_VH = 200704;      // 2 stages x 2 KB
constexpr uint32_t SM_BIAS = 204800;    // 2 softmax groups x 2 buffers x 4 copies x 264 fp32
constexpr uint32_t SM_BAR = SM_BIAS + kBiasBytes;  // mbarriers, tmem base, flags
constexpr int kPrefillSmem = SM_BAR + 512 + 1024;

enum {
    B_QFULL = 0,
    B_KRAW = 1,    // +stage
    B_VRAW = 3,
    B_KREADY = 5,
    B_VREADY = 7,
    B_KEMPTY = 9,
    B_VEMPTY = 11,
    B_SFULL = 13,  // +tile
    B_PFULL = 15,
    B_ODONE = 17,
    B_DRAIN = 19,
    B_COUNT = 20
};

// kFill: also write the post-sconv keys/values to the paged cache and the new
// sconv state (a separate instantiation, so the plain prefill keeps its
// registers).
template <bool kFill>
__global__ void __launch_bounds__(512, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_kh,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_vh,
                    const __grid_constant__ CUtensorMap tm_out, const PrefillArgs a,
                    const FillArgs f) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bar = (uint64_t *)(smem + SM_BAR);
    uint32_t *tmem_slot = (uint32_t *)(bar + B_COUNT);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- work item: CTAs run grouped by (sequence, kv head), so the CTAs
    // resident at one time read the same keys/values (they stay in L2); inside
    // a group the heaviest query blocks come first.
    const int G = a.Hq / a.Hkv;
    const int per_group = a.nqb * G;
    const int grp = (int)(blockIdx.x / per_group), rem = (int)(blockIdx.x % per_group);
    const int b = grp / a.Hkv;
    const int kvh = grp % a.Hkv;
    const int qb = a.nqb - 1 - rem / G;
    const int h = kvh * G + rem % G;
    int r0[2], lo[2], hi[2];
    bool ok[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        r0[t] = qb * kQRows + t * 128;
        ok[t] = r0[t] < a.T;
        const int rmax = min(r0[t] + 127, a.T - 1);
        hi[t] = rmax >> 7;
        lo[t] = (a.window > 0) ? (max(0, r0[t] - a.window + 1) >> 7) : 0;
    }
    const int ulo = lo[0];
    const int uhi = ok[1] ? hi[1] : hi[0];

    // ---- setup
    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t cnt = 1;
            if (i == B_PFULL || i == B_PFULL + 1) cnt = 128;
            if (i == B_KREADY || i == B_KREADY + 1 || i == B_VREADY || i == B_VREADY + 1) cnt = 64;
            mbar_init(&bar[i], cnt);
        }
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
            softmax_role(a, (float *)(smem + SM_BIAS) + t * 2 * kBiasBuf, &bar[B_SFULL],
                         &bar[B_ODONE], abort_flag, tbase, t, h, r0[t], a.T, lo[t], hi[t], 3 + t,
                         0, 0u, [&](int tt) { mbar_arrive(&bar[B_PFULL + tt]); },
                         TmaStoreEpilogue{a, smem + SM_Q + t * 32768, &tm_out, b, h, r0[t], 3 + t});
    } else if (warp < 12) {
        // ========================== sconv transform: warps 8-9 keys, 10-11 values ==
        setmaxnreg_dec80();
        const bool is_v = warp >= 10;
        const int v = threadIdx.x - (is_v ? 320 : 256);
        const int bar_id = is_v ? 2 : 1;
        // taps of this thread's 8 channels, held for the whole block
        f32x2 w[4][4];
        load_taps(w, (is_v ? a.w_v : a.w_k) + ((long)kvh * 128 + 8 * (v & 15)) * 4);
        uint64_t *raw_full = &bar[is_v ? B_VRAW : B_KRAW];
        uint64_t *ready = &bar[is_v ? B_VREADY : B_KREADY];
        const uint32_t tiles = sb + (is_v ? SM_V : SM_K);
        const uint32_t hists = sb + (is_v ? SM_VH : SM_KH);
        // with a cache to fill, the block of the kv group's first head writes
        // the key tiles this query block owns (2qb up to its last tile)
        const bool writer = kFill && h == kvh * G && f.k_cache != nullptr;
        bool dead = false;
        int it = 0;
        for (int n = ulo; n <= uhi; ++n, ++it) {
            const int st = it & 1;
            if (!dead) dead = !mbar_wait(&raw_full[st], (it >> 1) & 1, abort_flag, a.status);
            if (dead) {
                named_bar_sync(bar_id, 64);  // keep the group's barrier count matched
                continue;
            }
            // thread v: column v % 16, rows 32 (v / 16) .. +32 of the 128-row tile
            sconv_rows(tiles + st * 32768, hists + st * 2048, 16384, w, v & 15, 32 * (v >> 4), 32,
                       bar_id, 64);
            if (kFill && writer && n >= 2 * qb) {
                uint16_t *gdst = cache_rows(f, a, is_v ? f.v_cache : f.k_cache, b, kvh, n, 0, 8 * (v & 15));
                if (gdst) store_rows(tiles + st * 32768, 16384, v & 15, 32 * (v >> 4), 32, gdst, a.T - n * 128);
            }
            fence_proxy_async_smem();
            mbar_arrive(&ready[st]);
        }
    } else {
        setmaxnreg_dec64();
        if (kFill && warp == 14 && h == kvh * G && f.k_state && uhi == (a.T - 1) >> 7) {
            // the new sconv state, by the block that owns the last key tile
            write_sconv_state(f, a, b, kvh, lane);
        } else if (warp == 12 && lane == 0) {
            // ============================================== TMA producer ==
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_kh);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_vh);
            mbar_arrive_expect_tx(&bar[B_QFULL], 65536);
            for (int t = 0; t < 2; ++t)
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_4d(smem + SM_Q + t * 32768 + hf * 16384, &tm_q, &bar[B_QFULL],
                                hf * 64, r0[t], h, b);
            int kis = 0, vis = 0;  // key / value tile loads issued
            for (int n = ulo; n <= uhi; ++n) {
                const int it = n - ulo, st = it & 1;
                const uint32_t ph = ((it >> 1) & 1) ^ 1;
                if (!mbar_wait(&bar[B_KEMPTY + st], ph, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&bar[B_KRAW + st], 32768 + 2048);
                for (int hf = 0; hf < 2; ++hf) {
                    tma_load_4d(smem + SM_K + st * 32768 + hf * 16384, &tm_k, &bar[B_KRAW + st],
                                hf * 64, n * 128, kvh, b);
                    tma_load_4d(smem + SM_KH + st * 2048 + hf * 1024, &tm_kh, &bar[B_KRAW + st],
                                hf * 64, n * 128 - 8, kvh, b);
                }
                ++kis;
                if (!mbar_wait(&bar[B_VEMPTY + st], ph, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&bar[B_VRAW + st], 32768 + 2048);
                for (int hf = 0; hf < 2; ++hf) {
                    tma_load_4d(smem + SM_V + st * 32768 + hf * 16384, &tm_v, &bar[B_VRAW + st],
                                hf * 64, n * 128, kvh, b);
                    tma_load_4d(smem + SM_VH + st * 2048 + hf * 1024, &tm_vh, &bar[B_VRAW + st],
                                hf * 64, n * 128 - 8, kvh, b);
                }
                ++vis;
            }
            // drain: every load issued has landed before the block may exit
            mbar_wait(&bar[B_QFULL], 0, nullptr, a.status);
            for (int k = max(0, kis - 2); k < kis; ++k)
                mbar_wait(&bar[B_KRAW + (k & 1)], (k >> 1) & 1, nullptr, a.status);
            for (int k = max(0, vis - 2); k < vis; ++k)
                mbar_wait(&bar[B_VRAW + (k & 1)], (k >> 1) & 1, nullptr, a.status);
        } else if (warp == 13 && lane == 0) {
            // ================================================ MMA issuer ==
            const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_pv = idesc_bf16(128, 128, 0, 1);
            auto in_range = [&](int t, int n) { return ok[t] && n >= lo[t] && n <= hi[t]; };
            auto issue_qk = [&](int t, int st) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint64_t ad = sw128_desc(sb + SM_Q + t * 32768 + koff, 16, 1024);
                    const uint64_t bd = sw128_desc(sb + SM_K + st * 32768 + koff, 16, 1024);
                    umma_ss(tbase + t * 128, ad, bd, id_qk, ks > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](int t, int st, bool acc) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t bd = sw128_desc(sb + SM_V + st * 32768 + ks * 2048, 16384, 1024);
                    umma_ts(tbase + 256 + t * 128, tbase + t * 128 + ks * 8, bd, id_pv,
                            (acc || ks > 0) ? 1u : 0u);
                }
            };
            bool alive = mbar_wait(&bar[B_QFULL], 0, abort_flag, a.status);
            if (alive) alive = mbar_wait(&bar[B_KREADY], 0, abort_flag, a.status);
            if (alive) {
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (in_range(t, ulo)) {
                        issue_qk(t, 0);
                        tc_commit(&bar[B_SFULL + t]);
                    }
                tc_commit(&bar[B_KEMPTY]);
                int it = 0;
                for (int n = ulo; n <= uhi && alive; ++n, ++it) {
                    const int st = it & 1, st1 = (it + 1) & 1;
                    const uint32_t ph1 = ((it + 1) >> 1) & 1;
                    if (!mbar_wait(&bar[B_VREADY + st], (it >> 1) & 1, abort_flag, a.status)) break;
                    tc_fence_after();
                    const bool has_next = n < uhi;
                    bool got_next = false;
                    for (int t = 0; t < 2 && alive; ++t) {
                        if (in_range(t, n)) {
                            if (!mbar_wait(&bar[B_PFULL + t], (n - lo[t]) & 1, abort_flag, a.status)) {
                                alive = false;
                                break;
                            }
                            tc_fence_after();
                            issue_pv(t, st, n > lo[t]);
                        }
                        if (has_next && in_range(t, n + 1)) {
                            if (!got_next) {
                                if (!mbar_wait(&bar[B_KREADY + st1], ph1, abort_flag, a.status)) {
                                    alive = false;
                                    break;
                                }
                                tc_fence_after();
                                got_next = true;
                            }
                            issue_qk(t, st1);
                            tc_commit(&bar[B_SFULL + t]);
                        }
                    }
                    if (!alive) break;
                    if (has_next) {
                        if (!got_next && !mbar_wait(&bar[B_KREADY + st1], ph1, abort_flag, a.status))
                            break;
                        tc_commit(&bar[B_KEMPTY + st1]);
                    }
                    tc_commit(&bar[B_VEMPTY + st]);
                    for (int t = 0; t < 2; ++t)
                        if (ok[t] && n == hi[t]) tc_commit(&bar[B_ODONE + t]);
                }
            }
            // every MMA issued has completed before TMEM is released
            tc_commit(&bar[B_DRAIN]);
            mbar_wait(&bar[B_DRAIN], 0, nullptr, a.status);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

cudaError_t launch_attn_prefill(const inkling_prefill_params &p, const CUtensorMap *maps,
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
    a.nqb = (p.seq_len + kQRows - 1) / kQRows;
    const long grid = (long)a.B * a.Hq * a.nqb;
    if (grid == 0) return cudaSuccess;
    const bool fill = f.k_cache != nullptr || f.k_state != nullptr;
    auto kernel = fill ? attn_prefill_kernel<true> : attn_prefill_kernel<false>;
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPrefillSmem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)grid, 512, kPrefillSmem, stream>>>(maps[0], maps[1], maps[2], maps[3],
                                                         maps[4], maps[5], a, f);
    return cudaGetLastError();
}

}  // namespace inkling
