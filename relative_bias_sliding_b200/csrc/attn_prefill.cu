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
//   8-11  sconv transform: converts the raw key / value tile in place
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
#include "common.cuh"

namespace inkling {

constexpr int kQRows = 256;
constexpr uint32_t SM_Q = 0;            // 2 tiles x 32 KB
constexpr uint32_t SM_K = 65536;        // 2 stages x 32 KB
constexpr uint32_t SM_V = 131072;       // 2 stages x 32 KB
constexpr uint32_t SM_KH = 196608;      // 2 stages x 2 KB (8 history rows x 2 halves)
constexpr uint32_t SM_VH = 200704;      // 2 stages x 2 KB
constexpr uint32_t SM_W = 204800;       // w_k (2 KB) + w_v (2 KB) of this kv head
constexpr uint32_t SM_BAR = 208896;     // mbarriers, tmem base, abort flag, verdict
constexpr int kPrefillSmem = 208896 + 512 + 1024;

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

struct PrefillArgs {
    const float *w_k, *w_v, *bias;
    uint16_t *out;
    float *lse;
    int32_t *status;
    int B, T, Hq, Hkv, window, d_max, nqb;
};

// Register split per warpgroup: 2 x 128 softmax threads at 184, 128 sconv
// threads at 96, 128 producer/MMA/idle threads at 48: 47104 + 12288 + 6144 =
// 65536 = 512 threads x the 128 registers the kernel launches with (ptxas
// reports 128), so the increase never waits on registers that do not exist.
INK_DEV void setmaxnreg_inc184() { asm volatile("setmaxnreg.inc.sync.aligned.u32 184;"); }
INK_DEV void setmaxnreg_dec96() { asm volatile("setmaxnreg.dec.sync.aligned.u32 96;"); }
INK_DEV void setmaxnreg_dec48() { asm volatile("setmaxnreg.dec.sync.aligned.u32 48;"); }

// Convert one raw 128-row key or value tile (TMA layout: two 64-column halves
// of 128 rows x 128 bytes, 128-byte swizzle) into its sconv output, in place.
// Thread u owns 16-byte column c = u % 16 (8 channels) and rows 16g..16g+15,
// g = u / 16; the 3 rows before its first row come from the tile itself, or
// for g = 0 from the 8-row history box loaded with the tile.
INK_DEV void sconv_tile_inplace(uint32_t tile, uint32_t hist, const float *wsm, int u) {
    const int c = u & 15, g = u >> 4;
    const int half = c >> 3, cc = c & 7;
    float w[8][4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 t4 = *(const float4 *)(wsm + (c * 8 + e) * 4);
        w[e][0] = t4.x; w[e][1] = t4.y; w[e][2] = t4.z; w[e][3] = t4.w;
    }
    float h3[8], h2[8], h1[8];
    if (g == 0) {
        const uint32_t hb = hist + half * 1024;
        unpack8(lds128(hb + 5 * 128 + ((cc ^ 5) << 4)), h3);
        unpack8(lds128(hb + 6 * 128 + ((cc ^ 6) << 4)), h2);
        unpack8(lds128(hb + 7 * 128 + ((cc ^ 7) << 4)), h1);
    } else {
        const uint32_t tb = tile + half * 16384;
        const int r = 16 * g;
        unpack8(lds128(tb + (r - 3) * 128 + ((cc ^ ((r - 3) & 7)) << 4)), h3);
        unpack8(lds128(tb + (r - 2) * 128 + ((cc ^ ((r - 2) & 7)) << 4)), h2);
        unpack8(lds128(tb + (r - 1) * 128 + ((cc ^ ((r - 1) & 7)) << 4)), h1);
    }
    named_bar_sync(1, 128);  // every history row read before any row is overwritten
    const uint32_t tb = tile + half * 16384;
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
        const int r = 16 * g + i;
        const uint32_t addr = tb + r * 128 + ((cc ^ (r & 7)) << 4);
        float x[8];
        unpack8(lds128(addr), x);
        sts128(addr, sconv8(w, h3, h2, h1, x));
#pragma unroll
        for (int e = 0; e < 8; ++e) { h3[e] = h2[e]; h2[e] = h1[e]; h1[e] = x[e]; }
    }
}

__global__ void __launch_bounds__(512, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_kh,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_vh, const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bar = (uint64_t *)(smem + SM_BAR);
    uint32_t *tmem_slot = (uint32_t *)(bar + B_COUNT);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float *w_sm = (float *)(smem + SM_W);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- work item: heaviest query blocks first, heads of one kv group adjacent
    const int bh = a.B * a.Hq;
    const int qb = a.nqb - 1 - (int)(blockIdx.x / bh);
    const int b = (int)(blockIdx.x % bh) / a.Hq;
    const int h = (int)(blockIdx.x % bh) % a.Hq;
    const int G = a.Hq / a.Hkv;
    const int kvh = h / G;
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
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bar[i], (i == B_PFULL || i == B_PFULL + 1) ? 128 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 13) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp >= 8 && warp < 12) {
        const int u = threadIdx.x - 256;
        const float4 *wk = (const float4 *)(a.w_k + (long)kvh * 512);
        const float4 *wv = (const float4 *)(a.w_v + (long)kvh * 512);
        ((float4 *)w_sm)[u] = wk[u];
        ((float4 *)(w_sm + 512))[u] = wv[u];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp < 8) {
        // ================================================== softmax (2 WGs) ==
        setmaxnreg_inc184();
        const int t = warp >> 2;
        const int u = threadIdx.x & 127;
        if (ok[t]) {
            const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
            const uint32_t s_col = tl + t * 128, o_col = tl + 256 + t * 128;
            const int i = r0[t] + u;
            const float scale = 0.08838834764831845f;  // 1/sqrt(128)
            const float kLog2e = 1.4426950408889634f;
            const float kTau = 5.545177444479562f;       // 8 ln 2
            const float *bias_h = a.bias + (long)h * (a.d_max + 1);
            const int W = a.window, Dm = a.d_max, T = a.T;
            float m_ref = -INFINITY, l = 0.f;
            int k = 0;
            bool aborted = false;
            for (int n = lo[t]; n <= hi[t]; ++n, ++k) {
                if (!mbar_wait_warp(&bar[B_SFULL + t], k & 1, abort_flag, a.status)) {
                    aborted = true;
                    break;
                }
                tc_fence_after();
                uint32_t sr[128];
                tmem_ld32(s_col + 0, sr + 0);
                tmem_ld32(s_col + 32, sr + 32);
                tmem_ld32(s_col + 64, sr + 64);
                tmem_ld32(s_col + 96, sr + 96);
                tmem_wait_ld();
                float x[128];
                const int j0 = n * 128;
                const int dist0 = i - j0;  // distance of key j0 + c is dist0 - c
                const bool full = (dist0 - 127 >= 0) && (W <= 0 || dist0 < W) && (j0 + 127 < T);
                float mx = -INFINITY;
                if (full && dist0 <= Dm) {
                    const float *bp = bias_h + dist0;
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        x[c] = fmaf(__uint_as_float(sr[c]), scale, __ldg(bp - c));
                        mx = fmaxf(mx, x[c]);
                    }
                } else if (full && dist0 - 127 >= Dm) {
                    const float bc = __ldg(bias_h + Dm);
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        x[c] = fmaf(__uint_as_float(sr[c]), scale, bc);
                        mx = fmaxf(mx, x[c]);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const int dist = dist0 - c;
                        const bool allowed = dist >= 0 && (W <= 0 || dist < W) && (j0 + c < T);
                        const float bv = allowed ? __ldg(bias_h + min(dist, Dm)) : 0.f;
                        x[c] = allowed ? fmaf(__uint_as_float(sr[c]), scale, bv) : -INFINITY;
                        mx = fmaxf(mx, x[c]);
                    }
                }
                // lazy rescale: move the reference only when the max grows by > tau
                const bool grow = mx > m_ref + kTau;
                float alpha = 1.f;
                if (grow) {
                    alpha = ex2((m_ref - mx) * kLog2e);
                    l *= alpha;
                    m_ref = mx;
                }
                const float mneg = (m_ref == -INFINITY) ? 0.f : -m_ref * kLog2e;
                {
                    uint32_t pk[64];
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        const float p0 = ex2(fmaf(x[2 * c], kLog2e, mneg));
                        const float p1 = ex2(fmaf(x[2 * c + 1], kLog2e, mneg));
                        l += p0 + p1;
                        pk[c] = pack_bf16(p0, p1);
                    }
                    tmem_st32(s_col + 0, pk + 0);
                    tmem_st32(s_col + 32, pk + 32);
                }
                // O rescale after P is out of registers (keeps the peak low); the
                // P.V MMA of this tile is issued only after p_full
                if (k > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                    for (int cb = 0; cb < 4; ++cb) {
                        uint32_t orr[32];
                        tmem_ld32(o_col + cb * 32, orr);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
                        tmem_st32(o_col + cb * 32, orr);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar[B_PFULL + t]);
            }
            // epilogue: O / l -> bf16
            if (!aborted && mbar_wait_warp(&bar[B_ODONE + t], 0, abort_flag, a.status)) {
                tc_fence_after();
                const float inv = (l > 0.f) ? 1.f / l : 0.f;
                uint4 *dst = (uint4 *)(a.out + (((long)b * T + i) * a.Hq + h) * 128);
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t orr[32];
                    tmem_ld32(o_col + cb * 32, orr);
                    tmem_wait_ld();
                    if (i < T) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 v;
                            v.x = pack_bf16(__uint_as_float(orr[q4 * 8 + 0]) * inv,
                                            __uint_as_float(orr[q4 * 8 + 1]) * inv);
                            v.y = pack_bf16(__uint_as_float(orr[q4 * 8 + 2]) * inv,
                                            __uint_as_float(orr[q4 * 8 + 3]) * inv);
                            v.z = pack_bf16(__uint_as_float(orr[q4 * 8 + 4]) * inv,
                                            __uint_as_float(orr[q4 * 8 + 5]) * inv);
                            v.w = pack_bf16(__uint_as_float(orr[q4 * 8 + 6]) * inv,
                                            __uint_as_float(orr[q4 * 8 + 7]) * inv);
                            dst[cb * 4 + q4] = v;
                        }
                    }
                }
                if (a.lse && i < T)
                    a.lse[((long)b * a.Hq + h) * T + i] = (l > 0.f) ? m_ref + __logf(l) : -INFINITY;
            }
        }
    } else if (warp < 12) {
        // ============================================ sconv transform (WG2) ==
        setmaxnreg_dec96();
        const int u = threadIdx.x - 256;
        volatile int *verdict = abort_flag + 1;
        // one thread waits (bounded); the whole group learns the verdict at a
        // named barrier, so no warp can be left alone inside a barrier
        auto group_wait = [&](uint64_t *br, uint32_t parity) {
            if (u == 0) *verdict = mbar_wait(br, parity, abort_flag, a.status) ? 1 : 0;
            named_bar_sync(1, 128);
            const bool good = *verdict != 0;
            if (good) (void)mbar_try_wait(br, parity);
            named_bar_sync(1, 128);  // verdict read by all before it is rewritten
            return good;
        };
        int it = 0;
        for (int n = ulo; n <= uhi; ++n, ++it) {
            const int st = it & 1;
            const uint32_t ph = (it >> 1) & 1;
            if (!group_wait(&bar[B_KRAW + st], ph)) break;
            sconv_tile_inplace(sb + SM_K + st * 32768, sb + SM_KH + st * 2048, w_sm, u);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (u == 0) mbar_arrive(&bar[B_KREADY + st]);
            if (!group_wait(&bar[B_VRAW + st], ph)) break;
            sconv_tile_inplace(sb + SM_V + st * 32768, sb + SM_VH + st * 2048, w_sm + 512, u);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (u == 0) mbar_arrive(&bar[B_VREADY + st]);
        }
    } else {
        setmaxnreg_dec48();
        if (warp == 12 && lane == 0) {
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
    PrefillArgs a;
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
    a.nqb = (p.seq_len + kQRows - 1) / kQRows;
    const long grid = (long)a.B * a.Hq * a.nqb;
    if (grid == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPrefillSmem);
    if (e != cudaSuccess) return e;
    attn_prefill_kernel<<<(unsigned)grid, 512, kPrefillSmem, stream>>>(maps[0], maps[1], maps[2],
                                                                      maps[3], maps[4], a);
    return cudaGetLastError();
}

}  // namespace inkling
