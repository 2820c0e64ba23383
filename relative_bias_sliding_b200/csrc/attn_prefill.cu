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
#include "common.cuh"

namespace inkling {

constexpr int kQRows = 256;
constexpr uint32_t SM_Q = 0;            // 2 tiles x 32 KB
constexpr uint32_t SM_K = 65536;        // 2 stages x 32 KB
constexpr uint32_t SM_V = 131072;       // 2 stages x 32 KB
constexpr uint32_t SM_KH = 196608;      // 2 stages x 2 KB (8 history rows x 2 halves)
constexpr uint32_t SM_VH = 200704;      // 2 stages x 2 KB
constexpr uint32_t SM_BIAS = 204800;    // 2 softmax groups x 2 buffers x 4 copies x 264 fp32
constexpr int kBiasCopy = 264;          // floats per shifted copy (== 8 mod 32: conflict-free)
constexpr int kBiasBuf = 4 * kBiasCopy;
constexpr uint32_t SM_BAR = SM_BIAS + 2 * 2 * kBiasBuf * 4;  // mbarriers, tmem base, flags
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

struct PrefillArgs {
    const float *w_k, *w_v, *bias;
    uint16_t *out;
    float *lse;
    int32_t *status;
    int B, T, Hq, Hkv, window, d_max, nqb;
};

// Register split per warpgroup: 2 x 128 softmax threads at 176, 128 sconv
// threads at 112, 128 producer/MMA/idle threads at 48: 45056 + 14336 + 6144 =
// 65536 = 512 threads x the 128 registers the kernel launches with (ptxas
// reports 128), so the increase never waits on registers that do not exist.
INK_DEV void setmaxnreg_inc176() { asm volatile("setmaxnreg.inc.sync.aligned.u32 176;"); }
INK_DEV void setmaxnreg_dec112() { asm volatile("setmaxnreg.dec.sync.aligned.u32 112;"); }
INK_DEV void setmaxnreg_dec48() { asm volatile("setmaxnreg.dec.sync.aligned.u32 48;"); }

// Convert one raw 128-row key or value tile (TMA layout: two 64-column halves
// of 128 rows x 128 bytes, 128-byte swizzle) into its sconv output, in place,
// with 64 threads.  Thread v owns 16-byte column c = v % 16 (8 channels) and
// rows 32g..32g+31, g = v / 16; the 3 rows before its first row come from the
// tile itself, or for g = 0 from the 8-row history box loaded with the tile.
// w[tap][pair] holds the taps of channel pairs (2p, 2p+1) of this column.
INK_DEV void sconv_tile_group(uint32_t tile, uint32_t hist, const f32x2 (&w)[4][4], int v,
                              int bar_id) {
    const int c = v & 15, g = v >> 4;
    const int half = c >> 3, cc = c & 7;
    const uint32_t tb = tile + half * 16384;
    f32x2 h3[4], h2[4], h1[4];
    auto load = [&](uint32_t base, int r, f32x2(&dst)[4]) {
        const uint4 q = lds128(base + r * 128 + ((cc ^ (r & 7)) << 4));
        dst[0] = bf2_to_f2(q.x);
        dst[1] = bf2_to_f2(q.y);
        dst[2] = bf2_to_f2(q.z);
        dst[3] = bf2_to_f2(q.w);
    };
    if (g == 0) {
        const uint32_t hb = hist + half * 1024;
        load(hb, 5, h3);
        load(hb, 6, h2);
        load(hb, 7, h1);
    } else {
        load(tb, 32 * g - 3, h3);
        load(tb, 32 * g - 2, h2);
        load(tb, 32 * g - 1, h1);
    }
    named_bar_sync(bar_id, 64);  // every history row read before any row is overwritten
#pragma unroll 4
    for (int i = 0; i < 32; ++i) {
        const int r = 32 * g + i;
        const uint32_t addr = tb + r * 128 + ((cc ^ (r & 7)) << 4);
        f32x2 x[4];
        load(tb, r, x);
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            // same order as the decode append: w3*x[t-3], +w2*x[t-2], +w1*x[t-1], +w0*x[t]
            f32x2 acc = fmul2(w[3][p], h3[p]);
            acc = ffma2(w[2][p], h2[p], acc);
            acc = ffma2(w[1][p], h1[p], acc);
            acc = ffma2(w[0][p], x[p], acc);
            o[p] = f2_to_bf2(acc);
        }
        sts128(addr, make_uint4(o[0], o[1], o[2], o[3]));
#pragma unroll
        for (int p = 0; p < 4; ++p) { h3[p] = h2[p]; h2[p] = h1[p]; h1[p] = x[p]; }
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
        setmaxnreg_inc176();
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
            float *bias_sm = (float *)(smem + SM_BIAS) + t * 2 * kBiasBuf;
            const int o_rd = 127 - u, sh = o_rd & 3;  // this row's start in the staged diagonal
            bool dead = false;
            int k = 0;
            for (int n = lo[t]; n <= hi[t]; ++n, ++k) {
                const int j0 = n * 128;
                // Stage the bias diagonal of this (query tile, key tile) pair:
                // R[q] = bias[h, clamp(top - q, 0, d_max)], q = 0..254, top = r0 - j0 + 127,
                // as 4 copies shifted by 0..3 floats so that row u reads R[127-u+c],
                // c = 0..127, with aligned 16-byte loads.  Double-buffered by tile parity.
                float *bb = bias_sm + (k & 1) * kBiasBuf;
                {
                    const int top = r0[t] - j0 + 127;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int q = 2 * u + e;
                        if (q < 255) {
                            const float bv = __ldg(bias_h + min(max(top - q, 0), Dm));
#pragma unroll
                            for (int s4 = 0; s4 < 4; ++s4)
                                if (q >= s4) bb[s4 * kBiasCopy + q - s4] = bv;
                        }
                    }
                }
                named_bar_sync(3 + t, 128);
                if (!dead) dead = !mbar_wait_warp(&bar[B_SFULL + t], k & 1, abort_flag, a.status);
                if (dead) continue;  // keep stepping through the group barrier
                tc_fence_after();
                uint32_t sr[128];
                tmem_ld32(s_col + 0, sr + 0);
                tmem_ld32(s_col + 32, sr + 32);
                tmem_ld32(s_col + 64, sr + 64);
                tmem_ld32(s_col + 96, sr + 96);
                tmem_wait_ld();
                const float4 *rp = (const float4 *)(bb + sh * kBiasCopy + (o_rd - sh));
                float x[128];
                const int dist0 = i - j0;  // distance of key j0 + c is dist0 - c
                const bool full = (dist0 - 127 >= 0) && (W <= 0 || dist0 < W) && (j0 + 127 < T);
                if (full) {
                    const f32x2 sc2 = pk2(scale, scale);
#pragma unroll
                    for (int c4 = 0; c4 < 32; ++c4) {
                        const float4 b4 = rp[c4];
                        const f32x2 xa = ffma2(pk2(__uint_as_float(sr[4 * c4]),
                                                   __uint_as_float(sr[4 * c4 + 1])),
                                               sc2, pk2(b4.x, b4.y));
                        const f32x2 xb = ffma2(pk2(__uint_as_float(sr[4 * c4 + 2]),
                                                   __uint_as_float(sr[4 * c4 + 3])),
                                               sc2, pk2(b4.z, b4.w));
                        upk2(xa, x[4 * c4], x[4 * c4 + 1]);
                        upk2(xb, x[4 * c4 + 2], x[4 * c4 + 3]);
                    }
                } else {
#pragma unroll
                    for (int c4 = 0; c4 < 32; ++c4) {
                        const float4 b4 = rp[c4];
                        const float bq[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = 4 * c4 + e;
                            const int dist = dist0 - c;
                            const bool allowed = dist >= 0 && (W <= 0 || dist < W) && (j0 + c < T);
                            x[c] = allowed ? fmaf(__uint_as_float(sr[c]), scale, bq[e]) : -INFINITY;
                        }
                    }
                }
                // row max: 8 independent chains of 3-input max
                float m8[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) m8[q] = fmaxf(x[2 * q], x[2 * q + 1]);
#pragma unroll
                for (int c = 16; c < 128; c += 16)
#pragma unroll
                    for (int q = 0; q < 8; ++q) m8[q] = max3f(m8[q], x[c + 2 * q], x[c + 2 * q + 1]);
                const float mx = fmaxf(max3f(m8[0], m8[1], m8[2]),
                                       max3f(max3f(m8[3], m8[4], m8[5]), m8[6], m8[7]));
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
                    const f32x2 l2e2 = pk2(kLog2e, kLog2e), mneg2 = pk2(mneg, mneg);
                    f32x2 acc[4] = {0ull, 0ull, 0ull, 0ull};
                    uint32_t pk[64];
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        const f32x2 tt = ffma2(pk2(x[2 * c], x[2 * c + 1]), l2e2, mneg2);
                        float t0, t1;
                        upk2(tt, t0, t1);
                        const float p0 = ex2(t0), p1 = ex2(t1);
                        acc[c & 3] = fadd2(acc[c & 3], pk2(p0, p1));
                        pk[c] = pack_bf16(p0, p1);
                    }
                    tmem_st32(s_col + 0, pk + 0);
                    tmem_st32(s_col + 32, pk + 32);
                    const f32x2 s01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
                    float la, lb;
                    upk2(s01, la, lb);
                    l += la + lb;
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
            const bool aborted = dead;
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
        setmaxnreg_dec112();
        const bool is_v = warp >= 10;
        const int v = threadIdx.x - (is_v ? 320 : 256);
        const int bar_id = is_v ? 2 : 1;
        // taps of this thread's 8 channels, as channel pairs, held for the whole block
        f32x2 w[4][4];
        {
            const float *wg = (is_v ? a.w_v : a.w_k) + ((long)kvh * 128 + 8 * (v & 15)) * 4;
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int tap = 0; tap < 4; ++tap)
                    w[tap][p] = pk2(__ldg(wg + (2 * p) * 4 + tap), __ldg(wg + (2 * p + 1) * 4 + tap));
        }
        uint64_t *raw_full = &bar[is_v ? B_VRAW : B_KRAW];
        uint64_t *ready = &bar[is_v ? B_VREADY : B_KREADY];
        const uint32_t tiles = sb + (is_v ? SM_V : SM_K);
        const uint32_t hists = sb + (is_v ? SM_VH : SM_KH);
        bool dead = false;
        int it = 0;
        for (int n = ulo; n <= uhi; ++n, ++it) {
            const int st = it & 1;
            if (!dead) dead = !mbar_wait(&raw_full[st], (it >> 1) & 1, abort_flag, a.status);
            if (dead) {
                named_bar_sync(bar_id, 64);  // keep the group's barrier count matched
                continue;
            }
            sconv_tile_group(tiles + st * 32768, hists + st * 2048, w, v, bar_id);
            fence_proxy_async_smem();
            mbar_arrive(&ready[st]);
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
