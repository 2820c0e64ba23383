// attn_decode_mq.cu — multi-token decode on tcgen05 tensor cores: the q_len
// newest tokens of each sequence (the draft tokens of speculative decoding /
// multi-token prediction; vLLM Recipes "thinkingmachines/Inkling", Overview,
// MTP bullet: up to 9 tokens per forward step) attend to the paged cache.
// Query qi of sequence s sits at position L - q_len + qi and sees keys up to
// itself, inside the window, with the bias at its own distance.
//
// One thread block = one (sequence, kv head, split).  All G * q_len (token,
// head) rows of the kv head (at most 80) form one 128-row tile: a single 3-D
// TMA box gathers them (q viewed as [S*q_len, Hq, d], box {64, G, q_len}),
// rows ordered r = qi*G + g.  Key tiles are 64 tokens, half a cache block
// (two 64-column TMA boxes each for keys and values, 128-byte swizzle), keys
// in 3 stages and values in 2, so a block needs ~108 KB of shared memory and
// 256 TMEM columns and two blocks share an SM: one's softmax runs while the
// other waits on its tiles.
//   S = Q K^T: tcgen05 M=128 N=64 into one of two TMEM buffers, so the MMA
//     of key tile k+1 runs while the softmax works on tile k;
//   P (bf16) over the first 32 columns of its S buffer; O += P V (TMEM A);
//   the softmax (4 warps, thread = row = TMEM lane) reads each row's bias
//     from per-head diagonals staged in shared memory (head stride 4 mod 32
//     floats: the 4 tokens x 8 heads of a warp hit distinct banks), masks the
//     row's columns outside its causal/window range, and rescales O only when
//     its running maximum grows by more than 8 (log2 units), after the
//     previous P.V has completed.
// The key range of a sequence (union of its rows' windows) is cut into
// `splits` runs of tiles on separate blocks; with more than one split the
// block writes unnormalised partials (max in log2 units, sum, O) that
// decode_combine_kernel merges, as for single-token decode.
#include "common.cuh"

#include <type_traits>

namespace inkling {

cudaError_t launch_decode_combine(const float *part_o, const float *part_ml, uint16_t *out, float *lse,
                                  long rows, int splits, cudaStream_t stream);

// A (sequence, token, head) row this call could not compute (length out of
// range, or a bounded wait gave up) reads NaN in out and lse; with splits, a
// NaN partial makes the merged row NaN.
__device__ __noinline__ void decode_nan_row(uint16_t *out, float *lse, float *part_ml, int splits,
                                            long pair, long pbase, int split) {
    const float nanv = __int_as_float(0x7fc00000);
    if (splits == 1) {
        const uint32_t nb = 0x7fc07fc0u;
        uint4 *dst = (uint4 *)(out + pair * 128);
        for (int c = 0; c < 16; ++c) dst[c] = make_uint4(nb, nb, nb, nb);
        if (lse) lse[pair] = nanv;
    } else {
        const long pi = (pair - pbase) * splits + split;
        part_ml[pi * 2] = nanv;
        part_ml[pi * 2 + 1] = nanv;
    }
}

constexpr int kMqTile = 64;                       // keys per tile (half a cache block)
constexpr int kMqHead = 100;                      // floats per head diagonal (>= 63 + 10, == 4 mod 32)
constexpr int kMqBiasBuf = 8 * kMqHead;
// The query tile holds at most 80 rows (two 10 KB d halves).  The M=128 MMA
// also reads rows 80..127 of each half, which lie in the next half or in the
// first key stage: those rows' S, P and O are never used.
constexpr uint32_t kMqQHalf = 10240;              // 80 rows x 128 B
constexpr int kMqKStages = 3;                     // keys: 3 stages, values: 2
constexpr uint32_t MQ_Q = 0;
constexpr uint32_t MQ_K = 2 * kMqQHalf;           // 3 stages x 16 KB (two 64-row d halves)
constexpr uint32_t MQ_V = MQ_K + kMqKStages * 16384;  // 2 stages x 16 KB
constexpr uint32_t MQ_BIAS = MQ_V + 2 * 16384;    // 2 buffers of staged diagonals
constexpr uint32_t MQ_BAR = MQ_BIAS + 2 * kMqBiasBuf * 4;
constexpr int kMqSmem = MQ_BAR + 256 + 1024;

enum {
    M_QFULL = 0,
    M_KFULL = 1,    // +key stage
    M_VFULL = 4,    // +value stage
    M_KEMPTY = 6,
    M_VEMPTY = 9,
    M_SFULL = 11,   // +S buffer
    M_PFULL = 13,   // +S buffer (128 arrivals)
    M_OREADY = 15,  // one phase per P.V issued
    M_DRAIN = 16,
    M_ODONE = 17,   // the last P.V has completed (one phase)
    M_COUNT = 18
};

struct DecodeMqArgs {
    const int32_t *block_table, *seq_lens;
    const float *bias;
    uint16_t *out;
    float *lse;
    float *part_o, *part_ml;
    int32_t *status;
    int S, Q, Hq, Hkv, G, max_blocks, num_blocks, window, d_max, splits;
    // sequences [0, s_whole) run unsplit (one block per kv head, output
    // written directly); sequences [s_whole, S) in `splits` key-range pieces
    // whose partials start at row pbase = s_whole * Q * Hq
    int s_whole;
    long pbase;
};

__global__ void __launch_bounds__(192, 2)
decode_mq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const DecodeMqArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bar = (uint64_t *)(smem + MQ_BAR);
    uint32_t *tmem_slot = (uint32_t *)(bar + M_COUNT);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blocks of the whole sequences first (they are dispatched first), then
    // the pieces of the others
    const int nwhole = a.s_whole * a.Hkv;
    int s, kvh, split, splits;
    if ((int)blockIdx.x < nwhole) {
        s = blockIdx.x % a.s_whole;
        kvh = blockIdx.x / a.s_whole;
        split = 0;
        splits = 1;
    } else {
        const int j = blockIdx.x - nwhole, Sr = a.S - a.s_whole;
        s = a.s_whole + j % Sr;
        kvh = (j / Sr) % a.Hkv;
        split = j / (Sr * a.Hkv);
        splits = a.splits;
    }
    const int Q = a.Q, G = a.G, rows = G * Q;

    // key tiles of this sequence (union of its rows' windows) and this split
    const int L = a.seq_lens[s];
    const bool bad_len = (L < Q || L > a.max_blocks * 128);
    const int klo = (a.window > 0) ? max(0, L - Q - a.window + 1) : 0;
    int ta = 0, tb = 0;
    if (!bad_len) {
        const int t_lo = klo / kMqTile, t_hi = (L - 1) / kMqTile;
        const int per = (t_hi - t_lo + splits) / splits;
        ta = min(t_hi + 1, t_lo + split * per);
        tb = min(t_hi + 1, ta + per);
    } else if (threadIdx.x == 0 && split == 0 && kvh == 0) {
        report_status(a.status, INKLING_STATUS_BAD_LENGTH);
    }
    const int nt = tb - ta;

    if (threadIdx.x == 0) {
        for (int i = 0; i < M_COUNT; ++i)
            mbar_init(&bar[i], (i == M_PFULL || i == M_PFULL + 1) ? 128 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp < 4) {
        // ============================================ softmax (thread = row) ==
        const int u = threadIdx.x;
        const bool rv = u < rows;
        // a warp whose 32 rows are all padding (G * q_len <= 96) computes
        // nothing: it stages bias, keeps the barrier and arrives on P_FULL
        // (its P rows are never read for an output)
        const bool live = warp * 32 < rows;
        const int qi = rv ? u / G : 0, g = rv ? u % G : 0;
        const int h = kvh * G + g;
        const int ipos = L - Q + qi;  // this row's query position
        const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
        const uint32_t o_col = tl + 128;
        const float scale = 0.08838834764831845f;  // 1/sqrt(128)
        const float kLog2e = 1.4426950408889634f;
        const float kTau = 5.545177444479562f;     // 8 ln 2
        const int W = a.window, Dm = a.d_max;
        float m_ref = -INFINITY, l = 0.f;
        const int o_rd = Q - 1 - qi;     // start of this row in its head's diagonal
        const int span = Q + kMqTile - 1;  // staged values per head
        bool dead = bad_len;
        // diagonal of head g for key tile k: R[kk] = bias[h_g, clamp(L-1-j0-kk, 0, d_max)]
        // (row qi reads R[Q-1-qi + c] for column c); thread t holds elements
        // t, t+128, ... of the G x span values, fetched one tile ahead and
        // stored under the next barrier
        constexpr int kPer = (8 * (10 + kMqTile - 1) + 127) / 128;  // G <= 8, Q <= 10
        float nxt[kPer];
        // this thread's (head, offset) pairs, the same for every tile (-1: none)
        int egg[kPer], ekk[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = threadIdx.x + 128 * i;
            egg[i] = e < G * span ? e / span : -1;
            ekk[i] = e < G * span ? e % span : 0;
        }
        auto fetch = [&](int k) {
            const int top = L - 1 - (ta + k) * kMqTile;
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if (egg[i] >= 0)
                    nxt[i] = __ldg(a.bias + (long)(kvh * G + egg[i]) * (Dm + 1) +
                                   min(max(top - ekk[i], 0), Dm));
        };
        auto stage = [&](int k) {
            float *bb = (float *)(smem + MQ_BIAS) + (k & 1) * kMqBiasBuf;
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if (egg[i] >= 0) bb[egg[i] * kMqHead + ekk[i]] = nxt[i];
        };
        if (nt > 0) {
            fetch(0);
            stage(0);
        }
        for (int k = 0; k < nt; ++k) {
            const int j0 = (ta + k) * kMqTile;
            const float *bb = (const float *)(smem + MQ_BIAS) + (k & 1) * kMqBiasBuf;
            named_bar_sync(1, 128);  // tile k's diagonals are staged; tile k-1's reads are done
            if (k + 1 < nt) fetch(k + 1);
            if (!live) {
                mbar_arrive(&bar[M_PFULL + (k & 1)]);
                if (k + 1 < nt) stage(k + 1);
                continue;
            }
            if (!dead) dead = !mbar_wait_warp(&bar[M_SFULL + (k & 1)], (k >> 1) & 1, abort_flag, a.status);
            if (dead) {
                if (k + 1 < nt) stage(k + 1);
                continue;  // keep stepping through the group barrier
            }
            tc_fence_after();
            const uint32_t s_col = tl + (k & 1) * kMqTile;
            uint32_t sr[64];
            tmem_ld32(s_col + 0, sr + 0);
            tmem_ld32(s_col + 32, sr + 32);
            tmem_wait_ld();
            // columns this row may see: ipos - j0 - c in [0, W).  The choice
            // of path is warp-uniform and padding rows (whose S, P and O are
            // never read) take no part in it: a warp that held both paths ran
            // both, one after the other
            const int dist0 = ipos - j0;
            const int cmax = rv ? min(kMqTile - 1, dist0) : kMqTile - 1;
            const int cmin = (rv && W > 0) ? max(0, dist0 - W + 1) : 0;
            const bool full = __all_sync(0xffffffffu, cmin == 0 && cmax == kMqTile - 1);
            const float *rb = bb + g * kMqHead + o_rd;
            float x[64];
            float m8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
            const f32x2 sc2 = pk2(scale, scale);
            auto logits = [&](auto masked) {
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) {
                    float4 b4[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        b4[j] = make_float4(rb[32 * cb + 4 * j], rb[32 * cb + 4 * j + 1],
                                            rb[32 * cb + 4 * j + 2], rb[32 * cb + 4 * j + 3]);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int c = 32 * cb + 4 * j;
                        const f32x2 xa = ffma2(pk2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                               sc2, pk2(b4[j].x, b4[j].y));
                        const f32x2 xb = ffma2(pk2(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])),
                                               sc2, pk2(b4[j].z, b4[j].w));
                        upk2(xa, x[c], x[c + 1]);
                        upk2(xb, x[c + 2], x[c + 3]);
                        if (decltype(masked)::value) {
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                x[c + e] = (c + e >= cmin && c + e <= cmax) ? x[c + e] : -INFINITY;
                        }
                        m8[j] = max3f(max3f(m8[j], x[c], x[c + 1]), x[c + 2], x[c + 3]);
                    }
                }
            };
            if (full)
                logits(std::false_type{});
            else
                logits(std::true_type{});
            const float mx =
                fmaxf(max3f(m8[0], m8[1], m8[2]), max3f(max3f(m8[3], m8[4], m8[5]), m8[6], m8[7]));
            const bool grow = rv && mx > m_ref + kTau;
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
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const f32x2 tt = ffma2(pk2(x[2 * c], x[2 * c + 1]), l2e2, mneg2);
                    float t0, t1;
                    upk2(tt, t0, t1);
                    const float p0 = ex2(t0), p1 = ex2(t1);
                    acc[c & 3] = fadd2(acc[c & 3], pk2(p0, p1));
                    pk[c] = pack_bf16(p0, p1);
                }
                tmem_st32(s_col, pk);
                const f32x2 s01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
                float la, lb;
                upk2(s01, la, lb);
                l += la + lb;
            }
            // O rescale, after the previous tile's P.V has completed (at most
            // that phase can have completed: the next P.V waits for this P)
            if (k > 0 && __any_sync(0xffffffffu, grow)) {
                if (!mbar_wait_warp(&bar[M_OREADY], (k - 1) & 1, abort_flag, a.status)) {
                    dead = true;
                } else {
                    tc_fence_after();
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
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar[M_PFULL + (k & 1)]);
            if (k + 1 < nt) stage(k + 1);
        }
        // epilogue: the last P.V has completed.  It has a one-phase barrier of
        // its own: a parity wait on M_OREADY could match the phase of the P.V
        // two tiles back if the one before it had not completed yet
        const bool have_o = live && !dead && nt > 0 &&
                            mbar_wait_warp(&bar[M_ODONE], 0, abort_flag, a.status);
        if (have_o) tc_fence_after();
        uint32_t ob[128];
        if (have_o) {
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tmem_ld32(o_col + cb * 32, ob + cb * 32);
            tmem_wait_ld();
        }
        auto o = [&](int i) { return __uint_as_float(ob[i]); };
        if (rv && !bad_len && !*abort_flag) {
            const long pair = ((long)s * Q + qi) * a.Hq + h;
            if (splits == 1) {
                const float inv = (l > 0.f) ? 1.f / l : 0.f;
                uint4 *dst = (uint4 *)(a.out + pair * 128);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    uint4 v;
                    v.x = pack_bf16(o(8 * c + 0) * inv, o(8 * c + 1) * inv);
                    v.y = pack_bf16(o(8 * c + 2) * inv, o(8 * c + 3) * inv);
                    v.z = pack_bf16(o(8 * c + 4) * inv, o(8 * c + 5) * inv);
                    v.w = pack_bf16(o(8 * c + 6) * inv, o(8 * c + 7) * inv);
                    dst[c] = v;
                }
                if (a.lse) a.lse[pair] = (l > 0.f) ? m_ref + __logf(l) : -INFINITY;
            } else {
                const long pi = (pair - a.pbase) * splits + split;
                float4 *po = (float4 *)(a.part_o + pi * 128);
                if (have_o) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        po[c] = make_float4(o(4 * c), o(4 * c + 1), o(4 * c + 2), o(4 * c + 3));
                }
                // an empty split (or row) contributes nothing: max -inf
                a.part_ml[pi * 2] = (have_o && l > 0.f) ? m_ref * kLog2e : -INFINITY;
                a.part_ml[pi * 2 + 1] = have_o ? l : 0.f;
            }
        }
    } else if (warp == 4 && lane == 0) {
        // ============================================== TMA producer ==
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (nt > 0) {
            mbar_arrive_expect_tx(&bar[M_QFULL], 2 * rows * 128);
            tma_load_3d(smem + MQ_Q, &tm_q, &bar[M_QFULL], 0, kvh * G, s * Q);
            tma_load_3d(smem + MQ_Q + kMqQHalf, &tm_q, &bar[M_QFULL], 64, kvh * G, s * Q);
        }
        // cache row of key tile k (half n % 2 of cache block n / 2)
        auto tile_row = [&](int k) {
            int blk = a.block_table[(long)s * a.max_blocks + (ta + k) / 2];
            if (blk < 0 || blk >= a.num_blocks) {
                report_status(a.status, INKLING_STATUS_BAD_BLOCK);
                blk = 0;  // keep the pipeline running on a valid block
            }
            return (blk * a.Hkv + kvh) * 128 + ((ta + k) & 1) * kMqTile;
        };
        // Loads in the order their stages free up: K0 K1 K2 V0 K3 V1 K4 V2 ...
        // V(k) waits for P.V(k-2), K(k+3) for QK^T(k), and the MMA runs
        // QK^T(k) before P.V(k-1).  Keys are fetched three tiles ahead, values
        // two.
        int kk = 0, vv = 0;
        while (kk < nt || vv < nt) {
            if (kk < nt && kk < vv + kMqKStages) {
                const int st = kk % kMqKStages;
                const int row = tile_row(kk);
                if (!mbar_wait(&bar[M_KEMPTY + st], ((kk / kMqKStages) & 1) ^ 1, abort_flag, a.status))
                    break;
                mbar_arrive_expect_tx(&bar[M_KFULL + st], 16384);
                tma_load_2d(smem + MQ_K + st * 16384, &tm_k, &bar[M_KFULL + st], 0, row);
                tma_load_2d(smem + MQ_K + st * 16384 + 8192, &tm_k, &bar[M_KFULL + st], 64, row);
                ++kk;
            } else {
                const int st = vv & 1;
                const int row = tile_row(vv);
                if (!mbar_wait(&bar[M_VEMPTY + st], ((vv >> 1) & 1) ^ 1, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&bar[M_VFULL + st], 16384);
                tma_load_2d(smem + MQ_V + st * 16384, &tm_v, &bar[M_VFULL + st], 0, row);
                tma_load_2d(smem + MQ_V + st * 16384 + 8192, &tm_v, &bar[M_VFULL + st], 64, row);
                ++vv;
            }
        }
        // drain: every load issued has landed before the block may exit
        if (nt > 0) mbar_wait(&bar[M_QFULL], 0, nullptr, a.status);
        for (int k = max(0, kk - kMqKStages); k < kk; ++k)
            mbar_wait(&bar[M_KFULL + k % kMqKStages], (k / kMqKStages) & 1, nullptr, a.status);
        for (int k = max(0, vv - 2); k < vv; ++k)
            mbar_wait(&bar[M_VFULL + (k & 1)], (k >> 1) & 1, nullptr, a.status);
    } else if (warp == 5 && lane == 0) {
        // ================================================ MMA issuer ==
        const uint32_t id_qk = idesc_bf16(128, kMqTile, 0, 0);
        const uint32_t id_pv = idesc_bf16(128, 128, 0, 1);
        auto issue_qk = [&](int k) {
            const int st = k % kMqKStages;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad =
                    sw128_desc(sb + MQ_Q + (ks >> 2) * kMqQHalf + (ks & 3) * 32, 16, 1024);
                const uint64_t bd =
                    sw128_desc(sb + MQ_K + st * 16384 + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                umma_ss(tbase + (k & 1) * kMqTile, ad, bd, id_qk, ks > 0 ? 1u : 0u);
            }
        };
        auto issue_pv = [&](int k) {
            const int st = k & 1;
#pragma unroll
            for (int ks = 0; ks < kMqTile / 16; ++ks) {
                const uint64_t bd = sw128_desc(sb + MQ_V + st * 16384 + ks * 2048, 8192, 1024);
                umma_ts(tbase + 128, tbase + (k & 1) * kMqTile + ks * 8, bd, id_pv,
                        (k > 0 || ks > 0) ? 1u : 0u);
            }
        };
        bool alive = nt == 0 || mbar_wait(&bar[M_QFULL], 0, abort_flag, a.status);
        // QK(0) QK(1) | PV(0) QK(2) | PV(1) QK(3) | ...: the QK^T of the next
        // tile runs while the softmax works on the current one
        for (int k = 0; k <= nt && alive; ++k) {
            if (k < nt) {
                if (!mbar_wait(&bar[M_KFULL + k % kMqKStages], (k / kMqKStages) & 1, abort_flag,
                               a.status))
                    break;
                tc_fence_after();
                issue_qk(k);
                tc_commit(&bar[M_SFULL + (k & 1)]);
                tc_commit(&bar[M_KEMPTY + k % kMqKStages]);
            }
            if (k >= 1) {
                const int kp = k - 1;
                if (!mbar_wait(&bar[M_PFULL + (kp & 1)], (kp >> 1) & 1, abort_flag, a.status) ||
                    !mbar_wait(&bar[M_VFULL + (kp & 1)], (kp >> 1) & 1, abort_flag, a.status))
                    break;
                tc_fence_after();
                issue_pv(kp);
                tc_commit(&bar[M_OREADY]);
                tc_commit(&bar[M_VEMPTY + (kp & 1)]);
                if (kp == nt - 1) tc_commit(&bar[M_ODONE]);
            }
        }
        // every MMA issued has completed before TMEM is released
        tc_commit(&bar[M_DRAIN]);
        mbar_wait(&bar[M_DRAIN], 0, nullptr, a.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
    // rows this call could not compute read NaN: after the block's work, so
    // that the main loop's code stays as it is without this rare path (in the
    // epilogue it cost the kernel 6%)
    if (warp < 4 && (int)threadIdx.x < rows && (bad_len || *abort_flag))
        decode_nan_row(a.out, a.lse, a.part_ml, splits,
                       ((long)s * Q + threadIdx.x / G) * a.Hq + kvh * G + threadIdx.x % G, a.pbase,
                       split);
}

// s_whole: sequences [0, s_whole) run unsplit, the rest in `splits` pieces
// (s_whole == num_seqs: no partials; 0: every sequence split).
cudaError_t launch_attn_decode_mq(const inkling_decode_params &p, int splits, int s_whole,
                                  void *workspace, const CUtensorMap &tm_q,
                                  const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                                  cudaStream_t stream) {
    DecodeMqArgs a;
    a.block_table = p.block_table;
    a.seq_lens = p.seq_lens;
    a.bias = p.bias;
    a.out = (uint16_t *)p.out;
    a.lse = p.lse;
    a.status = p.status;
    a.S = p.num_seqs;
    a.Q = p.q_len;
    a.Hq = p.num_q_heads;
    a.Hkv = p.num_kv_heads;
    a.G = p.num_q_heads / p.num_kv_heads;
    a.max_blocks = p.max_blocks;
    a.num_blocks = p.num_blocks;
    a.window = p.window;
    a.d_max = p.d_max;
    if (splits == 1) s_whole = p.num_seqs;
    a.splits = splits;
    a.s_whole = s_whole;
    a.pbase = (long)s_whole * p.q_len * p.num_q_heads;
    const long rows_part = (long)(p.num_seqs - s_whole) * p.q_len * p.num_q_heads;
    a.part_o = (float *)workspace;
    a.part_ml = rows_part > 0 ? (float *)workspace + rows_part * splits * 128 : nullptr;
    cudaError_t e = cudaFuncSetAttribute(decode_mq_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kMqSmem);
    if (e != cudaSuccess) return e;
    const long grid = (long)s_whole * p.num_kv_heads +
                      (long)(p.num_seqs - s_whole) * p.num_kv_heads * splits;
    if (grid == 0) return cudaSuccess;
    decode_mq_tc_kernel<<<(unsigned)grid, 192, kMqSmem, stream>>>(tm_q, tm_k, tm_v, a);
    e = cudaGetLastError();
    if (e != cudaSuccess || rows_part == 0) return e;
    return launch_decode_combine(a.part_o, a.part_ml, a.out + a.pbase * 128,
                                 a.lse ? a.lse + a.pbase : nullptr, rows_part, splits, stream);
}

}  // namespace inkling
