// prefill_common.cuh — pieces shared by the two prefill kernels (one CTA per
// query block, or a 2-CTA cluster sharing every key/value tile): arguments,
// the register split, the in-place sconv transform of a raw key/value tile and
// the softmax role of one 128-row query tile.
#pragma once

#include "common.cuh"

#include <type_traits>

namespace inkling {

constexpr int kQRows = 256;     // query rows per CTA: two 128-row tiles
constexpr int kBiasCopy = 264;  // floats per shifted bias copy (== 8 mod 32: conflict-free)
constexpr int kBiasBuf = 4 * kBiasCopy;
constexpr int kBiasBytes = 2 * 2 * kBiasBuf * 4;  // 2 query tiles x 2 buffers

struct PrefillArgs {
    const float *w_k, *w_v, *bias;
    uint16_t *out;
    float *lse;
    int32_t *status;
    int B, T, Hq, Hkv, window, d_max, nqb;
};

// Optional outputs of the prefill (a kernel argument of its own, so that the
// plain prefill's argument block and registers are those without them):
// post-sconv keys/values into the paged cache [num_blocks, Hkv, 128, 128]
// through block_table [B, max_blocks], and the new sconv state
// [B, 3, Hkv*128] (the last 3 raw rows of k_raw / v_raw).
struct FillArgs {
    uint16_t *k_cache, *v_cache, *k_state, *v_state;
    const int32_t *block_table;
    const uint16_t *k_raw, *v_raw;
    int max_blocks, num_blocks;
};

// Where the converted rows of key tile n go in the paged cache: the address of
// tile row 0 (token n*128 + row_base) at channel `ch` of kv head kvh.  A block
// id outside the pool is reported and gives nullptr (nothing is written).
INK_DEV uint16_t *cache_rows(const FillArgs &f, const PrefillArgs &a, uint16_t *cache, int b,
                             int kvh, int n, int row_base, int ch) {
    const int blk = __ldg(f.block_table + (long)b * f.max_blocks + n);
    if (blk < 0 || blk >= f.num_blocks) {
        report_status(a.status, INKLING_STATUS_BAD_BLOCK);
        return nullptr;
    }
    return cache + (((long)blk * a.Hkv + kvh) * 128 + row_base) * 128 + ch;
}

// New sconv state of (sequence b, kv head kvh) after a prefill of T tokens
// from zero history: rows T-3..T-1 of the raw keys/values (zero where the
// index is negative), for both K and V.  One warp; 16-byte copies.
INK_DEV void write_sconv_state(const FillArgs &f, const PrefillArgs &a, int b, int kvh, int lane) {
    const long C = (long)a.Hkv * 128;
    for (int k = lane; k < 2 * 3 * 16; k += 32) {
        const bool v = k >= 48;
        const int m = (k % 48) >> 4, chunk = k & 15;
        const int t = a.T - 3 + m;
        const uint16_t *raw = v ? f.v_raw : f.k_raw;
        uint16_t *state = v ? f.v_state : f.k_state;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (t >= 0) val = *(const uint4 *)(raw + (((long)b * a.T + t) * a.Hkv + kvh) * 128 + chunk * 8);
        *(uint4 *)(state + ((long)b * 3 + m) * C + (long)kvh * 128 + chunk * 8) = val;
    }
}

// Register split per warpgroup: 2 x 128 softmax threads at 184, 128 sconv
// threads at 80, 128 producer/MMA/idle threads at 64: 47104 + 10240 + 8192 =
// 65536 = 512 threads x the 128 registers the kernels launch with (ptxas
// reports 128), so the increase never waits on registers that do not exist.
// (At 48 the MMA issuer spills, and its loads from local memory sit on the
// S -> softmax -> P -> MMA chain.)
INK_DEV void setmaxnreg_inc184() { asm volatile("setmaxnreg.inc.sync.aligned.u32 184;"); }
INK_DEV void setmaxnreg_dec80() { asm volatile("setmaxnreg.dec.sync.aligned.u32 80;"); }
INK_DEV void setmaxnreg_dec64() { asm volatile("setmaxnreg.dec.sync.aligned.u32 64;"); }
// The split of the cache-filling CTA-pair prefill: its sconv warps also store
// the converted tiles to the paged cache, and its producer / MMA group tracks
// the fill, so they get 96 and 80 registers and the softmax groups 168:
// 2 x 128 x 168 + 128 x 96 + 128 x 80 = 65536.  Measured on the
// sliding-window workload: 687 TFLOP/s against 655 with the plain split (the
// plain prefill keeps its split: 696 against 689).
INK_DEV void setmaxnreg_inc168() { asm volatile("setmaxnreg.inc.sync.aligned.u32 168;"); }
INK_DEV void setmaxnreg_dec96() { asm volatile("setmaxnreg.dec.sync.aligned.u32 96;"); }
// The splits of the paged prefill, which has no sconv warps: its four idle
// warps keep the minimum, and the softmax groups take most of the rest.
// Persistent walk: 8 x 192 + 4 x 24 + 4 x 104 = 2048; one item per CTA:
// 8 x 200 + 4 x 24 + 4 x 88 = 2048 (16 warps x 128, the launch's registers).
INK_DEV void setmaxnreg_inc192() { asm volatile("setmaxnreg.inc.sync.aligned.u32 192;"); }
INK_DEV void setmaxnreg_inc200() { asm volatile("setmaxnreg.inc.sync.aligned.u32 200;"); }
INK_DEV void setmaxnreg_dec24() { asm volatile("setmaxnreg.dec.sync.aligned.u32 24;"); }
INK_DEV void setmaxnreg_dec104() { asm volatile("setmaxnreg.dec.sync.aligned.u32 104;"); }
INK_DEV void setmaxnreg_dec88() { asm volatile("setmaxnreg.dec.sync.aligned.u32 88;"); }

// Taps of 8 consecutive channels starting at `wg` ([C, 4] fp32), as channel
// pairs: w[tap][p] = (w[2p][tap], w[2p+1][tap]).
INK_DEV void load_taps(f32x2 (&w)[4][4], const float *wg) {
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int tap = 0; tap < 4; ++tap)
            w[tap][p] = pk2(__ldg(wg + (2 * p) * 4 + tap), __ldg(wg + (2 * p + 1) * 4 + tap));
}

// In-place sconv of rows [row0, row0 + nrows) of one 16-byte column of a raw
// key/value tile.  The tile is TMA-loaded with 128-byte swizzle as 64-column
// halves of 128-byte rows (`half_bytes` apart); the 8-row history box (rows
// -8..-1, halves 1 KB apart) supplies the 3 rows before row 0.  Column `c`
// (0..15) selects half c/8 and chunk c%8.  All `nthreads` threads of the group
// read their 3 history rows before a named barrier; only then is anything
// overwritten.
INK_DEV void sconv_rows(uint32_t tile, uint32_t hist, uint32_t half_bytes, const f32x2 (&w)[4][4],
                        int c, int row0, int nrows, int bar_id, int nthreads) {
    const int half = c >> 3, cc = c & 7;
    const uint32_t tb = tile + half * half_bytes;
    f32x2 h3[4], h2[4], h1[4];
    auto load = [&](uint32_t base, int r, f32x2(&dst)[4]) {
        const uint4 q = lds128(base + r * 128 + ((cc ^ (r & 7)) << 4));
        dst[0] = bf2_to_f2(q.x);
        dst[1] = bf2_to_f2(q.y);
        dst[2] = bf2_to_f2(q.z);
        dst[3] = bf2_to_f2(q.w);
    };
    if (row0 == 0) {
        const uint32_t hb = hist + half * 1024;
        load(hb, 5, h3);
        load(hb, 6, h2);
        load(hb, 7, h1);
    } else {
        load(tb, row0 - 3, h3);
        load(tb, row0 - 2, h2);
        load(tb, row0 - 1, h1);
    }
    named_bar_sync(bar_id, nthreads);  // every history row read before any row is overwritten
#pragma unroll 4
    for (int i = 0; i < nrows; ++i) {
        const int r = row0 + i;
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

// Copy of the rows [row0, row0 + nrows) of column `c` that this thread has just
// converted (same layout as sconv_rows) to the paged cache: tile row r goes to
// gdst + r*128 (gdst = tile row 0 at this column's channels) when r < gvalid.
// Only the calling thread's own shared-memory writes are read, so no barrier
// is needed; a separate pass keeps the transform's registers unchanged.
INK_DEV void store_rows(uint32_t tile, uint32_t half_bytes, int c, int row0, int nrows,
                        uint16_t *gdst, int gvalid) {
    const uint32_t tb = tile + (c >> 3) * half_bytes;
    const int cc = c & 7;
    for (int i = 0; i < nrows; ++i) {
        const int r = row0 + i;
        if (r >= gvalid) break;
        *(uint4 *)(gdst + (long)r * 128) = lds128(tb + r * 128 + ((cc ^ (r & 7)) << 4));
    }
}

// Normalised output of one query row: O / l from tensor memory as 16 chunks of
// 8 bf16 (16 bytes), handed to store(c, chunk) for c = 0..15.
template <class Store>
INK_DEV void emit_row(uint32_t o_col, float l, Store store) {
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
        uint32_t orr[32];
        tmem_ld32(o_col + cb * 32, orr);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(orr[q4 * 8 + 0]) * inv, __uint_as_float(orr[q4 * 8 + 1]) * inv);
            v.y = pack_bf16(__uint_as_float(orr[q4 * 8 + 2]) * inv, __uint_as_float(orr[q4 * 8 + 3]) * inv);
            v.z = pack_bf16(__uint_as_float(orr[q4 * 8 + 4]) * inv, __uint_as_float(orr[q4 * 8 + 5]) * inv);
            v.w = pack_bf16(__uint_as_float(orr[q4 * 8 + 6]) * inv, __uint_as_float(orr[q4 * 8 + 7]) * inv);
            store(cb * 4 + q4, v);
        }
    }
}

// Epilogue of the dense prefill: the normalised bf16 O tile is staged in
// `stage` (the query tile's shared-memory buffer, free once the last QK^T of
// the tile has completed) in the same 128-byte-swizzled layout, and one thread
// writes it with two bulk tensor stores through `tm_out`, a [B, T, Hq, 128]
// map (rows past the sequence end are clipped).  Every thread of the group
// calls it (the named barrier counts 128).
struct TmaStoreEpilogue {
    const PrefillArgs &a;
    uint8_t *stage;
    const CUtensorMap *tm_out;
    int b, h, r0, bar_id;
    INK_DEV void operator()(bool have_o, int u, int i, float l, float m_ref, uint32_t o_col,
                            volatile int *abort_flag) const {
        if (have_o) {
            emit_row(o_col, l, [&](int c, uint4 v) {
                *(uint4 *)(stage + (c >> 3) * 16384 + u * 128 + (((c & 7) ^ (u & 7)) << 4)) = v;
            });
            if (a.lse && i < a.T)
                a.lse[((long)b * a.Hq + h) * a.T + i] = (l > 0.f) ? m_ref + __logf(l) : -INFINITY;
            fence_proxy_async_smem();
        } else if (i < a.T) {
            // a bounded wait gave up: the row reads NaN (the status word says why)
            const uint32_t nb = 0x7fc07fc0u;
            uint16_t *dst = a.out + (((long)b * a.T + i) * a.Hq + h) * 128;
#pragma unroll
            for (int c = 0; c < 16; ++c) *(uint4 *)(dst + c * 8) = make_uint4(nb, nb, nb, nb);
            if (a.lse) a.lse[((long)b * a.Hq + h) * a.T + i] = __int_as_float(0x7fc00000);
        }
        // every warp of the group reaches this barrier (have_o is uniform per warp)
        named_bar_sync(bar_id, 128);
        if (u == 0 && have_o && !*abort_flag) {
            tma_store_4d(tm_out, stage, 0, r0, h, b);
            tma_store_4d(tm_out, stage + 16384, 64, r0, h, b);
            bulk_commit_group();
            bulk_wait_read_all();
        }
    }
};

// Softmax of one 128-row query tile (the calling warpgroup; thread = row =
// TMEM lane), over key tiles lo..hi, then the epilogue.  Row u of the tile is
// the query at sequence position pos0 + u; keys exist at positions
// 0 .. key_end-1.  S lives in TMEM columns [128t, 128t+128), O in
// [256+128t, ...); P (bf16) is written over the first 64 columns of S.
// `signal_p(t)` is called by every thread once its P and O updates are
// complete and fenced; it must tell the MMA issuer.  `bias_sm` holds this
// tile's two bias-diagonal buffers; `bar_id` is a named barrier private to
// this warpgroup.  At the end every thread calls
// epilogue(have_o, u, pos0 + u, l, m_ref, o_col, abort_flag).
// `k_base` counts the key tiles this group processed before (for the parities
// of S_FULL and of the bias buffers when the group walks several work items),
// `o_phase` is the parity of this item's O_DONE phase.
template <class SignalP, class Epilogue>
INK_DEV void softmax_role(const PrefillArgs &a, float *bias_sm, uint64_t *s_full, uint64_t *o_done,
                          volatile int *abort_flag, uint32_t tbase, int t, int h, int pos0,
                          int key_end, int lo, int hi, int bar_id, int k_base, uint32_t o_phase,
                          SignalP signal_p, const Epilogue &epilogue) {
    const int u = threadIdx.x & 127;
    const uint32_t tl = tbase + ((uint32_t)(((threadIdx.x >> 5) & 3) * 32) << 16);
    const uint32_t s_col = tl + t * 128, o_col = tl + 256 + t * 128;
    const int i = pos0 + u;
    const float scale = 0.08838834764831845f;  // 1/sqrt(128)
    const float kLog2e = 1.4426950408889634f;
    const float kTau = 5.545177444479562f;     // 8 ln 2
    const float *bias_h = a.bias + (long)h * (a.d_max + 1);
    const int W = a.window, Dm = a.d_max, T = key_end;
    float m_ref = -INFINITY, l = 0.f;
    const int o_rd = 127 - u, sh = o_rd & 3;  // this row's start in the staged diagonal
    // an item started after an abort waits on nothing: its barriers may be
    // phases behind, where a parity test could pass on an older phase; its
    // rows are written as NaN (warp-uniform, for the warp-wide TMEM loads)
    bool dead = __any_sync(0xffffffffu, *abort_flag != 0);
    int k = 0;
    for (int n = lo; n <= hi; ++n, ++k) {
        const int j0 = n * 128;
        // Stage the bias diagonal of this (query tile, key tile) pair:
        // R[q] = bias[h, clamp(top - q, 0, d_max)], q = 0..254, top = pos0 - j0 + 127,
        // as 4 copies shifted by 0..3 floats so that row u reads R[127-u+c],
        // c = 0..127, with aligned 16-byte loads.  Double-buffered by tile parity.
        const int kk = k_base + k;
        float *bb = bias_sm + (kk & 1) * kBiasBuf;
        {
            const int top = pos0 - j0 + 127;
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
        named_bar_sync(bar_id, 128);
        if (!dead) dead = !mbar_wait_warp(&s_full[t], kk & 1, abort_flag, a.status);
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
        // the keys this row may see in this tile are the columns cmin..cmax:
        // dist0 - c >= 0, dist0 - c < W (when windowed) and j0 + c < T
        const int cmax = min(min(127, dist0), T - 1 - j0);
        const int cmin = (W > 0) ? max(0, dist0 - W + 1) : 0;
        // one path per warp: a warp holding both would run both (rows of a
        // window or chunk edge that falls inside the warp)
        const bool full = __all_sync(0xffffffffu, cmin == 0 && cmax == 127);
        // logits and row max, 32 columns at a time: the 8 bias loads of a batch
        // are issued together, and 8 independent 3-input max chains run
        // alongside.  Rows of a partial tile take the same paired FMAs and then
        // mask the columns outside cmin..cmax (a compare of the unrolled column
        // index against two bounds), in a separate copy of the loop so that
        // full rows pay nothing for it.
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
        const f32x2 sc2 = pk2(scale, scale);
        auto logits = [&](auto masked) {
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float4 b4[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) b4[j] = rp[cb * 8 + j];
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
        // O rescale after P is out of registers (keeps the peak low); the P.V
        // MMA of this tile is issued only after the P signal
        if (k > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t orr[32];
                tmem_ld32(o_col + cb * 32, orr);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
                tmem_st32(o_col + cb * 32, orr);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        signal_p(t);
    }
    const bool have_o = !dead && mbar_wait_warp(&o_done[t], o_phase, abort_flag, a.status);
    if (have_o) tc_fence_after();
    epilogue(have_o, u, i, l, m_ref, o_col, abort_flag);
}

}  // namespace inkling
