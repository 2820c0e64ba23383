// attn_decode.cu — single-token decode over the paged KV cache, split-KV
// (vLLM Recipes "thinkingmachines/Inkling": Overview "Attention" bullet —
// GQA at head size 128 with a learned relative-position term added to the
// pre-softmax logits, sliding-window or full layers; 128-token cache blocks
// from the `--block-size 128` launch option; 1M-token context).
//
// Design (HBM-bound: each key/value byte is read once, 8 query heads share it):
//  * grid = num_seqs x Hkv x num_splits thread blocks; a block owns one kv head
//    of one sequence and a contiguous run of 64-key chunks of its key range.
//  * warp 4 is the producer: it reads block ids from the block table (one
//    coalesced load per 32 blocks) and issues TMA loads of 64-key halves of a
//    cache block (keys and values, 128-byte swizzled, 32 KB per stage) into a
//    3-stage mbarrier ring.
//  * warps 0-3 each take 16 keys of a chunk: S = Q K^T with mma.sync m16n8k16
//    (rows = the 8 query heads of the group, padded to 16), logits in log2
//    units plus bias, online softmax with quad shuffles, O += P V with the
//    P accumulator fragment reused as the A operand and V read by
//    ldmatrix.trans.  No tcgen05 here: at 8 flop/byte the tensor work is a
//    small fraction of the stream time and mma.sync keeps it in registers.
//  * the 4 warps merge through shared memory; with one split the block writes
//    the bf16 output, otherwise an unnormalised partial (m, l, O) that
//    decode_combine_kernel merges.
#include <mutex>

#include "common.cuh"

namespace inkling {

constexpr int kDecStages = 3;
constexpr int kDecStageBytes = 32768;  // 64 keys x 128 d x bf16, keys + values
constexpr int kDecSmem = kDecStages * kDecStageBytes + 1024 /*align*/ + 256 /*barriers*/;

struct DecodeArgs {
    const uint16_t *q;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const float *bias;
    uint16_t *out;
    float *lse;
    float *part_o;   // [S, Hq, splits, 128]
    float *part_ml;  // [S, Hq, splits, 2] (max in log2 units, sum)
    int32_t *status;
    int S, Hq, Hkv, G, max_blocks, num_blocks, window, d_max, splits;
    // sequences [0, s_whole) run unsplit (output written directly); sequences
    // [s_whole, S) in `splits` key-range pieces whose partials start at row
    // pbase = s_whole * Hq
    int s_whole;
    long pbase;
};

INK_DEV void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
INK_DEV void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
INK_DEV void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of (row r, 16-byte chunk cc of a 128-byte row) in a
// 128-byte-swizzled tile whose base is 1024-byte aligned
INK_DEV uint32_t sw128_off(int r, int cc) { return (uint32_t)(r * 128 + ((cc ^ (r & 7)) << 4)); }

__global__ void __launch_bounds__(160, 2)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = (uint64_t *)(smem + kDecStages * kDecStageBytes);
    uint64_t *empty = full + kDecStages;
    volatile int *abort_flag = (volatile int *)(empty + kDecStages);

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

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // key range of this sequence and this split, in 64-key chunks
    const int L = a.seq_lens[s];
    const bool bad_len = (L < 1 || L > a.max_blocks * 128);
    const int lo = (a.window > 0) ? max(0, L - a.window) : 0;
    int ca = 0, cb = 0;
    if (!bad_len) {
        const int c_lo = lo >> 6, c_hi = (L + 63) >> 6;
        const int per = (c_hi - c_lo + splits - 1) / splits;
        ca = min(c_hi, c_lo + split * per);
        cb = min(c_hi, ca + per);
    } else if (threadIdx.x == 0 && split == 0 && kvh == 0) {
        report_status(a.status, INKLING_STATUS_BAD_LENGTH);
    }

    if (warp == 4) {
        // ------------------------------------------------------- producer --
        int cur_batch = -1, my_id = 0, issued = 0;
        for (int c = ca; c < cb; ++c) {
            const int bi = c >> 1;
            if ((bi >> 5) != cur_batch) {
                cur_batch = bi >> 5;
                const int idx = cur_batch * 32 + lane;
                my_id = (idx < a.max_blocks) ? a.block_table[(long)s * a.max_blocks + idx] : 0;
            }
            int blk = __shfl_sync(0xffffffffu, my_id, bi & 31);
            int ok = 1;
            if (lane == 0) {
                const int k = c - ca, st = k % kDecStages;
                ok = mbar_wait(&empty[st], ((k / kDecStages) & 1) ^ 1, abort_flag, a.status);
                if (ok) {
                    if (blk < 0 || blk >= a.num_blocks) {
                        report_status(a.status, INKLING_STATUS_BAD_BLOCK);
                        blk = 0;  // keep the pipeline running on a valid block
                    }
                    const int row = (blk * a.Hkv + kvh) * 128 + (c & 1) * 64;
                    uint8_t *kb = smem + st * kDecStageBytes;
                    mbar_arrive_expect_tx(&full[st], kDecStageBytes);
                    tma_load_2d(kb, &tm_k, &full[st], 0, row);
                    tma_load_2d(kb + 8192, &tm_k, &full[st], 64, row);
                    tma_load_2d(kb + 16384, &tm_v, &full[st], 0, row);
                    tma_load_2d(kb + 24576, &tm_v, &full[st], 64, row);
                    ++issued;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
        }
        // drain: every load issued has landed before the block may exit
        if (lane == 0) {
            for (int k = max(0, issued - kDecStages); k < issued; ++k)
                mbar_wait(&full[k % kDecStages], (k / kDecStages) & 1, nullptr, a.status);
        }
    } else {
        // --------------------------------------------------------- compute --
        const int g = lane >> 2, t = lane & 3;
        const bool row_ok = g < a.G;
        const int h = kvh * a.G + (row_ok ? g : 0);
        const uint16_t *qrow = a.q + ((long)s * a.Hq + h) * 128;
        uint32_t qa[8][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qa[ks][0] = row_ok ? *(const uint32_t *)(qrow + 16 * ks + 2 * t) : 0u;
            qa[ks][2] = row_ok ? *(const uint32_t *)(qrow + 16 * ks + 8 + 2 * t) : 0u;
            qa[ks][1] = 0u;
            qa[ks][3] = 0u;
        }
        const float kLog2e = 1.4426950408889634f;
        const float c1 = kLog2e * 0.08838834764831845f;  // log2(e) / sqrt(128)
        const float *bias_h = a.bias + (long)h * (a.d_max + 1);

        float o[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float m = -INFINITY, l = 0.f;

        const uint32_t sbase = smem_u32(smem);
        for (int c = ca; c < cb; ++c) {
            const int k = c - ca, st = k % kDecStages;
            // bias for this thread's 4 keys, fetched before the wait
            float bv[2][2];
            int jj[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int j = c * 64 + warp * 16 + nt * 8 + 2 * t + e;
                    jj[nt][e] = j;
                    const int dist = L - 1 - j;
                    const bool ok = row_ok && j >= lo && j < L;
                    bv[nt][e] = ok ? __ldg(bias_h + min(dist, a.d_max)) : 0.f;
                }
            if (!mbar_wait_warp(&full[st], (k / kDecStages) & 1, abort_flag, a.status)) break;

            const uint32_t kst = sbase + st * kDecStageBytes;
            const uint32_t vst = kst + 16384;
            // S = Q K^T over this warp's 16 keys (two n-tiles of 8)
            float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            {
                const int r = warp * 16 + ((lane >> 4) & 1) * 8 + (lane & 7);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int cc = 2 * (ks & 3) + ((lane >> 3) & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kst + (ks >> 2) * 8192 + sw128_off(r, cc), b0, b1, b2, b3);
                    mma16816(sacc[0], qa[ks], b0, b1);
                    mma16816(sacc[1], qa[ks], b2, b3);
                }
            }
            // logits (log2 units), mask, online softmax
            float x[2][2];
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int j = jj[nt][e];
                    const bool ok = row_ok && j >= lo && j < L;
                    x[nt][e] = ok ? fmaf(sacc[nt][e], c1, bv[nt][e] * kLog2e) : -INFINITY;
                    mx = fmaxf(mx, x[nt][e]);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m, mx);
            const float alpha = (m == -INFINITY) ? 0.f : ex2(m - m_new);
            float p[2][2], psum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    p[nt][e] = (x[nt][e] == -INFINITY) ? 0.f : ex2(x[nt][e] - m_new);
                    psum += p[nt][e];
                }
            l = l * alpha + psum;
            m = m_new;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                o[i][0] *= alpha;
                o[i][1] *= alpha;
            }
            uint32_t pa[4];
            pa[0] = pack_bf16(p[0][0], p[0][1]);
            pa[1] = 0u;
            pa[2] = pack_bf16(p[1][0], p[1][1]);
            pa[3] = 0u;
            // O += P V over the 16 keys, 16 n-tiles of 8 head-dim columns
            {
                const int r = warp * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
                for (int mm = 0; mm < 8; ++mm) {
                    const int ch = 2 * mm + (lane >> 4);  // 16-byte chunk of d
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vst + (ch >> 3) * 8192 + sw128_off(r, ch & 7), b0, b1, b2, b3);
                    mma16816(o[2 * mm], pa, b0, b1);
                    mma16816(o[2 * mm + 1], pa, b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);

        // merge the 4 warps through shared memory (the ring is idle now)
        named_bar_sync(1, 128);
        float *red_o = (float *)smem;                  // [4][8][128]
        float *red_ml = red_o + 4 * 8 * 128;           // [4][8][2]
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            red_o[(warp * 8 + g) * 128 + i * 8 + 2 * t] = o[i][0];
            red_o[(warp * 8 + g) * 128 + i * 8 + 2 * t + 1] = o[i][1];
        }
        if (t == 0) {
            red_ml[(warp * 8 + g) * 2] = m;
            red_ml[(warp * 8 + g) * 2 + 1] = l;
        }
        named_bar_sync(1, 128);
        const int u = threadIdx.x;  // 0..127
        const int gg = u >> 4, d0 = (u & 15) * 8;
        if (gg < a.G && (bad_len || *abort_flag)) {
            // a row this call could not compute (its length is out of range, or
            // a bounded wait gave up) reads NaN, so that a caller without a
            // status word cannot take it, or another call's partial, for a
            // result; with splits the NaN partial makes the merged row NaN
            const float nanv = __int_as_float(0x7fc00000);
            const int hh = kvh * a.G + gg;
            if (splits == 1) {
                const uint32_t nb = 0x7fc07fc0u;
                *(uint4 *)(a.out + ((long)s * a.Hq + hh) * 128 + d0) = make_uint4(nb, nb, nb, nb);
                if (a.lse && (u & 15) == 0) a.lse[(long)s * a.Hq + hh] = nanv;
            } else if ((u & 15) == 0) {
                const long pi = ((long)s * a.Hq + hh - a.pbase) * splits + split;
                a.part_ml[pi * 2] = nanv;
                a.part_ml[pi * 2 + 1] = nanv;
            }
        } else if (gg < a.G) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) M = fmaxf(M, red_ml[(w * 8 + gg) * 2]);
            float f[4], Ls = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float mw = red_ml[(w * 8 + gg) * 2];
                f[w] = (mw == -INFINITY) ? 0.f : ex2(mw - M);
                Ls += f[w] * red_ml[(w * 8 + gg) * 2 + 1];
            }
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) v = fmaf(f[w], red_o[(w * 8 + gg) * 128 + d0 + e], v);
                acc[e] = v;
            }
            const int hh = kvh * a.G + gg;
            if (splits == 1) {
                const float inv = (Ls > 0.f) ? 1.f / Ls : 0.f;
                uint4 pk;
                pk.x = pack_bf16(acc[0] * inv, acc[1] * inv);
                pk.y = pack_bf16(acc[2] * inv, acc[3] * inv);
                pk.z = pack_bf16(acc[4] * inv, acc[5] * inv);
                pk.w = pack_bf16(acc[6] * inv, acc[7] * inv);
                *(uint4 *)(a.out + ((long)s * a.Hq + hh) * 128 + d0) = pk;
                if (a.lse && (u & 15) == 0)
                    a.lse[(long)s * a.Hq + hh] =
                        (Ls > 0.f) ? (M + __log2f(Ls)) * 0.6931471805599453f : -INFINITY;
            } else {
                const long pi = ((long)s * a.Hq + hh - a.pbase) * splits + split;
                float4 *po = (float4 *)(a.part_o + pi * 128 + d0);
                po[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                po[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
                if ((u & 15) == 0) {
                    a.part_ml[pi * 2] = M;
                    a.part_ml[pi * 2 + 1] = Ls;
                }
            }
        }
    }
    __syncthreads();
}

// Log-sum-exp merge of the splits of each (sequence, token, query head) row.
// A block of 8 warps merges 8 / WPR rows, WPR warps per row: warp w of a row
// takes every WPR-th split (lane l holds dims 4l..4l+3) with four splits'
// loads in flight, and the row's warps meet in shared memory in a fixed
// order.  WPR grows with the split count (1 below 8 splits, 8 from 32 on).  A
// single warp per row walking 148 splits in turn was latency-bound: 45 us for
// the 64 rows of a 1M-token batch-1 decode, 6% of that step (0.710 -> 0.682
// ms with 8 warps per row).
constexpr int kCombWarps = 8;

template <int WPR>
__global__ void __launch_bounds__(kCombWarps * 32)
decode_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml,
                      uint16_t *__restrict__ out, float *__restrict__ lse, long rows, int splits) {
    __shared__ float s_m[kCombWarps];
    __shared__ float s_ls[kCombWarps];
    __shared__ float4 s_acc[kCombWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = warp % WPR, w0 = warp - sub;  // this row's first warp
    const long pair = (long)blockIdx.x * (kCombWarps / WPR) + warp / WPR;
    const bool live = pair < rows;
    const float *ml = part_ml + (live ? pair : 0) * splits * 2;
    float M = -INFINITY;
    if (live)
        for (int sp = sub * 32 + lane; sp < splits; sp += WPR * 32) M = fmaxf(M, ml[sp * 2]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (WPR > 1) {
        if (lane == 0) s_m[warp] = M;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < WPR; ++w) M = fmaxf(M, s_m[w0 + w]);
    }
    float Ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 *po = (const float4 *)(part_o + (live ? pair : 0) * splits * 128) + lane;
    if (live) {
#pragma unroll 4
        for (int sp = sub; sp < splits; sp += WPR) {
            const float msp = ml[sp * 2];
            const float lsp = ml[sp * 2 + 1];
            const float4 v = po[sp * 32];
            // an empty split (no key in range) carries m = -inf and takes no
            // weight; a NaN partial passes into Ls and the output
            if (msp != -INFINITY) {
                const float f = ex2(msp - M);
                Ls = fmaf(f, lsp, Ls);
                acc.x = fmaf(f, v.x, acc.x);
                acc.y = fmaf(f, v.y, acc.y);
                acc.z = fmaf(f, v.z, acc.z);
                acc.w = fmaf(f, v.w, acc.w);
            }
        }
    }
    if (WPR > 1) {
        s_acc[warp][lane] = acc;
        if (lane == 0) s_ls[warp] = Ls;
        __syncthreads();
        if (sub != 0) return;
        acc = s_acc[w0][lane];
        Ls = s_ls[w0];
#pragma unroll
        for (int w = 1; w < WPR; ++w) {
            const float4 b = s_acc[w0 + w][lane];
            acc.x += b.x;
            acc.y += b.y;
            acc.z += b.z;
            acc.w += b.w;
            Ls += s_ls[w0 + w];
        }
    }
    if (!live) return;
    // a NaN partial makes Ls, the output and the lse NaN
    const float inv = (Ls > 0.f) ? 1.f / Ls : 0.f;
    uint2 pk;
    pk.x = pack_bf16(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16(acc.z * inv, acc.w * inv);
    *(uint2 *)(out + pair * 128 + lane * 4) = pk;
    if (lse && lane == 0)
        lse[pair] = (Ls > 0.f) ? (M + __log2f(Ls)) * 0.6931471805599453f
                               : (Ls == 0.f ? -INFINITY : Ls);
}

template <int WPR>
static cudaError_t launch_combine_wpr(const float *part_o, const float *part_ml, uint16_t *out,
                                      float *lse, long rows, int splits, cudaStream_t stream) {
    const long per = kCombWarps / WPR;
    decode_combine_kernel<WPR><<<(unsigned)((rows + per - 1) / per), kCombWarps * 32, 0, stream>>>(
        part_o, part_ml, out, lse, rows, splits);
    return cudaGetLastError();
}

cudaError_t launch_decode_combine(const float *part_o, const float *part_ml, uint16_t *out, float *lse,
                                  long rows, int splits, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    if (splits >= 32) return launch_combine_wpr<8>(part_o, part_ml, out, lse, rows, splits, stream);
    if (splits >= 16) return launch_combine_wpr<4>(part_o, part_ml, out, lse, rows, splits, stream);
    if (splits >= 8) return launch_combine_wpr<2>(part_o, part_ml, out, lse, rows, splits, stream);
    return launch_combine_wpr<1>(part_o, part_ml, out, lse, rows, splits, stream);
}

// s_whole: sequences [0, s_whole) run unsplit, the rest in `splits` pieces
// (s_whole == num_seqs: no partials; 0: every sequence split).
cudaError_t launch_attn_decode(const inkling_decode_params &p, int splits, int s_whole,
                               void *workspace, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                               cudaStream_t stream) {
    DecodeArgs a;
    a.q = (const uint16_t *)p.q;
    a.block_table = p.block_table;
    a.seq_lens = p.seq_lens;
    a.bias = p.bias;
    a.out = (uint16_t *)p.out;
    a.lse = p.lse;
    a.part_o = (float *)workspace;
    a.status = p.status;
    a.S = p.num_seqs;
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
    a.pbase = (long)s_whole * p.num_q_heads;
    const long rows_part = (long)(p.num_seqs - s_whole) * p.num_q_heads;
    a.part_ml = rows_part > 0 ? (float *)workspace + rows_part * splits * 128 : nullptr;
    const long grid = (long)s_whole * p.num_kv_heads +
                      (long)(p.num_seqs - s_whole) * p.num_kv_heads * splits;
    if (grid == 0) return cudaSuccess;
    cudaError_t e0 = cudaFuncSetAttribute(decode_split_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    if (e0 != cudaSuccess) return e0;
    decode_split_kernel<<<(unsigned)grid, 160, kDecSmem, stream>>>(tm_k, tm_v, a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || rows_part == 0) return e;
    return launch_decode_combine(a.part_o, a.part_ml, a.out + a.pbase * 128,
                                 a.lse ? a.lse + a.pbase : nullptr, rows_part, splits, stream);
}

// ---------------------------------------------------------------------------
// Split-KV partials in a buffer the library owns, for callers that cannot
// allocate device memory themselves (see inkling_attn_decode_static).  The
// array is part of this module: every device that loads the library holds
// kDecodeStaticScratchBytes of it until the process exits.  Host code never
// dereferences the symbol; it asks the runtime for the device address (with
// that device current) and hands that address to the kernels.  The address
// is kept per device together with the unique id of the CUDA context it was
// resolved in, and resolved again when the current context is another one
// (after cudaDeviceReset, or under a context the caller made current).
constexpr size_t kDecodeStaticScratchBytes = (size_t)8 << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeStaticScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// unique id of the current CUDA context; false when no context is current or
// the driver does not provide the entry points
static bool current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = (CtxGetCurrentFn)p;
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (CtxGetIdFn)p;
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

cudaError_t decode_static_scratch(void **ptr, size_t *bytes) {
    static std::mutex mu;
    static void *addr[64] = {nullptr};
    static unsigned long long ctx_of[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(mu);
    if (have_id && addr[dev] != nullptr && ctx_of[dev] == id) {
        *ptr = addr[dev];
        *bytes = kDecodeStaticScratchBytes;
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    // the runtime has made its context current if none was
    if (!have_id) have_id = current_context_id(&id);
    addr[dev] = have_id ? p : nullptr;  // without an id, resolve on every call
    ctx_of[dev] = id;
    *ptr = p;
    *bytes = kDecodeStaticScratchBytes;
    return cudaSuccess;
}

}  // namespace inkling
