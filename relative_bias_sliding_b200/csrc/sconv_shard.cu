// sconv_shard.cu — the output short convolution sharded over channels across
// tensor-parallel ranks, fused with its reduce-scatter and all-gather over
// peer memory (vLLM Recipes "thinkingmachines/Inkling": Overview, "Short
// convolution" — the sconv is sharded across the channel dimension with a
// reduce-scatter / all-gather so that neither its cache nor its compute is
// replicated on every rank; Performance — sconv-aware TP sharding, each rank
// storing only its channel shard of the sconv cache).
//
// Under tensor parallelism the input of the output sconv arrives as one
// partial sum per rank (the output of a row-parallel projection).  Rank r
// owns channels [r*Cs, (r+1)*Cs), Cs = C / n_ranks.  One launch on rank r:
//   1. reduce-scatter: for its channels, sum the n_ranks partials (plain
//      16-byte loads, from peers over NVLink), in fp32 in rank order, and
//      round once to bf16;
//   2. the causal window-4 sconv of that sum, with the 3 rows before t = 0
//      from rank r's state shard [B, 3, Cs] (the summed raw rows), the same
//      fp32 FMA order and one bf16 rounding as inkling_sconv_out;
//   3. all-gather: store the result into the output buffer of every rank
//      (plain 16-byte stores, to peers over NVLink).
// So the transfer overlaps the arithmetic row by row and no intermediate
// buffer exists.  No TMA and no multicast are used.
//
// One thread owns 8 consecutive channels of one sequence and a run of up to
// 64 tokens (its 3 history rows are summed again from the partials, or come
// from the state in the first run); the first run's thread writes the new
// state after reading the old one.
#include "common.cuh"

namespace inkling {

constexpr int kShardRun = 64;
constexpr int kMaxRanks = INKLING_SHARD_MAX_RANKS;

struct ShardArgs {
    const uint4 *x[kMaxRanks];  // partial sums [B, T, C] of every rank
    uint4 *y[kMaxRanks];        // outputs [B, T, C] of every rank
    const float4 *w;            // [C, 4] taps
    uint4 *state;               // [B, 3, Cs] this rank's state shard, or null
    int n, B, T, chunks, cs_chunks, c0_chunk;
};

// the reduce-scatter of one 16-byte row chunk: fp32 sum over ranks in rank
// order, one bf16 rounding; returns the 8 summed raw values (as bf16 bits)
INK_DEV uint4 sum_parts(const ShardArgs &a, long off) {
    float acc[8];
    unpack8(a.x[0][off], acc);
#pragma unroll
    for (int r = 1; r < kMaxRanks; ++r) {
        if (r >= a.n) break;
        float v[8];
        unpack8(a.x[r][off], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += v[e];
    }
    uint4 o;
    o.x = pack_bf16(acc[0], acc[1]);
    o.y = pack_bf16(acc[2], acc[3]);
    o.z = pack_bf16(acc[4], acc[5]);
    o.w = pack_bf16(acc[6], acc[7]);
    return o;
}

__global__ void __launch_bounds__(128)
sconv_out_sharded_kernel(const ShardArgs a) {
    const int runs = (a.T + kShardRun - 1) / kShardRun;
    const long gid = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long)a.B * a.cs_chunks * runs) return;
    const int lc = (int)(gid % a.cs_chunks);  // chunk within the shard
    const int run = (int)((gid / a.cs_chunks) % runs);
    const int b = (int)(gid / ((long)a.cs_chunks * runs));
    const int chunk = a.c0_chunk + lc;         // chunk within all C channels

    float wt[8][4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 t = a.w[chunk * 8 + e];
        wt[e][0] = t.x; wt[e][1] = t.y; wt[e][2] = t.z; wt[e][3] = t.w;
    }
    auto off = [&](int t) { return ((long)b * a.T + t) * a.chunks + chunk; };
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const int t0 = run * kShardRun, t1 = min(a.T, t0 + kShardRun);
    uint4 r3, r2, r1;
    if (run == 0) {
        r3 = a.state ? a.state[((long)b * 3 + 0) * a.cs_chunks + lc] : zero;
        r2 = a.state ? a.state[((long)b * 3 + 1) * a.cs_chunks + lc] : zero;
        r1 = a.state ? a.state[((long)b * 3 + 2) * a.cs_chunks + lc] : zero;
    } else {
        r3 = sum_parts(a, off(t0 - 3));
        r2 = sum_parts(a, off(t0 - 2));
        r1 = sum_parts(a, off(t0 - 1));
    }
    const uint4 s3 = r3, s2 = r2, s1 = r1;
    float h3[8], h2[8], h1[8];
    unpack8(r3, h3);
    unpack8(r2, h2);
    unpack8(r1, h1);
    uint4 last[3] = {s3, s2, s1};  // the last 3 summed raw rows seen
    for (int t = t0; t < t1; ++t) {
        const long o = off(t);
        const uint4 xs = sum_parts(a, o);
        float xv[8];
        unpack8(xs, xv);
        const uint4 yv = sconv8(wt, h3, h2, h1, xv);
#pragma unroll
        for (int r = 0; r < kMaxRanks; ++r)
            if (r < a.n) a.y[r][o] = yv;
#pragma unroll
        for (int e = 0; e < 8; ++e) { h3[e] = h2[e]; h2[e] = h1[e]; h1[e] = xv[e]; }
        last[0] = last[1];
        last[1] = last[2];
        last[2] = xs;
    }
    if (run == 0 && a.state) {
        // new state: the last 3 summed raw rows of (old state, x); the first
        // run holds them when T <= 64, else they are summed again
        uint4 ns[3];
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            const int t = a.T - 3 + m;
            ns[m] = (a.T <= kShardRun) ? last[m] : sum_parts(a, off(t));
        }
#pragma unroll
        for (int m = 0; m < 3; ++m) a.state[((long)b * 3 + m) * a.cs_chunks + lc] = ns[m];
    }
}

cudaError_t launch_sconv_out_sharded(const inkling_sconv_out_sharded_params &p,
                                     cudaStream_t stream) {
    ShardArgs a = {};
    for (int r = 0; r < p.n_ranks; ++r) {
        a.x[r] = (const uint4 *)p.x_parts[r];
        a.y[r] = (uint4 *)p.y_parts[r];
    }
    a.w = (const float4 *)p.w;
    a.state = (uint4 *)p.state;
    a.n = p.n_ranks;
    a.B = p.batch;
    a.T = p.seq_len;
    a.chunks = p.channels / 8;
    a.cs_chunks = a.chunks / p.n_ranks;
    a.c0_chunk = p.rank * a.cs_chunks;
    const long runs = (p.seq_len + kShardRun - 1) / kShardRun;
    const long threads = (long)p.batch * a.cs_chunks * runs;
    if (threads == 0) return cudaSuccess;
    sconv_out_sharded_kernel<<<(unsigned)((threads + 127) / 128), 128, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace inkling
