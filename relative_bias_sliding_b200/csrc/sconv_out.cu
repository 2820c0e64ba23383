// sconv_out.cu — the window-4 short convolution on the attention output
// (vLLM Recipes "thinkingmachines/Inkling", Overview, "Short convolution":
// each layer applies four window-4 sconv modules, on attention keys, values,
// output and MoE output).  y[b,t,c] = sum_k w[c,k] x[b,t-k,c] over the
// channels of the attention output (C = Hq*128), with the 3 raw rows before
// t = 0 taken from a rolling state (or zero), one bf16 rounding.
//
// One thread owns 8 consecutive channels of one sequence and a run of up to
// kOutRun (64) consecutive tokens, with 4 row loads in flight: history from the
// state (first run) or from x, 16-byte loads and stores, the same fp32 FMA
// order as the key/value sconv.
// The first run's thread also writes the new state (the last 3 raw rows of
// (old state, x)) after reading the old one.  HBM-bound: x read once (plus 3
// history rows per run), y written once.
#include "common.cuh"

namespace inkling {

constexpr int kOutRun = 64;

__global__ void __launch_bounds__(128)
sconv_out_kernel(const uint4 *__restrict__ x, const float4 *__restrict__ w, uint4 *state,
                 uint4 *__restrict__ y, int B, int T, int chunks) {
    const int runs = (T + kOutRun - 1) / kOutRun;
    const long gid = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long)B * chunks * runs) return;
    const int chunk = (int)(gid % chunks);
    const int run = (int)((gid / chunks) % runs);
    const int b = (int)(gid / ((long)chunks * runs));

    float wt[8][4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 t = w[chunk * 8 + e];
        wt[e][0] = t.x; wt[e][1] = t.y; wt[e][2] = t.z; wt[e][3] = t.w;
    }
    auto row = [&](int t) { return x[((long)b * T + t) * chunks + chunk]; };
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const int t0 = run * kOutRun, t1 = min(T, t0 + kOutRun);
    uint4 r3, r2, r1;
    if (run == 0) {
        r3 = state ? state[((long)b * 3 + 0) * chunks + chunk] : zero;
        r2 = state ? state[((long)b * 3 + 1) * chunks + chunk] : zero;
        r1 = state ? state[((long)b * 3 + 2) * chunks + chunk] : zero;
    } else {
        r3 = row(t0 - 3);
        r2 = row(t0 - 2);
        r1 = row(t0 - 1);
    }
    const uint4 s3 = r3, s2 = r2, s1 = r1;
    float h3[8], h2[8], h1[8];
    unpack8(r3, h3);
    unpack8(r2, h2);
    unpack8(r1, h1);
#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
        float xv[8];
        unpack8(row(t), xv);
        y[((long)b * T + t) * chunks + chunk] = sconv8(wt, h3, h2, h1, xv);
#pragma unroll
        for (int e = 0; e < 8; ++e) { h3[e] = h2[e]; h2[e] = h1[e]; h1[e] = xv[e]; }
    }
    if (run == 0 && state) {
        uint4 ns[3];
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            const int idx = T + m;  // index in the stream (old state: 0..2, x: 3..T+2)
            ns[m] = idx >= 3 ? row(idx - 3) : (idx == 0 ? s3 : (idx == 1 ? s2 : s1));
        }
#pragma unroll
        for (int m = 0; m < 3; ++m) state[((long)b * 3 + m) * chunks + chunk] = ns[m];
    }
}

cudaError_t launch_sconv_out(const inkling_sconv_out_params &p, cudaStream_t stream) {
    const int chunks = p.channels / 8;
    const long runs = (p.seq_len + kOutRun - 1) / kOutRun;
    const long threads = (long)p.batch * chunks * runs;
    if (threads == 0) return cudaSuccess;
    const long grid = (threads + 127) / 128;
    sconv_out_kernel<<<(unsigned)grid, 128, 0, stream>>>(
        (const uint4 *)p.x, (const float4 *)p.w, (uint4 *)p.state, (uint4 *)p.y, p.batch,
        p.seq_len, chunks);
    return cudaGetLastError();
}

}  // namespace inkling
