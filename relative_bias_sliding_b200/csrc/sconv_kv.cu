// sconv_kv.cu — decode-side sconv append (vLLM Recipes "thinkingmachines/
// Inkling", Overview, "Short convolution": window-4 sconv on keys and values,
// its state managed like the KV cache of a sliding-window layer).  The same
// call appends one decode token, a few draft tokens or a whole prefill chunk.
#include "common.cuh"

namespace inkling {

// One thread owns 8 consecutive channels of one sequence's keys or values and
// a run of up to kRun consecutive new tokens: it reads the 3 raw tokens before
// its run (from the state for the first run, from the new tokens otherwise),
// convolves each token of the run and writes the bf16 result to the token's
// slot in the paged cache (block_table[s, pos/128], slot pos%128).  The thread
// of the first run also writes the new state, the last 3 raw tokens of
// (old state, new tokens), after it has read the old one; no other thread
// touches the state.  Memory-bound: 16-byte loads and stores, one pass, 8
// tokens' loads in flight per thread.
//
// The two-pass prefill runs the same kernel on a whole prompt with three
// internal modes that the public append never takes: zero_hist (zero raw
// history before the first new token, the old state not read; a NULL state is
// then not written either), seq_lens NULL (every length is n_new) and
// block_table NULL (scratch blocks: sequence s owns blocks s*max_blocks ... in
// order, and the slots past its end in its last block are zeroed).
constexpr int kRun = 32;

__global__ void __launch_bounds__(128)
sconv_kv_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                const float4 *__restrict__ w_k, const float4 *__restrict__ w_v,
                uint4 *__restrict__ k_state, uint4 *__restrict__ v_state,
                uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                const int32_t *__restrict__ block_table, const int32_t *__restrict__ seq_lens,
                int32_t *status, int S, int n_new, int Hkv, int max_blocks, int num_blocks,
                bool zero_hist) {
    const int chunks = Hkv * 16;  // 8-channel chunks per token (C = Hkv*128)
    const int runs = (n_new + kRun - 1) / kRun;
    const long gid = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long)S * 2 * chunks * runs) return;
    const int chunk = (int)(gid % chunks);
    const int which = (int)((gid / chunks) & 1);  // 0 = keys, 1 = values
    const int run = (int)((gid / (2 * chunks)) % runs);
    const int s = (int)(gid / (2L * chunks * runs));

    const uint4 *xin = which ? v_new : k_new;
    const float4 *wt = which ? w_v : w_k;
    uint4 *state = which ? v_state : k_state;
    uint4 *cache = which ? v_cache : k_cache;

    const int L = seq_lens ? seq_lens[s] : n_new;
    if (L < n_new || L > max_blocks * 128) {
        report_status(status, INKLING_STATUS_BAD_LENGTH);
        return;
    }
    float w[8][4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 t = wt[chunk * 8 + e];
        w[e][0] = t.x; w[e][1] = t.y; w[e][2] = t.z; w[e][3] = t.w;
    }
    // raw history: state [S, 3, C] (oldest first) or new tokens [S, n_new, C]
    const int t0 = run * kRun, t1 = min(n_new, t0 + kRun);
    auto new_tok = [&](int t) { return xin[((long)s * n_new + t) * chunks + chunk]; };
    uint4 r3, r2, r1;
    if (run == 0 && zero_hist) {
        r3 = r2 = r1 = make_uint4(0u, 0u, 0u, 0u);
    } else if (run == 0) {
        r3 = state[((long)s * 3 + 0) * chunks + chunk];
        r2 = state[((long)s * 3 + 1) * chunks + chunk];
        r1 = state[((long)s * 3 + 2) * chunks + chunk];
    } else {
        r3 = new_tok(t0 - 3);
        r2 = new_tok(t0 - 2);
        r1 = new_tok(t0 - 1);
    }
    const uint4 s3 = r3, s2 = r2, s1 = r1;  // the old state, for the first run
    float h3[8], h2[8], h1[8];
    unpack8(r3, h3);
    unpack8(r2, h2);
    unpack8(r1, h1);

    const int kvh = chunk >> 4, e16 = chunk & 15;  // kv head, 16-byte column in the row
    // the cache blocks this run writes: a run of kRun (32) tokens spans at
    // most two 128-token blocks, whose ids are read once
    const int pfirst = L - n_new + t0;
    const int q0 = pfirst >> 7, q1 = (L - n_new + t1 - 1) >> 7;
    auto block_of = [&](int q) {
        return block_table ? block_table[(long)s * max_blocks + q] : s * max_blocks + q;
    };
    const int blk0 = block_of(q0);
    const int blk1 = (q1 != q0) ? block_of(q1) : blk0;
    const bool bad0 = blk0 < 0 || blk0 >= num_blocks, bad1 = blk1 < 0 || blk1 >= num_blocks;
    if (bad0 || bad1) report_status(status, INKLING_STATUS_BAD_BLOCK);
    // 8 tokens' loads in flight, then their convolutions in order
    for (int tb = t0; tb < t1; tb += 8) {
        uint4 raw[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            raw[j] = (tb + j < t1) ? new_tok(tb + j) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (tb + j >= t1) break;
            float x[8];
            unpack8(raw[j], x);
            const uint4 y = sconv8(w, h3, h2, h1, x);
            const int pos = pfirst + (tb - t0) + j;
            const bool second = (pos >> 7) != q0;
            if (!(second ? bad1 : bad0))
                cache[(((long)(second ? blk1 : blk0) * Hkv + kvh) * 128 + (pos & 127)) * 16 + e16] = y;
#pragma unroll
            for (int e = 0; e < 8; ++e) { h3[e] = h2[e]; h2[e] = h1[e]; h1[e] = x[e]; }
        }
    }
    if (!block_table && run == runs - 1 && (L & 127)) {
        // scratch blocks: zero the slots past the sequence end in its last
        // block (the attention reads whole blocks and multiplies those slots
        // by zero probabilities, which stale NaN or Inf bits would survive)
        const long blk = (long)s * max_blocks + ((L - 1) >> 7);
        uint4 *dst = cache + ((blk * Hkv + kvh) * 128) * 16 + e16;
        for (int slot = L & 127; slot < 128; ++slot) dst[(long)slot * 16] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (run == 0 && state) {
        // new state: the last 3 of (old state s3 s2 s1, new tokens 0..n_new-1)
        uint4 ns[3];
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            const int idx = n_new + m;  // index in the concatenated stream of 3 + n_new
            ns[m] = idx >= 3 ? new_tok(idx - 3) : (idx == 0 ? s3 : (idx == 1 ? s2 : s1));
        }
#pragma unroll
        for (int m = 0; m < 3; ++m) state[((long)s * 3 + m) * chunks + chunk] = ns[m];
    }
}

cudaError_t launch_sconv_kv(const inkling_sconv_params &p, cudaStream_t stream, bool zero_hist) {
    const long runs = (p.n_new + kRun - 1) / kRun;
    const long threads = (long)p.num_seqs * 2 * p.num_kv_heads * 16 * runs;
    if (threads == 0) return cudaSuccess;
    const int block = 128;
    const long grid = (threads + block - 1) / block;
    sconv_kv_kernel<<<(unsigned)grid, block, 0, stream>>>(
        (const uint4 *)p.k_new, (const uint4 *)p.v_new, (const float4 *)p.w_k,
        (const float4 *)p.w_v, (uint4 *)p.k_state, (uint4 *)p.v_state, (uint4 *)p.k_cache,
        (uint4 *)p.v_cache, p.block_table, p.seq_lens, p.status, p.num_seqs, p.n_new,
        p.num_kv_heads, p.max_blocks, p.num_blocks, zero_hist);
    return cudaGetLastError();
}

// Self-test of the bounded waits every kernel of this library uses: one thread
// waits on an mbarrier phase that nothing will complete, with a short limit;
// the wait gives up, reports INKLING_STATUS_TIMEOUT and the kernel returns.
__global__ void wait_timeout_probe_kernel(int32_t *status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    __syncthreads();
}

cudaError_t launch_wait_timeout_probe(int32_t *status, uint32_t limit_us, cudaStream_t stream) {
    wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(status, (uint64_t)limit_us * 1000ull);
    return cudaGetLastError();
}

}  // namespace inkling
