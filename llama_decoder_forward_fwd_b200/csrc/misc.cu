// Small kernels at the ends of a pass: the embedding lookup that starts the
// residual stream, the hidden-state output of the layer-stack-only path, and the
// RoPE cos/sin tables built once at model creation.
#include "common.cuh"
#include "kernels.cuh"

namespace lfw {

constexpr int EMB_THREADS = 256;

// h[m] = E[tok[m]] ("Building llama3 from scratch": the embedding layer maps each
// token id to its row of tok_embeddings) or the given hidden state, plus the first
// layer's RMSNorm inputs: hw[m] = h[m] * w and ss[m] = sum h[m]^2. Each thread
// moves 8 consecutive elements per step with 16-byte accesses, so a row costs one
// memory round trip.
template <typename WT>
__global__ void __launch_bounds__(EMB_THREADS) embed_kernel(const EmbedArgs a) {
    __shared__ float red[EMB_THREADS / 32];
    const int m = blockIdx.x;
    pdl_trigger();
    pdl_wait();
    const WT* wn = reinterpret_cast<const WT*>(a.wnorm);
    WT* hw = reinterpret_cast<WT*>(a.hw) + (long long)m * a.D;
    WT* hw_lo = a.hw_lo ? reinterpret_cast<WT*>(a.hw_lo) + (long long)m * a.D : nullptr;
    float* h = a.h + (long long)m * a.D;
    const WT* src = nullptr;
    const float* hsrc = nullptr;
    if (a.h_in) {
        hsrc = a.h_in + (long long)m * a.D;
    } else {
        int tok = a.tok[m];
        if (threadIdx.x == 0) LFW_CHECK(tok >= 0 && tok < a.vocab, a.err, BC_TOKEN);
        tok = tok < 0 ? 0 : (tok >= a.vocab ? a.vocab - 1 : tok);  // never read outside the table
        src = reinterpret_cast<const WT*>(a.E) + (long long)tok * a.D;
    }
    float ss = 0.f;
    for (int i = threadIdx.x * 8; i < a.D; i += EMB_THREADS * 8) {  // D % 8 == 0
        float v[8], w[8];
        if (hsrc) {
            const float4 x0 = *reinterpret_cast<const float4*>(hsrc + i);
            const float4 x1 = *reinterpret_cast<const float4*>(hsrc + i + 4);
            v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w; v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = to_f<WT>(src[i + j]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = to_f<WT>(wn[i + j]);
        reinterpret_cast<float4*>(h + i)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(h + i)[1] = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const WT xw = from_f<WT>(v[j] * w[j]);
            hw[i + j] = xw;
            if (hw_lo) hw_lo[i + j] = from_f<WT>(v[j] * w[j] - to_f<WT>(xw));
            ss += v[j] * v[j];
        }
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < EMB_THREADS / 32; ++w) t += red[w];
        a.ss[m] = t;
    }
}

cudaError_t launch_embed(const EmbedArgs& a, bool bf16, cudaStream_t s, bool pdl) {
    if (bf16) return launch_k(embed_kernel<__nv_bfloat16>, dim3(a.M), EMB_THREADS, 0, s, pdl, a);
    return launch_k(embed_kernel<float>, dim3(a.M), EMB_THREADS, 0, s, pdl, a);
}

__global__ void finish_hidden_kernel(const float* h, float* h_out, long long n, int32_t* seq_len, int B,
                                     int advance) {
    pdl_trigger();
    pdl_wait();
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        h_out[i] = h[i];
    if (blockIdx.x == 0 && threadIdx.x < B) seq_len[threadIdx.x] += advance;
}

cudaError_t launch_finish_hidden(const float* h, float* h_out, long long n, int32_t* seq_len, int B, int advance,
                                 cudaStream_t s, bool pdl) {
    long long blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    if (blocks < 1) blocks = 1;
    return launch_k(finish_hidden_kernel, dim3((unsigned)blocks), dim3(256), 0, s, pdl, h, h_out, n, seq_len, B,
                    advance);
}

// cos/sin of p * theta^(-2i/head_dim) for p < n_pos, i < head_dim/2 (llama3.np
// page, "RoPE #1": positions times frequencies, then cos and sin), evaluated in
// double precision and stored as fp32.
__global__ void rope_table_kernel(float* cosv, float* sinv, int n_pos, int half, double theta, int head_dim) {
    const long long n = (long long)n_pos * half;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const int p = (int)(idx / half), i = (int)(idx % half);
        const double freq = pow(theta, -2.0 * i / head_dim);
        double sn, cs;
        sincos((double)p * freq, &sn, &cs);
        cosv[idx] = (float)cs;
        sinv[idx] = (float)sn;
    }
}

cudaError_t launch_rope_tables(float* cosv, float* sinv, int n_pos, int half, double theta, int head_dim,
                               cudaStream_t s) {
    rope_table_kernel<<<256, 256, 0, s>>>(cosv, sinv, n_pos, half, theta, head_dim);
    return cudaGetLastError();
}

// ---- wait probe: the bounded-wait path run on purpose ------------------
// An mbarrier armed for 16 bytes that no copy delivers: the bounded wait gives
// up after limit_ns, records DERR_PROBE_WAIT and returns. Nothing is left in
// flight (no copy was issued), so the CTA retires normally.
__global__ void wait_probe_mbar_kernel(uint64_t limit_ns, uint32_t* err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar, 16);
        mbar_wait(&bar, 0, err, DERR_PROBE_WAIT, limit_ns);
    }
}
// A grid barrier that is never reached: each CTA arrives once (the counter
// starts at zero), but barrier index 1 waits for 2 * gridDim.x arrivals. The
// first CTA to give up after limit_ns records DERR_PROBE_WAIT; the other sees the
// error word and leaves too.
__global__ void wait_probe_grid_kernel(uint64_t limit_ns, uint32_t* err, unsigned* counter) {
    grid_barrier(counter, 1, blockDim.x, err, DERR_PROBE_WAIT, limit_ns);
}

cudaError_t launch_wait_probe(int which, uint64_t limit_ns, uint32_t* err, unsigned* counter, cudaStream_t s) {
    if (which == 0) {
        wait_probe_mbar_kernel<<<1, 32, 0, s>>>(limit_ns, err);
        return cudaGetLastError();
    }
    if (which != 1 || !counter) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(counter, 0, 4, s);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // both CTAs resident: the wait is the only thing that stops them
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, wait_probe_grid_kernel, limit_ns, err, counter);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(counter, 0, 4, s);
}

}  // namespace lfw
