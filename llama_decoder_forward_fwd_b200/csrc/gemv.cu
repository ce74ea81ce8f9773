// Decode projections: y[m][n] = sum_k x[m][k] W[n][k] for M <= 16 token rows,
// streaming the weight matrix from HBM once ("KV cache" on the llama3.np page:
// in the decode phase only the newest token is projected, so every projection
// is a matrix-vector product bound by the weight bytes).
//
// bf16 kernel. A warp owns a tile of 16 weight rows and a slice of K and runs
// mma.sync m16n8k16 with the weights as the A operand (16 rows) and the token
// rows as B (8 or 16 columns). Lane (g = lane/4, t = lane%4) loads 16
// contiguous bf16 of rows g and g+8 at k0 + 16t (two 16-byte loads per row per
// 64-wide k block). Because a dot product does not depend on the order of k,
// the fragment's logical k index is mapped onto these physical offsets: for the
// j-th MMA of the block, lane t's logical k pairs (2t, 2t+1) and (2t+8, 2t+9)
// take physical k0 + 16t + 4j + {0,1} and {2,3}. The B operand (x) is loaded
// with the same map, so the product is unchanged while every weight load is a
// full 16-byte vector. KSPLIT warps share a tile (split K inside the CTA) and
// combine their fragments in shared memory.
#include "epilogue.cuh"

#include <float.h>
#include <limits.h>

namespace lfw {

constexpr int GEMV_THREADS = 256;

template <int EPI>
DEVI int gemv_tile_rows() { return EPI == EPI_SWIGLU ? 8 : 16; }

int gemv_num_tiles(int kind, int N) { return kind == EPI_SWIGLU ? (N + 7) / 8 : (N + 15) / 16; }

DEVI uint32_t w_of(const uint4& a, const uint4& b, int i) {
    const uint4& v = i < 4 ? a : b;
    const int j = i & 3;
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Per-row RMSNorm scale of the M token rows into smem (warp per row, lanes over parts).
DEVI void compute_rinv(const NormIn& n, int M, int m0, float* rinv_s) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int m = warp; m < M; m += GEMV_THREADS / 32) {
        float s = 0.f;
        if (n.ss != nullptr) {
            const float* p = n.ss + n.row0 + (long long)(m0 + m) * n.row_step;
            for (int i = lane; i < n.nparts; i += 32) s += p[(long long)i * n.ld];
            s = warp_sum(s);
        }
        if (lane == 0) rinv_s[m] = n.ss ? rsqrtf(s * n.inv_dim + n.eps) : 1.f;
    }
}

// Last CTA of the grid reduces the per-tile argmax partials: next[m] and the
// cache-length advance ("Predicción de tokens").
DEVI void logits_finish(const Epi& e, int M, int ntiles, int* last_s) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(e.am_counter, 1u);
        *last_s = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!*last_s) return;
    __threadfence();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int m = warp; m < M; m += GEMV_THREADS / 32) {
        float bv = -FLT_MAX;
        int bi = INT_MAX;
        for (int t = lane; t < ntiles; t += 32)
            am_merge(bv, bi, __ldcg(e.am_val + (long long)t * M + m), __ldcg(e.am_idx + (long long)t * M + m));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            am_merge(bv, bi, ov, oi);
        }
        if (lane == 0) {
            e.next_tok[m] = bi;
            if (e.seq_len) e.seq_len[m] += e.advance;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) *e.am_counter = 0u;
}

template <int NB, int KSPLIT, int EPI>
__global__ void __launch_bounds__(GEMV_THREADS) gemv_bf16_kernel(const GemvArgs<__nv_bfloat16> a) {
    constexpr int TPC = 8 / KSPLIT;  // 16-row tiles per CTA
    constexpr int NM = NB / 8;       // n8 MMAs per k16 step
    constexpr int U = 2;             // 64-wide k blocks in flight per warp
    __shared__ float red_s[KSPLIT > 1 ? GEMV_THREADS * 4 * NM : 1];
    __shared__ float rinv_s[16];
    __shared__ int last_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tl = warp / KSPLIT, ks = warp - tl * KSPLIT;
    const int tile = blockIdx.x * TPC + tl;
    const int g = lane >> 2, t4 = lane & 3;
    const int M = a.M, K = a.K;

    const __nv_bfloat16* wr0 = nullptr;
    const __nv_bfloat16* wr1 = nullptr;
    int lr0, lr1;
    if (EPI == EPI_SWIGLU) {
        lr0 = tile * 8 + g;
        lr1 = lr0;
        if (lr0 < a.N) {
            wr0 = a.W[0] + (size_t)lr0 * K;
            wr1 = a.W[1] + (size_t)lr0 * K;
        }
    } else if (EPI == EPI_QKV_ROPE) {
        lr0 = tile * 16 + 2 * g;
        lr1 = lr0 + 1;
        if (lr0 < a.N) {
            int s = 0, r = lr0;
            while (s < 2 && r >= a.seg_rows[s]) {
                r -= a.seg_rows[s];
                ++s;
            }
            wr0 = a.W[s] + (size_t)r * K;
            wr1 = wr0 + K;
        }
    } else {
        lr0 = tile * 16 + g;
        lr1 = lr0 + 8;
        if (lr0 < a.N) wr0 = a.W[0] + (size_t)lr0 * K;
        if (lr1 < a.N) wr1 = a.W[0] + (size_t)lr1 * K;
    }

    const int nkb = (K + 63) >> 6;
    const int per = (nkb + KSPLIT - 1) / KSPLIT;
    const int kb_beg = ks * per;
    const int kb_end = min(nkb, kb_beg + per);
    const uint4 z4 = make_uint4(0, 0, 0, 0);

    auto load_w = [&](int kb, uint4(&w)[4]) {
        const int k = kb * 64 + t4 * 16;
        const bool in0 = kb < kb_end && k < K, in1 = kb < kb_end && k + 8 < K;
        w[0] = (wr0 && in0) ? ld_stream_v4(wr0 + k) : z4;
        w[1] = (wr0 && in1) ? ld_stream_v4(wr0 + k + 8) : z4;
        w[2] = (wr1 && in0) ? ld_stream_v4(wr1 + k) : z4;
        w[3] = (wr1 && in1) ? ld_stream_v4(wr1 + k + 8) : z4;
    };

    // Weights do not depend on the previous kernel: start streaming them first.
    uint4 wc[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) load_w(kb_beg + u, wc[u]);
    pdl_trigger();
    pdl_wait();

    float c[NM][4];
#pragma unroll
    for (int n = 0; n < NM; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0.f;

    for (int kb = kb_beg; kb < kb_end; kb += U) {
        uint4 wn[U][4];
#pragma unroll
        for (int u = 0; u < U; ++u) load_w(kb + U + u, wn[u]);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = (kb + u) * 64 + t4 * 16;
            uint4 xa[NM], xb[NM];
#pragma unroll
            for (int n = 0; n < NM; ++n) {
                const int mrow = g + 8 * n;
                const bool ok = mrow < M && kb + u < kb_end;
                const __nv_bfloat16* xp = a.x + (size_t)mrow * a.ldx + k;
                xa[n] = (ok && k < K) ? *reinterpret_cast<const uint4*>(xp) : z4;
                xb[n] = (ok && k + 8 < K) ? *reinterpret_cast<const uint4*>(xp + 8) : z4;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t af[4];
                af[0] = w_of(wc[u][0], wc[u][1], 2 * j);
                af[1] = w_of(wc[u][2], wc[u][3], 2 * j);
                af[2] = w_of(wc[u][0], wc[u][1], 2 * j + 1);
                af[3] = w_of(wc[u][2], wc[u][3], 2 * j + 1);
#pragma unroll
                for (int n = 0; n < NM; ++n)
                    mma_bf16_16816(c[n], af, w_of(xa[n], xb[n], 2 * j), w_of(xa[n], xb[n], 2 * j + 1));
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int i = 0; i < 4; ++i) wc[u][i] = wn[u][i];
    }

    if (KSPLIT > 1) {
#pragma unroll
        for (int n = 0; n < NM; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) red_s[(threadIdx.x * NM + n) * 4 + i] = c[n][i];
    }
    compute_rinv(a.epi.norm, M, a.m0, rinv_s);
    __syncthreads();
    if (KSPLIT > 1 && ks == 0) {
        for (int s = 1; s < KSPLIT; ++s) {
            const int src = (tl * KSPLIT + s) * 32 + lane;
#pragma unroll
            for (int n = 0; n < NM; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) c[n][i] += red_s[(src * NM + n) * 4 + i];
        }
    }

    const Epi& e = a.epi;
    if (ks == 0) {
        float ssum[NM][2];
        float bv[NM][2];
        int bi[NM][2];
#pragma unroll
        for (int n = 0; n < NM; ++n)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int m = n * 8 + 2 * t4 + h;
                ssum[n][h] = 0.f;
                bv[n][h] = -FLT_MAX;
                bi[n][h] = INT_MAX;
                if (m >= M) continue;
                const int mg = a.m0 + m;           // token index
                const float r = rinv_s[m];
                const float v0 = c[n][h] * r;      // logical row lr0
                const float v1 = c[n][2 + h] * r;  // logical row lr1
                if (EPI == EPI_STORE_F32) {
                    if (lr0 < a.N) e.y[(size_t)mg * e.ldy + lr0] = v0;
                    if (lr1 < a.N) e.y[(size_t)mg * e.ldy + lr1] = v1;
                } else if (EPI == EPI_QKV_ROPE) {
                    if (lr0 < a.N) epi_qkv_pair<__nv_bfloat16>(e, mg, lr0, v0, v1);
                } else if (EPI == EPI_SWIGLU) {
                    if (lr0 < a.N)
                        reinterpret_cast<__nv_bfloat16*>(e.g_out)[(size_t)mg * e.F + lr0] =
                            __float2bfloat16_rn(swiglu(v0, v1));
                } else if (EPI == EPI_RESID) {
                    float s = 0.f;
                    if (lr0 < a.N) {
                        const float hn = epi_resid1<__nv_bfloat16>(e, mg, lr0, v0);
                        s += hn * hn;
                    }
                    if (lr1 < a.N) {
                        const float hn = epi_resid1<__nv_bfloat16>(e, mg, lr1, v1);
                        s += hn * hn;
                    }
                    ssum[n][h] = s;
                } else if (EPI == EPI_LOGITS) {
                    if (lr0 < a.N) {
                        if (e.logits) e.logits[(size_t)m * e.ld_logits + lr0] = v0;
                        am_merge(bv[n][h], bi[n][h], v0, lr0);
                    }
                    if (lr1 < a.N) {
                        if (e.logits) e.logits[(size_t)m * e.ld_logits + lr1] = v1;
                        am_merge(bv[n][h], bi[n][h], v1, lr1);
                    }
                }
            }
        if (EPI == EPI_RESID || EPI == EPI_LOGITS) {
            // Reduce over the 8 row groups g (lanes with equal t4).
#pragma unroll
            for (int n = 0; n < NM; ++n)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        if (EPI == EPI_RESID) {
                            ssum[n][h] += __shfl_xor_sync(0xffffffffu, ssum[n][h], o);
                        } else {
                            const float ov = __shfl_xor_sync(0xffffffffu, bv[n][h], o);
                            const int oi = __shfl_xor_sync(0xffffffffu, bi[n][h], o);
                            am_merge(bv[n][h], bi[n][h], ov, oi);
                        }
                    }
                    const int m = n * 8 + 2 * t4 + h;
                    if (g == 0 && m < M) {
                        if (EPI == EPI_RESID) {
                            e.ss_out[(size_t)tile * e.ss_out_ld + a.m0 + m] = ssum[n][h];
                        } else {
                            e.am_val[(size_t)tile * M + m] = bv[n][h];
                            e.am_idx[(size_t)tile * M + m] = bi[n][h];
                        }
                    }
                }
        }
    }
    if (EPI == EPI_LOGITS) logits_finish(e, M, gridDim.x * TPC, &last_s);
}

// fp32 kernel (CUDA cores): a warp owns a pair of logical rows, a CTA 8 pairs.
template <int EPI>
__global__ void __launch_bounds__(GEMV_THREADS) gemv_f32_kernel(const GemvArgs<float> a) {
    __shared__ float rinv_s[16];
    __shared__ float ss_s[8][16];
    __shared__ float amv_s[8][16];
    __shared__ int ami_s[8][16];
    __shared__ int last_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.x * 8 + warp;
    const int M = a.M, K = a.K;
    const float* wr0 = nullptr;
    const float* wr1 = nullptr;
    int lr0, lr1;
    if (EPI == EPI_SWIGLU) {
        lr0 = lr1 = pair;
        if (pair < a.N) {
            wr0 = a.W[0] + (size_t)pair * K;
            wr1 = a.W[1] + (size_t)pair * K;
        }
    } else if (EPI == EPI_QKV_ROPE) {
        lr0 = 2 * pair;
        lr1 = lr0 + 1;
        if (lr0 < a.N) {
            int s = 0, r = lr0;
            while (s < 2 && r >= a.seg_rows[s]) {
                r -= a.seg_rows[s];
                ++s;
            }
            wr0 = a.W[s] + (size_t)r * K;
            wr1 = wr0 + K;
        }
    } else {
        lr0 = 2 * pair;
        lr1 = lr0 + 1;
        if (lr0 < a.N) wr0 = a.W[0] + (size_t)lr0 * K;
        if (lr1 < a.N) wr1 = a.W[0] + (size_t)lr1 * K;
    }
    pdl_trigger();
    pdl_wait();
    float acc0[16], acc1[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc0[m] = acc1[m] = 0.f;
    for (int k = lane * 4; k < K; k += 128) {
        const float4 w0 = wr0 ? *reinterpret_cast<const float4*>(wr0 + k) : make_float4(0, 0, 0, 0);
        const float4 w1 = wr1 ? *reinterpret_cast<const float4*>(wr1 + k) : make_float4(0, 0, 0, 0);
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            if (m < M) {
                const float4 x = *reinterpret_cast<const float4*>(a.x + (size_t)m * a.ldx + k);
                acc0[m] += w0.x * x.x + w0.y * x.y + w0.z * x.z + w0.w * x.w;
                acc1[m] += w1.x * x.x + w1.y * x.y + w1.z * x.z + w1.w * x.w;
            }
        }
    }
    compute_rinv(a.epi.norm, M, a.m0, rinv_s);
    __syncthreads();
    const Epi& e = a.epi;
    float my0 = 0.f, my1 = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const float s0 = warp_sum(acc0[m]), s1 = warp_sum(acc1[m]);
        if (lane == m) {
            my0 = s0;
            my1 = s1;
        }
    }
    float ss = 0.f, bv = -FLT_MAX;
    int bi = INT_MAX;
    if (lane < M) {
        const int m = lane;
        const int mg = a.m0 + m;  // token index
        const float r = rinv_s[m];
        const float v0 = my0 * r, v1 = my1 * r;
        if (EPI == EPI_STORE_F32) {
            if (lr0 < a.N) e.y[(size_t)mg * e.ldy + lr0] = v0;
            if (lr1 < a.N) e.y[(size_t)mg * e.ldy + lr1] = v1;
        } else if (EPI == EPI_QKV_ROPE) {
            if (lr0 < a.N) epi_qkv_pair<float>(e, mg, lr0, v0, v1);
        } else if (EPI == EPI_SWIGLU) {
            if (lr0 < a.N) reinterpret_cast<float*>(e.g_out)[(size_t)mg * e.F + lr0] = swiglu(v0, v1);
        } else if (EPI == EPI_RESID) {
            if (lr0 < a.N) {
                const float hn = epi_resid1<float>(e, mg, lr0, v0);
                ss += hn * hn;
            }
            if (lr1 < a.N) {
                const float hn = epi_resid1<float>(e, mg, lr1, v1);
                ss += hn * hn;
            }
        } else if (EPI == EPI_LOGITS) {
            if (lr0 < a.N) {
                if (e.logits) e.logits[(size_t)m * e.ld_logits + lr0] = v0;
                am_merge(bv, bi, v0, lr0);
            }
            if (lr1 < a.N) {
                if (e.logits) e.logits[(size_t)m * e.ld_logits + lr1] = v1;
                am_merge(bv, bi, v1, lr1);
            }
        }
    }
    if (EPI == EPI_RESID || EPI == EPI_LOGITS) {
        if (lane < 16) {
            ss_s[warp][lane] = ss;
            amv_s[warp][lane] = bv;
            ami_s[warp][lane] = bi;
        }
        __syncthreads();
        if (threadIdx.x < M) {
            const int m = threadIdx.x;
            if (EPI == EPI_RESID) {
                float s = 0.f;
                for (int w = 0; w < 8; ++w) s += ss_s[w][m];
                e.ss_out[(size_t)blockIdx.x * e.ss_out_ld + a.m0 + m] = s;
            } else {
                float v = -FLT_MAX;
                int i = INT_MAX;
                for (int w = 0; w < 8; ++w) am_merge(v, i, amv_s[w][m], ami_s[w][m]);
                e.am_val[(size_t)blockIdx.x * M + m] = v;
                e.am_idx[(size_t)blockIdx.x * M + m] = i;
            }
        }
    }
    if (EPI == EPI_LOGITS) logits_finish(e, M, gridDim.x, &last_s);
}

// ---------------------------------------------------------------- launchers
template <int NB, int KS>
static cudaError_t launch_bf16_ks(const GemvArgs<__nv_bfloat16>& a, int ntiles, cudaStream_t s, bool pdl) {
    const dim3 grid((ntiles + (8 / KS) - 1) / (8 / KS));
    switch (a.epi.kind) {
        case EPI_STORE_F32: return launch_k(gemv_bf16_kernel<NB, KS, EPI_STORE_F32>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_QKV_ROPE: return launch_k(gemv_bf16_kernel<NB, KS, EPI_QKV_ROPE>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_SWIGLU: return launch_k(gemv_bf16_kernel<NB, KS, EPI_SWIGLU>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_RESID: return launch_k(gemv_bf16_kernel<NB, KS, EPI_RESID>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_LOGITS: return launch_k(gemv_bf16_kernel<NB, KS, EPI_LOGITS>, grid, GEMV_THREADS, 0, s, pdl, a);
    }
    return cudaErrorInvalidValue;
}

template <int NB>
static cudaError_t launch_bf16_nb(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl) {
    const int ntiles = gemv_num_tiles(a.epi.kind, a.N);
    // Enough warps in flight to cover HBM latency: about 16 warps per SM.
    const int want = 148 * 16;
    if (ntiles * 4 < want) return launch_bf16_ks<NB, 8>(a, ntiles, s, pdl);
    if (ntiles * 2 < want) return launch_bf16_ks<NB, 4>(a, ntiles, s, pdl);
    if (ntiles < want) return launch_bf16_ks<NB, 2>(a, ntiles, s, pdl);
    return launch_bf16_ks<NB, 1>(a, ntiles, s, pdl);
}

cudaError_t launch_gemv_bf16(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl) {
    if (a.M < 1 || a.M > 16 || a.K % 8 != 0) return cudaErrorInvalidValue;
    return a.M <= 8 ? launch_bf16_nb<8>(a, s, pdl) : launch_bf16_nb<16>(a, s, pdl);
}

cudaError_t launch_gemv_f32(const GemvArgs<float>& a, cudaStream_t s, bool pdl) {
    if (a.M < 1 || a.M > 16 || a.K % 4 != 0) return cudaErrorInvalidValue;
    const int pairs = a.epi.kind == EPI_SWIGLU ? a.N : (a.N + 1) / 2;
    const dim3 grid((pairs + 7) / 8);
    switch (a.epi.kind) {
        case EPI_STORE_F32: return launch_k(gemv_f32_kernel<EPI_STORE_F32>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_QKV_ROPE: return launch_k(gemv_f32_kernel<EPI_QKV_ROPE>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_SWIGLU: return launch_k(gemv_f32_kernel<EPI_SWIGLU>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_RESID: return launch_k(gemv_f32_kernel<EPI_RESID>, grid, GEMV_THREADS, 0, s, pdl, a);
        case EPI_LOGITS: return launch_k(gemv_f32_kernel<EPI_LOGITS>, grid, GEMV_THREADS, 0, s, pdl, a);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lfw
