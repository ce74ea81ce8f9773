// Decode projections y[m][n] = sum_k x[m][k] W[n][k] for M <= 16 token rows: one
// launch per projection. The bf16 kernel is the TMA-fed producer/consumer
// pipeline of gemv_core.cuh; the fp32 kernel runs on CUDA cores.
#include "gemv_core.cuh"

namespace lfw {

constexpr int GEMV_THREADS = 256;

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


// bf16 projection: one CTA per SM, GV_STAGES units in flight per CTA. The launch is
// cooperative (every CTA resident), so a row tile split over several CTAs is
// finished by its first CTA, which waits for the other CTAs' pieces; they publish
// them as soon as they reach the end of their part and move on.
// Ring depth: 8 stages (128 KB) for the layer projections, about the bytes an SM
// has in flight at its share of HBM bandwidth under load (measured at the
// Llama-3-8B shape: 3.51 ms per decode token against 3.58 with 5 stages, 3.51 with
// 7 or 9, 3.57 with 10); the lm_head, one long stream of 1 GB, keeps 10 stages
// (163 against 172 us with 5). With 16 token columns (NB = 16: 5 to 16 tokens, or
// their split parts) the residual projections (wo, and w2 with its long rows) keep 7
// stages, so that 16 token rows of a CTA's k blocks of the 14336-wide FFN input (49
// blocks at the Llama-3-8B shape) fit the staging buffer (batch 16: 7.26 -> 7.05 ms
// per decode step); with one token (NB = 8) the deeper ring is the better use of the
// shared memory.
template <int NB, int EPI> constexpr bool gv_wide_xs() { return NB == 16 && EPI == EPI_RESID; }
template <int NB, int EPI> constexpr int gv_stages() { return EPI == EPI_LOGITS ? 10 : gv_wide_xs<NB, EPI>() ? 7 : 8; }
constexpr int GV_THREADS = GV_CONSUMERS + 32;   // 8 consumer warps + 1 producer warp
// Token rows staged in shared memory when the CTA's k blocks of them fit.
template <int NB, int EPI> constexpr int gv_xs_bytes() { return (gv_wide_xs<NB, EPI>() ? 98 : 56) * 1024 + 256; }
template <int NB, int EPI> constexpr int gv_smem() {
    return 1024 + gv_stages<NB, EPI>() * GV_UNIT_BYTES + gv_xs_bytes<NB, EPI>() + 2 * gv_stages<NB, EPI>() * 8 + 64;
}

template <int NB, int EPI, bool SPLIT>
__global__ void __launch_bounds__(GV_THREADS, gv_stages<NB, EPI>() > 6 ? 1 : 2)
    gemv_bf16_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                     const __grid_constant__ CUtensorMap tm2, const GemvArgs<__nv_bfloat16> a, int ntiles, int nku,
                     int max_pieces) {
    constexpr int GV_STAGES = gv_stages<NB, EPI>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem + GV_STAGES * GV_UNIT_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + GV_STAGES * GV_UNIT_BYTES + gv_xs_bytes<NB, EPI>());
    __shared__ float rinv_s[16];
    __shared__ float rred_s[8][16];
    GvRing ring{smem, full, full + GV_STAGES, GV_STAGES, 0, 0u, 0};
    const int warp = threadIdx.x >> 5;
    const GvWork w = gv_work(ntiles, nku);

    if (threadIdx.x == 0) {
        for (int i = 0; i < GV_STAGES; ++i) {
            mbar_init(&ring.full[i], 1);
            mbar_init(&ring.empty[i], 8);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tm0);
        tma_prefetch_desc(&tm1);
        tma_prefetch_desc(&tm2);
    }
    __syncthreads();
    pdl_trigger();

    if (warp == 8) {
        // producer: weights do not depend on the previous kernel
        if ((threadIdx.x & 31) == 0) {
            const bool ok = gv_produce(ring, w, EPI == EPI_SWIGLU, &tm0, &tm1, &tm2, a.seg_rows[0], a.seg_rows[1],
                                       a.epi.err, DERR_GEMV_PRODUCER_WAIT);
            gv_drain(ring, ok ? w.u1 - w.u0 : GV_STAGES, a.epi.err, DERR_GEMV_PRODUCER_WAIT);
        }
        pdl_wait();
        return;
    }

    // consumers
    pdl_wait();
    GvX X;
    X.x = a.x;
    X.ldx = a.ldx;
    X.M = a.M;
    X.K = a.K;
    // the k blocks this CTA's units read: kb0, kb0 + 1, ... (mod nku)
    const bool all_k = w.u1 - w.u0 >= nku || w.u1 <= w.u0;
    X.kb0 = all_k ? 0 : (int)(w.u0 % nku);
    X.nku = nku;
    X.Kp = (all_k ? nku : (int)(w.u1 - w.u0)) * GV_BK;
    X.xlo = SPLIT ? a.x_lo : nullptr;
    X.MX = SPLIT ? 2 * a.M : a.M;
    X.xs = (long long)X.MX * X.Kp * 2 <= gv_xs_bytes<NB, EPI>() ? xs : nullptr;
    gv_prologue(const_cast<__nv_bfloat16*>(X.xs), a.x, a.ldx, a.M, a.K, X.Kp, a.epi.norm, a.m0, rinv_s, rred_s, X.kb0,
                nku, X.xlo);
    gv_consume<NB, EPI, SPLIT>(ring, w, X, a.N, a.m0, rinv_s, a.epi, a.ws, max_pieces, a.epi.err,
                               DERR_GEMV_CONSUMER_WAIT);
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
template <int NB, int EPI, bool SPLIT>
static cudaError_t launch_bf16_e(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl) {
    static bool smem_set = false;
    if (!smem_set) {
        cudaError_t e = cudaFuncSetAttribute(gemv_bf16_kernel<NB, EPI, SPLIT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, gv_smem<NB, EPI>());
        if (e != cudaSuccess) return e;
        smem_set = true;
    }
    if (!a.tmw[0]) return cudaErrorInvalidValue;
    const GemvPlan p = gemv_plan(EPI, a.N, a.K, a.num_sms, 1);
    if ((size_t)p.ntiles * p.max_pieces * GV_PIECE_FLOATS > a.ws.part_floats || p.ntiles > a.ws.tiles_cap ||
        !a.ws.warp_cnt)
        return cudaErrorInvalidValue;
    const CUtensorMap& m0 = *a.tmw[0];
    const CUtensorMap& m1 = a.tmw[1] ? *a.tmw[1] : m0;
    const CUtensorMap& m2 = a.tmw[2] ? *a.tmw[2] : m0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(GV_THREADS);
    cfg.dynamicSmemBytes = gv_smem<NB, EPI>();
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemv_bf16_kernel<NB, EPI, SPLIT>, m0, m1, m2, a, p.ntiles, p.nkb, p.max_pieces);
}

template <int NB, bool SPLIT>
static cudaError_t launch_bf16_nb(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl) {
    switch (a.epi.kind) {
        case EPI_STORE_F32: return launch_bf16_e<NB, EPI_STORE_F32, SPLIT>(a, s, pdl);
        case EPI_QKV_ROPE: return launch_bf16_e<NB, EPI_QKV_ROPE, SPLIT>(a, s, pdl);
        case EPI_SWIGLU: return launch_bf16_e<NB, EPI_SWIGLU, SPLIT>(a, s, pdl);
        case EPI_RESID: return launch_bf16_e<NB, EPI_RESID, SPLIT>(a, s, pdl);
        case EPI_LOGITS: return launch_bf16_e<NB, EPI_LOGITS, SPLIT>(a, s, pdl);
    }
    return cudaErrorInvalidValue;
}

int gemv_num_tiles(int kind, int N) {
    // row tiles of the decode projection: 128 rows (64 w1 + 64 w3 rows for SwiGLU)
    return kind == EPI_SWIGLU ? (N + 63) / 64 : (N + 127) / 128;
}

// One CTA per SM (never more CTAs than units); max_pieces bounds how many CTAs
// share one row tile.
GemvPlan gemv_plan(int kind, int N, int K, int num_sms, int) {
    GemvPlan p;
    p.ntiles = gemv_num_tiles(kind, N);
    p.nkb = (K + GV_BK - 1) / GV_BK;  // units per tile
    p.TB = (long long)p.ntiles * p.nkb;
    p.grid = (long long)num_sms < p.TB ? num_sms : (int)p.TB;
    if (p.grid < 1) p.grid = 1;
    long long mp = 1;
    for (long long t = 0; t < p.ntiles; ++t) {
        const long long cf = ((t * p.nkb + 1) * p.grid - 1) / p.TB;
        const long long cl = (((t + 1) * p.nkb) * p.grid - 1) / p.TB;
        if (cl - cf + 1 > mp) mp = cl - cf + 1;
    }
    p.max_pieces = (int)mp;
    return p;
}

size_t gemv_scratch_floats(int kind, int N, int K, int num_sms) {
    const GemvPlan p = gemv_plan(kind, N, K, num_sms, 1);
    return (size_t)p.ntiles * p.max_pieces * GV_PIECE_FLOATS;
}

cudaError_t launch_gemv_bf16(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl) {
    if (a.M < 1 || a.M > 16 || a.K % 8 != 0) return cudaErrorInvalidValue;
    if (a.x_lo && a.M <= 8)  // split activations: 2M B-operand columns
        return a.M <= 4 ? launch_bf16_nb<8, true>(a, s, pdl) : launch_bf16_nb<16, true>(a, s, pdl);
    return a.M <= 8 ? launch_bf16_nb<8, false>(a, s, pdl) : launch_bf16_nb<16, false>(a, s, pdl);
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
