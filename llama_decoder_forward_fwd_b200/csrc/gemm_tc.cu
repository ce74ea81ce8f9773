// Prefill projections on the 5th-generation tensor cores: C = A W^T with
// A = activations [M][K] bf16 and W = a weight matrix [N][K] bf16 ("Building
// llama3 from scratch": q_per_token = x @ wq_head^T, here for all tokens and all
// heads at once), fp32 accumulation in tensor memory.
//
// Persistent kernel, one CTA per SM, 10 warps:
//   warp 0     TMA producer: streams 128x64 A tiles and 256x64 B tiles into a
//              4-stage shared-memory ring (128-byte swizzle), one mbarrier per
//              stage for "full" (transaction bytes) and one for "empty".
//   warp 1     allocates 512 TMEM columns and issues tcgen05.mma (M=128, N=256,
//              K=16; four per 64-wide k block) from one elected thread into one
//              of two 256-column accumulators, committing "empty" per stage and
//              "accumulator full" per tile.
//   warps 2-9  epilogue, two warps per 32-lane quarter (rows) of the accumulator,
//              each half of the columns: tcgen05.ld, the fused epilogue (RMSNorm
//              scale, RoPE + KV-cache append, SwiGLU, or residual add) and stores,
//              with each chunk's global operands loaded a chunk ahead; then release
//              the accumulator so the MMA warp can start the tile after next.
// Tiles are visited m-fastest so CTAs running together share weight tiles in L2.
#include "epilogue.cuh"

namespace lfw {

constexpr int G_STAGES = 4;
constexpr int G_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB
constexpr int G_B_BYTES = GEMM_BN * GEMM_BK * 2;  // 32 KB
constexpr int G_STAGE_BYTES = G_A_BYTES + G_B_BYTES;
constexpr int G_SMEM_BYTES = G_STAGES * G_STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr int G_THREADS = 320;
constexpr uint32_t G_TMEM_COLS = 512;

struct GemmKernelParams {
    int seg_cols[3];
    int M, N, K;
    Epi epi;
};

template <int EPI>
__global__ void __launch_bounds__(G_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                   const GemmKernelParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G_STAGES * G_STAGE_BYTES);
    uint64_t* empty = full + G_STAGES;
    uint64_t* tfull = empty + G_STAGES;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* err = p.epi.err;
    __shared__ float ss_half[2][GEMM_BM];  // residual epilogue: the row sums of squares of the two halves

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < G_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 8);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
        tma_prefetch_desc(&tmB2);
    }
    if (warp == 1) {
        tc_alloc(tmem_slot, G_TMEM_COLS);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_trigger();
    pdl_wait();

    const int num_m = (p.M + GEMM_BM - 1) / GEMM_BM;
    const int num_n = (EPI == EPI_SWIGLU) ? p.N / (GEMM_BN / 2) : p.N / GEMM_BN;
    const int total = num_m * num_n;
    const int nk = p.K / GEMM_BK;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const int mb = tile % num_m, nb = tile / num_m;
                const CUtensorMap* b0;
                const CUtensorMap* b1;
                int r0, r1;
                if (EPI == EPI_SWIGLU) {
                    b0 = &tmB0;
                    b1 = &tmB1;
                    r0 = r1 = nb * (GEMM_BN / 2);
                } else {
                    // each 128-row half of the tile from the segment (wq, wk, wv) holding it
                    auto seg_of = [&](int c, int& row) -> const CUtensorMap* {
                        int s = 0;
                        while (s < 2 && c >= p.seg_cols[s]) {
                            c -= p.seg_cols[s];
                            ++s;
                        }
                        row = c;
                        return (s == 0) ? &tmB0 : (s == 1) ? &tmB1 : &tmB2;
                    };
                    b0 = seg_of(nb * GEMM_BN, r0);
                    b1 = seg_of(nb * GEMM_BN + GEMM_BN / 2, r1);
                }
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, err, DERR_GEMM_PRODUCER_WAIT)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * G_STAGE_BYTES;
                    uint8_t* sb = sa + G_A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], G_STAGE_BYTES);
                    tma_load_2d(sa, &tmA, &full[stage], kb * GEMM_BK, mb * GEMM_BM);
                    tma_load_2d(sb, b0, &full[stage], kb * GEMM_BK, r0);
                    tma_load_2d(sb + G_B_BYTES / 2, b1, &full[stage], kb * GEMM_BK, r1);
                    if (++stage == G_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let copies already issued land before the CTA can exit.
                for (int i = 0; i < G_STAGES; ++i) mbar_wait(&full[i], 0, nullptr, 0);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(GEMM_BM, GEMM_BN);
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, err, DERR_GEMM_MMA_WAIT)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * GEMM_BN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&full[stage], phase, err, DERR_GEMM_MMA_WAIT)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * G_STAGE_BYTES);
                    const uint32_t sb = sa + G_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
                        tc_mma_f16(d_tmem, smem_desc_sw128(sa + kk * 32), smem_desc_sw128(sb + kk * 32), idesc,
                                   (kb | kk) != 0);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == G_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                tc_commit(&tfull[acc]);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..9) ----------------
        // Warps w and w+4 share TMEM lane quarter w % 4 (32 rows of the tile); the
        // first takes the tile's first 128 columns, the second the last 128 (for
        // SwiGLU: the first and last two 32-column chunks of the w1 and w3 halves).
        // The global operands of a chunk (residual h and norm weights, RoPE cos/sin)
        // and the row's RMSNorm scale are loaded one chunk ahead, the first ones
        // before the accumulator is waited for, so the stores do not wait on them.
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int half = (warp - 2) >> 2;
        const int row_in_tile = quarter * 32 + lane;
        const Epi& e = p.epi;
        constexpr int NCH = EPI == EPI_SWIGLU ? 2 : 4;  // 32-column chunks per warp
        // After a failed (timed-out) wait a warp stops waiting but keeps walking the
        // tiles, so the two warps of a lane quarter always meet at their named barriers.
        bool ok = true;
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            const int mb = tile % num_m, nb = tile / num_m;
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            const int m = mb * GEMM_BM + row_in_tile;
            const bool valid = m < p.M;
            const float rinv = valid ? row_rinv(e.norm, m) : 0.f;
            // operands of chunk ch: columns c0(ch) .. c0(ch)+31
            auto col0 = [&](int ch) { return nb * GEMM_BN + half * (GEMM_BN / 2) + ch * 32; };
            float4 opa[8], opb[8];  // RESID: h (8 float4) and norm weights (4 uint4 in opb[0..3]);
                                    // QKV: cos (opa[0..3]) and sin (opb[0..3]) of the chunk's 16 pairs
            auto load_ops = [&](int ch) {
                if (!valid) return;
                const int c0 = col0(ch);
                if (EPI == EPI_RESID) {
                    const float4* hp = reinterpret_cast<const float4*>(e.h + (size_t)m * e.D + c0);
#pragma unroll
                    for (int i = 0; i < 8; ++i) opa[i] = hp[i];
                    const float4* wp = reinterpret_cast<const float4*>(reinterpret_cast<const __nv_bfloat16*>(e.wnext) + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) opb[i] = wp[i];
                } else if (EPI == EPI_QKV_ROPE) {
                    const int Hd = e.H * e.d, Hkd = e.Hk * e.d;
                    if (c0 < Hd + Hkd) {
                        const int b = m / e.T;
                        const int pos = e.pos0[b] + (m - b * e.T);
                        if (pos >= 0 && pos < e.S_max) {
                            const long long ti = (long long)pos * (e.d >> 1) + ((c0 % e.d) >> 1);
                            const float4* cp = reinterpret_cast<const float4*>(e.rope_cos + ti);
                            const float4* sp = reinterpret_cast<const float4*>(e.rope_sin + ti);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                opa[i] = cp[i];
                                opb[i] = sp[i];
                            }
                        }
                    }
                }
            };
            if (EPI == EPI_RESID || EPI == EPI_QKV_ROPE) load_ops(0);
            if (ok && !mbar_wait(&tfull[acc], acc_phase, err, DERR_GEMM_EPI_WAIT)) ok = false;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * GEMM_BN;
            if (EPI == EPI_SWIGLU) {
                const int n0 = nb * (GEMM_BN / 2);
#pragma unroll 1
                for (int cc = 0; cc < NCH; ++cc) {
                    const int ch = half * NCH + cc;
                    uint32_t ra[32], rc[32];
                    tc_ld_32x32b_x32(tbase + ch * 32, ra);
                    tc_ld_32x32b_x32(tbase + GEMM_BN / 2 + ch * 32, rc);
                    tc_wait_ld();
                    if (valid) {
                        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(e.g_out) + (size_t)m * e.F + n0 + ch * 32;
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            float v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                v[i] = swiglu(__uint_as_float(ra[j + i]) * rinv, __uint_as_float(rc[j + i]) * rinv);
                            store8<__nv_bfloat16>(dst + j, v);
                        }
                    }
                }
            } else {
                float ss = 0.f;
#pragma unroll 1
                for (int cc = 0; cc < NCH; ++cc) {
                    uint32_t r[32];
                    tc_ld_32x32b_x32(tbase + half * (GEMM_BN / 2) + cc * 32, r);
                    // this chunk's operands are in opa/opb; fetch the next chunk's while
                    // the accumulator values arrive
                    float4 ca[8], cb[4];
#pragma unroll
                    for (int i = 0; i < 8; ++i) ca[i] = opa[i];
#pragma unroll
                    for (int i = 0; i < 4; ++i) cb[i] = opb[i];
                    if ((EPI == EPI_RESID || EPI == EPI_QKV_ROPE) && cc + 1 < NCH) load_ops(cc + 1);
                    tc_wait_ld();
                    if (!valid) continue;
                    const int c0 = col0(cc);
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        float v[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[j + i]) * rinv;
                        if (EPI == EPI_STORE_F32) {
                            store8<float>(e.y + (size_t)m * e.ldy + c0 + j, v);
                        } else if (EPI == EPI_QKV_ROPE) {
                            const int Hd = e.H * e.d, Hkd = e.Hk * e.d;
                            const int c = c0 + j;
                            const int b = m / e.T;
                            const int pos = e.pos0[b] + (m - b * e.T);
                            if (!LFW_CHECK(pos >= 0 && pos < e.S_max, e.err, BC_CACHE_POS)) continue;
                            if (c < Hd + Hkd) {
                                // pairs 4j/8 .. of the chunk: cos/sin elements j/2 .. j/2+3
                                const float4 cs = ca[j >> 3], sn = cb[j >> 3];
                                const float cv[4] = {cs.x, cs.y, cs.z, cs.w}, sv[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    const float x0 = v[2 * q], x1 = v[2 * q + 1];
                                    v[2 * q] = x0 * cv[q] - x1 * sv[q];
                                    v[2 * q + 1] = x0 * sv[q] + x1 * cv[q];
                                }
                            }
                            if (c < Hd) {
                                store8<__nv_bfloat16>(reinterpret_cast<__nv_bfloat16*>(e.q_out) + (size_t)m * Hd + c, v);
                            } else {
                                int kc = c - Hd;
                                const bool isv = kc >= Hkd;
                                if (isv) kc -= Hkd;
                                const int kvh = kc / e.d, dd = kc - kvh * e.d;
                                __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(isv ? e.v_cache : e.k_cache);
                                store8<__nv_bfloat16>(base + ((long long)(b * e.Hk + kvh) * e.S_max + pos) * e.d + dd, v);
                            }
                        } else if (EPI == EPI_RESID) {
                            float* hp = e.h + (size_t)m * e.D + c0 + j;
                            const float4 h0 = ca[j >> 2], h1 = ca[(j >> 2) + 1];
                            float hn[8] = {h0.x + v[0], h0.y + v[1], h0.z + v[2], h0.w + v[3],
                                           h1.x + v[4], h1.y + v[5], h1.z + v[6], h1.w + v[7]};
                            store8<float>(hp, hn);
                            const float4 wf = cb[j >> 3];
                            const uint4 wv = make_uint4(__float_as_uint(wf.x), __float_as_uint(wf.y),
                                                        __float_as_uint(wf.z), __float_as_uint(wf.w));
                            float hw[8];
                            hw[0] = hn[0] * bf16lo(wv.x);
                            hw[1] = hn[1] * bf16hi(wv.x);
                            hw[2] = hn[2] * bf16lo(wv.y);
                            hw[3] = hn[3] * bf16hi(wv.y);
                            hw[4] = hn[4] * bf16lo(wv.z);
                            hw[5] = hn[5] * bf16hi(wv.z);
                            hw[6] = hn[6] * bf16lo(wv.w);
                            hw[7] = hn[7] * bf16hi(wv.w);
                            store8<__nv_bfloat16>(reinterpret_cast<__nv_bfloat16*>(e.hw_out) + (size_t)m * e.D + c0 + j,
                                                  hw);
#pragma unroll
                            for (int i = 0; i < 8; ++i) ss += hn[i] * hn[i];
                        }
                    }
                }
                if (EPI == EPI_RESID) {
                    // the row's sum of squares over the tile: the two halves' sums, added
                    // in a fixed order
                    ss_half[half][row_in_tile] = ss;
                    named_bar_sync(1 + quarter, 64);
                    if (half == 0 && valid)
                        e.ss_out[(size_t)nb * e.ss_out_ld + m] = ss + ss_half[1][row_in_tile];
                    named_bar_sync(1 + quarter, 64);  // the slots are rewritten by the next tile
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tc_dealloc(tmem_base, G_TMEM_COLS);
    }
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t s, bool pdl) {
    if (a.M < 1 || a.K % GEMM_BK != 0) return cudaErrorInvalidValue;
    const int kind = a.epi.kind;
    if (kind == EPI_SWIGLU ? (a.N % (GEMM_BN / 2) != 0) : (a.N % GEMM_BN != 0)) return cudaErrorInvalidValue;
    if (kind == EPI_LOGITS) return cudaErrorInvalidValue;
    GemmKernelParams p;
    for (int i = 0; i < 3; ++i) p.seg_cols[i] = a.seg_cols[i];
    p.M = a.M;
    p.N = a.N;
    p.K = a.K;
    p.epi = a.epi;
    const int num_m = (a.M + GEMM_BM - 1) / GEMM_BM;
    const int num_n = kind == EPI_SWIGLU ? a.N / (GEMM_BN / 2) : a.N / GEMM_BN;
    const int total = num_m * num_n;
    const dim3 grid(total < a.num_sms ? total : a.num_sms);
    const CUtensorMap& b0 = *a.tmB[0];
    const CUtensorMap& b1 = a.tmB[1] ? *a.tmB[1] : *a.tmB[0];
    const CUtensorMap& b2 = a.tmB[2] ? *a.tmB[2] : *a.tmB[0];
    auto go = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        return launch_k(kern, grid, dim3(G_THREADS), G_SMEM_BYTES, s, pdl, *a.tmA, b0, b1, b2, p);
    };
    switch (kind) {
        case EPI_STORE_F32: return go(gemm_tc_kernel<EPI_STORE_F32>);
        case EPI_QKV_ROPE: return go(gemm_tc_kernel<EPI_QKV_ROPE>);
        case EPI_SWIGLU: return go(gemm_tc_kernel<EPI_SWIGLU>);
        case EPI_RESID: return go(gemm_tc_kernel<EPI_RESID>);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lfw
