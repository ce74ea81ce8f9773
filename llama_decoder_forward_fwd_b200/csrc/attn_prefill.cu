// Causal grouped-query attention for a block of prompt tokens (prefill).
//
// What it computes ("Resumen ...", "Implementación de la atención" and
// "Atención multi-head"; llama3.np, "GQA" and "Scaled Dot-Product Attention"):
// for query head h of the token at position p, scores q.k_j / sqrt(d) over keys
// j <= p of KV head h / G (G = n_heads / n_kv_heads), future keys masked, softmax,
// weighted sum of values, heads concatenated.
//
// Layout of the work. A CTA owns 128 "rows" of one (sequence, KV head): row r is
// (token t = r / G, query head kvh*G + r % G), so the G query heads that share a
// KV head sit in one CTA and every K/V tile is loaded once for all of them.
// K and V tiles of 64 keys x 128 dims come from the KV cache by TMA (two
// 64-dim halves with the 128-byte swizzle) into a 2-stage ring. Each of the 8
// warps runs mma.sync m16n8k16 on its 16 rows: S = Q K^T (ldmatrix from the
// swizzled tiles), an online softmax in registers (running max and sum in the
// log2 domain), and O += P V with P reused from the S registers.
#include "common.cuh"
#include "kernels.cuh"

#include <math.h>

namespace lfw {

constexpr int FA_THREADS = 256;
constexpr int FA_ROWS = 128;
constexpr int FA_KT = 64;
constexpr int FA_D = 128;
constexpr int FA_Q_BYTES = FA_ROWS * FA_D * 2;   // 32 KB
constexpr int FA_KV_BYTES = FA_KT * FA_D * 2;    // 16 KB per K or V tile
constexpr int FA_SMEM = 1024 + FA_Q_BYTES + 4 * FA_KV_BYTES + 64;

DEVI uint32_t kv_addr(uint32_t base, int key, int chunk) {
    // chunk: 16-byte column chunk 0..15 of the 128-dim row; halves are 8 KB apart.
    return base + (chunk >> 3) * (FA_KT * 128) + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
}

__global__ void __launch_bounds__(FA_THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const AttnPrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Ks = smem;                       // 2 stages x 16 KB
    uint8_t* Vs = smem + 2 * FA_KV_BYTES;     // 2 stages x 16 KB
    uint8_t* Qs = smem + 4 * FA_KV_BYTES;     // 32 KB
    uint64_t* barK = reinterpret_cast<uint64_t*>(Qs + FA_Q_BYTES);
    uint64_t* barV = barK + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int G = a.H / a.Hk;
    const int rb = gridDim.x - 1 - blockIdx.x;  // longest rows first
    const int b = blockIdx.y / a.Hk, kvh = blockIdx.y % a.Hk;
    const int HD = a.H * FA_D;

    pdl_trigger();
    pdl_wait();
    const int p0 = a.pos0[b];

    const int row0 = rb * FA_ROWS;
    const int t_last = min(a.T - 1, (row0 + FA_ROWS - 1) / G);
    const int p_max = min(p0 + t_last, a.S_max - 1);  // never read past this head's cache rows
    const int nkt = p_max / FA_KT + 1;
    const long long kv_row0 = a.row_base + (long long)(b * a.Hk + kvh) * a.S_max;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&barK[i], 1);
            mbar_init(&barV[i], 1);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        for (int kt = 0; kt < 2 && kt < nkt; ++kt) {
            mbar_arrive_expect_tx(&barK[kt], FA_KV_BYTES);
            tma_load_2d(Ks + kt * FA_KV_BYTES, &tmK, &barK[kt], 0, (int)(kv_row0 + kt * FA_KT));
            tma_load_2d(Ks + kt * FA_KV_BYTES + FA_KV_BYTES / 2, &tmK, &barK[kt], 64, (int)(kv_row0 + kt * FA_KT));
            mbar_arrive_expect_tx(&barV[kt], FA_KV_BYTES);
            tma_load_2d(Vs + kt * FA_KV_BYTES, &tmV, &barV[kt], 0, (int)(kv_row0 + kt * FA_KT));
            tma_load_2d(Vs + kt * FA_KV_BYTES + FA_KV_BYTES / 2, &tmV, &barV[kt], 64, (int)(kv_row0 + kt * FA_KT));
        }
    }

    // Stage this CTA's 128 query rows in shared memory (16-byte chunks XOR-swizzled by row).
    for (int idx = threadIdx.x; idx < FA_ROWS * 16; idx += FA_THREADS) {
        const int r = idx >> 4, c = idx & 15;
        const int rg = row0 + r;
        const int t = rg / G, h = kvh * G + (rg - t * G);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < a.T)
            v = *reinterpret_cast<const uint4*>(a.q + ((long long)(b * a.T + t) * a.H + h) * FA_D + c * 8);
        *reinterpret_cast<uint4*>(Qs + r * 256 + ((c ^ (r & 7)) << 4)) = v;
    }
    __syncthreads();

    uint32_t qf[8][4];
    {
        const uint32_t qbase = smem_u32(Qs);
        const int j = lane >> 3, i = lane & 7;
        const int r = warp * 16 + (j & 1) * 8 + i;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c = 2 * kk + (j >> 1);
            ldsm_x4(qf[kk], qbase + r * 256 + ((c ^ (r & 7)) << 4));
        }
    }

    // Positions of this lane's two rows (g and g+8 of the warp's 16); -1 if no token.
    int prow[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int rg = row0 + warp * 16 + g + 8 * hh;
        const int t = rg / G;
        prow[hh] = t < a.T ? p0 + t : -1;
    }
    const int wr_first = row0 + warp * 16, wr_last = row0 + warp * 16 + 15;
    const int w_plo = (wr_first / G < a.T) ? p0 + wr_first / G : INT_MAX;
    const int w_phi = (wr_first / G < a.T) ? p0 + min(a.T - 1, wr_last / G) : -1;

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    const float sl2 = a.scale_log2;
    bool ok = true;

    for (int kt = 0; kt < nkt; ++kt) {
        const int st = kt & 1;
        const uint32_t ph = (kt >> 1) & 1;
        const bool active = ok && (kt * FA_KT <= w_phi);
        if (ok && !mbar_wait(&barK[st], ph, a.err, DERR_ATTN_TMA_WAIT)) ok = false;
        if (active && ok) {
            const uint32_t kb = smem_u32(Ks + st * FA_KV_BYTES);
            float s[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
            {
                const int j = lane >> 3, i = lane & 7;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
                    for (int np = 0; np < 4; ++np) {
                        uint32_t r[4];
                        const int key = (2 * np + (j >> 1)) * 8 + i;
                        ldsm_x4(r, kv_addr(kb, key, 2 * kk + (j & 1)));
                        mma_bf16_16816(s[2 * np], qf[kk], r[0], r[1]);
                        mma_bf16_16816(s[2 * np + 1], qf[kk], r[2], r[3]);
                    }
                }
            }
            const bool need_mask = (kt * FA_KT + FA_KT - 1) > w_plo;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float mx = -INFINITY;
#pragma unroll
                for (int n = 0; n < 8; ++n)
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        float v = s[n][2 * hh + e2] * sl2;
                        if (need_mask) {
                            const int key = kt * FA_KT + n * 8 + 2 * t4 + e2;
                            if (key > prow[hh]) v = -INFINITY;
                        }
                        s[n][2 * hh + e2] = v;
                        mx = fmaxf(mx, v);
                    }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float mnew = fmaxf(mrow[hh], mx);
                const float muse = (mnew == -INFINITY) ? 0.f : mnew;
                const float alpha = exp2f(mrow[hh] - muse);
                mrow[hh] = mnew;
                float sum = 0.f;
#pragma unroll
                for (int n = 0; n < 8; ++n)
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const float pv = exp2f(s[n][2 * hh + e2] - muse);
                        s[n][2 * hh + e2] = pv;
                        sum += pv;
                    }
                lrow[hh] = lrow[hh] * alpha + sum;
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    o[n][2 * hh] *= alpha;
                    o[n][2 * hh + 1] *= alpha;
                }
            }
            if (!mbar_wait(&barV[st], ph, a.err, DERR_ATTN_TMA_WAIT)) ok = false;
            if (ok) {
                const uint32_t vb = smem_u32(Vs + st * FA_KV_BYTES);
                const int j = lane >> 3, i = lane & 7;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t pf[4];
                    pf[0] = pack_bf16x2(s[2 * ks][0], s[2 * ks][1]);
                    pf[1] = pack_bf16x2(s[2 * ks][2], s[2 * ks][3]);
                    pf[2] = pack_bf16x2(s[2 * ks + 1][0], s[2 * ks + 1][1]);
                    pf[3] = pack_bf16x2(s[2 * ks + 1][2], s[2 * ks + 1][3]);
                    const int key = ks * 16 + (j & 1) * 8 + i;
#pragma unroll
                    for (int dp = 0; dp < 8; ++dp) {
                        uint32_t r[4];
                        ldsm_x4_t(r, kv_addr(vb, key, 2 * dp + (j >> 1)));
                        mma_bf16_16816(o[2 * dp], pf, r[0], r[1]);
                        mma_bf16_16816(o[2 * dp + 1], pf, r[2], r[3]);
                    }
                }
            }
        } else if (ok) {
            if (!mbar_wait(&barV[st], ph, a.err, DERR_ATTN_TMA_WAIT)) ok = false;
        }
        __syncthreads();
        if (threadIdx.x == 0 && kt + 2 < nkt) {
            const int nt = kt + 2;
            mbar_arrive_expect_tx(&barK[st], FA_KV_BYTES);
            tma_load_2d(Ks + st * FA_KV_BYTES, &tmK, &barK[st], 0, (int)(kv_row0 + nt * FA_KT));
            tma_load_2d(Ks + st * FA_KV_BYTES + FA_KV_BYTES / 2, &tmK, &barK[st], 64, (int)(kv_row0 + nt * FA_KT));
            mbar_arrive_expect_tx(&barV[st], FA_KV_BYTES);
            tma_load_2d(Vs + st * FA_KV_BYTES, &tmV, &barV[st], 0, (int)(kv_row0 + nt * FA_KT));
            tma_load_2d(Vs + st * FA_KV_BYTES + FA_KV_BYTES / 2, &tmV, &barV[st], 64, (int)(kv_row0 + nt * FA_KT));
        }
    }

    // Normalise and store this lane's two rows.
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float l = lrow[hh];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int rg = row0 + warp * 16 + g + 8 * hh;
        const int t = rg / G, h = kvh * G + (rg - t * G);
        if (t >= a.T || prow[hh] < 0) continue;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16* dst = a.out + (long long)(b * a.T + t) * HD + h * FA_D + 2 * t4;
#pragma unroll
        for (int n = 0; n < 16; ++n)
            *reinterpret_cast<uint32_t*>(dst + n * 8) = pack_bf16x2(o[n][2 * hh] * inv, o[n][2 * hh + 1] * inv);
    }
}

cudaError_t launch_attn_prefill(const AttnPrefillArgs& a, cudaStream_t s, bool pdl) {
    if (a.H % a.Hk != 0 || a.T < 1) return cudaErrorInvalidValue;
    const int G = a.H / a.Hk;
    const dim3 grid((a.T * G + FA_ROWS - 1) / FA_ROWS, a.B * a.Hk);
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM);
    if (e != cudaSuccess) return e;
    return launch_k(attn_prefill_kernel, grid, dim3(FA_THREADS), FA_SMEM, s, pdl, *a.tmK, *a.tmV, a);
}

}  // namespace lfw
