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

// Order-preserving key of (logit, token id) for a 64-bit atomicMax: a larger
// logit wins, and among equal logits the lower id ("the highest value is the
// next token"; ties go to the lowest id).
DEVI unsigned long long am_key(float v, int idx) {
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}
DEVI int am_key_index(unsigned long long k) { return (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull)); }

// Decode projection kernel: a TMA-fed CTA pipeline.
//
// Work unit = one 128-row x 64-wide tile of the weight matrix (16 KB, one TMA
// tensor copy with the 128-byte swizzle). The units of all row tiles, in
// (row tile, k) order, are split into equal contiguous ranges, one per CTA (one
// CTA per SM), so every SM streams the same number of bytes. Warp 8 is the
// producer and keeps GV_STAGES units in flight in a shared-memory ring (full /
// empty mbarriers). Each of the 8 consumer warps owns 16 of the 128 rows and
// consumes every unit with mma.sync m16n8k16 (weights as A, read from the
// swizzled tile; token rows as B, staged in shared memory): no reduction between
// warps is needed. A row tile whose k range is split over several CTAs leaves
// one partial per CTA; the CTA that completes the tile (atomic counter, no
// waiting) adds the partials in CTA order, which keeps results deterministic,
// and its warps run the fused epilogue on their own rows.
constexpr int GV_ROWS = 128;                    // rows per tile (8 warps x 16)
constexpr int GV_BK = 64;                       // k per unit
constexpr int GV_UNIT_BYTES = GV_ROWS * GV_BK * 2;
constexpr int GV_STAGES = 5;                    // ~110 KB per CTA: two CTAs (of consecutive
                                                // launches) can share an SM
constexpr int GV_THREADS = 288;                 // 8 consumer warps + 1 producer warp
constexpr int GV_XS_BYTES = 28 * 1024 + 256;    // token rows staged whole when they fit
constexpr int GV_SMEM = 1024 + GV_STAGES * GV_UNIT_BYTES + GV_XS_BYTES + 2 * GV_STAGES * 8 + 64;

DEVI long long cta_of_unit(long long u, long long G, long long TU) { return ((u + 1) * G - 1) / TU; }

template <int NB, int EPI>
__global__ void __launch_bounds__(GV_THREADS, 2)
    gemv_bf16_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                     const __grid_constant__ CUtensorMap tm2, const GemvArgs<__nv_bfloat16> a, int ntiles, int nku,
                     long long TU, int max_pieces) {
    constexpr int NM = NB / 8;   // n8 MMAs per k16 step
    constexpr int FR = 4 * NM;   // accumulator floats per lane
    constexpr int TR = EPI == EPI_SWIGLU ? GV_ROWS / 2 : GV_ROWS;  // logical rows per tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem + GV_STAGES * GV_UNIT_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + GV_STAGES * GV_UNIT_BYTES + GV_XS_BYTES);
    uint64_t* empty = full + GV_STAGES;
    __shared__ float rinv_s[16];
    __shared__ float rred_s[8][16];
    __shared__ int last_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int M = a.M, K = a.K;
    const long long G = gridDim.x;
    const long long u0 = blockIdx.x * TU / G, u1 = (blockIdx.x + 1) * TU / G;

    if (threadIdx.x == 0) {
        for (int i = 0; i < GV_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 8);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tm0);
        tma_prefetch_desc(&tm1);
        tma_prefetch_desc(&tm2);
    }
    __syncthreads();
    pdl_trigger();

    if (warp == 8) {
        // ---------------- producer: weights do not depend on the previous kernel ----
        if (lane == 0) {
            // (tile, k unit) of u tracked incrementally: no division in the loop
            int tile = (int)(u0 / nku), kb = (int)(u0 % nku);
            int st = 0;
            uint32_t ph = 0;
            for (long long u = u0; u < u1; ++u) {
                if (!mbar_wait(&empty[st], ph ^ 1u, a.epi.err, DERR_GEMV_PRODUCER_WAIT)) break;
                const int kx = kb * GV_BK;
                uint8_t* dst = stages + st * GV_UNIT_BYTES;
                mbar_arrive_expect_tx(&full[st], GV_UNIT_BYTES);
                if (EPI == EPI_SWIGLU) {
                    tma_load_2d(dst, &tm0, &full[st], kx, tile * TR);                      // w1 rows
                    tma_load_2d(dst + GV_UNIT_BYTES / 2, &tm1, &full[st], kx, tile * TR);  // w3 rows
                } else {
                    int r = tile * GV_ROWS, sgm = 0;
                    while (sgm < 2 && r >= a.seg_rows[sgm] && a.seg_rows[sgm] > 0) {
                        r -= a.seg_rows[sgm];
                        ++sgm;
                    }
                    tma_load_2d(dst, sgm == 0 ? &tm0 : sgm == 1 ? &tm1 : &tm2, &full[st], kx, r);
                }
                if (++kb == nku) {
                    kb = 0;
                    ++tile;
                }
                if (++st == GV_STAGES) {
                    st = 0;
                    ph ^= 1u;
                }
            }
        }
        pdl_wait();
        return;
    }

    // ---------------- consumers ----------------
    pdl_wait();
    const int Kp = nku * GV_BK;  // K padded to the unit width (the TMA box fills zeros past K)
    const bool x_in_smem = (long long)M * Kp * 2 <= GV_XS_BYTES;
    if (x_in_smem)
        for (int i = threadIdx.x * 8; i < M * Kp; i += 256 * 8) {
            const int m = i / Kp, k = i - m * Kp;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (k < K) v = *reinterpret_cast<const uint4*>(a.x + (size_t)m * a.ldx + k);
            *reinterpret_cast<uint4*>(xs + i) = v;
        }
    {
        // RMSNorm scale of each token row from the producer's partial sums of h^2.
        const NormIn& n = a.epi.norm;
        float part[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) part[m] = 0.f;
        if (n.ss != nullptr)
            for (int p = threadIdx.x; p < n.nparts; p += 256)
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    if (m < M) part[m] += n.ss[(long long)p * n.ld + n.row0 + (long long)(a.m0 + m) * n.row_step];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float v = warp_sum(part[m]);
            if (lane == 0) rred_s[warp][m] = v;
        }
        named_bar_sync(1, 256);
        if (threadIdx.x < 16) {
            float t = 0.f;
            for (int w = 0; w < 8; ++w) t += rred_s[w][threadIdx.x];
            rinv_s[threadIdx.x] = n.ss ? rsqrtf(t * n.inv_dim + n.eps) : 1.f;
        }
        named_bar_sync(1, 256);
    }

    // This warp's two A rows (g and g + 8) inside a stage and their logical rows.
    const int srow0 = EPI == EPI_SWIGLU ? warp * 8 + g : warp * 16 + g;
    const int srow1 = EPI == EPI_SWIGLU ? GV_ROWS / 2 + warp * 8 + g : warp * 16 + g + 8;
    auto lrow = [&](int tile, int which) -> int {
        const int lr = EPI == EPI_SWIGLU ? tile * TR + warp * 8 + g : tile * TR + warp * 16 + g + 8 * which;
        return lr < a.N ? lr : -1;
    };

    const Epi& e = a.epi;
    auto epilogue = [&](int tile, float (&c)[NM][4]) {
        const int lr0 = lrow(tile, 0), lr1 = lrow(tile, 1);
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
                const float r = m < M ? rinv_s[m] : 0.f;
                const float v0 = c[n][h] * r;      // A row g
                const float v1 = c[n][2 + h] * r;  // A row g + 8
                if (EPI == EPI_QKV_ROPE) {
                    // RoPE pairs (2i, 2i+1) sit in A rows g and g^1: lanes lane and lane^4.
                    const float p0 = __shfl_xor_sync(0xffffffffu, v0, 4);
                    const float p1 = __shfl_xor_sync(0xffffffffu, v1, 4);
                    if (m < M && (g & 1) == 0) {
                        const int mg = a.m0 + m;
                        if (lr0 >= 0) epi_qkv_pair<__nv_bfloat16>(e, mg, lr0, v0, p0);
                        if (lr1 >= 0) epi_qkv_pair<__nv_bfloat16>(e, mg, lr1, v1, p1);
                    }
                    continue;
                }
                if (m >= M) continue;
                const int mg = a.m0 + m;
                if (EPI == EPI_STORE_F32) {
                    if (lr0 >= 0) e.y[(size_t)mg * e.ldy + lr0] = v0;
                    if (lr1 >= 0) e.y[(size_t)mg * e.ldy + lr1] = v1;
                } else if (EPI == EPI_SWIGLU) {
                    if (lr0 >= 0)
                        reinterpret_cast<__nv_bfloat16*>(e.g_out)[(size_t)mg * e.F + lr0] =
                            __float2bfloat16_rn(swiglu(v0, v1));
                } else if (EPI == EPI_RESID) {
                    float sq = 0.f;
                    if (lr0 >= 0) {
                        const float hn = epi_resid1<__nv_bfloat16>(e, mg, lr0, v0);
                        sq += hn * hn;
                    }
                    if (lr1 >= 0) {
                        const float hn = epi_resid1<__nv_bfloat16>(e, mg, lr1, v1);
                        sq += hn * hn;
                    }
                    ssum[n][h] = sq;
                } else if (EPI == EPI_LOGITS) {
                    if (lr0 >= 0) {
                        if (e.logits) e.logits[(size_t)m * e.ld_logits + lr0] = v0;
                        am_merge(bv[n][h], bi[n][h], v0, lr0);
                    }
                    if (lr1 >= 0) {
                        if (e.logits) e.logits[(size_t)m * e.ld_logits + lr1] = v1;
                        am_merge(bv[n][h], bi[n][h], v1, lr1);
                    }
                }
            }
        if (EPI == EPI_RESID || EPI == EPI_LOGITS) {
#pragma unroll
            for (int n = 0; n < NM; ++n)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {  // over the 8 row groups g
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
                        if (EPI == EPI_RESID)  // one part per 16 rows, like the other producers of h
                            e.ss_out[(size_t)(tile * 8 + warp) * e.ss_out_ld + a.m0 + m] = ssum[n][h];
                        else if (bi[n][h] != INT_MAX)
                            atomicMax(a.ws.am_best + m, am_key(bv[n][h], bi[n][h]));
                    }
                }
        }
        if (EPI == EPI_LOGITS) {
            // The last of the ntiles * 8 warp epilogues turns the packed maxima into token ids.
            __syncwarp();
            unsigned prev = 0;
            if (lane == 0) {
                __threadfence();
                prev = atomicAdd(a.ws.done_cnt, 1u);
            }
            prev = __shfl_sync(0xffffffffu, prev, 0);
            if (prev == (unsigned)(ntiles * 8 - 1)) {
                __threadfence();
                if (lane < M) {
                    const unsigned long long k = __ldcg(a.ws.am_best + lane);
                    e.next_tok[lane] = am_key_index(k);
                    if (e.seq_len) e.seq_len[lane] += e.advance;
                    a.ws.am_best[lane] = 0ull;
                }
                if (lane == 0) *a.ws.done_cnt = 0u;
            }
        }
    };

    const uint4 z4 = make_uint4(0, 0, 0, 0);
    float c[NM][4];
#pragma unroll
    for (int n = 0; n < NM; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0.f;
    int ctile = (int)(u0 / nku), ckb = (int)(u0 % nku);  // (tile, k unit) of u, tracked incrementally
    int st = 0;
    uint32_t ph = 0;
    const uint32_t xbase = smem_u32(xs);
    for (long long u = u0; u < u1; ++u) {
        if (!mbar_wait(&full[st], ph, a.epi.err, DERR_GEMV_CONSUMER_WAIT)) break;
        const uint32_t sp = smem_u32(stages + st * GV_UNIT_BYTES);
        const int kx = ckb * GV_BK;
        // swizzled 16-byte chunks 2*t4 and 2*t4+1 of rows srow0 and srow1
        const uint32_t a0 = sp + srow0 * 128, a1 = sp + srow1 * 128;
        const int c0 = 2 * t4, c1 = 2 * t4 + 1;
        uint4 w0, w1, w2, w3;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w0.x), "=r"(w0.y), "=r"(w0.z), "=r"(w0.w) : "r"(a0 + ((c0 ^ (srow0 & 7)) << 4)));
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w1.x), "=r"(w1.y), "=r"(w1.z), "=r"(w1.w) : "r"(a0 + ((c1 ^ (srow0 & 7)) << 4)));
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w2.x), "=r"(w2.y), "=r"(w2.z), "=r"(w2.w) : "r"(a1 + ((c0 ^ (srow1 & 7)) << 4)));
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w3.x), "=r"(w3.y), "=r"(w3.z), "=r"(w3.w) : "r"(a1 + ((c1 ^ (srow1 & 7)) << 4)));
        uint4 xa[NM], xb[NM];
        const int k = kx + t4 * 16;
#pragma unroll
        for (int n = 0; n < NM; ++n) {
            const int mrow = g + 8 * n;
            if (x_in_smem) {
                const uint32_t xp = xbase + (uint32_t)(mrow * Kp + k) * 2;
                xa[n] = z4;
                xb[n] = z4;
                if (mrow < M) {
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(xa[n].x), "=r"(xa[n].y), "=r"(xa[n].z), "=r"(xa[n].w) : "r"(xp));
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(xb[n].x), "=r"(xb[n].y), "=r"(xb[n].z), "=r"(xb[n].w) : "r"(xp + 16));
                }
            } else {
                const __nv_bfloat16* xp = a.x + (size_t)mrow * a.ldx + k;
                xa[n] = (mrow < M && k < K) ? *reinterpret_cast<const uint4*>(xp) : z4;
                xb[n] = (mrow < M && k + 8 < K) ? *reinterpret_cast<const uint4*>(xp + 8) : z4;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);  // the stage's data is in registers
        if (++st == GV_STAGES) {
            st = 0;
            ph ^= 1u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t af[4];
            af[0] = w_of(w0, w1, 2 * j);
            af[1] = w_of(w2, w3, 2 * j);
            af[2] = w_of(w0, w1, 2 * j + 1);
            af[3] = w_of(w2, w3, 2 * j + 1);
#pragma unroll
            for (int n = 0; n < NM; ++n)
                mma_bf16_16816(c[n], af, w_of(xa[n], xb[n], 2 * j), w_of(xa[n], xb[n], 2 * j + 1));
        }
        const int tile = ctile;
        if (++ckb == nku) {
            ckb = 0;
            ++ctile;
        }
        if (u + 1 != u1 && ckb != 0) continue;
        // ---- end of this CTA's part of a row tile ----
        const long long tu0 = (long long)tile * nku;
        const long long cf = cta_of_unit(tu0, G, TU), cl = cta_of_unit(tu0 + nku - 1, G, TU);
        if (cf == cl) {
            epilogue(tile, c);
        } else {
            float* base = a.ws.part + (size_t)tile * max_pieces * (8 * 32 * 8);
            float* mine = base + (size_t)(blockIdx.x - cf) * (8 * 32 * 8) + (warp * 32 + lane) * 8;
#pragma unroll
            for (int n = 0; n < NM; ++n)
                *reinterpret_cast<float4*>(mine + 4 * n) = make_float4(c[n][0], c[n][1], c[n][2], c[n][3]);
            __threadfence();
            named_bar_sync(1, 256);
            if (threadIdx.x == 0) {
                const unsigned prev = atomicAdd(a.ws.tile_cnt + tile, 1u);
                last_s = prev == (unsigned)(cl - cf);
                if (last_s) a.ws.tile_cnt[tile] = 0u;
            }
            named_bar_sync(1, 256);
            if (last_s) {
                __threadfence();
                float t[NM][4];
#pragma unroll
                for (int n = 0; n < NM; ++n) t[n][0] = t[n][1] = t[n][2] = t[n][3] = 0.f;
                for (long long p = 0; p <= cl - cf; ++p) {
                    const float* src = base + (size_t)p * (8 * 32 * 8) + (warp * 32 + lane) * 8;
#pragma unroll
                    for (int n = 0; n < NM; ++n) {
                        const float4 v = __ldcg(reinterpret_cast<const float4*>(src + 4 * n));
                        t[n][0] += v.x;
                        t[n][1] += v.y;
                        t[n][2] += v.z;
                        t[n][3] += v.w;
                    }
                }
                epilogue(tile, t);
            }
        }
#pragma unroll
        for (int n = 0; n < NM; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0.f;
    }
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
template <int NB, int EPI>
static cudaError_t launch_bf16_e(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(gemv_bf16_kernel<NB, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, GV_SMEM);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    if (!a.tmw[0]) return cudaErrorInvalidValue;
    const GemvPlan p = gemv_plan(EPI, a.N, a.K, a.num_sms, 1);
    if ((size_t)p.ntiles * p.max_pieces * 8 * 32 * 8 > a.ws.part_floats || p.ntiles > a.ws.tiles_cap)
        return cudaErrorInvalidValue;
    const CUtensorMap& m0 = *a.tmw[0];
    const CUtensorMap& m1 = a.tmw[1] ? *a.tmw[1] : m0;
    const CUtensorMap& m2 = a.tmw[2] ? *a.tmw[2] : m0;
    return launch_k(gemv_bf16_kernel<NB, EPI>, dim3(p.grid), GV_THREADS, GV_SMEM, s, pdl, m0, m1, m2, a, p.ntiles,
                    p.nkb, p.TB, p.max_pieces);
}

template <int NB>
static cudaError_t launch_bf16_nb(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl) {
    switch (a.epi.kind) {
        case EPI_STORE_F32: return launch_bf16_e<NB, EPI_STORE_F32>(a, s, pdl);
        case EPI_QKV_ROPE: return launch_bf16_e<NB, EPI_QKV_ROPE>(a, s, pdl);
        case EPI_SWIGLU: return launch_bf16_e<NB, EPI_SWIGLU>(a, s, pdl);
        case EPI_RESID: return launch_bf16_e<NB, EPI_RESID>(a, s, pdl);
        case EPI_LOGITS: return launch_bf16_e<NB, EPI_LOGITS>(a, s, pdl);
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
    return (size_t)p.ntiles * p.max_pieces * 8 * 32 * 8;
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
