// Building blocks of the streaming bf16 decode projection y[m][n] = sum_k x[m][k] W[n][k]
// (M <= 16 token rows), shared by the single-projection kernel (gemv.cu) and
// the fused decode-step kernel (decode_step.cu).
//
// In the decode phase only the newest token of each sequence is projected ("KV
// cache" on the llama3.np page), so every projection is a matrix-vector product
// bound by the bytes of its weight matrix, which are streamed from HBM once.
//
// Work unit = one 128-row x 64-wide tile of the weight matrix (16 KB, one TMA
// tensor copy with the 128-byte swizzle; for SwiGLU, 64 rows of w1 and the same
// 64 rows of w3). The units of all row tiles, in (row tile, k) order, are split
// into equal contiguous ranges, one per CTA, so every SM streams the same number
// of bytes. One producer warp keeps a shared-memory ring of units full (full /
// empty mbarriers); eight consumer warps each own 16 of a tile's 128 rows and
// consume every unit with mma.sync m16n8k16 (weights as the A operand, token
// rows as B), so no reduction between warps is needed. A row tile whose k range
// is split over several CTAs leaves one partial per CTA, added in CTA order (so
// results are deterministic) by the tile's first CTA, which reaches the tile
// last (at the end of its range): each of its warps waits for the other CTAs'
// pieces of its own 16 rows and runs the fused epilogue. The other CTAs publish
// their pieces and move on. Both kernels that use this are launched
// cooperatively, so every CTA is resident while the first ones wait.
//
// Fragment layout: lane (g = lane/4, t = lane%4) reads 16 contiguous bf16 of its
// rows g and g+8 at k0 + 16t. Because a dot product does not depend on the order
// of k, the fragment's logical k index is mapped onto these physical offsets:
// for the j-th MMA of a 64-wide unit, lane t's logical k pairs (2t, 2t+1) and
// (2t+8, 2t+9) take physical k0 + 16t + 4j + {0,1} and {2,3}. The B operand (x)
// is read with the same map, so the product is unchanged while every shared-
// memory read is a full 16-byte vector.
//
// Activations written earlier in the same launch by other CTAs (x, h, the
// RMSNorm partial sums) are read with ld.global.cg (L2, never a stale L1 line).
//
// Split activations (SPLIT): in decode the producer of x also leaves its bf16
// rounding remainder x_lo = bf16(x - bf16(x)). The B operand then holds 2M
// columns, token m's bf16 part in column 2m and its remainder in column 2m + 1,
// and the epilogue adds the two columns: the product sees x to about 16
// significant bits instead of 8. A matrix-vector product is bound by its weight
// bytes, and the extra columns fit in the MMA tile the tokens already occupy
// (M <= 4) or in a second one (M <= 8), so the weight stream is unchanged.
#pragma once
#include "epilogue.cuh"

#include <float.h>
#include <limits.h>

namespace lfw {

constexpr int GV_ROWS = 128;                      // rows per tile (8 warps x 16)
constexpr int GV_BK = 64;                         // k per unit
constexpr int GV_UNIT_BYTES = GV_ROWS * GV_BK * 2;
constexpr int GV_CONSUMERS = 256;                 // 8 consumer warps; warp 8 is the producer
constexpr int GV_PIECE_FLOATS = 8 * 32 * 8;       // one CTA's partial of a 128-row tile (NB <= 16)

DEVI uint32_t w_of(const uint4& a, const uint4& b, int i) {
    const uint4& v = i < 4 ? a : b;
    const int j = i & 3;
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Order-preserving key of (logit, token id) for a 64-bit atomicMax: a larger
// logit wins, and among equal logits the lower id ("Predicción de tokens": the
// token with the largest logit comes next; ties go to the lowest id).
DEVI unsigned long long am_key(float v, int idx) {
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}
DEVI int am_key_index(unsigned long long k) { return (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull)); }

// Shared-memory ring of weight units. The producer and the consumers each keep
// their own copy of (st, ph) and advance it once per unit, in the same order.
struct GvRing {
    uint8_t* stages;
    uint64_t* full;   // [n] producer -> consumers (one arrival + transaction bytes)
    uint64_t* empty;  // [n] consumers -> producer (8 arrivals, one per consumer warp)
    int n;
    int st;
    uint32_t ph;
    long long issued; // producer: copies issued so far
};
DEVI void ring_next(GvRing& r) {
    if (++r.st == r.n) {
        r.st = 0;
        r.ph ^= 1u;
    }
}

// One projection's unit range for this CTA. The units are split over
// G = min(grid, units) CTAs, so every CTA that takes part has at least one unit
// (CTAs beyond G get none); a row tile's pieces then come from consecutive CTAs.
struct GvWork {
    int ntiles, nku;   // row tiles; 64-wide k units per tile
    long long TU;      // all units
    long long G;       // CTAs taking part
    long long u0, u1;  // this CTA's units
};
DEVI GvWork gv_work(int ntiles, int nku) {
    GvWork w;
    w.ntiles = ntiles;
    w.nku = nku;
    w.TU = (long long)ntiles * nku;
    w.G = (long long)gridDim.x < w.TU ? (long long)gridDim.x : w.TU;
    if (blockIdx.x < w.G) {
        w.u0 = blockIdx.x * w.TU / w.G;
        w.u1 = (blockIdx.x + 1) * w.TU / w.G;
    } else {
        w.u0 = w.u1 = w.TU;
    }
    return w;
}
// CTA whose range holds unit u.
DEVI long long cta_of_unit(long long u, long long G, long long TU) { return ((u + 1) * G - 1) / TU; }

// Producer (one lane): TMA copies of this CTA's units into the ring. For SwiGLU a
// unit is 64 rows of w1 (tm0) and the same rows of w3 (tm1); otherwise it is 128
// rows of the row-wise concatenation of up to three segments of seg0, seg1, ...
// rows (every segment a multiple of 128 rows, so no tile straddles two).
// Returns false if the consumers stopped freeing stages (bounded wait).
DEVI bool gv_produce(GvRing& r, const GvWork& w, bool swiglu, const CUtensorMap* tm0, const CUtensorMap* tm1,
                     const CUtensorMap* tm2, int seg0, int seg1, uint32_t* err, uint32_t code) {
    int tile = (int)(w.u0 / w.nku), kb = (int)(w.u0 % w.nku);  // tracked incrementally: no division in the loop
    for (long long u = w.u0; u < w.u1; ++u) {
        if (!mbar_wait(&r.empty[r.st], r.ph ^ 1u, err, code)) return false;
        uint8_t* dst = r.stages + r.st * GV_UNIT_BYTES;
        const int kx = kb * GV_BK;
        mbar_arrive_expect_tx(&r.full[r.st], GV_UNIT_BYTES);
        if (swiglu) {
            tma_load_2d(dst, tm0, &r.full[r.st], kx, tile * (GV_ROWS / 2));
            tma_load_2d(dst + GV_UNIT_BYTES / 2, tm1, &r.full[r.st], kx, tile * (GV_ROWS / 2));
        } else {
            int row = tile * GV_ROWS;
            const CUtensorMap* m = tm0;
            if (seg0 > 0 && row >= seg0) {
                row -= seg0;
                m = tm1;
                if (seg1 > 0 && row >= seg1) {
                    row -= seg1;
                    m = tm2;
                }
            }
            tma_load_2d(dst, m, &r.full[r.st], kx, row);
        }
        if (++kb == w.nku) {
            kb = 0;
            ++tile;
        }
        ++r.issued;
        ring_next(r);
    }
    return true;
}

// Producer, before it exits: wait (bounded) for the copies of the last
// min(issued, n) units, so no bulk copy is still writing this CTA's shared memory
// when it retires. In a run without errors the consumers have already waited
// for all of them and this returns at once.
DEVI void gv_drain(const GvRing& r, long long issued, uint32_t* err, uint32_t code) {
    int st = r.st;
    uint32_t ph = r.ph;
    for (long long i = 0; i < r.n && i < issued; ++i) {
        if (st == 0) {
            st = r.n - 1;
            ph ^= 1u;
        } else {
            --st;
        }
        mbar_wait(&r.full[st], ph, err, code);
    }
}

// Consumers (256 threads), at the start of a projection: copy the token rows of x
// (row stride ldx, K % 8 == 0) into shared memory (when xs is not null), and
// compute each row's RMSNorm scale from the partial sums of h^2 left by the
// producer of the input (1 where the input is not normed). Every load of the
// first batch is issued before any is used, so the prologue costs about one
// memory round trip. Ends with a barrier of the consumers.
// Only the 64-wide k blocks the CTA's units read are copied, kb0, kb0 + 1, ...
// (wrapping at nku, the blocks of a row), Kp / 64 of them: xs is [rows][Kp] with
// slot s holding k block (kb0 + s) mod nku, zero past K. Every CTA of a launch
// reads its own few blocks, and a range of many token rows still fits.
DEVI void gv_prologue(__nv_bfloat16* xs, const __nv_bfloat16* x, int ldx, int M, int K, int Kp, const NormIn& n,
                      int m0, float* rinv_s, float (*rred_s)[16], int kb0 = 0, int nku = 1 << 30,
                      const __nv_bfloat16* xlo = nullptr) {
    constexpr int XB = 14;  // 16-byte loads per thread per batch: one batch covers the split rows of K = 14336
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // partial sums: the first part of each row, loads only
    float part[16];
    const bool has0 = n.ss != nullptr && (int)threadIdx.x < n.nparts;
#pragma unroll
    for (int m = 0; m < 16; ++m)
        part[m] = (has0 && m < M) ? __ldcg(n.ss + (long long)threadIdx.x * n.ld + n.row0 + (long long)(m0 + m) * n.row_step)
                                  : 0.f;
    // token rows, XB loads in flight per thread
    if (xs != nullptr) {
        const int total = (xlo ? 2 * M : M) * Kp;  // with xlo: row 2m = x[m], row 2m + 1 = xlo[m]
        for (int i0 = threadIdx.x * 8; i0 < total; i0 += GV_CONSUMERS * 8 * XB) {
            uint4 v[XB];
#pragma unroll
            for (int j = 0; j < XB; ++j) {
                const int i = i0 + j * GV_CONSUMERS * 8;
                v[j] = make_uint4(0, 0, 0, 0);
                if (i < total) {
                    const int r = i / Kp, ks = i - r * Kp;
                    int kb = kb0 + ks / GV_BK;
                    if (kb >= nku) kb -= nku;
                    const int k = kb * GV_BK + (ks & (GV_BK - 1));
                    const __nv_bfloat16* src = xlo ? ((r & 1) ? xlo : x) + (size_t)(r >> 1) * ldx : x + (size_t)r * ldx;
                    if (k < K) v[j] = __ldcg(reinterpret_cast<const uint4*>(src + k));
                }
            }
#pragma unroll
            for (int j = 0; j < XB; ++j) {
                const int i = i0 + j * GV_CONSUMERS * 8;
                if (i < total) *reinterpret_cast<uint4*>(xs + i) = v[j];
            }
        }
    }
    // remaining parts
    if (n.ss != nullptr)
        for (int p = threadIdx.x + GV_CONSUMERS; p < n.nparts; p += GV_CONSUMERS)
#pragma unroll
            for (int m = 0; m < 16; ++m)
                if (m < M) part[m] += __ldcg(n.ss + (long long)p * n.ld + n.row0 + (long long)(m0 + m) * n.row_step);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const float v = warp_sum(part[m]);
        if (lane == 0) rred_s[warp][m] = v;
    }
    named_bar_sync(1, GV_CONSUMERS);
    if (threadIdx.x < 16) {
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += rred_s[w][threadIdx.x];
        rinv_s[threadIdx.x] = n.ss ? rsqrtf(t * n.inv_dim + n.eps) : 1.f;
    }
    named_bar_sync(1, GV_CONSUMERS);
}

// Token rows of one projection as the consumers see them.
struct GvX {
    const __nv_bfloat16* x;  // [M][ldx] in global memory
    int ldx, M, K, Kp;       // Kp: the row stride of xs, a whole number of 64-wide k blocks
    const __nv_bfloat16* xs; // [MX][Kp] copy in shared memory, or nullptr
    int kb0 = 0, nku = 1 << 30;  // slot s of xs holds k block (kb0 + s) mod nku
    const __nv_bfloat16* xlo = nullptr;  // split activations: the remainders, [M][ldx]
    int MX = 0;                          // B-operand columns: M, or 2M when split
};

// Operands of a tile's epilogue that live in global memory: for the residual
// epilogue the old h values and the next norm weight of this lane's rows, for the
// QKV epilogue the RoPE cos/sin of its rows at each token's position. They are
// loaded when the tile's first unit is consumed -- only the CTA that holds the
// tile's first unit runs its epilogue -- so they have arrived by the tile's end
// instead of adding dependent L2 round trips to the end of the kernel.
template <int NB>
struct GvEpiOps {
    float a[NB / 8][2][2];  // [n][h][row g / g+8]: residual h, or RoPE cos
    float b[NB / 8][2][2];  // RoPE sin
    float w[2];             // next norm weight of rows g / g+8
};

// Token of accumulator column (n, h): 2t4 + h of n-tile n, or with split
// activations the column pair (2t4, 2t4 + 1) of n-tile n, token n*4 + t4 (h = 0).
template <bool SPLIT>
DEVI int gv_token(int n, int h, int t4) { return SPLIT ? n * 4 + t4 : n * 8 + 2 * t4 + h; }

template <int NB, int EPI, bool SPLIT = false>
DEVI void gv_epi_prefetch(GvEpiOps<NB>& op, int tile, int N, int M, int m0, const Epi& e) {
    if (EPI != EPI_RESID && EPI != EPI_QKV_ROPE) return;
    constexpr int NM = NB / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    int lr[2];
    lr[0] = tile * GV_ROWS + warp * 16 + g;
    lr[1] = lr[0] + 8;
    if (EPI == EPI_RESID) {
#pragma unroll
        for (int q = 0; q < 2; ++q)
            op.w[q] = lr[q] < N ? to_f<__nv_bfloat16>(reinterpret_cast<const __nv_bfloat16*>(e.wnext)[lr[q]]) : 0.f;
    }
#pragma unroll
    for (int n = 0; n < NM; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = gv_token<SPLIT>(n, h, t4);
            const int mg = m0 + m;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                op.a[n][h][q] = 0.f;
                op.b[n][h][q] = 0.f;
                if (SPLIT && h == 1) continue;
                if (m >= M || lr[q] >= N) continue;
                if (EPI == EPI_RESID) {
                    op.a[n][h][q] = __ldcg(e.h + (long long)mg * e.D + lr[q]);
                } else if ((g & 1) == 0 && lr[q] < (e.H + e.Hk) * e.d) {
                    const int bq = mg / e.T;
                    const int pos = e.pos0[bq] + (mg - bq * e.T);
                    if (!LFW_CHECK(pos >= 0 && pos < e.S_max, e.err, BC_ROPE_POS)) continue;
                    const long long ti = (long long)pos * (e.d >> 1) + ((lr[q] % e.d) >> 1);
                    op.a[n][h][q] = e.rope_cos[ti];
                    op.b[n][h][q] = e.rope_sin[ti];
                }
            }
        }
}

// QKV epilogue for one (even, odd) column pair with its RoPE cos/sin given:
// rotate q and k, write q, append k and v to the cache at the token's position
// (as epi_qkv_pair).
DEVI void gv_qkv_pair(const Epi& e, int m, int col, float v0, float v1, float cs, float sn) {
    const int Hd = e.H * e.d, Hkd = e.Hk * e.d;
    const int b = m / e.T;
    const int pos = e.pos0[b] + (m - b * e.T);
    if (!LFW_CHECK(pos >= 0 && pos < e.S_max, e.err, BC_CACHE_POS)) return;
    if (col < Hd + Hkd) {
        const float r0 = v0 * cs - v1 * sn;
        const float r1 = v0 * sn + v1 * cs;
        v0 = r0;
        v1 = r1;
    }
    if (col < Hd) {
        store2<__nv_bfloat16>(reinterpret_cast<__nv_bfloat16*>(e.q_out) + (long long)m * Hd + col, v0, v1);
    } else {
        int cc = col - Hd;
        const bool isv = cc >= Hkd;
        if (isv) cc -= Hkd;
        const int kvh = cc / e.d, dd = cc - kvh * e.d;
        __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(isv ? e.v_cache : e.k_cache);
        store2<__nv_bfloat16>(base + ((long long)(b * e.Hk + kvh) * e.S_max + pos) * e.d + dd, v0, v1);
    }
}

// Fused epilogue of one warp's 16 rows of a finished row tile (accumulators c,
// before the RMSNorm scale; global operands in op).
template <int NB, int EPI, bool SPLIT = false>
DEVI void gv_epilogue(int tile, const float (&c)[NB / 8][4], int N, int M, int m0, const float* rinv_s, const Epi& e,
                      const GemvScratch& ws, int ntiles, const GvEpiOps<NB>& op) {
    constexpr int NM = NB / 8;
    constexpr int TR = EPI == EPI_SWIGLU ? GV_ROWS / 2 : GV_ROWS;  // logical rows per tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    auto lrow = [&](int which) -> int {
        const int lr = EPI == EPI_SWIGLU ? tile * TR + warp * 8 + g : tile * TR + warp * 16 + g + 8 * which;
        return lr < N ? lr : -1;
    };
    const int lr0 = lrow(0), lr1 = lrow(1);
    float ssum[NM][2];
    float bv[NM][2];
    int bi[NM][2];
#pragma unroll
    for (int n = 0; n < NM; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = gv_token<SPLIT>(n, h, t4);
            ssum[n][h] = 0.f;
            bv[n][h] = -FLT_MAX;
            bi[n][h] = INT_MAX;
            if (SPLIT && h == 1) continue;  // (uniform over the warp)
            const float r = m < M ? rinv_s[m] : 0.f;
            const float v0 = (SPLIT ? c[n][0] + c[n][1] : c[n][h]) * r;          // A row g
            const float v1 = (SPLIT ? c[n][2] + c[n][3] : c[n][2 + h]) * r;      // A row g + 8
            if (EPI == EPI_QKV_ROPE) {
                // RoPE pairs (2i, 2i+1) sit in A rows g and g^1: lanes lane and lane^4.
                const float p0 = __shfl_xor_sync(0xffffffffu, v0, 4);
                const float p1 = __shfl_xor_sync(0xffffffffu, v1, 4);
                if (m < M && (g & 1) == 0) {
                    const int mg = m0 + m;
                    if (lr0 >= 0) gv_qkv_pair(e, mg, lr0, v0, p0, op.a[n][h][0], op.b[n][h][0]);
                    if (lr1 >= 0) gv_qkv_pair(e, mg, lr1, v1, p1, op.a[n][h][1], op.b[n][h][1]);
                }
                continue;
            }
            if (m >= M) continue;
            const int mg = m0 + m;
            if (EPI == EPI_STORE_F32) {
                if (lr0 >= 0) e.y[(size_t)mg * e.ldy + lr0] = v0;
                if (lr1 >= 0) e.y[(size_t)mg * e.ldy + lr1] = v1;
            } else if (EPI == EPI_SWIGLU) {
                if (lr0 >= 0) {
                    const float gv = swiglu(v0, v1);
                    const __nv_bfloat16 hi = __float2bfloat16_rn(gv);
                    reinterpret_cast<__nv_bfloat16*>(e.g_out)[(size_t)mg * e.F + lr0] = hi;
                    if (e.g_lo_out)
                        reinterpret_cast<__nv_bfloat16*>(e.g_lo_out)[(size_t)mg * e.F + lr0] =
                            __float2bfloat16_rn(gv - __bfloat162float(hi));
                }
            } else if (EPI == EPI_RESID) {
                // residual add and the next norm's input hw = h * w (as epi_resid1,
                // with h and w from the prefetch), and its remainder when asked
                float sq = 0.f;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int lr = q ? lr1 : lr0;
                    if (lr < 0) continue;
                    const float hn = op.a[n][h][q] + (q ? v1 : v0);
                    e.h[(long long)mg * e.D + lr] = hn;
                    const float xw = hn * op.w[q];
                    const __nv_bfloat16 hi = __float2bfloat16_rn(xw);
                    reinterpret_cast<__nv_bfloat16*>(e.hw_out)[(long long)mg * e.D + lr] = hi;
                    if (e.hw_lo_out)
                        reinterpret_cast<__nv_bfloat16*>(e.hw_lo_out)[(long long)mg * e.D + lr] =
                            __float2bfloat16_rn(xw - __bfloat162float(hi));
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
                if (SPLIT && h == 1) continue;
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
                const int m = gv_token<SPLIT>(n, h, t4);
                if (g == 0 && m < M) {
                    if (EPI == EPI_RESID)  // one part per 16 rows
                        e.ss_out[(size_t)(tile * 8 + warp) * e.ss_out_ld + m0 + m] = ssum[n][h];
                    else if (bi[n][h] != INT_MAX)
                        atomicMax(ws.am_best + m, am_key(bv[n][h], bi[n][h]));
                }
            }
    }
    if (EPI == EPI_LOGITS) {
        // The last of the ntiles * 8 warp epilogues turns the packed maxima into
        // token ids and advances the cache lengths.
        __syncwarp();
        unsigned prev = 0;
        if (lane == 0) {
            __threadfence();
            prev = atomicAdd(ws.done_cnt, 1u);
        }
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == (unsigned)(ntiles * 8 - 1)) {
            __threadfence();
            if (lane < M) {
                const unsigned long long k = __ldcg(ws.am_best + lane);
                e.next_tok[lane] = am_key_index(k);
                if (e.seq_len && LFW_CHECK(e.seq_len[lane] + e.advance <= e.S_max || e.S_max == 0, e.err,
                                           BC_SEQ_ADVANCE))
                    e.seq_len[lane] += e.advance;
                ws.am_best[lane] = 0ull;
            }
            if (lane == 0) *ws.done_cnt = 0u;
        }
    }
}

// Consumers (256 threads): this CTA's units of one projection, with the split-
// tile reduction and the epilogues. A failed (timed-out) wait is recorded in
// *err; the warp then stops waiting and runs the rest of its control flow on
// whatever the stage holds, so every consumer warp still reaches every barrier.
template <int NB, int EPI, bool SPLIT = false>
DEVI bool gv_consume(GvRing& r, const GvWork& w, const GvX& X, int N, int m0, const float* rinv_s, const Epi& e,
                     const GemvScratch& ws, int max_pieces, uint32_t* err, uint32_t code) {
    constexpr int NM = NB / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int M = X.M, K = X.K;
    const int MX = SPLIT ? 2 * M : M;  // B-operand columns
    const long long G = w.G;
    bool ok = true;
    // this warp's two A rows (g and g + 8) inside a stage
    const int srow0 = EPI == EPI_SWIGLU ? warp * 8 + g : warp * 16 + g;
    const int srow1 = EPI == EPI_SWIGLU ? GV_ROWS / 2 + warp * 8 + g : warp * 16 + g + 8;
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    float c[NM][4];
#pragma unroll
    for (int n = 0; n < NM; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0.f;
    int ctile = (int)(w.u0 / w.nku), ckb = (int)(w.u0 % w.nku);
    const uint32_t xbase = X.xs ? smem_u32(X.xs) : 0u;
    GvEpiOps<NB> ops;
    for (long long u = w.u0; u < w.u1; ++u) {
        // this CTA holds the tile's first unit, so it runs the tile's epilogue
        if (ckb == 0) gv_epi_prefetch<NB, EPI, SPLIT>(ops, ctile, N, M, m0, e);
        if (ok && !mbar_wait(&r.full[r.st], r.ph, err, code)) ok = false;
        const uint32_t sp = smem_u32(r.stages + r.st * GV_UNIT_BYTES);
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
            if (X.xs) {
                int slot = kx / GV_BK - X.kb0;
                if (slot < 0) slot += X.nku;
                const uint32_t xp = xbase + (uint32_t)(mrow * X.Kp + slot * GV_BK + t4 * 16) * 2;
                xa[n] = z4;
                xb[n] = z4;
                if (mrow < MX) {
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(xa[n].x), "=r"(xa[n].y), "=r"(xa[n].z), "=r"(xa[n].w) : "r"(xp));
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(xb[n].x), "=r"(xb[n].y), "=r"(xb[n].z), "=r"(xb[n].w) : "r"(xp + 16));
                }
            } else {
                const __nv_bfloat16* xp = (SPLIT ? ((mrow & 1) ? X.xlo : X.x) + (size_t)(mrow >> 1) * X.ldx
                                                 : X.x + (size_t)mrow * X.ldx) + k;
                xa[n] = (mrow < MX && k < K) ? __ldcg(reinterpret_cast<const uint4*>(xp)) : z4;
                xb[n] = (mrow < MX && k + 8 < K) ? __ldcg(reinterpret_cast<const uint4*>(xp + 8)) : z4;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&r.empty[r.st]);  // the stage's data is in registers
        ring_next(r);
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
        if (++ckb == w.nku) {
            ckb = 0;
            ++ctile;
        }
        if (u + 1 != w.u1 && ckb != 0) continue;
        // ---- end of this CTA's part of a row tile ----
        const long long tu0 = (long long)tile * w.nku;
        const long long cf = cta_of_unit(tu0, G, w.TU), cl = cta_of_unit(tu0 + w.nku - 1, G, w.TU);
        if (cf == cl) {
            gv_epilogue<NB, EPI, SPLIT>(tile, c, N, M, m0, rinv_s, e, ws, w.ntiles, ops);
        } else {
            // Every CTA of the tile but the first publishes its piece, one warp's rows
            // at a time; the first CTA's warps wait for their rows' pieces.
            float* base = ws.part + (size_t)tile * max_pieces * GV_PIECE_FLOATS + (warp * 32 + lane) * 8;
            unsigned* cnt = ws.warp_cnt + tile * 8 + warp;
            const long long pc = blockIdx.x - cf;
            if (pc != 0) {
                float* mine = base + (size_t)pc * GV_PIECE_FLOATS;
#pragma unroll
                for (int n = 0; n < NM; ++n)
                    *reinterpret_cast<float4*>(mine + 4 * n) = make_float4(c[n][0], c[n][1], c[n][2], c[n][3]);
                __syncwarp();
                if (lane == 0) red_release_add(cnt, 1u);
                __syncwarp();
            } else {
                if (lane == 0) {
                    const unsigned want = (unsigned)(cl - cf);
                    if (ok && ld_acquire_gpu(cnt) < want) {
                        const uint64_t t0 = globaltimer();
                        while (ld_acquire_gpu(cnt) < want) {
                            if (globaltimer() - t0 > kWaitLimitNs) {
                                atomicCAS(err, 0u, code);
                                break;
                            }
                        }
                    }
                    *cnt = 0u;
                }
                __syncwarp();
                float t[NM][4];
#pragma unroll
                for (int n = 0; n < NM; ++n) t[n][0] = c[n][0], t[n][1] = c[n][1], t[n][2] = c[n][2], t[n][3] = c[n][3];
                for (long long p = 1; p <= cl - cf; ++p) {
                    const float* src = base + (size_t)p * GV_PIECE_FLOATS;
#pragma unroll
                    for (int n = 0; n < NM; ++n) {
                        const float4 v = __ldcg(reinterpret_cast<const float4*>(src + 4 * n));
                        t[n][0] += v.x;
                        t[n][1] += v.y;
                        t[n][2] += v.z;
                        t[n][3] += v.w;
                    }
                }
                gv_epilogue<NB, EPI, SPLIT>(tile, t, N, M, m0, rinv_s, e, ws, w.ntiles, ops);
            }
        }
#pragma unroll
        for (int n = 0; n < NM; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0.f;
    }
    return ok;
}

}  // namespace lfw
