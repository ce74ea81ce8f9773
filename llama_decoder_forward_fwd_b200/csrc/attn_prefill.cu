// Causal grouped-query attention for a block of prompt tokens (prefill), on the
// 5th-generation tensor cores.
//
// What it computes ("Resumen ...", "Implementación de la atención" and
// "Atención multi-head"; llama3.np, "GQA" and "Scaled Dot-Product Attention"):
// for query head h of the token at position p, scores q.k_j / sqrt(d) over keys
// j <= p of KV head h / G (G = n_heads / n_kv_heads), future keys masked, softmax,
// weighted sum of values, heads concatenated.
//
// Layout of the work. A work item is 128 "rows" of one (sequence, KV head): row r
// is (token t = r / G, query head kvh*G + r % G), so the G query heads that share a
// KV head sit together and every K/V tile is loaded once for all of them. The
// kernel is persistent (one CTA per SM, TMEM allocated once): each CTA runs a
// fixed sequence of items, longest causal rows first, and every role walks the
// same sequence, so the barrier phases follow one running tile count. Keys go in
// tiles of 128, d = 128. Eleven warps:
//   warps 0, 10  TMA producers, one thread each: K tiles (warp 0) and V tiles
//              (warp 10), two 64-dim halves in the 128-byte swizzle, from the KV
//              cache into 2-stage rings with their own barriers;
//   warp 1     allocates 512 TMEM columns and issues tcgen05.mma from one thread:
//              S = Q K^T (M = 128 rows, N = 128 keys, K = d) into one of two S
//              accumulators, and O += P V (N = d, K = keys; P read from tensor
//              memory, V from shared memory MN-major, as it lies in the cache) into
//              the O accumulator;
//   warps 2-9  softmax, two threads per row (its TMEM lane), 64 keys each:
//              tcgen05.ld of the row of S, causal mask, the row's maximum (shared
//              between the pair through shared memory), P = 2^(s - m) in the log2
//              domain stored with tcgen05.st to tensor memory in bf16 (two buffers)
//              as the A operand of the PV product, partial sums; at the end
//              tcgen05.ld of O / sum.
// Keeping P in tensor memory leaves shared memory to the Q, K and V operands and the
// TMA writes (160 KB a tile instead of 224 with P there).
// The MMA thread issues S for tile j+2 as soon as P of tile j is written, and the
// softmax of tile j+1 does not wait for PV of tile j (unless O must be rescaled),
// so the tensor cores and the softmax warps work at the same time.
// The softmax warps stage the next item's query rows (in the swizzled layout, one
// memory round trip) once they have released P of the item's last tile, while that
// PV product runs, so the MMA thread starts the next item's S products while they
// write out O.
// O is rescaled (tcgen05.ld, scale, tcgen05.st) only when a row's maximum grows
// by more than 2^8 over the maximum its P values were taken against (the
// conditional rescaling of FlashAttention-4): P stays below 256, exact in the
// final normalisation, which divides by a sum taken against the same maximum.
#include "common.cuh"
#include "kernels.cuh"

#include <math.h>

namespace lfw {

constexpr int FA_THREADS = 352;
constexpr int FA_V_WARP = 10;                   // the V producer
constexpr int FA_ROWS = 128;
constexpr int FA_KT = 128;                      // keys per tile
constexpr int FA_D = 128;
constexpr int FA_HALF = 128 * 128;              // [128 rows][64 bf16]: 16 KB
constexpr int FA_TILE = 2 * FA_HALF;            // a K, V, Q or P tile: 32 KB
constexpr int FA_SMEM = 1024 + 5 * FA_TILE + 256 + 1024;  // K, V (2 stages each), Q, barriers, row sums
constexpr uint32_t FA_TMEM_COLS = 512;          // S (2 x 128 columns), O (128), P (2 x 64)
constexpr uint32_t FA_TMEM_O = 256;
constexpr uint32_t FA_TMEM_P = 384;             // P in bf16, two keys per column, two buffers of 64
constexpr float FA_RESCALE_LOG2 = 8.f;

// 2^x by the special-function unit (ex2.approx, flush-to-zero): relative error of
// a few ulp, far below the bf16 rounding that P gets next; 2^-inf = +0.
DEVI float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe, for a share of the elements so that the special-function
// unit is not the only one computing exponentials, two values at a time with the
// packed fp32 operations of sm_100 (one instruction per pair): x = n + f with n the
// nearest integer (added to the exponent field) and f in [-0.5, 0.5], 2^f by a
// cubic fitted to minimise the relative error (at most 1.5e-4 in fp32 arithmetic,
// far below the bf16 rounding P gets next). x is clamped at -126, so a masked
// score gives 2^-126 instead of 0: nothing at the scale of the row's sum.
DEVI float2 ex2_poly2(float2 x) {
    x.x = fmaxf(x.x, -126.f);
    x.y = fmaxf(x.y, -126.f);
    // 1.5 * 2^23: n lands in the low mantissa bits of t
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
    const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);  // x - n, exact as a subtraction
    float2 p = __ffma2_rn(make_float2(0.05517166f, 0.05517166f), f, make_float2(0.24261114f, 0.24261114f));
    p = __ffma2_rn(p, f, make_float2(0.69326097f, 0.69326097f));
    p = __ffma2_rn(p, f, make_float2(0.99992806f, 0.99992806f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// max(a, b, c) in one instruction (three-input max of sm_100).
DEVI float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// D (+)= A B with A in tensor memory (M = 128 rows in the lanes, two bf16 of a row
// per 32-bit column along K) and B described in shared memory.
DEVI void tc_mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// A work item: the 128 rows of one (sequence, KV head) starting at row0.
struct FaItem {
    int b, kvh, row0, p0, nkt;
    long long kv_row0;  // cache row of this (sequence, KV head)'s position 0
};

__global__ void __launch_bounds__(FA_THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const AttnPrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // V stages sit below Q, so every operand read stays inside the allocation.
    uint8_t* Ks = smem;                  // 2 stages
    uint8_t* Vs = smem + 2 * FA_TILE;    // 2 stages
    uint8_t* Qs = smem + 4 * FA_TILE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 5 * FA_TILE);
    float* lsum = reinterpret_cast<float*>(smem + 5 * FA_TILE + 256);  // [half][row]: the pair's row sums
    uint64_t* k_full = bars;
    uint64_t* k_empty = bars + 2;
    uint64_t* v_full = bars + 4;
    uint64_t* v_empty = bars + 6;
    uint64_t* s_full = bars + 8;
    uint64_t* p_full = bars + 10;
    uint64_t* pv_done = bars + 12;
    uint64_t* q_full = bars + 14;    // the next item's Q is staged (items after the first)
    uint64_t* mma_done = bars + 15;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
    // [tile parity][half][row]: the pair's partial maxima, in fp16 (both threads take
    // the maximum of the two rounded values, so they agree on it; the maximum only
    // offsets the exponent)
    __shared__ __half red_max[2][2][FA_ROWS];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.H / a.Hk;
    const int nbh = a.B * a.Hk;
    const int nrb = (a.T * G + FA_ROWS - 1) / FA_ROWS;
    const int total = nrb * nbh;
    uint32_t* err = a.err;

    // Items are numbered longest causal rows first (item k: row block nrb-1-k/nbh of
    // (sequence, KV head) k % nbh); CTA c takes items c, 2g-1-c, 2g+c, ... (g CTAs),
    // which balances the rows' lengths over the CTAs.
    auto item_of = [&](int ki) -> int {
        const int k = ki * (int)gridDim.x + ((ki & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
        return k < total ? k : -1;
    };
    auto describe = [&](int k) -> FaItem {
        FaItem it;
        const int bh = k % nbh;
        it.b = bh / a.Hk;
        it.kvh = bh % a.Hk;
        it.row0 = (nrb - 1 - k / nbh) * FA_ROWS;
        it.p0 = a.pos0[it.b];
        const int t_last = min(a.T - 1, (it.row0 + FA_ROWS - 1) / G);
        const int p_max = min(it.p0 + t_last, a.S_max - 1);  // the last key any row of the item sees
        it.nkt = max(p_max, 0) / FA_KT + 1;
        it.kv_row0 = a.row_base + (long long)(it.b * a.Hk + it.kvh) * a.S_max;
        return it;
    };
    auto load_kv = [&](uint8_t* dst, const CUtensorMap* tm, uint64_t* bar, long long kv_row0, int j) {
        const int y = (int)(kv_row0 + (long long)j * FA_KT);
        mbar_arrive_expect_tx(bar, FA_TILE);
        for (int h = 0; h < 2; ++h)
            for (int kb = 0; kb < 2; ++kb) tma_load_2d(dst + h * FA_HALF + kb * (FA_HALF / 2), tm, bar, h * 64, y + kb * 64);
    };
    // Stage an item's 128 query rows as the A operand of S = Q K^T: two 64-dim
    // halves of [128 rows][128 bytes], 16-byte chunks XOR-swizzled by row; 16 loads
    // per thread are in flight before any is stored.
    auto stage_q = [&](const FaItem& it, int tid, int nthr) {
        constexpr int QB = 16;
        for (int base = tid; base < FA_ROWS * 16; base += nthr * QB) {
            uint4 v[QB];
#pragma unroll
            for (int i = 0; i < QB; ++i) {
                const int idx = base + i * nthr;
                const int r = idx >> 4, c = idx & 15;
                const int rg = it.row0 + r;
                const int t = rg / G, h = it.kvh * G + (rg - t * G);
                v[i] = make_uint4(0, 0, 0, 0);
                if (idx < FA_ROWS * 16 && t < a.T)
                    v[i] = __ldcg(reinterpret_cast<const uint4*>(a.q + ((long long)(it.b * a.T + t) * a.H + h) * FA_D + c * 8));
            }
#pragma unroll
            for (int i = 0; i < QB; ++i) {
                const int idx = base + i * nthr;
                const int r = idx >> 4, c = idx & 15;
                if (idx < FA_ROWS * 16)
                    *reinterpret_cast<uint4*>(Qs + (c >> 3) * FA_HALF + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = v[i];
            }
        }
    };

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 256);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(q_full, 256);
        mbar_init(mma_done, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tc_alloc(tmem_slot, FA_TMEM_COLS);
        tc_relinquish();
    }

    pdl_trigger();
    pdl_wait();
    // The first item: the producer issues its first two K and V tiles (the stages are
    // free), then every thread helps to stage its Q.
    const FaItem it0 = describe(item_of(0));  // the grid never exceeds the items
    if (warp == 0 && lane == 0) {
        for (int j = 0; j < 2 && j < it0.nkt; ++j) {
            load_kv(Ks + j * FA_TILE, &tmK, &k_full[j], it0.kv_row0, j);
            load_kv(Vs + j * FA_TILE, &tmV, &v_full[j], it0.kv_row0, j);
        }
    }
    stage_q(it0, threadIdx.x, FA_THREADS);
    fence_proxy_async();  // the tensor cores read Q through the async proxy
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 || warp == FA_V_WARP) {
        // ---------------- producers: K tiles (warp 0) and V tiles (the last warp) ----------------
        // Each ring has its own thread, so a K tile is requested as soon as its stage
        // is free (the S product two tiles back is complete), not after the V tile
        // ahead of it, whose stage frees only when a PV product completes.
        const bool is_v = warp == FA_V_WARP;
        uint8_t* ring = is_v ? Vs : Ks;
        const CUtensorMap* tm = is_v ? &tmV : &tmK;
        uint64_t* full = is_v ? v_full : k_full;
        uint64_t* empty = is_v ? v_empty : k_empty;
        int last[2] = {it0.nkt > 0 ? 0 : -1, it0.nkt > 1 ? 1 : -1};  // last running tile loaded per stage
        bool ok = true;
        int g = 0;  // running tile index over this CTA's items
        for (int ki = 0; ok; ++ki) {
            const int k = item_of(ki);
            if (k < 0) break;
            const FaItem it = describe(k);
            if (lane == 0 && !is_v) (void)LFW_CHECK(it.p0 >= 0 && it.p0 + a.T <= a.S_max, err, BC_ATTN_POS);
            const int j0 = ki == 0 ? min(2, it.nkt) : 0;
            if (lane == 0) {
                for (int j = j0; j < it.nkt && ok; ++j) {
                    const int gg = g + j, st = gg & 1;
                    if (!mbar_wait(&empty[st], ((gg >> 1) & 1) ^ 1u, err, DERR_ATTN_TMA_WAIT)) {
                        ok = false;
                        break;
                    }
                    load_kv(ring + st * FA_TILE, tm, &full[st], it.kv_row0, j);
                    last[st] = gg;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            g += it.nkt;
        }
        if (!ok && lane == 0) {
            // let copies already issued land before the CTA can exit
            for (int st = 0; st < 2; ++st)
                if (last[st] >= 0) mbar_wait(&full[st], (last[st] >> 1) & 1, nullptr, 0);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(FA_ROWS, FA_KT);
            constexpr uint32_t idO = idesc_bf16_f32_bmn(FA_ROWS, FA_D);
            const uint32_t qa = smem_u32(Qs);
            auto issue_s = [&](int gg) -> bool {
                const int st = gg & 1;
                if (!mbar_wait(&k_full[st], (gg >> 1) & 1, err, DERR_ATTN_MMA_WAIT)) return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(Ks + st * FA_TILE);
#pragma unroll
                for (int kk = 0; kk < FA_D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * FA_HALF + (kk & 3) * 32;
                    tc_mma_f16(tmem_base + st * FA_KT, smem_desc_sw128(qa + off), smem_desc_sw128(ka + off), idS,
                               kk != 0);
                }
                tc_commit(&k_empty[st]);
                tc_commit(&s_full[st]);
                return true;
            };
            bool ok = true;
            int g = 0;
            for (int ki = 0; ok; ++ki) {
                const int k = item_of(ki);
                if (k < 0) break;
                const int nkt = describe(k).nkt;
                if (ki > 0 && !mbar_wait(q_full, (ki - 1) & 1, err, DERR_ATTN_MMA_WAIT)) break;
                tc_fence_after();
                ok = issue_s(g);
                if (ok && nkt > 1) ok = issue_s(g + 1);
                for (int j = 0; j < nkt && ok; ++j) {
                    const int gg = g + j, st = gg & 1;  // K/V stage, S accumulator and P buffer
                    if (!mbar_wait(&p_full[st], (gg >> 1) & 1, err, DERR_ATTN_MMA_WAIT)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&v_full[st], (gg >> 1) & 1, err, DERR_ATTN_MMA_WAIT)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t va = smem_u32(Vs + st * FA_TILE), pj = tmem_base + FA_TMEM_P + st * 64;
#pragma unroll
                    for (int kk = 0; kk < FA_KT / 16; ++kk) {
                        // A = P from TMEM: keys 16kk.. are columns 8kk.. of the P buffer; B = V:
                        // the same 16 key rows, all 128 dims (the second 64-dim half FA_HALF
                        // bytes on). The item's first product overwrites O: the softmax
                        // threads read the previous item's O before they released this P.
                        tc_mma_f16_ta(tmem_base + FA_TMEM_O, pj + kk * 8, smem_desc_sw128_mn(va + kk * 2048, FA_HALF),
                                      idO, (j | kk) != 0);
                    }
                    tc_commit(&v_empty[st]);
                    tc_commit(&pv_done[st]);
                    if (j + 2 < nkt) ok = issue_s(gg + 2);
                }
                g += nkt;
            }
            tc_commit(mma_done);  // arrives once every MMA issued above has completed
        }
    } else {
        // ---------------- softmax (warps 2..9): two threads per row ----------------
        // Warps w and w+4 share TMEM lane quarter w % 4 (the rows); the first takes
        // keys 0..63 of each tile, the second keys 64..127. They agree on the row's
        // maximum through shared memory and keep their own partial sums, added at
        // the end through two free TMEM columns.
        const int q4 = warp & 3;             // the TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;    // which 64 keys of a tile, and 64 dims of O
        const int r = q4 * 32 + lane;
        const uint32_t lane_base = tmem_base + ((uint32_t)(q4 * 32) << 16);
        const float sl2 = a.scale_log2;
        bool ok = true;
        int g = 0;
        for (int ki = 0;; ++ki) {
            const int k = item_of(ki);
            if (k < 0) break;
            const FaItem it = describe(k);
            const int rg = it.row0 + r;
            const int t = rg / G, h = it.kvh * G + (rg - t * G);
            const int prow = t < a.T ? it.p0 + t : -1;
            float m_used = -INFINITY, l = 0.f;   // m_used in the log2 domain
            for (int j = 0; j < it.nkt; ++j) {
                const int gg = g + j, sb = gg & 1;
                if (ok && !mbar_wait(&s_full[sb], (gg >> 1) & 1, err, DERR_ATTN_SOFTMAX_WAIT)) ok = false;
                tc_fence_after();
                float s[64];
                {
                    uint32_t u[2][32];
#pragma unroll
                    for (int c = 0; c < 2; ++c) tc_ld_32x32b_x32(lane_base + sb * FA_KT + half * 64 + c * 32, u[c]);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(u[c][i]);
                }
                // raw maximum (the scale is positive), four independent chains
                const int key0 = j * FA_KT + half * 64;
                if (key0 + 63 > prow) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (key0 + i > prow) s[i] = -INFINITY;
                }
                float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
                for (int i = 4; i < 64; i += 2) mx4[(i >> 1) & 3] = fmax3(mx4[(i >> 1) & 3], s[i], s[i + 1]);
                const __half mine = __float2half_ru(fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2);
                red_max[sb][half][r] = mine;
                named_bar_sync(1 + q4, 64);
                const float mx = fmaxf(__half2float(mine), __half2float(red_max[sb][half ^ 1][r]));
                const float m_new = fmaxf(m_used, mx);
                const bool need = m_new > m_used + FA_RESCALE_LOG2;  // false while the row has seen no key
                const float alpha = need ? ex2_approx(m_used - m_new) : 1.f;
                // P buffer sb is free once PV of running tile gg-2 has completed
                if (gg >= 2 && ok && !mbar_wait(&pv_done[sb], ((gg - 2) >> 1) & 1, err, DERR_ATTN_SOFTMAX_WAIT))
                    ok = false;
                if (j > 0 && __any_sync(0xffffffffu, need)) {
                    // rescale this thread's 64 dims of O: PV of the previous tile has
                    // completed, PV of this one waits for this P
                    const int pg = gg - 1;
                    if (ok && !mbar_wait(&pv_done[pg & 1], (pg >> 1) & 1, err, DERR_ATTN_SOFTMAX_WAIT)) ok = false;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 2; ++c) {
                        uint32_t u[32];
                        tc_ld_32x32b_x32(lane_base + FA_TMEM_O + half * 64 + c * 32, u);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const float2 o = __fmul2_rn(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                                                        make_float2(alpha, alpha));
                            u[i] = __float_as_uint(o.x);
                            u[i + 1] = __float_as_uint(o.y);
                        }
                        tc_st_32x32b_x32(lane_base + FA_TMEM_O + half * 64 + c * 32, u);
                    }
                    tc_wait_st();
                }
                if (need) {
                    l *= alpha;
                    m_used = m_new;
                }
                const float muse = m_used == -INFINITY ? 0.f : m_used;
                // scores to exponents, exponentials and partial sums on pairs of keys
                // (packed fp32: one instruction per pair)
                const float2 sl2x2 = make_float2(sl2, sl2), nmx2 = make_float2(-muse, -muse);
                float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                uint32_t pw[32];  // this thread's 64 keys of P in bf16 pairs: TMEM columns of its lane
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float2 p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __ffma2_rn(make_float2(s[c * 8 + 2 * e], s[c * 8 + 2 * e + 1]), sl2x2, nmx2);
                        // a quarter of the exponentials on the FMA pipe
                        p[e] = e < 3 ? make_float2(ex2_approx(x.x), ex2_approx(x.y)) : ex2_poly2(x);
                        sum2[e & 1] = __fadd2_rn(sum2[e & 1], p[e]);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) pw[c * 4 + e] = pack_bf16x2(p[e].x, p[e].y);
                }
                l += (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
                // P buffer sb in TMEM: the A operand of the PV product (row = lane, key
                // pairs along the columns)
                tc_st_32x32b_x32(lane_base + FA_TMEM_P + sb * 64 + half * 32, pw);
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[sb]);
            }
            {
                // the item's last S product is complete, so Q is free: stage the next
                // item's query rows while PV of the last tile runs; the MMA thread then
                // starts the next item's S products while this item's output is written
                const int kn = item_of(ki + 1);
                if (kn >= 0) {
                    stage_q(describe(kn), threadIdx.x - 64, 256);
                    fence_proxy_async();
                    mbar_arrive(q_full);
                }
            }
            // PV of the item's last tile (and so every earlier one) has completed
            const int gl = g + it.nkt - 1;
            if (ok && !mbar_wait(&pv_done[gl & 1], (gl >> 1) & 1, err, DERR_ATTN_SOFTMAX_WAIT)) ok = false;
            tc_fence_after();
            // the row's sum is the two halves' sums (both taken against the same
            // maximum), exchanged through shared memory (the partner reads the value
            // before the next tile's barrier, so one slot per half suffices)
            lsum[half * FA_ROWS + r] = l;
            named_bar_sync(1 + q4, 64);
            l += lsum[(half ^ 1) * FA_ROWS + r];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* dst = a.out + ((long long)(it.b * a.T + t) * a.H + h) * FA_D + half * 64;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                uint32_t u[32];
                tc_ld_32x32b_x32(lane_base + FA_TMEM_O + half * 64 + c * 32, u);
                tc_wait_ld();
                if (prow >= 0) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        const uint4 v = make_uint4(pack_bf16x2(__uint_as_float(u[i]) * inv, __uint_as_float(u[i + 1]) * inv),
                                                   pack_bf16x2(__uint_as_float(u[i + 2]) * inv, __uint_as_float(u[i + 3]) * inv),
                                                   pack_bf16x2(__uint_as_float(u[i + 4]) * inv, __uint_as_float(u[i + 5]) * inv),
                                                   pack_bf16x2(__uint_as_float(u[i + 6]) * inv, __uint_as_float(u[i + 7]) * inv));
                        *reinterpret_cast<uint4*>(dst + c * 32 + i) = v;
                    }
                }
            }
            g += it.nkt;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        // every MMA has completed before the accumulators are freed
        if (lane == 0) mbar_wait(mma_done, 0, err, DERR_ATTN_MMA_WAIT);
        __syncwarp();
        tc_fence_after();
        tc_dealloc(tmem_base, FA_TMEM_COLS);
    }
}

cudaError_t launch_attn_prefill(const AttnPrefillArgs& a, cudaStream_t s, bool pdl) {
    if (a.H % a.Hk != 0 || a.T < 1) return cudaErrorInvalidValue;
    const int G = a.H / a.Hk;
    const long long items = (long long)((a.T * G + FA_ROWS - 1) / FA_ROWS) * a.B * a.Hk;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    // persistent: one CTA per SM (the shared memory allows no second), never more CTAs than items
    const int sms = current_num_sms();
    const dim3 grid((unsigned)(items < sms ? items : sms));
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM);
    if (e != cudaSuccess) return e;
    return launch_k(attn_prefill_kernel, grid, dim3(FA_THREADS), FA_SMEM, s, pdl, *a.tmK, *a.tmV, a);
}

}  // namespace lfw
