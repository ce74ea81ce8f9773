// Decode attention streamed in 32-key units through the fused decode step's
// shared-memory ring (decode_step.cu).
//
// A unit is the K and V tiles of 32 consecutive keys of one (sequence, KV head)
// group: two 64-dim halves of 32 rows x 128 bytes each for K and for V, loaded by
// TMA with the 128-byte swizzle into one 16 KB ring stage. A group's keys are
// 0 .. len (the new token sits at position len), so it has ceil((len + 1) / 32)
// units, and the units of all groups, in group order, are split evenly over the
// CTAs. The step computes S = Q K^T and P V with mma.sync m16n8k16 from the
// swizzled tiles (the group's query heads padded to 16 rows) and an online
// softmax in the log2 domain ("Implementación de la atención"; "GQA" and
// "Scaled Dot-Product Attention" on the llama3.np page).
#pragma once
#include "common.cuh"
#include "kernels.cuh"

#include <math.h>

namespace lfw {

constexpr int AK = 32;  // keys per attention unit (K and V tiles of 32 x 128 bf16 = 16 KB)

// Swizzled address of 16-byte chunk `chunk` (0..15) of key row `key` in a K or V
// tile of an attention unit: two 64-dim halves of 32 rows x 128 B, 4 KB apart.
DEVI uint32_t kv32_addr(uint32_t base, int key, int chunk) {
    return base + (chunk >> 3) * (AK * 128) + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
}
// Attention units of a group: keys 0 .. len (the new token at position len).
DEVI int group_units(const int* s_len, int grp, int Hk) { return (s_len[grp / Hk] + AK) / AK; }

// This CTA's share of the attention units (the same for every layer).
struct AttnSplit {
    long long U, G, u0, u1;  // all units, CTAs taking part, this CTA's range
    int g0, j0;              // group and tile of unit u0
    long long cum0;          // first unit of group g0
};
DEVI AttnSplit attn_split(const int* s_len, int B, int Hk) {
    AttnSplit sp;
    long long U = 0;
    for (int gr = 0; gr < B * Hk; ++gr) U += group_units(s_len, gr, Hk);
    sp.U = U;
    sp.G = (long long)gridDim.x < U ? (long long)gridDim.x : U;
    if (blockIdx.x < sp.G) {
        sp.u0 = blockIdx.x * U / sp.G;
        sp.u1 = (blockIdx.x + 1) * U / sp.G;
    } else {
        sp.u0 = sp.u1 = U;
    }
    long long c = 0;
    int gr = 0;
    while (gr < B * Hk) {
        const int n = group_units(s_len, gr, Hk);
        if (c + n > sp.u0) break;
        c += n;
        ++gr;
    }
    sp.g0 = gr;
    sp.j0 = (int)(sp.u0 - c);
    sp.cum0 = c;
    return sp;
}

// ---- one warp's attention over 32-key units, on the tensor cores -----------
// Used by the cluster decode attention (attn_cluster.cu). A group's query rows (at most 8: the query heads
// of one KV head) sit in a 16-row tile of 256-byte rows in shared memory (rows
// past the group's zero, 16-byte chunks swizzled by row). For each unit the warp
// computes S = Q K^T (m16n8k16, queries as A, the unit's key rows as B), keeps an
// online softmax of query row g = lane / 4 (running max and sum, log2 domain),
// and accumulates the transposed output O^T += V^T P^T: the value tile read with
// transposed 8x8 loads is the A operand and the lane's own probabilities of row
// g are the B operand, so the 128 x 8 accumulator takes 32 registers.
constexpr int AW_REC = 132;  // a row's record: m, l, two pads, O[128]
__host__ __device__ constexpr int attn_scratch_bytes(int R) { return 4096 + 8 * R * AW_REC * 4; }

struct AttnAcc {
    float o[8][4];  // m-tile mt: dims mt*16 + g and + 8, rows 2t and 2t + 1
    float m, l;     // row g: running max (log2 domain) and this lane's part of the sum
};
DEVI void attn_acc_init(AttnAcc& A) {
#pragma unroll
    for (int n = 0; n < 8; ++n) A.o[n][0] = A.o[n][1] = A.o[n][2] = A.o[n][3] = 0.f;
    A.m = -INFINITY;
    A.l = 0.f;
}

// Query rows r < R (row r at q + r * row_stride) into the 16-row tile at qsm,
// zero past R; threads tid < 256 copy one 16-byte chunk each, others nothing.
DEVI void attn_q_tile(uint8_t* qsm, const __nv_bfloat16* q, size_t row_stride, int R, int tid) {
    if (tid >= 256) return;
    const int r = tid >> 4, c = tid & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < R) v = __ldcg(reinterpret_cast<const uint4*>(q + (size_t)r * row_stride + c * 8));
    *reinterpret_cast<uint4*>(qsm + r * 256 + ((c ^ (r & 7)) << 4)) = v;
}

// One unit: keys key0 .. key0 + 31 (those after position p0 masked), key tile at
// kb and value tile at kb + 8 KB in shared memory, query tile at qbase.
DEVI void attn_unit(AttnAcc& A, uint32_t kb, uint32_t qbase, int key0, int p0, float scale_log2) {
    const int lane = threadIdx.x & 31;
    const int t4 = lane & 3, j8 = lane >> 3, i8 = lane & 7;
    const uint32_t vb = kb + 2 * AK * 128;
    const int qr = (j8 & 1) * 8 + i8;  // this lane's query-tile row for ldmatrix
    const uint32_t qrow = qbase + qr * 256;
    // S = Q K^T: 16 query rows (rows 8..15 zero) x 32 keys
    float sc[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll 2
    for (int kk = 0; kk < 8; ++kk) {
        uint32_t qa[4];
        ldsm_x4(qa, qrow + (((2 * kk + (j8 >> 1)) ^ (qr & 7)) << 4));
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t rr[4];
            ldsm_x4(rr, kv32_addr(kb, (2 * np + (j8 >> 1)) * 8 + i8, 2 * kk + (j8 & 1)));
            mma_bf16_16816(sc[2 * np], qa, rr[0], rr[1]);
            mma_bf16_16816(sc[2 * np + 1], qa, rr[2], rr[3]);
        }
    }
    // online softmax of row g over the unit's keys
    float mx = -INFINITY;
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            float v = sc[n][e2] * scale_log2;
            if (key0 + n * 8 + 2 * t4 + e2 > p0) v = -INFINITY;
            sc[n][e2] = v;
            mx = fmaxf(mx, v);
        }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mnew = fmaxf(A.m, mx);
    const float muse = mnew == -INFINITY ? 0.f : mnew;
    const float alpha = exp2f(A.m - muse);
    A.m = mnew;
    float sum = 0.f;
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const float pv = exp2f(sc[n][e2] - muse);
            sc[n][e2] = pv;
            sum += pv;
        }
    A.l = A.l * alpha + sum;
    // the accumulators hold rows 2t and 2t + 1, whose factors sit in lanes 8t and 8t + 4
    const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * t4);
    const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * t4 + 4);
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        A.o[n][0] *= a0;
        A.o[n][1] *= a1;
        A.o[n][2] *= a0;
        A.o[n][3] *= a1;
    }
    // O^T += V^T P^T
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t b0 = pack_bf16x2(sc[2 * ks][0], sc[2 * ks][1]);
        const uint32_t b1 = pack_bf16x2(sc[2 * ks + 1][0], sc[2 * ks + 1][1]);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t va[4];
            ldsm_x4_t(va, kv32_addr(vb, ks * 16 + (j8 >> 1) * 8 + i8, 2 * mt + (j8 & 1)));
            mma_bf16_16816(A.o[mt], va, b0, b1);
        }
    }
}

// This warp's state of rows r < R into wst[warp][r][AW_REC] (m, l, O[128]).
DEVI void attn_acc_store(AttnAcc& A, float* wst, int warp, int R) {
    const int lane = threadIdx.x & 31, g8 = lane >> 2, t4 = lane & 3;
    A.l += __shfl_xor_sync(0xffffffffu, A.l, 1);
    A.l += __shfl_xor_sync(0xffffffffu, A.l, 2);
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
        const int row = 2 * t4 + e2;
        if (row >= R) continue;
        float* w = wst + ((size_t)warp * R + row) * AW_REC + 4;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            w[mt * 16 + g8] = A.o[mt][e2];
            w[mt * 16 + g8 + 8] = A.o[mt][2 + e2];
        }
    }
    if (t4 == 0 && g8 < R) {
        float* w = wst + ((size_t)warp * R + g8) * AW_REC;
        w[0] = A.m;
        w[1] = A.l;
    }
}

// Log-sum-exp merge of (m2, l2, O2) into (M, L, O) for four output dims.
DEVI void lse_merge(float& M, float& L, float (&O)[4], float m2, float l2, const float4& o2) {
    const float mn = fmaxf(M, m2);
    const float mu = mn == -INFINITY ? 0.f : mn;
    const float sa = exp2f(M - mu), sb = exp2f(m2 - mu);
    L = L * sa + l2 * sb;
    O[0] = O[0] * sa + o2.x * sb;
    O[1] = O[1] * sa + o2.y * sb;
    O[2] = O[2] * sa + o2.z * sb;
    O[3] = O[3] * sa + o2.w * sb;
    M = mn;
}

// Merge of the NW warps' records for row r, dims d4 .. d4 + 3: the common max
// first, then the scaled sums in warp order (every read issued up front).
template <int NW>
DEVI void attn_merge_warps(const float* wst, int R, int r, int d4, float& M, float& L, float (&O)[4]) {
    float m[NW], l[NW];
    float4 o[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const float* ws = wst + ((size_t)w * R + r) * AW_REC;
        m[w] = ws[0];
        l[w] = ws[1];
        o[w] = *reinterpret_cast<const float4*>(ws + 4 + d4);
    }
    M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, m[w]);
    const float mu = M == -INFINITY ? 0.f : M;
    L = 0.f;
    O[0] = O[1] = O[2] = O[3] = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const float sc = exp2f(m[w] - mu);
        L += sc * l[w];
        O[0] += sc * o[w].x;
        O[1] += sc * o[w].y;
        O[2] += sc * o[w].z;
        O[3] += sc * o[w].w;
    }
}

}  // namespace lfw
