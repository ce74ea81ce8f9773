// One work item of split-KV decode attention, run by the single-launch kernel
// of attn_decode.cu (the workspace and the allocation-free entry points; the
// fused decode step streams its attention through its own ring instead).
//
// Causal grouped-query attention of a few new tokens against the KV cache
// ("Implementación de la atención"; "GQA", "Scaled Dot-Product Attention" and
// "KV cache" on the llama3.np page): query head h at position p attends to keys
// 0..p of KV head h / G with scores q.k / sqrt(d) and a softmax.
//
// A work item is one (sequence, KV head, chunk of query rows) and one
// contiguous slice ("split") of the keys. The rows of a KV head are its G query
// heads at each query token, flattened as t*G + h; a chunk holds up to 16 of
// them (whole tokens when G <= 16, part of one token's heads when G > 16), so
// each key and value row is read once for all the rows of a chunk. Each of the
// NW warps takes 32-key groups of the split. Lane j loads the whole key row j
// into registers and the value slice (dims 4l..4l+3) of all 32 keys, every load
// issued before the first use, so a group costs one memory round trip. Lane j
// scores key j for every row against the query rows, which all lanes read from
// shared memory as broadcasts; the warp keeps an online softmax (running max
// and sum, log2 domain) and accumulates P V. The warps' states, then the
// splits' states (m, l, o), are merged by the log-sum-exp rule; the split merge
// is done by whichever CTA of the group finishes last (an atomic counter, no
// waiting), which also resets the counter.
//
// Queries, keys and values are read with ld.global.cg (cached in L2 only);
// each byte is used by one CTA.
#pragma once
#include "common.cuh"
#include "kernels.cuh"

#include <math.h>

namespace lfw {

constexpr int AD_GK = 32;  // keys per group (one per lane)
constexpr int AD_DMAX = 128;
constexpr int AD_MAX_SPLITS = 64;

// Shared-memory floats one work item needs: query rows, then per-warp (m, l),
// then per-warp partial outputs.
constexpr int attn_scratch_floats(int RMAX, int NW) { return RMAX * AD_DMAX + 2 * NW * RMAX + NW * RMAX * AD_DMAX; }

template <typename KT> DEVI void unpack16(const uint4& u, float (&v)[16 / sizeof(KT)]);
template <> DEVI void unpack16<float>(const uint4& u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y); v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
}
template <> DEVI void unpack16<__nv_bfloat16>(const uint4& u, float (&v)[8]) {
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}
// Four consecutive elements as raw bits (8 bytes of bf16 or 16 bytes of fp32).
template <typename KT> struct Vec4;
template <> struct Vec4<float> { using T = uint4; };
template <> struct Vec4<__nv_bfloat16> { using T = uint2; };
DEVI void to4(const uint4& u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y); v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
}
DEVI void to4(const uint2& u, float (&v)[4]) { v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y); }

// Runs work item (split, b, kvh, qc) with the first NW warps of the CTA
// (synchronised by named barrier 1). scratch: attn_scratch_floats(RMAX, NW)
// floats of 16-byte aligned shared memory; last_s: one shared int. VBATCH value
// rows and up to KMAX 16-byte chunks of a key row are loaded together (smaller
// batches: fewer registers, less latency hidden per warp).
template <typename KT, int RMAX, int NW, int VBATCH = (sizeof(KT) == 2 ? AD_GK : AD_GK / 2), int KMAX = 16>
DEVI void attn_split_item(const AttnDecodeArgs& a, int split, int b, int kvh, int qc, float* scratch, int* last_s) {
    static_assert(AD_GK % VBATCH == 0, "value batches must tile the key group");
    constexpr int NT = NW * 32;
    constexpr int EPC = 16 / sizeof(KT);  // elements per 16-byte chunk
    constexpr int NCH = AD_DMAX / EPC;    // chunks of a full-width key row
    constexpr int KBATCH = NCH < KMAX ? NCH : KMAX;  // key-row chunks loaded together
    using V4 = typename Vec4<KT>::T;
    // qs (query rows * log2(e)/sqrt(d)) during the keys, then the split weights
    // and sums sm_m/sm_l [RMAX][64] each during the split merge.
    float* qbuf = scratch;
    float(*wm)[RMAX] = reinterpret_cast<float(*)[RMAX]>(scratch + RMAX * AD_DMAX);
    float(*wl)[RMAX] = reinterpret_cast<float(*)[RMAX]>(scratch + RMAX * AD_DMAX + NW * RMAX);
    float(*wo)[RMAX][AD_DMAX] = reinterpret_cast<float(*)[RMAX][AD_DMAX]>(scratch + RMAX * AD_DMAX + 2 * NW * RMAX);
    float(*qs)[AD_DMAX] = reinterpret_cast<float(*)[AD_DMAX]>(qbuf);
    float(*sm_m)[AD_MAX_SPLITS] = reinterpret_cast<float(*)[AD_MAX_SPLITS]>(qbuf);
    float(*sm_l)[AD_MAX_SPLITS] = reinterpret_cast<float(*)[AD_MAX_SPLITS]>(qbuf + RMAX * AD_MAX_SPLITS);
    static_assert(2 * AD_MAX_SPLITS <= AD_DMAX, "split merge scratch must fit in the query buffer");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.H / a.Hk, d = a.d;
    const int R = a.rows;  // rows r of this item: (token, head) row0 + r, flattened as t*G + h
    const int HD = a.H * d;
    const int nch = d / EPC;
    const KT* q = reinterpret_cast<const KT*>(a.q);
    const long long head_off = (long long)(b * a.Hk + kvh) * a.S_max * d;
    const KT* kc = reinterpret_cast<const KT*>(a.kc) + head_off;
    const KT* vc = reinterpret_cast<const KT*>(a.vc) + head_off;

    const int p0 = a.pos0[b];
    if (threadIdx.x == 0) LFW_CHECK(p0 >= 0 && p0 + a.T <= a.S_max, a.err, BC_ATTN_POS);
    const int row0 = qc * R;
    const int t_last = min(a.T - 1, (row0 + R - 1) / G);
    // keys [0, limit) are visible to some row; never read past the cache
    const int limit = min(p0 + t_last + 1, a.S_max);
    int chunk = (limit + a.n_splits - 1) / a.n_splits;
    chunk = (chunk + AD_GK - 1) & ~(AD_GK - 1);
    const int kbeg = split * chunk;
    const int kend = min(limit, kbeg + chunk);

    // The first key-row batch and value batch of this warp's first group are
    // requested now, so their latency overlaps the query staging below.
    const bool own_dims = 4 * lane < d;
    uint4 kr0[KBATCH];
    V4 vr0[VBATCH];
    auto load_first = [&](int kb) {
        const int jj0 = kb + lane;
        const uint4* kp = reinterpret_cast<const uint4*>(kc + (long long)(jj0 < kend ? jj0 : kb) * d);
#pragma unroll
        for (int c = 0; c < KBATCH; ++c) kr0[c] = (c < nch && kb < kend) ? __ldcg(kp + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int jj = 0; jj < VBATCH; ++jj) {
            if (kb + jj < kend && own_dims) vr0[jj] = __ldcg(reinterpret_cast<const V4*>(vc + (long long)(kb + jj) * d + 4 * lane));
            else vr0[jj] = V4{};
        }
    };
    load_first(kbeg + warp * AD_GK);

    // Query rows, pre-scaled by log2(e)/sqrt(d): 4 elements per thread per step.
    for (int idx = threadIdx.x; idx < RMAX * (AD_DMAX / 4); idx += NT) {
        const int r = idx / (AD_DMAX / 4), dd = (idx % (AD_DMAX / 4)) * 4;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        const int t = (row0 + r) / G, hq = (row0 + r) % G;
        if (r < R && t < a.T && dd < d)
            to4(__ldcg(reinterpret_cast<const V4*>(q + (long long)(b * a.T + t) * HD + (kvh * G + hq) * d + dd)), v);
        *reinterpret_cast<float4*>(&qs[r][dd]) =
            make_float4(v[0] * a.scale_log2, v[1] * a.scale_log2, v[2] * a.scale_log2, v[3] * a.scale_log2);
    }
    int plim[RMAX];  // last visible key of each row (-1: no row)
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        const int t = (row0 + r) / G;
        plim[r] = (r < R && t < a.T) ? p0 + t : -1;
    }
    named_bar_sync(1, NT);

    float m[RMAX], l[RMAX], o[RMAX][4];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
        o[r][0] = o[r][1] = o[r][2] = o[r][3] = 0.f;
    }

    for (int kb = kbeg + warp * AD_GK; kb < kend; kb += NW * AD_GK) {
        const int j = kb + lane;
        const bool jv = j < kend;
        const int nk = min(AD_GK, kend - kb);
        // This lane's key row, KBATCH 16-byte chunks per batch with every load of a
        // batch issued before its first use (one batch for bf16 rows).
        const uint4* kp = reinterpret_cast<const uint4*>(kc + (long long)(jv ? j : kb) * d);
        float s[RMAX];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) s[r] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < NCH; c0 += KBATCH) {
            if (c0 >= nch) break;
            uint4 kr[KBATCH];
#pragma unroll
            for (int c = 0; c < KBATCH; ++c)
                kr[c] = c0 == 0 ? kr0[c] : ((c0 + c < nch) ? __ldcg(kp + c0 + c) : make_uint4(0, 0, 0, 0));
#pragma unroll
            for (int c = 0; c < KBATCH; ++c) {
                if (c0 + c < nch) {
                    float kv[EPC];
                    unpack16<KT>(kr[c], kv);
#pragma unroll
                    for (int r = 0; r < RMAX; ++r) {
#pragma unroll
                        for (int e = 0; e < EPC; e += 4) {
                            const float4 qv = *reinterpret_cast<const float4*>(&qs[r][(c0 + c) * EPC + e]);  // broadcast
                            s[r] += qv.x * kv[e] + qv.y * kv[e + 1] + qv.z * kv[e + 2] + qv.w * kv[e + 3];
                        }
                    }
                }
            }
        }
        float p[RMAX];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            const float sv = (jv && j <= plim[r]) ? s[r] : -INFINITY;
            const float mx = warp_max(sv);
            const float mnew = fmaxf(m[r], mx);
            const float muse = (mnew == -INFINITY) ? 0.f : mnew;
            const float alpha = exp2f(m[r] - muse);
            p[r] = exp2f(sv - muse);
            l[r] = l[r] * alpha + warp_sum(p[r]);
            m[r] = mnew;
#pragma unroll
            for (int e = 0; e < 4; ++e) o[r][e] *= alpha;
        }
        // Value slices of VBATCH keys per batch, all loads of a batch issued first.
#pragma unroll
        for (int j0 = 0; j0 < AD_GK; j0 += VBATCH) {
            V4 vr[VBATCH];
#pragma unroll
            for (int jj = 0; jj < VBATCH; ++jj) {
                if (j0 == 0)
                    vr[jj] = vr0[jj];
                else if (j0 + jj < nk && own_dims)
                    vr[jj] = __ldcg(reinterpret_cast<const V4*>(vc + (long long)(kb + j0 + jj) * d + 4 * lane));
                else
                    vr[jj] = V4{};
            }
#pragma unroll
            for (int jj = 0; jj < VBATCH; ++jj) {
                float vv[4];
                to4(vr[jj], vv);
#pragma unroll
                for (int r = 0; r < RMAX; ++r) {
                    const float pj = __shfl_sync(0xffffffffu, p[r], j0 + jj);
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[r][e] += pj * vv[e];
                }
            }
        }
        if (kb + NW * AD_GK < kend) load_first(kb + NW * AD_GK);
    }

    // Merge the NW warps.
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (lane == 0) {
            wm[warp][r] = m[r];
            wl[warp][r] = l[r];
        }
        if (own_dims) *reinterpret_cast<float4*>(&wo[warp][r][4 * lane]) = make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
    }
    named_bar_sync(1, NT);
    const long long rec = d + 4;  // m, l, 2 pad, o[d]: o starts 16-byte aligned
    const long long grp = ((long long)(b * a.Hk + kvh) * a.n_qchunks + qc);
    float* part = a.ws_part + grp * R * a.n_splits * rec;
    for (int idx = threadIdx.x; idx < R * d; idx += NT) {
        const int r = idx / d, dd = idx % d;
        float M = -INFINITY;
        for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w][r]);
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, O = 0.f;
        for (int w = 0; w < NW; ++w) {
            const float sc = exp2f(wm[w][r] - Mu);
            L += sc * wl[w][r];
            O += sc * wo[w][r][dd];
        }
        float* pr = part + ((long long)r * a.n_splits + split) * rec;
        pr[4 + dd] = O;
        if (dd == 0) {
            pr[0] = M;
            pr[1] = L;
        }
    }

    // The last split of this group merges all splits.
    named_bar_sync(1, NT);
    if (threadIdx.x == 0) {
        const unsigned prev = atom_add_acq_rel(a.ws_count + grp, 1u);
        *last_s = (prev == (unsigned)(a.n_splits - 1));
    }
    named_bar_sync(1, NT);
    if (!*last_s) return;
    const int ns = a.n_splits;
    for (int idx = threadIdx.x; idx < R * ns; idx += NT) {
        const int r = idx / ns, sp = idx % ns;
        const float* pr = part + ((long long)r * ns + sp) * rec;
        sm_m[r][sp] = __ldcg(pr);
        sm_l[r][sp] = __ldcg(pr + 1);
    }
    named_bar_sync(1, NT);
    // Split weights w_s = exp2(m_s - max) / sum_s exp2(m_s - max) l_s, kept in sm_m.
    for (int r = threadIdx.x; r < R; r += NT) {
        float M = -INFINITY;
        for (int sp = 0; sp < ns; ++sp) M = fmaxf(M, sm_m[r][sp]);
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f;
        for (int sp = 0; sp < ns; ++sp) {
            const float w = exp2f(sm_m[r][sp] - Mu);
            sm_m[r][sp] = w;
            L += w * sm_l[r][sp];
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        for (int sp = 0; sp < ns; ++sp) sm_m[r][sp] *= inv;
    }
    named_bar_sync(1, NT);
    // Each thread owns (row, 4 dims) outputs and sums the weighted splits; the
    // loads of different splits are independent, so they overlap.
    KT* out = reinterpret_cast<KT*>(a.out);
    const int dq = d / 4;
    for (int idx = threadIdx.x; idx < R * dq; idx += NT) {
        const int r = idx / dq, d4 = (idx % dq) * 4;
        const float* pr = part + (long long)r * ns * rec + 4 + d4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int sp = 0; sp < ns; ++sp) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(pr + (long long)sp * rec));
            const float w = sm_m[r][sp];
            acc.x += w * v.x;
            acc.y += w * v.y;
            acc.z += w * v.z;
            acc.w += w * v.w;
        }
        const int t = (row0 + r) / G, hq = (row0 + r) % G;
        if (t < a.T) {
            KT* dst = out + (long long)(b * a.T + t) * HD + (kvh * G + hq) * d + d4;
            dst[0] = from_f<KT>(acc.x);
            dst[1] = from_f<KT>(acc.y);
            dst[2] = from_f<KT>(acc.z);
            dst[3] = from_f<KT>(acc.w);
        }
    }
    if (threadIdx.x == 0) a.ws_count[grp] = 0u;
}

}  // namespace lfw
