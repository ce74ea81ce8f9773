// Causal grouped-query attention of a few new tokens against the KV cache,
// split over the keys (decode phase; also the fp32 path's prefill).
//
// Same mathematics as the prefill kernel ("Implementación de la atención";
// "GQA", "Scaled Dot-Product Attention" and "KV cache" on the llama3.np page):
// query head h at position p attends to keys 0..p of KV head h / G with scores
// q.k / sqrt(d) and a softmax.
//
// A CTA owns one (sequence, KV head, chunk of query tokens) and one contiguous
// slice ("split") of the keys; its rows are the G query heads of the KV head for
// each query token, so each key and value row is read once for the whole group.
// Lane j of a warp scores key j of a 32-key group for every row, the warp keeps
// an online softmax (running max and sum, log2 domain), and accumulates
// P V with lane l owning dims 4l..4l+3. The 4 warps' states and then the splits'
// states (m, l, o) are merged by the log-sum-exp rule; the merge across
// splits is done by whichever CTA of the (sequence, head, chunk) finishes last
// (an atomic counter, no waiting), which also resets the counter.
#include "common.cuh"
#include "kernels.cuh"

#include <math.h>

namespace lfw {

constexpr int AD_THREADS = 128;
constexpr int AD_DMAX = 128;

template <typename KT> DEVI void load8(const KT* p, float (&v)[8]);
template <> DEVI void load8<float>(const float* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <> DEVI void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}
template <typename KT> DEVI void load4(const KT* p, float (&v)[4]);
template <> DEVI void load4<float>(const float* p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <> DEVI void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
}

template <typename KT, int RMAX>
__global__ void __launch_bounds__(AD_THREADS) attn_decode_kernel(const AttnDecodeArgs a) {
    __shared__ __align__(16) float qs[RMAX][AD_DMAX];
    __shared__ float wm[4][RMAX], wl[4][RMAX];
    __shared__ __align__(16) float wo[4][RMAX][AD_DMAX];
    __shared__ int last_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, qc = blockIdx.z;
    const int b = blockIdx.y / a.Hk, kvh = blockIdx.y % a.Hk;
    const int G = a.H / a.Hk, d = a.d;
    const int R = a.tq * G;
    const int HD = a.H * d;
    const KT* q = reinterpret_cast<const KT*>(a.q);
    const long long head_off = (long long)(b * a.Hk + kvh) * a.S_max * d;
    const KT* kc = reinterpret_cast<const KT*>(a.kc) + head_off;
    const KT* vc = reinterpret_cast<const KT*>(a.vc) + head_off;

    pdl_trigger();
    pdl_wait();
    const int p0 = a.pos0[b];
    const int t_first = qc * a.tq;
    const int t_last = min(a.T - 1, t_first + a.tq - 1);
    // keys [0, limit) are visible to some row; never read past the cache
    const int limit = min(p0 + t_last + 1, a.S_max);
    int chunk = (limit + a.n_splits - 1) / a.n_splits;
    chunk = (chunk + 31) & ~31;
    const int kbeg = split * chunk;
    const int kend = min(limit, kbeg + chunk);

    // Query rows, pre-scaled by log2(e)/sqrt(d).
    for (int idx = threadIdx.x; idx < RMAX * AD_DMAX; idx += AD_THREADS) {
        const int r = idx / AD_DMAX, dd = idx % AD_DMAX;
        float v = 0.f;
        const int t = t_first + r / G;
        if (r < R && t < a.T && dd < d) {
            const int h = kvh * G + r % G;
            v = to_f<KT>(q[(long long)(b * a.T + t) * HD + h * d + dd]) * a.scale_log2;
        }
        qs[r][dd] = v;
    }
    int plim[RMAX];  // last visible key of each row (-1: no row)
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        const int t = t_first + r / G;
        plim[r] = (r < R && t < a.T) ? p0 + t : -1;
    }
    __syncthreads();

    float m[RMAX], l[RMAX], o[RMAX][4];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
        o[r][0] = o[r][1] = o[r][2] = o[r][3] = 0.f;
    }
    const bool own_dims = 4 * lane < d;

    for (int kb = kbeg + warp * 32; kb < kend; kb += 4 * 32) {
        const int j = kb + lane;
        const bool jv = j < kend;
        float s[RMAX];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) s[r] = 0.f;
        if (jv) {
            const KT* kp = kc + (long long)j * d;
            for (int dd = 0; dd < d; dd += 8) {
                float kv[8];
                load8<KT>(kp + dd, kv);
#pragma unroll
                for (int r = 0; r < RMAX; ++r) {
                    const float4 qa = *reinterpret_cast<const float4*>(&qs[r][dd]);
                    const float4 qb = *reinterpret_cast<const float4*>(&qs[r][dd + 4]);
                    s[r] += qa.x * kv[0] + qa.y * kv[1] + qa.z * kv[2] + qa.w * kv[3] + qb.x * kv[4] +
                            qb.y * kv[5] + qb.z * kv[6] + qb.w * kv[7];
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
            for (int i = 0; i < 4; ++i) o[r][i] *= alpha;
        }
        const int nv = min(32, kend - kb);
        for (int jj = 0; jj < nv; ++jj) {
            float vv[4] = {0.f, 0.f, 0.f, 0.f};
            if (own_dims) load4<KT>(vc + (long long)(kb + jj) * d + 4 * lane, vv);
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                const float pj = __shfl_sync(0xffffffffu, p[r], jj);
#pragma unroll
                for (int i = 0; i < 4; ++i) o[r][i] += pj * vv[i];
            }
        }
    }

    // Merge the 4 warps.
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (lane == 0) {
            wm[warp][r] = m[r];
            wl[warp][r] = l[r];
        }
        if (own_dims) *reinterpret_cast<float4*>(&wo[warp][r][4 * lane]) = make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
    }
    __syncthreads();
    const long long rec = d + 2;
    const long long grp = ((long long)(b * a.Hk + kvh) * a.n_qchunks + qc);
    float* part = a.ws_part + grp * R * a.n_splits * rec;
    for (int idx = threadIdx.x; idx < R * d; idx += AD_THREADS) {
        const int r = idx / d, dd = idx % d;
        float M = -INFINITY;
        for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w][r]);
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, O = 0.f;
        for (int w = 0; w < 4; ++w) {
            const float sc = exp2f(wm[w][r] - Mu);
            L += sc * wl[w][r];
            O += sc * wo[w][r][dd];
        }
        float* pr = part + ((long long)r * a.n_splits + split) * rec;
        pr[2 + dd] = O;
        if (dd == 0) {
            pr[0] = M;
            pr[1] = L;
        }
    }

    // The last split CTA of this group merges all splits.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(a.ws_count + grp, 1u);
        last_s = (prev == (unsigned)(a.n_splits - 1));
    }
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    KT* out = reinterpret_cast<KT*>(a.out);
    for (int idx = threadIdx.x; idx < R * d; idx += AD_THREADS) {
        const int r = idx / d, dd = idx % d;
        const int t = t_first + r / G;
        if (t >= a.T) continue;
        const int h = kvh * G + r % G;
        const float* pr = part + (long long)r * a.n_splits * rec;
        float M = -INFINITY;
        for (int sp = 0; sp < a.n_splits; ++sp) M = fmaxf(M, __ldcg(pr + sp * rec));
        float L = 0.f, O = 0.f;
        for (int sp = 0; sp < a.n_splits; ++sp) {
            const float sc = exp2f(__ldcg(pr + sp * rec) - M);
            L += sc * __ldcg(pr + sp * rec + 1);
            O += sc * __ldcg(pr + sp * rec + 2 + dd);
        }
        out[(long long)(b * a.T + t) * HD + h * d + dd] = from_f<KT>(O / L);
    }
    if (threadIdx.x == 0) a.ws_count[grp] = 0u;
}

AttnDecodePlan attn_decode_plan(int B, int T, int H, int Hk, int d, int max_keys, int num_sms) {
    AttnDecodePlan p;
    const int G = H / Hk;
    p.tq = G >= 16 ? 1 : (16 / G < T ? 16 / G : T);
    if (p.tq < 1) p.tq = 1;
    p.n_qchunks = (T + p.tq - 1) / p.tq;
    const int groups = B * Hk * p.n_qchunks;
    int ns = (2 * num_sms + groups - 1) / groups;
    const int by_len = (max_keys + 127) / 128;
    if (ns > by_len) ns = by_len;
    if (ns > 64) ns = 64;
    if (ns < 1) ns = 1;
    p.n_splits = ns;
    p.part_floats = (size_t)groups * p.tq * G * ns * (d + 2);
    p.counters = groups;
    return p;
}

cudaError_t launch_attn_decode(const AttnDecodeArgs& a, bool bf16, cudaStream_t s, bool pdl) {
    const int G = a.H / a.Hk;
    const int R = a.tq * G;
    if (a.H % a.Hk != 0 || R > 16 || a.d > AD_DMAX || a.d % 8 != 0) return cudaErrorInvalidValue;
    const dim3 grid(a.n_splits, a.B * a.Hk, a.n_qchunks);
    if (bf16) {
        if (R <= 4) return launch_k(attn_decode_kernel<__nv_bfloat16, 4>, grid, AD_THREADS, 0, s, pdl, a);
        if (R <= 8) return launch_k(attn_decode_kernel<__nv_bfloat16, 8>, grid, AD_THREADS, 0, s, pdl, a);
        return launch_k(attn_decode_kernel<__nv_bfloat16, 16>, grid, AD_THREADS, 0, s, pdl, a);
    }
    if (R <= 4) return launch_k(attn_decode_kernel<float, 4>, grid, AD_THREADS, 0, s, pdl, a);
    if (R <= 8) return launch_k(attn_decode_kernel<float, 8>, grid, AD_THREADS, 0, s, pdl, a);
    return launch_k(attn_decode_kernel<float, 16>, grid, AD_THREADS, 0, s, pdl, a);
}

}  // namespace lfw
