// Split-KV decode attention as its own launch (decode phase; also the fp32
// path's prefill): one CTA of 4 warps per work item of attn_core.cuh, grid
// (splits, sequences x KV heads, query-token chunks).
#include "attn_core.cuh"

namespace lfw {

constexpr int AD_WARPS = 4;
constexpr int AD_KEYS_PER_CTA = 704;
constexpr int AD_THREADS = AD_WARPS * 32;

template <typename KT, int RMAX>
__global__ void __launch_bounds__(AD_THREADS) attn_decode_kernel(const AttnDecodeArgs a) {
    __shared__ __align__(16) float scratch[attn_scratch_floats(RMAX, AD_WARPS)];
    __shared__ int last_s;
    pdl_trigger();
    pdl_wait();
    attn_split_item<KT, RMAX, AD_WARPS>(a, blockIdx.x, blockIdx.y / a.Hk, blockIdx.y % a.Hk, blockIdx.z, scratch,
                                        &last_s);
}

AttnDecodePlan attn_decode_plan(int B, int T, int H, int Hk, int d, int max_keys, int num_sms) {
    AttnDecodePlan p;
    const int G = H / Hk;
    // Rows of a work item: the G query heads of 16/G whole tokens when G <= 16,
    // else 16 of the G heads of one token (multi-query models).
    int tq = G >= 16 ? 1 : (16 / G < T ? 16 / G : T);
    if (tq < 1) tq = 1;
    p.rows = G >= 16 ? 16 : tq * G;
    p.n_qchunks = (int)(((long long)T * G + p.rows - 1) / p.rows);
    const int groups = B * Hk * p.n_qchunks;
    // The kernel's register use leaves room for two CTAs per SM. Split so that all
    // CTAs are resident at once (1.75 per SM: one wave, no tail) unless that
    // leaves a CTA more than AD_KEYS_PER_CTA keys, then split by length instead.
    // Measured on B200 (Llama-3-8B heads): batch 1 over 2304 keys is fastest at
    // 24-32 splits, batch 4 over ~2k keys at 8, batch 16 over 4k-8k keys at 12;
    // fewer splits leave SMs idle, more pay each CTA's fixed cost (query staging,
    // one load round trip, the partial write and the split merge) more often.
    // Every split keeps at least 32 keys.
    const int fill = (num_sms * 7 / 4) / groups;
    const int by_len = (max_keys + AD_KEYS_PER_CTA - 1) / AD_KEYS_PER_CTA;
    const int cap = (max_keys + AD_GK - 1) / AD_GK;
    int ns = by_len > fill ? by_len : fill;
    if (ns > cap) ns = cap;
    if (ns > AD_MAX_SPLITS) ns = AD_MAX_SPLITS;
    if (ns < 1) ns = 1;
    p.n_splits = ns;
    p.part_floats = (size_t)groups * p.rows * ns * (d + 4);
    p.counters = groups;
    return p;
}

template <typename KT, int RMAX>
static cudaError_t launch_one(const AttnDecodeArgs& a, cudaStream_t s, bool pdl) {
    const dim3 grid(a.n_splits, a.B * a.Hk, a.n_qchunks);
    return launch_k(attn_decode_kernel<KT, RMAX>, grid, AD_THREADS, 0, s, pdl, a);
}

cudaError_t launch_attn_decode(const AttnDecodeArgs& a, bool bf16, cudaStream_t s, bool pdl) {
    const int R = a.rows;
    if (a.H % a.Hk != 0 || R < 1 || R > 16 || a.d > AD_DMAX || a.d % 8 != 0 || a.n_splits > AD_MAX_SPLITS)
        return cudaErrorInvalidValue;
    if (bf16) {
        if (R <= 4) return launch_one<__nv_bfloat16, 4>(a, s, pdl);
        if (R <= 8) return launch_one<__nv_bfloat16, 8>(a, s, pdl);
        return launch_one<__nv_bfloat16, 16>(a, s, pdl);
    }
    if (R <= 4) return launch_one<float, 4>(a, s, pdl);
    if (R <= 8) return launch_one<float, 8>(a, s, pdl);
    return launch_one<float, 16>(a, s, pdl);
}

}  // namespace lfw
