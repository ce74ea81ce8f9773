// Fused projection epilogues shared by the decode GEMV and the prefill GEMM.
//
// RMSNorm ("Building llama3 from scratch", RMSNorm code block: x * rsqrt(mean(x^2)
// + eps) * w) is split across two kernels: the producer of the residual stream h
// stores hw = h * w (the norm weight of the next sub-layer) and a partial sum of
// h^2 per row; the consumer projection computes acc = hw W^T and multiplies each
// row by rinv = rsqrt(sum / dim + eps) here, before the rest of its epilogue.
// Since rinv is a per-row scalar this equals projecting the normalised input.
#pragma once
#include "common.cuh"
#include "kernels.cuh"

namespace lfw {

DEVI float row_rinv(const NormIn& n, int m) {
    if (n.ss == nullptr) return 1.f;
    const float* p = n.ss + n.row0 + (long long)m * n.row_step;
    float s = 0.f;
    for (int i = 0; i < n.nparts; ++i) s += p[(long long)i * n.ld];
    return rsqrtf(s * n.inv_dim + n.eps);
}

template <typename AT> DEVI void store2(AT* p, float a, float b);
template <> DEVI void store2<float>(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
template <> DEVI void store2<__nv_bfloat16>(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
}
// Eight consecutive values (16-byte aligned destination for bf16, 32-byte for fp32).
template <typename AT> DEVI void store8(AT* p, const float (&v)[8]);
template <> DEVI void store8<float>(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <> DEVI void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = u;
}

// RoPE (llama3.np page, "RoPE #1" and "RoPE #2"): the pair (x[2i], x[2i+1]) of a
// query or key head at position p is rotated by angle p * theta^(-2i/d), with the
// cos/sin of every (p, i) precomputed in a table. Values are rotated in fp32.
DEVI void rope_pair(const Epi& e, int pos, int col_in_head, float& v0, float& v1) {
    const int half = e.d >> 1;
    const int i = col_in_head >> 1;
    const float c = e.rope_cos[(long long)pos * half + i];
    const float s = e.rope_sin[(long long)pos * half + i];
    const float r0 = v0 * c - v1 * s;
    const float r1 = v0 * s + v1 * c;
    v0 = r0;
    v1 = r1;
}

// QKV epilogue for one (even, odd) column pair of the concatenated [q; k; v]
// projection output of token m: rotate q and k, write q, append k and v to the
// cache at the token's position ("KV cache" on the llama3.np page).
template <typename AT>
DEVI void epi_qkv_pair(const Epi& e, int m, int c, float v0, float v1) {
    const int Hd = e.H * e.d, Hkd = e.Hk * e.d;
    const int b = m / e.T;
    const int pos = e.pos0[b] + (m - b * e.T);
    if (!LFW_CHECK(pos >= 0 && pos < e.S_max, e.err, BC_CACHE_POS)) return;
    if (c < Hd + Hkd) rope_pair(e, pos, c % e.d, v0, v1);
    if (c < Hd) {
        store2<AT>(reinterpret_cast<AT*>(e.q_out) + (long long)m * Hd + c, v0, v1);
    } else {
        int cc = c - Hd;
        const bool isv = cc >= Hkd;
        if (isv) cc -= Hkd;
        const int kvh = cc / e.d, dd = cc - kvh * e.d;
        AT* base = reinterpret_cast<AT*>(isv ? e.v_cache : e.k_cache);
        store2<AT>(base + ((long long)(b * e.Hk + kvh) * e.S_max + pos) * e.d + dd, v0, v1);
    }
}

// Same for eight consecutive columns c .. c+7 (c % 8 == 0, head_dim % 8 == 0).
template <typename AT>
DEVI void epi_qkv8(const Epi& e, int m, int c, float (&v)[8]) {
    const int Hd = e.H * e.d, Hkd = e.Hk * e.d;
    const int b = m / e.T;
    const int pos = e.pos0[b] + (m - b * e.T);
    if (!LFW_CHECK(pos >= 0 && pos < e.S_max, e.err, BC_CACHE_POS)) return;
    if (c < Hd + Hkd) {
        const int ch = c % e.d;
#pragma unroll
        for (int j = 0; j < 8; j += 2) rope_pair(e, pos, ch + j, v[j], v[j + 1]);
    }
    if (c < Hd) {
        store8<AT>(reinterpret_cast<AT*>(e.q_out) + (long long)m * Hd + c, v);
    } else {
        int cc = c - Hd;
        const bool isv = cc >= Hkd;
        if (isv) cc -= Hkd;
        const int kvh = cc / e.d, dd = cc - kvh * e.d;
        AT* base = reinterpret_cast<AT*>(isv ? e.v_cache : e.k_cache);
        store8<AT>(base + ((long long)(b * e.Hk + kvh) * e.S_max + pos) * e.d + dd, v);
    }
}

// SwiGLU ("Feed Forward" on the llama3.np page; w1 is the SiLU-gated branch,
// w3 the linear one): g = silu(a) * c.
DEVI float swiglu(float a, float c) { return silu(a) * c; }

// Residual add ("Red feed-forward": the sub-layer output is added back), plus
// the next RMSNorm's input hw = h * w. Returns the new h for the sum of squares.
template <typename AT>
DEVI float epi_resid1(const Epi& e, int m, int n, float v) {
    float* hp = e.h + (long long)m * e.D + n;
    const float hn = __ldcg(hp) + v;  // h may have been written by another CTA earlier in this launch
    *hp = hn;
    const float w = to_f<AT>(reinterpret_cast<const AT*>(e.wnext)[n]);
    reinterpret_cast<AT*>(e.hw_out)[(long long)m * e.D + n] = from_f<AT>(hn * w);
    return hn;
}

// Argmax partial: the better of (va, ia) and (vb, ib); the lower index wins ties
// ("Predicción de tokens": the highest logit is the next token).
DEVI void am_merge(float& va, int& ia, float vb, int ib) {
    if (vb > va || (vb == va && ib < ia)) {
        va = vb;
        ia = ib;
    }
}

}  // namespace lfw
