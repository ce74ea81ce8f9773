// C ABI of the decoder (declared in include/llama_fwd.h): model creation, the
// per-layer driver for prefill and decode, decode-step CUDA graphs, the KV-cache
// accessors and the single-operation entry points.
//
// One pass over a batch ("Resumen ...": embedding, then for every layer RMSNorm,
// attention, residual, RMSNorm, SwiGLU, residual; final RMSNorm, logits, argmax):
//   embed          h = E[tok]; hw = h * attention_norm[0]; ss = sum h^2
//   per layer l    QKV projection (RMSNorm scale, RoPE, KV-cache append)
//                  attention (flash kernel for bf16 prompts, split-KV otherwise)
//                  wo projection + residual (writes hw = h * ffn_norm[l], ss)
//                  w1/w3 projection + SwiGLU (RMSNorm scale)
//                  w2 projection + residual (writes hw = h * next norm weight, ss)
//   head           last-position lm_head with RMSNorm scale + argmax (+ cache lengths)
// Projections of more than 16 tokens run on the tcgen05 GEMM (bf16), otherwise on
// the streaming decode GEMV. With LLM_FLAG_PDL, launches use programmatic
// dependent launch so a kernel's prologue overlaps the previous kernel's tail.
#include "../../include/llama_fwd.h"
#include "errors.cuh"
#include "kernels.cuh"

#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <map>
#include <string>
#include <tuple>
#include <vector>

using namespace lfw;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

#define CK(x)                                                                                 \
    do {                                                                                      \
        cudaError_t e_ = (x);                                                                 \
        if (e_ != cudaSuccess) return fail(LLM_ERR_CUDA, "%s: %s", #x, cudaGetErrorString(e_)); \
    } while (0)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 tensor map over [rows][inner] (row-major), box [box_rows][box_inner],
// 128-byte swizzle (box_inner * 2 must be 128).
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
               uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms_current() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct LayerW {
    const void *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *w1, *w3, *w2;
};

// RMSNorm partial sums written by a residual projection with N output rows.
int bf16_gemv_ss_parts(int N) { return gemv_num_tiles(EPI_RESID, N) * 8; }  // one per 16 rows of a 128-row tile
int f32_gemv_ss_parts(int N) { return (N + 15) / 16; }                     // one per CTA of 16 rows

__device__ uint32_t g_op_err;  // device error word of the single-operation entry points

}  // namespace

int lfw::set_error(int code, const char* msg) { return fail(code, "%s", msg); }
int lfw::current_num_sms() { return num_sms_current(); }

struct llm_model {
    llm_config cfg;
    int dev = 0, num_sms = 148;
    cudaStream_t stream = nullptr;
    bool own_stream = false;
    bool bf16 = true;
    size_t esz = 2;  // element size of weights / activations / cache
    int M_max = 0;   // token rows per call
    // weights
    const void *tok_emb = nullptr, *out = nullptr, *final_norm = nullptr;
    std::vector<LayerW> L;
    // activations and scratch
    float* h = nullptr;
    void *hw = nullptr, *q = nullptr, *o = nullptr, *g = nullptr;
    // bf16 remainders of hw, o and g (split activations of the decode projections)
    // and whether the last writer of each left them
    void *hw_lo = nullptr, *o_lo = nullptr, *g_lo = nullptr;
    bool hw_lo_ok = false, o_lo_ok = false, g_lo_ok = false;
    float* ss = nullptr;
    int ss_ld = 0;
    void *kc = nullptr, *vc = nullptr;
    long long layer_elems = 0;  // elements of one layer's K (or V) cache
    float *rope_cos = nullptr, *rope_sin = nullptr;
    float* am_val = nullptr;
    int* am_idx = nullptr;
    unsigned* am_counter = nullptr;
    GemvScratch gws;
    float* attn_ws = nullptr;
    unsigned* attn_cnt = nullptr;
    size_t attn_ws_floats = 0, attn_cnt_n = 0;
    int32_t *d_tok = nullptr, *d_next = nullptr, *seq_len = nullptr;
    float* d_logits = nullptr;
    uint32_t* d_err = nullptr;
    float* taps = nullptr;
    int taps_tokens = 0;
    std::vector<int> host_len;
    // tensor maps (bf16 models)
    CUtensorMap tm_hw, tm_o, tm_g, tm_kc, tm_vc, tm_head;
    CUtensorMap tm_k32, tm_v32;  // the K and V caches in 32-row boxes (decode attention units)
    bool kv32_ok = false;
    std::vector<CUtensorMap> tm_w;
    bool gemm_ok = false;
    // fused decode step (bf16): device copies of the weight tensor maps and norm
    // pointers, and the grid-barrier counter
    bool fused = false;
    int smem_optin = 0;
    CUtensorMap* d_tmaps = nullptr;
    const void** d_norms = nullptr;
    unsigned* ds_bar = nullptr;
    unsigned* probe_cnt = nullptr;  // grid-barrier counter of the wait probe
    // per-launch CUDA-event timing (LLM_FLAG_KERNEL_TIMING)
    bool timing = false;
    bool capturing = false;
    bool pdl = false;  // programmatic dependent launch between consecutive kernels
    struct TimeRec {
        int kind;
        cudaEvent_t a, b;
    };
    std::vector<TimeRec> trecs;      // direct launches since the last report
    std::vector<TimeRec> cap_recs;   // event nodes of the graph being captured
    double kt_ms[LLM_K_COUNT] = {};  // accumulated from graph replays
    int64_t kt_n[LLM_K_COUNT] = {};
    std::vector<cudaEvent_t> ev_pool;
    // decode graphs keyed by (B, n_splits, logits requested)
    struct Graph {
        cudaGraphExec_t exec;
        std::vector<TimeRec> recs;  // timing event pairs inside the graph
    };
    std::map<std::tuple<int, int, int>, Graph> graphs;
    std::vector<void*> allocs;
};

namespace {

cudaEvent_t pool_event(llm_model* m) {
    if (!m->ev_pool.empty()) {
        cudaEvent_t e = m->ev_pool.back();
        m->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets one kernel launch with an event pair when timing is on. Inside a
// graph capture the events become event-record nodes of the graph, so each
// replay timestamps the kernel on the device with no host gap in between.
struct KTimer {
    llm_model* m;
    int kind;
    cudaEvent_t a = nullptr;
    KTimer(llm_model* mm, int k) : m(mm), kind(k) {
        if (m->timing && m->trecs.size() < 1000000) {
            a = pool_event(m);
            if (m->capturing) cudaEventRecordWithFlags(a, m->stream, cudaEventRecordExternal);
            else cudaEventRecord(a, m->stream);
        }
    }
    ~KTimer() {
        if (a) {
            cudaEvent_t b = pool_event(m);
            if (m->capturing) {
                cudaEventRecordWithFlags(b, m->stream, cudaEventRecordExternal);
                m->cap_recs.push_back({kind, a, b});
            } else {
                cudaEventRecord(b, m->stream);
                m->trecs.push_back({kind, a, b});
            }
        }
    }
};

int dev_alloc(llm_model* m, void** p, size_t bytes) {
    if (bytes == 0) bytes = 16;
    cudaError_t e = cudaMalloc(p, bytes);
    if (e != cudaSuccess) return fail(LLM_ERR_CUDA, "cudaMalloc(%zu): %s", bytes, cudaGetErrorString(e));
    m->allocs.push_back(*p);
    return LLM_OK;
}

int validate_config(const llm_config* c) {
    if (c->dim <= 0 || c->n_layers <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
        c->ffn_hidden <= 0 || c->max_seq_len <= 0 || c->max_batch <= 0)
        return fail(LLM_ERR_BAD_CONFIG, "non-positive size in config");
    if (c->n_heads % c->n_kv_heads != 0) return fail(LLM_ERR_BAD_CONFIG, "n_heads %% n_kv_heads != 0");
    if (c->n_heads * c->head_dim != c->dim) return fail(LLM_ERR_BAD_CONFIG, "n_heads * head_dim != dim");
    if (c->head_dim % 8 != 0 || c->head_dim > 128) return fail(LLM_ERR_BAD_CONFIG, "head_dim must be a multiple of 8, <= 128");
    if (c->dim % 8 != 0 || c->ffn_hidden % 8 != 0) return fail(LLM_ERR_BAD_CONFIG, "dim and ffn_hidden must be multiples of 8");
    if (c->dtype != LLM_F32 && c->dtype != LLM_BF16) return fail(LLM_ERR_BAD_CONFIG, "dtype must be LLM_F32 or LLM_BF16");
    if (c->has_embed_and_head && c->vocab <= 0) return fail(LLM_ERR_BAD_CONFIG, "vocab must be positive");
    if (c->max_batch > 16) return fail(LLM_ERR_BAD_CONFIG, "max_batch > 16");
    if (c->dtype == LLM_BF16 && ((c->n_heads * c->head_dim) % 128 != 0 || (c->n_kv_heads * c->head_dim) % 128 != 0))
        return fail(LLM_ERR_BAD_CONFIG, "bf16 models need n_heads*head_dim and n_kv_heads*head_dim multiples of 128");
    if (!(c->norm_eps >= 0.f) || !(c->rope_theta > 0.f)) return fail(LLM_ERR_BAD_CONFIG, "bad norm_eps or rope_theta");
    return LLM_OK;
}

NormIn norm_in(const llm_model* m, int nparts, int row0 = 0, int row_step = 1) {
    NormIn n;
    n.ss = m->ss;
    n.nparts = nparts;
    n.ld = m->ss_ld;
    n.row0 = row0;
    n.row_step = row_step;
    n.inv_dim = 1.f / (float)m->cfg.dim;
    n.eps = m->cfg.norm_eps;
    return n;
}

// One projection with fused epilogue, over M token rows.
//   kind QKV: W = {wq, wk, wv}; SWIGLU: W = {w1, w3}; RESID/others: W = {w}
//   tms: tensor-map indices of the weight segments (bf16 GEMM path)
int project(llm_model* m, int l, int kind, int tkind, const void* x, const CUtensorMap* tmA, int K, int N,
            const void* const* W, const int* seg, const int* tms, const Epi& epi, int M, int* nparts_out) {
    const llm_config& c = m->cfg;
    const bool use_gemm = m->bf16 && M > 16 && m->gemm_ok;
    KTimer timer(m, tkind);
    if (use_gemm) {
        GemmArgs ga;
        ga.tmA = tmA;
        for (int i = 0; i < 3; ++i) ga.tmB[i] = tms[i] >= 0 ? &m->tm_w[(size_t)l * TM_PER_LAYER + tms[i]] : nullptr;
        for (int i = 0; i < 3; ++i) ga.seg_cols[i] = seg[i];
        ga.M = M;
        ga.N = N;
        ga.K = K;
        ga.num_sms = m->num_sms;
        ga.epi = epi;
        CK(launch_gemm_tc(ga, m->stream, m->pdl));
        if (nparts_out) *nparts_out = c.dim / GEMM_BN;
        if (kind == EPI_RESID) m->hw_lo_ok = false;
        if (kind == EPI_SWIGLU) m->g_lo_ok = false;
        return LLM_OK;
    }
    // the input's remainders, when its producer left them
    const void* x_lo = x == m->hw ? (m->hw_lo_ok ? m->hw_lo : nullptr)
                     : x == m->o  ? (m->o_lo_ok ? m->o_lo : nullptr)
                     : x == m->g  ? (m->g_lo_ok ? m->g_lo : nullptr) : nullptr;
    Epi ep = epi;
    if (m->bf16 && kind == EPI_RESID) ep.hw_lo_out = m->hw_lo;
    if (m->bf16 && kind == EPI_SWIGLU) ep.g_lo_out = m->g_lo;
    for (int r0 = 0; r0 < M; r0 += 16) {
        const int rows = M - r0 < 16 ? M - r0 : 16;
        if (m->bf16) {
            GemvArgs<__nv_bfloat16> ga;
            for (int i = 0; i < 3; ++i) ga.W[i] = reinterpret_cast<const __nv_bfloat16*>(W[i]);
            for (int i = 0; i < 3; ++i) {
                int t = tms[i];
                if (kind == EPI_SWIGLU && t == TM_W1) t = TM_W1G;
                if (kind == EPI_SWIGLU && t == TM_W3) t = TM_W3G;
                ga.tmw[i] = t >= 0 ? &m->tm_w[(size_t)l * TM_PER_LAYER + t] : nullptr;
            }
            for (int i = 0; i < 3; ++i) ga.seg_rows[i] = seg[i];
            ga.N = N;
            ga.K = K;
            ga.x = reinterpret_cast<const __nv_bfloat16*>(x) + (size_t)r0 * K;
            ga.x_lo = x_lo ? reinterpret_cast<const __nv_bfloat16*>(x_lo) + (size_t)r0 * K : nullptr;
            ga.ldx = K;
            ga.M = rows;
            ga.m0 = r0;
            ga.num_sms = m->num_sms;
            ga.ws = m->gws;
            ga.epi = ep;
            CK(launch_gemv_bf16(ga, m->stream, m->pdl));
        } else {
            GemvArgs<float> ga;
            for (int i = 0; i < 3; ++i) ga.W[i] = reinterpret_cast<const float*>(W[i]);
            for (int i = 0; i < 3; ++i) ga.seg_rows[i] = seg[i];
            ga.N = N;
            ga.K = K;
            ga.x = reinterpret_cast<const float*>(x) + (size_t)r0 * K;
            ga.ldx = K;
            ga.M = rows;
            ga.m0 = r0;
            ga.epi = epi;
            CK(launch_gemv_f32(ga, m->stream, m->pdl));
        }
    }
    if (nparts_out) *nparts_out = m->bf16 ? bf16_gemv_ss_parts(N) : f32_gemv_ss_parts(N);
    if (kind == EPI_RESID) m->hw_lo_ok = m->bf16;
    if (kind == EPI_SWIGLU) m->g_lo_ok = m->bf16;
    return LLM_OK;
}

Epi base_epi(llm_model* m, int M, int T) {
    Epi e;
    e.M = M;
    e.T = T;
    e.S_max = m->cfg.max_seq_len;
    e.err = m->d_err;
    return e;
}

// The launches of one layer, in order.
enum { PH_QKV, PH_ATTN, PH_WO, PH_W13, PH_W2, PH_PER_LAYER };

// Phase p (PH_QKV .. PH_W2) of layer l over M = B*T token rows, each as its
// own launch. *nparts: partial sums of h^2 that describe the current RMSNorm input
// hw (set by the residual phases).
int run_phase(llm_model* m, int l, int p, int B, int T, int max_keys, int* nparts) {
    const llm_config& c = m->cfg;
    const int M = B * T, D = c.dim, H = c.n_heads, Hk = c.n_kv_heads, d = c.head_dim, F = c.ffn_hidden;
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
    const LayerW& w = m->L[l];
    char* kbase = reinterpret_cast<char*>(m->kc) + (size_t)l * m->layer_elems * m->esz;
    char* vbase = reinterpret_cast<char*>(m->vc) + (size_t)l * m->layer_elems * m->esz;
    switch (p) {
        case PH_QKV: {  // QKV + RoPE + cache append
            Epi e = base_epi(m, M, T);
            e.kind = EPI_QKV_ROPE;
            e.norm = norm_in(m, *nparts);
            e.pos0 = m->seq_len;
            e.rope_cos = m->rope_cos;
            e.rope_sin = m->rope_sin;
            e.H = H;
            e.Hk = Hk;
            e.d = d;
            e.S_max = c.max_seq_len;
            e.q_out = m->q;
            e.k_cache = kbase;
            e.v_cache = vbase;
            const void* W[3] = {w.wq, w.wk, w.wv};
            const int seg[3] = {H * d, Hk * d, Hk * d};
            const int tms[3] = {TM_WQ, TM_WK, TM_WV};
            return project(m, l, EPI_QKV_ROPE, LLM_K_QKV, m->hw, &m->tm_hw, D, (H + 2 * Hk) * d, W, seg, tms, e, M,
                           nullptr);
        }
        case PH_ATTN: {
            KTimer attn_timer(m, LLM_K_ATTN);
            if (T > 1 && m->bf16 && d == 128) {
                AttnPrefillArgs a;
                a.tmK = &m->tm_kc;
                a.tmV = &m->tm_vc;
                a.row_base = (long long)l * c.max_batch * Hk * c.max_seq_len;
                a.S_max = c.max_seq_len;
                a.q = reinterpret_cast<const __nv_bfloat16*>(m->q);
                a.out = reinterpret_cast<__nv_bfloat16*>(m->o);
                a.pos0 = m->seq_len;
                a.B = B;
                a.T = T;
                a.H = H;
                a.Hk = Hk;
                a.scale_log2 = scale_log2;
                a.err = m->d_err;
                CK(launch_attn_prefill(a, m->stream, m->pdl));
                m->o_lo_ok = false;
            } else if (T == 1 && m->bf16 && m->kv32_ok && attn_cluster_size(B, H, Hk, d, m->num_sms) > 0) {
                AttnClusterArgs a;
                a.q = reinterpret_cast<const __nv_bfloat16*>(m->q);
                a.out = reinterpret_cast<__nv_bfloat16*>(m->o);
                a.pos0 = m->seq_len;
                a.B = B;
                a.H = H;
                a.Hk = Hk;
                a.S_max = c.max_seq_len;
                a.row_base = (long long)l * c.max_batch * Hk * c.max_seq_len;
                a.rows_per_seq = (long long)Hk * c.max_seq_len;
                a.out_lo = reinterpret_cast<__nv_bfloat16*>(m->o_lo);
                a.cs = attn_cluster_size(B, H, Hk, d, m->num_sms);
                a.scale_log2 = scale_log2;
                a.err = m->d_err;
                CK(launch_attn_cluster(a, &m->tm_k32, &m->tm_v32, m->stream));
                m->o_lo_ok = true;
            } else {
                const AttnDecodePlan pl = attn_decode_plan(B, T, H, Hk, d, max_keys, m->num_sms);
                if (pl.part_floats > m->attn_ws_floats || pl.counters > m->attn_cnt_n)
                    return fail(LLM_ERR_UNSUPPORTED, "attention scratch too small for this call");
                AttnDecodeArgs a;
                a.q = m->q;
                a.kc = kbase;
                a.vc = vbase;
                a.out = m->o;
                a.pos0 = m->seq_len;
                a.B = B;
                a.T = T;
                a.H = H;
                a.Hk = Hk;
                a.d = d;
                a.S_max = c.max_seq_len;
                a.n_splits = pl.n_splits;
                a.rows = pl.rows;
                a.n_qchunks = pl.n_qchunks;
                a.ws_part = m->attn_ws;
                a.ws_count = m->attn_cnt;
                a.scale_log2 = scale_log2;
                a.err = m->d_err;
                CK(launch_attn_decode(a, m->bf16, m->stream, m->pdl));
                m->o_lo_ok = false;
            }
            return LLM_OK;
        }
        case PH_WO: {  // wo + residual; writes the ffn_norm input
            Epi e = base_epi(m, M, T);
            e.kind = EPI_RESID;
            e.h = m->h;
            e.D = D;
            e.hw_out = m->hw;
            e.wnext = w.ffn_norm;
            e.ss_out = m->ss;
            e.ss_out_ld = m->ss_ld;
            const void* W[3] = {w.wo, nullptr, nullptr};
            const int seg[3] = {D, 0, 0};
            const int tms[3] = {TM_WO, -1, -1};
            return project(m, l, EPI_RESID, LLM_K_WO, m->o, &m->tm_o, H * d, D, W, seg, tms, e, M, nparts);
        }
        case PH_W13: {  // w1, w3 + SwiGLU
            Epi e = base_epi(m, M, T);
            e.kind = EPI_SWIGLU;
            e.norm = norm_in(m, *nparts);
            e.g_out = m->g;
            e.F = F;
            const void* W[3] = {w.w1, w.w3, nullptr};
            const int seg[3] = {F, 0, 0};
            const int tms[3] = {TM_W1, TM_W3, -1};
            return project(m, l, EPI_SWIGLU, LLM_K_W13, m->hw, &m->tm_hw, D, F, W, seg, tms, e, M, nullptr);
        }
        default: {  // w2 + residual; writes the next norm's input
            Epi e = base_epi(m, M, T);
            e.kind = EPI_RESID;
            e.h = m->h;
            e.D = D;
            e.hw_out = m->hw;
            e.wnext = (l + 1 < c.n_layers) ? m->L[l + 1].attn_norm : (m->final_norm ? m->final_norm : w.ffn_norm);
            e.ss_out = m->ss;
            e.ss_out_ld = m->ss_ld;
            const void* W[3] = {w.w2, nullptr, nullptr};
            const int seg[3] = {D, 0, 0};
            const int tms[3] = {TM_W2, -1, -1};
            return project(m, l, EPI_RESID, LLM_K_W2, m->g, &m->tm_g, F, D, W, seg, tms, e, M, nparts);
        }
    }
}

// Decoder layers over M = B*T token rows; h/hw/ss hold the embedding output.
int run_layers(llm_model* m, int B, int T, int max_keys) {
    const llm_config& c = m->cfg;
    const int M = B * T, D = c.dim;
    int nparts = 1;
    for (int l = 0; l < c.n_layers; ++l) {
        for (int p = 0; p < PH_PER_LAYER; ++p) {
            const int rc = run_phase(m, l, p, B, T, max_keys, &nparts);
            if (rc) return rc;
        }
        if (m->taps)
            CK(cudaMemcpyAsync(m->taps + (size_t)l * m->M_max * D, m->h, (size_t)M * D * sizeof(float),
                               cudaMemcpyDeviceToDevice, m->stream));
    }
    m->taps_tokens = M;
    return LLM_OK;
}

// Final RMSNorm + lm_head + argmax on the last position of each sequence.
int run_head(llm_model* m, int B, int T, int nparts, int32_t* next, float* logits) {
    const llm_config& c = m->cfg;
    Epi e = base_epi(m, B, 1);
    e.kind = EPI_LOGITS;
    e.norm = norm_in(m, nparts, T - 1, T);
    e.logits = logits;
    e.ld_logits = c.vocab;
    e.am_val = m->am_val;
    e.am_idx = m->am_idx;
    e.am_counter = m->am_counter;
    e.next_tok = next;
    e.seq_len = m->seq_len;
    e.advance = T;
    const void* Wout = c.tie_embeddings ? m->tok_emb : m->out;
    KTimer timer(m, LLM_K_HEAD);
    if (m->bf16) {
        GemvArgs<__nv_bfloat16> ga;
        ga.W[0] = reinterpret_cast<const __nv_bfloat16*>(Wout);
        ga.N = c.vocab;
        ga.K = c.dim;
        ga.x = reinterpret_cast<const __nv_bfloat16*>(m->hw) + (size_t)(T - 1) * c.dim;
        ga.x_lo = m->hw_lo_ok ? reinterpret_cast<const __nv_bfloat16*>(m->hw_lo) + (size_t)(T - 1) * c.dim : nullptr;
        ga.ldx = T * c.dim;
        ga.M = B;
        ga.num_sms = m->num_sms;
        ga.ws = m->gws;
        ga.tmw[0] = &m->tm_head;
        ga.epi = e;
        CK(launch_gemv_bf16(ga, m->stream, m->pdl));
    } else {
        GemvArgs<float> ga;
        ga.W[0] = reinterpret_cast<const float*>(Wout);
        ga.N = c.vocab;
        ga.K = c.dim;
        ga.x = reinterpret_cast<const float*>(m->hw) + (size_t)(T - 1) * c.dim;
        ga.ldx = T * c.dim;
        ga.M = B;
        ga.epi = e;
        CK(launch_gemv_f32(ga, m->stream, m->pdl));
    }
    return LLM_OK;
}

int last_nparts(const llm_model* m, int M) {
    // Producer of the final hw/ss: the last layer's w2 projection.
    if (m->bf16 && M > 16 && m->gemm_ok) return m->cfg.dim / GEMM_BN;
    return m->bf16 ? bf16_gemv_ss_parts(m->cfg.dim) : f32_gemv_ss_parts(m->cfg.dim);
}

int check_batch(llm_model* m, int B, int T) {
    if (B < 1 || B > m->cfg.max_batch) return fail(LLM_ERR_BATCH, "B=%d outside [1, %d]", B, m->cfg.max_batch);
    if (T < 1) return fail(LLM_ERR_BAD_ARG, "T=%d < 1", T);
    if ((long long)B * T > m->M_max) return fail(LLM_ERR_BATCH, "B*T=%lld > max_tokens=%d", (long long)B * T, m->M_max);
    for (int b = 0; b < B; ++b)
        if (m->host_len[b] + T > m->cfg.max_seq_len)
            return fail(LLM_ERR_SEQ_OVERFLOW, "sequence %d: length %d + %d > max_seq_len %d", b, m->host_len[b], T,
                        m->cfg.max_seq_len);
    return LLM_OK;
}

int max_keys_after(const llm_model* m, int B, int T) {
    int mk = 1;
    for (int b = 0; b < B; ++b) mk = m->host_len[b] + T > mk ? m->host_len[b] + T : mk;
    return mk;
}

int run_embed(llm_model* m, const int32_t* tok, const float* h_in, int M) {
    EmbedArgs ea;
    ea.tok = tok;
    ea.E = m->tok_emb;
    ea.h_in = h_in;
    ea.h = m->h;
    ea.hw = m->hw;
    ea.hw_lo = m->hw_lo;  // null for fp32 models
    m->hw_lo_ok = m->bf16;
    ea.wnorm = m->L[0].attn_norm;
    ea.ss = m->ss;
    ea.M = M;
    ea.D = m->cfg.dim;
    ea.vocab = m->cfg.vocab;
    ea.err = m->d_err;
    KTimer timer(m, LLM_K_EMBED);
    CK(launch_embed(ea, m->bf16, m->stream, m->pdl));
    return LLM_OK;
}

DecodeStepPlan fused_plan(const llm_model* m, int B, int max_keys) {
    const llm_config& c = m->cfg;
    return decode_step_plan(B, c.dim, c.n_heads, c.n_kv_heads, c.head_dim, c.ffn_hidden, c.vocab,
                            c.has_embed_and_head, max_keys, m->num_sms, m->smem_optin);
}

// Arguments of the fused decode step for B sequences.
DecodeStepArgs ds_args(llm_model* m, int B, const DecodeStepPlan& p) {
    const llm_config& c = m->cfg;
    DecodeStepArgs a;
    a.B = B;
    a.D = c.dim;
    a.H = c.n_heads;
    a.Hk = c.n_kv_heads;
    a.d = c.head_dim;
    a.F = c.ffn_hidden;
    a.vocab = c.vocab;
    a.S_max = c.max_seq_len;
    a.n_layers = c.n_layers;
    a.eps = c.norm_eps;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)c.head_dim));
    a.has_head = c.has_embed_and_head;
    a.n_stages = p.n_stages;
    a.xs_bytes = p.xs_bytes;
    for (int i = 0; i < 5; ++i) a.max_pieces[i] = p.max_pieces[i];
    a.tmaps = m->d_tmaps;
    a.norms = m->d_norms;
    a.tok_emb = m->tok_emb;
    a.kc = m->kc;
    a.vc = m->vc;
    a.layer_elems = m->layer_elems;
    a.kv_rows_per_layer = m->layer_elems / c.head_dim;
    a.seq_len = m->seq_len;
    a.h = m->h;
    a.hw = reinterpret_cast<__nv_bfloat16*>(m->hw);
    a.ss = m->ss;
    a.ss_ld = m->ss_ld;
    a.q = reinterpret_cast<__nv_bfloat16*>(m->q);
    a.o = reinterpret_cast<__nv_bfloat16*>(m->o);
    a.g = reinterpret_cast<__nv_bfloat16*>(m->g);
    a.rope_cos = m->rope_cos;
    a.rope_sin = m->rope_sin;
    a.ws = m->gws;
    a.attn_part = m->attn_ws;
    a.attn_cnt = m->attn_cnt;
    a.bar = m->ds_bar;
    a.err = m->d_err;
    return a;
}

int ds_check(llm_model* m, const DecodeStepPlan& p) {
    if (!p.supported) return fail(LLM_ERR_UNSUPPORTED, "fused decode kernel does not support this shape");
    if (p.part_floats > m->gws.part_floats || p.tiles > m->gws.tiles_cap || p.attn_part_floats > m->attn_ws_floats ||
        p.attn_counters > m->attn_cnt_n)
        return fail(LLM_ERR_UNSUPPORTED, "fused decode kernel scratch too small for this call");
    return LLM_OK;
}

// One decode step of every sequence b < B as a single fused launch (token ids,
// or hidden states for a bare layer stack).
int run_fused_step(llm_model* m, int B, const int32_t* tok, const float* h_in, float* h_out, int32_t* next,
                   float* logits) {
    const DecodeStepPlan p = fused_plan(m, B, max_keys_after(m, B, 1));
    const int rc = ds_check(m, p);
    if (rc) return rc;
    DecodeStepArgs a = ds_args(m, B, p);
    a.tok = tok;
    a.h_in = h_in;
    a.h_out = h_out;
    a.next = next;
    a.logits = logits;
    KTimer timer(m, LLM_K_STEP);
    CK(cudaMemsetAsync(m->ds_bar, 0, 4, m->stream));
    CK(launch_decode_step(a, p, m->stream));
    m->hw_lo_ok = m->o_lo_ok = m->g_lo_ok = false;
    return LLM_OK;
}

// The device work of one decode step (captured into a graph when enabled).
int decode_core(llm_model* m, int B, const int32_t* tok, int32_t* next, float* logits) {
    if (m->fused) return run_fused_step(m, B, tok, nullptr, nullptr, next, logits);
    int rc = run_embed(m, tok, nullptr, B);
    if (rc) return rc;
    rc = run_layers(m, B, 1, max_keys_after(m, B, 1));
    if (rc) return rc;
    return run_head(m, B, 1, last_nparts(m, B), next, logits);
}

}  // namespace

extern "C" {

const char* llm_last_error(void) { return g_last_error.c_str(); }

void llm_model_free(llm_model* m) {
    if (!m) return;
    if (m->stream) cudaStreamSynchronize(m->stream);
    for (auto& kv : m->graphs) {
        cudaGraphExecDestroy(kv.second.exec);
        for (auto& r : kv.second.recs) {
            cudaEventDestroy(r.a);
            cudaEventDestroy(r.b);
        }
    }
    for (auto& r : m->trecs) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    for (cudaEvent_t e : m->ev_pool) cudaEventDestroy(e);
    for (void* p : m->allocs) cudaFree(p);
    if (m->own_stream && m->stream) cudaStreamDestroy(m->stream);
    delete m;
}

int llm_model_init(const llm_config* cfg, const llm_weights* w, void* stream, llm_model** out) {
    if (!out) return fail(LLM_ERR_NULL_PTR, "out is NULL");
    *out = nullptr;
    if (!cfg || !w) return fail(LLM_ERR_NULL_PTR, "cfg or weights is NULL");
    int rc = validate_config(cfg);
    if (rc) return rc;
    const llm_config& c = *cfg;
    if (c.has_embed_and_head && (!w->tok_emb || !w->final_norm || (!c.tie_embeddings && !w->out)))
        return fail(LLM_ERR_NULL_PTR, "embedding, final norm or lm_head weight is NULL");
    if (!w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo || !w->ffn_norm || !w->w1 || !w->w3 || !w->w2)
        return fail(LLM_ERR_NULL_PTR, "a per-layer weight array is NULL");
    for (int l = 0; l < c.n_layers; ++l) {
        const void* ps[9] = {w->attn_norm[l], w->wq[l], w->wk[l], w->wv[l], w->wo[l],
                             w->ffn_norm[l],  w->w1[l], w->w3[l], w->w2[l]};
        for (int i = 0; i < 9; ++i) {
            if (!ps[i]) return fail(LLM_ERR_NULL_PTR, "layer %d weight %d is NULL", l, i);
            if (!aligned16(ps[i])) return fail(LLM_ERR_BAD_ARG, "layer %d weight %d not 16-byte aligned", l, i);
        }
    }

    llm_model* m = new llm_model();
    m->cfg = c;
    if (m->cfg.max_tokens <= 0) m->cfg.max_tokens = c.max_batch * c.max_seq_len;
    m->bf16 = c.dtype == LLM_BF16;
    m->esz = m->bf16 ? 2 : 4;
    m->M_max = m->cfg.max_tokens > c.max_batch ? m->cfg.max_tokens : c.max_batch;
    m->host_len.assign(c.max_batch, 0);
    m->timing = (c.flags & LLM_FLAG_KERNEL_TIMING) != 0;
    m->pdl = (c.flags & LLM_FLAG_PDL) != 0;
    m->tok_emb = w->tok_emb;
    m->out = w->out;
    m->final_norm = w->final_norm;
    for (int l = 0; l < c.n_layers; ++l)
        m->L.push_back({w->attn_norm[l], w->wq[l], w->wk[l], w->wv[l], w->wo[l], w->ffn_norm[l], w->w1[l], w->w3[l],
                        w->w2[l]});
    auto bail = [&](int code) {
        llm_model_free(m);
        return code;
    };
    if (cudaGetDevice(&m->dev) != cudaSuccess) return bail(fail(LLM_ERR_CUDA, "no CUDA device"));
    cudaDeviceGetAttribute(&m->num_sms, cudaDevAttrMultiProcessorCount, m->dev);
    if (stream) {
        m->stream = reinterpret_cast<cudaStream_t>(stream);
    } else {
        if (cudaStreamCreate(&m->stream) != cudaSuccess) return bail(fail(LLM_ERR_CUDA, "cudaStreamCreate failed"));
        m->own_stream = true;
    }

    const int D = c.dim, H = c.n_heads, Hk = c.n_kv_heads, d = c.head_dim, F = c.ffn_hidden;
    const size_t Mx = (size_t)m->M_max, es = m->esz;
    // residual stream and projection inputs/outputs
#define MALLOC_OR_BAIL(ptr, bytes)                                                  \
    do {                                                                            \
        int r_ = dev_alloc(m, reinterpret_cast<void**>(&(ptr)), (size_t)(bytes));    \
        if (r_ != LLM_OK) return bail(r_);                                          \
    } while (0)
    MALLOC_OR_BAIL(m->h, Mx * D * 4);
    MALLOC_OR_BAIL(m->hw, Mx * D * es);
    MALLOC_OR_BAIL(m->q, Mx * H * d * es);
    MALLOC_OR_BAIL(m->o, Mx * H * d * es);
    MALLOC_OR_BAIL(m->g, Mx * F * es);
    if (m->bf16) {
        MALLOC_OR_BAIL(m->hw_lo, Mx * D * es);
        MALLOC_OR_BAIL(m->o_lo, Mx * H * d * es);
        MALLOC_OR_BAIL(m->g_lo, Mx * F * es);
    }
    m->ss_ld = (int)Mx;
    const int parts = (bf16_gemv_ss_parts(D) > f32_gemv_ss_parts(D) ? bf16_gemv_ss_parts(D) : f32_gemv_ss_parts(D)) + 8;
    MALLOC_OR_BAIL(m->ss, (size_t)parts * Mx * 4);
    m->layer_elems = (long long)c.max_batch * Hk * c.max_seq_len * d;
    MALLOC_OR_BAIL(m->kc, (size_t)c.n_layers * m->layer_elems * es);
    MALLOC_OR_BAIL(m->vc, (size_t)c.n_layers * m->layer_elems * es);
    MALLOC_OR_BAIL(m->rope_cos, (size_t)c.max_seq_len * (d / 2) * 4);
    MALLOC_OR_BAIL(m->rope_sin, (size_t)c.max_seq_len * (d / 2) * 4);
    const int vt = c.has_embed_and_head ? (c.vocab + 15) / 16 + 8 : 8;  // fp32 head: one argmax part per CTA
    MALLOC_OR_BAIL(m->am_val, (size_t)vt * c.max_batch * 4);
    MALLOC_OR_BAIL(m->am_idx, (size_t)vt * c.max_batch * 4);
    MALLOC_OR_BAIL(m->am_counter, 64);
    {
        // Attention scratch: the largest split-KV plan any call can request
        // (decode, and prefill of fp32 or non-128 head_dim models). The plan's
        // size is not monotone in T (the split count fills the GPU per group), so
        // every T is evaluated; a plan is a few integer operations.
        size_t pf = 0, cn = 0;
        const int Tmax = (m->bf16 && d == 128) ? 1 : (int)(Mx < (size_t)c.max_seq_len ? Mx : c.max_seq_len);
        for (int B = 1; B <= c.max_batch; ++B)
            for (int T = 1; T <= Tmax && (size_t)B * T <= Mx; ++T) {
                const AttnDecodePlan p = attn_decode_plan(B, T, H, Hk, d, c.max_seq_len, m->num_sms);
                pf = p.part_floats > pf ? p.part_floats : pf;
                cn = p.counters > cn ? p.counters : cn;
            }
        if (!(m->bf16 && d == 128)) {
            for (int B = 1; B <= c.max_batch; ++B) {
                const int T = (int)(Mx / B < (size_t)c.max_seq_len ? Mx / B : c.max_seq_len);
                if (T < 1) continue;
                const AttnDecodePlan p = attn_decode_plan(B, T, H, Hk, d, c.max_seq_len, m->num_sms);
                pf = p.part_floats > pf ? p.part_floats : pf;
                cn = p.counters > cn ? p.counters : cn;
            }
        }
        m->attn_ws_floats = pf;
        m->attn_cnt_n = cn;
        MALLOC_OR_BAIL(m->attn_ws, pf * 4);
        MALLOC_OR_BAIL(m->attn_cnt, cn * 4);
    }
    if (m->bf16) {
        // Streaming GEMV scratch, sized for the largest projection of this model.
        const int shapes[5][3] = {{EPI_QKV_ROPE, (H + 2 * Hk) * d, D}, {EPI_RESID, D, H * d}, {EPI_SWIGLU, F, D},
                                  {EPI_RESID, D, F}, {EPI_LOGITS, c.has_embed_and_head ? c.vocab : 16, D}};
        size_t pf = 0;
        int tiles = 0;
        for (auto& sh : shapes) {
            const size_t f = gemv_scratch_floats(sh[0], sh[1], sh[2], m->num_sms);
            pf = f > pf ? f : pf;
            const int t = gemv_num_tiles(sh[0], sh[1]);
            tiles = t > tiles ? t : tiles;
        }
        m->gws.part_floats = pf;
        m->gws.tiles_cap = tiles;
        MALLOC_OR_BAIL(m->gws.part, pf * 4);
        MALLOC_OR_BAIL(m->gws.am_best, 16 * 8);
        MALLOC_OR_BAIL(m->gws.done_cnt, 16);
        MALLOC_OR_BAIL(m->gws.warp_cnt, (size_t)tiles * 8 * 4);
    }
    MALLOC_OR_BAIL(m->d_tok, (size_t)c.max_batch * 4);
    MALLOC_OR_BAIL(m->d_next, (size_t)c.max_batch * 4);
    MALLOC_OR_BAIL(m->seq_len, (size_t)c.max_batch * 4);
    if (c.has_embed_and_head) MALLOC_OR_BAIL(m->d_logits, (size_t)c.max_batch * c.vocab * 4);
    MALLOC_OR_BAIL(m->d_err, 64);
    MALLOC_OR_BAIL(m->probe_cnt, 16);
    if (c.flags & LLM_FLAG_DEBUG_TAPS) MALLOC_OR_BAIL(m->taps, (size_t)c.n_layers * Mx * D * 4);

    if (cudaMemsetAsync(m->am_counter, 0, 64, m->stream) != cudaSuccess ||
        cudaMemsetAsync(m->attn_cnt, 0, m->attn_cnt_n * 4, m->stream) != cudaSuccess ||
        cudaMemsetAsync(m->seq_len, 0, (size_t)c.max_batch * 4, m->stream) != cudaSuccess ||
        cudaMemsetAsync(m->d_err, 0, 64, m->stream) != cudaSuccess ||
        cudaMemsetAsync(m->ss, 0, (size_t)parts * Mx * 4, m->stream) != cudaSuccess ||
        // attention reads whole 32-key tiles: positions past a sequence's length are
        // masked, and zeroed here so that they never hold a non-finite pattern
        cudaMemsetAsync(m->kc, 0, (size_t)c.n_layers * m->layer_elems * es, m->stream) != cudaSuccess ||
        cudaMemsetAsync(m->vc, 0, (size_t)c.n_layers * m->layer_elems * es, m->stream) != cudaSuccess ||
        (m->bf16 && (cudaMemsetAsync(m->gws.am_best, 0, 16 * 8, m->stream) != cudaSuccess ||
                     cudaMemsetAsync(m->gws.done_cnt, 0, 16, m->stream) != cudaSuccess ||
                     cudaMemsetAsync(m->gws.warp_cnt, 0, (size_t)m->gws.tiles_cap * 8 * 4, m->stream) != cudaSuccess)))
        return bail(fail(LLM_ERR_CUDA, "cudaMemsetAsync failed"));
    if (launch_rope_tables(m->rope_cos, m->rope_sin, c.max_seq_len, d / 2, (double)c.rope_theta, d, m->stream) !=
        cudaSuccess)
        return bail(fail(LLM_ERR_CUDA, "rope table kernel failed"));

    // Tensor maps (bf16 only): weights for the decode GEMV (128-row boxes, 64-row
    // boxes of w1/w3 for the SwiGLU tiles) and the prefill GEMM, activations for
    // the GEMM, the KV cache for the flash attention.
    if (m->bf16) {
        bool ok = true;
        m->tm_w.resize((size_t)c.n_layers * TM_PER_LAYER);
        for (int l = 0; l < c.n_layers && ok; ++l) {
            CUtensorMap* t = &m->tm_w[(size_t)l * TM_PER_LAYER];
            const LayerW& lw = m->L[l];
            ok = make_tmap(&t[TM_WQ], lw.wq, D, (uint64_t)H * d, 64, 128) &&
                 make_tmap(&t[TM_WK], lw.wk, D, (uint64_t)Hk * d, 64, 128) &&
                 make_tmap(&t[TM_WV], lw.wv, D, (uint64_t)Hk * d, 64, 128) &&
                 make_tmap(&t[TM_WO], lw.wo, (uint64_t)H * d, D, 64, 128) &&
                 make_tmap(&t[TM_W1], lw.w1, D, F, 64, 128) && make_tmap(&t[TM_W3], lw.w3, D, F, 64, 128) &&
                 make_tmap(&t[TM_W2], lw.w2, F, D, 64, 128) && make_tmap(&t[TM_W1G], lw.w1, D, F, 64, 64) &&
                 make_tmap(&t[TM_W3G], lw.w3, D, F, 64, 64);
        }
        if (ok && c.has_embed_and_head)
            ok = make_tmap(&m->tm_head, c.tie_embeddings ? m->tok_emb : m->out, D, c.vocab, 64, 128);
        if (ok) ok = make_tmap(&m->tm_hw, m->hw, D, Mx, 64, 128) && make_tmap(&m->tm_o, m->o, H * d, Mx, 64, 128) &&
                     make_tmap(&m->tm_g, m->g, F, Mx, 64, 128);
        if (!ok) return bail(fail(LLM_ERR_CUDA, "cuTensorMapEncodeTiled failed"));
        // the QKV output in whole 256-column tiles, each half from one of wq, wk, wv
        m->gemm_ok = D % GEMM_BN == 0 && (H * d) % (GEMM_BN / 2) == 0 && (Hk * d) % (GEMM_BN / 2) == 0 &&
                     ((H + 2 * Hk) * d) % GEMM_BN == 0 && F % (GEMM_BN / 2) == 0 && D % GEMM_BK == 0 &&
                     F % GEMM_BK == 0 && (H * d) % GEMM_BK == 0;
        if (d == 128) {
            const uint64_t rows = (uint64_t)c.n_layers * c.max_batch * Hk * c.max_seq_len;
            if (!make_tmap(&m->tm_kc, m->kc, d, rows, 64, 64) || !make_tmap(&m->tm_vc, m->vc, d, rows, 64, 64) ||
                !make_tmap(&m->tm_k32, m->kc, d, rows, 64, 32) || !make_tmap(&m->tm_v32, m->vc, d, rows, 64, 32))
                return bail(fail(LLM_ERR_CUDA, "cuTensorMapEncodeTiled (KV cache) failed"));
            m->kv32_ok = true;
        }
    }
    // Fused decode step: supported shapes only, sized for every batch size at the
    // longest cache; its scratch is the decode projection's and the attention's.
    if (m->bf16 && (c.flags & LLM_FLAG_FUSED_DECODE) && !(c.flags & LLM_FLAG_DEBUG_TAPS)) {
        cudaDeviceGetAttribute(&m->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, m->dev);
        int coop = 0;
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, m->dev);
        bool ok = coop != 0;
        size_t pf = 0, af = 0, ac = 0;
        int tiles = 0;
        for (int B = 1; B <= c.max_batch && ok; ++B) {
            const DecodeStepPlan p = fused_plan(m, B, c.max_seq_len);
            ok = p.supported;
            pf = p.part_floats > pf ? p.part_floats : pf;
            af = p.attn_part_floats > af ? p.attn_part_floats : af;
            ac = p.attn_counters > ac ? p.attn_counters : ac;
            tiles = p.tiles > tiles ? p.tiles : tiles;
        }
        if (ok) {
            if (pf > m->gws.part_floats) {
                MALLOC_OR_BAIL(m->gws.part, pf * 4);
                m->gws.part_floats = pf;
            }
            if (tiles > m->gws.tiles_cap) {
                MALLOC_OR_BAIL(m->gws.warp_cnt, (size_t)tiles * 8 * 4);
                m->gws.tiles_cap = tiles;
                if (cudaMemsetAsync(m->gws.warp_cnt, 0, (size_t)tiles * 8 * 4, m->stream) != cudaSuccess)
                    return bail(fail(LLM_ERR_CUDA, "cudaMemsetAsync failed"));
            }
            if (af > m->attn_ws_floats) {
                MALLOC_OR_BAIL(m->attn_ws, af * 4);
                m->attn_ws_floats = af;
            }
            if (ac > m->attn_cnt_n) {
                MALLOC_OR_BAIL(m->attn_cnt, ac * 4);
                m->attn_cnt_n = ac;
                if (cudaMemsetAsync(m->attn_cnt, 0, ac * 4, m->stream) != cudaSuccess)
                    return bail(fail(LLM_ERR_CUDA, "cudaMemsetAsync failed"));
            }
            const size_t ntm = (size_t)c.n_layers * TM_PER_LAYER + 3;
            std::vector<CUtensorMap> tms(m->tm_w);
            tms.push_back(c.has_embed_and_head ? m->tm_head : m->tm_w[0]);
            tms.push_back(m->tm_k32);  // the whole K and V caches, 32-row boxes (attention units)
            tms.push_back(m->tm_v32);
            std::vector<const void*> norms;
            for (int l = 0; l < c.n_layers; ++l) {
                norms.push_back(m->L[l].attn_norm);
                norms.push_back(m->L[l].ffn_norm);
            }
            norms.push_back(m->final_norm ? m->final_norm : m->L[c.n_layers - 1].ffn_norm);
            MALLOC_OR_BAIL(m->d_tmaps, ntm * sizeof(CUtensorMap));
            MALLOC_OR_BAIL(m->d_norms, norms.size() * sizeof(void*));
            MALLOC_OR_BAIL(m->ds_bar, 64);
            if (cudaMemcpyAsync(m->d_tmaps, tms.data(), ntm * sizeof(CUtensorMap), cudaMemcpyHostToDevice,
                                m->stream) != cudaSuccess ||
                cudaMemcpyAsync(m->d_norms, norms.data(), norms.size() * sizeof(void*), cudaMemcpyHostToDevice,
                                m->stream) != cudaSuccess ||
                cudaMemsetAsync(m->ds_bar, 0, 64, m->stream) != cudaSuccess)
                return bail(fail(LLM_ERR_CUDA, "fused decode step setup copies failed"));
            m->fused = true;
        }
    }
    if (cudaStreamSynchronize(m->stream) != cudaSuccess) return bail(fail(LLM_ERR_CUDA, "init sync failed"));
    *out = m;
    return LLM_OK;
}

int llm_prefill(llm_model* m, const int32_t* tokens, int B, int T, int32_t* next, float* logits) {
    if (!m || !tokens || !next) return fail(LLM_ERR_NULL_PTR, "model, tokens or next is NULL");
    if (!m->cfg.has_embed_and_head) return fail(LLM_ERR_BAD_CONFIG, "model has no embedding/lm_head");
    int rc = check_batch(m, B, T);
    if (rc) return rc;
    rc = run_embed(m, tokens, nullptr, B * T);
    if (rc) return rc;
    rc = run_layers(m, B, T, max_keys_after(m, B, T));
    if (rc) return rc;
    rc = run_head(m, B, T, last_nparts(m, B * T), next, logits);
    if (rc) return rc;
    for (int b = 0; b < B; ++b) m->host_len[b] += T;
    return LLM_OK;
}

int llm_prefill_hidden(llm_model* m, const float* h_in, int B, int T, float* h_out) {
    if (!m || !h_in || !h_out) return fail(LLM_ERR_NULL_PTR, "model, h_in or h_out is NULL");
    if (!aligned16(h_in) || !aligned16(h_out)) return fail(LLM_ERR_BAD_ARG, "h_in and h_out must be 16-byte aligned");
    int rc = check_batch(m, B, T);
    if (rc) return rc;
    rc = run_embed(m, nullptr, h_in, B * T);
    if (rc) return rc;
    rc = run_layers(m, B, T, max_keys_after(m, B, T));
    if (rc) return rc;
    {
        KTimer timer(m, LLM_K_OUT);
        CK(launch_finish_hidden(m->h, h_out, (long long)B * T * m->cfg.dim, m->seq_len, B, T, m->stream, m->pdl));
    }
    for (int b = 0; b < B; ++b) m->host_len[b] += T;
    return LLM_OK;
}

int llm_decode_step(llm_model* m, int B, const int32_t* in_tok, int32_t* next, float* logits) {
    if (!m || !in_tok || !next) return fail(LLM_ERR_NULL_PTR, "model, in_tok or next is NULL");
    if (!m->cfg.has_embed_and_head) return fail(LLM_ERR_BAD_CONFIG, "model has no embedding/lm_head");
    int rc = check_batch(m, B, 1);
    if (rc) return rc;
    const size_t V = (size_t)m->cfg.vocab;
    if (m->cfg.flags & LLM_FLAG_CUDA_GRAPH) {
        const int mk = max_keys_after(m, B, 1);
        // the fused step splits the attention at run time from the cache lengths
        const int ns = m->fused ? 0
                                : attn_decode_plan(B, 1, m->cfg.n_heads, m->cfg.n_kv_heads, m->cfg.head_dim, mk,
                                                   m->num_sms).n_splits;
        const auto key = std::make_tuple(B, ns, logits ? 1 : 0);
        auto it = m->graphs.find(key);
        if (it == m->graphs.end()) {
            cudaGraph_t graph = nullptr;
            CK(cudaStreamBeginCapture(m->stream, cudaStreamCaptureModeThreadLocal));
            m->capturing = true;
            m->cap_recs.clear();
            rc = decode_core(m, B, m->d_tok, m->d_next, logits ? m->d_logits : nullptr);
            m->capturing = false;
            cudaError_t ec = cudaStreamEndCapture(m->stream, &graph);
            if (rc) {
                if (graph) cudaGraphDestroy(graph);
                return rc;
            }
            if (ec != cudaSuccess) return fail(LLM_ERR_CUDA, "graph capture: %s", cudaGetErrorString(ec));
            cudaGraphExec_t exec = nullptr;
            ec = cudaGraphInstantiate(&exec, graph, 0);
            cudaGraphDestroy(graph);
            if (ec != cudaSuccess) return fail(LLM_ERR_CUDA, "graph instantiate: %s", cudaGetErrorString(ec));
            it = m->graphs.emplace(key, llm_model::Graph{exec, m->cap_recs}).first;
            m->cap_recs.clear();
        }
        CK(cudaMemcpyAsync(m->d_tok, in_tok, (size_t)B * 4, cudaMemcpyDeviceToDevice, m->stream));
        CK(cudaGraphLaunch(it->second.exec, m->stream));
        if (!it->second.recs.empty()) {  // timing: read this replay's event pairs
            CK(cudaStreamSynchronize(m->stream));
            for (const auto& r : it->second.recs) {
                float ms = 0.f;
                CK(cudaEventElapsedTime(&ms, r.a, r.b));
                m->kt_ms[r.kind] += ms;
                m->kt_n[r.kind] += 1;
            }
        }
        CK(cudaMemcpyAsync(next, m->d_next, (size_t)B * 4, cudaMemcpyDeviceToDevice, m->stream));
        if (logits)
            CK(cudaMemcpyAsync(logits, m->d_logits, (size_t)B * V * 4, cudaMemcpyDeviceToDevice, m->stream));
    } else {
        rc = decode_core(m, B, in_tok, next, logits);
        if (rc) return rc;
    }
    for (int b = 0; b < B; ++b) m->host_len[b] += 1;
    return LLM_OK;
}

int llm_decode_step_hidden(llm_model* m, int B, const float* h_in, float* h_out) {
    if (!m || !m->fused) return llm_prefill_hidden(m, h_in, B, 1, h_out);
    if (!h_in || !h_out) return fail(LLM_ERR_NULL_PTR, "h_in or h_out is NULL");
    if (!aligned16(h_in) || !aligned16(h_out)) return fail(LLM_ERR_BAD_ARG, "h_in and h_out must be 16-byte aligned");
    int rc = check_batch(m, B, 1);
    if (rc) return rc;
    rc = run_fused_step(m, B, nullptr, h_in, h_out, nullptr, nullptr);
    if (rc) return rc;
    for (int b = 0; b < B; ++b) m->host_len[b] += 1;
    return LLM_OK;
}

int llm_kv_cache_reset(llm_model* m) {
    if (!m) return fail(LLM_ERR_NULL_PTR, "model is NULL");
    CK(cudaMemsetAsync(m->seq_len, 0, (size_t)m->cfg.max_batch * 4, m->stream));
    for (auto& x : m->host_len) x = 0;
    return LLM_OK;
}

int llm_kv_cache_view(llm_model* m, void** k, void** v, int64_t strides[4]) {
    if (!m || !k || !v || !strides) return fail(LLM_ERR_NULL_PTR, "NULL argument");
    const llm_config& c = m->cfg;
    *k = m->kc;
    *v = m->vc;
    strides[3] = c.head_dim;
    strides[2] = (int64_t)c.max_seq_len * c.head_dim;
    strides[1] = (int64_t)c.n_kv_heads * strides[2];
    strides[0] = (int64_t)c.max_batch * strides[1];
    return LLM_OK;
}

int llm_kv_cache_set_lens(llm_model* m, const int32_t* lens, int B) {
    if (!m || !lens) return fail(LLM_ERR_NULL_PTR, "NULL argument");
    if (B < 1 || B > m->cfg.max_batch) return fail(LLM_ERR_BATCH, "B=%d outside [1, %d]", B, m->cfg.max_batch);
    for (int b = 0; b < B; ++b)
        if (lens[b] < 0 || lens[b] > m->cfg.max_seq_len) return fail(LLM_ERR_SEQ_OVERFLOW, "length %d out of range", lens[b]);
    CK(cudaMemcpyAsync(m->seq_len, lens, (size_t)B * 4, cudaMemcpyHostToDevice, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    for (int b = 0; b < B; ++b) m->host_len[b] = lens[b];
    return LLM_OK;
}

int llm_kv_cache_get_lens(llm_model* m, int32_t* lens, int B) {
    if (!m || !lens) return fail(LLM_ERR_NULL_PTR, "NULL argument");
    if (B < 1 || B > m->cfg.max_batch) return fail(LLM_ERR_BATCH, "B=%d outside [1, %d]", B, m->cfg.max_batch);
    CK(cudaMemcpyAsync(lens, m->seq_len, (size_t)B * 4, cudaMemcpyDeviceToHost, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    return LLM_OK;
}

int llm_debug_tap(llm_model* m, int layer, float* dst, size_t dst_elems) {
    if (!m || !dst) return fail(LLM_ERR_NULL_PTR, "NULL argument");
    if (!m->taps) return fail(LLM_ERR_BAD_CONFIG, "model built without LLM_FLAG_DEBUG_TAPS");
    if (layer < 0 || layer >= m->cfg.n_layers) return fail(LLM_ERR_BAD_ARG, "layer %d out of range", layer);
    const size_t n = (size_t)m->taps_tokens * m->cfg.dim;
    if (dst_elems < n) return fail(LLM_ERR_BAD_ARG, "dst holds %zu elements, need %zu", dst_elems, n);
    CK(cudaMemcpyAsync(dst, m->taps + (size_t)layer * m->M_max * m->cfg.dim, n * 4, cudaMemcpyDeviceToDevice,
                       m->stream));
    return LLM_OK;
}

int llm_kernel_times(llm_model* m, int n, double* total_ms, int64_t* launches, int reset) {
    if (!m || (n > 0 && (!total_ms || !launches))) return fail(LLM_ERR_NULL_PTR, "NULL argument");
    CK(cudaStreamSynchronize(m->stream));
    for (const auto& r : m->trecs) {
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, r.a, r.b));
        m->kt_ms[r.kind] += ms;
        m->kt_n[r.kind] += 1;
        m->ev_pool.push_back(r.a);
        m->ev_pool.push_back(r.b);
    }
    m->trecs.clear();
    for (int i = 0; i < n; ++i) {
        total_ms[i] = i < LLM_K_COUNT ? m->kt_ms[i] : 0.0;
        launches[i] = i < LLM_K_COUNT ? m->kt_n[i] : 0;
    }
    if (reset)
        for (int i = 0; i < LLM_K_COUNT; ++i) {
            m->kt_ms[i] = 0.0;
            m->kt_n[i] = 0;
        }
    return LLM_OK;
}

int llm_debug_wait_probe(llm_model* m, int which, double limit_ms) {
    if (!m) return fail(LLM_ERR_NULL_PTR, "model is NULL");
    if ((which != 0 && which != 1) || !(limit_ms > 0.0) || limit_ms > 10000.0)
        return fail(LLM_ERR_BAD_ARG, "which must be 0 or 1 and limit_ms in (0, 10000]");
    CK(launch_wait_probe(which, (uint64_t)(limit_ms * 1e6), m->d_err, m->probe_cnt, m->stream));
    return LLM_OK;
}

// The status of a nonzero device error word (bounds-check codes carry their site).
static int device_error(uint32_t err) {
    if ((err & 0xFF000000u) == lfw::DERR_BOUNDS) {
        static const char* site[] = {"?", "token id outside [0, vocab)", "KV-cache append position outside [0, max_seq_len)",
                                     "RoPE table row outside [0, max_seq_len)", "attention over positions beyond the cache",
                                     "cache length advanced past max_seq_len", "decode position outside [0, max_seq_len)"};
        const uint32_t s = err & 0xFFu;
        return fail(LLM_ERR_DEVICE_BOUNDS, "device bounds check failed: %s (code 0x%x)", site[s < 7 ? s : 0], err);
    }
    return fail(LLM_ERR_DEVICE_TIMEOUT, "device wait timed out (code 0x%x)", err);
}

int llm_synchronize(llm_model* m) {
    if (!m) return fail(LLM_ERR_NULL_PTR, "model is NULL");
    CK(cudaStreamSynchronize(m->stream));
    uint32_t err = 0;
    CK(cudaMemcpy(&err, m->d_err, 4, cudaMemcpyDeviceToHost));
    if (err) {
        cudaMemset(m->d_err, 0, 4);
        return device_error(err);
    }
    return LLM_OK;
}

int llm_build_flags(void) {
#ifdef LLM_BOUNDS_CHECK
    return LLM_BUILD_BOUNDS_CHECK;
#else
    return 0;
#endif
}

// ---------------------------------------------------------------- single operations
static uint32_t* op_err_ptr() {
    uint32_t* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_op_err) != cudaSuccess) return nullptr;
    return p;
}

int llm_op_synchronize(void* stream) {
    CK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    uint32_t* p = op_err_ptr();
    if (!p) return fail(LLM_ERR_CUDA, "cudaGetSymbolAddress of the operations' error word failed");
    uint32_t err = 0;
    CK(cudaMemcpy(&err, p, 4, cudaMemcpyDeviceToHost));
    if (err) {
        cudaMemset(p, 0, 4);
        return device_error(err);
    }
    return LLM_OK;
}

int llm_op_gemm_bf16(const void* A, const void* B, float* C, int M, int N, int K, void* stream) {
    if (!A || !B || !C) return fail(LLM_ERR_NULL_PTR, "NULL operand");
    if (M < 1 || N < 1 || K < 1 || K % GEMM_BK != 0 || N % GEMM_BN != 0)
        return fail(LLM_ERR_BAD_ARG, "need M >= 1, K %% 64 == 0, N %% 256 == 0");
    if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return fail(LLM_ERR_BAD_ARG, "operands must be 16-byte aligned");
    CUtensorMap ta, tb;
    if (!make_tmap(&ta, A, K, M, 64, 128) || !make_tmap(&tb, B, K, N, 64, 128))
        return fail(LLM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    GemmArgs ga;
    ga.tmA = &ta;
    ga.tmB[0] = &tb;
    ga.seg_cols[0] = N;
    ga.M = M;
    ga.N = N;
    ga.K = K;
    ga.num_sms = num_sms_current();
    ga.epi.kind = EPI_STORE_F32;
    ga.epi.M = M;
    ga.epi.y = C;
    ga.epi.ldy = N;
    ga.epi.err = op_err_ptr();
    CK(launch_gemm_tc(ga, reinterpret_cast<cudaStream_t>(stream), false));
    return LLM_OK;
}

// Workspace layout of the single-operation GEMV: [tile counters | packed maxima
// | done counter | partial fragments], each part 256-byte aligned.
static size_t gemv_ws_layout(int N, int K, size_t* off_part, GemvScratch* ws, void* base) {
    const int sms = num_sms_current();
    const int tiles = gemv_num_tiles(EPI_STORE_F32, N);
    const size_t pf = gemv_scratch_floats(EPI_STORE_F32, N, K, sms);
    const size_t o_wcnt = 0;
    const size_t o_best = (o_wcnt + (size_t)tiles * 8 * 4 + 255) & ~size_t(255);
    const size_t o_done = o_best + 256;
    const size_t o_part = o_done + 256;
    if (off_part) *off_part = o_part;
    if (ws && base) {
        char* b = reinterpret_cast<char*>(base);
        ws->warp_cnt = reinterpret_cast<unsigned*>(b + o_wcnt);
        ws->tiles_cap = tiles;
        ws->am_best = reinterpret_cast<unsigned long long*>(b + o_best);
        ws->done_cnt = reinterpret_cast<unsigned*>(b + o_done);
        ws->part = reinterpret_cast<float*>(b + o_part);
        ws->part_floats = pf;
    }
    return o_part + pf * 4;
}

size_t llm_op_gemv_workspace(int N, int K) {
    if (N < 1 || K < 8 || K % 8 != 0) return 0;
    return gemv_ws_layout(N, K, nullptr, nullptr, nullptr);
}

int llm_op_gemv_bf16(const void* x, const void* W, float* y, int M, int N, int K, void* workspace,
                     size_t workspace_bytes, void* stream) {
    if (!x || !W || !y || !workspace) return fail(LLM_ERR_NULL_PTR, "NULL operand or workspace");
    if (M < 1 || M > 16 || N < 1 || K < 8 || K % 8 != 0) return fail(LLM_ERR_BAD_ARG, "need 1 <= M <= 16, K %% 8 == 0");
    if (!aligned16(x) || !aligned16(W) || !aligned16(workspace))
        return fail(LLM_ERR_BAD_ARG, "operands must be 16-byte aligned");
    GemvArgs<__nv_bfloat16> ga;
    size_t off_part = 0;
    if (workspace_bytes < gemv_ws_layout(N, K, &off_part, &ga.ws, workspace))
        return fail(LLM_ERR_BAD_ARG, "workspace too small");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    CK(cudaMemsetAsync(workspace, 0, off_part, s));
    CUtensorMap tw;
    if (!make_tmap(&tw, W, K, N, 64, 128)) return fail(LLM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    ga.tmw[0] = &tw;
    ga.W[0] = reinterpret_cast<const __nv_bfloat16*>(W);
    ga.N = N;
    ga.K = K;
    ga.x = reinterpret_cast<const __nv_bfloat16*>(x);
    ga.ldx = K;
    ga.M = M;
    ga.num_sms = num_sms_current();
    ga.epi.kind = EPI_STORE_F32;
    ga.epi.M = M;
    ga.epi.y = y;
    ga.epi.ldy = N;
    CK(launch_gemv_bf16(ga, s, false));
    return LLM_OK;
}

int llm_op_attention_prefill(const void* q, const void* kcache, const void* vcache, const int32_t* pos0, void* out,
                             int B, int T, int H, int Hk, int d, int S_max, int dtype, void* stream) {
    int rc = lfw::attn_op_check(q, kcache, vcache, pos0, out, B, T, H, Hk, d, S_max, dtype);
    if (rc) return rc;
    if (dtype != LLM_BF16 || d != 128) return fail(LLM_ERR_UNSUPPORTED, "flash kernel needs bf16 and d == 128");
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)B * Hk * S_max;
    if (!make_tmap(&tk, kcache, d, rows, 64, 64) || !make_tmap(&tv, vcache, d, rows, 64, 64))
        return fail(LLM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    AttnPrefillArgs a;
    a.tmK = &tk;
    a.tmV = &tv;
    a.row_base = 0;
    a.S_max = S_max;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.pos0 = pos0;
    a.B = B;
    a.T = T;
    a.H = H;
    a.Hk = Hk;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
    a.err = op_err_ptr();
    CK(launch_attn_prefill(a, reinterpret_cast<cudaStream_t>(stream), false));
    return LLM_OK;
}

size_t llm_op_attention_decode_workspace(int B, int T, int H, int Hk, int d) {
    if (B < 1 || T < 1 || H < 1 || Hk < 1 || H % Hk != 0 || d < 1) return 0;
    const AttnDecodePlan p = attn_decode_plan(B, T, H, Hk, d, 1 << 30, num_sms_current());
    return ((p.part_floats * 4 + 255) & ~size_t(255)) + p.counters * 4;
}

int llm_op_attention_decode(const void* q, const void* kcache, const void* vcache, const int32_t* pos0, void* out,
                            int B, int T, int H, int Hk, int d, int S_max, int dtype, void* workspace,
                            size_t workspace_bytes, void* stream) {
    int rc = lfw::attn_op_check(q, kcache, vcache, pos0, out, B, T, H, Hk, d, S_max, dtype);
    if (rc) return rc;
    if (!workspace) return fail(LLM_ERR_NULL_PTR, "workspace is NULL");
    // planned for keys up to the cache length; the workspace size (any length) covers it
    const AttnDecodePlan p = attn_decode_plan(B, T, H, Hk, d, S_max, num_sms_current());
    const size_t part_bytes = (p.part_floats * 4 + 255) & ~size_t(255);
    if (workspace_bytes < part_bytes + p.counters * 4 || !aligned16(workspace))
        return fail(LLM_ERR_BAD_ARG, "workspace too small or misaligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    AttnDecodeArgs a;
    a.q = q;
    a.kc = kcache;
    a.vc = vcache;
    a.out = out;
    a.pos0 = pos0;
    a.B = B;
    a.T = T;
    a.H = H;
    a.Hk = Hk;
    a.d = d;
    a.S_max = S_max;
    a.n_splits = p.n_splits;
    a.rows = p.rows;
    a.n_qchunks = p.n_qchunks;
    a.ws_part = reinterpret_cast<float*>(workspace);
    a.ws_count = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(workspace) + part_bytes);
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
    a.err = op_err_ptr();
    CK(cudaMemsetAsync(a.ws_count, 0, p.counters * 4, s));
    CK(launch_attn_decode(a, dtype == LLM_BF16, s, false));
    return LLM_OK;
}

int llm_op_attention_decode_cluster(const void* q, const void* kcache, const void* vcache, const int32_t* pos0,
                                    void* out, int B, int H, int Hk, int S_max, void* stream) {
    int rc = lfw::attn_op_check(q, kcache, vcache, pos0, out, B, 1, H, Hk, 128, S_max, LLM_BF16);
    if (rc) return rc;
    const int cs = attn_cluster_size(B, H, Hk, 128, num_sms_current());
    if (cs < 1) return fail(LLM_ERR_UNSUPPORTED, "cluster attention does not support this shape");
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)B * Hk * S_max;
    if (!make_tmap(&tk, kcache, 128, rows, 64, 32) || !make_tmap(&tv, vcache, 128, rows, 64, 32))
        return fail(LLM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    AttnClusterArgs a;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.pos0 = pos0;
    a.B = B;
    a.H = H;
    a.Hk = Hk;
    a.S_max = S_max;
    a.row_base = 0;
    a.rows_per_seq = (long long)Hk * S_max;
    a.cs = cs;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt(128.0));
    a.err = op_err_ptr();
    CK(launch_attn_cluster(a, &tk, &tv, reinterpret_cast<cudaStream_t>(stream)));
    return LLM_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- shared with attn_decode_static.cu
uint32_t* lfw::op_err_word() { return op_err_ptr(); }

int lfw::attn_op_check(const void* q, const void* kc, const void* vc, const int32_t* pos0, const void* out, int B,
                       int T, int H, int Hk, int d, int S_max, int dtype) {
    if (!q || !kc || !vc || !pos0 || !out) return fail(LLM_ERR_NULL_PTR, "NULL operand");
    if (B < 1 || T < 1 || H < 1 || Hk < 1 || H % Hk != 0 || S_max < 1 || d < 8 || d % 8 != 0 || d > 128)
        return fail(LLM_ERR_BAD_ARG, "bad attention shape");
    if (dtype != LLM_F32 && dtype != LLM_BF16) return fail(LLM_ERR_BAD_ARG, "bad dtype");
    if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(out))
        return fail(LLM_ERR_BAD_ARG, "operands must be 16-byte aligned");
    return LLM_OK;
}
