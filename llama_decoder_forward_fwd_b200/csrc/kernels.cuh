// Parameter blocks and host launchers of the decoder's kernels.
//
// Data layout in device memory (one model):
//   h      fp32 [tokens][dim]            residual stream
//   hw     act  [tokens][dim]            h * (next RMSNorm weight), the projection input;
//                                        its per-row RMS scale is applied in the consumer's epilogue
//   ss     fp32 [parts][ss_ld]           partial sums of h^2 per row, written by the producer of h
//   q      act  [tokens][n_heads*head_dim]      post-RoPE queries
//   o      act  [tokens][n_heads*head_dim]      attention output (heads concatenated)
//   g      act  [tokens][ffn_hidden]     silu(w1 x) * (w3 x)
//   K, V   act  [layer][batch][kv_head][position][head_dim]
// "act" is bf16 for bf16 models and fp32 for fp32 models. A token row m belongs
// to sequence b = m / T at position pos0[b] + (m % T).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace lfw {

enum EpiKind : int {
    EPI_STORE_F32 = 0,  // y[m][n] = acc
    EPI_QKV_ROPE = 1,   // rotate q/k pairs, write q and append k, v to the cache
    EPI_SWIGLU = 2,     // g[m][n] = silu(acc_w1) * acc_w3
    EPI_RESID = 3,      // h[m][n] += acc; hw = h * wnext; partial sum of h^2
    EPI_LOGITS = 4,     // logits (optional) + greedy argmax, last-CTA reduction
};

// The RMSNorm scale of a projection input that was stored as h * w:
// rinv[m] = 1 / sqrt(sum_p ss[p * ld + row0 + m * row_step] / dim + eps).
struct NormIn {
    const float* ss = nullptr;  // nullptr: input is not normed (no scaling)
    int nparts = 0, ld = 0, row0 = 0, row_step = 1;
    float inv_dim = 0.f, eps = 0.f;
};

struct Epi {
    int kind = EPI_STORE_F32;
    int M = 0;  // output rows (tokens)
    int T = 1;  // tokens per sequence
    NormIn norm;
    // EPI_STORE_F32
    float* y = nullptr;
    int ldy = 0;
    // EPI_QKV_ROPE
    const int32_t* pos0 = nullptr;
    const float* rope_cos = nullptr;  // [max_seq][head_dim/2]
    const float* rope_sin = nullptr;
    int H = 0, Hk = 0, d = 0, S_max = 0;
    void* q_out = nullptr;
    void* k_cache = nullptr;  // this layer: [batch][Hk][S_max][d]
    void* v_cache = nullptr;
    // EPI_SWIGLU
    void* g_out = nullptr;
    void* g_lo_out = nullptr;  // bf16 remainder of g (split activations; may be null)
    int F = 0;
    // EPI_RESID
    float* h = nullptr;
    int D = 0;
    void* hw_out = nullptr;
    void* hw_lo_out = nullptr;  // bf16 remainder of hw (split activations; may be null)
    const void* wnext = nullptr;
    float* ss_out = nullptr;
    int ss_out_ld = 0;
    // EPI_LOGITS
    float* logits = nullptr;
    int ld_logits = 0;
    float* am_val = nullptr;  // [tiles][M]
    int* am_idx = nullptr;
    unsigned* am_counter = nullptr;  // zero between launches; the last CTA resets it
    int32_t* next_tok = nullptr;
    int32_t* seq_len = nullptr;  // when set: seq_len[m] += advance, by the last CTA
    int advance = 0;
    uint32_t* err = nullptr;
};

// Tensor maps of one layer's weights, in this order per layer: 128-row boxes
// for the decode projection and the prefill GEMM, and 64-row boxes of w1 and
// w3 for the SwiGLU tiles of the decode projection.
enum { TM_WQ, TM_WK, TM_WV, TM_WO, TM_W1, TM_W3, TM_W2, TM_W1G, TM_W3G, TM_PER_LAYER };

// ---- decode projection: y = x W^T for M <= 16 token rows ---------------
// Device scratch of the streaming bf16 GEMV. Counters and packed maxima must be
// zero before the first launch; every launch leaves them zero again.
struct GemvScratch {
    float* part = nullptr;                  // partial fragments of split tiles
    size_t part_floats = 0;
    int tiles_cap = 0;                      // row tiles the counters below cover
    unsigned long long* am_best = nullptr;  // [16] packed (logit, id) maxima
    unsigned* done_cnt = nullptr;           // [1] tiles finished (argmax)
    unsigned* warp_cnt = nullptr;           // [tiles_cap * 8] pieces published per (tile, warp)
                                            // (fused decode step: the tile's owner waits for them)
};
struct GemvPlan {
    int ntiles, nkb, grid, max_pieces;
    long long TB;
};
GemvPlan gemv_plan(int kind, int N, int K, int num_sms, int occ);
// Partial-buffer floats any launch of this shape can need.
size_t gemv_scratch_floats(int kind, int N, int K, int num_sms);

template <typename T>
struct GemvArgs {
    const T* W[3] = {nullptr, nullptr, nullptr};  // QKV: wq, wk, wv; SWIGLU: w1, w3; else W[0]
    int seg_rows[3] = {0, 0, 0};                  // rows of each segment
    int N = 0;                                    // logical output rows (SWIGLU: ffn_hidden)
    int K = 0;
    const T* x = nullptr;  // [M][ldx]
    const T* x_lo = nullptr;  // bf16 kernel, M <= 8: the bf16 remainders of x (split activations)
    int ldx = 0;
    int M = 0;   // rows in this launch (<= 16)
    int m0 = 0;  // token index of row 0 (the epilogue sees token m0 + m)
    int num_sms = 148;
    GemvScratch ws;                                           // bf16 kernel only
    const CUtensorMap* tmw[3] = {nullptr, nullptr, nullptr};  // bf16 kernel: box 64 x 128 rows
                                                              // (SwiGLU: w1, w3 with 64-row boxes)
    Epi epi;
};
// Row tiles of the bf16 decode projection (128 rows; 64 w1 + 64 w3 rows for SwiGLU).
int gemv_num_tiles(int kind, int N);
// Parts of the RMSNorm partial sums a projection with N output rows writes (one per 16 rows).
inline int gemv_ss_parts(int N) { return (N + 15) / 16; }
cudaError_t launch_gemv_bf16(const GemvArgs<__nv_bfloat16>& a, cudaStream_t s, bool pdl);
cudaError_t launch_gemv_f32(const GemvArgs<float>& a, cudaStream_t s, bool pdl);

// ---- prefill projection on tcgen05 ------------------------------------
struct GemmArgs {
    const CUtensorMap* tmA = nullptr;                          // activations [rows][K] bf16
    const CUtensorMap* tmB[3] = {nullptr, nullptr, nullptr};   // weight segments [rows][K] bf16
    int seg_cols[3] = {0, 0, 0};  // output columns of each segment (SWIGLU: seg 0 = ffn_hidden)
    int M = 0, N = 0, K = 0;      // N: total output columns (SWIGLU: ffn_hidden)
    int num_sms = 148;
    Epi epi;
};
constexpr int GEMM_BM = 128, GEMM_BN = 256, GEMM_BK = 64;
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t s, bool pdl);

// ---- attention --------------------------------------------------------
struct AttnPrefillArgs {
    const CUtensorMap* tmK = nullptr;  // 2-D view of the K cache: [rows][head_dim] bf16
    const CUtensorMap* tmV = nullptr;
    long long row_base = 0;            // cache row of (batch 0, kv head 0, position 0) of this layer
    int S_max = 0;
    const __nv_bfloat16* q = nullptr;  // [B*T][H*d]
    __nv_bfloat16* out = nullptr;      // [B*T][H*d]
    const int32_t* pos0 = nullptr;
    int B = 0, T = 0, H = 0, Hk = 0;
    float scale_log2 = 0.f;            // log2(e) / sqrt(d)
    uint32_t* err = nullptr;
};
cudaError_t launch_attn_prefill(const AttnPrefillArgs& a, cudaStream_t s, bool pdl);

struct AttnDecodeArgs {
    const void* q = nullptr;   // [B*T][H*d]
    const void* kc = nullptr;  // this layer: [batch][Hk][S_max][d]
    const void* vc = nullptr;
    void* out = nullptr;       // [B*T][H*d]
    const int32_t* pos0 = nullptr;
    int B = 0, T = 0, H = 0, Hk = 0, d = 0, S_max = 0;
    // a work item: `rows` consecutive (token, head-in-group) rows r = t*G + h of one KV head
    int n_splits = 1, rows = 1, n_qchunks = 1;
    float* ws_part = nullptr;       // split partials (m, l, o[d])
    unsigned* ws_count = nullptr;   // [B*Hk*n_qchunks], zero between launches
    float scale_log2 = 0.f;
    uint32_t* err = nullptr;
};
struct AttnDecodePlan {
    int n_splits, rows, n_qchunks;
    size_t part_floats, counters;
};
AttnDecodePlan attn_decode_plan(int B, int T, int H, int Hk, int d, int max_keys, int num_sms);
cudaError_t launch_attn_decode(const AttnDecodeArgs& a, bool bf16, cudaStream_t s, bool pdl);

// Decode attention of one new token per sequence on the tensor cores, one
// thread-block cluster per group of up to 8 query heads of one (sequence, KV
// head) (attn_cluster.cu): bf16, head_dim 128. Needs no global scratch.
struct AttnClusterArgs {
    const __nv_bfloat16* q = nullptr;  // [B][H*128]
    __nv_bfloat16* out = nullptr;      // [B][H*128]
    __nv_bfloat16* out_lo = nullptr;   // [B][H*128] bf16 remainder of the output, or null
    const int32_t* pos0 = nullptr;     // [B] position of the new token (cache length before it)
    int B = 0, H = 0, Hk = 0, S_max = 0;
    long long row_base = 0;            // cache row of (sequence 0, KV head 0, position 0) in the maps
    long long rows_per_seq = 0;        // cache rows between consecutive sequences
    int cs = 1;                        // CTAs per group (the cluster size, 1..8)
    float scale_log2 = 0.f;
    uint32_t* err = nullptr;
};
// Groups of the launch, and CTAs per group on num_sms SMs (0: shape not supported).
int attn_cluster_groups(int B, int H, int Hk);
int attn_cluster_size(int B, int H, int Hk, int d, int num_sms);
// tmK, tmV: the K and V caches as [rows][128] bf16 with 32-row, 64-column boxes.
cudaError_t launch_attn_cluster(const AttnClusterArgs& a, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                cudaStream_t s);

// ---- fused decode step (bf16): the whole model in one persistent launch ----
struct DecodeStepArgs {
    int B = 0, D = 0, H = 0, Hk = 0, d = 0, F = 0, vocab = 0, S_max = 0, n_layers = 0;
    float eps = 0.f, scale_log2 = 0.f;
    int has_head = 0;
    int n_stages = 0, xs_bytes = 0;  // shared memory: ring stages; token rows / query tile
    int max_pieces[5] = {1, 1, 1, 1, 1};  // split-tile slots of QKV, wo, w1/w3, w2, lm_head
    // inputs and outputs of the step
    const int32_t* tok = nullptr;  // [B] token ids (models with embedding and head)
    const float* h_in = nullptr;   // [B][D] hidden states (layer stack only)
    float* h_out = nullptr;        // [B][D]
    int32_t* next = nullptr;       // [B] greedy next tokens
    float* logits = nullptr;       // [B][vocab] or nullptr
    // weights
    const CUtensorMap* tmaps = nullptr;  // device: TM_PER_LAYER maps per layer, then the lm_head map,
                                         // then the K and V cache maps (box 64 dims x 32 rows)
    const void* const* norms = nullptr;  // device: attention_norm[l], ffn_norm[l] per layer, then the final norm
    const void* tok_emb = nullptr;
    // state and activations (layouts as above)
    void* kc = nullptr;
    void* vc = nullptr;
    long long layer_elems = 0;        // elements of one layer's K (or V) cache
    long long kv_rows_per_layer = 0;  // its rows of head_dim elements
    int32_t* seq_len = nullptr;
    float* h = nullptr;
    __nv_bfloat16* hw = nullptr;
    float* ss = nullptr;
    int ss_ld = 0;
    __nv_bfloat16* q = nullptr;
    __nv_bfloat16* o = nullptr;
    __nv_bfloat16* g = nullptr;
    const float* rope_cos = nullptr;
    const float* rope_sin = nullptr;
    // scratch (counters zero between launches; *bar zeroed before each launch)
    GemvScratch ws;
    float* attn_part = nullptr;  // per (group, piece, warp): O[R][16], m[R], l[R]
    unsigned* attn_cnt = nullptr;  // per (group, warp), zero between launches
    unsigned* bar = nullptr;
    uint32_t* err = nullptr;
};
struct DecodeStepPlan {
    bool supported;
    int grid, n_stages, xs_bytes, smem;
    int max_pieces[5];
    size_t part_floats;  // split-tile partial floats needed
    int tiles;           // tile counters needed
    size_t attn_part_floats, attn_counters;
};
DecodeStepPlan decode_step_plan(int B, int D, int H, int Hk, int d, int F, int vocab, int has_head, int max_keys,
                                int num_sms, int smem_optin);
cudaError_t launch_decode_step(const DecodeStepArgs& a, const DecodeStepPlan& p, cudaStream_t s);

// ---- small kernels ----------------------------------------------------
struct EmbedArgs {
    const int32_t* tok = nullptr;  // token ids [M] (when h_in is null)
    const void* E = nullptr;       // [vocab][D] model dtype
    const float* h_in = nullptr;   // or given hidden states [M][D]
    float* h = nullptr;
    void* hw = nullptr;
    void* hw_lo = nullptr;         // bf16 models: the remainder hw - bf16(hw), or null
    const void* wnorm = nullptr;   // first layer's attention_norm
    float* ss = nullptr;           // [1][M]
    int M = 0, D = 0, vocab = 0;
    uint32_t* err = nullptr;       // bounds-checking build: out-of-range token ids
};
cudaError_t launch_embed(const EmbedArgs& a, bool bf16, cudaStream_t s, bool pdl);
// h_out = h; seq_len[b] += advance for b < B.
cudaError_t launch_finish_hidden(const float* h, float* h_out, long long n, int32_t* seq_len, int B,
                                 int advance, cudaStream_t s, bool pdl);
cudaError_t launch_rope_tables(float* cosv, float* sinv, int n_pos, int half, double theta, int head_dim,
                               cudaStream_t s);

// A wait that cannot complete, bounded by limit_ns, on the library's own wait
// code: which = 0 an mbarrier expecting bytes that never arrive (one CTA),
// which = 1 a grid barrier of a cooperative launch of two CTAs whose target
// counts three arrivals. Either records its code in *err and returns.
cudaError_t launch_wait_probe(int which, uint64_t limit_ns, uint32_t* err, unsigned* counter, cudaStream_t s);

// Record msg as the calling thread's last error (llm_last_error) and return code.
int set_error(int code, const char* msg);

// Shared by the single-operation attention entry points: argument checks of the
// split-KV and flash attention calls (0 or an LLM_ERR_* code, recorded), the
// device error word their kernels report into, and the current device's SM count.
int attn_op_check(const void* q, const void* kc, const void* vc, const int32_t* pos0, const void* out, int B, int T,
                  int H, int Hk, int d, int S_max, int dtype);
uint32_t* op_err_word();
int current_num_sms();

// Launch helper: programmatic stream serialization when pdl is set.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace lfw
