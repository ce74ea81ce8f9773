/*
 * llama_fwd.h: C ABI of a Llama-2/3 decoder forward pass (prefill plus
 * KV-cached greedy decode) on one NVIDIA B200 (sm_100a).
 *
 * What the calls compute. The pages this library follows define the
 * decoder step by step, and every call below names its source by page title and
 * section:
 *   - "Building llama3 from scratch": params.json fields (the config struct), the
 *     checkpoint tensor names and [out, in] shapes (the weights struct), the
 *     embedding lookup, the RMSNorm code block, the per-head view of wq.
 *   - "Model Llama 3 yang Diimplementasikan dengan NumPy Murni" (llama3.np):
 *     "RoPE #1/#2", "QKV", "KV cache", "GQA", "Scaled Dot-Product Attention",
 *     "Feed Forward", "Linear" (last-position logits), "Generasi" (prefill and
 *     decode phases).
 *   - "Resumen de una implementación desde cero del modelo LLaMA-3": attention
 *     with a future-token mask and softmax, multi-head concat, SwiGLU, residuals,
 *     final RMSNorm, logits, argmax as the next token.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers on the model's device;
 *     "host" pointers are ordinary CPU memory.
 *   - Matrices are row-major. Weight matrices are [out, in]: y = x W^T.
 *   - Work is queued on the model's CUDA stream and is asynchronous: device
 *     outputs are valid after llm_synchronize() or a sync of that stream.
 *   - Every int-returning call returns LLM_OK (0) or a negative LLM_ERR_* code
 *     and never aborts the process. llm_last_error() gives a message for the
 *     last failure on the calling thread.
 *   - Argument errors (null pointers, sizes beyond the limits given at init,
 *     unsupported shapes) are detected on the host before anything is queued.
 *   - Device-side waits are bounded; a wait that runs out sets the model's
 *     error word, which llm_synchronize() reports as LLM_ERR_DEVICE_TIMEOUT.
 *   - The library also comes as a bounds-checking build (liblfwd_checked.so,
 *     compiled with -DLLM_BOUNDS_CHECK, same entry points): before the accesses
 *     whose indices come from run-time data (token ids, cache positions and
 *     lengths) its kernels check them; a failed check skips the access and sets
 *     the error word, which llm_synchronize() (or llm_op_synchronize() for the
 *     single operations) reports as LLM_ERR_DEVICE_BOUNDS, naming the check.
 *     The normal build compiles these checks out (it clamps token ids).
 */
#ifndef LLAMA_FWD_H
#define LLAMA_FWD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define LLM_OK                   0
#define LLM_ERR_BAD_CONFIG      (-1)  /* inconsistent or unsupported config */
#define LLM_ERR_NULL_PTR        (-2)  /* a required pointer is NULL */
#define LLM_ERR_SEQ_OVERFLOW    (-3)  /* cache length + new tokens > max_seq_len */
#define LLM_ERR_BATCH           (-4)  /* B < 1, B > max_batch, or B*T > max_tokens */
#define LLM_ERR_CUDA            (-5)  /* a CUDA runtime/driver call failed */
#define LLM_ERR_DEVICE_TIMEOUT  (-6)  /* a bounded device-side wait ran out */
#define LLM_ERR_UNSUPPORTED     (-7)  /* valid request this build does not implement */
#define LLM_ERR_BAD_ARG         (-8)  /* other invalid argument (e.g. a size) */
#define LLM_ERR_DEVICE_BOUNDS   (-9)  /* a device-side index check failed
                                         (bounds-checking build only) */

/* ---- build flags (llm_build_flags) -------------------------------------- */
#define LLM_BUILD_BOUNDS_CHECK  1   /* compiled with -DLLM_BOUNDS_CHECK */

/* ---- element types ----------------------------------------------------- */
#define LLM_F32   0   /* weights, activations and KV cache in fp32 */
#define LLM_BF16  1   /* bf16 weights/activations/KV cache, fp32 accumulation
                         and fp32 residual stream */

/* ---- config flags ------------------------------------------------------ */
#define LLM_FLAG_CUDA_GRAPH  1  /* replay decode steps from captured CUDA graphs */
#define LLM_FLAG_DEBUG_TAPS  2  /* keep each layer's output hidden state (see llm_debug_tap) */
#define LLM_FLAG_KERNEL_TIMING 4 /* time every launch with CUDA events (see llm_kernel_times);
                                    with LLM_FLAG_CUDA_GRAPH the events are nodes of the decode
                                    graph and each decode step synchronises to read them */
#define LLM_FLAG_PDL           8 /* let each kernel launch while the previous one drains
                                    (programmatic dependent launch); off by default because it
                                    unbalances the persistent one-CTA-per-SM projections */
#define LLM_FLAG_FUSED_DECODE  16 /* run each bf16 decode step as one persistent launch (the
                                    whole model: every layer's projections and attention and the
                                    lm_head, separated by grid barriers) instead of one launch per
                                    projection and attention; needs head_dim 128, a dim that is
                                    a multiple of 256 and at most 16 query heads per KV head,
                                    and is not used with LLM_FLAG_DEBUG_TAPS; other models
                                    decode with the per-kernel path */

/* ---- kernel kinds reported by llm_kernel_times ------------------------- */
#define LLM_K_EMBED    0   /* embedding lookup / hidden-state load */
#define LLM_K_QKV      1   /* QKV projection + RoPE + KV-cache append */
#define LLM_K_ATTN     2   /* attention (flash or split-KV) */
#define LLM_K_WO       3   /* wo projection + residual */
#define LLM_K_W13      4   /* w1/w3 projection + SwiGLU */
#define LLM_K_W2       5   /* w2 projection + residual */
#define LLM_K_HEAD     6   /* final norm + lm_head + argmax */
#define LLM_K_OUT      7   /* hidden-state output */
#define LLM_K_STEP     8   /* fused decode step: the whole model in one launch */
#define LLM_K_COUNT    9

/*
 * Model hyper-parameters: the params.json fields of "Building llama3 from
 * scratch" (dim, n_layers, n_heads, n_kv_heads, vocab_size, norm_eps, rope_theta),
 * plus the FFN hidden size given explicitly and the capacity limits.
 *   head_dim       must equal dim / n_heads, be a multiple of 8 and at most
 *                  128; n_heads % n_kv_heads == 0 (any group size: multi-head,
 *                  grouped-query, multi-query).
 *   dim, ffn_hidden multiples of 8; for LLM_BF16 also n_heads*head_dim and
 *                  n_kv_heads*head_dim multiples of 128.
 *   max_seq_len    KV-cache positions per sequence.
 *   max_batch      sequences (B) per call, at most 16.
 *   max_tokens     B*T per prefill call (0 means max_batch * max_seq_len).
 *   dtype          LLM_F32 or LLM_BF16 (type of every weight buffer).
 *   tie_embeddings lm_head reuses tok_emb (weights.out ignored).
 *   has_embed_and_head  0 for a bare layer stack driven by the *_hidden calls.
 */
typedef struct llm_config {
    int dim, n_layers, n_heads, n_kv_heads, head_dim, ffn_hidden, vocab;
    int max_seq_len, max_batch, max_tokens;
    float norm_eps, rope_theta;
    int dtype;
    int tie_embeddings;
    int has_embed_and_head;
    int flags;
} llm_config;

/*
 * Weights: device pointers of element type config.dtype, owned by the caller,
 * which must keep them alive and unchanged until llm_model_free(). Names follow
 * the checkpoint keys listed in "Building llama3 from scratch". Per-layer
 * fields are host arrays of n_layers device pointers (copied at init).
 *   tok_emb    [vocab, dim]          (NULL when has_embed_and_head == 0)
 *   out        [vocab, dim]          lm_head; NULL when tied
 *   final_norm [dim]
 *   attn_norm, ffn_norm [dim]
 *   wq [n_heads*head_dim, dim], wk/wv [n_kv_heads*head_dim, dim],
 *   wo [dim, n_heads*head_dim], w1/w3 [ffn_hidden, dim], w2 [dim, ffn_hidden]
 * Every device pointer must be 16-byte aligned.
 */
typedef struct llm_weights {
    const void *tok_emb, *out, *final_norm;
    const void *const *attn_norm, *const *wq, *const *wk, *const *wv, *const *wo;
    const void *const *ffn_norm, *const *w1, *const *w3, *const *w2;
} llm_weights;

typedef struct llm_model llm_model;

/*
 * Create a model on the current CUDA device. stream is a cudaStream_t on which
 * every later call queues its work; NULL makes the model create and own a
 * blocking stream (ordered with the legacy default stream) instead. The
 * library allocates and owns the KV cache [n_layers][max_batch][n_kv_heads]
 * [max_seq_len][head_dim] (element type dtype), the RoPE cos/sin tables, the
 * activations and the scratch; llm_model_free() releases them. All cache
 * lengths start at 0. On failure *out is NULL.
 */
int llm_model_init(const llm_config* cfg, const llm_weights* w, void* stream, llm_model** out);

/*
 * Prefill phase ("Generasi": the whole prompt at once). tokens: device int32
 * [B, T]. Sequence b's tokens take positions len[b] .. len[b]+T-1, where len[b]
 * is its current cache length (0 after init/reset); their K and V are appended to
 * the cache and len[b] grows by T. Writes next[b] (device int32 [B]) = argmax of
 * the logits at the last position (ties: lowest id), and, when logits is not
 * NULL, those logits (device fp32 [B, vocab]).
 * Errors: NULL_PTR, BATCH, SEQ_OVERFLOW, BAD_CONFIG (model built without
 * embedding/head).
 */
int llm_prefill(llm_model* m, const int32_t* tokens, int B, int T, int32_t* next, float* logits);

/*
 * Prefill of the layer stack on given hidden states, with no embedding, final
 * norm or lm_head. h_in: device fp32 [B, T, dim]; h_out: device fp32 [B, T, dim],
 * the last layer's output; both 16-byte aligned (else LLM_ERR_BAD_ARG).
 * Positions and cache growth as in llm_prefill.
 */
int llm_prefill_hidden(llm_model* m, const float* h_in, int B, int T, float* h_out);

/*
 * One decode step ("KV cache": only the newest token is projected; "Generasi":
 * decode phase). in_tok: device int32 [B], the token at position len[b] of
 * sequence b; next: device int32 [B], the greedy next token; logits: optional
 * device fp32 [B, vocab]. Grows len[b] by 1. B may differ from the last
 * prefill's B; sequences b < B are advanced.
 */
int llm_decode_step(llm_model* m, int B, const int32_t* in_tok, int32_t* next, float* logits);

/* As llm_decode_step, on hidden states: h_in, h_out device fp32 [B, dim]. */
int llm_decode_step_hidden(llm_model* m, int B, const float* h_in, float* h_out);

/* Set every sequence's cache length to 0 (cache contents are left in place). */
int llm_kv_cache_reset(llm_model* m);

/*
 * Direct access to the cache for callers that fill it themselves. *k and *v get
 * the device base pointers of K and V (element type dtype; entries hold
 * post-RoPE keys and plain values). strides[0..3] get the element strides of
 * [layer, batch, kv_head, position]; head_dim is contiguous. The memory stays
 * owned by the model.
 */
int llm_kv_cache_view(llm_model* m, void** k, void** v, int64_t strides[4]);

/* Set (host int32 [B]) or read back the cache lengths of sequences 0..B-1. */
int llm_kv_cache_set_lens(llm_model* m, const int32_t* lens, int B);
int llm_kv_cache_get_lens(llm_model* m, int32_t* lens, int B);

/*
 * Copy the output hidden state of decoder layer `layer` (fp32 residual stream,
 * [tokens, dim] with tokens = B*T of the last prefill or B of the last decode
 * step) into dst (device fp32, dst_elems elements at least). Needs
 * LLM_FLAG_DEBUG_TAPS at init.
 */
int llm_debug_tap(llm_model* m, int layer, float* dst, size_t dst_elems);

/*
 * Per-kind kernel time recorded since the last reset (LLM_FLAG_KERNEL_TIMING).
 * Synchronises the stream, then writes total milliseconds and launch counts of
 * kinds 0..n-1 (see LLM_K_*) into the host arrays total_ms[n] and launches[n];
 * reset != 0 clears the record afterwards. Kernels are timed with a CUDA event
 * pair each on the model's stream, so kernels that would otherwise overlap
 * their neighbours' tails run back to back while timing is on. Directly
 * launched kernels include any host launch gap in their time; decode steps
 * replayed from a graph (LLM_FLAG_CUDA_GRAPH) do not.
 */
int llm_kernel_times(llm_model* m, int n, double* total_ms, int64_t* launches, int reset);

/*
 * Failure detection, exercised on purpose: queues on the model's stream a
 * kernel that enters one of the library's bounded device waits with a target
 * that is never reached, bounded by limit_ms (0 < limit_ms <= 10000) instead of
 * the usual 4 s: which = 0 an mbarrier wait for bytes no copy delivers, which = 1
 * a grid barrier of a two-CTA cooperative launch that waits for twice the
 * arrivals its CTAs make.
 * The wait gives up, records its code in the model's device error word and the
 * kernel returns: nothing faults or hangs, and the next llm_synchronize()
 * returns LLM_ERR_DEVICE_TIMEOUT (clearing the word) while the model stays
 * usable. The pages have no counterpart: this is a diagnostic of the library.
 * Returns LLM_OK once queued, LLM_ERR_BAD_ARG or LLM_ERR_CUDA otherwise.
 */
int llm_debug_wait_probe(llm_model* m, int which, double limit_ms);

/* Wait for the model's stream; report a CUDA error, a device-side timeout
 * (LLM_ERR_DEVICE_TIMEOUT) or, in the bounds-checking build, a failed device
 * index check (LLM_ERR_DEVICE_BOUNDS). Clears the model's error word. */
int llm_synchronize(llm_model* m);

/* LLM_BUILD_BOUNDS_CHECK if this library is the bounds-checking build, else 0.
 * A host-only query: needs no GPU. */
int llm_build_flags(void);

/* Release everything the model allocated. NULL is accepted. */
void llm_model_free(llm_model* m);

/* Message describing the last failure on this thread ("" if none). */
const char* llm_last_error(void);

/* ======================================================================
 * Single-operation entry points. Each runs one of the model's kernels on
 * caller-provided device buffers, on `stream` (a cudaStream_t, NULL: default).
 * ==================================================================== */

/* Wait for `stream` and report the single operations' device error word as
 * llm_synchronize() does for a model (a device timeout or, in the
 * bounds-checking build, a failed index check); clears the word. The word is
 * shared by all single operations of the process. */
int llm_op_synchronize(void* stream);

/*
 * C = A B^T on the tensor cores (the prefill projection kernel, tcgen05/TMEM
 * fed by TMA). A: device bf16 [M, K]; B: device bf16 [N, K]; C: device fp32
 * [M, N]. fp32 accumulation. Needs K % 64 == 0, N % 256 == 0, 16-byte aligned
 * pointers; M >= 1 is arbitrary. Source: "Building llama3 from scratch", the
 * projection q_per_token = x @ wq_head^T, here for whole matrices.
 */
int llm_op_gemm_bf16(const void* A, const void* B, float* C, int M, int N, int K, void* stream);

/*
 * y = x W^T for a few rows (the decode projection kernel, streaming W once).
 * x: device bf16 [M, K] with M <= 16; W: device bf16 [N, K]; y: device fp32
 * [M, N]. Needs K % 8 == 0. workspace: device scratch of at least
 * llm_op_gemv_workspace(N, K) bytes, 16-byte aligned, contents arbitrary (the
 * call clears the part it needs); calls sharing one workspace must not overlap
 * in time. The kernel is launched cooperatively (one CTA per SM, all resident
 * at once); where the device cannot host that, the call returns LLM_ERR_CUDA.
 * Source: the per-token projection q_per_token = x @ wq_head^T of
 * "Building llama3 from scratch", for the decode phase of llama3.np "Generasi".
 */
size_t llm_op_gemv_workspace(int N, int K);
int llm_op_gemv_bf16(const void* x, const void* W, float* y, int M, int N, int K, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * Causal grouped-query attention over a KV cache for a block of new tokens
 * ("Implementación de la atención" and "Atención multi-head" in "Resumen ...";
 * "GQA" and "Scaled Dot-Product Attention" in llama3.np).
 *   q:      device [B, T, H, d], element type dtype, RoPE already applied
 *   kcache, vcache: device [B, Hk, S_max, d] (one layer's cache), dtype
 *   pos0:   device int32 [B]; query t of sequence b sits at position pos0[b]+t
 *           and attends to keys 0 .. pos0[b]+t of its sequence
 *   out:    device [B, T, H*d], dtype
 * Scale 1/sqrt(d); query head h reads KV head h / (H/Hk).
 * llm_op_attention_prefill is the flash (tensor-core) kernel: dtype LLM_BF16,
 * d == 128. llm_op_attention_decode is the split-KV kernel: any dtype,
 * d <= 128 with d % 8 == 0, any T and any H/Hk (multi-query included); it
 * splits the keys by the cache length S_max and needs a device scratch buffer of
 * llm_op_attention_decode_workspace(...) bytes (16-byte aligned, contents
 * arbitrary; the kernel leaves it ready for the next call, so calls sharing one
 * buffer must not overlap in time).
 */
int llm_op_attention_prefill(const void* q, const void* kcache, const void* vcache,
                             const int32_t* pos0, void* out, int B, int T, int H, int Hk,
                             int d, int S_max, int dtype, void* stream);
size_t llm_op_attention_decode_workspace(int B, int T, int H, int Hk, int d);
int llm_op_attention_decode(const void* q, const void* kcache, const void* vcache,
                            const int32_t* pos0, void* out, int B, int T, int H, int Hk,
                            int d, int S_max, int dtype, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Decode attention of one new token per sequence on the tensor cores, as the
 * bf16 decode path runs it ("Implementación de la atención"; llama3.np "GQA",
 * "Scaled Dot-Product Attention", "KV cache"): out[b][h] = softmax over keys
 * 0..pos0[b] of q[b][h] . K[b][h/G][j] / sqrt(128), times V[b][h/G][j].
 *   q, out: [B][H*128] bf16; kcache, vcache: [B][Hk][S_max][128] bf16 holding
 *   positions 0..pos0[b] (the new token's key and value included); pos0: [B]
 *   int32 (0 <= pos0[b] < S_max); H a multiple of Hk. Device pointers,
 *   16-byte aligned, owned by the caller; no workspace: a thread-block cluster
 *   per (sequence, KV head, up to 8 of its query heads) streams 32-key K/V
 *   tiles by TMA and merges its CTAs' partial results in distributed shared
 *   memory. The probabilities enter the P V product rounded to bf16 (fp32
 *   accumulation).
 *   Errors: LLM_ERR_NULL_PTR, LLM_ERR_BAD_ARG (shape, alignment), LLM_ERR_CUDA.
 */
int llm_op_attention_decode_cluster(const void* q, const void* kcache, const void* vcache,
                                    const int32_t* pos0, void* out, int B, int H, int Hk,
                                    int S_max, void* stream);

/*
 * The split-KV decode attention of llm_op_attention_decode, for callers that
 * cannot allocate device memory: code running while a stream is captured into
 * a CUDA graph (cudaMalloc cannot be captured), plug-ins whose host
 * application owns every device allocation, and latency-critical loops where
 * an allocation could synchronise the device. The pages have no counterpart:
 * this is a deployment convenience, not a step of the decoder.
 *   Same arguments, checks, split plan (from S_max) and results as
 *   llm_op_attention_decode, without the workspace: the scratch is a fixed
 *   array inside the library (8 MiB of per-split partial results and 4096 merge
 *   counters), held by every GPU that loads the library until the process
 *   exits. The call allocates nothing (no cudaMalloc, cudaFree or allocating
 *   library routine).
 *   Shapes that need more scratch than that return LLM_ERR_BAD_ARG before
 *   anything is queued: a call needs B * Hk * ceil(T * G / rows) * rows *
 *   splits * (d + 4) floats (G = H / Hk; rows = 16 when G >= 16, else
 *   G * min(floor(16 / G), T); splits as llm_op_attention_decode plans them). With 32 query heads,
 *   8 KV heads and head_dim 128, one new token per sequence fits for every
 *   B <= 16 and S_max <= 16384.
 *   The first call in a CUDA context (once per device, and again after
 *   cudaDeviceReset) looks up the array's device address (cudaGetSymbolAddress);
 *   make that first call before any stream capture.
 *   Every call uses the same array and zeroes its counters first, so calls
 *   whose kernels may overlap on the GPU (other streams, other host threads)
 *   race with each other and must not be issued.
 */
int llm_op_attention_decode_static(const void* q, const void* kcache, const void* vcache,
                                   const int32_t* pos0, void* out, int B, int T, int H, int Hk,
                                   int d, int S_max, int dtype, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* LLAMA_FWD_H */
