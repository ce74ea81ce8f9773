// Split-KV decode attention for callers that cannot allocate device memory.
//
// llm_op_attention_decode takes its scratch (per-split partial results and
// merge counters) from the caller. Some callers cannot provide it: code that
// runs while a stream is being captured into a CUDA graph (cudaMalloc is not a
// stream operation and cannot be captured), plug-ins whose host application
// owns every device allocation, and latency-critical loops where an allocation
// could synchronise the device. This entry point runs the same kernel, with the
// same argument checks, split plan and error word, on a fixed-size scratch array
// that lives in this file, so a call allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it until the process exits. In host code its name is only a
// host-side stand-in, not a device address; the real address is looked up with
// cudaGetSymbolAddress, with the device current, the first time the entry point
// runs in a CUDA context (so once per device, and again after cudaDeviceReset
// has replaced the device's primary context). That first call should come
// before any stream capture.
#include "../../include/llama_fwd.h"
#include "kernels.cuh"

#include <math.h>
#include <mutex>

namespace {

constexpr size_t kScratchPartBytes = 8u << 20;  // per-split partial results
constexpr size_t kScratchCountBytes = 16u << 10;  // merge counters (4 bytes each)
constexpr size_t kScratchBytes = kScratchPartBytes + kScratchCountBytes;

__device__ __align__(256) unsigned char g_attn_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct Slot {
    void* ctx;   // the CUDA context the address belongs to
    void* addr;  // device address of g_attn_scratch in it
};
Slot g_slot[kMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);

// The driver's cuCtxGetCurrent, through the runtime's entry-point query (the
// library does not link libcuda directly).
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    return fn;
}

// Device address of the scratch array in the current context, looked up on the
// first call in that context.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CtxGetCurrentFn get = ctx_get_current();
    void* ctx = nullptr;
    if (!get || get(&ctx) != 0) return cudaErrorDeviceUninitialized;
    if (!ctx) {
        // no context yet: a runtime call on the device creates its primary context
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attn_scratch);
        if (e != cudaSuccess) return e;
        if (get(&ctx) != 0 || !ctx) return cudaErrorDeviceUninitialized;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_slot[dev].ctx != ctx || !g_slot[dev].addr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attn_scratch);
        if (e != cudaSuccess) return e;
        g_slot[dev].ctx = ctx;
        g_slot[dev].addr = p;
    }
    *out = g_slot[dev].addr;
    return cudaSuccess;
}

}  // namespace

extern "C" int llm_op_attention_decode_static(const void* q, const void* kcache, const void* vcache,
                                              const int32_t* pos0, void* out, int B, int T, int H, int Hk, int d,
                                              int S_max, int dtype, void* stream) {
    int rc = lfw::attn_op_check(q, kcache, vcache, pos0, out, B, T, H, Hk, d, S_max, dtype);
    if (rc) return rc;
    // planned for keys up to the cache length, as llm_op_attention_decode plans
    const lfw::AttnDecodePlan plan = lfw::attn_decode_plan(B, T, H, Hk, d, S_max, lfw::current_num_sms());
    // Sizes beyond the fixed scratch are rejected before anything is queued.
    if (plan.part_floats * 4 > kScratchPartBytes || plan.counters * 4 > kScratchCountBytes)
        return lfw::set_error(LLM_ERR_BAD_ARG,
                              "attention shape needs more than the static scratch (8 MiB of partials, 4096 counters)");
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess)
        return lfw::set_error(LLM_ERR_CUDA, "cudaGetSymbolAddress of the static attention scratch failed");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    lfw::AttnDecodeArgs a;
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
    a.n_splits = plan.n_splits;
    a.rows = plan.rows;
    a.n_qchunks = plan.n_qchunks;
    a.ws_part = reinterpret_cast<float*>(base);
    a.ws_count = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(base) + kScratchPartBytes);
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
    a.err = lfw::op_err_word();
    // The counters must start at zero; the previous call's partials need no clearing.
    if (cudaMemsetAsync(a.ws_count, 0, plan.counters * 4, s) != cudaSuccess)
        return lfw::set_error(LLM_ERR_CUDA, "cudaMemsetAsync of the attention counters failed");
    if (lfw::launch_attn_decode(a, dtype == LLM_BF16, s, false) != cudaSuccess)
        return lfw::set_error(LLM_ERR_CUDA, "attention kernel launch failed");
    return LLM_OK;
}
