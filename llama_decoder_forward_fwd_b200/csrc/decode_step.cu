// Fused decode step: one whole decode step of a bf16 model (embedding, every
// layer's QKV projection with RoPE and KV-cache append, attention, wo projection
// with residual, w1/w3 projection with SwiGLU, w2 projection with residual, and
// the lm_head with greedy argmax) in a single persistent launch with one CTA per
// SM ("Resumen ..." and "Predicción de tokens" on "Implementación de LLaMA3 en
// Python puro"; "Transformer Block" on the llama3.np page).
//
// Why one launch: a decode step streams every weight once (16 GB for the 8B
// shape) but runs ~160 dependent projections, each only tens of microseconds
// long. Launched one by one, each pays its pipeline fill and drain, its launch,
// and a tail while its last CTAs finish, and HBM idles in between. Here the
// phases are separated by grid-wide barriers instead of kernel boundaries, and
// the producer warp of every CTA never waits for a phase to end: weights do not
// depend on activations, so it streams the next phase's units into its shared-
// memory ring while the consumers are still in the previous phase (or in the
// attention phase, which reads the KV cache with its own loads). The ring
// (12 stages of 16 KB at the 8B shape, batch 1) keeps HBM busy through each
// barrier.
//
// Phase order per layer: QKV -> attention -> wo -> w1/w3 -> w2, each ending in a
// grid barrier (the data dependency is all-to-all: every projection row needs
// the whole input vector). The arithmetic of each phase is the same code as the
// per-projection kernels (gemv_core.cuh, attn_core.cuh), so results agree with
// the layer-by-layer path up to the split of the k sums over CTAs (which is a
// function of the grid size only, so a given GPU gives bit-identical steps).
//
// Barrier waits, ring waits and the final drain are all bounded; a timeout
// records an error code and every CTA leaves at its next barrier.
#include "attn_core.cuh"
#include "gemv_core.cuh"

#include <math.h>

namespace lfw {

constexpr int DS_THREADS = GV_CONSUMERS + 32;  // 8 consumer warps + 1 producer warp
constexpr int DS_NW = GV_CONSUMERS / 32;
constexpr int DS_MAX_STAGES = 16;
constexpr int DS_MIN_STAGES = 8;
constexpr int DS_SMEM_SLACK = 1024 + 2 * DS_MAX_STAGES * 8 + 64;  // alignment, mbarriers

DEVI int cdiv(int a, int b) { return (a + b - 1) / b; }

DEVI NormIn ds_norm(const DecodeStepArgs& a, int nparts) {
    NormIn n;
    n.ss = a.ss;
    n.nparts = nparts;
    n.ld = a.ss_ld;
    n.row0 = 0;
    n.row_step = 1;
    n.inv_dim = 1.f / (float)a.D;
    n.eps = a.eps;
    return n;
}

// Embedding (or given hidden states) into h, plus the first RMSNorm's inputs:
// hw = h * attention_norm[0] and one partial sum of h^2 per 256 columns.
// One warp per (token, 256-column chunk), 8 columns per lane.
DEVI void ds_embed(const DecodeStepArgs& a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = a.D, nch = D / 256, items = a.B * nch;
    const __nv_bfloat16* wn = reinterpret_cast<const __nv_bfloat16*>(a.norms[0]);
    for (int it = blockIdx.x * DS_NW + warp; it < items; it += gridDim.x * DS_NW) {
        const int m = it / nch, c = it - m * nch;
        const int col = c * 256 + lane * 8;
        float v[8];
        if (a.h_in) {
            const float4 x0 = *reinterpret_cast<const float4*>(a.h_in + (size_t)m * D + col);
            const float4 x1 = *reinterpret_cast<const float4*>(a.h_in + (size_t)m * D + col + 4);
            v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w; v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
        } else {
            int tok = a.tok[m];
            tok = tok < 0 ? 0 : (tok >= a.vocab ? a.vocab - 1 : tok);
            const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.tok_emb) +
                                                            (size_t)tok * D + col);
            v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
            v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
        }
        const uint4 wu = *reinterpret_cast<const uint4*>(wn + col);
        const float w[8] = {bf16lo(wu.x), bf16hi(wu.x), bf16lo(wu.y), bf16hi(wu.y),
                            bf16lo(wu.z), bf16hi(wu.z), bf16lo(wu.w), bf16hi(wu.w)};
        float* hp = a.h + (size_t)m * D + col;
        reinterpret_cast<float4*>(hp)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(hp)[1] = make_float4(v[4], v[5], v[6], v[7]);
        uint4 o;
        o.x = pack_bf16x2(v[0] * w[0], v[1] * w[1]);
        o.y = pack_bf16x2(v[2] * w[2], v[3] * w[3]);
        o.z = pack_bf16x2(v[4] * w[4], v[5] * w[5]);
        o.w = pack_bf16x2(v[6] * w[6], v[7] * w[7]);
        *reinterpret_cast<uint4*>(a.hw + (size_t)m * D + col) = o;
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) ss += v[j] * v[j];
        ss = warp_sum(ss);
        if (lane == 0) a.ss[(size_t)c * a.ss_ld + m] = ss;
    }
}

// 9 warps per CTA put 3 warps on one of the SM's four register partitions
// (16K registers each), so a thread gets at most 168 registers.
template <int NB, int RMAX>
__global__ void __launch_bounds__(DS_THREADS, 1) decode_step_kernel(const DecodeStepArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xs_raw = smem + (size_t)a.n_stages * GV_UNIT_BYTES;  // token rows, or attention scratch
    uint64_t* full = reinterpret_cast<uint64_t*>(xs_raw + a.xs_bytes);
    __shared__ float rinv_s[16];
    __shared__ float rred_s[8][16];
    __shared__ int last_s;
    GvRing ring{smem, full, full + a.n_stages, a.n_stages, 0, 0u};
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int B = a.B, D = a.D, Hd = a.H * a.d, Hkd = a.Hk * a.d, F = a.F;
    const int nku_D = cdiv(D, GV_BK), nku_Hd = cdiv(Hd, GV_BK), nku_F = cdiv(F, GV_BK);
    const int nt_qkv = cdiv(Hd + 2 * Hkd, GV_ROWS), nt_D = cdiv(D, GV_ROWS), nt_F = cdiv(F, GV_ROWS / 2);
    const int nt_V = cdiv(a.vocab, GV_ROWS);

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.n_stages; ++i) {
            mbar_init(&ring.full[i], 1);
            mbar_init(&ring.empty[i], DS_NW);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == DS_NW) {
        // ---------------- producer: every phase's weight units, back to back ----------------
        if (lane == 0) {
            bool ok = true;
            long long issued = 0;
            for (int l = 0; l < a.n_layers && ok; ++l) {
                const CUtensorMap* t = a.tmaps + (size_t)l * TM_PER_LAYER;
                GvWork w = gv_work(nt_qkv, nku_D);
                ok = ok && gv_produce(ring, w, false, t + TM_WQ, t + TM_WK, t + TM_WV, Hd, Hkd, a.err, DERR_MK_PRODUCER_WAIT);
                issued += w.u1 - w.u0;
                w = gv_work(nt_D, nku_Hd);
                ok = ok && gv_produce(ring, w, false, t + TM_WO, t + TM_WO, t + TM_WO, 0, 0, a.err, DERR_MK_PRODUCER_WAIT);
                issued += w.u1 - w.u0;
                w = gv_work(nt_F, nku_D);
                ok = ok && gv_produce(ring, w, true, t + TM_W1G, t + TM_W3G, t + TM_W3G, 0, 0, a.err, DERR_MK_PRODUCER_WAIT);
                issued += w.u1 - w.u0;
                w = gv_work(nt_D, nku_F);
                ok = ok && gv_produce(ring, w, false, t + TM_W2, t + TM_W2, t + TM_W2, 0, 0, a.err, DERR_MK_PRODUCER_WAIT);
                issued += w.u1 - w.u0;
            }
            if (ok && a.has_head) {
                const CUtensorMap* th = a.tmaps + (size_t)a.n_layers * TM_PER_LAYER;
                const GvWork w = gv_work(nt_V, nku_D);
                ok = gv_produce(ring, w, false, th, th, th, 0, 0, a.err, DERR_MK_PRODUCER_WAIT);
                issued += w.u1 - w.u0;
            }
            // After a failed wait the ring was full: at least n copies were issued.
            gv_drain(ring, ok ? issued : (long long)ring.n, a.err, DERR_MK_PRODUCER_WAIT);
        }
        return;
    }

    // ---------------- consumers ----------------
    unsigned nbar = 0;
    auto barrier = [&]() -> bool {
        return grid_barrier(a.bar, nbar++, GV_CONSUMERS, a.err, DERR_GRID_BARRIER_WAIT);
    };
    auto token_rows = [&](const __nv_bfloat16* x, int K) -> GvX {
        GvX X;
        X.x = x;
        X.ldx = K;
        X.M = B;
        X.K = K;
        X.Kp = cdiv(K, GV_BK) * GV_BK;
        X.xs = (long long)B * X.Kp * 2 <= a.xs_bytes ? reinterpret_cast<const __nv_bfloat16*>(xs_raw) : nullptr;
        if (X.xs) gv_stage_x(reinterpret_cast<__nv_bfloat16*>(xs_raw), x, K, B, K, X.Kp);
        return X;
    };
    Epi base;
    base.M = B;
    base.T = 1;
    base.err = a.err;

    ds_embed(a);
    if (!barrier()) return;
    int nparts = D / 256;  // partial sums of h^2 written by the embedding
    const int resid_parts = nt_D * 8;  // ... and by every residual projection (one per 16 rows)

    for (int l = 0; l < a.n_layers; ++l) {
        __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(a.kc) + (size_t)l * a.layer_elems;
        __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(a.vc) + (size_t)l * a.layer_elems;
        // QKV + RoPE + cache append
        {
            Epi e = base;
            e.kind = EPI_QKV_ROPE;
            e.pos0 = a.seq_len;
            e.rope_cos = a.rope_cos;
            e.rope_sin = a.rope_sin;
            e.H = a.H;
            e.Hk = a.Hk;
            e.d = a.d;
            e.S_max = a.S_max;
            e.q_out = a.q;
            e.k_cache = kc;
            e.v_cache = vc;
            const GvX X = token_rows(a.hw, D);
            gv_rinv(ds_norm(a, nparts), B, 0, rinv_s, rred_s);
            gv_consume<NB, EPI_QKV_ROPE>(ring, gv_work(nt_qkv, nku_D), X, Hd + 2 * Hkd, 0, rinv_s, e, a.ws,
                                         a.max_pieces[0], &last_s, a.err, DERR_MK_CONSUMER_WAIT);
            if (!barrier()) return;
        }
        // attention over the cache (the new token's K and V included)
        {
            AttnDecodeArgs aa;
            aa.q = a.q;
            aa.kc = kc;
            aa.vc = vc;
            aa.out = a.o;
            aa.pos0 = a.seq_len;
            aa.B = B;
            aa.T = 1;
            aa.H = a.H;
            aa.Hk = a.Hk;
            aa.d = a.d;
            aa.S_max = a.S_max;
            aa.n_splits = a.n_splits;
            aa.tq = 1;
            aa.n_qchunks = 1;
            aa.ws_part = a.attn_part;
            aa.ws_count = a.attn_cnt;
            aa.scale_log2 = a.scale_log2;
            aa.err = a.err;
            const int items = B * a.Hk * a.n_splits;
            for (int it = blockIdx.x; it < items; it += gridDim.x) {
                const int grp = it / a.n_splits, split = it - grp * a.n_splits;
                attn_split_item<__nv_bfloat16, RMAX, DS_NW, 16, 8>(aa, split, grp / a.Hk, grp % a.Hk, 0,
                                                               reinterpret_cast<float*>(xs_raw), &last_s);
                named_bar_sync(1, GV_CONSUMERS);  // the scratch is reused by the next item
            }
            if (!barrier()) return;
        }
        // wo + residual; writes the ffn_norm input
        {
            Epi e = base;
            e.kind = EPI_RESID;
            e.h = a.h;
            e.D = D;
            e.hw_out = a.hw;
            e.wnext = a.norms[2 * l + 1];
            e.ss_out = a.ss;
            e.ss_out_ld = a.ss_ld;
            const GvX X = token_rows(a.o, Hd);
            gv_rinv(NormIn(), B, 0, rinv_s, rred_s);
            gv_consume<NB, EPI_RESID>(ring, gv_work(nt_D, nku_Hd), X, D, 0, rinv_s, e, a.ws, a.max_pieces[1],
                                      &last_s, a.err, DERR_MK_CONSUMER_WAIT);
            nparts = resid_parts;
            if (!barrier()) return;
        }
        // w1, w3 + SwiGLU
        {
            Epi e = base;
            e.kind = EPI_SWIGLU;
            e.g_out = a.g;
            e.F = F;
            const GvX X = token_rows(a.hw, D);
            gv_rinv(ds_norm(a, nparts), B, 0, rinv_s, rred_s);
            gv_consume<NB, EPI_SWIGLU>(ring, gv_work(nt_F, nku_D), X, F, 0, rinv_s, e, a.ws, a.max_pieces[2],
                                       &last_s, a.err, DERR_MK_CONSUMER_WAIT);
            if (!barrier()) return;
        }
        // w2 + residual; writes the next norm's input
        {
            Epi e = base;
            e.kind = EPI_RESID;
            e.h = a.h;
            e.D = D;
            e.hw_out = a.hw;
            e.wnext = l + 1 < a.n_layers ? a.norms[2 * (l + 1)] : a.norms[2 * a.n_layers];
            e.ss_out = a.ss;
            e.ss_out_ld = a.ss_ld;
            const GvX X = token_rows(a.g, F);
            gv_rinv(NormIn(), B, 0, rinv_s, rred_s);
            gv_consume<NB, EPI_RESID>(ring, gv_work(nt_D, nku_F), X, D, 0, rinv_s, e, a.ws, a.max_pieces[3],
                                      &last_s, a.err, DERR_MK_CONSUMER_WAIT);
            if (!barrier()) return;
        }
    }

    if (a.has_head) {
        // final RMSNorm + lm_head + greedy argmax; the last warp epilogue writes the
        // next tokens and advances the cache lengths
        Epi e = base;
        e.kind = EPI_LOGITS;
        e.logits = a.logits;
        e.ld_logits = a.vocab;
        e.next_tok = a.next;
        e.seq_len = a.seq_len;
        e.advance = 1;
        const GvX X = token_rows(a.hw, D);
        gv_rinv(ds_norm(a, nparts), B, 0, rinv_s, rred_s);
        gv_consume<NB, EPI_LOGITS>(ring, gv_work(nt_V, nku_D), X, a.vocab, 0, rinv_s, e, a.ws, a.max_pieces[4],
                                   &last_s, a.err, DERR_MK_CONSUMER_WAIT);
    } else {
        // layer stack only: hand out the hidden states and advance the cache lengths
        const long long n4 = (long long)B * D / 4;
        for (long long i = (long long)blockIdx.x * GV_CONSUMERS + threadIdx.x; i < n4; i += (long long)gridDim.x * GV_CONSUMERS)
            reinterpret_cast<float4*>(a.h_out)[i] = __ldcg(reinterpret_cast<const float4*>(a.h) + i);
        if (blockIdx.x == 0 && threadIdx.x < B) a.seq_len[threadIdx.x] += 1;
    }
}

// ---------------------------------------------------------------- host side
static long long host_cta_of_unit(long long u, long long G, long long TU) { return ((u + 1) * G - 1) / TU; }

// Most CTAs that share one row tile when ntiles x nku units are split over
// min(G, units) CTAs (as the kernel's gv_work does).
static int pieces_for(int ntiles, int nku, int grid) {
    const long long TU = (long long)ntiles * nku;
    const long long G = grid < TU ? grid : TU;
    long long mp = 1;
    for (long long t = 0; t < ntiles; ++t) {
        const long long cf = host_cta_of_unit(t * nku, G, TU), cl = host_cta_of_unit((t + 1) * nku - 1, G, TU);
        if (cl - cf + 1 > mp) mp = cl - cf + 1;
    }
    return (int)mp;
}

static int hcdiv(int a, int b) { return (a + b - 1) / b; }
static int rmax_of(int G) { return G <= 4 ? 4 : (G <= 8 ? 8 : 16); }

DecodeStepPlan decode_step_plan(int B, int D, int H, int Hk, int d, int F, int vocab, int has_head, int max_keys,
                                int num_sms, int smem_optin) {
    DecodeStepPlan p = {};
    p.grid = num_sms;
    const int Hd = H * d, Hkd = Hk * d;
    const int G = H / Hk;
    p.supported = B >= 1 && B <= 16 && D % 256 == 0 && Hd % GV_ROWS == 0 && Hkd % GV_ROWS == 0 && F % 8 == 0 &&
                  d % 8 == 0 && d <= AD_DMAX && H % Hk == 0 && G <= 16;
    if (!p.supported) return p;
    p.rmax = rmax_of(G);
    // attention splits: minimise rounds x (per-round overhead + keys per split)
    {
        const int groups = B * Hk;
        long long best = -1;
        int best_ns = 1;
        const int cap = hcdiv(max_keys, AD_GK) < AD_MAX_SPLITS ? hcdiv(max_keys, AD_GK) : AD_MAX_SPLITS;
        for (int ns = 1; ns <= (cap > 1 ? cap : 1); ++ns) {
            const long long rounds = ((long long)groups * ns + num_sms - 1) / num_sms;
            const long long cost = rounds * (64 + hcdiv(max_keys, ns));
            if (best < 0 || cost < best) {
                best = cost;
                best_ns = ns;
            }
        }
        p.n_splits = best_ns;
        p.attn_part_floats = (size_t)groups * G * best_ns * (d + 4);
        p.attn_counters = (size_t)groups;
    }
    // shared memory: token-row copies that fit next to at least DS_MIN_STAGES ring
    // stages, the attention scratch, and as many more stages as fit
    const int avail = smem_optin - DS_SMEM_SLACK - 1024;  // 1 KB for the static shared variables
    const int attn_bytes = attn_scratch_floats(p.rmax, DS_NW) * 4;
    int xs = attn_bytes;
    const int ks[3] = {D, Hd, F};
    for (int K : ks) {
        const int need = B * hcdiv(K, GV_BK) * GV_BK * 2;
        if (need <= avail - DS_MIN_STAGES * GV_UNIT_BYTES && need > xs) xs = need;
    }
    xs = (xs + 1023) & ~1023;
    int st = (avail - xs) / GV_UNIT_BYTES;
    if (st > DS_MAX_STAGES) st = DS_MAX_STAGES;
    if (st < 2) {
        p.supported = false;
        return p;
    }
    p.n_stages = st;
    p.xs_bytes = xs;
    p.smem = DS_SMEM_SLACK + st * GV_UNIT_BYTES + xs;
    // split-tile partial slots per phase (QKV, wo, w1/w3, w2, lm_head)
    p.max_pieces[0] = pieces_for(hcdiv(Hd + 2 * Hkd, GV_ROWS), hcdiv(D, GV_BK), num_sms);
    p.max_pieces[1] = pieces_for(hcdiv(D, GV_ROWS), hcdiv(Hd, GV_BK), num_sms);
    p.max_pieces[2] = pieces_for(hcdiv(F, GV_ROWS / 2), hcdiv(D, GV_BK), num_sms);
    p.max_pieces[3] = pieces_for(hcdiv(D, GV_ROWS), hcdiv(F, GV_BK), num_sms);
    p.max_pieces[4] = has_head ? pieces_for(hcdiv(vocab, GV_ROWS), hcdiv(D, GV_BK), num_sms) : 1;
    const int nts[5] = {hcdiv(Hd + 2 * Hkd, GV_ROWS), hcdiv(D, GV_ROWS), hcdiv(F, GV_ROWS / 2), hcdiv(D, GV_ROWS),
                        has_head ? hcdiv(vocab, GV_ROWS) : 1};
    p.part_floats = 0;
    p.tiles = 0;
    for (int i = 0; i < 5; ++i) {
        const size_t f = (size_t)nts[i] * p.max_pieces[i] * GV_PIECE_FLOATS;
        p.part_floats = f > p.part_floats ? f : p.part_floats;
        p.tiles = nts[i] > p.tiles ? nts[i] : p.tiles;
    }
    return p;
}

template <int NB, int RMAX>
static cudaError_t launch_ds(const DecodeStepArgs& a, int smem, int grid, cudaStream_t s) {
    static int attr_smem = 0;
    if (attr_smem < smem) {
        const cudaError_t e =
            cudaFuncSetAttribute(decode_step_kernel<NB, RMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_smem = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DS_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    // Cooperative: the launch fails rather than run if the CTAs cannot all be
    // resident at once, which the grid barriers need.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_step_kernel<NB, RMAX>, a);
}

cudaError_t launch_decode_step(const DecodeStepArgs& a, const DecodeStepPlan& p, cudaStream_t s) {
    if (!p.supported || a.B < 1 || a.B > 16) return cudaErrorInvalidValue;
    if (a.B <= 8) {
        if (p.rmax == 4) return launch_ds<8, 4>(a, p.smem, p.grid, s);
        if (p.rmax == 8) return launch_ds<8, 8>(a, p.smem, p.grid, s);
        return launch_ds<8, 16>(a, p.smem, p.grid, s);
    }
    if (p.rmax == 4) return launch_ds<16, 4>(a, p.smem, p.grid, s);
    if (p.rmax == 8) return launch_ds<16, 8>(a, p.smem, p.grid, s);
    return launch_ds<16, 16>(a, p.smem, p.grid, s);
}

}  // namespace lfw
