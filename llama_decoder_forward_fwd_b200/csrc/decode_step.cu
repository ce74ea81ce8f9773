// Fused decode step: one whole decode step of a bf16 model (embedding, every
// layer's QKV projection with RoPE and KV-cache append, attention, wo projection
// with residual, w1/w3 projection with SwiGLU, w2 projection with residual, and
// the lm_head with greedy argmax) in a single persistent launch with one CTA per
// SM ("Resumen de una implementación desde cero del modelo LLaMA-3": attention
// and feed-forward repeated over every layer, then "Predicción de tokens";
// "手撕Llama3第1层", section 6: the stacked transformer blocks).
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
// the whole input vector). The projections are the code of the per-projection
// kernel (gemv_core.cuh), except that a split row tile is finished by its first
// CTA. The attention phase streams the KV cache through the same ring: a unit
// is the K and V tiles of 32 keys of one (sequence, KV head) group, and the
// units of all groups are split evenly over the CTAs. Each consumer warp owns
// 16 of the 128 output dims: it computes S = Q K^T for the group's query heads
// (padded to 16 rows) with mma.sync from the swizzled tiles, keeps the online
// softmax (running max and sum, log2 domain) and accumulates P V for its dims.
// A group split over several CTAs is merged by its first CTA (log-sum-exp
// rule, pieces in CTA order). The ring may have fetched the tile that holds the
// new token before this step's QKV phase wrote its key and value, so the CTA
// that owns that tile patches the row from the cache before using it.
// Reductions are split by a function of the grid size and the cache lengths
// only, so a given GPU gives bit-identical steps.
//
// Barrier waits, ring waits and the final drain are all bounded; a timeout
// records an error code and every CTA leaves at its next barrier.
#include "attn_ring.cuh"
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
// Producer: the TMA copies of this CTA's attention units of layer l (K and V
// tiles of 32 keys, each as two 64-dim boxes).
DEVI bool attn_produce(GvRing& r, const DecodeStepArgs& a, int l, const AttnSplit& sp, const int* s_len) {
    const CUtensorMap* tk = a.tmaps + (size_t)a.n_layers * TM_PER_LAYER + 1;
    const CUtensorMap* tv = tk + 1;
    int gr = sp.g0, j = sp.j0;
    int n = sp.u0 < sp.u1 ? group_units(s_len, gr, a.Hk) : 0;
    for (long long u = sp.u0; u < sp.u1; ++u) {
        if (!mbar_wait(&r.empty[r.st], r.ph ^ 1u, a.err, DERR_MK_PRODUCER_WAIT)) return false;
        uint8_t* dst = r.stages + r.st * GV_UNIT_BYTES;
        const int row = (int)((long long)l * a.kv_rows_per_layer + (long long)gr * a.S_max + j * AK);
        mbar_arrive_expect_tx(&r.full[r.st], GV_UNIT_BYTES);
        tma_load_2d(dst, tk, &r.full[r.st], 0, row);
        tma_load_2d(dst + AK * 128, tk, &r.full[r.st], 64, row);
        tma_load_2d(dst + 2 * AK * 128, tv, &r.full[r.st], 0, row);
        tma_load_2d(dst + 3 * AK * 128, tv, &r.full[r.st], 64, row);
        if (++j == n) {
            j = 0;
            ++gr;
            if (u + 1 < sp.u1) n = group_units(s_len, gr, a.Hk);
        }
        ++r.issued;
        ring_next(r);
    }
    return true;
}

// Consumers: this CTA's attention units of layer l (see the file comment).
// qsm: 4 KB of 1024-aligned shared memory for the group's query rows.
DEVI void attn_consume(GvRing& ring, const DecodeStepArgs& a, int l, const AttnSplit& sp, const int* s_len,
                       uint8_t* qsm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3, j8 = lane >> 3, i8 = lane & 7;
    const int Hk = a.Hk, R = a.H / a.Hk, HD = a.H * 128;
    const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(a.kc) + (size_t)l * a.layer_elems;
    const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(a.vc) + (size_t)l * a.layer_elems;
    const uint32_t qbase = smem_u32(qsm);
    const long long G = sp.G;
    bool ok = true;
    int gr = sp.g0, jt = sp.j0, n_g = 0, p0 = 0;
    long long cum = sp.cum0;
    bool fresh = true;
    uint32_t qf[8][4];
    float o[2][4], mrow[2], lrow[2];
    uint4 patch = make_uint4(0, 0, 0, 0);

    // Publishes this CTA's piece of group gr, or (first CTA of the group) merges
    // all pieces, and writes the group's attention output rows.
    auto finish_group = [&]() {
        const int b = gr / Hk, kvh = gr % Hk;
        const long long cf = cta_of_unit(cum, G, sp.U), cl = cta_of_unit(cum + n_g - 1, G, sp.U);
        const long long pc = blockIdx.x - cf;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            lrow[hh] += __shfl_xor_sync(0xffffffffu, lrow[hh], 1);
            lrow[hh] += __shfl_xor_sync(0xffffffffu, lrow[hh], 2);
        }
        const size_t rec_floats = 18 * (size_t)R;  // per warp: O[R][16], m[R], l[R]
        float* recs = a.attn_part + (size_t)gr * gridDim.x * 8 * rec_floats;
        unsigned* cnt = a.attn_cnt + gr * 8 + warp;
        if (cf != cl && pc != 0) {
            float* rec = recs + ((size_t)pc * 8 + warp) * rec_floats;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = g8 + 8 * hh;
                if (row >= R) continue;
#pragma unroll
                for (int n = 0; n < 2; ++n)
                    *reinterpret_cast<float2*>(rec + row * 16 + n * 8 + 2 * t4) = make_float2(o[n][2 * hh], o[n][2 * hh + 1]);
                if (t4 == 0) {
                    rec[16 * R + row] = mrow[hh];
                    rec[17 * R + row] = lrow[hh];
                }
            }
            __syncwarp();
            if (lane == 0) red_release_add(cnt, 1u);
            __syncwarp();
            return;
        }
        if (cf != cl) {
            if (lane == 0) {
                const unsigned want = (unsigned)(cl - cf);
                if (ld_acquire_gpu(cnt) < want) {
                    const uint64_t t0 = globaltimer();
                    while (ld_acquire_gpu(cnt) < want) {
                        if (globaltimer() - t0 > kWaitLimitNs) {
                            atomicCAS(a.err, 0u, DERR_MK_CONSUMER_WAIT);
                            break;
                        }
                    }
                }
                *cnt = 0u;
            }
            __syncwarp();
            // log-sum-exp merge of the pieces, in CTA order; the loads of PB pieces
            // are issued together
            constexpr int PB = 2;
            const int np = (int)(cl - cf);
            for (int p0 = 1; p0 <= np; p0 += PB) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int row = g8 + 8 * hh;
                    if (row >= R) continue;
                    float mp[PB], lp[PB];
                    float2 o0[PB], o1[PB];
#pragma unroll
                    for (int q = 0; q < PB; ++q) {
                        if (p0 + q > np) continue;
                        const float* rec = recs + ((size_t)(p0 + q) * 8 + warp) * rec_floats;
                        mp[q] = __ldcg(rec + 16 * R + row);
                        lp[q] = __ldcg(rec + 17 * R + row);
                        o0[q] = __ldcg(reinterpret_cast<const float2*>(rec + row * 16 + 2 * t4));
                        o1[q] = __ldcg(reinterpret_cast<const float2*>(rec + row * 16 + 8 + 2 * t4));
                    }
#pragma unroll
                    for (int q = 0; q < PB; ++q) {
                        if (p0 + q > np) continue;
                        const float mn = fmaxf(mrow[hh], mp[q]);
                        const float mu = mn == -INFINITY ? 0.f : mn;
                        const float sa = exp2f(mrow[hh] - mu), sb = exp2f(mp[q] - mu);
                        lrow[hh] = lrow[hh] * sa + lp[q] * sb;
                        o[0][2 * hh] = o[0][2 * hh] * sa + o0[q].x * sb;
                        o[0][2 * hh + 1] = o[0][2 * hh + 1] * sa + o0[q].y * sb;
                        o[1][2 * hh] = o[1][2 * hh] * sa + o1[q].x * sb;
                        o[1][2 * hh + 1] = o[1][2 * hh + 1] * sa + o1[q].y * sb;
                        mrow[hh] = mn;
                    }
                }
            }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = g8 + 8 * hh;
            if (row >= R) continue;
            const float inv = lrow[hh] > 0.f ? 1.f / lrow[hh] : 0.f;
            __nv_bfloat16* dst = a.o + (size_t)b * HD + (kvh * R + row) * 128 + 16 * warp + 2 * t4;
#pragma unroll
            for (int n = 0; n < 2; ++n)
                *reinterpret_cast<uint32_t*>(dst + n * 8) = pack_bf16x2(o[n][2 * hh] * inv, o[n][2 * hh + 1] * inv);
        }
    };

    for (long long u = sp.u0; u < sp.u1; ++u) {
        if (fresh) {
            // entering group gr: its query rows (zero past R), and the new token's
            // key and value row if this CTA holds the group's last tile
            const int b = gr / Hk, kvh = gr % Hk;
            n_g = group_units(s_len, gr, Hk);
            p0 = s_len[b];
            named_bar_sync(1, GV_CONSUMERS);  // the previous group's query rows are no longer read
            if (warp == 0 && cum + n_g - 1 < sp.u1) {
                const __nv_bfloat16* src = (lane < 16 ? kc : vc) + ((size_t)gr * a.S_max + p0) * 128 + (lane & 15) * 8;
                patch = __ldcg(reinterpret_cast<const uint4*>(src));
            }
            {
                const int r = threadIdx.x >> 4, c = threadIdx.x & 15;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (r < R) v = __ldcg(reinterpret_cast<const uint4*>(a.q + (size_t)b * HD + (kvh * R + r) * 128 + c * 8));
                *reinterpret_cast<uint4*>(qsm + r * 256 + ((c ^ (r & 7)) << 4)) = v;
            }
            named_bar_sync(1, GV_CONSUMERS);
            {
                const int r = (j8 & 1) * 8 + i8;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int c = 2 * kk + (j8 >> 1);
                    ldsm_x4(qf[kk], qbase + r * 256 + ((c ^ (r & 7)) << 4));
                }
            }
#pragma unroll
            for (int n = 0; n < 2; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            mrow[0] = mrow[1] = -INFINITY;
            lrow[0] = lrow[1] = 0.f;
            fresh = false;
        }
        if (ok && !mbar_wait(&ring.full[ring.st], ring.ph, a.err, DERR_MK_CONSUMER_WAIT)) ok = false;
        const uint32_t kb = smem_u32(ring.stages + ring.st * GV_UNIT_BYTES);
        const uint32_t vb = kb + 2 * AK * 128;
        const int key0 = jt * AK;
        if (key0 <= p0 && p0 < key0 + AK) {
            // the new token's row, written by this step's QKV phase
            if (warp == 0) {
                const uint32_t dst = kv32_addr(lane < 16 ? kb : vb, p0 - key0, lane & 15);
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(patch.x), "r"(patch.y), "r"(patch.z),
                             "r"(patch.w)
                             : "memory");
                fence_proxy_async();  // before the stage is handed back to the TMA writes
            }
            named_bar_sync(1, GV_CONSUMERS);
        }
        // S = Q K^T: 16 (padded) query rows x 32 keys
        float sc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t rr[4];
                ldsm_x4(rr, kv32_addr(kb, (2 * np + (j8 >> 1)) * 8 + i8, 2 * kk + (j8 & 1)));
                mma_bf16_16816(sc[2 * np], qf[kk], rr[0], rr[1]);
                mma_bf16_16816(sc[2 * np + 1], qf[kk], rr[2], rr[3]);
            }
        }
        // online softmax over the unit's keys (keys after the new token masked)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float mx = -INFINITY;
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    float v = sc[n][2 * hh + e2] * a.scale_log2;
                    if (key0 + n * 8 + 2 * t4 + e2 > p0) v = -INFINITY;
                    sc[n][2 * hh + e2] = v;
                    mx = fmaxf(mx, v);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float mnew = fmaxf(mrow[hh], mx);
            const float muse = mnew == -INFINITY ? 0.f : mnew;
            const float alpha = exp2f(mrow[hh] - muse);
            mrow[hh] = mnew;
            float sum = 0.f;
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const float pv = exp2f(sc[n][2 * hh + e2] - muse);
                    sc[n][2 * hh + e2] = pv;
                    sum += pv;
                }
            lrow[hh] = lrow[hh] * alpha + sum;
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                o[n][2 * hh] *= alpha;
                o[n][2 * hh + 1] *= alpha;
            }
        }
        // O += P V for this warp's 16 dims
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t pf[4];
            pf[0] = pack_bf16x2(sc[2 * ks][0], sc[2 * ks][1]);
            pf[1] = pack_bf16x2(sc[2 * ks][2], sc[2 * ks][3]);
            pf[2] = pack_bf16x2(sc[2 * ks + 1][0], sc[2 * ks + 1][1]);
            pf[3] = pack_bf16x2(sc[2 * ks + 1][2], sc[2 * ks + 1][3]);
            uint32_t rr[4];
            ldsm_x4_t(rr, kv32_addr(vb, ks * 16 + (j8 & 1) * 8 + i8, 2 * warp + (j8 >> 1)));
            mma_bf16_16816(o[0], pf, rr[0], rr[1]);
            mma_bf16_16816(o[1], pf, rr[2], rr[3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring.empty[ring.st]);
        ring_next(ring);
        if (++jt == n_g) {
            finish_group();
            cum += n_g;
            ++gr;
            jt = 0;
            fresh = true;
        }
    }
    if (!fresh) finish_group();
}

template <int NB>
__global__ void __launch_bounds__(DS_THREADS, 1) decode_step_kernel(const DecodeStepArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xs_raw = smem + (size_t)a.n_stages * GV_UNIT_BYTES;  // token rows, or attention scratch
    uint64_t* full = reinterpret_cast<uint64_t*>(xs_raw + a.xs_bytes);
    __shared__ float rinv_s[16];
    __shared__ float rred_s[8][16];
    __shared__ int s_len[16];  // cache lengths before this step (the new token's positions)
    GvRing ring{smem, full, full + a.n_stages, a.n_stages, 0, 0u, 0};
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
    if (threadIdx.x < B) {
        s_len[threadIdx.x] = a.seq_len[threadIdx.x];
        LFW_CHECK(s_len[threadIdx.x] >= 0 && s_len[threadIdx.x] < a.S_max, a.err, BC_DECODE_POS);
    }
    __syncthreads();
    const AttnSplit asp = attn_split(s_len, B, a.Hk);

    if (warp == DS_NW) {
        // ---------------- producer: every phase's units, back to back ----------------
        if (lane == 0) {
            bool ok = true;
            long long issued = 0;
            for (int l = 0; l < a.n_layers && ok; ++l) {
                const CUtensorMap* t = a.tmaps + (size_t)l * TM_PER_LAYER;
                GvWork w = gv_work(nt_qkv, nku_D);
                ok = ok && gv_produce(ring, w, false, t + TM_WQ, t + TM_WK, t + TM_WV, Hd, Hkd, a.err, DERR_MK_PRODUCER_WAIT);
                issued += w.u1 - w.u0;
                ok = ok && attn_produce(ring, a, l, asp, s_len);
                issued += asp.u1 - asp.u0;
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
    // Projection prologue: token rows into shared memory when they fit, RMSNorm scales.
    auto token_rows = [&](const __nv_bfloat16* x, int K, const NormIn& nrm) -> GvX {
        GvX X;
        X.x = x;
        X.ldx = K;
        X.M = B;
        X.K = K;
        X.Kp = cdiv(K, GV_BK) * GV_BK;
        X.xs = (long long)B * X.Kp * 2 <= a.xs_bytes ? reinterpret_cast<const __nv_bfloat16*>(xs_raw) : nullptr;
        gv_prologue(const_cast<__nv_bfloat16*>(X.xs), x, K, B, K, X.Kp, nrm, 0, rinv_s, rred_s);
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
            e.pos0 = s_len;  // this step's positions, already in shared memory
            e.rope_cos = a.rope_cos;
            e.rope_sin = a.rope_sin;
            e.H = a.H;
            e.Hk = a.Hk;
            e.d = a.d;
            e.S_max = a.S_max;
            e.q_out = a.q;
            e.k_cache = kc;
            e.v_cache = vc;
            const GvX X = token_rows(a.hw, D, ds_norm(a, nparts));
            gv_consume<NB, EPI_QKV_ROPE>(ring, gv_work(nt_qkv, nku_D), X, Hd + 2 * Hkd, 0, rinv_s, e, a.ws,
                                         a.max_pieces[0], a.err, DERR_MK_CONSUMER_WAIT);
            if (!barrier()) return;
        }
        // attention over the cache (the new token's K and V included)
        attn_consume(ring, a, l, asp, s_len, xs_raw);
        if (!barrier()) return;
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
            const GvX X = token_rows(a.o, Hd, NormIn());
            gv_consume<NB, EPI_RESID>(ring, gv_work(nt_D, nku_Hd), X, D, 0, rinv_s, e, a.ws, a.max_pieces[1],
                                      a.err, DERR_MK_CONSUMER_WAIT);
            nparts = resid_parts;
            if (!barrier()) return;
        }
        // w1, w3 + SwiGLU
        {
            Epi e = base;
            e.kind = EPI_SWIGLU;
            e.g_out = a.g;
            e.F = F;
            const GvX X = token_rows(a.hw, D, ds_norm(a, nparts));
            gv_consume<NB, EPI_SWIGLU>(ring, gv_work(nt_F, nku_D), X, F, 0, rinv_s, e, a.ws, a.max_pieces[2],
                                       a.err, DERR_MK_CONSUMER_WAIT);
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
            const GvX X = token_rows(a.g, F, NormIn());
            gv_consume<NB, EPI_RESID>(ring, gv_work(nt_D, nku_F), X, D, 0, rinv_s, e, a.ws, a.max_pieces[3],
                                      a.err, DERR_MK_CONSUMER_WAIT);
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
        const GvX X = token_rows(a.hw, D, ds_norm(a, nparts));
        gv_consume<NB, EPI_LOGITS>(ring, gv_work(nt_V, nku_D), X, a.vocab, 0, rinv_s, e, a.ws, a.max_pieces[4],
                                   a.err, DERR_MK_CONSUMER_WAIT);
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

DecodeStepPlan decode_step_plan(int B, int D, int H, int Hk, int d, int F, int vocab, int has_head, int max_keys,
                                int num_sms, int smem_optin) {
    (void)max_keys;
    DecodeStepPlan p = {};
    p.grid = num_sms;
    const int Hd = H * d, Hkd = Hk * d;
    p.supported = B >= 1 && B <= 16 && D % 256 == 0 && Hd % GV_ROWS == 0 && Hkd % GV_ROWS == 0 && F % 8 == 0 &&
                  d == 128 && H % Hk == 0 && H / Hk <= 16;
    if (!p.supported) return p;
    const int R = H / Hk;
    // attention: per (group, piece) records of 8 warps x 18 R floats; counters per (group, warp)
    p.attn_part_floats = (size_t)B * Hk * num_sms * 8 * 18 * R;
    p.attn_counters = (size_t)B * Hk * 8;
    // shared memory: the query tile (4 KB), token-row copies that fit next to at
    // least DS_MIN_STAGES ring stages, and as many more stages as fit
    const int avail = smem_optin - DS_SMEM_SLACK - 1024;  // 1 KB for the static shared variables
    int xs = 4096;
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

template <int NB>
static cudaError_t launch_ds(const DecodeStepArgs& a, int smem, int grid, cudaStream_t s) {
    static int attr_smem = 0;
    if (attr_smem < smem) {
        const cudaError_t e =
            cudaFuncSetAttribute(decode_step_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_smem = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DS_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    // Cooperative: the launch fails rather than run if the CTAs cannot all be
    // resident at once, which the grid barriers and the merges need.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_step_kernel<NB>, a);
}

cudaError_t launch_decode_step(const DecodeStepArgs& a, const DecodeStepPlan& p, cudaStream_t s) {
    if (!p.supported || a.B < 1 || a.B > 16) return cudaErrorInvalidValue;
    return a.B <= 8 ? launch_ds<8>(a, p.smem, p.grid, s) : launch_ds<16>(a, p.smem, p.grid, s);
}

}  // namespace lfw
