// Decode attention with one thread-block cluster per (sequence, KV head) group.
//
// Causal grouped-query attention of the newest token of each sequence against
// its KV cache ("Implementación de la atención"; "GQA", "Scaled Dot-Product
// Attention" and "KV cache" on the llama3.np page): query head h attends to
// keys 0 .. p (p the new token's position) of KV head h / G, scores q.k /
// sqrt(d), softmax, weighted sum of values.
//
// A group is a sequence's KV head with up to 8 of its query heads (a KV head
// with more, as in multi-query attention, makes several groups, each reading
// the head's keys and values). Its keys are cut into 32-key units (the K and V
// tiles of 32 positions, 16 KB) and split evenly over the cs CTAs of its cluster. In each CTA a producer
// warp streams the CTA's units by TMA into a ring of shared-memory stages (one
// copy of each tile, shared by all the group's query heads), and the eight
// consumer warps take the units in turn, computing S = Q K^T, an online softmax
// and O^T += V^T P^T on the tensor cores (attn_ring.cuh). The warps' states are
// merged in shared memory, then the CTAs' partial results are merged by the
// cluster's first CTA, which reads them from its peers' shared memory
// (distributed shared memory, after a cluster barrier) in rank order and writes
// the group's output. No global scratch and no atomics: the split merge costs
// two cluster barriers instead of global round trips.
#include "attn_ring.cuh"

namespace lfw {

constexpr int AC_UNIT = 4 * AK * 128;             // one unit: K and V tiles of 32 keys (16 KB)
constexpr int AC_CONSUMERS = 320;                 // 10 warps: a round of 10 units per CTA
constexpr int AC_THREADS = AC_CONSUMERS + 32;     // + the producer warp
constexpr int AC_STAGES = 10;
constexpr int AC_RMAX = 8;                        // query rows of a group
constexpr int AC_PIECE_BYTES = AC_RMAX * AW_REC * 4;
constexpr int AC_SCRATCH = 4096 + (AC_CONSUMERS / 32) * AC_RMAX * AW_REC * 4;  // query tile, warps' records
constexpr int AC_SMEM = 1024 + AC_STAGES * AC_UNIT + AC_SCRATCH + AC_PIECE_BYTES +
                        2 * AC_STAGES * 8 + 64;

DEVI void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
DEVI uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
DEVI uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
DEVI float ld_dsmem_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
DEVI float4 ld_dsmem_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Four output dims at element offset off: O / L in bf16, and the bf16 remainder
// (split activations for the next projection) when asked.
DEVI void attn_out4(const AttnClusterArgs& a, int off, const float (&O)[4], float L) {
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const float v[4] = {O[0] * inv, O[1] * inv, O[2] * inv, O[3] * inv};
    uint2 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    *reinterpret_cast<uint2*>(a.out + off) = u;
    if (a.out_lo) {
        uint2 r;
        r.x = pack_bf16x2(v[0] - bf16lo(u.x), v[1] - bf16hi(u.x));
        r.y = pack_bf16x2(v[2] - bf16lo(u.y), v[3] - bf16hi(u.y));
        *reinterpret_cast<uint2*>(a.out_lo + off) = r;
    }
}

__global__ void __launch_bounds__(AC_THREADS, 1)
    attn_cluster_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const AttnClusterArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* scratch = stages + AC_STAGES * AC_UNIT;        // query tile, then the warps' records
    float* piece = reinterpret_cast<float*>(scratch + AC_SCRATCH);  // [R][AW_REC]
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(piece) + AC_PIECE_BYTES);
    uint64_t* empty = full + AC_STAGES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = a.cs > 1 ? cluster_ctarank() : 0u;
    // group: (sequence, KV head, chunk of at most 8 of its query heads)
    const int G = a.H / a.Hk, chunks = (G + AC_RMAX - 1) / AC_RMAX;
    const int gr = blockIdx.y / chunks, chunk = blockIdx.y % chunks;
    const int b = gr / a.Hk, kvh = gr % a.Hk;
    const int R = G - chunk * AC_RMAX < AC_RMAX ? G - chunk * AC_RMAX : AC_RMAX;
    const int head0 = kvh * G + chunk * AC_RMAX;  // first query head of the group
    int p0 = a.pos0[b];
    if (threadIdx.x == 0) LFW_CHECK(p0 >= 0 && p0 < a.S_max, a.err, BC_ATTN_POS);
    p0 = p0 < 0 ? 0 : (p0 >= a.S_max ? a.S_max - 1 : p0);
    const int U = (p0 + AK) / AK;  // units covering keys 0 .. p0
    const int u0 = (int)((long long)rank * U / a.cs), u1 = (int)((long long)(rank + 1) * U / a.cs);
    const int n = u1 - u0;
    const long long row0 = a.row_base + (long long)b * a.rows_per_seq + (long long)kvh * a.S_max;

    if (threadIdx.x == 0) {
        for (int i = 0; i < AC_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    __syncthreads();

    if (warp == AC_CONSUMERS / 32) {
        // producer: this CTA's units, K and V tiles of 32 keys as four 64-dim boxes
        if (lane == 0) {
            bool ok = true;
            for (int i = 0; i < n && ok; ++i) {
                const int st = i % AC_STAGES;
                if (i >= AC_STAGES) ok = mbar_wait(&empty[st], ((i / AC_STAGES) - 1) & 1, a.err, DERR_ATTN_TMA_WAIT);
                if (!ok) break;
                uint8_t* dst = stages + st * AC_UNIT;
                const int row = (int)(row0 + (long long)(u0 + i) * AK);
                mbar_arrive_expect_tx(&full[st], AC_UNIT);
                tma_load_2d(dst, &tmK, &full[st], 0, row);
                tma_load_2d(dst + AK * 128, &tmK, &full[st], 64, row);
                tma_load_2d(dst + 2 * AK * 128, &tmV, &full[st], 0, row);
                tma_load_2d(dst + 3 * AK * 128, &tmV, &full[st], 64, row);
            }
            // no copy may still be writing shared memory when the CTA retires
            for (int i = n - AC_STAGES > 0 ? n - AC_STAGES : 0; i < n; ++i)
                mbar_wait(&full[i % AC_STAGES], (i / AC_STAGES) & 1, a.err, DERR_ATTN_TMA_WAIT);
        }
        __syncwarp();
    } else {
        // consumers: the group's query rows, then units i = warp, warp + 8, ...
        attn_q_tile(scratch, a.q + (size_t)b * a.H * 128 + (size_t)head0 * 128, 128, R, threadIdx.x);
        named_bar_sync(1, AC_CONSUMERS);
        float* wst = reinterpret_cast<float*>(scratch + 4096);
        AttnAcc acc;
        attn_acc_init(acc);
        for (int i = warp; i < n; i += AC_CONSUMERS / 32) {
            const int st = i % AC_STAGES;
            mbar_wait(&full[st], (i / AC_STAGES) & 1, a.err, DERR_ATTN_TMA_WAIT);
            attn_unit(acc, smem_u32(stages + st * AC_UNIT), smem_u32(scratch), (u0 + i) * AK, p0, a.scale_log2);
            fence_proxy_async();  // the stage's reads before the TMA writes that refill it
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        attn_acc_store(acc, wst, warp, R);
        named_bar_sync(1, AC_CONSUMERS);
        if ((int)threadIdx.x < R * 32) {
            const int r = threadIdx.x >> 5, d4 = (threadIdx.x & 31) * 4;
            float M, L, O[4];
            attn_merge_warps<AC_CONSUMERS / 32>(wst, R, r, d4, M, L, O);
            if (a.cs == 1) {
                attn_out4(a, b * a.H * 128 + (head0 + r) * 128 + d4, O, L);
            } else {
                float* pr = piece + r * AW_REC;
                *reinterpret_cast<float4*>(pr + 4 + d4) = make_float4(O[0], O[1], O[2], O[3]);
                if (d4 == 0) {
                    pr[0] = M;
                    pr[1] = L;
                }
            }
        }
    }
    if (a.cs == 1) return;
    // the cluster's first CTA merges the pieces of every rank, in rank order
    cluster_sync_all();
    if (rank == 0 && (int)threadIdx.x < R * 32) {
        const int r = threadIdx.x >> 5, d4 = (threadIdx.x & 31) * 4;
        const uint32_t base = smem_u32(piece + r * AW_REC);
        // every rank's record is read before any is used (cs <= 8)
        float mp[8], lp[8];
        float4 op[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (q >= a.cs) break;
            const uint32_t pa = map_rank(base, (uint32_t)q);
            mp[q] = ld_dsmem_f32(pa);
            lp[q] = ld_dsmem_f32(pa + 4);
            op[q] = ld_dsmem_f32x4(pa + 16 + 4 * d4);
        }
        float M = -INFINITY, L = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (q >= a.cs) break;
            lse_merge(M, L, O, mp[q], lp[q], op[q]);
        }
        attn_out4(a, b * a.H * 128 + (head0 + r) * 128 + d4, O, L);
    }
    cluster_sync_all();  // every piece stays in place until the first CTA has read it
}

int attn_cluster_groups(int B, int H, int Hk) { return B * Hk * ((H / Hk + AC_RMAX - 1) / AC_RMAX); }

int attn_cluster_size(int B, int H, int Hk, int d, int num_sms) {
    if (d != 128 || Hk < 1 || H % Hk != 0 || B < 1) return 0;
    const int groups = attn_cluster_groups(B, H, Hk);
    int cs = 1;
    while (cs < 8 && groups * cs < num_sms) cs *= 2;
    return cs;
}

cudaError_t launch_attn_cluster(const AttnClusterArgs& a, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                cudaStream_t s) {
    if (a.cs < 1 || a.cs > 8 || a.Hk < 1 || a.H % a.Hk != 0 || !tmK || !tmV) return cudaErrorInvalidValue;
    static bool attr = false;
    if (!attr) {
        const cudaError_t e = cudaFuncSetAttribute(attn_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   AC_SMEM);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.cs, attn_cluster_groups(a.B, a.H, a.Hk));
    cfg.blockDim = dim3(AC_THREADS);
    cfg.dynamicSmemBytes = AC_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = a.cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_cluster_kernel, *tmK, *tmV, a);
}

}  // namespace lfw
