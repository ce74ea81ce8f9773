// Decode attention streamed in 32-key units through the fused decode step's
// shared-memory ring (decode_step.cu).
//
// A unit is the K and V tiles of 32 consecutive keys of one (sequence, KV head)
// group: two 64-dim halves of 32 rows x 128 bytes each for K and for V, loaded by
// TMA with the 128-byte swizzle into one 16 KB ring stage. A group's keys are
// 0 .. len (the new token sits at position len), so it has ceil((len + 1) / 32)
// units, and the units of all groups, in group order, are split evenly over the
// CTAs. The step computes S = Q K^T and P V with mma.sync m16n8k16 from the
// swizzled tiles (the group's query heads padded to 16 rows) and an online
// softmax in the log2 domain ("Implementación de la atención"; "GQA" and
// "Scaled Dot-Product Attention" on the llama3.np page).
#pragma once
#include "common.cuh"
#include "kernels.cuh"

namespace lfw {

constexpr int AK = 32;  // keys per attention unit (K and V tiles of 32 x 128 bf16 = 16 KB)

// Swizzled address of 16-byte chunk `chunk` (0..15) of key row `key` in a K or V
// tile of an attention unit: two 64-dim halves of 32 rows x 128 B, 4 KB apart.
DEVI uint32_t kv32_addr(uint32_t base, int key, int chunk) {
    return base + (chunk >> 3) * (AK * 128) + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
}
// Attention units of a group: keys 0 .. len (the new token at position len).
DEVI int group_units(const int* s_len, int grp, int Hk) { return (s_len[grp / Hk] + AK) / AK; }

// This CTA's share of the attention units (the same for every layer).
struct AttnSplit {
    long long U, G, u0, u1;  // all units, CTAs taking part, this CTA's range
    int g0, j0;              // group and tile of unit u0
    long long cum0;          // first unit of group g0
};
DEVI AttnSplit attn_split(const int* s_len, int B, int Hk) {
    AttnSplit sp;
    long long U = 0;
    for (int gr = 0; gr < B * Hk; ++gr) U += group_units(s_len, gr, Hk);
    sp.U = U;
    sp.G = (long long)gridDim.x < U ? (long long)gridDim.x : U;
    if (blockIdx.x < sp.G) {
        sp.u0 = blockIdx.x * U / sp.G;
        sp.u1 = (blockIdx.x + 1) * U / sp.G;
    } else {
        sp.u0 = sp.u1 = U;
    }
    long long c = 0;
    int gr = 0;
    while (gr < B * Hk) {
        const int n = group_units(s_len, gr, Hk);
        if (c + n > sp.u0) break;
        c += n;
        ++gr;
    }
    sp.g0 = gr;
    sp.j0 = (int)(sp.u0 - c);
    sp.cum0 = c;
    return sp;
}

}  // namespace lfw
