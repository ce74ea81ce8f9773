// Codes of the device error word that kernels set (first one wins) and the
// host reads back: bounded waits that ran out, and the failed index checks of
// the bounds-checking build. Shared by device code and the host library.
#pragma once

#include <stdint.h>

namespace lfw {

// Device error word codes (first one wins).
enum : uint32_t {
    DERR_NONE = 0,
    DERR_GEMM_PRODUCER_WAIT = 0x101,
    DERR_GEMM_MMA_WAIT = 0x102,
    DERR_GEMM_EPI_WAIT = 0x103,
    DERR_ATTN_TMA_WAIT = 0x201,
    DERR_ATTN_MMA_WAIT = 0x202,
    DERR_ATTN_SOFTMAX_WAIT = 0x203,
    DERR_GEMV_PRODUCER_WAIT = 0x301,
    DERR_GEMV_CONSUMER_WAIT = 0x302,
    DERR_GRID_BARRIER_WAIT = 0x401,
    DERR_MK_PRODUCER_WAIT = 0x402,
    DERR_MK_CONSUMER_WAIT = 0x403,
    DERR_PROBE_WAIT = 0x501,  // the wait probe (a wait that cannot complete)
    DERR_BOUNDS = 0x06000000,  // | the check site (bounds-checking build)
};

// Check sites of the bounds-checking build (the low bits of DERR_BOUNDS codes).
enum : uint32_t {
    BC_TOKEN = 1,        // a token id outside [0, vocab)
    BC_CACHE_POS = 2,    // a KV-cache append position outside [0, S_max)
    BC_ROPE_POS = 3,     // a RoPE table row outside [0, S_max)
    BC_ATTN_POS = 4,     // attention over positions beyond the cache
    BC_SEQ_ADVANCE = 5,  // a cache length advanced past S_max
    BC_DECODE_POS = 6,   // a decode position outside [0, S_max)
};

}  // namespace lfw
