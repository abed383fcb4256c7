// dropout.cuh -- the LoRA-dropout mask of the adapter's input ("QLoRA & PEFT family" 3.4,
// dropout 0.05 - 0.1; the lora_dropout setting of the configuration in "How does QLoRA work for
// training?"). Inverted dropout: element e of the activation (e = offset + m k_in + k) survives
// when the 32-bit draw of a counter-based generator is >= thr = floor(p 2^32); survivors are
// scaled by 1 / (1 - p), which the kernels fold into the adapter scale s.
//
// The generator is Philox4x32 with 10 rounds (Salmon, Moraes, Dror and Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011): element e takes word e mod 4 of the block drawn at
// counter (e / 4 low word, e / 4 high word, 0, 0) with key (seed low word, seed high word).
#pragma once

#include <stdint.h>

#include "kernels.h"

namespace qn {

// Four 32-bit words for counter block `blk` under `seed`.
__device__ __forceinline__ uint4 philox_block(uint64_t seed, uint64_t blk) {
    uint32_t x0 = static_cast<uint32_t>(blk), x1 = static_cast<uint32_t>(blk >> 32), x2 = 0u, x3 = 0u;
    uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t lo0 = 0xD2511F53u * x0, hi0 = __umulhi(0xD2511F53u, x0);
        const uint32_t lo1 = 0xCD9E8D57u * x2, hi1 = __umulhi(0xCD9E8D57u, x2);
        const uint32_t y0 = hi1 ^ x1 ^ k0, y2 = hi0 ^ x3 ^ k1;
        x0 = y0;
        x1 = lo1;
        x2 = y2;
        x3 = lo0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return make_uint4(x0, x1, x2, x3);
}

__device__ __forceinline__ uint32_t philox_word(const uint4 &v, uint32_t i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Keep bits of the n (<= 32) consecutive elements e0 .. e0 + n - 1 (bit i for element e0 + i).
__device__ __forceinline__ uint32_t dropout_keep_bits(const DropoutArgs &d, uint64_t e0, int n) {
    uint32_t bits = 0u;
    uint64_t blk = ~uint64_t(0);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    for (int i = 0; i < n; ++i) {
        const uint64_t e = e0 + static_cast<uint64_t>(i);
        if ((e >> 2) != blk) {
            blk = e >> 2;
            v = philox_block(d.seed, blk);
        }
        if (philox_word(v, static_cast<uint32_t>(e & 3)) >= d.thr) bits |= 1u << i;
    }
    return bits;
}

// bf16 pair (lo, hi halves) with the halves whose keep bit is clear set to +0.
__device__ __forceinline__ uint32_t mask_pair(uint32_t v, uint32_t keep2) {
    return (v & ((keep2 & 1u) ? 0x0000ffffu : 0u)) | (v & ((keep2 & 2u) ? 0xffff0000u : 0u));
}

}  // namespace qn
