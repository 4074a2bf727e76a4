// Bit operations on 64-bit holder masks in shared memory (one bit per rank),
// used by the split's and the assign's per-expert tables.
#pragma once
#include <cstdint>

namespace lb {

// Bit b (0..63) of a 64-bit mask in shared memory, set or cleared with a
// 32-bit atomic on the word that holds it.  A hot expert's tens of holders
// hit one mask at once; with 64-bit atomics that step of the assign's prep
// took about 3.7 us for 63 holders, with these about 0.9 us.
__device__ __forceinline__ void or_bit64(uint64_t *m, int b) {
    atomicOr(reinterpret_cast<unsigned *>(m) + (b >> 5), 1u << (b & 31));
}
// true if this call cleared the bit (it was set before)
__device__ __forceinline__ bool clear_bit64(uint64_t *m, int b) {
    const unsigned bit = 1u << (b & 31);
    return (atomicAnd(reinterpret_cast<unsigned *>(m) + (b >> 5), ~bit) & bit) != 0u;
}

}  // namespace lb
