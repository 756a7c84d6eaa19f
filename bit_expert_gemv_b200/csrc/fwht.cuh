// Unnormalised Walsh-Hadamard butterflies over one 1024-block held by a warp.
// The transform is a product of one butterfly per index bit, so any
// assignment of the 10 element-index bits to (5 lane bits, 5 register bits)
// works: stages over lane bits pair lanes, stages over register bits pair
// registers.  Callers choose the element of (lane, register) they load and
// read back the same element.  Natural (Sylvester) order.
#pragma once

namespace gale {

__device__ __forceinline__ void fwht1024_warp(float (&v)[32], int lane) {
    // partner lane differs in bit s
#pragma unroll 1
    for (int s = 0; s < 5; ++s) {
        const bool upper = (lane >> s) & 1;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            float o = __shfl_xor_sync(0xffffffffu, v[i], 1 << s);
            v[i] = upper ? (o - v[i]) : (v[i] + o);
        }
    }
    // partner register differs in bit s
#pragma unroll
    for (int s = 0; s < 5; ++s) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & (1 << s)) continue;
            float a = v[i], b = v[i | (1 << s)];
            v[i] = a + b;
            v[i | (1 << s)] = a - b;
        }
    }
}

}  // namespace gale
