// Unnormalised Walsh-Hadamard butterflies over one 1024-block held by a warp.
// The transform is a product of one butterfly per index bit, so any
// assignment of the 10 element-index bits to (5 lane bits, 5 register bits)
// works: stages over lane bits pair lanes, stages over register bits pair
// registers.  Callers choose the element of (lane, register) they load and
// read back the same element.  Natural (Sylvester) order.
#pragma once

namespace gale {

// Unnormalised butterflies over the register index of v (5 index bits).
__device__ __forceinline__ void fwht32_regs(float (&v)[32]) {
#pragma unroll
    for (int s = 0; s < 5; ++s) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & (1 << s)) continue;
            const float a = v[i], b = v[i | (1 << s)];
            v[i] = a + b;
            v[i | (1 << s)] = a - b;
        }
    }
}

// The same 32-point transform in constant geometry: every stage adds and
// subtracts adjacent registers and writes the sums to the lower and the
// differences to the upper half, so the stage loop needs no unrolling (small
// code for paths that run once per launch).  Five stages give the natural
// (Sylvester) order.
__device__ __forceinline__ void fwht32_cg(float (&v)[32]) {
#pragma unroll 1
    for (int s = 0; s < 5; ++s) {
        float w[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            w[i] = v[2 * i] + v[2 * i + 1];
            w[i + 16] = v[2 * i] - v[2 * i + 1];
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = w[i];
    }
}

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
    fwht32_regs(v);
}

}  // namespace gale
