// Device helpers shared by the libspecverify kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define SV_DEV __device__ __forceinline__

namespace sv {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC'11). Ten rounds of the 4x32 S-box: two 32x32->64 products
// whose halves are xored into the other words, with the key advanced by the
// two Weyl constants between rounds.
// ---------------------------------------------------------------------------
struct PhiloxKey { uint32_t k0, k1; };

SV_DEV uint4 philox4x32_10(uint4 x, PhiloxKey key) {
    uint32_t k0 = key.k0, k1 = key.k1;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t a = 0xD2511F53u * x.x;              // low half of M0*x0
        const uint32_t ah = __umulhi(0xD2511F53u, x.x);    // high half
        const uint32_t c = 0xCD9E8D57u * x.z;
        const uint32_t ch = __umulhi(0xCD9E8D57u, x.z);
        uint4 y;
        y.x = ch ^ x.y ^ k0;
        y.y = c;
        y.z = ah ^ x.w ^ k1;
        y.w = a;
        x = y;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return x;
}

// Uniform in [0,1) with 24 random bits, exact in fp32: counter {c0, c1, tag, 0}.
SV_DEV float philox_uniform(PhiloxKey key, uint32_t c0, uint32_t c1, uint32_t tag) {
    const uint4 w = philox4x32_10(make_uint4(c0, c1, tag, 0u), key);
    return (float)(w.x >> 8) * (1.0f / 16777216.0f);
}

// ---------------------------------------------------------------------------
// Small reductions.
// ---------------------------------------------------------------------------
SV_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

SV_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

SV_DEV int warp_or(int v) {
    return __reduce_or_sync(0xffffffffu, (unsigned)v);
}

// bf16 bits -> float (exact).
SV_DEV float bf16_bits_to_float(uint16_t h) {
    return __uint_as_float(((uint32_t)h) << 16);
}

}  // namespace sv
