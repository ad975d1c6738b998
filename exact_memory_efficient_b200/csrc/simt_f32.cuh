// simt_f32.cuh -- warp-level helpers shared by the fp32 SIMT kernels.
//
// A warp owns one row of D = 32 * DPL floats: lane l holds the DPL consecutive
// dims [DPL*l, DPL*l + DPL).  Dot products of that row with 32 other rows are
// formed as per-lane partial sums and finished by a butterfly reduce-scatter
// that leaves the total for row j in lane j.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mea {
namespace simt {

constexpr float kLog2e = 1.4426950408889634f;

template <int DPL>
__device__ __forceinline__ void load_dims(const float* __restrict__ p, float (&x)[DPL]) {
    if constexpr (DPL == 4) {
        float4 t = __ldg(reinterpret_cast<const float4*>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else if constexpr (DPL == 2) {
        float2 t = __ldg(reinterpret_cast<const float2*>(p));
        x[0] = t.x; x[1] = t.y;
    } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) x[i] = __ldg(p + i);
    }
}

template <int DPL>
__device__ __forceinline__ void store_dims(float* p, const float (&x)[DPL]) {
    if constexpr (DPL == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    } else if constexpr (DPL == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) p[i] = x[i];
    }
}

// Butterfly reduce-scatter: on entry every lane holds 32 partial sums v[0..31]
// (one per key of the group); on exit lane l returns the warp-wide total of
// entry l.  31 shuffles for 32 keys.
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], unsigned lane) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const bool hi = lane & 16u;
        float send = hi ? v[k] : v[k + 16];
        float keep = hi ? v[k + 16] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const bool hi = lane & 8u;
        float send = hi ? v[k] : v[k + 8];
        float keep = hi ? v[k + 8] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const bool hi = lane & 4u;
        float send = hi ? v[k] : v[k + 4];
        float keep = hi ? v[k + 4] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const bool hi = lane & 2u;
        float send = hi ? v[k] : v[k + 2];
        float keep = hi ? v[k + 2] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    {
        const bool hi = lane & 1u;
        float send = hi ? v[0] : v[1];
        float keep = hi ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
    return v[0];
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace simt
}  // namespace mea
