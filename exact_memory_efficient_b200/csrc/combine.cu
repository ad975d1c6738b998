// combine.cu -- merge attention results computed over disjoint key ranges.
//
// Method: the chunk-summary merge of "Self-attention Does Not Need O(n^2)
// Memory" (English summary, the bullet on summarising the results of key/value
// chunks) with the two-block formulas of "当注意力成为瓶颈" (section IO感知),
// written for normalised parts: part r holds O_r and lse_r over its own keys,
// and the result over all of them is
//     lse = ln sum_r e^{lse_r},     O = sum_r e^{lse_r - lse} O_r.
// This is the merge step of a key (sequence) split: each part can come from a
// different GPU.  The parts are given as an array of R device pointers (local
// buffers, slices of a gathered buffer, or another GPU's memory), so the same
// kernel serves a merge after a collective gather and a merge that reads the
// peers' parts directly.
//
// Memory-bound: one thread per (row, 8 head dims) reads the R lse values of its
// row and R 16-byte (bf16) or 32-byte (fp32) pieces of the O rows.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mea {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void load8(const uint16_t* p, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void store8(uint16_t* p, const float (&x)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                              pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}
__device__ __forceinline__ void store8(float* p, const float (&x)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

// MAXR: the parts this instantiation handles (4, 8 or 16), so that the per-part
// registers of a small merge stay few and many threads stay resident.
template <typename T, int MAXR>
__global__ void __launch_bounds__(256) combine_kernel(const CombineArgs a) {
    const int groups = a.D / 8;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= a.rows * groups) return;
    const long long row = idx / groups;
    const int g = (int)(idx - row * groups);

    float lv[MAXR];
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
        lv[r] = (r < a.R) ? a.lse_parts[r][row] : -INFINITY;
        M = fmaxf(M, lv[r]);
    }
    // every part's piece is loaded before any weight is known (one round trip
    // to memory); a part without keys (lse = -inf, weight 0) is then dropped by
    // a select, so whatever its o holds (even NaN) never reaches the result
    float x[MAXR][8];
#pragma unroll
    for (int r = 0; r < MAXR; ++r)
        if (r < a.R) load8(static_cast<const T*>(a.o_parts[r]) + row * a.D + 8 * g, x[r]);
    // a row whose parts are all empty has no keys at all: its sum of exponentials
    // is 0, so lse = ln 0 = -inf, and its o is written as 0 (every weight is 0)
    const bool no_keys = (M == -INFINITY);
    const float Mref = no_keys ? 0.f : M;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    float L = 0.f;
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
        if (r < a.R) {
            const float w = ex2_approx((lv[r] - Mref) * kLog2e);
            const bool use = w != 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = use ? fmaf(w, x[r][i], acc[i]) : acc[i];
            L += w;
        }
    }
    const float inv = no_keys ? 0.f : 1.f / L;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= inv;
    store8(static_cast<T*>(a.o) + row * a.D + 8 * g, acc);
    if (g == 0) a.lse[row] = no_keys ? -INFINITY : M + __log2f(L) * kLn2;
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t stream) {
    const long long threads = a.rows * (a.D / 8);
    if (threads == 0) return cudaSuccess;
    const long long blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    auto run = [&](auto kern) { kern<<<(unsigned)blocks, 256, 0, stream>>>(a); };
    if (bf16) {
        if (a.R <= 4) run(combine_kernel<uint16_t, 4>);
        else if (a.R <= 8) run(combine_kernel<uint16_t, 8>);
        else run(combine_kernel<uint16_t, kCombineMaxParts>);
    } else {
        if (a.R <= 4) run(combine_kernel<float, 4>);
        else if (a.R <= 8) run(combine_kernel<float, 8>);
        else run(combine_kernel<float, kCombineMaxParts>);
    }
    return cudaGetLastError();
}

}  // namespace mea
