// bwd_f32.cu -- fp32 SIMT backward of exact attention.
//
// Method: "Self-attention Does Not Need O(n^2) Memory" (English summary, the
// bullet on differentiation): nothing of the forward is stored but o and lse;
// the probabilities are recomputed, P_ij = exp(scale q_i.k_j - lse_i).  With
// lse known every P_ij is final, so sums over keys or over queries split into
// independent parts that simply add: no running maximum and no rescaling is
// needed here.  The gradient formulas are ordinary softmax calculus:
//   D_i = sum_d dO_id O_id,   dP_ij = dO_i.v_j,   dS_ij = P_ij (dP_ij - D_i),
//   dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i,   dV_j = sum_i P_ij dO_i.
//
// Three launches, no atomics, deterministic:
//   bwd_f32_pre_kernel    warp per query row: D_i.
//   bwd_f32_dq_kernel     warp per (query row, key slice): dQ_i.
//   bwd_f32_dkdv_kernel   warp per (key row, query slice): dK_j, dV_j.
// Inside a CTA the slices of one row are summed through shared memory in a
// fixed order.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"
#include "simt_f32.cuh"

namespace mea {
namespace {

using simt::kLog2e;
using simt::load_dims;
using simt::reduce_scatter32;
using simt::store_dims;
using simt::warp_sum;

// P = exp(scale * s - lse): the difference is formed by one fused multiply-add
// (one rounding), then exponentiated in base 2.
__device__ __forceinline__ float prob(float s, float scale, float lse) {
    return ex2_approx(fmaf(s, scale, -lse) * kLog2e);
}

template <int DPL>
__global__ void __launch_bounds__(256)
bwd_f32_pre_kernel(const float* __restrict__ o, const float* __restrict__ dO, float* __restrict__ delta,
                   long long rows) {
    constexpr int D = 32 * DPL;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const unsigned lane = lane_id();
    float a[DPL], b[DPL];
    load_dims<DPL>(o + row * D + DPL * lane, a);
    load_dims<DPL>(dO + row * D + DPL * lane, b);
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) t = fmaf(a[i], b[i], t);
    t = warp_sum(t);
    if (lane == 0) delta[row] = t;
}

// Sum the per-warp partial rows of one output row (warps r*wpr .. r*wpr+wpr-1
// of the CTA) in warp order; returns the total in the first warp of the group.
template <int DPL>
__device__ __forceinline__ void sum_slices(float (&part)[8][32 * DPL], float (&acc)[DPL], int warp, int wpr,
                                           int slice, unsigned lane) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) part[warp][DPL * lane + i] = acc[i];
    __syncthreads();
    if (slice == 0) {
        for (int w = 1; w < wpr; ++w)
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[i] += part[warp + w][DPL * lane + i];
    }
}

template <int DPL>
__global__ void __launch_bounds__(256)
bwd_f32_dq_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                  const float* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ delta,
                  float* __restrict__ dq, int Nq, int Nk, float scale, int rows_per_cta, int warps_per_row,
                  bool accumulate) {
    constexpr int D = 32 * DPL;
    __shared__ float part[8][32 * DPL];
    const unsigned lane = lane_id();
    const int warp = (int)warp_id();
    const int r_local = warp / warps_per_row;
    const int slice = warp % warps_per_row;
    const int bh = blockIdx.y;
    const int row = blockIdx.x * rows_per_cta + r_local;
    const bool row_ok = (r_local < rows_per_cta) && (row < Nq);
    const float* kh = k + (size_t)bh * Nk * D;
    const float* vh = v + (size_t)bh * Nk * D;

    float acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
    if (row_ok) {
        const size_t ri = (size_t)bh * Nq + row;
        float qv[DPL], dov[DPL];
        load_dims<DPL>(q + ri * D + DPL * lane, qv);
        load_dims<DPL>(dO + ri * D + DPL * lane, dov);
        const float lse_i = lse[ri];
        const float d_i = delta[ri];
        for (int j0 = 32 * slice; j0 < Nk; j0 += 32 * warps_per_row) {
            const int nvalid = min(32, Nk - j0);
            float ps[32], pd[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float kv[DPL], vv[DPL];
                if (j < nvalid) {
                    load_dims<DPL>(kh + (size_t)(j0 + j) * D + DPL * lane, kv);
                    load_dims<DPL>(vh + (size_t)(j0 + j) * D + DPL * lane, vv);
                } else {
#pragma unroll
                    for (int i = 0; i < DPL; ++i) kv[i] = vv[i] = 0.f;
                }
                float ts = 0.f, td = 0.f;
#pragma unroll
                for (int i = 0; i < DPL; ++i) {
                    ts = fmaf(qv[i], kv[i], ts);
                    td = fmaf(dov[i], vv[i], td);
                }
                ps[j] = ts;
                pd[j] = td;
            }
            const float s = reduce_scatter32(ps, lane);    // q_i . k_{j0+lane}
            const float dp = reduce_scatter32(pd, lane);   // dO_i . v_{j0+lane}
            const float p = ((int)lane < nvalid) ? prob(s, scale, lse_i) : 0.f;
            const float ds = p * (dp - d_i);
#pragma unroll 8
            for (int j = 0; j < 32; ++j) {
                const float dsj = __shfl_sync(0xffffffffu, ds, j);
                if (j < nvalid) {
                    float kv[DPL];
                    load_dims<DPL>(kh + (size_t)(j0 + j) * D + DPL * lane, kv);
#pragma unroll
                    for (int i = 0; i < DPL; ++i) acc[i] = fmaf(dsj, kv[i], acc[i]);
                }
            }
        }
    }
    sum_slices<DPL>(part, acc, warp, warps_per_row, slice, lane);
    if (row_ok && slice == 0) {
        float* dst = dq + ((size_t)bh * Nq + row) * D + DPL * lane;
        float out[DPL];
        if (accumulate) {   // fp32 sum of an accumulating caller: add the unscaled dS K
            load_dims<DPL>(dst, out);
#pragma unroll
            for (int i = 0; i < DPL; ++i) out[i] += acc[i];
        } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) out[i] = scale * acc[i];
        }
        store_dims<DPL>(dst, out);
    }
}

template <int DPL>
__global__ void __launch_bounds__(256)
bwd_f32_dkdv_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                    const float* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ delta,
                    float* __restrict__ dk, float* __restrict__ dv, int Nq, int Nk, float scale, int rows_per_cta,
                    int warps_per_row, bool accumulate) {
    constexpr int D = 32 * DPL;
    __shared__ float part[8][32 * DPL];
    const unsigned lane = lane_id();
    const int warp = (int)warp_id();
    const int r_local = warp / warps_per_row;
    const int slice = warp % warps_per_row;
    const int bh = blockIdx.y;
    const int key = blockIdx.x * rows_per_cta + r_local;
    const bool key_ok = (r_local < rows_per_cta) && (key < Nk);
    const float* qh = q + (size_t)bh * Nq * D;
    const float* doh = dO + (size_t)bh * Nq * D;
    const float* lseh = lse + (size_t)bh * Nq;
    const float* dh = delta + (size_t)bh * Nq;

    float acc_k[DPL], acc_v[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc_k[i] = acc_v[i] = 0.f;
    if (key_ok) {
        const size_t kj = (size_t)bh * Nk + key;
        float kv[DPL], vv[DPL];
        load_dims<DPL>(k + kj * D + DPL * lane, kv);
        load_dims<DPL>(v + kj * D + DPL * lane, vv);
        for (int i0 = 32 * slice; i0 < Nq; i0 += 32 * warps_per_row) {
            const int nvalid = min(32, Nq - i0);
            float ps[32], pd[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float qv[DPL], dov[DPL];
                if (i < nvalid) {
                    load_dims<DPL>(qh + (size_t)(i0 + i) * D + DPL * lane, qv);
                    load_dims<DPL>(doh + (size_t)(i0 + i) * D + DPL * lane, dov);
                } else {
#pragma unroll
                    for (int t = 0; t < DPL; ++t) qv[t] = dov[t] = 0.f;
                }
                float ts = 0.f, td = 0.f;
#pragma unroll
                for (int t = 0; t < DPL; ++t) {
                    ts = fmaf(qv[t], kv[t], ts);
                    td = fmaf(dov[t], vv[t], td);
                }
                ps[i] = ts;
                pd[i] = td;
            }
            const float s = reduce_scatter32(ps, lane);    // q_{i0+lane} . k_j
            const float dp = reduce_scatter32(pd, lane);   // dO_{i0+lane} . v_j
            float p = 0.f, ds = 0.f;
            if ((int)lane < nvalid) {
                p = prob(s, scale, lseh[i0 + lane]);
                ds = p * (dp - dh[i0 + lane]);
            }
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                const float pi = __shfl_sync(0xffffffffu, p, i);
                const float dsi = __shfl_sync(0xffffffffu, ds, i);
                if (i < nvalid) {
                    float qv[DPL], dov[DPL];
                    load_dims<DPL>(qh + (size_t)(i0 + i) * D + DPL * lane, qv);
                    load_dims<DPL>(doh + (size_t)(i0 + i) * D + DPL * lane, dov);
#pragma unroll
                    for (int t = 0; t < DPL; ++t) {
                        acc_v[t] = fmaf(pi, dov[t], acc_v[t]);
                        acc_k[t] = fmaf(dsi, qv[t], acc_k[t]);
                    }
                }
            }
        }
    }
    sum_slices<DPL>(part, acc_k, warp, warps_per_row, slice, lane);
    __syncthreads();  // part[] is reused for dV
    sum_slices<DPL>(part, acc_v, warp, warps_per_row, slice, lane);
    if (key_ok && slice == 0) {
        const size_t kj = ((size_t)bh * Nk + key) * D + DPL * lane;
        float out[DPL];
        if (accumulate) {   // fp32 sums of an accumulating caller: add the unscaled dS^T Q and P^T dO
            float prev[DPL];
            load_dims<DPL>(dk + kj, out);
            load_dims<DPL>(dv + kj, prev);
#pragma unroll
            for (int i = 0; i < DPL; ++i) {
                out[i] += acc_k[i];
                prev[i] += acc_v[i];
            }
            store_dims<DPL>(dk + kj, out);
            store_dims<DPL>(dv + kj, prev);
        } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) out[i] = scale * acc_k[i];
            store_dims<DPL>(dk + kj, out);
            store_dims<DPL>(dv + kj, acc_v);
        }
    }
}

template <int DPL>
cudaError_t launch_dpl(const F32BwdArgs& a, cudaStream_t stream, unsigned phases) {
    if (phases & kBwdPhasePre) {
        const long long rows = (long long)a.BH * a.Nq;
        if (rows > 0) {
            bwd_f32_pre_kernel<DPL><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(a.o, a.dO, a.delta, rows);
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    if (phases & kBwdPhaseMain) {
        {
            dim3 grid((a.Nq + a.q_rows_per_cta - 1) / a.q_rows_per_cta, a.BH);
            bwd_f32_dq_kernel<DPL><<<grid, 256, 0, stream>>>(a.q, a.k, a.v, a.dO, a.lse, a.delta, a.dq, a.Nq, a.Nk,
                                                             a.scale, a.q_rows_per_cta, 8 / a.q_rows_per_cta,
                                                             a.accumulate);
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        dim3 grid((a.Nk + a.k_rows_per_cta - 1) / a.k_rows_per_cta, a.BH);
        bwd_f32_dkdv_kernel<DPL><<<grid, 256, 0, stream>>>(a.q, a.k, a.v, a.dO, a.lse, a.delta, a.dk, a.dv, a.Nq,
                                                           a.Nk, a.scale, a.k_rows_per_cta, 8 / a.k_rows_per_cta,
                                                           a.accumulate);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_bwd_f32(const F32BwdArgs& a, cudaStream_t stream, unsigned phases) {
    switch (a.D) {
        case 32: return launch_dpl<1>(a, stream, phases);
        case 64: return launch_dpl<2>(a, stream, phases);
        case 96: return launch_dpl<3>(a, stream, phases);
        case 128: return launch_dpl<4>(a, stream, phases);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace mea
