// fwd_f32.cu -- fp32 SIMT forward: exact attention with O(1) state per row.
//
// Method: "Self-attention Does Not Need O(n^2) Memory" (English summary,
// method bullets 1-4).  Each query row is owned by a warp that walks its keys
// 32 at a time keeping the running maximum m, the running exp-sum l and the
// rescaled weighted-value accumulator acc; normalisation happens once at the
// end.  Long key ranges are split into chunks processed by the CTAs of one
// thread-block cluster (and, inside a CTA, by several warps); every chunk
// leaves a summary (m, l, acc) and the summaries are merged with the two-block
// formulas of "当注意力成为瓶颈" (section IO感知), through distributed
// shared memory, so no global scratch memory is used.
//
// Layout: lane l of a warp owns the DPL consecutive head dims [DPL*l, DPL*l+DPL)
// of q, acc and of every key/value row it reads (D = 32 * DPL).
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"
#include "simt_f32.cuh"

namespace cg = cooperative_groups;

namespace mea {
namespace {

using simt::kLog2e;
using simt::load_dims;
using simt::reduce_scatter32;
using simt::store_dims;
using simt::warp_max;
using simt::warp_sum;

// exp(x) for x <= 0 via the hardware base-2 exponential.
__device__ __forceinline__ float exp_nonpos(float x) { return ex2_approx(x * kLog2e); }

// One chunk summary: running max, exp-sum and accumulator of one row.
template <int DPL>
struct RowState {
    float m;
    float l;  // warp-uniform after finalisation
    float acc[DPL];
};

// Merge (m2, l2, acc2) into (m, l, acc): both rescaled to the larger maximum.
template <int DPL>
__device__ __forceinline__ void merge_into(RowState<DPL>& a, float m2, float l2, const float (&acc2)[DPL]) {
    const float m = fmaxf(a.m, m2);
    if (m == -INFINITY) return;  // both empty
    const float wa = exp_nonpos(a.m - m);
    const float wb = exp_nonpos(m2 - m);
    a.l = a.l * wa + l2 * wb;
#pragma unroll
    for (int i = 0; i < DPL; ++i) a.acc[i] = a.acc[i] * wa + acc2[i] * wb;
    a.m = m;
}

// Shared-memory record of one warp's (or one CTA's) summary for one row.
template <int DPL>
struct alignas(16) Summary {
    float acc[32 * DPL];
    float m;
    float l;
    float pad[2];
};

// Up to 16 warps per CTA for D <= 64 (a single query row then gets 16 warps of
// key slices, for more loads in flight), 8 otherwise (register budget).
template <int DPL>
constexpr int kMaxWarps = (DPL <= 2) ? 16 : 8;

template <int DPL>
__global__ void __launch_bounds__(32 * kMaxWarps<DPL>)
fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
               float* __restrict__ o, float* __restrict__ lse,
               int Nq, int Nk, float scale, int rows_per_cta, int warps_per_row, int chunk_len) {
    constexpr int D = 32 * DPL;
    __shared__ Summary<DPL> warp_sum_s[kMaxWarps<DPL>];   // one per warp
    __shared__ Summary<DPL> cta_sum_s[8];                 // one per row of this CTA (read by cluster rank 0)

    cg::cluster_group cluster = cg::this_cluster();
    const unsigned nranks = cluster.num_blocks();
    const unsigned rank = cluster.block_rank();

    const unsigned lane = lane_id();
    const unsigned warp = warp_id();
    const int r_local = warp / warps_per_row;       // row within CTA
    const int kg = warp % warps_per_row;            // key sub-group of this warp
    const int bh = blockIdx.z;
    const int row = blockIdx.y * rows_per_cta + r_local;
    const bool row_ok = (r_local < rows_per_cta) && (row < Nq);

    const int c_begin = rank * chunk_len;
    const int c_end = min(Nk, c_begin + chunk_len);

    const float* kh = k + (size_t)bh * Nk * D;
    const float* vh = v + (size_t)bh * Nk * D;

    RowState<DPL> st;
    st.m = -INFINITY;
    st.l = 0.f;  // per-lane partial until the end of the loop
#pragma unroll
    for (int i = 0; i < DPL; ++i) st.acc[i] = 0.f;

    if (row_ok) {
        float qv[DPL];
        load_dims<DPL>(q + ((size_t)bh * Nq + row) * D + DPL * lane, qv);

        for (int j0 = c_begin + 32 * kg; j0 < c_end; j0 += 32 * warps_per_row) {
            const int nvalid = min(32, c_end - j0);
            // Value rows do not depend on the scores: for D <= 64 (DPL <= 2) they
            // are loaded together with the key rows, so both streams are in flight
            // at once (this loop is bound by memory latency, not arithmetic).
            constexpr bool kVEarly = DPL <= 2;
            float vbuf[kVEarly ? 32 : 1][DPL];
            // scores of the 32 keys of this group, reduce-scattered to lane j
            float pd[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float kv[DPL];
                if (j < nvalid) {
                    load_dims<DPL>(kh + (size_t)(j0 + j) * D + DPL * lane, kv);
                    if constexpr (kVEarly) load_dims<DPL>(vh + (size_t)(j0 + j) * D + DPL * lane, vbuf[j]);
                } else {
#pragma unroll
                    for (int i = 0; i < DPL; ++i) kv[i] = 0.f;
                    if constexpr (kVEarly) {
#pragma unroll
                        for (int i = 0; i < DPL; ++i) vbuf[j][i] = 0.f;
                    }
                }
                float t = 0.f;
#pragma unroll
                for (int i = 0; i < DPL; ++i) t = fmaf(qv[i], kv[i], t);
                pd[j] = t;
            }
            // scale multiplies the fp32-accumulated dot product
            float s = scale * reduce_scatter32(pd, lane);
            if ((int)lane >= nvalid) s = -INFINITY;
            const float m_new = fmaxf(st.m, warp_max(s));
            const float alpha = exp_nonpos(st.m - m_new);
            const float p = exp_nonpos(s - m_new);
            st.l = st.l * alpha + p;
#pragma unroll
            for (int i = 0; i < DPL; ++i) st.acc[i] *= alpha;
            st.m = m_new;
            if constexpr (kVEarly) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, p, j);   // 0 past nvalid
#pragma unroll
                    for (int i = 0; i < DPL; ++i) st.acc[i] = fmaf(pj, vbuf[j][i], st.acc[i]);
                }
            } else {
#pragma unroll 8
                for (int j = 0; j < 32; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, p, j);
                    if (j < nvalid) {
                        float vv[DPL];
                        load_dims<DPL>(vh + (size_t)(j0 + j) * D + DPL * lane, vv);
#pragma unroll
                        for (int i = 0; i < DPL; ++i) st.acc[i] = fmaf(pj, vv[i], st.acc[i]);
                    }
                }
            }
        }
    }
    st.l = warp_sum(st.l);

    // ---- merge the warps_per_row warps of each row inside the CTA
    Summary<DPL>& ws = warp_sum_s[warp];
#pragma unroll
    for (int i = 0; i < DPL; ++i) ws.acc[DPL * lane + i] = st.acc[i];
    if (lane == 0) { ws.m = st.m; ws.l = st.l; }
    __syncthreads();
    if (kg == 0 && r_local < rows_per_cta) {
        for (int w = 1; w < warps_per_row; ++w) {
            const Summary<DPL>& o2 = warp_sum_s[warp + w];
            float a2[DPL];
#pragma unroll
            for (int i = 0; i < DPL; ++i) a2[i] = o2.acc[DPL * lane + i];
            merge_into<DPL>(st, o2.m, o2.l, a2);
        }
        Summary<DPL>& cs = cta_sum_s[r_local];
#pragma unroll
        for (int i = 0; i < DPL; ++i) cs.acc[DPL * lane + i] = st.acc[i];
        if (lane == 0) { cs.m = st.m; cs.l = st.l; }
    }

    // ---- merge the chunks held by the CTAs of the cluster (distributed smem)
    if (nranks > 1) cluster.sync(); else __syncthreads();
    if (rank == 0 && kg == 0 && row_ok) {
        for (unsigned c = 1; c < nranks; ++c) {
            const Summary<DPL>* rs = cluster.map_shared_rank(&cta_sum_s[r_local], c);
            float a2[DPL];
#pragma unroll
            for (int i = 0; i < DPL; ++i) a2[i] = rs->acc[DPL * lane + i];
            merge_into<DPL>(st, rs->m, rs->l, a2);
        }
        const float inv_l = 1.f / st.l;
        float out[DPL];
#pragma unroll
        for (int i = 0; i < DPL; ++i) out[i] = st.acc[i] * inv_l;
        store_dims<DPL>(o + ((size_t)bh * Nq + row) * D + DPL * lane, out);
        if (lane == 0) lse[(size_t)bh * Nq + row] = st.m + logf(st.l);
    }
    // keep every CTA's shared memory alive until rank 0 has read it
    if (nranks > 1) cluster.sync();
}

template <int DPL>
cudaError_t launch_dpl(const F32FwdArgs& a, cudaStream_t stream) {
    auto kern = fwd_f32_kernel<DPL>;
    cudaError_t e = cudaSuccess;
    if (a.chunks > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.chunks, (a.Nq + a.rows_per_cta - 1) / a.rows_per_cta, a.BH);
    cfg.blockDim = dim3(32 * a.rows_per_cta * a.warps_per_row, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.chunks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a.q, a.k, a.v, a.o, a.lse, a.Nq, a.Nk, a.scale,
                              a.rows_per_cta, a.warps_per_row, a.chunk_len);
}

}  // namespace

cudaError_t launch_fwd_f32(const F32FwdArgs& a, cudaStream_t stream) {
    switch (a.D) {
        case 32: return launch_dpl<1>(a, stream);
        case 64: return launch_dpl<2>(a, stream);
        case 96: return launch_dpl<3>(a, stream);
        case 128: return launch_dpl<4>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace mea
