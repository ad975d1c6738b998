// fwd_bf16.cu -- bf16 forward on the 5th-generation tensor cores (sm_100a).
//
// Method: "Self-attention Does Not Need O(n^2) Memory" (English summary,
// method bullets 1-4): keys/values are consumed block by block; each query row
// keeps a running maximum, a running exp-sum and a rescaled accumulator, and
// is normalised once at the end.  Per key block j the recurrence is the
// incremental form of the two-block formulas of "当注意力成为瓶颈"
// (section IO感知):  m' = max(m, rowmax S_j),  l' = l e^(m-m') + sum e^(S_j-m'),
// O' = O e^(m-m') + e^(S_j-m') V_j.
//
// One CTA owns two 128-row query tiles of one (batch, head) and streams all
// key/value tiles (128 keys each) through a shared-memory ring:
//   warp 0      TMEM allocator, then TMA producer (Q once, then K_0, V_0,
//               K_1, V_1, ... ; no multicast)
//   warp 1      MMA issuer (one thread): S_t = Q_t K_j^T into TMEM, then
//               O_t += P_t V_j with P_t read from TMEM
//   warps 2-5   softmax of query tile 0, warps 6-9 softmax of query tile 1
//               (warp w reaches TMEM lanes 32*(w%4) .. 32*(w%4)+31):
//               one thread per query row (TMEM lane), tcgen05.ld of S,
//               exp2 with scale*log2(e) folded in, P written back to TMEM as
//               bf16 over the S columns, O rescaled in TMEM when the reference
//               maximum moves.
// TMEM (512 columns): S_0 [0,128)  S_1 [128,256)  O_0 [256,256+D)  O_1 [384,384+D).
//
// Reference maximum: a row's exponentials are taken relative to a reference
// value m_ref that is raised to the true running maximum only when the new
// block maximum exceeds it by more than 8 (base-2 units).  Then every
// exponential is <= 2^8, nothing overflows, and because O, l and the final
// lse all use the same m_ref the result is the same exact softmax; it only
// saves O rescales.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mea {
namespace {

constexpr int kTileM = 128;       // query rows per tile
constexpr int kTileN = 128;       // keys per tile
constexpr int kThreads = 320;     // 10 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct FwdCfg {
    static constexpr int kTileBytes = kTileN * D * 2;         // one K or V tile
    static constexpr int kQBytes = kTileM * D * 2;            // one Q tile
    static constexpr int kStages = (D == 128) ? 4 : 6;
    static constexpr int kBoxBytes = 128 * 128;               // one 64-column box of 128 rows
    static constexpr int kSmemData = 2 * kQBytes + kStages * kTileBytes;
    static constexpr int kSmemBytes = kSmemData + 1024 /*barriers*/ + 1024 /*alignment slack*/;
};

struct FwdBarriers {
    uint64_t q_full;
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t s_full[2];
    uint64_t p_ready[2];
    uint64_t o_final;
    uint64_t drain;
    unsigned tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ o,
                float* __restrict__ lse, int Nq, int Nk, float scale) {
    using Cfg = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                               // Q_0 then Q_1
    uint8_t* sRing = smem + 2 * Cfg::kQBytes;         // kStages tiles
    FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(smem + Cfg::kSmemData);

    const unsigned warp = warp_id();
    const unsigned lane = lane_id();
    const int bh = blockIdx.y;
    const int m0 = blockIdx.x * (2 * kTileM);
    const int n_kv = (Nk + kTileN - 1) / kTileN;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_ready[t], 128);
        }
        mbar_init(&bars->o_final, 1);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tmem = bars->tmem_base;
    volatile int* abort_flag = &bars->abort_flag;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(&bars->q_full, 2 * Cfg::kQBytes);
            for (int t = 0; t < 2; ++t)
                for (int b = 0; b < D / 64; ++b)
                    tma_load_3d(sQ + t * Cfg::kQBytes + b * Cfg::kBoxBytes, &tm_q, &bars->q_full,
                                b * 64, m0 + t * kTileM, bh);
            const int n_tiles = 2 * n_kv;
            int issued = 0;
            for (int c = 0; c < n_tiles; ++c) {
                const int s = c % Cfg::kStages;
                if (c >= Cfg::kStages) {
                    if (!mbar_wait(&bars->empty[s], ((c / Cfg::kStages) - 1) & 1, abort_flag)) break;
                }
                uint8_t* dst = sRing + s * Cfg::kTileBytes;
                const CUtensorMap* tm = (c & 1) ? &tm_v : &tm_k;
                const int key0 = (c >> 1) * kTileN;
                mbar_arrive_expect_tx(&bars->full[s], Cfg::kTileBytes);
                for (int b = 0; b < D / 64; ++b)
                    tma_load_3d(dst + b * Cfg::kBoxBytes, tm, &bars->full[s], b * 64, key0, bh);
                issued = c + 1;
            }
            // Never leave with copies in flight: wait until the last loads landed.
            for (int c = (issued > Cfg::kStages ? issued - Cfg::kStages : 0); c < issued; ++c)
                mbar_wait(&bars->full[c % Cfg::kStages], (c / Cfg::kStages) & 1, nullptr);
            mbar_wait(&bars->q_full, 0, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // The issuing thread does as little as possible between tcgen05.mma
        // instructions: descriptors are built once and stepped by 32-bit adds
        // of compile-time offsets; ring stages are tracked incrementally.
        if (lane == 0) {
            constexpr unsigned idesc_s = make_idesc_bf16(128, kTileN, 0, 0);
            constexpr unsigned idesc_o = make_idesc_bf16(128, D, 0, 1);
            const uint32_t q_lo0 = desc_lo_kmajor(smem_u32(sQ));
            const uint32_t q_lo1 = desc_lo_kmajor(smem_u32(sQ + Cfg::kQBytes));
            const uint32_t ring_k_lo = desc_lo_kmajor(smem_u32(sRing));
            const uint32_t ring_v_lo = desc_lo_mnmajor(smem_u32(sRing));
            constexpr uint32_t kStageStep = Cfg::kTileBytes >> 4;   // start-field step between ring stages
            const unsigned tS0 = tmem, tS1 = tmem + 128u, tO0 = tmem + 256u, tO1 = tmem + 384u;
            bool ok = mbar_wait(&bars->q_full, 0, abort_flag);
            int stage = 0;
            unsigned phase = 0;
            // consume one ring tile: wait until it landed, return its stage offset (16-byte units)
            auto next_tile = [&](uint32_t& off, int& st_used) -> bool {
                if (!mbar_wait(&bars->full[stage], phase, abort_flag)) return false;
                off = (uint32_t)stage * kStageStep;
                st_used = stage;
                if (++stage == Cfg::kStages) { stage = 0; phase ^= 1u; }
                return true;
            };
            auto issue_s = [&](unsigned tS, uint32_t q_lo, uint32_t k_off) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss_lo(tS, q_lo + kmajor_step(kk), ring_k_lo + k_off + kmajor_step(kk), idesc_s, kk > 0);
            };
            auto issue_pv = [&](unsigned tO, unsigned tS, uint32_t v_off, unsigned acc0) {
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk)
                    mma_ts_lo(tO, tS + kk * 8, ring_v_lo + v_off + mnmajor_step(kk), idesc_o, (acc0 | kk) ? 1u : 0u);
            };
            uint32_t k_off = 0;
            int k_stage = 0;
            if (ok) ok = next_tile(k_off, k_stage);
            if (ok) {
                tc_fence_after();
                issue_s(tS0, q_lo0, k_off);
                mma_commit(&bars->s_full[0]);
                issue_s(tS1, q_lo1, k_off);
                mma_commit(&bars->s_full[1]);
                mma_commit(&bars->empty[k_stage]);
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                const bool more = (j + 1 < n_kv);
                const unsigned acc0 = j > 0 ? 1u : 0u;
                uint32_t v_off = 0;
                int v_stage = 0;
                if (!(ok = next_tile(v_off, v_stage))) break;
                // tile 0: O_0 += P_0 V_j, then S_0 = Q_0 K_{j+1}^T
                if (!(ok = mbar_wait(&bars->p_ready[0], j & 1, abort_flag))) break;
                tc_fence_after();
                issue_pv(tO0, tS0, v_off, acc0);
                if (more) {
                    if (!(ok = next_tile(k_off, k_stage))) break;
                    tc_fence_after();
                    issue_s(tS0, q_lo0, k_off);
                    mma_commit(&bars->s_full[0]);
                }
                // tile 1: O_1 += P_1 V_j, then S_1 = Q_1 K_{j+1}^T
                if (!(ok = mbar_wait(&bars->p_ready[1], j & 1, abort_flag))) break;
                tc_fence_after();
                issue_pv(tO1, tS1, v_off, acc0);
                mma_commit(&bars->empty[v_stage]);
                if (more) {
                    issue_s(tS1, q_lo1, k_off);
                    mma_commit(&bars->s_full[1]);
                    mma_commit(&bars->empty[k_stage]);
                }
            }
            if (ok) mma_commit(&bars->o_final);
            // drain: every MMA issued above has completed before TMEM is freed
            mma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, nullptr);
        }
    } else {
        // ------------------------------------------------ softmax / epilogue
        const int t = (warp - 2) >> 2;                     // query tile of these four warps
        const unsigned sub = warp & 3;                     // TMEM sub-partition (lanes 32*sub..)
        const int r = sub * 32 + lane;                     // row within the tile
        const unsigned lane_off = (sub * 32u) << 16;
        const unsigned tS = tmem + lane_off + (t ? 128u : 0u);
        const unsigned tO = tmem + lane_off + (t ? 384u : 256u);
        const float c_log2 = scale * kLog2e;
        float m_ref = -INFINITY;  // reference maximum, base-2 units of scale*s
        float l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            if (!(ok = mbar_wait(&bars->s_full[t], j & 1, abort_flag))) break;
            tc_fence_after();
            uint32_t sr[kTileN];
#pragma unroll
            for (int c0 = 0; c0 < kTileN; c0 += 32)
                tmem_ld32(tS + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[c0]));
            tmem_wait_ld();
            const int nvalid = Nk - j * kTileN;
            if (nvalid < kTileN) {
#pragma unroll
                for (int c = 0; c < kTileN; ++c)
                    if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
            }
            // row maximum as 8 independent chains (one thread owns the row, so a
            // single 128-long dependent chain would dominate the softmax latency)
            float mxa[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mxa[i] = __uint_as_float(sr[i]);
#pragma unroll
            for (int c = 8; c < kTileN; c += 8)
#pragma unroll
                for (int i = 0; i < 8; ++i) mxa[i] = fmaxf(mxa[i], __uint_as_float(sr[c + i]));
            const float mx = fmaxf(fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3])),
                                   fmaxf(fmaxf(mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7])));
            const float m_blk = mx * c_log2;
            float m_new = m_ref;
            bool rescale = false;
            float alpha = 1.f;
            if (j == 0) {
                m_new = m_blk;
            } else if (__any_sync(0xffffffffu, m_blk - m_ref > kRescaleThreshold)) {
                // warp-uniform decision: tcgen05.ld/st below are warp-collective
                m_new = fmaxf(m_ref, m_blk);
                alpha = ex2_approx(m_ref - m_new);
                rescale = true;
            }
            m_ref = m_new;
            l *= alpha;
            // row sum as 8 independent partial sums (same reason as the maximum)
            float rsa[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) rsa[i] = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < kTileN; c0 += 32) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c0 + c]), c_log2, -m_ref));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c0 + c + 1]), c_log2, -m_ref));
                    rsa[(c / 2) & 7] += p0 + p1;
                    pk[c / 2] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tS + c0 / 2, pk);
            }
            l += ((rsa[0] + rsa[1]) + (rsa[2] + rsa[3])) + ((rsa[4] + rsa[5]) + (rsa[6] + rsa[7]));
            if (rescale) {
                // PV_t(j-1) has completed (it was issued before S_t(j), whose
                // commit we waited on), so O_t can be rescaled in place.
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t ov[32];
                    tmem_ld32(tO + c0, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    tmem_st32(tO + c0, ov);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_ready[t]);
        }
        if (ok && mbar_wait(&bars->o_final, 0, abort_flag)) {
            tc_fence_after();
            const int row = m0 + t * kTileM + r;
            const float inv_l = 1.f / l;
            uint16_t* orow = o + ((size_t)bh * Nq + row) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(tO + c0, ov);
                tmem_wait_ld();
                if (row < Nq) {
                    uint32_t packed[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        packed[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l,
                                                __uint_as_float(ov[2 * i + 1]) * inv_l);
                    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                }
            }
            if (row < Nq) lse[(size_t)bh * Nq + row] = (m_ref + __log2f(l)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_d(const Bf16FwdArgs& a, cudaStream_t stream) {
    using Cfg = FwdCfg<D>;
    auto kern = fwd_bf16_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid((a.Nq + 2 * kTileM - 1) / (2 * kTileM), a.BH, 1);
    kern<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.o, a.lse, a.Nq, a.Nk, a.scale);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const Bf16FwdArgs& a, cudaStream_t stream) {
    if (a.D == 64) return launch_d<64>(a, stream);
    if (a.D == 128) return launch_d<128>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace mea
