// bwd_bf16.cu -- bf16 backward on the 5th-generation tensor cores (sm_100a).
//
// Method: "Self-attention Does Not Need O(n^2) Memory" (English summary,
// method bullet on differentiation): nothing of size n x n is stored by the
// forward; the backward recomputes the probabilities block by block from the
// saved per-row lse (checkpointing), P = exp(scale q k^T - lse).  The gradient
// formulas are ordinary softmax calculus:
//     dV = P^T dO,  dP = dO V^T,  D_i = sum_d dO_id O_id,  dS = P o (dP - D),
//     dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels on one stream:
//   bwd_pre      D_i = sum_d dO_id O_id (fp32) and zeroes the fp32 dQ accumulator.
//   bwd_main     one CTA per (batch*head, 128-key tile); loops over 128-query
//                tiles.  Everything is computed transposed (keys on TMEM lanes):
//                  S^T  = K Q_i^T          (smem x smem -> TMEM)
//                  dP^T = V dO_i^T         (smem x smem -> TMEM)
//                  dV  += P^T dO_i         (P^T from TMEM, bf16)
//                  dQ_i^T = K^T dS^T       (both from smem, bf16) -> fp32 TMA reduce-add
//                  dK  += dS^T Q_i         (both from smem, bf16)
//                dS^T is written once, to swizzled shared memory, where it is
//                the MN-major B operand of dQ^T and the K-major A operand of
//                dK.  dQ^T is issued before dK, so the dQ warps copy it out of
//                TMEM (and dP^T of the next tile can take its columns) while
//                dK runs.
//                dQ is formed transposed so that TMEM lanes are head dims: each
//                warp of the dQ warpgroup stages [64 queries x 32 head dims] of
//                it in shared memory and one TMA reduce-add sends it to the dQ
//                accumulator.  For D = 64 the MMA still has M = 128; lanes
//                64..127 hold products with the V tile that follows K in
//                shared memory and are ignored.
//   bwd_dq_final dq = bf16(scale * dQacc).
//
// Roles in bwd_main (512 threads, four warpgroups):
//   warp 0       TMEM allocator, then TMA producer (K, V once; then Q_i, dO_i;
//                no multicast)
//   warp 1       MMA issuer (one thread)
//   warps 4-11   two compute warpgroups: thread (warp w, lane) owns key row
//                32*(w%4)+lane (the TMEM lane warp w can reach) and query half
//                (w-4)/4 of every tile: P^T (to TMEM) and dS^T (to smem)
//   warps 12-15  dQ warpgroup: copies dQ_i^T out of TMEM (freeing it at once),
//                stages it in its own shared-memory buffer and hands it to the
//                TMA engine as fp32 reduce-adds into the dQ accumulator; also
//                stages the lse / D values of later query tiles.
// Shared memory (D = 128): K, V 32 KB each; Q ring 2 x 32 KB; dO 32 KB (one
// buffer: dead after dV(i)); dS^T 32 KB; dQ staging 32 KB; lse/D 2 KB.
// Every thread runs within 128 registers (512 threads x 128 = the register
// file); P^T is kept in registers as packed bf16 pairs to make that fit.
// TMEM: S^T [0,128)  dP^T [128,256)  dV [256,256+D)  dK [256+D, 256+2D)
//       dQ^T (128 query columns): D=128 reuses the dP^T columns, D=64 uses [384,512).
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mea {
namespace {

constexpr int kTile = 128;
constexpr int kThreads = 512;
constexpr int kComputeThreads = 256;
constexpr int kDrainThreads = 128;
// Persistent backward CTAs pay off while an item's query loop is short
// (B32 H8 N512: 12 % faster); at 32 query tiles per item they measured 18 % slower.
constexpr int kBwdPersistMaxQTiles = 8;
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ pre

// delta = sum_d dO * O (fp32) per query row, and the row of the fp32 dQ
// accumulator := 0.  HBM-bound: each lane loads 16 bytes (8 bf16) of O and of
// dO, D/8 lanes share a row, and a warp keeps kPreRows rows of loads in flight
// before reducing (one 4-byte load per lane and row left too few bytes in
// flight to stream HBM).
constexpr int kPreRows = 4;   // row groups per warp per pass
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dO,
                                                      float* __restrict__ delta, float* __restrict__ dq_acc,
                                                      long long rows) {
    constexpr int LPR = D / 8;          // lanes per row
    constexpr int RPW = 32 / LPR;       // rows per warp and row group
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR, l = lane % LPR;
    const long long warp_g = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long row0 = warp_g * (RPW * kPreRows) + sub;
    uint4 ov[kPreRows], dv[kPreRows];
#pragma unroll
    for (int u = 0; u < kPreRows; ++u) {
        const long long r = row0 + u * RPW;
        if (r < rows) {
            ov[u] = *reinterpret_cast<const uint4*>(o + r * D + 8 * l);
            dv[u] = *reinterpret_cast<const uint4*>(dO + r * D + 8 * l);
        } else {
            ov[u] = dv[u] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int u = 0; u < kPreRows; ++u) {
        const uint32_t ow[4] = {ov[u].x, ov[u].y, ov[u].z, ov[u].w};
        const uint32_t dw[4] = {dv[u].x, dv[u].y, dv[u].z, dv[u].w};
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            acc = fmaf(__uint_as_float(ow[c] << 16), __uint_as_float(dw[c] << 16), acc);
            acc = fmaf(__uint_as_float(ow[c] & 0xffff0000u), __uint_as_float(dw[c] & 0xffff0000u), acc);
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        const long long r = row0 + u * RPW;
        if (r < rows) {
            if (l == 0) delta[r] = acc;
            if (dq_acc != nullptr) {   // accumulating callers own (and keep) their dQ accumulator
                float4* z = reinterpret_cast<float4*>(dq_acc + r * D) + 2 * l;
                z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
                z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
}

// ------------------------------------------------------------- finalise

// dq = bf16(scale * dQacc): each thread converts kFinalVecs float4 groups, all
// loads issued before the first store.
constexpr int kFinalVecs = 4;
__global__ void __launch_bounds__(256) bwd_dq_final_kernel(const float* __restrict__ dq_acc, uint16_t* __restrict__ dq,
                                                           long long n4, float scale) {
    const long long base = (long long)blockIdx.x * blockDim.x * kFinalVecs + threadIdx.x;
    float4 a[kFinalVecs];
#pragma unroll
    for (int u = 0; u < kFinalVecs; ++u) {
        const long long i = base + (long long)u * blockDim.x;
        a[u] = i < n4 ? reinterpret_cast<const float4*>(dq_acc)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kFinalVecs; ++u) {
        const long long i = base + (long long)u * blockDim.x;
        if (i < n4) {
            uint2 r;
            r.x = pack_bf16x2(a[u].x * scale, a[u].y * scale);
            r.y = pack_bf16x2(a[u].z * scale, a[u].w * scale);
            reinterpret_cast<uint2*>(dq)[i] = r;
        }
    }
}

// fp32 accumulator -> output dtype: out = mul * acc (bf16 round to nearest even, or fp32)
__global__ void accum_convert_kernel(const float* __restrict__ acc, void* __restrict__ out, long long n4, float mul,
                                     bool bf16) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4 a = reinterpret_cast<const float4*>(acc)[i];
    if (bf16) {
        uint2 r;
        r.x = pack_bf16x2(a.x * mul, a.y * mul);
        r.y = pack_bf16x2(a.z * mul, a.w * mul);
        reinterpret_cast<uint2*>(out)[i] = r;
    } else {
        reinterpret_cast<float4*>(out)[i] = make_float4(a.x * mul, a.y * mul, a.z * mul, a.w * mul);
    }
}

// ----------------------------------------------------------------- main

template <int D, bool PERSIST>
struct BwdCfg {
    static constexpr int kKVBytes = kTile * D * 2;      // one K (or V, Q, dO) tile
    static constexpr int kDSBytes = kTile * kTile * 2;  // dS^T tile, bf16
    static constexpr int kStageBytes = 4 * 64 * 32 * 4; // dQ staging: 4 warps x [64 queries x 32 floats]
    static constexpr int kBoxBytes = 128 * 128;
    // K/V buffers: persistent CTAs load the next item's K and V into the
    // other buffer while the current item finishes.  V must follow K in each
    // buffer (read as K^T rows 64..127 at D = 64).
    static constexpr int kKVBufs = PERSIST ? 2 : 1;
    static constexpr int kKVBufBytes = 2 * kKVBytes;
    static constexpr int offK = 0;
    static constexpr int offV = kKVBytes;
    static constexpr int offQ = kKVBufs * kKVBufBytes;  // Q_i ring, 2 stages
    static constexpr int offDO = offQ + 2 * kKVBytes;   // dO_i, single buffer (dead after dV(i))
    static constexpr int offDS = offDO + kKVBytes;
    static constexpr int offStage = offDS + kDSBytes;
    static constexpr int offStats = offStage + kStageBytes;    // lse2[2][128], delta[2][128]
    static constexpr int offBars = offStats + 4 * kTile * 4;
    static constexpr int kSmemBytes = offBars + 256;
    static constexpr bool kDqInDp = (D == 128);
    static constexpr unsigned colS = 0, colDP = 128, colDV = 256, colDK = 256 + D;
    static constexpr unsigned colDQ = kDqInDp ? 128u : 384u;   // 128 columns (queries)
};

struct BwdBarriers {
    uint64_t kv_full[2];
    uint64_t kv_empty[2];
    uint64_t q_full[2];
    uint64_t q_empty[2];
    uint64_t do_full, do_empty;
    uint64_t s_full, dp_full, dq_full;
    uint64_t p_ready, ds_ready, dq_free;
    uint64_t stats[2];
    uint64_t final_done;
    uint64_t acc_free;
    uint64_t drain;
    unsigned tmem_base;
    int abort_flag;
};

// bf16 A operand packed in TMEM by the two compute warpgroups: query half g
// occupies columns [64 g, 64 g + 32) of its region.
__device__ __forceinline__ unsigned packed_col(int kk) { return (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8; }

// Work items are (batch*head, 128-key tile) pairs.  Without PERSIST each CTA
// owns one (grid = key tiles x heads, as before); with PERSIST a grid of at
// most one CTA per SM walks items c, c + G, c + 2G, ...: the next item's K, V
// load into the other buffer and its first S^T is issued while the current
// item's last tile and epilogue are still in flight.  The query tiles of all
// of a CTA's items form one sequence T = li * n_q + i; every per-tile barrier
// takes its phase from T.
template <int D, bool PERSIST>
__global__ void __launch_bounds__(kThreads, 1)
bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dq, const float* __restrict__ lse,
                const float* __restrict__ delta, uint16_t* __restrict__ dk, uint16_t* __restrict__ dv,
                float* __restrict__ dk_acc, float* __restrict__ dv_acc, int BH, int Nq, int Nk, float scale) {
    using Cfg = BwdCfg<D, PERSIST>;
    extern __shared__ __align__(1024) uint8_t smem[];
    BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + Cfg::offBars);
    float* s_lse2 = reinterpret_cast<float*>(smem + Cfg::offStats);          // [2][128]
    float* s_delta = s_lse2 + 2 * kTile;                                      // [2][128]

    const unsigned warp = warp_id();
    const unsigned lane = lane_id();
    const int n_q = (Nq + kTile - 1) / kTile;
    const int n_kt = (Nk + kTile - 1) / kTile;
    const int n_items = PERSIST ? BH * n_kt : 1;
    const int first = PERSIST ? (int)blockIdx.x : 0;
    const int stride = PERSIST ? (int)gridDim.x : 1;
    const int my_items = first < n_items ? (n_items - first + stride - 1) / stride : 0;
    const int total = my_items * n_q;   // query tiles of this CTA over all its items
    // (bh, first key) of this CTA's li-th item
    auto item_bh = [&](int li) -> int { return PERSIST ? (first + li * stride) / n_kt : (int)blockIdx.y; };
    auto item_n0 = [&](int li) -> int {
        return (PERSIST ? (first + li * stride) % n_kt : (int)blockIdx.x) * kTile;
    };

    if ((smem_u32(smem) & 1023u) != 0) {     // swizzle atoms need 1024-byte alignment
        if (threadIdx.x == 0) flag_timeout();
        return;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        mbar_init(&bars->do_full, 1);
        mbar_init(&bars->do_empty, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->p_ready, kComputeThreads);
        mbar_init(&bars->ds_ready, kComputeThreads);
        mbar_init(&bars->dq_free, kDrainThreads);
        mbar_init(&bars->stats[0], kDrainThreads);
        mbar_init(&bars->stats[1], kDrainThreads);
        mbar_init(&bars->final_done, 1);
        mbar_init(&bars->acc_free, kComputeThreads);
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
    uint8_t* sQ = smem + Cfg::offQ;
    uint8_t* sDO = smem + Cfg::offDO;
    uint8_t* sDS = smem + Cfg::offDS;
    uint8_t* sStage = smem + Cfg::offStage;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_do);
            // K, V of item li into buffer li % kKVBufs, once the item that used it last is done
            auto load_kv = [&](int li) -> bool {
                const int b = li % Cfg::kKVBufs;
                if (li >= Cfg::kKVBufs &&
                    !mbar_wait(&bars->kv_empty[b], ((li / Cfg::kKVBufs) - 1) & 1, abort_flag))
                    return false;
                uint8_t* sK = smem + b * Cfg::kKVBufBytes + Cfg::offK;
                uint8_t* sV = smem + b * Cfg::kKVBufBytes + Cfg::offV;
                const int bh = item_bh(li), n0 = item_n0(li);
                mbar_arrive_expect_tx(&bars->kv_full[b], 2 * Cfg::kKVBytes);
                for (int bx = 0; bx < D / 64; ++bx) {
                    tma_load_3d(sK + bx * Cfg::kBoxBytes, &tm_k, &bars->kv_full[b], bx * 64, n0, bh);
                    tma_load_3d(sV + bx * Cfg::kBoxBytes, &tm_v, &bars->kv_full[b], bx * 64, n0, bh);
                }
                return true;
            };
            // Q_T: 2-stage ring (Q_{T+1} is read by S^T(T+1) before dK(T) frees Q_T).
            // dO_T: single buffer, reloaded once dV(T) and dP^T(T) have read it.
            // tile T's (query tile, batch*head) without a division per tile: the
            // producer walks T in order, so the item is tracked incrementally
            auto tile_of = [&](int T, int& i, int& bh) {
                const int li = PERSIST ? T / n_q : 0;
                i = T - li * n_q;
                bh = item_bh(li);
            };
            auto load_q = [&](int T) {
                int i, bh;
                tile_of(T, i, bh);
                mbar_arrive_expect_tx(&bars->q_full[T & 1], Cfg::kKVBytes);
                for (int bx = 0; bx < D / 64; ++bx)
                    tma_load_3d(sQ + (T & 1) * Cfg::kKVBytes + bx * Cfg::kBoxBytes, &tm_q, &bars->q_full[T & 1],
                                bx * 64, i * kTile, bh);
            };
            auto load_do = [&](int T) {
                int i, bh;
                tile_of(T, i, bh);
                mbar_arrive_expect_tx(&bars->do_full, Cfg::kKVBytes);
                for (int bx = 0; bx < D / 64; ++bx)
                    tma_load_3d(sDO + bx * Cfg::kBoxBytes, &tm_do, &bars->do_full, bx * 64, i * kTile, bh);
            };
            int q_issued = 0, do_issued = 0, kv_issued = 0;
            bool ok = total > 0 && load_kv(0);
            if (ok) {
                kv_issued = 1;
                load_q(0);
                load_do(0);
                q_issued = do_issued = 1;
                if (total > 1) { load_q(1); q_issued = 2; }
            }
            for (int T = 0; ok && T < total; ++T) {
                // the next item's K, V as soon as its buffer frees (persistent CTAs)
                if (PERSIST && kv_issued < my_items && kv_issued * n_q <= T + n_q) {
                    if (!(ok = load_kv(kv_issued))) break;
                    ++kv_issued;
                }
                // dO_{T+1} as soon as dV(T) has read dO_T, before Q_{T+2}
                // (whose buffer frees only after dK(T))
                if (T + 1 < total) {
                    if (!(ok = mbar_wait(&bars->do_empty, T & 1, abort_flag))) break;
                    load_do(T + 1);
                    do_issued = T + 2;
                }
                if (T + 2 < total) {
                    if (!(ok = mbar_wait(&bars->q_empty[T & 1], (T >> 1) & 1, abort_flag))) break;
                    load_q(T + 2);
                    q_issued = T + 3;
                }
            }
            // Never leave with copies in flight: wait until the last loads landed.
            for (int T = (q_issued > 2 ? q_issued - 2 : 0); T < q_issued; ++T)
                mbar_wait(&bars->q_full[T & 1], (T >> 1) & 1, nullptr);
            if (do_issued > 0) mbar_wait(&bars->do_full, (do_issued - 1) & 1, nullptr);
            for (int li = (kv_issued > Cfg::kKVBufs ? kv_issued - Cfg::kKVBufs : 0); li < kv_issued; ++li)
                mbar_wait(&bars->kv_full[li % Cfg::kKVBufs], (li / Cfg::kKVBufs) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // Descriptors are built once and stepped by 32-bit adds of compile-time
        // offsets, so the issuing thread keeps the tensor pipe fed.
        if (lane == 0) {
            constexpr unsigned idesc_t = make_idesc_bf16(128, 128, 0, 0);   // S^T, dP^T
            constexpr unsigned idesc_g = make_idesc_bf16(128, D, 0, 1);     // dV, dK (A in TMEM)
            constexpr unsigned idesc_q = make_idesc_bf16(128, 128, 1, 1);   // dQ^T (A = K^T, B = dS^T, MN-major)
            constexpr unsigned idesc_k = make_idesc_bf16(128, D, 0, 1);     // dK (A = dS^T K-major, B = Q MN-major)
            constexpr uint32_t kKVBufStep = Cfg::kKVBufBytes >> 4;          // start-field step between K/V buffers
            const uint32_t k_lo0 = desc_lo_kmajor(smem_u32(smem + Cfg::offK));   // K as A of S^T
            const uint32_t kt_lo0 = desc_lo_mnmajor(smem_u32(smem + Cfg::offK)); // K^T as A of dQ^T
            const uint32_t v_lo0 = desc_lo_kmajor(smem_u32(smem + Cfg::offV));
            const uint32_t ds_lo = desc_lo_mnmajor(smem_u32(sDS));          // dS^T as B of dQ^T
            const uint32_t dsk_lo = desc_lo_kmajor(smem_u32(sDS));          // dS^T as A of dK
            const uint32_t do_k_lo = desc_lo_kmajor(smem_u32(sDO));         // dO as B of dP^T
            const uint32_t do_mn_lo = desc_lo_mnmajor(smem_u32(sDO));       // dO as B of dV
            const uint32_t q_k_lo0 = desc_lo_kmajor(smem_u32(sQ));
            const uint32_t q_mn_lo0 = desc_lo_mnmajor(smem_u32(sQ));
            constexpr uint32_t kQStep = Cfg::kKVBytes >> 4;                  // start-field step between Q stages
            const unsigned tS = tmem + Cfg::colS, tDP = tmem + Cfg::colDP, tDV = tmem + Cfg::colDV,
                           tDK = tmem + Cfg::colDK, tDQ = tmem + Cfg::colDQ;
            // S^T(T) = K Q_T^T into the S columns (once Q_T and the item's K have landed)
            auto issue_s = [&](int T, int li, bool new_item) -> bool {
                const int b = li % Cfg::kKVBufs;
                if (new_item && !mbar_wait(&bars->kv_full[b], (li / Cfg::kKVBufs) & 1, abort_flag)) return false;
                if (!mbar_wait(&bars->q_full[T & 1], (T >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_lo = k_lo0 + (uint32_t)b * kKVBufStep;
                const uint32_t q_lo = q_k_lo0 + (uint32_t)(T & 1) * kQStep;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss_lo(tS, k_lo + kmajor_step(kk), q_lo + kmajor_step(kk), idesc_t, kk > 0);
                mma_commit(&bars->s_full);
                return true;
            };
            bool ok = total > 0 && issue_s(0, 0, true);
            for (int li = 0; ok && li < my_items; ++li) {
                const uint32_t kvoff = (uint32_t)(li % Cfg::kKVBufs) * kKVBufStep;
                const uint32_t kt_lo = kt_lo0 + kvoff;
                const uint32_t v_lo = v_lo0 + kvoff;
                for (int i = 0; i < n_q; ++i) {
                    const int T = li * n_q + i;
                    const uint32_t q_mn_lo = q_mn_lo0 + (uint32_t)(T & 1) * kQStep;
                    const unsigned acc0 = i > 0 ? 1u : 0u;
                    // dP^T = V dO_T^T  (D=128: dP columns held dQ_{T-1} until the dQ warps copied it out)
                    if (!(ok = mbar_wait(&bars->do_full, T & 1, abort_flag))) break;
                    if (Cfg::kDqInDp && T > 0) {
                        if (!(ok = mbar_wait(&bars->dq_free, (T - 1) & 1, abort_flag))) break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss_lo(tDP, v_lo + kmajor_step(kk), do_k_lo + kmajor_step(kk), idesc_t, kk > 0);
                    mma_commit(&bars->dp_full);
                    // dV += P^T dO_T; the item's first dV and dK overwrite the
                    // accumulators, which the previous item's epilogue must have read
                    if (!(ok = mbar_wait(&bars->p_ready, T & 1, abort_flag))) break;
                    if (i == 0 && li > 0 && !(ok = mbar_wait(&bars->acc_free, (li - 1) & 1, abort_flag))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        mma_ts_lo(tDV, tS + packed_col(kk), do_mn_lo + mnmajor_step(kk), idesc_g, (acc0 | kk) ? 1u : 0u);
                    mma_commit(&bars->do_empty);           // dO_T read by dP^T(T) and dV(T)
                    // Software pipeline: S^T(T+1) -- of this item, or of the next
                    // one (persistent CTAs) -- right after dV(T)
                    if (T + 1 < total && !(ok = issue_s(T + 1, (i + 1 < n_q) ? li : li + 1, i + 1 == n_q))) break;
                    // dQ_T^T = K^T dS^T first, so the dQ warps copy it out while dK
                    // runs; dK += dS^T Q_T then reads dS^T from shared memory too
                    if (!(ok = mbar_wait(&bars->ds_ready, T & 1, abort_flag))) break;
                    tc_fence_after();
                    if (!Cfg::kDqInDp && T > 0) {
                        if (!(ok = mbar_wait(&bars->dq_free, (T - 1) & 1, abort_flag))) break;
                        tc_fence_after();
                    }
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        mma_ss_lo(tDQ, kt_lo + mnmajor_step(kk), ds_lo + mnmajor_step(kk), idesc_q, kk > 0);
                    mma_commit(&bars->dq_full);
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        mma_ss_lo(tDK, dsk_lo + kmajor_step(kk), q_mn_lo + mnmajor_step(kk), idesc_k, (acc0 | kk) ? 1u : 0u);
                    mma_commit(&bars->q_empty[T & 1]);
                }
                if (!ok) break;
                mma_commit(&bars->final_done);                  // the item's dV, dK are complete
                mma_commit(&bars->kv_empty[li % Cfg::kKVBufs]);  // and its K, V are no longer read
            }
            mma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, nullptr);
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------ compute warps
        const int g = (warp - 4) >> 2;                 // query half of every tile
        const unsigned sub = warp & 3;
        const int kr = sub * 32 + lane;                // key row within the tile (TMEM lane)
        const unsigned lane_off = (sub * 32u) << 16;
        const float c_log2 = scale * kLog2e;
        uint32_t pp[32];   // P^T of the current tile as packed bf16 pairs (exactly what dV used)
        // ---- P^T = exp2(scale*log2e * S^T - lse2), query half g, tile T of an item whose keys start at n0
        auto do_p = [&](int T, int n0) -> bool {
            const bool key_ok = (n0 + kr) < Nk;
            const float* l2 = s_lse2 + (T & 1) * kTile + 64 * g;
            if (!mbar_wait(&bars->stats[T & 1], (T >> 1) & 1, abort_flag)) return false;
            if (!mbar_wait(&bars->s_full, T & 1, abort_flag)) return false;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t sr[32];
                tmem_ld32(tmem + lane_off + Cfg::colS + 64 * g + 32 * h, sr);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float p0 = key_ok ? ex2_approx(fmaf(__uint_as_float(sr[2 * c]), c_log2, -l2[32 * h + 2 * c])) : 0.f;
                    const float p1 =
                        key_ok ? ex2_approx(fmaf(__uint_as_float(sr[2 * c + 1]), c_log2, -l2[32 * h + 2 * c + 1])) : 0.f;
                    pp[16 * h + c] = pack_bf16x2(p0, p1);
                }
                // packed P^T overwrites S^T columns this thread has already read
                tmem_st16(tmem + lane_off + Cfg::colS + 64 * g + 16 * h, *reinterpret_cast<const uint32_t(*)[16]>(&pp[16 * h]));
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_ready);
            return true;
        };
        // ---- dS^T = P^T o (dP^T - delta): bf16 to shared memory (for dQ and dK)
        auto do_ds = [&](int T) -> bool {
            const float* dl = s_delta + (T & 1) * kTile + 64 * g;
            if (!mbar_wait(&bars->dp_full, T & 1, abort_flag)) return false;
            // dp_full(T) was committed after dQ(T-1) and dK(T-1), the readers of the dS buffer
            tc_fence_after();
            // dS^T (keys x queries) in shared memory: MN-major operand, query block g,
            // row = key, 16-byte chunk c of the 128-byte row swizzled by (key mod 8).
            uint8_t* row = sDS + g * Cfg::kBoxBytes + kr * 128;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t dr[32];
                tmem_ld32(tmem + lane_off + Cfg::colDP + 64 * g + 32 * h, dr);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int q = 32 * h + 2 * c;
                    const uint32_t pr = pp[16 * h + c];
                    const float d0 = __uint_as_float(pr << 16) * (__uint_as_float(dr[2 * c]) - dl[q]);
                    const float d1 = __uint_as_float(pr & 0xffff0000u) * (__uint_as_float(dr[2 * c + 1]) - dl[q + 1]);
                    pk[c] = pack_bf16x2(d0, d1);
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int pc = (4 * h + c) ^ (kr & 7);
                    *reinterpret_cast<uint4*>(row + pc * 16) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_ready);
            return true;
        };
        // Order per tile: dS(T), then P(T+1) (overlapping dK(T), dQ(T) on the
        // tensor cores, and, at the end of an item, its epilogue); the dQ warps
        // drain dQ(T) meanwhile.
        bool ok = total > 0 && do_p(0, item_n0(0));
        for (int li = 0; ok && li < my_items; ++li) {
            const int n0 = item_n0(li);
            for (int i = 0; i < n_q; ++i) {
                const int T = li * n_q + i;
                if (!(ok = do_ds(T))) break;
                if (T + 1 < total && !(ok = do_p(T + 1, (i + 1 < n_q) ? n0 : item_n0(li + 1)))) break;
            }
            if (!ok) break;
            // ---- epilogue of the item: dV, dK (scaled) rows of its keys, or, for an
            //      accumulating caller, dV and the unscaled dS^T Q added to its fp32 sums
            if (!(ok = mbar_wait(&bars->final_done, li & 1, abort_flag))) break;
            tc_fence_after();
            const int bh = item_bh(li);
            const int key = n0 + kr;
            const bool key_ok = key < Nk;
            const bool accumulate = dk_acc != nullptr;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const unsigned col = (which == 0 ? Cfg::colDV : Cfg::colDK) + g * (D / 2);
                const float mul = (which == 0 || accumulate) ? 1.f : scale;
                const size_t off = ((size_t)bh * Nk + key) * D + g * (D / 2);
#pragma unroll
                for (int c0 = 0; c0 < D / 2; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + col + c0, r);
                    tmem_wait_ld();
                    if (key_ok && accumulate) {
                        float4* f4 = reinterpret_cast<float4*>((which == 0 ? dv_acc : dk_acc) + off + c0);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            float4 x = f4[c];
                            x.x += __uint_as_float(r[4 * c]);
                            x.y += __uint_as_float(r[4 * c + 1]);
                            x.z += __uint_as_float(r[4 * c + 2]);
                            x.w += __uint_as_float(r[4 * c + 3]);
                            f4[c] = x;
                        }
                    } else if (key_ok) {
                        uint32_t pk[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            pk[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * mul, __uint_as_float(r[2 * c + 1]) * mul);
                        uint4* d4 = reinterpret_cast<uint4*>((which == 0 ? dv : dk) + off + c0);
#pragma unroll
                        for (int c = 0; c < 4; ++c) d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                    }
                }
            }
            // dV, dK have been read: the next item's first dV and dK may overwrite them
            tc_fence_before();
            mbar_arrive(&bars->acc_free);
        }
    } else if (warp >= 12) {
        // ------------------------------------------------ dQ warps (+ lse/D staging)
        const unsigned sub = warp & 3;
        const int d = sub * 32 + lane;                 // TMEM lane = head dim of dQ^T
        const unsigned lane_off = (sub * 32u) << 16;
        const bool active = d < D;                     // D = 64: lanes 64..127 hold nothing useful
        const int j = threadIdx.x - 384;               // 0..127
        float* stage = reinterpret_cast<float*>(sStage + sub * 8192);   // this warp: 64 rows x 32 floats
        auto stage_stats = [&](int T, int li, int i) {
            const size_t base = (size_t)item_bh(li) * Nq;
            const int row = i * kTile + j;
            s_lse2[(T & 1) * kTile + j] = (row < Nq) ? lse[base + row] * kLog2e : INFINITY;
            s_delta[(T & 1) * kTile + j] = (row < Nq) ? delta[base + row] : 0.f;
            mbar_arrive(&bars->stats[T & 1]);
        };
        // one half (64 queries) of dQ^T from registers to this warp's staging
        // buffer as [query][32 head dims], then one TMA reduce-add (not waited for)
        auto stage_and_reduce = [&](const uint32_t (&v)[64], int q0, int bh) {
            if (active) {
#pragma unroll
                for (int c = 0; c < 64; ++c) stage[c * 32 + lane] = __uint_as_float(v[c]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && active && q0 < Nq) {
                tma_reduce_add_3d(&tm_dq, stage, 32 * sub, q0, bh);
                bulk_commit_group();
            }
        };
        auto staging_reusable = [&]() {                // the TMA engine has read the staging buffer
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
        };
        // (item, query tile) of tile T + 2, advanced incrementally
        int s_li = 0, s_i = 0;
        auto advance = [&]() {
            if (++s_i == n_q) { s_i = 0; ++s_li; }
        };
        if (total > 0) { stage_stats(0, s_li, s_i); advance(); }
        if (total > 1) { stage_stats(1, s_li, s_i); advance(); }
        bool ok = true;
        int li = 0, i = 0, bh = item_bh(0);
        for (int T = 0; ok && T < total; ++T) {
            if (T > 0 && ++i == n_q) {
                i = 0;
                bh = item_bh(++li);
            }
            if (!(ok = mbar_wait(&bars->dq_full, T & 1, abort_flag))) break;
            tc_fence_after();
            uint32_t v[64];
            tmem_ld32(tmem + lane_off + Cfg::colDQ, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld32(tmem + lane_off + Cfg::colDQ + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tmem_wait_ld();
            stage_and_reduce(v, i * kTile, bh);
            tmem_ld32(tmem + lane_off + Cfg::colDQ + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld32(tmem + lane_off + Cfg::colDQ + 96, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->dq_free);               // dQ^T columns may be overwritten now
            // tile T's lse/D are no longer read (dS(T) is done): slot T&1 takes tile T+2
            if (T + 2 < total) {
                stage_stats(T + 2, s_li, s_i);
                advance();
            }
            staging_reusable();
            stage_and_reduce(v, i * kTile + 64, bh);
            staging_reusable();
        }
        if (lane == 0) bulk_wait_all();                // every reduce-add has completed
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool PERSIST>
cudaError_t launch_main(const Bf16BwdArgs& a, cudaStream_t stream) {
    using Cfg = BwdCfg<D, PERSIST>;
    static_assert(Cfg::kSmemBytes <= 232448, "shared memory budget");
    auto kern = bwd_main_kernel<D, PERSIST>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int n_kt = (a.Nk + kTile - 1) / kTile;
    dim3 grid(n_kt, a.BH, 1);
    if (PERSIST) {
        const long long items = (long long)n_kt * a.BH;
        grid = dim3((unsigned)(items < a.sm_count ? items : a.sm_count), 1, 1);
    }
    kern<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_do, a.tm_dq_acc, a.lse, a.delta,
                                                      a.dk, a.dv, a.dk_acc, a.dv_acc, a.BH, a.Nq, a.Nk, a.scale);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_accum_convert(const float* acc, void* out, long long n, float mul, bool bf16, cudaStream_t stream) {
    const long long n4 = n / 4;
    if (n4 == 0) return cudaSuccess;
    const int tpb = 256;
    accum_convert_kernel<<<(unsigned)((n4 + tpb - 1) / tpb), tpb, 0, stream>>>(acc, out, n4, mul, bf16);
    return cudaGetLastError();
}

cudaError_t launch_bwd_bf16(const Bf16BwdArgs& a, cudaStream_t stream, unsigned phases) {
    const long long rows = (long long)a.BH * a.Nq;
    if ((phases & kBwdPhasePre) && rows > 0) {
        const long long rows_per_warp = (long long)(32 / (a.D / 8)) * kPreRows;
        const long long warps = (rows + rows_per_warp - 1) / rows_per_warp;
        const unsigned blocks = (unsigned)((warps + 7) / 8);
        if (a.D == 64)
            bwd_pre_kernel<64><<<blocks, 256, 0, stream>>>(a.o, a.dO, a.delta, a.dq_acc, rows);
        else if (a.D == 128)
            bwd_pre_kernel<128><<<blocks, 256, 0, stream>>>(a.o, a.dO, a.delta, a.dq_acc, rows);
        else
            return cudaErrorInvalidValue;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaSuccess;
    if (phases & kBwdPhaseMain) {
        // D = 64 with few query tiles per key tile: persistent CTAs (two K/V
        // buffers fit), whose next item's loads overlap the current item's end;
        // otherwise one CTA per (head, key tile)
        const bool persist = a.D == 64 && (a.Nq + kTile - 1) / kTile <= kBwdPersistMaxQTiles;
        e = (a.D == 64) ? (persist ? launch_main<64, true>(a, stream) : launch_main<64, false>(a, stream))
            : (a.D == 128) ? launch_main<128, false>(a, stream)
                           : cudaErrorInvalidValue;
        if (e != cudaSuccess) return e;
    }
    if ((phases & kBwdPhaseFinal) && rows > 0) {
        const long long n4 = rows * a.D / 4;
        const int tpb = 256;
        const long long per_block = (long long)tpb * kFinalVecs;
        bwd_dq_final_kernel<<<(unsigned)((n4 + per_block - 1) / per_block), tpb, 0, stream>>>(a.dq_acc, a.dq, n4,
                                                                                              a.scale);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace mea
