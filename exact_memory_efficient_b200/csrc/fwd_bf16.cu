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
//               O_t += P_t V_j with P_t read from TMEM, in two halves of
//               64 keys (the first as soon as the softmax has stored it)
//   warps 2-5   softmax of TMEM slot 0, warps 6-9 of slot 1 (warp w reaches
//               TMEM lanes 32*(w%4) .. 32*(w%4)+31): one thread per query row
//               (TMEM lane), tcgen05.ld of S, exp2 with scale*log2(e) folded
//               in, P written back to TMEM as bf16 over the S columns, O
//               rescaled in TMEM when the reference maximum moves.
// TMEM (512 columns): S_0 [0,128)  S_1 [128,256)  O_0 [256,256+D)  O_1 [384,384+D).
// With two live query tiles slot t holds query tile t.  A CTA whose rows all
// fit in its first tile (decode, or the last pair of a ragged Nq) runs both
// slots on that tile over alternate key tiles and merges the two summaries at
// the end, so one slot's softmax still overlaps the other's MMAs.
//
// Instantiations: F8 takes e4m3 Q and K (S on kind::f8f6f4; V, P, O bf16);
// DEEP (launches with Nq <= 128 at D = 128) keeps one Q buffer and gives the
// rest of shared memory to a six-stage K/V ring.
//
// Key split (decode-shaped calls): when a grid would leave most SMs idle (few
// query tiles x heads), the keys of each (batch, head, query tile) are split
// over the CTAs of a thread-block cluster.  Each CTA runs the recurrence over
// its chunk and leaves the chunk summary of every row -- its reference maximum,
// exp-sum and unnormalised accumulator -- in its shared memory; the CTAs then
// merge the summaries through distributed shared memory with the two-block
// formulas, each writing a slice of the head dims of O (and the first, lse).
// No global scratch is used.
//
// Reference maximum: a row's exponentials are taken relative to a reference
// value m_ref that is raised to the true running maximum only when the new
// block maximum exceeds it by more than 8 (base-2 units).  Then every
// exponential is <= 2^8, nothing overflows, and because O, l and the final
// lse all use the same m_ref the result is the same exact softmax; it only
// saves O rescales.
#include <cooperative_groups.h>
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
// Bit 13 of a kind::f16 / kind::f8f6f4 instruction descriptor: operand A negated.
constexpr unsigned kIdescNegateA = 1u << 13;

// F8: Q and K are e4m3 (one byte per element) and S = Q K^T runs as
// kind::f8f6f4; V, P and O stay bf16.  DEEP: for launches whose CTAs all hold
// a single query tile (decode): one Q buffer, and the space of the second one
// plus the rest of shared memory goes to the K/V ring (such launches stream
// K/V with little compute per byte and gain from the deeper prefetch).
template <int D, bool F8 = false, bool DEEP = false>
struct FwdCfg {
    static constexpr int kQKElem = F8 ? 1 : 2;                // bytes per Q/K element
    static constexpr int kQKBox = 128 / kQKElem;              // Q/K elements per 128-byte box row
    static constexpr int kKBytes = kTileN * D * kQKElem;      // one K tile
    static constexpr int kVBytes = kTileN * D * 2;            // one V tile
    static constexpr int kTileBytes = kVBytes;                // one ring stage (a K tile uses its start)
    static constexpr int kQBytes = kTileM * D * kQKElem;      // one Q tile
    static constexpr int kQTiles = DEEP ? 1 : 2;                // Q buffers
    static constexpr int kStages = DEEP ? 6 : (F8 ? ((D == 128) ? 5 : 7) : ((D == 128) ? 4 : 6));
    static constexpr int kBoxBytes = 128 * 128;               // one 128-byte-wide box of 128 rows
    static constexpr int kSmemData = kQTiles * kQBytes + kStages * kTileBytes;
    static constexpr int kSmemBytes = kSmemData + 1024 /*barriers*/ + 1024 /*alignment slack*/;
};

struct FwdBarriers {
    uint64_t q_full;
    uint64_t full[8];    // ring stages (at most 8)
    uint64_t empty[8];
    uint64_t s_full[2];
    uint64_t p_half[2];   // P columns 0..63 of tile t are in TMEM
    uint64_t p_ready[2];
    uint64_t o_final;
    uint64_t merge_ready;
    uint64_t drain;
    unsigned tmem_base;
    int abort_flag;
};

// Chunk summaries for the cluster merge live where Q and the K/V ring were
// (free once the last MMA has completed): rows of D floats padded to D + 4 so
// that one row per lane is written without shared-memory bank conflicts.
template <int D>
__device__ __forceinline__ float* part_row(uint8_t* smem, int t, int r) {
    return reinterpret_cast<float*>(smem) + ((size_t)t * kTileM + r) * (D + 4);
}
template <int D>
__device__ __forceinline__ float* part_ml(uint8_t* smem, int t, int r) {
    return reinterpret_cast<float*>(smem) + (size_t)2 * kTileM * (D + 4) + ((size_t)t * kTileM + r) * 2;
}
static_assert(2 * 128 * (128 + 4) * 4 + 2 * 128 * 2 * 4 <= FwdCfg<128>::kSmemData, "merge area (D=128)");
static_assert(2 * 128 * (128 + 4) * 4 + 2 * 128 * 2 * 4 <= FwdCfg<128, true>::kSmemData, "merge area (D=128, fp8)");
static_assert(FwdCfg<128, true, true>::kStages <= 8 && FwdCfg<64, false, true>::kStages <= 8, "ring barriers");
static_assert(FwdCfg<128, true, true>::kSmemBytes <= 227 * 1024 && FwdCfg<128, false, true>::kSmemBytes <= 227 * 1024,
              "shared memory");
static_assert(2 * 128 * (64 + 4) * 4 + 2 * 128 * 2 * 4 <= FwdCfg<64>::kSmemData, "merge area (D=64)");

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int D, bool F8, bool DEEP>
__global__ void __launch_bounds__(kThreads, 1)
fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ o,
                float* __restrict__ lse, int Nq, int Nk, float scale, int chunk_len) {
    using Cfg = FwdCfg<D, F8, DEEP>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the shared-memory address (not of the generic
    // pointer: in a cluster launch each CTA's shared window can sit at a
    // different generic offset) for the 128-byte-swizzle atoms
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sQ = smem;                               // Q_0 then Q_1
    uint8_t* sRing = smem + Cfg::kQTiles * Cfg::kQBytes;   // kStages tiles
    FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(smem + Cfg::kSmemData);

    const unsigned warp = warp_id();
    const unsigned lane = lane_id();
    const int bh = blockIdx.y;
    // key split over the CTAs of a cluster (one CTA per cluster when not split)
    unsigned nranks, rank;
    asm("mov.u32 %0, %%cluster_nctarank;" : "=r"(nranks));
    asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    const int m0 = (blockIdx.x / nranks) * (2 * kTileM);
    // A CTA whose rows all fall in its first query tile (decode-shaped calls,
    // the last tile pair of a ragged Nq) issues no work for the second tile.
    const bool two = !DEEP && (m0 + kTileM) < Nq;   // DEEP launches have Nq <= 128
    const int c_begin = (nranks > 1) ? (int)rank * chunk_len : 0;
    const int c_end = (nranks > 1) ? min(Nk, c_begin + chunk_len) : Nk;
    const int n_kv = (c_end > c_begin) ? (c_end - c_begin + kTileN - 1) / kTileN : 0;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_half[t], 128);
            mbar_init(&bars->p_ready[t], 128);
        }
        mbar_init(&bars->o_final, 1);
        mbar_init(&bars->merge_ready, 128);
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
            const int n_qt = two ? 2 : 1;
            mbar_arrive_expect_tx(&bars->q_full, n_qt * Cfg::kQBytes);
            for (int t = 0; t < n_qt; ++t)
                for (int b = 0; b < D / Cfg::kQKBox; ++b)
                    tma_load_3d(sQ + t * Cfg::kQBytes + b * Cfg::kBoxBytes, &tm_q, &bars->q_full,
                                b * Cfg::kQKBox, m0 + t * kTileM, bh);
            const int n_tiles = 2 * n_kv;
            int issued = 0;
            for (int c = 0; c < n_tiles; ++c) {
                const int s = c % Cfg::kStages;
                if (c >= Cfg::kStages) {
                    if (!mbar_wait(&bars->empty[s], ((c / Cfg::kStages) - 1) & 1, abort_flag)) break;
                }
                uint8_t* dst = sRing + s * Cfg::kTileBytes;
                const bool is_v = c & 1;
                const CUtensorMap* tm = is_v ? &tm_v : &tm_k;
                const int key0 = c_begin + (c >> 1) * kTileN;
                const int bw = is_v ? 64 : Cfg::kQKBox;               // elements per box row
                mbar_arrive_expect_tx(&bars->full[s], is_v ? Cfg::kVBytes : Cfg::kKBytes);
                for (int b = 0; b < D / bw; ++b)
                    tma_load_3d(dst + b * Cfg::kBoxBytes, tm, &bars->full[s], b * bw, key0, bh);
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
            // scale < 0: S is formed as (-Q) K^T (the instruction's A-negate bit)
            // and the softmax uses |scale|, so its running maximum is that of the
            // scaled scores with either sign
            const unsigned s_neg = scale < 0.f ? kIdescNegateA : 0u;
            const unsigned idesc_s = make_idesc_bf16(128, kTileN, 0, 0) | s_neg;
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
                if constexpr (F8) {
                    // K = 32 e4m3 elements per instruction: the same 32-byte step
                    const unsigned idesc_s8 = make_idesc_e4m3(128, kTileN) | s_neg;
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk)
                        mma_ss_lo_f8(tS, q_lo + kmajor_step(kk), ring_k_lo + k_off + kmajor_step(kk), idesc_s8,
                                     kk > 0);
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss_lo(tS, q_lo + kmajor_step(kk), ring_k_lo + k_off + kmajor_step(kk), idesc_s, kk > 0);
                }
            };
            // In a cluster launch (key split) P V is issued per 64-column block of V,
            // each block addressed by its start address: on this part, an MMA on
            // a CTA of cluster rank 1 read the second 64-element block of an
            // MN-major B operand wrongly when reaching it through the
            // descriptor's leading-byte offset (rank 0 and non-cluster launches
            // were correct).  The single N = D instruction is kept otherwise.
            const bool pv_by_block = (D > 64) && (nranks > 1);
            // P V over the keys [16 kk0, 16 kk1) of the tile (K steps kk0..kk1-1)
            auto issue_pv = [&](unsigned tO, unsigned tS, uint32_t v_off, unsigned acc0, int kk0, int kk1) {
                if (pv_by_block) {
                    constexpr unsigned idesc_o64 = make_idesc_bf16(128, 64, 0, 1);
#pragma unroll
                    for (int blk = 0; blk < D / 64; ++blk)
#pragma unroll
                        for (int kk = kk0; kk < kk1; ++kk)
                            mma_ts_lo(tO + 64 * blk, tS + kk * 8,
                                      ring_v_lo + v_off + blk * (Cfg::kBoxBytes >> 4) + mnmajor_step(kk), idesc_o64,
                                      (acc0 | kk) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int kk = kk0; kk < kk1; ++kk)
                        mma_ts_lo(tO, tS + kk * 8, ring_v_lo + v_off + mnmajor_step(kk), idesc_o, (acc0 | kk) ? 1u : 0u);
                }
            };
            // P V in two halves: the first four K steps as soon as the softmax has
            // stored P's first 64 columns, the rest once the whole P is in TMEM
            auto pv_halves = [&](int t, unsigned parity, uint32_t v_off, unsigned acc0) -> bool {
                const unsigned tO = t ? tO1 : tO0, tS = t ? tS1 : tS0;
                if (!mbar_wait(&bars->p_half[t], parity, abort_flag)) return false;
                tc_fence_after();
                issue_pv(tO, tS, v_off, acc0, 0, kTileN / 32);
                if (!mbar_wait(&bars->p_ready[t], parity, abort_flag)) return false;
                tc_fence_after();
                issue_pv(tO, tS, v_off, acc0, kTileN / 32, kTileN / 16);
                return true;
            };
            uint32_t k_off = 0;
            int k_stage = 0;
            if (!two) {
                // One live query tile: the two TMEM slots run the recurrence for
                // the same rows over alternate key tiles (slot t takes tiles
                // t, t+2, ...), so one slot's softmax overlaps the other's MMAs.
                // Ring tiles are still taken in the producer's order K_0, V_0,
                // K_1, V_1, ...; a slot's V tile is held until its P is ready.
                uint32_t v_off[2] = {0, 0};
                int v_stage[2] = {0, 0};
                for (int t = 0; ok && t < 2 && t < n_kv; ++t) {
                    if (!(ok = next_tile(k_off, k_stage))) break;
                    tc_fence_after();
                    issue_s(t ? tS1 : tS0, q_lo0, k_off);
                    mma_commit(&bars->s_full[t]);
                    mma_commit(&bars->empty[k_stage]);
                    ok = next_tile(v_off[t], v_stage[t]);
                }
                for (int j = 0; ok && j < n_kv; ++j) {
                    const int t = j & 1;
                    const int i = j >> 1;  // iteration of slot t
                    if (!(ok = pv_halves(t, i & 1, v_off[t], i > 0 ? 1u : 0u))) break;
                    mma_commit(&bars->empty[v_stage[t]]);
                    if (j + 2 < n_kv) {
                        if (!(ok = next_tile(k_off, k_stage))) break;
                        tc_fence_after();
                        issue_s(t ? tS1 : tS0, q_lo0, k_off);
                        mma_commit(&bars->s_full[t]);
                        mma_commit(&bars->empty[k_stage]);
                        ok = next_tile(v_off[t], v_stage[t]);
                    }
                }
            }
            if (two && ok && n_kv > 0) ok = next_tile(k_off, k_stage);
            if (two && ok && n_kv > 0) {
                tc_fence_after();
                issue_s(tS0, q_lo0, k_off);
                mma_commit(&bars->s_full[0]);
                issue_s(tS1, q_lo1, k_off);
                mma_commit(&bars->s_full[1]);
                mma_commit(&bars->empty[k_stage]);
            }
            for (int j = 0; two && ok && j < n_kv; ++j) {
                const bool more = (j + 1 < n_kv);
                const unsigned acc0 = j > 0 ? 1u : 0u;
                uint32_t v_off = 0;
                int v_stage = 0;
                if (!(ok = next_tile(v_off, v_stage))) break;
                // tile 0: O_0 += P_0 V_j, then S_0 = Q_0 K_{j+1}^T
                if (!(ok = pv_halves(0, j & 1, v_off, acc0))) break;
                if (more) {
                    if (!(ok = next_tile(k_off, k_stage))) break;
                    tc_fence_after();
                    issue_s(tS0, q_lo0, k_off);
                    mma_commit(&bars->s_full[0]);
                }
                // tile 1: O_1 += P_1 V_j, then S_1 = Q_1 K_{j+1}^T
                if (!(ok = pv_halves(1, j & 1, v_off, acc0))) break;
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
        const int t = (warp - 2) >> 2;                     // TMEM slot of these four warps
        const unsigned sub = warp & 3;                     // TMEM sub-partition (lanes 32*sub..)
        const int r = sub * 32 + lane;                     // row within the query tile
        const unsigned lane_off = (sub * 32u) << 16;
        const unsigned tS = tmem + lane_off + (t ? 128u : 0u);
        const unsigned tO = tmem + lane_off + (t ? 384u : 256u);
        // With two live query tiles slot t owns query tile t and every key
        // tile; with one, both slots own query tile 0 and slot t takes the key
        // tiles t, t+2, ... (merged below).
        const bool split = !two;
        const int n_mine = split ? (n_kv + 1 - t) / 2 : n_kv;
        const int row0 = m0 + (split ? 0 : t * kTileM);
        // Rows at or past Nq are never stored and a row of O depends only on
        // the same row of P, so a warp whose 32 rows all lie past Nq only keeps
        // the handshake (its P lanes hold whatever S left there).
        const bool live = (row0 + (int)sub * 32) < Nq;
        float m_ref = -INFINITY;  // reference maximum, base-2 units of scale*s
        float l = 0.f;
        bool ok = true;
        if (!live) {
            for (int i = 0; i < n_mine; ++i) {
                if (!(ok = mbar_wait(&bars->s_full[t], i & 1, abort_flag))) break;
                mbar_arrive(&bars->p_half[t]);
                mbar_arrive(&bars->p_ready[t]);
            }
        } else {
            const float c_log2 = fabsf(scale) * kLog2e;   // S carries the sign (A negated)
            for (int it = 0; it < n_mine; ++it) {
                const int j = split ? 2 * it + t : it;  // key tile within this CTA's range
                if (!(ok = mbar_wait(&bars->s_full[t], it & 1, abort_flag))) break;
                tc_fence_after();
                uint32_t sr[kTileN];
#pragma unroll
                for (int c0 = 0; c0 < kTileN; c0 += 32)
                    tmem_ld32(tS + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[c0]));
                tmem_wait_ld();
                const int nvalid = c_end - (c_begin + j * kTileN);
                if (nvalid < kTileN) {
#pragma unroll
                    for (int c = 0; c < kTileN; ++c)
                        if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
                }
                // row maximum as 8 independent chains of 3-input maxima (one thread
                // owns the row, so a single 128-long dependent chain would dominate
                // the softmax latency; the softmax warps are issue-bound, so each
                // instruction should retire two new values)
                float mxa[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mxa[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]));
#pragma unroll
                for (int c = 16; c < kTileN; c += 16)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        mxa[i] = fmax3(mxa[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 8 + i]));
                const float mx = fmaxf(fmax3(mxa[0], mxa[1], mxa[2]),
                                       fmax3(fmax3(mxa[3], mxa[4], mxa[5]), mxa[6], mxa[7]));
                const float m_blk = mx * c_log2;
                float m_new = m_ref;
                bool rescale = false;
                float alpha = 1.f;
                if (it == 0) {
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
                    if (c0 == kTileN / 2 - 32 && !rescale) {
                        // P's first 64 columns are in TMEM and O needs no rescale:
                        // their P V steps may start
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&bars->p_half[t]);
                    }
                }
                l += ((rsa[0] + rsa[1]) + (rsa[2] + rsa[3])) + ((rsa[4] + rsa[5]) + (rsa[6] + rsa[7]));
                if (rescale) {
                    // PV_t of the previous key tile has completed (it was issued before
                    // S_t of this one, whose commit we waited on), so O_t can be rescaled
                    // in place; this warp's first-half signal waits for it, and P V
                    // starts only when all four warps have signalled
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
                if (rescale) mbar_arrive(&bars->p_half[t]);
                mbar_arrive(&bars->p_ready[t]);
            }
        }

        if (split && t == 1) {
            // hand this slot's (m_ref, l) to slot 0, whose warps read its O
            // straight from TMEM (same lanes); the merge area is free once the
            // last MMA has completed
            if (live && ok && mbar_wait(&bars->o_final, 0, abort_flag)) {
                float* ml = part_ml<D>(smem, 1, r);
                ml[0] = m_ref;
                ml[1] = l;
            }
            mbar_arrive(&bars->merge_ready);
        } else if (live && ok && mbar_wait(&bars->o_final, 0, abort_flag)) {
            tc_fence_after();
            const int row = row0 + r;
            // split mode: fold slot 1's summary of the same rows in with the
            // two-block formulas (slot 1 is empty when the range has one key tile)
            const bool with1 = split && n_kv >= 2;
            float w0 = 1.f, w1 = 0.f, M = m_ref, L = l;
            if (with1) {
                ok = mbar_wait(&bars->merge_ready, 0, abort_flag);
                const float* ml1 = part_ml<D>(smem, 1, r);
                const float m1 = ml1[0], l1 = ml1[1];
                M = fmaxf(m_ref, m1);
                w0 = ex2_approx(m_ref - M);
                w1 = ex2_approx(m1 - M);
                L = w0 * l + w1 * l1;
            }
            const unsigned tO1 = tmem + lane_off + 384u;
            const bool has = n_kv > 0;
            const float inv_L = 1.f / L;
            uint16_t* orow = o + ((size_t)bh * Nq + row) * D;
            float* prow = part_row<D>(smem, t, r);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t a0[16], a1[16];
                tmem_ld16(tO + c0, a0);
                if (with1) tmem_ld16(tO1 + c0, a1);
                tmem_wait_ld();
                float f[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    f[i] = w0 * __uint_as_float(a0[i]);
                    if (with1) f[i] = fmaf(w1, __uint_as_float(a1[i]), f[i]);
                }
                if (!ok || row >= Nq) continue;
                if (nranks == 1) {
                    uint32_t packed[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) packed[i] = pack_bf16x2(f[2 * i] * inv_L, f[2 * i + 1] * inv_L);
                    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
                    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                } else {
                    // chunk summary of this row for the cluster merge: the
                    // unnormalised accumulator (zero when this CTA's range is empty)
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        *reinterpret_cast<float4*>(prow + c0 + i) =
                            has ? make_float4(f[i], f[i + 1], f[i + 2], f[i + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            if (ok && row < Nq) {
                if (nranks == 1) {
                    lse[(size_t)bh * Nq + row] = (M + __log2f(L)) * kLn2;
                } else {
                    float* ml = part_ml<D>(smem, t, r);
                    ml[0] = has ? M : -INFINITY;
                    ml[1] = has ? L : 0.f;
                }
            }
        }
    }

    if (nranks > 1) {
        // every thread of every CTA of the cluster passes both barriers, also
        // on the abort path, so no CTA leaves while another reads its memory
        __syncwarp();
        cluster_sync_all();
        if (warp >= 2 && !*abort_flag) {
            // The merge is spread over the whole cluster: rank c finishes the
            // 4-column groups g = c, c + nranks, ... of every row, so each
            // thread issues all of its remote loads at once and no CTA does
            // more than its share.
            namespace cg = cooperative_groups;
            cg::cluster_group cluster = cg::this_cluster();
            constexpr int kGroups = D / 4;
            const int gpr = (kGroups - (int)rank + (int)nranks - 1) / (int)nranks;  // groups of this rank
            const int rows = min(2 * kTileM, Nq - m0);
            const int items = rows * gpr;
            for (int item = (int)threadIdx.x - 64; item < items; item += kThreads - 64) {
                const int i = item / gpr;                        // row within this CTA's tile pair
                const int g = (int)rank + (int)nranks * (item - i * gpr);
                const int t = i / kTileM;
                const int r = i - t * kTileM;
                float mc[16], lc[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    mc[c] = -INFINITY;
                    lc[c] = 0.f;
                    if (c < (int)nranks) {
                        const float* ml = cluster.map_shared_rank(part_ml<D>(smem, t, r), (unsigned)c);
                        mc[c] = ml[0];
                        lc[c] = ml[1];
                    }
                }
                float M = mc[0];
#pragma unroll
                for (int c = 1; c < 16; ++c) M = fmaxf(M, mc[c]);
                float L = 0.f;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    if (c < (int)nranks) {
                        const float w = ex2_approx(mc[c] - M);   // 0 for empty chunks (m = -inf)
                        const float* prow = cluster.map_shared_rank(part_row<D>(smem, t, r), (unsigned)c);
                        const float4 v = *reinterpret_cast<const float4*>(prow + 4 * g);
                        L = fmaf(w, lc[c], L);
                        acc.x = fmaf(w, v.x, acc.x);
                        acc.y = fmaf(w, v.y, acc.y);
                        acc.z = fmaf(w, v.z, acc.z);
                        acc.w = fmaf(w, v.w, acc.w);
                    }
                }
                const float inv_L = 1.f / L;
                const int row = m0 + i;
                uint16_t* orow = o + ((size_t)bh * Nq + row) * D;
                *reinterpret_cast<uint2*>(orow + 4 * g) =
                    make_uint2(pack_bf16x2(acc.x * inv_L, acc.y * inv_L), pack_bf16x2(acc.z * inv_L, acc.w * inv_L));
                if (g == 0) lse[(size_t)bh * Nq + row] = (M + __log2f(L)) * kLn2;
            }
        }
        cluster_sync_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool F8, bool DEEP>
cudaError_t launch_d(const Bf16FwdArgs& a, cudaStream_t stream) {
    using Cfg = FwdCfg<D, F8, DEEP>;
    auto kern = fwd_bf16_kernel<D, F8, DEEP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int q_tiles = (a.Nq + 2 * kTileM - 1) / (2 * kTileM);
    if (a.chunks <= 1) {
        dim3 grid(q_tiles, a.BH, 1);
        kern<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.o, a.lse, a.Nq, a.Nk, a.scale, 0);
        return cudaGetLastError();
    }
    if (a.chunks > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(q_tiles * a.chunks, a.BH, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.chunks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a.tm_q, a.tm_k, a.tm_v, a.o, a.lse, a.Nq, a.Nk, a.scale, a.chunk_len);
}

template <int D, bool F8, bool DEEP>
int max_active_clusters_d(int cluster) {
    using Cfg = FwdCfg<D, F8, DEEP>;
    auto kern = fwd_bf16_kernel<D, F8, DEEP>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) != cudaSuccess)
        return 0;
    if (cluster > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    return n;
}

}  // namespace

// The deep-ring variant is used at D = 128 when every CTA holds a single query
// tile (Nq <= 128).
bool use_deep(int D, int Nq) { return D == 128 && Nq <= kTileM; }

int fwd_bf16_max_active_clusters(int D, bool fp8_qk, int Nq, int cluster) {
    if (cluster < 1 || cluster > 16) return 0;
    const bool deep = use_deep(D, Nq);
    if (fp8_qk) {
        if (D != 128) return 0;
        return deep ? max_active_clusters_d<128, true, true>(cluster) : max_active_clusters_d<128, true, false>(cluster);
    }
    if (D == 64) return max_active_clusters_d<64, false, false>(cluster);
    if (D == 128)
        return deep ? max_active_clusters_d<128, false, true>(cluster) : max_active_clusters_d<128, false, false>(cluster);
    return 0;
}

cudaError_t launch_fwd_bf16(const Bf16FwdArgs& a, cudaStream_t stream) {
    const bool deep = use_deep(a.D, a.Nq);
    if (a.fp8_qk) {
        if (a.D != 128) return cudaErrorInvalidValue;
        return deep ? launch_d<128, true, true>(a, stream) : launch_d<128, true, false>(a, stream);
    }
    if (a.D == 64) return launch_d<64, false, false>(a, stream);
    if (a.D == 128) return deep ? launch_d<128, false, true>(a, stream) : launch_d<128, false, false>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace mea
