// fwd_persist.cu -- bf16 forward with persistent CTAs for short key ranges.
//
// Method: the recurrence of fwd_bf16.cu, from "Self-attention Does Not Need
// O(n^2) Memory" (English summary, method bullets 1-4) with the two-block
// formulas of "当注意力成为瓶颈" (section IO感知): per key block j,
// m' = max(m, rowmax S_j), l' = l e^(m-m') + sum e^(S_j-m'), O' = O e^(m-m') + e^(S_j-m') V_j,
// normalised once at the end.
//
// Why: with a few key tiles per (head, query-tile pair) the one-CTA-per-item
// forward spends much of each CTA on its fixed cost (barriers, TMEM, the Q
// load) and on filling and draining its pipeline.  Here a grid of at most one
// CTA per SM walks a fixed list of items (CTA c takes items c, c + G, c + 2G,
// ...), keeping its barriers, TMEM and K/V ring: the next item's Q is loaded
// as soon as the current item's last S has been issued, and its first S and
// the producer's K/V loads overlap the current item's epilogue.
//
// Items.  A pair item is one (head, query-tile pair): slot t holds query tile
// t and every key tile.  When the pair items do not fill the last round of
// the grid (n pairs over G CTAs leave r = n mod G of them for a last round in
// which most CTAs would idle), the last r pairs are listed instead as 2r
// single items of one query tile each, provided 2r <= G: the two slots of a
// single item run the recurrence for the same rows over alternate key tiles
// (slot t takes tiles t, t+2, ...); at the end they swap their row summaries
// through shared memory, fold them with the two-block formulas and each writes
// half of the head dims from both slots' O, so the last round takes about half
// the time of a pair round.
//
// Roles (320 threads) as in fwd_bf16.cu's two-tile path:
//   warp 0       TMEM allocator, then TMA producer (Q tiles per item; K_0, V_0,
//                K_1, V_1, ... of each item through the ring; no multicast)
//   warp 1       MMA issuer (one thread)
//   warps 2-5    softmax / epilogue of slot 0, warps 6-9 of slot 1
// Phases of the per-key-tile barriers run on across items (the parity is that
// of the slot's running key-tile count).  Per item, q_empty (Q may be
// replaced), o_final (O complete) and o_free[t] (slot t's O has been read by
// the epilogue, so the next item's first P V may overwrite it) complete once;
// merge_ready (both slots' row summaries are in shared memory) once per single
// item.
// TMEM: S_0 [0,128) S_1 [128,256) O_0 [256,256+D) O_1 [384,384+D).
//
// Used for bf16 Q/K/V when Nq is a multiple of 256, the keys are not split,
// and the key range is short.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mea {
namespace {

constexpr int kTileP = 128;
constexpr int kThreadsP = 320;
constexpr float kLog2eP = 1.4426950408889634f;
constexpr float kLn2P = 0.6931471805599453f;
constexpr float kRescaleThresholdP = 8.0f;
// Bit 13 of a kind::f16 instruction descriptor: operand A negated.
constexpr unsigned kIdescNegateAP = 1u << 13;

template <int D>
struct PersistCfg {
    static constexpr int kQBytes = kTileP * D * 2;
    static constexpr int kTileBytes = kTileP * D * 2;    // K or V tile
    static constexpr int kStages = D == 128 ? 4 : 6;
    static constexpr int kBoxBytes = 128 * 128;
    static constexpr int kSmemData = 2 * kQBytes + kStages * kTileBytes;
    static constexpr int kSmemBytes = kSmemData + 1024 /*barriers*/ + 1024 /*alignment slack*/;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct PersistBarriers {
    uint64_t q_full, q_empty;
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t s_full[2];
    uint64_t p_half[2];
    uint64_t p_ready[2];
    uint64_t o_final;
    uint64_t o_free[2];
    uint64_t merge_ready;
    uint64_t drain;
    unsigned tmem_base;
    int abort_flag;
};

// Item `item` of the list: the first n_pair_items are (head, query-tile pair)
// items in head-major order; the rest are the query tiles of the remaining
// pairs, one per item, in the same order.
struct PersistItem {
    int bh;
    int q0;       // first query row
    bool single;  // one query tile (both slots on its rows)
};

__device__ __forceinline__ PersistItem persist_item(int item, int pairs, int n_pair_items) {
    PersistItem it;
    it.single = item >= n_pair_items;
    const int p = it.single ? n_pair_items + ((item - n_pair_items) >> 1) : item;   // pair index
    it.bh = p / pairs;
    it.q0 = (p - it.bh * pairs) * (2 * kTileP) + (it.single ? ((item - n_pair_items) & 1) * kTileP : 0);
    return it;
}

// SINGLES: the item list may hold single query tiles (a launch whose list has
// none uses the instantiation without their code paths).
template <int D, bool SINGLES>
__global__ void __launch_bounds__(kThreadsP, 1)
fwd_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ o, float* __restrict__ lse,
                   int Nq, int Nk, float scale, int n_pair_items, int n_items) {
    using Cfg = PersistCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sQ = smem;
    uint8_t* sRing = smem + 2 * Cfg::kQBytes;
    // Both slots' (m_ref, l) per row of a single item go to the second Q tile's
    // buffer: single items come after every pair item of the list and load only
    // the first Q tile, so once a CTA reaches its first single item nothing
    // writes or reads that buffer any more.
    float* sMerge = reinterpret_cast<float*>(smem + Cfg::kQBytes);
    PersistBarriers* bars = reinterpret_cast<PersistBarriers*>(smem + Cfg::kSmemData);

    const unsigned warp = warp_id();
    const unsigned lane = lane_id();
    const int pairs = Nq / (2 * kTileP);             // query-tile pairs per head
    const int n_kv = (Nk + kTileP - 1) / kTileP;
    // this CTA's items: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int first = (int)blockIdx.x;
    const int stride = (int)gridDim.x;
    const int my_items = first < n_items ? (n_items - first + stride - 1) / stride : 0;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_half[t], 128);
            mbar_init(&bars->p_ready[t], 128);
            mbar_init(&bars->o_free[t], 128);
        }
        mbar_init(&bars->o_final, 1);
        mbar_init(&bars->merge_ready, 256);
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
            int c_glob = 0;       // ring tiles issued so far (all items)
            int q_issued = 0;     // items whose Q has been requested
            bool ok = true;
            for (int li = 0; ok && li < my_items; ++li) {
                const PersistItem itm = persist_item(first + li * stride, pairs, n_pair_items);
                const int n_qt = itm.single ? 1 : 2;
                if (li > 0 && !(ok = mbar_wait(&bars->q_empty, (li - 1) & 1, abort_flag))) break;
                mbar_arrive_expect_tx(&bars->q_full, n_qt * Cfg::kQBytes);
                for (int t = 0; t < n_qt; ++t)
                    for (int b = 0; b < D / 64; ++b)
                        tma_load_3d(sQ + t * Cfg::kQBytes + b * Cfg::kBoxBytes, &tm_q, &bars->q_full, b * 64,
                                    itm.q0 + t * kTileP, itm.bh);
                q_issued = li + 1;
                for (int c = 0; c < 2 * n_kv; ++c, ++c_glob) {
                    const int s = c_glob % Cfg::kStages;
                    if (c_glob >= Cfg::kStages &&
                        !(ok = mbar_wait(&bars->empty[s], ((c_glob / Cfg::kStages) - 1) & 1, abort_flag)))
                        break;
                    const CUtensorMap* tm = (c & 1) ? &tm_v : &tm_k;
                    mbar_arrive_expect_tx(&bars->full[s], Cfg::kTileBytes);
                    for (int b = 0; b < D / 64; ++b)
                        tma_load_3d(sRing + s * Cfg::kTileBytes + b * Cfg::kBoxBytes, tm, &bars->full[s], b * 64,
                                    (c >> 1) * kTileP, itm.bh);
                }
            }
            // never leave with copies in flight
            for (int c = (c_glob > Cfg::kStages ? c_glob - Cfg::kStages : 0); c < c_glob; ++c)
                mbar_wait(&bars->full[c % Cfg::kStages], (c / Cfg::kStages) & 1, nullptr);
            if (q_issued > 0) mbar_wait(&bars->q_full, (q_issued - 1) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            // scale < 0: S is formed as (-Q) K^T and the softmax uses |scale|
            const unsigned idesc_s = make_idesc_bf16(128, kTileP, 0, 0) | (scale < 0.f ? kIdescNegateAP : 0u);
            constexpr unsigned idesc_o = make_idesc_bf16(128, D, 0, 1);
            const uint32_t q_lo0 = desc_lo_kmajor(smem_u32(sQ));
            const uint32_t q_lo1 = desc_lo_kmajor(smem_u32(sQ + Cfg::kQBytes));
            const uint32_t ring_k_lo = desc_lo_kmajor(smem_u32(sRing));
            const uint32_t ring_v_lo = desc_lo_mnmajor(smem_u32(sRing));
            constexpr uint32_t kStageStep = Cfg::kTileBytes >> 4;
            const unsigned tS0 = tmem, tS1 = tmem + 128u, tO0 = tmem + 256u, tO1 = tmem + 384u;
            int stage = 0;
            unsigned phase = 0;
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
            auto pv_halves = [&](int t, unsigned parity, uint32_t v_off, unsigned acc0) -> bool {
                const unsigned tO = t ? tO1 : tO0, tS = t ? tS1 : tS0;
                if (!mbar_wait(&bars->p_half[t], parity, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileP / 32; ++kk)
                    mma_ts_lo(tO, tS + kk * 8, ring_v_lo + v_off + mnmajor_step(kk), idesc_o, (acc0 | kk) ? 1u : 0u);
                if (!mbar_wait(&bars->p_ready[t], parity, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = kTileP / 32; kk < kTileP / 16; ++kk)
                    mma_ts_lo(tO, tS + kk * 8, ring_v_lo + v_off + mnmajor_step(kk), idesc_o, 1u);
                return true;
            };
            bool ok = true;
            // key tiles completed by each slot (all items): phase of s_full / p_half / p_ready
            // (scalars, not an array indexed by the slot, so that they stay in registers)
            int cnt0 = 0, cnt1 = 0;
            for (int li = 0; ok && li < my_items; ++li) {
                const bool single = SINGLES && first + li * stride >= n_pair_items;
                // after a single item both slots read both O: the first P V of
                // either slot waits for both epilogues
                const bool prev_single = SINGLES && li > 0 && first + (li - 1) * stride >= n_pair_items;
                if (!(ok = mbar_wait(&bars->q_full, li & 1, abort_flag))) break;
                uint32_t k_off = 0;
                int k_stage = 0;
                if (single) {
                    // both slots on query tile 0 over alternate key tiles; the ring
                    // is still taken in the producer's order K_0, V_0, K_1, V_1, ...
                    // and a slot's V tile is held until its P is ready
                    uint32_t v_off0 = 0, v_off1 = 0;
                    int v_stage0 = 0, v_stage1 = 0;
                    for (int t = 0; ok && t < 2 && t < n_kv; ++t) {
                        if (!(ok = next_tile(k_off, k_stage))) break;
                        tc_fence_after();
                        issue_s(t ? tS1 : tS0, q_lo0, k_off);
                        mma_commit(&bars->s_full[t]);
                        mma_commit(&bars->empty[k_stage]);
                        if (t + 1 == n_kv) mma_commit(&bars->q_empty);   // Q read by its last S
                        ok = t ? next_tile(v_off1, v_stage1) : next_tile(v_off0, v_stage0);
                    }
                    for (int j = 0; ok && j < n_kv; ++j) {
                        const int t = j & 1;
                        // the first P V of a slot overwrites its O: the epilogue of
                        // the previous item must have read it
                        if (j < 2 && li > 0 && !(ok = mbar_wait(&bars->o_free[t], (li - 1) & 1, abort_flag))) break;
                        if (j == 0 && prev_single && !(ok = mbar_wait(&bars->o_free[1], (li - 1) & 1, abort_flag))) break;
                        if (!(ok = pv_halves(t, (t ? cnt1 : cnt0) & 1, t ? v_off1 : v_off0, j >= 2 ? 1u : 0u))) break;
                        if (t) ++cnt1; else ++cnt0;
                        mma_commit(&bars->empty[t ? v_stage1 : v_stage0]);
                        if (j + 2 < n_kv) {
                            if (!(ok = next_tile(k_off, k_stage))) break;
                            tc_fence_after();
                            issue_s(t ? tS1 : tS0, q_lo0, k_off);
                            mma_commit(&bars->s_full[t]);
                            mma_commit(&bars->empty[k_stage]);
                            if (j + 3 == n_kv) mma_commit(&bars->q_empty);
                            ok = t ? next_tile(v_off1, v_stage1) : next_tile(v_off0, v_stage0);
                        }
                    }
                } else {
                    if (!(ok = next_tile(k_off, k_stage))) break;
                    tc_fence_after();
                    issue_s(tS0, q_lo0, k_off);
                    mma_commit(&bars->s_full[0]);
                    issue_s(tS1, q_lo1, k_off);
                    mma_commit(&bars->s_full[1]);
                    mma_commit(&bars->empty[k_stage]);
                    if (n_kv == 1) mma_commit(&bars->q_empty);      // Q read by its last S
                    for (int j = 0; ok && j < n_kv; ++j) {
                        const bool more = (j + 1 < n_kv);
                        const unsigned acc0 = j > 0 ? 1u : 0u;
                        uint32_t v_off = 0;
                        int v_stage = 0;
                        if (!(ok = next_tile(v_off, v_stage))) break;
                        // the first P V of an item overwrites O: the epilogue of the
                        // previous item must have read it
                        if (j == 0 && li > 0 && !(ok = mbar_wait(&bars->o_free[0], (li - 1) & 1, abort_flag))) break;
                        if (j == 0 && prev_single && !(ok = mbar_wait(&bars->o_free[1], (li - 1) & 1, abort_flag))) break;
                        if (!(ok = pv_halves(0, cnt0 & 1, v_off, acc0))) break;
                        ++cnt0;
                        if (more) {
                            if (!(ok = next_tile(k_off, k_stage))) break;
                            tc_fence_after();
                            issue_s(tS0, q_lo0, k_off);
                            mma_commit(&bars->s_full[0]);
                        }
                        if (j == 0 && li > 0 && !(ok = mbar_wait(&bars->o_free[1], (li - 1) & 1, abort_flag))) break;
                        if (!(ok = pv_halves(1, cnt1 & 1, v_off, acc0))) break;
                        ++cnt1;
                        mma_commit(&bars->empty[v_stage]);
                        if (more) {
                            issue_s(tS1, q_lo1, k_off);
                            mma_commit(&bars->s_full[1]);
                            mma_commit(&bars->empty[k_stage]);
                            if (j + 2 == n_kv) mma_commit(&bars->q_empty);   // Q read by its last S
                        }
                    }
                }
                if (ok) mma_commit(&bars->o_final);
            }
            mma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, nullptr);
        }
    } else {
        // ------------------------------------------------ softmax / epilogue
        const int t = (warp - 2) >> 2;
        const unsigned sub = warp & 3;
        const int r = (int)sub * 32 + (int)lane;
        const unsigned lane_off = (sub * 32u) << 16;
        const unsigned tS = tmem + lane_off + (t ? 128u : 0u);
        const unsigned tO = tmem + lane_off + (t ? 384u : 256u);
        const float c_log2 = fabsf(scale) * kLog2eP;   // S carries the sign (A negated)
        bool ok = true;
        int kt = 0;         // key tiles completed by this slot (all items)
        int n_single = 0;   // single items completed by this CTA
        for (int li = 0; ok && li < my_items; ++li) {
            const int item = first + li * stride;
            const bool single = SINGLES && item >= n_pair_items;
            // a pair item's slot t owns query tile t and every key tile; a single
            // item's slots own its one tile and key tiles t, t+2, ...
            const int n_mine = single ? (n_kv + 1 - t) / 2 : n_kv;
            float m_ref = -INFINITY;
            float l = 0.f;
            for (int it = 0; it < n_mine; ++it, ++kt) {
                const int nvalid = Nk - (single ? 2 * it + t : it) * kTileP;   // keys from this tile on
                if (!(ok = mbar_wait(&bars->s_full[t], kt & 1, abort_flag))) break;
                tc_fence_after();
                uint32_t sr[kTileP];
#pragma unroll
                for (int c0 = 0; c0 < kTileP; c0 += 32) tmem_ld32(tS + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[c0]));
                tmem_wait_ld();
                if (nvalid < kTileP) {
#pragma unroll
                    for (int c = 0; c < kTileP; ++c)
                        if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
                }
                float mxa[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mxa[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]));
#pragma unroll
                for (int c = 16; c < kTileP; c += 16)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        mxa[i] = fmax3(mxa[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 8 + i]));
                const float mx = fmaxf(fmax3(mxa[0], mxa[1], mxa[2]), fmax3(fmax3(mxa[3], mxa[4], mxa[5]), mxa[6], mxa[7]));
                const float m_blk = mx * c_log2;
                float alpha = 1.f;
                bool rescale = false;
                if (it == 0) {
                    m_ref = m_blk;
                } else if (__any_sync(0xffffffffu, m_blk - m_ref > kRescaleThresholdP)) {
                    const float m_new = fmaxf(m_ref, m_blk);
                    alpha = ex2_approx(m_ref - m_new);
                    m_ref = m_new;
                    rescale = true;
                }
                l *= alpha;
                float rsa[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) rsa[i] = 0.f;
#pragma unroll
                for (int c0 = 0; c0 < kTileP; c0 += 32) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c0 + c]), c_log2, -m_ref));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c0 + c + 1]), c_log2, -m_ref));
                        rsa[(c / 2) & 7] += p0 + p1;
                        pk[c / 2] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tS + c0 / 2, pk);
                    if (c0 == kTileP / 2 - 32 && !rescale) {
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&bars->p_half[t]);
                    }
                }
                l += ((rsa[0] + rsa[1]) + (rsa[2] + rsa[3])) + ((rsa[4] + rsa[5]) + (rsa[6] + rsa[7]));
                if (rescale) {
                    // P V of this slot's previous key tile has completed (it was
                    // issued before S of this one, whose commit was waited on)
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
            if (!ok) break;
            // A single item's slots fold their summaries of the same rows
            // together with the two-block formulas and each writes half of the
            // head dims, reading both slots' O (slot 1 is empty when the item
            // has one key tile; its summary is then m = -inf, l = 0).
            const bool with1 = single && n_kv >= 2;
            // (the item's rows are found while the last P V is still running)
            const PersistItem itm = persist_item(item, pairs, n_pair_items);
            const int row = itm.q0 + (single ? 0 : t * kTileP) + r;
            float w0 = 1.f, w1 = 0.f, M = m_ref, L = l;
            if (single) {
                // the other slot has read the previous single item's summaries:
                // its o_free of the previous item completed after its epilogue
                if (li > 0 && !(ok = mbar_wait(&bars->o_free[t ^ 1], (li - 1) & 1, abort_flag))) break;
                sMerge[2 * (t * kTileP + r)] = m_ref;
                sMerge[2 * (t * kTileP + r) + 1] = l;
                mbar_arrive(&bars->merge_ready);
                if (!(ok = mbar_wait(&bars->merge_ready, n_single & 1, abort_flag))) break;
                ++n_single;
                const float m_o = sMerge[2 * ((t ^ 1) * kTileP + r)];
                const float l_o = sMerge[2 * ((t ^ 1) * kTileP + r) + 1];
                M = fmaxf(m_ref, m_o);
                const float w_self = ex2_approx(m_ref - M), w_oth = ex2_approx(m_o - M);
                L = w_self * l + w_oth * l_o;
                w0 = t ? w_oth : w_self;
                w1 = t ? w_self : w_oth;
            }
            if (!(ok = mbar_wait(&bars->o_final, li & 1, abort_flag))) break;
            tc_fence_after();
            const float inv_l = 1.f / L;
            const float s0 = w0 * inv_l, s1 = w1 * inv_l;
            // pair item: slot t writes every head dim of its own O; single item:
            // slot t writes dims [t D/2, (t+1) D/2) of O_0 s0 + O_1 s1
            const int c_begin = single ? t * (D / 2) : 0;
            const int n_chunks = single ? D / 32 : D / 16;
            const unsigned tOa = single ? tmem + lane_off + 256u : tO;
            const unsigned tOb = tmem + lane_off + 384u;
            uint16_t* orow = o + ((size_t)itm.bh * Nq + row) * D;
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                if (k >= n_chunks) break;
                const int c0 = c_begin + 16 * k;
                uint32_t a[16];
                float f[16];
                tmem_ld16(tOa + c0, a);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(a[i]) * s0;
                if (with1) {
                    tmem_ld16(tOb + c0, a);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) f[i] = fmaf(__uint_as_float(a[i]), s1, f[i]);
                }
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) packed[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
                uint4* dst = reinterpret_cast<uint4*>(orow + c0);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
            if (!single || t == 0) lse[(size_t)itm.bh * Nq + row] = (M + __log2f(L)) * kLn2P;
            // this slot's reads of O are done (a single item's O_0 and O_1 are
            // both read by both slots: the next item's first P V waits for both)
            tc_fence_before();
            mbar_arrive(&bars->o_free[t]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool SINGLES>
cudaError_t launch_persist_list(const Bf16FwdArgs& a, const PersistSchedule& sch, cudaStream_t stream) {
    using Cfg = PersistCfg<D>;
    auto kern = fwd_persist_kernel<D, SINGLES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)sch.grid, kThreadsP, Cfg::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.o, a.lse, a.Nq, a.Nk,
                                                                       a.scale, (int)sch.n_pair_items,
                                                                       (int)sch.n_items);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_persist(const Bf16FwdArgs& a, int sm_count, cudaStream_t stream) {
    const PersistSchedule sch = fwd_persist_schedule((long long)a.BH * (a.Nq / (2 * kTileP)), sm_count);
    if (sch.grid <= 0) return cudaSuccess;
    return sch.n_items > sch.n_pair_items ? launch_persist_list<D, true>(a, sch, stream)
                                          : launch_persist_list<D, false>(a, sch, stream);
}

}  // namespace

PersistSchedule fwd_persist_schedule(long long n_pairs, int sm_count) {
    PersistSchedule s;
    s.n_pair_items = n_pairs;
    s.n_items = n_pairs;
    s.grid = n_pairs < sm_count ? n_pairs : sm_count;
    if (n_pairs <= 0 || sm_count <= 0) return s;
    const long long rounds = n_pairs / sm_count;
    const long long rest = n_pairs - rounds * sm_count;   // pairs of a partial last round
    if (rest > 0 && 2 * rest <= sm_count) {
        s.n_pair_items = n_pairs - rest;
        s.n_items = n_pairs + rest;
        s.grid = rounds > 0 ? sm_count : 2 * rest;
    }
    return s;
}

bool fwd_persist_applies(int D, bool fp8_qk, int BH, int Nq, int Nk, int chunks, int sm_count) {
    if (!((D == 64 || D == 128) && !fp8_qk && chunks <= 1 && Nq >= 2 * kTileP && Nq % (2 * kTileP) == 0 && Nk >= 1))
        return false;
    const int max_keys = D == 64 ? kFwdPersistMaxKeys64 : kFwdPersistMaxKeys128;
    if (Nk <= max_keys) return true;
    // longer key ranges amortise a CTA's fixed cost by themselves, but where
    // the pairs leave a partial last round that single tiles can halve, the
    // item list still gains up to twice the key limit
    if (Nk > 2 * max_keys) return false;
    const PersistSchedule s = fwd_persist_schedule((long long)BH * (Nq / (2 * kTileP)), sm_count);
    return s.n_items > s.n_pair_items;
}

cudaError_t launch_fwd_persist(const Bf16FwdArgs& a, int sm_count, cudaStream_t stream) {
    if (!fwd_persist_applies(a.D, a.fp8_qk, a.BH, a.Nq, a.Nk, a.chunks, sm_count)) return cudaErrorInvalidValue;
    if ((long long)a.BH * (a.Nq / (2 * kTileP)) * 2 > 0x7fffffffLL) return cudaErrorInvalidValue;
    return a.D == 64 ? launch_persist<64>(a, sm_count, stream) : launch_persist<128>(a, sm_count, stream);
}

}  // namespace mea
