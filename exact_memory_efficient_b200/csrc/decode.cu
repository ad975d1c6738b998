// decode.cu -- split-KV forward for decode-shaped calls: few query rows per
// key/value head (R = (H / H_kv) * Nq <= 8) against a long key range.
//
// Method: the chunked formulation of "Self-attention Does Not Need O(n^2)
// Memory" (English summary, method bullets 1-4: keys and values in chunks, a
// running maximum, exp-sum and rescaled accumulator per row, one division at
// the end) with the chunk summaries merged by the two-block formulas of
// "当注意力成为瓶颈" (section IO感知).
//
// With R <= 8 rows per key/value head the work is 4*R*D flops per key against
// 2*D elements of K and V read once from HBM, so the launch is bound by HBM,
// not by the tensor cores: it is written for the memory system (bulk copies
// into a ring of shared-memory stages, a grid that covers every SM) and does
// its arithmetic on the CUDA cores in fp32.
//
// Phase 1, decode_partial_kernel, grid (B*H_kv, nsplit): each CTA takes one
// key chunk of one key/value head, for all R query rows of that head.
//   warp 8      producer: cp.async.bulk copies of 64-key K and V tiles
//               (contiguous rows of the [B*H_kv, Nk, D] tensors) into the ring.
//   warps 0-7   warp w takes keys [8w, 8w + 8) of every tile and keeps its own
//               running (m, l, acc) per row.  A key is shared by the whole
//               warp (1 or 8 rows per head) or by a half-warp (2 or 4 rows,
//               two keys at a time); each lane owns a slice of the head dims,
//               forms partial dot products for its keys x up to 4 rows, and a
//               butterfly reduce-scatter over the key's lanes leaves every
//               (key, row) score complete in one set of lanes; the score
//               is already in the base-2 domain (q is pre-multiplied by
//               scale * log2 e).  The maximum is refreshed only when a score
//               exceeds it by more than 2^8 (the rescale is exact whenever it
//               happens; skipping it only lets the weights grow up to 2^8),
//               and the weights reach every lane by shuffles for the P V
//               update of its dims.
//   end         the 8 warp summaries are merged through shared memory (the
//               drained ring); with one chunk per head the CTA writes o and
//               lse, otherwise the chunk summary (m, l, acc) goes to the
//               caller's workspace.
// Phase 2, decode_merge_kernel: merges the nsplit chunk summaries of each row.
// Both kernels are launched with programmatic stream serialisation: a grid may
// be scheduled while the kernel before it in the stream drains, and waits
// (griddepcontrol.wait) for that kernel's results before it touches global
// memory, so results are as with plain stream order while the launch and
// set-up of one kernel overlap the tail of the previous one.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mea {
namespace {

constexpr int kTK = kDecodeTileKeys;             // keys per tile
constexpr int kCompWarps = 8;                    // compute warps
constexpr int kKeysPerWarp = kTK / kCompWarps;   // keys of a tile per compute warp
constexpr int kThreads = 32 * (kCompWarps + 1);  // + producer warp
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;        // log2 of the largest weight left unrescaled

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// Lanes per key: 2 and 4 rows per head put 16 lanes (half a warp) on a key,
// so a warp reduces two keys' products at once over 16 lanes; 1 and 8 rows use
// the whole warp (one row's products are few; eight rows need the registers).
template <int RMAX>
constexpr int kLanesPerKey = (RMAX == 2 || RMAX == 4) ? 16 : 32;

template <typename T, int DPL, int RMAX>
struct DecCfg {
    static constexpr int D = 32 * DPL;
    static constexpr int LPK = kLanesPerKey<RMAX>;
    static constexpr int kGroups = 32 / LPK;              // key groups per warp (1 or 2)
    static constexpr int kKPG = kKeysPerWarp / kGroups;   // keys per group in a tile
    static constexpr int DL = D / LPK;                    // head dims per lane
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kTileBytes = kTK * kRowBytes;   // K or V part of a stage
    static constexpr int kStageBytes = 2 * kTileBytes;
    // several CTAs per SM where registers and the ring allow it (finer load
    // balance, more loads in flight): three with a two-stage ring for one row
    // per head (B1 H8 N16384 D128 bf16: 15.43 -> 15.09 us against two), two for
    // 2 and 4 rows (whose registers do not allow three)
    static constexpr int kMinBlocks = (RMAX <= 4 && kStageBytes <= 32768) ? (RMAX == 1 ? 3 : 2) : 1;
    static constexpr int kRingBudget = (kMinBlocks == 3 ? 64 : kMinBlocks == 2 ? 96 : 192) * 1024;
    static constexpr int kStages = kRingBudget / kStageBytes < 2 ? 2 : kRingBudget / kStageBytes;
    static constexpr int RR = RMAX < 4 ? RMAX : 4;        // rows per pass
    static constexpr int kPasses = RMAX / RR;
    static constexpr int kN = kKPG * RR;                  // values per reduce-scatter: 8, 16 or 32
    static constexpr int kSh = ilog2(LPK) - ilog2(kN);    // lane in group -> value: v = li >> kSh
    // merge scratch over the drained ring: acc, m, l of every warp and row
    static constexpr int kScratchBytes = kCompWarps * RMAX * (D + 2) * 4;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kSmemData = kRingBytes > kScratchBytes ? kRingBytes : kScratchBytes;
    static constexpr int kSmemBytes = kSmemData + 2 * 8 * kStages + 16;
    static_assert(RMAX == 1 || RMAX == 2 || RMAX == 4 || RMAX == 8, "RMAX");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// DPL consecutive elements of one row, as fp32.
__device__ __forceinline__ void load_row(const uint16_t* p, float (&x)[2]) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    x[0] = __uint_as_float(u << 16);
    x[1] = __uint_as_float(u & 0xffff0000u);
}
__device__ __forceinline__ void load_row(const uint16_t* p, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load_row(const uint16_t* p, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void load_row(const float* p, float (&x)[1]) { x[0] = *p; }
__device__ __forceinline__ void load_row(const float* p, float (&x)[2]) {
    const float2 u = *reinterpret_cast<const float2*>(p);
    x[0] = u.x;
    x[1] = u.y;
}
__device__ __forceinline__ void load_row(const float* p, float (&x)[3]) {
    x[0] = p[0];
    x[1] = p[1];
    x[2] = p[2];
}
__device__ __forceinline__ void load_row(const float* p, float (&x)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    x[0] = u.x;
    x[1] = u.y;
    x[2] = u.z;
    x[3] = u.w;
}
__device__ __forceinline__ void load_row(const float* p, float (&x)[6]) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const float2 u = reinterpret_cast<const float2*>(p)[i];
        x[2 * i] = u.x;
        x[2 * i + 1] = u.y;
    }
}
__device__ __forceinline__ void load_row(const float* p, float (&x)[8]) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float4 u = reinterpret_cast<const float4*>(p)[i];
        x[4 * i] = u.x;
        x[4 * i + 1] = u.y;
        x[4 * i + 2] = u.z;
        x[4 * i + 3] = u.w;
    }
}

__device__ __forceinline__ void store_out(uint16_t* p, float x) {
    *p = (uint16_t)(pack_bf16x2(x, 0.f) & 0xffffu);
}
__device__ __forceinline__ void store_out(float* p, float x) { *p = x; }

// (d0, d1) += (a0, a1) * (b0, b1) as one packed fp32 FMA (each lane rounded as fmaf)
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
        "mov.b64 pa, {%2, %3};\n\t"
        "mov.b64 pb, {%4, %5};\n\t"
        "mov.b64 pd, {%0, %1};\n\t"
        "fma.rn.f32x2 pd, pa, pb, pd;\n\t"
        "mov.b64 {%0, %1}, pd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Dot product of DPL-element slices: pairs through the packed FMA.
template <int DPL>
__device__ __forceinline__ float dot_slice(const float (&a)[DPL], const float (&b)[DPL]) {
    float d0 = 0.f, d1 = 0.f;
#pragma unroll
    for (int i = 0; i + 1 < DPL; i += 2) fma2(d0, d1, a[i], a[i + 1], b[i], b[i + 1]);
    if constexpr (DPL % 2 == 1) d0 = fmaf(a[DPL - 1], b[DPL - 1], d0);
    return d0 + d1;
}

// acc += p * v over a DPL-element slice, pairs through the packed FMA.
template <int DPL>
__device__ __forceinline__ void axpy_slice(float (&acc)[DPL], float p, const float (&v)[DPL]) {
#pragma unroll
    for (int i = 0; i + 1 < DPL; i += 2) fma2(acc[i], acc[i + 1], p, p, v[i], v[i + 1]);
    if constexpr (DPL % 2 == 1) acc[DPL - 1] = fmaf(p, v[DPL - 1], acc[DPL - 1]);
}

// Butterfly reduce-scatter of N values (N = 8, 16 or 32) over groups of L
// lanes (L = 16 or 32, aligned): on return the lane holds the group-wide sum of
// value v = (lane mod L) >> (log2 L - log2 N).  Each halving step exchanges
// half of the remaining values with the partner lane (lane ^ o); the lanes
// left holding the same value after the halving steps are summed by plain
// butterfly steps.
template <int N, int L>
__device__ __forceinline__ float reduce_scatter(float (&x)[N], unsigned lane) {
    static_assert(N <= L, "one value per lane at least");
#pragma unroll
    for (int st = 0; (N >> st) > 1; ++st) {
        const int o = (L / 2) >> st;
        const int h = (N >> st) / 2;
        const bool upper = (lane & (unsigned)o) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = upper ? x[i] : x[i + h];
            const float keep = upper ? x[i + h] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float s = x[0];
#pragma unroll
    for (int o = L / (2 * N); o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

template <typename T, int DPL, int RMAX>
__global__ void __launch_bounds__(kThreads, DecCfg<T, DPL, RMAX>::kMinBlocks)
decode_partial_kernel(const DecodeArgs a) {
    using C = DecCfg<T, DPL, RMAX>;
    constexpr int D = C::D;
    constexpr int RR = C::RR;
    constexpr int kSh = C::kSh;
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kSmemData);
    uint64_t* empty = full + C::kStages;
    int* abort_flag = reinterpret_cast<int*>(empty + C::kStages);
    int* issued_s = abort_flag + 1;

    const long long bh = blockIdx.x;
    const int c_begin = (int)blockIdx.y * a.chunk_len;
    const int c_end = min(a.Nk, c_begin + a.chunk_len);
    const int n_keys = c_end - c_begin;                 // >= 1 by the host's split
    const int n_tiles = (n_keys + kTK - 1) / kTK;
    const unsigned warp = warp_id();
    const unsigned lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCompWarps);
        }
        *abort_flag = 0;
        *issued_s = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // This grid may have been launched before the previous kernel of the stream
    // finished (programmatic stream serialisation): nothing global is touched
    // before that kernel's results are complete and visible.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the merge kernel may be scheduled from now on; it waits for this grid's results
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kCompWarps) {
        if (lane == 0) {
            const T* kg = static_cast<const T*>(a.k) + ((size_t)bh * a.Nk + c_begin) * D;
            const T* vg = static_cast<const T*>(a.v) + ((size_t)bh * a.Nk + c_begin) * D;
            int t = 0;
            for (; t < n_tiles; ++t) {
                const int s = t % C::kStages;
                if (t >= C::kStages && !mbar_wait(&empty[s], ((t / C::kStages) - 1) & 1, abort_flag)) break;
                const int keys = min(kTK, n_keys - t * kTK);
                const unsigned bytes = (unsigned)(keys * C::kRowBytes);
                uint8_t* st = smem + (size_t)s * C::kStageBytes;
                mbar_arrive_expect_tx(&full[s], 2 * bytes);
                bulk_load(st, kg + (size_t)t * kTK * D, bytes, &full[s]);
                bulk_load(st + C::kTileBytes, vg + (size_t)t * kTK * D, bytes, &full[s]);
            }
            *issued_s = t;
        }
    } else {
        // ---------------------------------------------------------- compute
        // Lane = (group g, lane-in-group li): group g takes keys
        // [8w + g*kKPG, 8w + (g+1)*kKPG) of every tile, and li owns head dims
        // [li*DL, (li+1)*DL) of q, of those keys' K/V rows and of acc.
        constexpr int LPK = C::LPK;
        constexpr int DL = C::DL;
        constexpr int kKPG = C::kKPG;
        const int w = (int)warp;
        const int g = (int)(lane / LPK);
        const int li = (int)(lane % LPK);
        float qr[RMAX][DL];
        {
            const float qs = a.scale * kLog2e;
            const T* qg = static_cast<const T*>(a.q) + (size_t)bh * a.R * D + li * DL;
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                if (r < a.R) {
                    load_row(qg + (size_t)r * D, qr[r]);
#pragma unroll
                    for (int i = 0; i < DL; ++i) qr[r][i] *= qs;
                } else {
#pragma unroll
                    for (int i = 0; i < DL; ++i) qr[r][i] = 0.f;
                }
            }
        }
        float acc[RMAX][DL];
#pragma unroll
        for (int r = 0; r < RMAX; ++r)
#pragma unroll
            for (int i = 0; i < DL; ++i) acc[r][i] = 0.f;
        // this lane's (key, row) value of the reduce-scatter, per pass
        const int v_mine = li >> kSh;
        const int j_mine = v_mine / RR;
        float m_mine[C::kPasses], l_mine[C::kPasses];
#pragma unroll
        for (int p = 0; p < C::kPasses; ++p) {
            m_mine[p] = -INFINITY;
            l_mine[p] = 0.f;
        }

        for (int t = 0; t < n_tiles; ++t) {
            const int s = t % C::kStages;
            if (!mbar_wait(&full[s], (t / C::kStages) & 1, abort_flag)) break;
            const int key0 = w * kKeysPerWarp + g * kKPG;            // first key of this group in the tile
            const T* ks = reinterpret_cast<const T*>(smem + (size_t)s * C::kStageBytes) + (size_t)key0 * D + li * DL;
            const T* vs = ks + C::kTileBytes / (int)sizeof(T);
            // keys of this group in this tile that exist; rows past them hold
            // stale or unwritten shared memory and are never used
            const int valid = min(kKPG, max(0, n_keys - t * kTK - key0));
#pragma unroll
            for (int p = 0; p < C::kPasses; ++p) {
                float part[C::kN];
#pragma unroll
                for (int j = 0; j < kKPG; ++j) {
                    float kf[DL];
                    load_row(ks + j * D, kf);
#pragma unroll
                    for (int rr = 0; rr < RR; ++rr) part[j * RR + rr] = dot_slice<DL>(qr[p * RR + rr], kf);
                }
                float sv = reduce_scatter<C::kN, LPK>(part, lane);
                sv = (j_mine < valid) ? sv : -INFINITY;
                float& m = m_mine[p];
                if (__any_sync(0xffffffffu, sv > m + kRescaleThreshold)) {
                    // exact maximum of this tile per row: over the lanes of the
                    // same row (key bits of the value index: lane bits 2-3 or
                    // 2-4; group: lane bit 4)
                    float tmax = sv;
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
                    const float mn = fmaxf(m, tmax);
                    const float alpha = (mn == -INFINITY) ? 1.f : ex2_approx(m - mn);
                    m = mn;
                    l_mine[p] *= alpha;
#pragma unroll
                    for (int rr = 0; rr < RR; ++rr) {
                        const float ar = __shfl_sync(0xffffffffu, alpha, rr << kSh);
#pragma unroll
                        for (int i = 0; i < DL; ++i) acc[p * RR + rr][i] *= ar;
                    }
                }
                const float pw = (m == -INFINITY) ? 0.f : ex2_approx(sv - m);
                l_mine[p] += pw;
#pragma unroll
                for (int j = 0; j < kKPG; ++j) {
                    float vf[DL];
                    if (j < valid) {
                        load_row(vs + j * D, vf);
                    } else {
#pragma unroll
                        for (int i = 0; i < DL; ++i) vf[i] = 0.f;
                    }
#pragma unroll
                    for (int rr = 0; rr < RR; ++rr) {
                        const float pj = __shfl_sync(0xffffffffu, pw, g * LPK + ((j * RR + rr) << kSh));
                        axpy_slice<DL>(acc[p * RR + rr], pj, vf);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        // exp-sum of this warp's keys per row: over the key lanes and groups of each row
#pragma unroll
        for (int p = 0; p < C::kPasses; ++p)
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) l_mine[p] += __shfl_xor_sync(0xffffffffu, l_mine[p], o);
        // the groups of a warp accumulate the same dims over different keys
        if constexpr (C::kGroups == 2) {
#pragma unroll
            for (int r = 0; r < RMAX; ++r)
#pragma unroll
                for (int i = 0; i < DL; ++i) acc[r][i] += __shfl_xor_sync(0xffffffffu, acc[r][i], 16);
        }

        // all compute warps are past the ring before it is reused as scratch
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kCompWarps) : "memory");
        float* sc_acc = reinterpret_cast<float*>(smem);                 // [warp][RMAX][D]
        float* sc_ml = sc_acc + kCompWarps * RMAX * D;                  // [warp][RMAX][2]
        if (g == 0) {
#pragma unroll
            for (int r = 0; r < RMAX; ++r)
#pragma unroll
                for (int i = 0; i < DL; ++i) sc_acc[(w * RMAX + r) * D + li * DL + i] = acc[r][i];
        }
#pragma unroll
        for (int p = 0; p < C::kPasses; ++p) {
            // lane (rr << kSh) holds row p*RR + rr (key 0 of the value index)
            if (g == 0 && (li & ((1 << kSh) - 1)) == 0 && j_mine == 0) {
                const int r = p * RR + v_mine;
                sc_ml[(w * RMAX + r) * 2] = m_mine[p];
                sc_ml[(w * RMAX + r) * 2 + 1] = l_mine[p];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kCompWarps) : "memory");
        if (!*abort_flag) {
            const bool direct = a.nsplit == 1;
            for (int e = (int)threadIdx.x; e < a.R * D; e += 32 * kCompWarps) {
                const int r = e / D;
                const int d = e - r * D;
                float M = -INFINITY;
#pragma unroll
                for (int ww = 0; ww < kCompWarps; ++ww) M = fmaxf(M, sc_ml[(ww * RMAX + r) * 2]);
                float L = 0.f, A = 0.f;
#pragma unroll
                for (int ww = 0; ww < kCompWarps; ++ww) {
                    const float mw = sc_ml[(ww * RMAX + r) * 2];
                    const float wt = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
                    L = fmaf(wt, sc_ml[(ww * RMAX + r) * 2 + 1], L);
                    A = fmaf(wt, sc_acc[(ww * RMAX + r) * D + d], A);
                }
                const size_t row = (size_t)bh * a.R + r;
                if (direct) {
                    store_out(static_cast<T*>(a.o) + row * D + d, A / L);
                    if (d == 0) a.lse[row] = (M + __log2f(L)) * kLn2;
                } else {
                    const size_t prow = ((size_t)bh * a.nsplit + blockIdx.y) * a.R + r;
                    a.part_acc[prow * D + d] = A;
                    if (d == 0) {
                        a.part_ml[prow * 2] = M;
                        a.part_ml[prow * 2 + 1] = L;
                    }
                }
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        // a wait gave up: let every copy still in flight land before the CTA
        // (and its shared memory) goes away
        const int issued = *issued_s;
        for (int t = issued - C::kStages < 0 ? 0 : issued - C::kStages; t < issued; ++t)
            mbar_wait(&full[t % C::kStages], (t / C::kStages) & 1, nullptr);
    }
}

// Merge of the chunk summaries: one CTA per row.  Thread (slice sl, group g)
// owns head dims [4g, 4g + 4) of the chunks c = sl, sl + S, ... and loads all
// of its chunks' (m, l, acc) before using any (one round trip to memory for up
// to 8 chunks per thread), folding them with the two-block formulas; the S
// slice summaries of each group are then folded through shared memory.
constexpr int kMergeThreads = 256;
constexpr int kMergeBatch = 8;

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(const DecodeArgs a) {
    __shared__ float4 s_acc[kMergeThreads];
    __shared__ float s_m[kMergeThreads];
    __shared__ float s_l[kMergeThreads];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // a following launch with programmatic serialisation may start its set-up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const long long row = blockIdx.x;
    const long long bh = row / a.R;
    const int r = (int)(row - bh * a.R);
    const int G = a.D / 4;
    const int S = kMergeThreads / G;
    const int t = (int)threadIdx.x;
    const int sl = t / G;
    const int g = t - sl * G;
    float M = -INFINITY, L = 0.f;
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    if (sl < S) {
        const size_t p0 = (size_t)bh * a.nsplit * a.R + r;   // chunk c: p0 + c * R
        for (int c0 = sl; c0 < a.nsplit; c0 += kMergeBatch * S) {
            float mc[kMergeBatch], lc[kMergeBatch];
            float4 x[kMergeBatch];
#pragma unroll
            for (int u = 0; u < kMergeBatch; ++u) {
                const int c = c0 + u * S;
                if (c < a.nsplit) {
                    const size_t p = p0 + (size_t)c * a.R;
                    mc[u] = a.part_ml[p * 2];
                    lc[u] = a.part_ml[p * 2 + 1];
                    x[u] = *reinterpret_cast<const float4*>(a.part_acc + p * a.D + 4 * g);
                } else {
                    mc[u] = -INFINITY;
                    lc[u] = 0.f;
                    x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int u = 0; u < kMergeBatch; ++u) {
                if (mc[u] == -INFINITY) continue;
                if (mc[u] > M) {
                    const float al = ex2_approx(M - mc[u]);   // 0 while M = -inf
                    L *= al;
                    A.x *= al;
                    A.y *= al;
                    A.z *= al;
                    A.w *= al;
                    M = mc[u];
                }
                const float wc = ex2_approx(mc[u] - M);
                L = fmaf(wc, lc[u], L);
                A.x = fmaf(wc, x[u].x, A.x);
                A.y = fmaf(wc, x[u].y, A.y);
                A.z = fmaf(wc, x[u].z, A.z);
                A.w = fmaf(wc, x[u].w, A.w);
            }
        }
    }
    s_m[t] = M;
    s_l[t] = L;
    s_acc[t] = A;
    __syncthreads();
    if (t < G) {
        float MM = -INFINITY;
        for (int k = 0; k < S; ++k) MM = fmaxf(MM, s_m[k * G + t]);
        float LL = 0.f;
        float4 AA = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < S; ++k) {
            const float mk = s_m[k * G + t];
            const float wk = (mk == -INFINITY) ? 0.f : ex2_approx(mk - MM);
            const float4 xk = s_acc[k * G + t];
            LL = fmaf(wk, s_l[k * G + t], LL);
            AA.x = fmaf(wk, xk.x, AA.x);
            AA.y = fmaf(wk, xk.y, AA.y);
            AA.z = fmaf(wk, xk.z, AA.z);
            AA.w = fmaf(wk, xk.w, AA.w);
        }
        const float inv = 1.f / LL;
        T* orow = static_cast<T*>(a.o) + row * a.D + 4 * t;
        if constexpr (sizeof(T) == 2) {
            *reinterpret_cast<uint2*>(orow) =
                make_uint2(pack_bf16x2(AA.x * inv, AA.y * inv), pack_bf16x2(AA.z * inv, AA.w * inv));
        } else {
            *reinterpret_cast<float4*>(orow) = make_float4(AA.x * inv, AA.y * inv, AA.z * inv, AA.w * inv);
        }
        if (t == 0) a.lse[row] = (MM + __log2f(LL)) * kLn2;
    }
}

template <typename T, int DPL, int RMAX>
cudaError_t launch_partial(const DecodeArgs& a, cudaStream_t stream) {
    using C = DecCfg<T, DPL, RMAX>;
    auto kern = decode_partial_kernel<T, DPL, RMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.BHkv, (unsigned)a.nsplit);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename T, int DPL>
cudaError_t dispatch_rows(const DecodeArgs& a, cudaStream_t stream) {
    if (a.R <= 1) return launch_partial<T, DPL, 1>(a, stream);
    if (a.R <= 2) return launch_partial<T, DPL, 2>(a, stream);
    if (a.R <= 4) return launch_partial<T, DPL, 4>(a, stream);
    return launch_partial<T, DPL, 8>(a, stream);
}

template <typename T, int DPL>
int blocks_rows(int R) {
    if (R <= 1) return DecCfg<T, DPL, 1>::kMinBlocks;
    if (R <= 2) return DecCfg<T, DPL, 2>::kMinBlocks;
    if (R <= 4) return DecCfg<T, DPL, 4>::kMinBlocks;
    return DecCfg<T, DPL, 8>::kMinBlocks;
}

}  // namespace

bool decode_supported(bool bf16, int D, int R) {
    if (R < 1 || R > kDecodeMaxRows) return false;
    if (bf16) return D == 64 || D == 128;
    return D == 32 || D == 64 || D == 96 || D == 128;
}

int decode_blocks_per_sm(bool bf16, int D, int R) {
    if (bf16) return D == 64 ? blocks_rows<uint16_t, 2>(R) : blocks_rows<uint16_t, 4>(R);
    switch (D) {
        case 32: return blocks_rows<float, 1>(R);
        case 64: return blocks_rows<float, 2>(R);
        case 96: return blocks_rows<float, 3>(R);
        default: return blocks_rows<float, 4>(R);
    }
}

cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t stream) {
    if (a.BHkv == 0 || a.R == 0) return cudaSuccess;
    if (a.BHkv > 0x7fffffffLL || a.nsplit < 1 || a.nsplit > 65535) return cudaErrorInvalidValue;
    cudaError_t e;
    if (bf16) e = a.D == 64 ? dispatch_rows<uint16_t, 2>(a, stream) : dispatch_rows<uint16_t, 4>(a, stream);
    else {
        switch (a.D) {
            case 32: e = dispatch_rows<float, 1>(a, stream); break;
            case 64: e = dispatch_rows<float, 2>(a, stream); break;
            case 96: e = dispatch_rows<float, 3>(a, stream); break;
            default: e = dispatch_rows<float, 4>(a, stream); break;
        }
    }
    if (e != cudaSuccess || a.nsplit == 1) return e;
    const long long blocks = a.BHkv * a.R;   // one CTA per row
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kMergeThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (bf16) e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<uint16_t>, a);
    else e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<float>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace mea
