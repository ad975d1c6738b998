// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernels.  Not installed; the public interface is include/mea_attn.h.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mea {

// fp32 SIMT forward (fwd_f32.cu).
struct F32FwdArgs {
    const float* q;
    const float* k;
    const float* v;
    float* o;
    float* lse;
    int BH, Nq, Nk, D;
    float scale;
    int rows_per_cta;   // query rows per CTA (one row per group of warps_per_row warps)
    int warps_per_row;  // warps sharing one row's keys inside a CTA
    int chunks;         // CTAs per cluster splitting the keys (1..16)
    int chunk_len;      // keys per chunk (multiple of 32)
};
cudaError_t launch_fwd_f32(const F32FwdArgs& a, cudaStream_t stream);

// Merge of results over disjoint key ranges (combine.cu).  Pointer arrays are
// passed by value; every part and the output are [rows, D] with rows = B*H*Nq.
constexpr int kCombineMaxParts = 16;
struct CombineArgs {
    const void* o_parts[kCombineMaxParts];
    const float* lse_parts[kCombineMaxParts];
    void* o;
    float* lse;
    long long rows;
    int D;
    int R;
};
cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t stream);

// fp32 SIMT backward (bwd_f32.cu).  Row term D_i in `delta` (workspace).
struct F32BwdArgs {
    const float* q;
    const float* k;
    const float* v;
    const float* o;
    const float* dO;
    const float* lse;
    float* dq;
    float* dk;
    float* dv;
    float* delta;       // [BH, Nq]
    int BH, Nq, Nk, D;
    float scale;
    int q_rows_per_cta;  // dQ kernel: query rows per CTA of 8 warps (1, 2, 4 or 8)
    int k_rows_per_cta;  // dK/dV kernel: key rows per CTA of 8 warps (1, 2, 4 or 8)
    // Accumulating callers: dq, dk, dv are fp32 sums that receive the unscaled
    // dS K, dS^T Q and P^T dO of this call (instead of being overwritten).
    bool accumulate = false;
};
cudaError_t launch_bwd_f32(const F32BwdArgs& a, cudaStream_t stream, unsigned phases);

// Split-KV forward for few query rows per key/value head (decode.cu).  q, o
// are [BHkv, R, D] (the R = G*Nq rows sharing one key/value head), k, v are
// [BHkv, Nk, D], bf16 or fp32.  With nsplit > 1 the chunk summaries go to
// part_acc [BHkv, nsplit, R, D] and part_ml [BHkv, nsplit, R, 2] (fp32) and a
// second kernel merges them; with nsplit == 1 the first kernel writes o, lse.
constexpr int kDecodeMaxRows = 8;
constexpr int kDecodeTileKeys = 64;
struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    float* part_acc;
    float* part_ml;
    long long BHkv;
    int R, Nk, D;
    float scale;
    int nsplit;     // key chunks per key/value head (grid y)
    int chunk_len;  // keys per chunk (multiple of kDecodeTileKeys)
};
bool decode_supported(bool bf16, int D, int R);
int decode_blocks_per_sm(bool bf16, int D, int R);   // CTAs of the partial kernel per SM
cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t stream);

// bf16 tcgen05 forward (fwd_bf16.cu).  Tensor maps are 3-D {D, N, B*H} bf16,
// 128-byte swizzle, box {64, 128, 1}.
struct Bf16FwdArgs {
    CUtensorMap tm_q, tm_k, tm_v;
    uint16_t* o;  // bf16 bits
    float* lse;
    int BH, Nq, Nk, D;
    float scale;
    int chunks;     // CTAs per cluster splitting the keys (1 = no split)
    int chunk_len;  // keys per chunk (multiple of 128) when chunks > 1
    bool fp8_qk = false;  // q, k are e4m3 (maps of uint8, box {128, 128, 1}); D = 128 only
};
cudaError_t launch_fwd_bf16(const Bf16FwdArgs& a, cudaStream_t stream);
// The same forward with persistent CTAs (fwd_persist.cu): at most one CTA per
// SM walks the (head, query-tile pair) items, for bf16 Q/K/V at D = 64 or 128
// when every item holds two full query tiles (Nq a multiple of 256), the keys
// are not split and the key range is short: Nk <= 2048 at D = 128, 4096 at
// D = 64 (longer ranges amortise a CTA's fixed cost by themselves), or up to
// twice that when the item list has single query tiles (fwd_persist_schedule).
constexpr int kFwdPersistMaxKeys128 = 2048;
constexpr int kFwdPersistMaxKeys64 = 4096;
bool fwd_persist_applies(int D, bool fp8_qk, int BH, int Nq, int Nk, int chunks, int sm_count);
cudaError_t launch_fwd_persist(const Bf16FwdArgs& a, int sm_count, cudaStream_t stream);
// Item list of the persistent forward for n_pairs (head, query-tile pair)
// items on sm_count SMs: the first n_pair_items are pairs; when the pairs of a
// partial last round number r with 2r <= sm_count, those r pairs are listed as
// 2r single query tiles instead (n_items = n_pairs + r).  grid = CTAs launched.
struct PersistSchedule {
    long long n_pair_items, n_items, grid;
};
PersistSchedule fwd_persist_schedule(long long n_pairs, int sm_count);
// Clusters of `cluster` CTAs of the tensor-core forward instantiation that a
// launch with these D, operand type and Nq uses that can be resident at once
// (cudaOccupancyMaxActiveClusters); 0 on failure.
int fwd_bf16_max_active_clusters(int D, bool fp8_qk, int Nq, int cluster);

// bf16 backward (bwd_bf16.cu).
struct Bf16BwdArgs {
    CUtensorMap tm_q, tm_k, tm_v, tm_do;
    CUtensorMap tm_dq_acc;  // fp32 {D, Nq, BH}, box {32, 64, 1}, no swizzle (TMA reduce-add target)
    const uint16_t* o;
    const uint16_t* dO;
    const float* lse;
    uint16_t* dq;
    uint16_t* dk;
    uint16_t* dv;
    float* dq_acc;  // workspace [BH, Nq, D] fp32 (zeroed by the preprocess phase); nullptr: not zeroed
    float* delta;   // workspace [BH, Nq] fp32: sum_d dO * O
    // Accumulating callers: dV and the unscaled dS^T Q are added to these fp32
    // [BH, Nk, D] sums instead of being written to dk, dv (nullptr otherwise).
    float* dk_acc = nullptr;
    float* dv_acc = nullptr;
    int BH, Nq, Nk, D;
    float scale;
    int sm_count = 1;   // persistent grids (D = 64): at most one CTA per SM
};
// Phases of the backward, run in this order on one workspace.
constexpr unsigned kBwdPhasePre = 1u;    // delta = rowsum(dO o O); dQ accumulator := 0
constexpr unsigned kBwdPhaseMain = 2u;   // dK, dV; dQ accumulated in fp32
constexpr unsigned kBwdPhaseFinal = 4u;  // dq = bf16(scale * dQ accumulator)
cudaError_t launch_bwd_bf16(const Bf16BwdArgs& a, cudaStream_t stream, unsigned phases);
// out[i] = mul * acc[i] as bf16 (round to nearest even) or fp32; n a multiple of 4.
cudaError_t launch_accum_convert(const float* acc, void* out, long long n, float mul, bool bf16, cudaStream_t stream);

}  // namespace mea
