/*
 * mea_attn.h -- C ABI of the exact memory-efficient attention library
 * (libmea_attn.so, sm_100a).
 *
 * The operation is exact softmax attention for every (batch, head):
 *
 *     O = softmax(scale * Q K^T) V,      lse_i = ln sum_j exp(scale * q_i . k_j)
 *
 * as defined in "Fast and memory-efficient exact attention" (section on the
 * mathematical form: softmax(QK^T / sqrt(d_k)) V) and computed the way
 * "Self-attention Does Not Need O(n^2) Memory" describes (English summary,
 * method bullets): keys and values are consumed block by block, each query row
 * keeps a running maximum score, a running sum of exponentials and a rescaled
 * weighted-value accumulator, and normalisation happens once at the end, so
 * the n x n score matrix is never stored.  The backward pass recomputes the
 * probabilities from lse instead of storing them (the same page's bullet on
 * differentiation by checkpointing).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are contiguous row-major [B, H, N, D] ("BHND"); d_v = d.
 *    q, o, dO, dq: [B, H, Nq, D];  k, v, dk, dv: [B, H, Nk, D];
 *    lse: [B, H, Nq] fp32 (natural log of the scaled scores' exp-sum).
 *  - Every pointer is caller-owned DEVICE memory.  The library never
 *    allocates, frees or synchronises inside fwd/bwd; scratch memory for the
 *    backward pass and the split-KV decode is the caller's `workspace`.
 *  - Tensor pointers (q, k, v, o, dO, dq, dk, dv, workspace) must be 16-byte
 *    aligned; lse must be 4-byte aligned.
 *  - `stream` is a cudaStream_t (CUstream) passed as void*; NULL means the
 *    legacy default stream.  Work is enqueued asynchronously; a returned
 *    MEA_OK means the arguments were valid and the launches were accepted.
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns an error status and leaves all outputs untouched.
 *    The library never aborts the process.
 *  - Device-side failures that do not stop a launch (a bounded wait that
 *    expired) set a per-device flag that mea_last_device_error() reports.
 *
 * Supported set
 *  - MEA_DTYPE_BF16: forward and backward, D in {64, 128}; inputs/outputs bf16,
 *    accumulation fp32 (tcgen05 tensor cores).
 *  - MEA_DTYPE_F32: forward and backward, D in {32, 64, 96, 128}; fp32
 *    throughout (SIMT kernels, no tensor cores).
 *  - e4m3 queries and keys with bf16 values and output: mea_attn_fwd_fp8, D = 128.
 *  - Key/value heads shared by groups of query heads: the _gqa entry points.
 *  - Results over disjoint key ranges (a key split) merged: mea_attn_combine.
 *  - Decode-shaped calls (at most 8 query rows per key/value head) over all
 *    SMs with a caller-given workspace: mea_attn_decode.
 *  - Any Nq >= 0 and Nk >= 1; partial tiles are masked.  No mask, no dropout.
 *  - B*H*max(Nq,Nk)*D < 2^40 elements, and B*H <= 65535 (one launch-grid
 *    dimension indexes the heads; the grouped-query entry points count
 *    B*H_kv).  Decode-shaped calls that the split-KV kernels take accept up
 *    to 2^31-1 heads.  The fp32 forward also needs ceil(Nq/8) <= 65535.
 *    Larger calls return MEA_ERR_UNSUPPORTED before any launch.
 */
#ifndef MEA_ATTN_H
#define MEA_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MEA_OK = 0,
    MEA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, Nk == 0 with rows, non-finite scale */
    MEA_ERR_UNSUPPORTED = 2,  /* head dim / dtype / direction outside the supported set */
    MEA_ERR_MISALIGNED = 3,   /* a pointer violates the alignment rule above */
    MEA_ERR_WORKSPACE = 4,    /* workspace missing or smaller than mea_attn_bwd_workspace_size */
    MEA_ERR_CUDA = 5,         /* a CUDA runtime/driver call or a launch failed */
    MEA_ERR_TIMEOUT = 6       /* a device-side bounded wait expired (see mea_last_device_error) */
} mea_status_t;

typedef enum {
    MEA_DTYPE_F32 = 0,
    MEA_DTYPE_BF16 = 1
} mea_dtype_t;

/*
 * Forward pass: o = softmax(scale * q k^T) v and lse, per (batch, head).
 *
 * Source: "Self-attention Does Not Need O(n^2) Memory" (English summary),
 * method bullets 1-4 (delayed normalisation, running maximum, key/value
 * blocks summarised and merged); the two-block merge formulas of
 * "当注意力成为瓶颈" (section IO感知).
 *
 * q,k,v   inputs (dtype), o output (dtype), lse output fp32 [B,H,Nq].
 * B,H     batch and heads (>= 0); Nq query rows (>= 0); Nk keys (>= 1 when
 *         B*H*Nq > 0); D head dim; scale multiplies q.k before the softmax.
 * Nq == 0 or B == 0 or H == 0 is a no-op returning MEA_OK.
 * Errors: MEA_ERR_INVALID_ARG, MEA_ERR_UNSUPPORTED, MEA_ERR_MISALIGNED,
 *         MEA_ERR_CUDA (launch failure).
 */
mea_status_t mea_attn_fwd(const void* q, const void* k, const void* v,
                          void* o, float* lse,
                          int B, int H, int Nq, int Nk, int D, float scale,
                          mea_dtype_t dtype, void* stream);

/*
 * Bytes of device workspace mea_attn_bwd needs for these sizes (written to
 * *bytes).  bf16: an fp32 dQ accumulator [B,H,Nq,D] and the fp32 row term
 * D_i = sum_d dO_id O_id [B,H,Nq], each 256-byte aligned.  fp32: the row term
 * only.  O(N*D), never O(N^2).  Errors: MEA_ERR_INVALID_ARG (null `bytes`,
 * negative size), MEA_ERR_UNSUPPORTED (dtype/D not supported).
 */
mea_status_t mea_attn_bwd_workspace_size(int B, int H, int Nq, int Nk, int D,
                                         mea_dtype_t dtype, size_t* bytes);

/*
 * Backward pass: gradients of sum(dO o O) with respect to q, k, v.
 *
 * Source: "Self-attention Does Not Need O(n^2) Memory" (English summary),
 * method bullet on differentiation: intermediate states are recomputed
 * (checkpointing), here P = exp(scale * q k^T - lse) from the forward's lse.
 * The gradient formulas are ordinary softmax calculus (the pages print none):
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_d dO_id O_id,  dS = P o (dP - D),
 *   dQ = scale dS K,  dK = scale dS^T Q.
 *
 * q,k,v,o,dO inputs (dtype); lse input fp32 [B,H,Nq] from mea_attn_fwd;
 * dq,dk,dv outputs (dtype).  workspace: device memory of at least
 * mea_attn_bwd_workspace_size() bytes, owned by the caller, contents on entry
 * ignored, clobbered on exit.  bf16: dq is accumulated in fp32 by reduce-adds
 * from many CTAs, so it is not bitwise deterministic run to run (dk, dv are).
 * fp32: dq, dk, dv are each summed by one CTA in a fixed order (bitwise
 * deterministic).  Nq == 0 writes zeros to dk, dv.  Errors as for
 * mea_attn_fwd plus MEA_ERR_WORKSPACE.
 */
mea_status_t mea_attn_bwd(const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dO,
                          void* dq, void* dk, void* dv,
                          int B, int H, int Nq, int Nk, int D, float scale,
                          mea_dtype_t dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * The backward pass in its three stream-ordered phases, for callers that want
 * to time or overlap them separately.  mea_attn_bwd(...) is exactly
 * mea_attn_bwd_phase(MEA_BWD_ALL, ...).  Every phase takes the full argument
 * list of mea_attn_bwd and validates it the same way; the phases must run in
 * the order PREPROCESS, MAIN, FINALIZE on the same workspace:
 *   MEA_BWD_PREPROCESS  D_i = sum_d dO_id O_id into the workspace; zeroes the
 *                       fp32 dQ accumulator.               (reads o, dO)
 *   MEA_BWD_MAIN        recomputes P from lse per key tile; writes dk, dv and
 *                       adds dS K into the dQ accumulator.  (reads q, k, v, dO, lse)
 *   MEA_BWD_FINALIZE    dq = bf16(scale * dQ accumulator). (writes dq)
 * For MEA_DTYPE_F32 the main phase writes dq, dk and dv directly and the
 * preprocess phase only computes D_i; the finalize phase does nothing.
 * Errors as for mea_attn_bwd; an unknown phase returns MEA_ERR_INVALID_ARG.
 */
typedef enum {
    MEA_BWD_ALL = 0,
    MEA_BWD_PREPROCESS = 1,
    MEA_BWD_MAIN = 2,
    MEA_BWD_FINALIZE = 3
} mea_bwd_phase_t;

mea_status_t mea_attn_bwd_phase(mea_bwd_phase_t phase,
                                const void* q, const void* k, const void* v,
                                const void* o, const float* lse, const void* dO,
                                void* dq, void* dk, void* dv,
                                int B, int H, int Nq, int Nk, int D, float scale,
                                mea_dtype_t dtype,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Shared key/value heads: grouped-query (1 < H_kv < H) and multi-query
 * (H_kv == 1) attention.
 *
 * Source: "当注意力成为瓶颈从on困境到线性复杂度的技术突围" (section
 * 推理优化：减少KV Cache): the query heads are split into groups and each
 * group shares one key/value head.  Reading adopted: the groups are
 * consecutive, so query head h uses key/value head h / (H / H_kv).  The
 * gradient of a shared key/value head is the sum over the query heads of its
 * group.
 *
 * Layout: q, o, dO, dq [B, H, Nq, D]; k, v, dk, dv [B, H_kv, Nk, D];
 * lse [B, H, Nq] fp32.  Because the G = H / H_kv query heads of a group are
 * consecutive, they form one contiguous [G*Nq, D] block of q, so each call
 * runs the kernels of mea_attn_fwd / mea_attn_bwd over B*H_kv heads of G*Nq
 * query rows: every key/value tile is loaded once per group, and dk, dv sum
 * over the group inside one accumulator (no atomics, deterministic).
 *
 * Arguments, ownership, alignment, supported dtypes and head dims, and errors
 * are those of the entry point without the suffix, plus: H_kv < 1 or H not a
 * multiple of H_kv returns MEA_ERR_INVALID_ARG; G*Nq above 2^31-1 returns
 * MEA_ERR_UNSUPPORTED.  H == 0 is a no-op for the forward; the backward then
 * writes zeros to dk, dv.  H_kv == H is exactly mea_attn_fwd / mea_attn_bwd.
 */
mea_status_t mea_attn_fwd_gqa(const void* q, const void* k, const void* v,
                              void* o, float* lse,
                              int B, int H, int H_kv, int Nq, int Nk, int D, float scale,
                              mea_dtype_t dtype, void* stream);

mea_status_t mea_attn_bwd_gqa_workspace_size(int B, int H, int H_kv, int Nq, int Nk, int D,
                                             mea_dtype_t dtype, size_t* bytes);

mea_status_t mea_attn_bwd_gqa(const void* q, const void* k, const void* v,
                              const void* o, const float* lse, const void* dO,
                              void* dq, void* dk, void* dv,
                              int B, int H, int H_kv, int Nq, int Nk, int D, float scale,
                              mea_dtype_t dtype,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward pass with e4m3 (FP8) queries and keys.
 *
 * Source: "当注意力成为瓶颈从on困境到线性复杂度的技术突围" (section
 * IO感知：重新审视硬件, the FlashAttention-3 paragraph on FP8 tensor cores).
 * Reading adopted: Q and K are stored as e4m3 with one dequantisation factor
 * each (q = q_descale * q8, k = k_descale * k8); V, the probabilities P and
 * the output stay bf16.  The operation is then exactly that of mea_attn_fwd
 * on the dequantised inputs:
 *     O = softmax(scale * q_descale * k_descale * q8 k8^T) v,
 *     lse_i = ln sum_j exp(scale * q_descale * k_descale * q8_i . k8_j).
 * S = q8 k8^T runs on the tensor cores as kind::f8f6f4 (each product of two
 * e4m3 values is exact in the fp32 accumulator); the rest is the bf16 path.
 *
 * q: e4m3 [B, H, Nq, D];  k: e4m3 [B, H_kv, Nk, D];  v: bf16 [B, H_kv, Nk, D];
 * o: bf16 [B, H, Nq, D];  lse: fp32 [B, H, Nq].  H_kv key/value heads are
 * shared by groups of H / H_kv query heads as in mea_attn_fwd_gqa (H_kv = H is
 * ordinary multi-head attention).  D = 128 only.  Pointers as for
 * mea_attn_fwd (16-byte aligned, lse 4-byte aligned).
 * Errors: MEA_ERR_INVALID_ARG (also for descale factors that are not finite
 * and positive), MEA_ERR_UNSUPPORTED (D != 128), MEA_ERR_MISALIGNED,
 * MEA_ERR_CUDA.
 */
mea_status_t mea_attn_fwd_fp8(const void* q, const void* k, const void* v,
                              void* o, float* lse,
                              int B, int H, int H_kv, int Nq, int Nk, int D, float scale,
                              float q_descale, float k_descale, void* stream);

/*
 * Merge of results computed over disjoint key ranges (key / sequence split).
 *
 * Source: "Self-attention Does Not Need O(n^2) Memory" (English summary, the
 * bullet on summarising the results of key/value chunks) with the two-block
 * formulas of "当注意力成为瓶颈从on困境到线性复杂度的技术突围" (section IO感知).
 * Part r is mea_attn_fwd's output (o_r, lse_r) over the r-th key range; the
 * merge gives exactly the attention over all keys:
 *     lse = ln sum_r exp(lse_r),     o = sum_r exp(lse_r - lse) o_r.
 * A part with lse = -inf (no keys) contributes nothing; a row whose parts all
 * have lse = -inf has no keys at all and gets o = 0 and lse = -inf.
 *
 * o_parts, lse_parts: HOST arrays of R device pointers (1 <= R <= 16); each
 * o part is [B, H, Nq, D] in `dtype`, each lse part [B, H, Nq] fp32.  The
 * pointers may address memory of other GPUs that this one can read (peer
 * access), so the merge can read remote parts directly.  o, lse: outputs of
 * the same shapes.  Pointers 16-byte (o) / 4-byte (lse) aligned; D a multiple
 * of 8, at most 256.  The backward of a key split needs no entry point of its
 * own: each range runs mea_attn_bwd_phase with the merged o and lse, the fp32
 * dQ accumulators of the ranges are summed between MAIN and FINALIZE, and dk,
 * dv stay with their range.
 * Errors: MEA_ERR_INVALID_ARG, MEA_ERR_UNSUPPORTED (R, D), MEA_ERR_MISALIGNED,
 * MEA_ERR_CUDA.
 */
mea_status_t mea_attn_combine(const void* const* o_parts, const float* const* lse_parts, int R,
                              void* o, float* lse, int B, int H, int Nq, int D,
                              mea_dtype_t dtype, void* stream);

/*
 * Split-KV forward for decode-shaped calls: few query rows per key/value head
 * against a long key range (token-by-token generation).
 *
 * Source: "Self-attention Does Not Need O(n^2) Memory" (Chinese summary,
 * section 方法详解: for a single query the scores and weighted values are
 * accumulated key by key with two running quantities, the weighted sum and the
 * total weight, plus the running maximum), its chunk summaries merged with the
 * two-block formulas of "当注意力成为瓶颈从on困境到线性复杂度的技术突围"
 * (section IO感知); the workload is the one the "overhead" page (section
 * 对模型开发与部署的影响) names for autoregressive generation, where every new
 * token attends to all previous ones.  The operation is exactly that of
 * mea_attn_fwd_gqa.
 *
 * With R = (H / H_kv) * Nq <= 8 rows per key/value head (and a head dim of the
 * dtype's supported set) the call reads K and V once with every SM of the
 * device: the keys of each head are cut into chunks, every CTA summarises one
 * chunk (running max, exp-sum, unnormalised fp32 accumulator) into
 * `workspace`, and a second kernel merges the summaries into o and lse.  With
 * more rows per head the call is mea_attn_fwd_gqa and `workspace` is unused.
 *
 * Arguments, layouts, alignment and dtypes are those of mea_attn_fwd_gqa.
 * workspace: caller-owned device memory of at least the size that
 * mea_attn_decode_workspace_size returns for the same shape on the device
 * current at the call (it depends on the device's SM count); 16-byte aligned;
 * its contents are scratch (no initialisation needed, nothing kept).  Size 0
 * (workspace may be NULL) when one chunk per head already fills the device or
 * the call has more than 8 rows per head.
 * Both kernels of the split path are launched with programmatic stream
 * serialisation: a kernel may begin its set-up while the previous kernel in
 * the stream drains, but reads or writes no global memory before that kernel
 * has completed, so ordering is that of a plain stream (graph capture works).
 * Errors: those of mea_attn_fwd_gqa, plus MEA_ERR_WORKSPACE (missing or too
 * small) and MEA_ERR_MISALIGNED for the workspace.
 */
mea_status_t mea_attn_decode_workspace_size(int B, int H, int H_kv, int Nq, int Nk, int D,
                                            mea_dtype_t dtype, size_t* bytes);

mea_status_t mea_attn_decode(const void* q, const void* k, const void* v,
                             void* o, float* lse,
                             int B, int H, int H_kv, int Nq, int Nk, int D, float scale,
                             mea_dtype_t dtype, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * Accumulating backward of one key range, for callers that split the keys
 * (and queries) over several calls -- sequence-parallel attention whose
 * key/value blocks visit every rank, as in the Ring Attention paragraph of
 * "当注意力成为瓶颈从on困境到线性复杂度的技术突围" (section 分布式：突破单卡限制).
 *
 * P = exp(scale q k^T - lse) is recomputed from the given lse, which must be
 * the merged lse over ALL keys (the checkpointing of "Self-attention Does Not
 * Need O(n^2) Memory", English summary, method bullet on differentiation), and
 * o the merged output.  Then every contribution of this key range is final and
 * contributions of disjoint key (or query) ranges simply add, so this call adds
 * to caller-owned fp32 sums:
 *     dq_acc [B, H, Nq, D] += dS K,   dk_acc [B, H, Nk, D] += dS^T Q,
 *     dv_acc [B, H, Nk, D] += P^T dO,   dS = P o (dO V^T - rowsum(dO o o)),
 * WITHOUT the softmax scale on dq_acc and dk_acc (dQ = scale dq_acc,
 * dK = scale dk_acc: see mea_attn_accum_convert).  The caller zeroes the sums
 * before the first call; they stay fp32 over any number of calls.
 *
 * q, o, dO [B, H, Nq, D] and k, v [B, H, Nk, D] in `dtype` (bf16: D in {64,
 * 128}; fp32: D in {32, 64, 96, 128}), lse [B, H, Nq] fp32; all device memory,
 * 16-byte aligned (lse 4-byte), caller-owned.  `workspace` (256-byte aligned,
 * at least mea_attn_bwd_accum_workspace_size bytes) holds the row term.  An
 * empty query or key range adds nothing (MEA_OK).  Asynchronous on `stream`;
 * dq_acc is summed by fp32 reduce-adds in no fixed order (bf16), dk_acc and
 * dv_acc in a fixed order.  Errors: MEA_ERR_INVALID_ARG, MEA_ERR_UNSUPPORTED,
 * MEA_ERR_MISALIGNED, MEA_ERR_WORKSPACE, MEA_ERR_CUDA.
 */
mea_status_t mea_attn_bwd_accum_workspace_size(int B, int H, int Nq, int Nk, int D, mea_dtype_t dtype,
                                               size_t* bytes);
mea_status_t mea_attn_bwd_accum(const void* q, const void* k, const void* v,
                                const void* o, const float* lse, const void* dO,
                                float* dq_acc, float* dk_acc, float* dv_acc,
                                int B, int H, int Nq, int Nk, int D, float scale,
                                mea_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * out[i] = mul * acc[i] for i < n, written as `dtype` (bf16 rounded to nearest
 * even, or fp32): turns the fp32 sums of mea_attn_bwd_accum into gradients
 * (mul = scale for dq and dk, 1 for dv).  acc, out: device memory, 16-byte
 * aligned; n a multiple of 4 (MEA_ERR_UNSUPPORTED otherwise).  Asynchronous on
 * `stream`.  Errors: MEA_ERR_INVALID_ARG, MEA_ERR_UNSUPPORTED,
 * MEA_ERR_MISALIGNED, MEA_ERR_CUDA.
 */
mea_status_t mea_attn_accum_convert(const float* acc, void* out, long long n, float mul, mea_dtype_t dtype,
                                    void* stream);

/*
 * Backward pass that allocates nothing and takes no workspace./*
 * Backward pass that allocates nothing and takes no workspace.  The paper has
 * no counterpart: this is a deployment convenience of this library.
 *
 * Some callers cannot call cudaMalloc or any allocator: a plugin inside an
 * inference runtime or framework whose device memory is owned and budgeted by
 * the host application, real-time or embedded code whose memory is fixed at
 * start-up, or code that holds no allocator handle at all.  For them the
 * scratch that mea_attn_bwd takes as `workspace` (fp32 dQ accumulator and row
 * term) lives in one static device array of MEA_NOALLOC_SCRATCH_BYTES (64 MiB)
 * compiled into the library; every GPU that loads the library holds that array
 * until the process exits.
 *
 * Arguments, layout, results and errors are those of mea_attn_bwd without the
 * workspace pair, for MEA_DTYPE_BF16 only (MEA_DTYPE_F32 returns
 * MEA_ERR_UNSUPPORTED).  Sizes whose workspace (mea_attn_bwd_workspace_size) exceeds
 * MEA_NOALLOC_SCRATCH_BYTES are rejected with MEA_ERR_WORKSPACE and a message
 * in mea_last_error_message().  The first call on each device resolves the
 * array's device address (cudaGetSymbolAddress) with that device current; make
 * that first call before any stream capture.  The address is remembered with
 * the unique id of the CUDA context it belongs to: after cudaDeviceReset, or
 * when another context becomes current, the next call resolves it again (so
 * that call, too, belongs before any capture).  All calls on a device share the
 * one array: calls that overlap on the GPU (different streams, or different
 * host threads without ordering) race on it and give wrong gradients; calls
 * ordered on one stream are safe.  Each call clears the part that must start
 * at zero itself.  It never calls cudaMalloc, cudaFree or any allocating
 * library routine.
 */
#define MEA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

mea_status_t mea_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                  const void* o, const float* lse, const void* dO,
                                  void* dq, void* dk, void* dv,
                                  int B, int H, int Nq, int Nk, int D, float scale,
                                  mea_dtype_t dtype, void* stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * flag.  Returns MEA_ERR_TIMEOUT if any kernel of this library gave up on a
 * bounded wait since the last call, MEA_ERR_CUDA if the synchronisation
 * itself failed, MEA_OK otherwise.
 */
mea_status_t mea_last_device_error(void* stream);

/*
 * Self-test of the device-side failure detection.  Launches one kernel on
 * `stream` whose only thread waits on an mbarrier that nothing ever completes,
 * using the same bounded wait every kernel of this library uses.  After the
 * wait's wall-clock limit (about one second) the kernel writes 1 to *gave_up
 * (device memory, 4-byte aligned), records the expiry in the device error
 * flag and returns normally: mea_last_device_error() then reports
 * MEA_ERR_TIMEOUT and the context stays usable.  Nothing faults, traps or
 * hangs.  Errors: MEA_ERR_INVALID_ARG, MEA_ERR_MISALIGNED, MEA_ERR_CUDA.
 */
mea_status_t mea_selftest_bounded_wait(int* gave_up, void* stream);

/* Static, human-readable name of a status code (never NULL). */
const char* mea_status_string(mea_status_t status);

/*
 * Text describing the most recent failure reported by this library on the
 * calling host thread (which call failed and the CUDA error, if any); empty
 * if none.  The pointer stays valid until the next call on the same thread.
 */
const char* mea_last_error_message(void);

/* Library ABI version: 100 * major + minor. */
int mea_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MEA_ATTN_H */
