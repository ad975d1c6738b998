// api.cu -- the C ABI declared in include/mea_attn.h: argument validation,
// dispatch, TMA tensor-map encoding and launches on the caller's stream.
// Nothing here allocates, frees or synchronises on the fwd/bwd paths.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "mea_attn.h"
#include "ptx.cuh"

namespace mea {
__device__ unsigned int g_device_error = 0;

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// will ever arrive on.  The wait gives up after its wall-clock limit, records
// the timeout in g_device_error and the kernel returns normally.
__global__ void selftest_wait_kernel(int* gave_up) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        const bool ok = mbar_wait(&bar, 0, nullptr);
        *gave_up = ok ? 0 : 1;
    }
}
}  // namespace mea

namespace {

constexpr int kMaxDevices = 64;

// Text of the most recent failure on this host thread (mea_last_error_message).
thread_local char g_err_msg[256] = "";

mea_status_t fail(mea_status_t st, const char* where, const char* detail) {
    std::snprintf(g_err_msg, sizeof(g_err_msg), "%s: %s", where, detail ? detail : "");
    return st;
}
mea_status_t fail_cuda(const char* where, cudaError_t e) {
    return fail(MEA_ERR_CUDA, where, cudaGetErrorString(e));
}

struct DeviceInfo {
    bool init = false;
    bool sm100 = false;
    int sm_count = 0;
    // clusters of the tensor-core forward (index 0: D = 64, 1: D = 128,
    // 2: D = 128 with e4m3 Q/K; +3 for the single-query-tile instantiations)
    // that can be resident at once, per cluster size; -1 until first queried
    int fwd_clusters[6][17];
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

mea_status_t device_info(DeviceInfo** out) {
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return fail_cuda("cudaGetDevice", ce);
    if (dev < 0 || dev >= kMaxDevices) return MEA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.init) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return fail(MEA_ERR_CUDA, "cudaDeviceGetAttribute", "failed");
        d.sm100 = (major == 10 && minor == 0);
        d.sm_count = sms;
        for (auto& row : d.fwd_clusters)
            for (int& n : row) n = -1;
        d.init = true;
    }
    if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return fail(MEA_ERR_CUDA, "cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled unavailable");
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (!d.sm100) return fail(MEA_ERR_UNSUPPORTED, "device", "compute capability 10.0 (sm_100a) required");
    *out = &d;
    return MEA_OK;
}

// Clusters of `size` CTAs of the bf16 forward that fit on the device at once
// (cached; 0 if the query fails, which only disables that cluster size).
int fwd_max_clusters(DeviceInfo* d, int D, bool fp8, int Nq, int size) {
    std::lock_guard<std::mutex> lk(g_mu);
    const int single = (D == 128 && Nq <= 128) ? 3 : 0;   // the kernel's deep-ring instantiation
    int& n = d->fwd_clusters[(fp8 ? 2 : (D == 128 ? 1 : 0)) + single][size];
    if (n < 0) n = mea::fwd_bf16_max_active_clusters(D, fp8, Nq, size);
    return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// 3-D bf16 map over [BH][N][D]: dims {D, N, BH}, box {64, 128, 1}, 128-byte swizzle,
// out-of-range rows read as zero.
mea_status_t make_map(CUtensorMap* m, const void* base, int BH, int N, int D) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[64];
        std::snprintf(buf, sizeof(buf), "CUresult %d", (int)r);
        return fail(MEA_ERR_CUDA, "cuTensorMapEncodeTiled", buf);
    }
    return MEA_OK;
}

// 3-D e4m3 map over [BH][N][D] with D = 128: dims {128, N, BH}, box {128, 128, 1}
// (one 128-byte row per element row), 128-byte swizzle, out-of-range rows read as zero.
mea_status_t make_map_u8(CUtensorMap* m, const void* base, int BH, int N, int D) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)N * D};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[64];
        std::snprintf(buf, sizeof(buf), "CUresult %d (e4m3)", (int)r);
        return fail(MEA_ERR_CUDA, "cuTensorMapEncodeTiled", buf);
    }
    return MEA_OK;
}

// 3-D fp32 map over the dQ accumulator [BH][Nq][D]: box {32, 64, 1}, no swizzle
// (target of the backward's TMA reduce-adds; x offsets are multiples of 32 floats).
mea_status_t make_map_f32_acc(CUtensorMap* m, void* base, int BH, int Nq, int D) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Nq, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)Nq * D * 4};
    cuuint32_t box[3] = {32, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[64];
        std::snprintf(buf, sizeof(buf), "CUresult %d (dQ accumulator)", (int)r);
        return fail(MEA_ERR_CUDA, "cuTensorMapEncodeTiled", buf);
    }
    return MEA_OK;
}

mea_status_t cuda_status(cudaError_t e, const char* where) {
    return e == cudaSuccess ? MEA_OK : fail_cuda(where, e);
}

// The tensor-core forward over BH heads: bf16 q, k (fp8 = false) or e4m3 q, k
// (fp8 = true, D = 128); bf16 v, o.  Arguments are validated by the caller.
mea_status_t tc_forward(const void* q, const void* k, const void* v, void* o, float* lse, int BH, int Nq, int Nk,
                        int D, float scale, bool fp8, DeviceInfo* dev, cudaStream_t s) {
    mea::Bf16FwdArgs a;
    mea_status_t st;
    a.fp8_qk = fp8;
    if ((st = (fp8 ? make_map_u8 : make_map)(&a.tm_q, q, BH, Nq, D)) != MEA_OK) return st;
    if ((st = (fp8 ? make_map_u8 : make_map)(&a.tm_k, k, BH, Nk, D)) != MEA_OK) return st;
    if ((st = make_map(&a.tm_v, v, BH, Nk, D)) != MEA_OK) return st;
    a.o = static_cast<uint16_t*>(o);
    a.lse = lse;
    a.BH = BH;
    a.Nq = Nq;
    a.Nk = Nk;
    a.D = D;
    a.scale = scale;
    if (BH > 65535) return MEA_ERR_UNSUPPORTED;
    // Split the keys over a cluster when the (query tile x head) grid would
    // leave more than half of the SMs idle, e.g. decode-shaped calls with a
    // handful of rows: the cluster size is the one that puts the most CTAs to
    // work while every cluster of the launch is resident at once (one wave),
    // with at least two key tiles per CTA.
    {
        const long long base = (long long)((Nq + 255) / 256) * BH;
        const int key_tiles = (Nk + 127) / 128;
        int chunks = 1;
        if (base * 2 <= dev->sm_count) {
            long long best = base;
            for (int c = 2; c <= 16 && key_tiles >= 2 * c; ++c) {
                if (base > fwd_max_clusters(dev, D, fp8, Nq, c)) continue;
                if (base * c > best) {
                    best = base * c;
                    chunks = c;
                }
            }
        }
        a.chunks = chunks;
        a.chunk_len = (int)round_up((size_t)((Nk + chunks - 1) / chunks), 128);
        if ((long long)((Nq + 255) / 256) * chunks > 0x7fffffffLL) return MEA_ERR_UNSUPPORTED;
    }
    if (mea::fwd_persist_applies(D, fp8, BH, Nq, Nk, a.chunks, dev->sm_count))
        return cuda_status(mea::launch_fwd_persist(a, dev->sm_count, s), "fwd_persist launch");
    return cuda_status(mea::launch_fwd_bf16(a, s), "fwd_bf16 launch");
}

// Split-KV decode plan for BHkv key/value heads of R query rows each: the key
// range of a head is cut into nsplit chunks of whole 64-key tiles so that the
// launch has at most one CTA per slot of the device (SMs x resident CTAs of
// the partial kernel) and every chunk holds at least one key.
struct DecodePlan {
    int nsplit = 1;
    int chunk_len = 0;
    size_t ws_bytes = 0;   // chunk summaries; 0 when nsplit == 1
};
DecodePlan decode_plan(const DeviceInfo* dev, long long BHkv, int R, int Nk, int D, bool bf16) {
    DecodePlan p;
    const long long tiles = ((long long)Nk + mea::kDecodeTileKeys - 1) / mea::kDecodeTileKeys;
    const long long slots = (long long)dev->sm_count * mea::decode_blocks_per_sm(bf16, D, R);
    long long n = 1;
    if (BHkv > 0 && BHkv < slots) n = slots / BHkv;
    if (n > tiles) n = tiles;
    if (n < 1) n = 1;
    const long long chunk_tiles = (tiles + n - 1) / n;
    p.nsplit = (int)((tiles + chunk_tiles - 1) / chunk_tiles);
    p.chunk_len = (int)(chunk_tiles * mea::kDecodeTileKeys);
    if (p.nsplit > 1) p.ws_bytes = (size_t)BHkv * p.nsplit * R * (D + 2) * sizeof(float);
    return p;
}

mea_status_t launch_decode_plan(const void* q, const void* k, const void* v, void* o, float* lse, long long BHkv,
                                int R, int Nk, int D, float scale, bool bf16, const DecodePlan& p, void* ws,
                                cudaStream_t s) {
    mea::DecodeArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.lse = lse;
    a.BHkv = BHkv;
    a.R = R;
    a.Nk = Nk;
    a.D = D;
    a.scale = scale;
    a.nsplit = p.nsplit;
    a.chunk_len = p.chunk_len;
    a.part_acc = static_cast<float*>(ws);
    a.part_ml = p.nsplit > 1 ? a.part_acc + (size_t)BHkv * p.nsplit * R * D : nullptr;
    return cuda_status(mea::launch_decode(a, bf16, s), "decode launch");
}

mea_status_t common_checks(int B, int H, int Nq, int Nk, int D, float scale, mea_dtype_t dtype) {
    if (dtype != MEA_DTYPE_F32 && dtype != MEA_DTYPE_BF16) return MEA_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || D <= 0) return MEA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return MEA_ERR_INVALID_ARG;
    if ((long long)B * H > 0x7fffffffLL) return MEA_ERR_INVALID_ARG;
    const long long maxn = Nq > Nk ? Nq : Nk;
    if ((long long)B * H * maxn * D >= (1LL << 40)) return MEA_ERR_INVALID_ARG;
    if (dtype == MEA_DTYPE_BF16 && D != 64 && D != 128) return MEA_ERR_UNSUPPORTED;
    if (dtype == MEA_DTYPE_F32 && (D % 32 != 0 || D > 128)) return MEA_ERR_UNSUPPORTED;
    return MEA_OK;
}


}  // namespace

extern "C" {

const char* mea_status_string(mea_status_t s) {
    switch (s) {
        case MEA_OK: return "MEA_OK";
        case MEA_ERR_INVALID_ARG: return "MEA_ERR_INVALID_ARG: invalid argument";
        case MEA_ERR_UNSUPPORTED: return "MEA_ERR_UNSUPPORTED: unsupported dtype, head dim, direction or device";
        case MEA_ERR_MISALIGNED: return "MEA_ERR_MISALIGNED: pointer misaligned";
        case MEA_ERR_WORKSPACE: return "MEA_ERR_WORKSPACE: workspace missing or too small";
        case MEA_ERR_CUDA: return "MEA_ERR_CUDA: CUDA call or launch failed";
        case MEA_ERR_TIMEOUT: return "MEA_ERR_TIMEOUT: a device-side bounded wait expired";
    }
    return "MEA_ERR_UNKNOWN";
}

int mea_version(void) { return 100; }

const char* mea_last_error_message(void) { return g_err_msg; }

mea_status_t mea_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                          int Nk, int D, float scale, mea_dtype_t dtype, void* stream) {
    mea_status_t st = common_checks(B, H, Nq, Nk, D, scale, dtype);
    if (st != MEA_OK) return st;
    const long long rows = (long long)B * H * Nq;
    if (rows == 0) return MEA_OK;
    if (Nk == 0) return MEA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !lse) return MEA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return MEA_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    if ((st = device_info(&dev)) != MEA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int BH = B * H;

    // Few rows per head: when one chunk per head already fills the device, the
    // split-KV decode kernel runs alone (no workspace needed).
    const bool bf16 = dtype == MEA_DTYPE_BF16;
    if (mea::decode_supported(bf16, D, Nq)) {
        const DecodePlan p = decode_plan(dev, BH, Nq, Nk, D, bf16);
        if (p.nsplit == 1) return launch_decode_plan(q, k, v, o, lse, BH, Nq, Nk, D, scale, bf16, p, nullptr, s);
    }

    if (dtype == MEA_DTYPE_F32) {
        mea::F32FwdArgs a;
        a.q = static_cast<const float*>(q);
        a.k = static_cast<const float*>(k);
        a.v = static_cast<const float*>(v);
        a.o = static_cast<float*>(o);
        a.lse = lse;
        a.BH = BH;
        a.Nq = Nq;
        a.Nk = Nk;
        a.D = D;
        a.scale = scale;
        if (Nq >= 8) { a.rows_per_cta = 8; a.warps_per_row = 1; }
        else if (Nq >= 4) { a.rows_per_cta = 4; a.warps_per_row = 2; }
        else if (Nq >= 2) { a.rows_per_cta = 2; a.warps_per_row = 4; }
        else { a.rows_per_cta = 1; a.warps_per_row = (D <= 64) ? 16 : 8; }   // 16 warps only within the
                                                                            // D <= 64 register budget
        const long long base = (long long)BH * ((Nq + a.rows_per_cta - 1) / a.rows_per_cta);
        const long long target = 2LL * dev->sm_count;
        int chunks = 1;
        while (chunks < 16 && base * chunks < target &&
               (long long)Nk / (2 * chunks) >= 2LL * 32 * a.warps_per_row)
            chunks *= 2;
        a.chunks = chunks;
        const long long per = (Nk + chunks - 1) / chunks;
        a.chunk_len = (int)round_up((size_t)per, 32);
        if ((long long)((Nq + a.rows_per_cta - 1) / a.rows_per_cta) > 65535 || BH > 65535)
            return MEA_ERR_UNSUPPORTED;
        return cuda_status(mea::launch_fwd_f32(a, s), "fwd_f32 launch");
    }

    return tc_forward(q, k, v, o, lse, BH, Nq, Nk, D, scale, false, dev, s);
}

mea_status_t mea_attn_bwd_workspace_size(int B, int H, int Nq, int Nk, int D, mea_dtype_t dtype, size_t* bytes) {
    if (bytes == nullptr) return MEA_ERR_INVALID_ARG;
    mea_status_t st = common_checks(B, H, Nq, Nk, D, 1.0f, dtype);
    if (st != MEA_OK) return st;
    const size_t rows = (size_t)B * H * Nq;
    if (dtype == MEA_DTYPE_F32) {
        // fp32: the row term only (dQ is summed per row in registers)
        *bytes = round_up(rows * sizeof(float), 256);
        return MEA_OK;
    }
    *bytes = round_up(rows * D * sizeof(float), 256) + round_up(rows * sizeof(float), 256);
    return MEA_OK;
}

mea_status_t mea_attn_bwd_phase(mea_bwd_phase_t phase, const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dO, void* dq, void* dk, void* dv, int B, int H, int Nq,
                                int Nk, int D, float scale, mea_dtype_t dtype, void* workspace,
                                size_t workspace_bytes, void* stream) {
    unsigned phases = 0;
    switch (phase) {
        case MEA_BWD_ALL: phases = mea::kBwdPhasePre | mea::kBwdPhaseMain | mea::kBwdPhaseFinal; break;
        case MEA_BWD_PREPROCESS: phases = mea::kBwdPhasePre; break;
        case MEA_BWD_MAIN: phases = mea::kBwdPhaseMain; break;
        case MEA_BWD_FINALIZE: phases = mea::kBwdPhaseFinal; break;
        default: return MEA_ERR_INVALID_ARG;
    }
    mea_status_t st = common_checks(B, H, Nq, Nk, D, scale, dtype);
    if (st != MEA_OK) return st;
    const int BH = B * H;
    if (BH == 0) return MEA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t esize = dtype == MEA_DTYPE_F32 ? 4 : 2;
    if (Nq == 0) {
        if (Nk == 0 || !(phases & mea::kBwdPhaseMain)) return MEA_OK;
        if (!dk || !dv) return MEA_ERR_INVALID_ARG;
        if (!aligned16(dk) || !aligned16(dv)) return MEA_ERR_MISALIGNED;
        const size_t n = (size_t)BH * Nk * D * esize;
        cudaError_t e = cudaMemsetAsync(dk, 0, n, s);
        if (e != cudaSuccess) return fail_cuda("cudaMemsetAsync", e);
        return cuda_status(cudaMemsetAsync(dv, 0, n, s), "cudaMemsetAsync");
    }
    if (Nk == 0) return MEA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return MEA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned4(lse))
        return MEA_ERR_MISALIGNED;
    size_t need = 0;
    if ((st = mea_attn_bwd_workspace_size(B, H, Nq, Nk, D, dtype, &need)) != MEA_OK) return st;
    if (workspace == nullptr || workspace_bytes < need) return MEA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MEA_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    if ((st = device_info(&dev)) != MEA_OK) return st;
    if (BH > 65535) return MEA_ERR_UNSUPPORTED;

    if (dtype == MEA_DTYPE_F32) {
        mea::F32BwdArgs f;
        f.q = static_cast<const float*>(q);
        f.k = static_cast<const float*>(k);
        f.v = static_cast<const float*>(v);
        f.o = static_cast<const float*>(o);
        f.dO = static_cast<const float*>(dO);
        f.lse = lse;
        f.dq = static_cast<float*>(dq);
        f.dk = static_cast<float*>(dk);
        f.dv = static_cast<float*>(dv);
        f.delta = static_cast<float*>(workspace);
        f.BH = BH;
        f.Nq = Nq;
        f.Nk = Nk;
        f.D = D;
        f.scale = scale;
        // Rows per CTA of 8 warps: fewer rows (more warps sharing one row's
        // loop) while the grid would leave SMs idle.
        auto rows_per_cta = [&](int rows) {
            int r = 8;
            while (r > 1 && (long long)BH * ((rows + r - 1) / r) < 2LL * dev->sm_count) r /= 2;
            return r;
        };
        f.q_rows_per_cta = rows_per_cta(Nq);
        f.k_rows_per_cta = rows_per_cta(Nk);
        return cuda_status(mea::launch_bwd_f32(f, s, phases), "bwd_f32 launch");
    }

    mea::Bf16BwdArgs a;
    if ((st = make_map(&a.tm_q, q, BH, Nq, D)) != MEA_OK) return st;
    if ((st = make_map(&a.tm_k, k, BH, Nk, D)) != MEA_OK) return st;
    if ((st = make_map(&a.tm_v, v, BH, Nk, D)) != MEA_OK) return st;
    if ((st = make_map(&a.tm_do, dO, BH, Nq, D)) != MEA_OK) return st;
    const size_t rows = (size_t)BH * Nq;
    a.o = static_cast<const uint16_t*>(o);
    a.dO = static_cast<const uint16_t*>(dO);
    a.lse = lse;
    a.dq = static_cast<uint16_t*>(dq);
    a.dk = static_cast<uint16_t*>(dk);
    a.dv = static_cast<uint16_t*>(dv);
    a.dq_acc = static_cast<float*>(workspace);
    if ((st = make_map_f32_acc(&a.tm_dq_acc, workspace, BH, Nq, D)) != MEA_OK) return st;
    a.delta = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round_up(rows * D * sizeof(float), 256));
    a.BH = BH;
    a.Nq = Nq;
    a.Nk = Nk;
    a.D = D;
    a.scale = scale;
    a.sm_count = dev->sm_count;
    return cuda_status(mea::launch_bwd_bf16(a, s, phases), "bwd_bf16 launch");
}

mea_status_t mea_attn_bwd_accum_workspace_size(int B, int H, int Nq, int Nk, int D, mea_dtype_t dtype,
                                               size_t* bytes) {
    if (bytes == nullptr) return MEA_ERR_INVALID_ARG;
    mea_status_t st = common_checks(B, H, Nq, Nk, D, 1.0f, dtype);
    if (st != MEA_OK) return st;
    *bytes = round_up((size_t)B * H * Nq * sizeof(float), 256);   // the row term D_i
    return MEA_OK;
}

mea_status_t mea_attn_bwd_accum(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                const void* dO, float* dq_acc, float* dk_acc, float* dv_acc, int B, int H, int Nq,
                                int Nk, int D, float scale, mea_dtype_t dtype, void* workspace,
                                size_t workspace_bytes, void* stream) {
    mea_status_t st = common_checks(B, H, Nq, Nk, D, scale, dtype);
    if (st != MEA_OK) return st;
    const int BH = B * H;
    if (BH == 0 || Nq == 0 || Nk == 0) return MEA_OK;   // an empty query or key range adds nothing
    if (!q || !k || !v || !o || !lse || !dO || !dq_acc || !dk_acc || !dv_acc) return MEA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(dq_acc) ||
        !aligned16(dk_acc) || !aligned16(dv_acc) || !aligned4(lse))
        return MEA_ERR_MISALIGNED;
    size_t need = 0;
    if ((st = mea_attn_bwd_accum_workspace_size(B, H, Nq, Nk, D, dtype, &need)) != MEA_OK) return st;
    if (workspace == nullptr || workspace_bytes < need) return MEA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MEA_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    if ((st = device_info(&dev)) != MEA_OK) return st;
    if (BH > 65535) return MEA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned phases = mea::kBwdPhasePre | mea::kBwdPhaseMain;
    if (dtype == MEA_DTYPE_F32) {
        mea::F32BwdArgs f;
        f.q = static_cast<const float*>(q);
        f.k = static_cast<const float*>(k);
        f.v = static_cast<const float*>(v);
        f.o = static_cast<const float*>(o);
        f.dO = static_cast<const float*>(dO);
        f.lse = lse;
        f.dq = dq_acc;
        f.dk = dk_acc;
        f.dv = dv_acc;
        f.delta = static_cast<float*>(workspace);
        f.BH = BH;
        f.Nq = Nq;
        f.Nk = Nk;
        f.D = D;
        f.scale = scale;
        f.accumulate = true;
        auto rows_per_cta = [&](int rows) {
            int r = 8;
            while (r > 1 && (long long)BH * ((rows + r - 1) / r) < 2LL * dev->sm_count) r /= 2;
            return r;
        };
        f.q_rows_per_cta = rows_per_cta(Nq);
        f.k_rows_per_cta = rows_per_cta(Nk);
        return cuda_status(mea::launch_bwd_f32(f, s, phases), "bwd_f32 accumulate launch");
    }
    mea::Bf16BwdArgs a;
    if ((st = make_map(&a.tm_q, q, BH, Nq, D)) != MEA_OK) return st;
    if ((st = make_map(&a.tm_k, k, BH, Nk, D)) != MEA_OK) return st;
    if ((st = make_map(&a.tm_v, v, BH, Nk, D)) != MEA_OK) return st;
    if ((st = make_map(&a.tm_do, dO, BH, Nq, D)) != MEA_OK) return st;
    // dS K goes straight into the caller's fp32 sum by the TMA reduce-adds
    if ((st = make_map_f32_acc(&a.tm_dq_acc, dq_acc, BH, Nq, D)) != MEA_OK) return st;
    a.o = static_cast<const uint16_t*>(o);
    a.dO = static_cast<const uint16_t*>(dO);
    a.lse = lse;
    a.dq = nullptr;
    a.dk = nullptr;
    a.dv = nullptr;
    a.dq_acc = nullptr;   // the preprocess phase leaves the caller's sum alone
    a.delta = static_cast<float*>(workspace);
    a.dk_acc = dk_acc;
    a.dv_acc = dv_acc;
    a.BH = BH;
    a.Nq = Nq;
    a.Nk = Nk;
    a.D = D;
    a.scale = scale;
    a.sm_count = dev->sm_count;
    return cuda_status(mea::launch_bwd_bf16(a, s, phases), "bwd_bf16 accumulate launch");
}

mea_status_t mea_attn_accum_convert(const float* acc, void* out, long long n, float mul, mea_dtype_t dtype,
                                    void* stream) {
    if (n < 0 || !std::isfinite(mul)) return MEA_ERR_INVALID_ARG;
    if (dtype != MEA_DTYPE_F32 && dtype != MEA_DTYPE_BF16) return MEA_ERR_UNSUPPORTED;
    if (n == 0) return MEA_OK;
    if (n % 4 != 0) return fail(MEA_ERR_UNSUPPORTED, "mea_attn_accum_convert", "n must be a multiple of 4");
    if (!acc || !out) return MEA_ERR_INVALID_ARG;
    if (!aligned16(acc) || !aligned16(out)) return MEA_ERR_MISALIGNED;
    return cuda_status(mea::launch_accum_convert(acc, out, n, mul, dtype == MEA_DTYPE_BF16,
                                                 static_cast<cudaStream_t>(stream)),
                       "accum_convert launch");
}

mea_status_t mea_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dO, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int D,
                          float scale, mea_dtype_t dtype, void* workspace, size_t workspace_bytes, void* stream) {
    return mea_attn_bwd_phase(MEA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, B, H, Nq, Nk, D, scale, dtype,
                              workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// Shared key/value heads.  The G = H / H_kv query heads of one group are
// consecutive in [B, H, Nq, D], so they are one contiguous [G*Nq, D] block:
// the group is a single "head" of G*Nq query rows over its key/value head,
// and the kernels above run unchanged over B*H_kv such heads.  lse, the dQ
// accumulator and the row term D_i follow the same [B*H_kv, G*Nq] view.
}  // extern "C"

namespace {
mea_status_t gqa_rows(int H, int H_kv, int Nq, int* rows) {
    if (H < 0 || H_kv < 1 || Nq < 0 || H % H_kv != 0)
        return fail(MEA_ERR_INVALID_ARG, "gqa", "H must be a multiple of H_kv >= 1");
    const long long r = (long long)(H / H_kv) * Nq;
    if (r > 0x7fffffffLL) return fail(MEA_ERR_UNSUPPORTED, "gqa", "(H / H_kv) * Nq exceeds 2^31-1");
    *rows = (int)r;
    return MEA_OK;
}
}  // namespace

extern "C" {

mea_status_t mea_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                              int H_kv, int Nq, int Nk, int D, float scale, mea_dtype_t dtype, void* stream) {
    int rows = 0;
    mea_status_t st = gqa_rows(H, H_kv, Nq, &rows);
    if (st != MEA_OK) return st;
    return mea_attn_fwd(q, k, v, o, lse, B, H_kv, rows, Nk, D, scale, dtype, stream);
}

mea_status_t mea_attn_decode_workspace_size(int B, int H, int H_kv, int Nq, int Nk, int D, mea_dtype_t dtype,
                                          size_t* bytes) {
    if (bytes == nullptr) return MEA_ERR_INVALID_ARG;
    int rows = 0;
    mea_status_t st = gqa_rows(H, H_kv, Nq, &rows);
    if (st != MEA_OK) return st;
    if ((st = common_checks(B, H_kv, rows, Nk, D, 1.0f, dtype)) != MEA_OK) return st;
    *bytes = 0;
    const bool bf16 = dtype == MEA_DTYPE_BF16;
    if ((long long)B * H_kv * rows == 0 || Nk == 0 || !mea::decode_supported(bf16, D, rows)) return MEA_OK;
    DeviceInfo* dev = nullptr;
    if ((st = device_info(&dev)) != MEA_OK) return st;
    *bytes = decode_plan(dev, (long long)B * H_kv, rows, Nk, D, bf16).ws_bytes;
    return MEA_OK;
}

mea_status_t mea_attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                             int H_kv, int Nq, int Nk, int D, float scale, mea_dtype_t dtype, void* workspace,
                             size_t workspace_bytes, void* stream) {
    int rows = 0;
    mea_status_t st = gqa_rows(H, H_kv, Nq, &rows);
    if (st != MEA_OK) return st;
    const bool bf16 = dtype == MEA_DTYPE_BF16;
    if (dtype != MEA_DTYPE_F32 && dtype != MEA_DTYPE_BF16) return MEA_ERR_INVALID_ARG;
    if (!mea::decode_supported(bf16, D, rows))   // many rows per head: the tensor-core / fp32 forward
        return mea_attn_fwd(q, k, v, o, lse, B, H_kv, rows, Nk, D, scale, dtype, stream);
    if ((st = common_checks(B, H_kv, rows, Nk, D, scale, dtype)) != MEA_OK) return st;
    const long long BHkv = (long long)B * H_kv;
    if (BHkv * rows == 0) return MEA_OK;
    if (Nk == 0) return MEA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !lse) return MEA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return MEA_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    if ((st = device_info(&dev)) != MEA_OK) return st;
    const DecodePlan p = decode_plan(dev, BHkv, rows, Nk, D, bf16);
    if (p.nsplit > 1) {
        if (workspace == nullptr || workspace_bytes < p.ws_bytes)
            return fail(MEA_ERR_WORKSPACE, "mea_attn_decode", "workspace missing or below mea_attn_decode_workspace_size");
        if (!aligned16(workspace)) return MEA_ERR_MISALIGNED;
    }
    return launch_decode_plan(q, k, v, o, lse, BHkv, rows, Nk, D, scale, bf16, p, workspace,
                              static_cast<cudaStream_t>(stream));
}

mea_status_t mea_attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                              int H_kv, int Nq, int Nk, int D, float scale, float q_descale, float k_descale,
                              void* stream) {
    int rows = 0;
    mea_status_t st = gqa_rows(H, H_kv, Nq, &rows);
    if (st != MEA_OK) return st;
    if (!std::isfinite(q_descale) || !std::isfinite(k_descale) || !(q_descale > 0.f) || !(k_descale > 0.f))
        return fail(MEA_ERR_INVALID_ARG, "mea_attn_fwd_fp8", "descale factors must be finite and positive");
    if ((st = common_checks(B, H_kv, rows, Nk, D, scale, MEA_DTYPE_BF16)) != MEA_OK) return st;
    if (D != 128) return fail(MEA_ERR_UNSUPPORTED, "mea_attn_fwd_fp8", "head dim 128 only");
    if ((long long)B * H_kv * rows == 0) return MEA_OK;
    if (Nk == 0) return MEA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !lse) return MEA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return MEA_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    if ((st = device_info(&dev)) != MEA_OK) return st;
    // the product of e4m3 values is exact in the fp32 accumulator, so the
    // descale factors fold into the softmax scale
    const float eff = scale * q_descale * k_descale;
    if (!std::isfinite(eff)) return MEA_ERR_INVALID_ARG;
    return tc_forward(q, k, v, o, lse, B * H_kv, rows, Nk, D, eff, true, dev, static_cast<cudaStream_t>(stream));
}

mea_status_t mea_attn_combine(const void* const* o_parts, const float* const* lse_parts, int R, void* o,
                              float* lse, int B, int H, int Nq, int D, mea_dtype_t dtype, void* stream) {
    if (dtype != MEA_DTYPE_F32 && dtype != MEA_DTYPE_BF16) return MEA_ERR_INVALID_ARG;
    if (R < 1 || R > mea::kCombineMaxParts)
        return fail(MEA_ERR_UNSUPPORTED, "mea_attn_combine", "1 to 16 parts");
    if (B < 0 || H < 0 || Nq < 0 || D <= 0) return MEA_ERR_INVALID_ARG;
    if (D % 8 != 0 || D > 256) return fail(MEA_ERR_UNSUPPORTED, "mea_attn_combine", "D a multiple of 8, at most 256");
    const long long rows = (long long)B * H * Nq;
    if (rows * D >= (1LL << 40)) return MEA_ERR_INVALID_ARG;
    if (rows == 0) return MEA_OK;
    if (!o_parts || !lse_parts || !o || !lse) return MEA_ERR_INVALID_ARG;
    mea::CombineArgs a;
    for (int r = 0; r < R; ++r) {
        if (!o_parts[r] || !lse_parts[r]) return MEA_ERR_INVALID_ARG;
        if (!aligned16(o_parts[r]) || !aligned4(lse_parts[r])) return MEA_ERR_MISALIGNED;
        a.o_parts[r] = o_parts[r];
        a.lse_parts[r] = lse_parts[r];
    }
    for (int r = R; r < mea::kCombineMaxParts; ++r) {
        a.o_parts[r] = nullptr;
        a.lse_parts[r] = nullptr;
    }
    if (!aligned16(o) || !aligned4(lse)) return MEA_ERR_MISALIGNED;
    a.o = o;
    a.lse = lse;
    a.rows = rows;
    a.D = D;
    a.R = R;
    DeviceInfo* dev = nullptr;
    mea_status_t st = device_info(&dev);
    if (st != MEA_OK) return st;
    return cuda_status(mea::launch_combine(a, dtype == MEA_DTYPE_BF16, static_cast<cudaStream_t>(stream)),
                       "combine launch");
}

mea_status_t mea_attn_bwd_gqa_workspace_size(int B, int H, int H_kv, int Nq, int Nk, int D, mea_dtype_t dtype,
                                             size_t* bytes) {
    int rows = 0;
    mea_status_t st = gqa_rows(H, H_kv, Nq, &rows);
    if (st != MEA_OK) return st;
    return mea_attn_bwd_workspace_size(B, H_kv, rows, Nk, D, dtype, bytes);
}

mea_status_t mea_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dO, void* dq, void* dk, void* dv, int B, int H, int H_kv, int Nq, int Nk,
                              int D, float scale, mea_dtype_t dtype, void* workspace, size_t workspace_bytes,
                              void* stream) {
    int rows = 0;
    mea_status_t st = gqa_rows(H, H_kv, Nq, &rows);
    if (st != MEA_OK) return st;
    return mea_attn_bwd_phase(MEA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, B, H_kv, rows, Nk, D, scale, dtype,
                              workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// Backward without any allocation, for callers that cannot allocate device
// memory (see mea_attn_bwd_noalloc in mea_attn.h).  The scratch lives in one
// file-scope device array that every device loading this library keeps until
// the process exits; host code may only use its address as returned by
// cudaGetSymbolAddress, never the array's name.
}  // extern "C"

namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)MEA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
// The array's device address, resolved once per device and remembered with
// the unique id of the context it was resolved in: a device reset (or any new
// context) loads the module again, possibly elsewhere, so a changed id means
// the address is resolved anew instead of handing a freed address to a kernel.
struct NoAllocScratch {
    void* ptr = nullptr;
    unsigned long long ctx_id = 0;
};
NoAllocScratch g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Id of the context current on this thread, 0 if none is current yet.
mea_status_t current_context_id(unsigned long long* id) {
    *id = 0;
    if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || f1 == nullptr ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess || f2 == nullptr)
            return fail(MEA_ERR_CUDA, "cudaGetDriverEntryPoint", "cuCtxGetCurrent/cuCtxGetId unavailable");
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return fail(MEA_ERR_CUDA, "cuCtxGetCurrent", "failed");
    if (ctx != nullptr && g_ctx_get_id(ctx, id) != CUDA_SUCCESS) return fail(MEA_ERR_CUDA, "cuCtxGetId", "failed");
    return MEA_OK;
}
}  // namespace

extern "C" {

mea_status_t mea_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                  const void* dO, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int D,
                                  float scale, mea_dtype_t dtype, void* stream) {
    mea_status_t st = common_checks(B, H, Nq, Nk, D, scale, dtype);
    if (st != MEA_OK) return st;
    if (dtype != MEA_DTYPE_BF16) return MEA_ERR_UNSUPPORTED;
    size_t need = 0;
    if ((st = mea_attn_bwd_workspace_size(B, H, Nq, Nk, D, dtype, &need)) != MEA_OK) return st;
    if (need > kNoAllocScratchBytes) {
        char buf[160];
        std::snprintf(buf, sizeof(buf), "these sizes need %zu bytes of scratch; the static scratch holds %zu bytes",
                      need, kNoAllocScratchBytes);
        return fail(MEA_ERR_WORKSPACE, "mea_attn_bwd_noalloc", buf);
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return MEA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    {
        // Set-up once per device (and again only if the device's context was
        // replaced), with that device current: resolve the device address of
        // the static scratch array.  Host code never passes the array's name.
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        unsigned long long ctx_id = 0;
        if ((st = current_context_id(&ctx_id)) != MEA_OK) return st;
        NoAllocScratch& s = g_noalloc[dev];
        if (s.ptr == nullptr || ctx_id == 0 || ctx_id != s.ctx_id) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the device's context current
            if (e != cudaSuccess || p == nullptr) return fail_cuda("cudaGetSymbolAddress(scratch)", e);
            if ((st = current_context_id(&ctx_id)) != MEA_OK) return st;
            s.ptr = p;
            s.ctx_id = ctx_id;
        }
        scratch = s.ptr;
    }
    // The preprocess phase re-zeroes the dQ accumulator and rewrites the row
    // term on every call, so nothing left by an earlier call is read.
    return mea_attn_bwd_phase(MEA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, B, H, Nq, Nk, D, scale, dtype, scratch,
                              kNoAllocScratchBytes, stream);
}

mea_status_t mea_selftest_bounded_wait(int* gave_up, void* stream) {
    if (gave_up == nullptr) return MEA_ERR_INVALID_ARG;
    if (!aligned4(gave_up)) return MEA_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    mea_status_t st = device_info(&dev);
    if (st != MEA_OK) return st;
    mea::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(gave_up);
    return cuda_status(cudaGetLastError(), "selftest launch");
}

mea_status_t mea_last_device_error(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda("cudaStreamSynchronize", e);
    unsigned int flag = 0;
    if (cudaMemcpyFromSymbol(&flag, mea::g_device_error, sizeof(flag)) != cudaSuccess) return MEA_ERR_CUDA;
    if (flag == 0) return MEA_OK;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(mea::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return MEA_ERR_CUDA;
    return (flag & 1u) ? MEA_ERR_TIMEOUT : MEA_ERR_CUDA;
}

}  // extern "C"
