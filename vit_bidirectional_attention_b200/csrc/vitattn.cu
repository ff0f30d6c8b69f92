// vitattn.cu -- host side of libvitattn: argument checks, TMA tensor-map
// encoding, kernel dispatch by padded head dimension and dtype, and the
// extern "C" entry points declared in include/vitattn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "vitattn.h"

#include "fwd_kernel.cuh"
#include "norm_rope_kernel.cuh"
#include "rope_kernel.cuh"

namespace {

using vitattn::FwdParams;
using SegDense = vitattn::SegTable<false>;
using SegVar = vitattn::SegTable<true>;
static_assert(vitattn::kMaxSegs == VITATTN_MAX_SEQS, "segment table size");

constexpr int kVersion = 10000;  // 1.0.0
constexpr int kMaxDevices = 64;
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s per in-kernel wait

thread_local int t_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return VITATTN_ERR_CUDA;
}

bool overlaps(const void* a, const void* b, uint64_t bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

// [a, a + la) and [b, b + lb) share a byte.
bool overlaps2(const void* a, uint64_t la, const void* b, uint64_t lb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + lb && y < x + la;
}

int check_args(const void* q, const void* k, const void* v, const void* out, int64_t B, int64_t N,
               int64_t H, int64_t D, float scale, int dtype) {
    if (!q || !k || !v || !out) return VITATTN_ERR_NULL;
    if (B < 1 || N < 1 || H < 1 || D < 1) return VITATTN_ERR_DIM;
    if (D < 16 || D > 128 || D % 8 != 0) return VITATTN_ERR_HEADDIM;
    if (dtype != VITATTN_BF16 && dtype != VITATTN_F16) return VITATTN_ERR_DTYPE;
    if (!std::isfinite(scale)) return VITATTN_ERR_SCALE;
    // sizes: TMA coordinates are int32, the per-batch stride must stay below 2^40 bytes,
    // and the grid is one CTA per (b, h, 256 query rows)
    if (N > (int64_t)INT32_MAX - 512 || H > (int64_t)INT32_MAX || B > (int64_t)INT32_MAX)
        return VITATTN_ERR_DIM;
    const uint64_t batch_stride = (uint64_t)N * (uint64_t)H * (uint64_t)D * 2u;
    if (batch_stride >= (1ull << 40)) return VITATTN_ERR_DIM;
    if ((uint64_t)B > (1ull << 62) / batch_stride) return VITATTN_ERR_DIM;
    const uint64_t work = (uint64_t)B * (uint64_t)H * (uint64_t)((N + 255) / 256);
    if (work > (uint64_t)INT32_MAX) return VITATTN_ERR_DIM;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                           reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out)) & 15u;
    if (mis) return VITATTN_ERR_ALIGN;
    const uint64_t bytes = batch_stride * (uint64_t)B;
    if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes))
        return VITATTN_ERR_ALIAS;
    return VITATTN_OK;
}

// Cross lengths: q, out [B, Lq, H, D]; k, v [B, Lk, H, D]; lse (optional) [B, H, Lq] f32.
int check_args_ext(const void* q, const void* k, const void* v, const void* out, const float* lse, int64_t B,
                   int64_t Lq, int64_t Lk, int64_t H, int64_t D, float scale, int dtype) {
    if (!q || !k || !v || !out) return VITATTN_ERR_NULL;
    if (Lk < 1) return VITATTN_ERR_DIM;
    // the query side and every shape limit as for self-attention of length Lq, then the key side
    int rc = check_args(q, q, q, out, B, Lq, H, D, scale, dtype);
    if (rc) return rc;
    rc = check_args(k, k, k, k, B, Lk, H, D, scale, dtype);
    if (rc && rc != VITATTN_ERR_ALIAS) return rc;  // k "aliasing" itself is the stand-in, not an error
    if ((reinterpret_cast<uintptr_t>(v) & 15u) || (reinterpret_cast<uintptr_t>(lse) & 15u)) return VITATTN_ERR_ALIGN;
    const uint64_t q_bytes = (uint64_t)B * (uint64_t)Lq * (uint64_t)H * (uint64_t)D * 2u;
    const uint64_t kv_bytes = (uint64_t)B * (uint64_t)Lk * (uint64_t)H * (uint64_t)D * 2u;
    if (overlaps2(out, q_bytes, k, kv_bytes) || overlaps2(out, q_bytes, v, kv_bytes)) return VITATTN_ERR_ALIAS;
    if (lse) {
        const uint64_t lse_bytes = (uint64_t)B * (uint64_t)H * (uint64_t)Lq * 4u;
        if (overlaps2(lse, lse_bytes, out, q_bytes) || overlaps2(lse, lse_bytes, q, q_bytes) ||
            overlaps2(lse, lse_bytes, k, kv_bytes) || overlaps2(lse, lse_bytes, v, kv_bytes))
            return VITATTN_ERR_ALIAS;
    }
    return VITATTN_OK;
}

// Grouped-query attention: q, out [B, N, H, D]; k, v [B, N, Hkv, D], H a multiple of Hkv.
int check_args_gqa(const void* q, const void* k, const void* v, const void* out, int64_t B, int64_t N,
                   int64_t H, int64_t Hkv, int64_t D, float scale, int dtype) {
    if (Hkv < 1 || H < 1 || H % Hkv != 0) return (!q || !k || !v || !out) ? VITATTN_ERR_NULL : VITATTN_ERR_DIM;
    // the query side (and every shape limit) as for multi-head attention, with k, v
    // standing in at the query's size only for the pointer checks
    int rc = check_args(q, q, q, out, B, N, H, D, scale, dtype);
    if (rc) return rc;
    if (!k || !v) return VITATTN_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15u) return VITATTN_ERR_ALIGN;
    const uint64_t out_bytes = (uint64_t)B * (uint64_t)N * (uint64_t)H * (uint64_t)D * 2u;
    const uint64_t kv_bytes = (uint64_t)B * (uint64_t)N * (uint64_t)Hkv * (uint64_t)D * 2u;
    if (overlaps2(out, out_bytes, k, kv_bytes) || overlaps2(out, out_bytes, v, kv_bytes)) return VITATTN_ERR_ALIAS;
    return VITATTN_OK;
}

// Token-strided inputs: element (b, i, h, d) of x at x + ((b*N + i)*ts_x + h*D + d)
// for x = q, k, v (ts_x elements between consecutive tokens, >= H*D, a multiple
// of 8 so that every token row starts on 16 bytes); out dense [B, N, H, D], or
// (internally, for head groups of the host-buffer entry) token-strided by
// out_ts likewise.  The inputs may overlap one another (views of one packed
// projection); out must not overlap any of them.
int check_args_strided(const void* q, const void* k, const void* v, const void* out, int64_t B, int64_t N,
                       int64_t H, int64_t D, const int64_t ts[3], float scale, int dtype, int64_t out_ts = 0) {
    if (!q || !k || !v || !out) return VITATTN_ERR_NULL;
    if (B < 1 || N < 1 || H < 1 || D < 1) return VITATTN_ERR_DIM;
    if (D < 16 || D > 128 || D % 8 != 0) return VITATTN_ERR_HEADDIM;
    if (dtype != VITATTN_BF16 && dtype != VITATTN_F16) return VITATTN_ERR_DTYPE;
    if (!std::isfinite(scale)) return VITATTN_ERR_SCALE;
    if (N > (int64_t)INT32_MAX - 512 || H > (int64_t)INT32_MAX || B > (int64_t)INT32_MAX) return VITATTN_ERR_DIM;
    const uint64_t row = (uint64_t)H * (uint64_t)D;  // elements of one token's heads
    if (row * 2u >= (1ull << 40)) return VITATTN_ERR_DIM;
    const uint64_t out_bytes_batch = (uint64_t)N * row * 2u;
    if (out_bytes_batch >= (1ull << 40) || (uint64_t)B > (1ull << 62) / out_bytes_batch) return VITATTN_ERR_DIM;
    const uint64_t work = (uint64_t)B * (uint64_t)H * (uint64_t)((N + 255) / 256);
    if (work > (uint64_t)INT32_MAX) return VITATTN_ERR_DIM;
    uint64_t extent[3];
    for (int i = 0; i < 3; ++i) {
        if (ts[i] < (int64_t)row || ts[i] % 8 != 0) return VITATTN_ERR_DIM;
        const uint64_t batch = (uint64_t)N * (uint64_t)ts[i] * 2u;  // bytes between batches (a TMA stride)
        if (batch >= (1ull << 40) || (uint64_t)B > (1ull << 62) / batch) return VITATTN_ERR_DIM;
        extent[i] = ((uint64_t)B * (uint64_t)N - 1u) * (uint64_t)ts[i] * 2u + row * 2u;
    }
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                           reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out)) & 15u;
    if (mis) return VITATTN_ERR_ALIGN;
    if (out_ts != 0 && (out_ts < (int64_t)row || out_ts % 8 != 0 ||
                        (uint64_t)N * (uint64_t)out_ts * 2u >= (1ull << 40)))
        return VITATTN_ERR_DIM;
    const uint64_t out_bytes = out_ts == 0 ? out_bytes_batch * (uint64_t)B
                                           : ((uint64_t)B * (uint64_t)N - 1u) * (uint64_t)out_ts * 2u + row * 2u;
    if (overlaps2(out, out_bytes, q, extent[0]) || overlaps2(out, out_bytes, k, extent[1]) ||
        overlaps2(out, out_bytes, v, extent[2]))
        return VITATTN_ERR_ALIAS;
    return VITATTN_OK;
}

// Ragged batch: q, k, v, out are [total, H, D] with total = cu_seqlens[num_seqs];
// cu_seqlens (host) starts at 0 and never decreases.
int check_args_varlen(const void* q, const void* k, const void* v, const void* out,
                      const int32_t* cu_seqlens, int64_t num_seqs, int64_t H, int64_t D, float scale,
                      int dtype) {
    if (!q || !k || !v || !out || !cu_seqlens) return VITATTN_ERR_NULL;
    if (num_seqs < 1 || num_seqs > vitattn::kMaxSegs || H < 1 || D < 1) return VITATTN_ERR_DIM;
    if (D < 16 || D > 128 || D % 8 != 0) return VITATTN_ERR_HEADDIM;
    if (dtype != VITATTN_BF16 && dtype != VITATTN_F16) return VITATTN_ERR_DTYPE;
    if (!std::isfinite(scale)) return VITATTN_ERR_SCALE;
    if (cu_seqlens[0] != 0) return VITATTN_ERR_SEQLENS;
    for (int64_t s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return VITATTN_ERR_SEQLENS;
    const int64_t total = cu_seqlens[num_seqs];
    // TMA token coordinates and per-item token offsets are int32
    if (total > (int64_t)INT32_MAX - 512 || H > (int64_t)INT32_MAX) return VITATTN_ERR_DIM;
    const uint64_t token_bytes = (uint64_t)H * (uint64_t)D * 2u;
    if (token_bytes >= (1ull << 40) || (uint64_t)total > (1ull << 62) / token_bytes) return VITATTN_ERR_DIM;
    uint64_t work = 0;
    for (int64_t s = 0; s < num_seqs; ++s)
        work += (uint64_t)H * (uint64_t)((cu_seqlens[s + 1] - cu_seqlens[s] + 127) / 128);
    if (work > (uint64_t)INT32_MAX) return VITATTN_ERR_DIM;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                           reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out)) & 15u;
    if (mis) return VITATTN_ERR_ALIGN;
    const uint64_t bytes = token_bytes * (uint64_t)total;
    if (bytes > 0 && (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes)))
        return VITATTN_ERR_ALIAS;
    return VITATTN_OK;
}

// QKV split + rope prologue: qkv [T, 3, H, D], cos/sin [T, D] f32, q/k/v [T, H, D].
// need_v = false: the q/k-only prologue (v stays in qkv), v is not an output.
int check_args_rope(const void* qkv, const float* cs, const float* sn, const void* q, const void* k,
                    const void* v, int64_t T, int64_t H, int64_t D, int dtype, bool need_v = true) {
    if (!qkv || !cs || !sn || !q || !k || (need_v && !v)) return VITATTN_ERR_NULL;
    if (!need_v) v = q;  // stands in for the absent output in the checks below
    if (T < 1 || H < 1 || D < 1) return VITATTN_ERR_DIM;
    if (D < 16 || D > 128 || D % 8 != 0) return VITATTN_ERR_HEADDIM;
    if (dtype != VITATTN_BF16 && dtype != VITATTN_F16) return VITATTN_ERR_DTYPE;
    if (H > (int64_t)INT32_MAX || T > (int64_t)1 << 40) return VITATTN_ERR_DIM;
    const uint64_t row_bytes = (uint64_t)H * (uint64_t)D * 2u;
    if (row_bytes >= (1ull << 40) || (uint64_t)T > (1ull << 60) / (3u * row_bytes)) return VITATTN_ERR_DIM;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(cs) |
                           reinterpret_cast<uintptr_t>(sn) | reinterpret_cast<uintptr_t>(q) |
                           reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15u;
    if (mis) return VITATTN_ERR_ALIGN;
    const uint64_t in_bytes = 3u * row_bytes * (uint64_t)T, out_bytes = row_bytes * (uint64_t)T;
    const uint64_t tab_bytes = (uint64_t)T * (uint64_t)D * 4u;
    const void* outs[3] = {q, k, v};
    const int nout = need_v ? 3 : 2;
    for (int i = 0; i < nout; ++i) {
        if (overlaps2(outs[i], out_bytes, qkv, in_bytes) || overlaps2(outs[i], out_bytes, cs, tab_bytes) ||
            overlaps2(outs[i], out_bytes, sn, tab_bytes))
            return VITATTN_ERR_ALIAS;
        for (int j = 0; j < i; ++j)
            if (overlaps(outs[i], outs[j], out_bytes)) return VITATTN_ERR_ALIAS;
    }
    return VITATTN_OK;
}

// The prologue with q/k RMS norm: the rope checks, plus two [D] f32 weight
// vectors (16-byte aligned, not overlapping an output) and a finite eps >= 0.
int check_args_norm_rope(const void* qkv, const float* cs, const float* sn, const float* qw, const float* kw,
                         float eps, const void* q, const void* k, const void* v, int64_t T, int64_t H,
                         int64_t D, int dtype, bool need_v = true) {
    int rc = check_args_rope(qkv, cs, sn, q, k, v, T, H, D, dtype, need_v);
    if (rc) return rc;
    if (!need_v) v = q;
    if (!qw || !kw) return VITATTN_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(qw) | reinterpret_cast<uintptr_t>(kw)) & 15u) return VITATTN_ERR_ALIGN;
    if (!std::isfinite(eps) || eps < 0.f) return VITATTN_ERR_SCALE;
    const uint64_t out_bytes = (uint64_t)H * (uint64_t)D * 2u * (uint64_t)T, w_bytes = (uint64_t)D * 4u;
    const void* outs[3] = {q, k, v};
    for (int i = 0; i < 3; ++i)
        if (overlaps2(outs[i], out_bytes, qw, w_bytes) || overlaps2(outs[i], out_bytes, kw, w_bytes))
            return VITATTN_ERR_ALIAS;
    return VITATTN_OK;
}

// ---------------------------------------------------------------- driver entry point

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Token-major [B, N, H, D] seen by TMA as 4-D {D, H, N, B} (innermost first);
// one box is `width` head-dim columns x 1 head x 128 tokens x 1 batch.
// `ts` is the element stride between consecutive tokens (H*D when dense).
bool encode_map(CUtensorMap* m, const void* ptr, int dtype, int64_t B, int64_t N, int64_t H,
                int64_t D, int width, int64_t ts) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)(D * 2), (cuuint64_t)(ts * 2), (cuuint64_t)(N * ts * 2)};
    const cuuint32_t box[4] = {(cuuint32_t)width, 1u, (cuuint32_t)vitattn::kTileRows, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUtensorMapSwizzle sw = width == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : width == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_32B;
    const CUtensorMapDataType dt =
        dtype == VITATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(m, dt, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- dispatch

// Kernel modes: one work item per CTA, CTAs looping over items, ragged batch,
// one split item (a query tile's key blocks in two halves) per CTA.
enum Mode { kModeItem = 0, kModeLoop = 1, kModeVarlen = 2, kModeSplit = 3, kNumModes = 4 };

template <int DP>
const void* kernel_of(bool bf, Mode mode) {
    switch (mode) {
        case kModeLoop:
            return bf ? reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, true, true, false>)
                      : reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, false, true, false>);
        case kModeVarlen:
            return bf ? reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, true, false, true>)
                      : reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, false, false, true>);
        case kModeSplit:
            return bf ? reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, true, false, false, true>)
                      : reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, false, false, false, true>);
        default:
            return bf ? reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, true, false, false>)
                      : reinterpret_cast<const void*>(vitattn::fwd_kernel<DP, false, false, false>);
    }
}

const void* pick_kernel(int dp, int dtype, Mode mode) {
    const bool bf = dtype == VITATTN_BF16;
    switch (dp) {
        case 16: return kernel_of<16>(bf, mode);
        case 32: return kernel_of<32>(bf, mode);
        case 48: return kernel_of<48>(bf, mode);
        case 64: return kernel_of<64>(bf, mode);
        case 80: return kernel_of<80>(bf, mode);
        case 96: return kernel_of<96>(bf, mode);
        case 112: return kernel_of<112>(bf, mode);
        case 128: return kernel_of<128>(bf, mode);
        default: return nullptr;
    }
}

// Per device: architecture verified once; per kernel instantiation: the
// dynamic shared-memory limit raised once.
struct DeviceState {
    bool checked = false;
    bool is_sm100 = false;
    int num_sms = 0;
    bool smem_set[9][2][kNumModes] = {};
};
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Architecture check and SM count, once per device.
int device_info(int* num_sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return VITATTN_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& st = g_dev[dev];
    if (!st.checked) {
        int major = 0, minor = 0;
        e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        st.is_sm100 = (major == 10 && minor == 0);
        e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        st.checked = true;
    }
    if (!st.is_sm100) return VITATTN_ERR_DEVICE;
    *num_sms = st.num_sms;
    return VITATTN_OK;
}

// Every pointer must address memory that the current device's kernels may
// read and write: its own device memory, managed memory, or pinned host
// memory mapped for it.  Plain (unregistered) host memory or another GPU's
// memory would be encoded into a tensor map and fault or be read across
// devices, so the call is refused before anything is enqueued.
int check_device_ptrs(std::initializer_list<const void*> ptrs) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    for (const void* ptr : ptrs) {
        if (!ptr) continue;
        cudaPointerAttributes a;
        e = cudaPointerGetAttributes(&a, ptr);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();  // clear the sticky-free error of the query
            return VITATTN_ERR_DEVICE;
        }
        if (a.type == cudaMemoryTypeUnregistered) return VITATTN_ERR_DEVICE;
        if (a.type == cudaMemoryTypeDevice && a.device != dev) return VITATTN_ERR_DEVICE;
        if (a.type == cudaMemoryTypeHost && a.devicePointer == nullptr) return VITATTN_ERR_DEVICE;
    }
    return VITATTN_OK;
}

// The dynamic shared-memory limit of one kernel instantiation, raised once per device.
int ensure_smem(int dp, int dtype, Mode mode, const void* fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    std::lock_guard<std::mutex> lock(g_mu);
    bool& done = g_dev[dev].smem_set[dp / 16][dtype][mode];
    if (!done) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 vitattn::smem_bytes(dp, mode == kModeLoop, mode == kModeSplit));
        if (e != cudaSuccess) return cuda_fail(e);
        done = true;
    }
    return VITATTN_OK;
}

// Tensor maps of q, k, v for every column-chunk width, and the shape fields.
// ts: token strides of q, k, v in elements (nullptr: dense, heads * D).
int fill_common(FwdParams* prm, const void* q, const void* k, const void* v, void* out, int64_t B,
                int64_t N, int64_t H, int64_t D, float scale, int dtype, int flags, int64_t Hkv = 0,
                int64_t Nk = 0, const int64_t* ts = nullptr) {
    std::memset(prm, 0, sizeof *prm);
    if (Hkv == 0) Hkv = H;  // multi-head: k and v have the query's head count
    if (Nk == 0) Nk = N;    // self-attention: as many keys as queries
    const int dp = (int)((D + 15) / 16 * 16);
    const void* src[3] = {q, k, v};
    const int64_t heads[3] = {H, Hkv, Hkv};
    const int64_t lens[3] = {N, Nk, Nk};
    const int nch = vitattn::chunk_count(dp);
    for (int c = 0; c < nch; ++c) {
        const int w = vitattn::chunk_width(dp, c);
        for (int m = 0; m < 3; ++m) {
            CUtensorMap* map = &prm->maps[m][vitattn::width_class(w)];
            const int64_t stride = ts ? ts[m] : heads[m] * D;
            if (!encode_map(map, src[m], dtype, B, lens[m], heads[m], D, w, stride))
                return cuda_fail(cudaErrorInvalidValue);
        }
    }
    prm->kv_group = (int)(H / Hkv);
    prm->Nk = (int)Nk;
    prm->out = out;
    prm->out_ts = (long long)(H * D);
    prm->B = (int)B;
    prm->N = (int)N;
    prm->H = (int)H;
    prm->D = (int)D;
    prm->scale_log2 = (float)((double)scale * 1.4426950408889634);
    prm->flags = flags;
    prm->timeout_ns = kWaitTimeoutNs;
    return VITATTN_OK;
}

template <class Seg>
int run_kernel(int dp, int dtype, Mode mode, unsigned grid, FwdParams* prm, Seg* seg,
               cudaStream_t stream) {
    const void* fn = pick_kernel(dp, dtype, mode);
    if (!fn) return VITATTN_ERR_HEADDIM;
    int rc = ensure_smem(dp, dtype, mode, fn);
    if (rc) return rc;
    void* args[2] = {prm, seg};
    cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(vitattn::kThreads), args,
                                     (size_t)vitattn::smem_bytes(dp, mode == kModeLoop, mode == kModeSplit), stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return VITATTN_OK;
}

// Cross-length / causal / LSE extras of the dense launch (all off by default).
struct Ext {
    int64_t Nk = 0;       // keys per (b, h); 0: N
    int causal = 0;       // aligned causal mask
    float* lse = nullptr; // optional [B, H, N] log-sum-exp output
    const int64_t* ts = nullptr;  // token strides of q, k, v in elements; nullptr: dense
    int64_t out_ts = 0;           // token stride of out in elements (with ts only); 0: dense
};

int launch(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N,
           int64_t H, int64_t D, float scale, int dtype, cudaStream_t stream, int flags, int64_t Hkv = 0,
           const Ext& ext = Ext()) {
    int rc = ext.ts   ? check_args_strided(q, k, v, out, B, N, H, D, ext.ts, scale, dtype, ext.out_ts)
             : ext.Nk ? check_args_ext(q, k, v, out, ext.lse, B, N, ext.Nk, H, D, scale, dtype)
             : Hkv    ? check_args_gqa(q, k, v, out, B, N, H, Hkv, D, scale, dtype)
                      : check_args(q, k, v, out, B, N, H, D, scale, dtype);
    if (rc) return rc;
    const int64_t Nk = ext.Nk ? ext.Nk : N;
    const int dp = (int)((D + 15) / 16 * 16);
    int num_sms = 0;
    rc = device_info(&num_sms);
    if (rc) return rc;
    rc = check_device_ptrs({q, k, v, out, ext.lse});
    if (rc) return rc;

    FwdParams prm;
    rc = fill_common(&prm, q, k, v, out, B, N, H, D, scale, dtype, flags, Hkv, Nk, ext.ts);
    if (rc) return rc;
    if (ext.out_ts) prm.out_ts = (long long)ext.out_ts;
    prm.causal = ext.causal ? 1 : 0;
    prm.causal_off = (int)(Nk - N);
    prm.lse = ext.lse;
    // Two query tiles per CTA share each K/V block (fewer K/V reads, two
    // softmax warpgroups in flight); one per CTA when two would leave SMs idle.
    const uint64_t pairs = (uint64_t)B * (uint64_t)H * (uint64_t)((N + 255) / 256);
    prm.tiles_per_cta = (N > 128 && pairs < (uint64_t)num_sms) ? 1 : 2;
    if (flags & vitattn::kFlagForceTwoTiles) prm.tiles_per_cta = 2;
    if (flags & vitattn::kFlagForceOneTile) prm.tiles_per_cta = 1;
    prm.n_qgroups = (int)((N + 128 * prm.tiles_per_cta - 1) / (128 * prm.tiles_per_cta));
    prm.n_items = (int)((uint64_t)B * (uint64_t)H * (uint64_t)prm.n_qgroups);
    prm.n_kblocks = (int)((Nk + 127) / 128);

    // Persistent grid (one CTA per SM, each looping over work items) when there
    // are more items than SMs, the items are short enough (at most 32 key
    // blocks) for the per-CTA start-up and epilogue to matter, and every item
    // has the same number of query tiles (all have two unless the last group
    // of a head is a single tile); otherwise one CTA per item.
    // The causal mask gives items different key-block counts, so it runs one
    // CTA per item, each (b, h)'s longest item first: the hardware's block
    // scheduler then hands the short items to whichever SM frees up first.
    const bool uniform = !prm.causal && (prm.tiles_per_cta == 1 || (N % 256 == 0 || N % 256 > 128));
    unsigned grid = (unsigned)prm.n_items;
    if (uniform && prm.n_items > num_sms && prm.n_kblocks <= 32) grid = (unsigned)num_sms;
    if (uniform && (flags & vitattn::kFlagTinyGrid) && grid > 3u) grid = 3u;
    const bool loop = grid < (unsigned)prm.n_items;
    // One query tile per item (two would leave SMs idle) and one CTA per
    // item: the tile's key blocks are split over the two softmax warpgroups,
    // so that the CTA's serial chain is half as long and both warpgroups
    // work (the unmasked case with at least four key blocks).
    const int split_from = (flags & vitattn::kFlagSplitFromTwo) ? 2 : 4;
    prm.split = !loop && !prm.causal && prm.tiles_per_cta == 1 && prm.n_kblocks >= split_from &&
                !(flags & vitattn::kFlagNoSplit);

    SegDense seg{0};
    return run_kernel(dp, dtype, loop ? kModeLoop : (prm.split ? kModeSplit : kModeItem), grid, &prm, &seg,
                      stream);
}

// Ragged batch: one CTA per work item (segment, head, group of query tiles).
int launch_varlen(const void* q, const void* k, const void* v, void* out, const int32_t* cu,
                  int64_t num_seqs, int64_t H, int64_t D, float scale, int dtype, cudaStream_t stream,
                  int flags) {
    int rc = check_args_varlen(q, k, v, out, cu, num_seqs, H, D, scale, dtype);
    if (rc) return rc;
    const int64_t total = cu[num_seqs];
    if (total == 0) return VITATTN_OK;  // no tokens: nothing to compute or write
    const int dp = (int)((D + 15) / 16 * 16);
    int num_sms = 0;
    rc = device_info(&num_sms);
    if (rc) return rc;
    rc = check_device_ptrs({q, k, v, out});
    if (rc) return rc;

    FwdParams prm;
    rc = fill_common(&prm, q, k, v, out, 1, total, H, D, scale, dtype, flags);
    if (rc) return rc;
    static thread_local SegVar seg;  // ~4 KB: kept off the stack
    std::memset(&seg, 0, sizeof seg);
    seg.n = (int)num_seqs;
    // two query tiles per item unless that leaves SMs idle (as for the dense layout)
    uint64_t pairs = 0;
    for (int64_t s = 0; s < num_seqs; ++s) pairs += (uint64_t)H * (uint64_t)((cu[s + 1] - cu[s] + 255) / 256);
    int tiles = pairs < (uint64_t)num_sms ? 1 : 2;
    if (flags & vitattn::kFlagForceTwoTiles) tiles = 2;
    if (flags & vitattn::kFlagForceOneTile) tiles = 1;
    int items = 0;
    for (int s = 0; s < (int)num_seqs; ++s) {
        seg.start[s] = cu[s];
        seg.len[s] = cu[s + 1] - cu[s];
        seg.qgroups[s] = (seg.len[s] + 128 * tiles - 1) / (128 * tiles);
        seg.item0[s] = items;
        items += (int)H * seg.qgroups[s];
    }
    seg.item0[num_seqs] = items;
    prm.tiles_per_cta = tiles;
    prm.n_items = items;
    return run_kernel(dp, dtype, kModeVarlen, (unsigned)items, &prm, &seg, stream);
}

// The prologue: a grid-stride kernel, 8 warps per block, at most 8 blocks per SM
// (a full SM); a warp takes a group of one token's heads per loop trip (two
// heads side by side per row of the group when D <= 64).
int launch_rope(const void* qkv, const float* cs, const float* sn, void* q, void* k, void* v, int64_t T,
                int64_t H, int64_t D, int dtype, cudaStream_t stream, bool copy_v = true) {
    int rc = check_args_rope(qkv, cs, sn, q, k, v, T, H, D, dtype, copy_v);
    if (rc) return rc;
    int num_sms = 0;
    rc = device_info(&num_sms);
    if (rc) return rc;
    rc = check_device_ptrs({qkv, cs, sn, q, k, copy_v ? v : nullptr});
    if (rc) return rc;
    const int hpw = vitattn::rope_heads_per_warp(copy_v) * vitattn::rope_lane_groups((int)D);  // per loop trip
    const uint64_t items = (uint64_t)T * (uint64_t)((H + hpw - 1) / hpw);
    const uint64_t per_block = (uint64_t)(vitattn::kRopeThreads / 32);
    const uint64_t want = (items + per_block - 1) / per_block;
    const unsigned grid = (unsigned)std::min<uint64_t>(want, (uint64_t)num_sms * 8u);
    auto qkv8 = static_cast<const uint8_t*>(qkv);
    auto q8 = static_cast<uint8_t*>(q), k8 = static_cast<uint8_t*>(k), v8 = static_cast<uint8_t*>(v);
    long long TT = (long long)T;
    int HH = (int)H, DD = (int)D;
    void* args[9] = {&qkv8, &cs, &sn, &q8, &k8, &v8, &TT, &HH, &DD};
    const bool bf = dtype == VITATTN_BF16;
    static const void* const fns[2][2][2] = {  // [bf16][copy v][pair]
        {{reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<false, false, false>),
          reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<false, false, true>)},
         {reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<false, true, false>),
          reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<false, true, true>)}},
        {{reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<true, false, false>),
          reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<true, false, true>)},
         {reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<true, true, false>),
          reinterpret_cast<const void*>(vitattn::qkv_rope_kernel<true, true, true>)}}};
    const void* fn = fns[bf ? 1 : 0][copy_v ? 1 : 0][vitattn::rope_pair((int)D) ? 1 : 0];
    cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(vitattn::kRopeThreads), args, 0, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return VITATTN_OK;
}

// The prologue with q/k RMS norm: as launch_rope, with a grid of the blocks
// that are resident at once (kNormRopeBlocksPerSm per SM).
int launch_norm_rope(const void* qkv, const float* cs, const float* sn, const float* qw, const float* kw,
                     float eps, void* q, void* k, void* v, int64_t T, int64_t H, int64_t D, int dtype,
                     cudaStream_t stream, bool copy_v = true) {
    int rc = check_args_norm_rope(qkv, cs, sn, qw, kw, eps, q, k, v, T, H, D, dtype, copy_v);
    if (rc) return rc;
    int num_sms = 0;
    rc = device_info(&num_sms);
    if (rc) return rc;
    rc = check_device_ptrs({qkv, cs, sn, qw, kw, q, k, copy_v ? v : nullptr});
    if (rc) return rc;
    const int hpw = vitattn::kRopeHeadsPerWarp * vitattn::rope_lane_groups((int)D);  // heads per loop trip
    const uint64_t items = (uint64_t)T * (uint64_t)((H + hpw - 1) / hpw);
    const uint64_t per_block = (uint64_t)(vitattn::kRopeThreads / 32);
    const uint64_t want = (items + per_block - 1) / per_block;
    const unsigned grid =
        (unsigned)std::min<uint64_t>(want, (uint64_t)num_sms * (uint64_t)vitattn::kNormRopeBlocksPerSm);
    auto qkv8 = static_cast<const uint8_t*>(qkv);
    auto q8 = static_cast<uint8_t*>(q), k8 = static_cast<uint8_t*>(k), v8 = static_cast<uint8_t*>(v);
    long long TT = (long long)T;
    int HH = (int)H, DD = (int)D;
    void* args[12] = {&qkv8, &cs, &sn, &qw, &kw, &eps, &q8, &k8, &v8, &TT, &HH, &DD};
    const bool bf = dtype == VITATTN_BF16;
    static const void* const fns[2][2][2] = {  // [bf16][copy v][pair]
        {{reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<false, false, false>),
          reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<false, false, true>)},
         {reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<false, true, false>),
          reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<false, true, true>)}},
        {{reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<true, false, false>),
          reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<true, false, true>)},
         {reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<true, true, false>),
          reinterpret_cast<const void*>(vitattn::qkv_norm_rope_kernel<true, true, true>)}}};
    const void* fn = fns[bf ? 1 : 0][copy_v ? 1 : 0][vitattn::rope_pair((int)D) ? 1 : 0];
    cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(vitattn::kRopeThreads), args, 0, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return VITATTN_OK;
}

// Launch (through `go`), synchronise, and read the kernel's status words.
template <class Go>
int checked_run(cudaStream_t stream, Go go) {
    const unsigned zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_vitattn_status, &zero, sizeof zero, 0,
                                            cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemcpyToSymbolAsync(g_vitattn_range, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                                stream);
    if (e != cudaSuccess) return cuda_fail(e);
    int rc = go();
    if (rc) return rc;
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned status = 0, range = 0;
    e = cudaMemcpyFromSymbol(&status, g_vitattn_status, sizeof status);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemcpyFromSymbol(&range, g_vitattn_range, sizeof range);
    if (e != cudaSuccess) return cuda_fail(e);
    if (status) return VITATTN_ERR_TIMEOUT;
    return range ? VITATTN_ERR_RANGE : VITATTN_OK;
}

int forward_checked(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N,
                    int64_t H, int64_t D, float scale, int dtype, cudaStream_t stream, int flags,
                    int64_t Hkv = 0, const Ext& ext = Ext()) {
    int rc = ext.ts   ? check_args_strided(q, k, v, out, B, N, H, D, ext.ts, scale, dtype)
             : ext.Nk ? check_args_ext(q, k, v, out, ext.lse, B, N, ext.Nk, H, D, scale, dtype)
             : Hkv    ? check_args_gqa(q, k, v, out, B, N, H, Hkv, D, scale, dtype)
                      : check_args(q, k, v, out, B, N, H, D, scale, dtype);
    if (rc) return rc;
    return checked_run(stream,
                       [&] { return launch(q, k, v, out, B, N, H, D, scale, dtype, stream, flags, Hkv, ext); });
}

int forward_varlen_checked(const void* q, const void* k, const void* v, void* out, const int32_t* cu,
                           int64_t num_seqs, int64_t H, int64_t D, float scale, int dtype,
                           cudaStream_t stream, int flags) {
    int rc = check_args_varlen(q, k, v, out, cu, num_seqs, H, D, scale, dtype);
    if (rc) return rc;
    return checked_run(stream, [&] {
        return launch_varlen(q, k, v, out, cu, num_seqs, H, D, scale, dtype, stream, flags);
    });
}

// ---------------------------------------------------------------- host-buffer entry

// The host-buffer entry cuts the work into groups so that copies and kernels
// overlap: the inputs of group c+1 travel host -> device while the kernel of
// group c runs and the output of group c-1 travels back.  A group is a run
// of whole images (at most kImageGroups groups: every copy call costs, so
// more, smaller groups of images measured slower) when the batch has at
// least kImageGroups images; otherwise each image is cut into groups of
// heads (every head of a token is independent), at most kHostChunks groups
// in all, copied as 2-D copies of the heads' columns (rows of at least
// kMinCopyRow bytes) and run through the token-strided attention with a
// token-strided output.  Two copy streams per (host thread, device) carry
// the two directions; the kernels run on the caller's stream.
constexpr int kHostChunks = 16;
constexpr int kImageGroups = 8;
constexpr int64_t kMinCopyRow = 512;

struct HostPipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t in[kHostChunks] = {}, ran[kHostChunks] = {}, out[kHostChunks] = {};
};
thread_local HostPipe t_pipe[kMaxDevices];

int host_pipe(int dev, HostPipe** out) {
    HostPipe& hp = t_pipe[dev];
    if (!hp.ready) {
        cudaError_t e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming);
        for (int c = 0; c < kHostChunks && e == cudaSuccess; ++c) {
            e = cudaEventCreateWithFlags(&hp.in[c], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.ran[c], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.out[c], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) return cuda_fail(e);
        hp.ready = true;
    }
    *out = &hp;
    return VITATTN_OK;
}

// How the host-buffer entry cuts [B, N, H, D]: `per_chunk` images per group
// when heads are not cut (groups_per_image == 1), else one image per group
// and its heads in groups_per_image near-equal parts: part g is heads
// g*H/G .. (g+1)*H/G - 1 (G = groups_per_image, integer division), each at
// least kMinCopyRow bytes of a token wide.
struct HostPlan {
    int64_t per_chunk;
    int groups_per_image, nchunks;
};

HostPlan host_plan(int64_t B, int64_t H, int64_t D) {
    HostPlan pl{};
    pl.groups_per_image = 1;
    if (B < kImageGroups && H > 1) {
        const int64_t want = (kHostChunks + B - 1) / B;              // groups per image wanted
        const int64_t min_hc = (kMinCopyRow + 2 * D - 1) / (2 * D);  // heads per copy row at least
        const int64_t g = std::min<int64_t>(std::min<int64_t>(want, H / min_hc), kHostChunks / B);
        if (g > 1) pl.groups_per_image = (int)g;
    }
    if (pl.groups_per_image > 1) {
        pl.per_chunk = 1;
        pl.nchunks = (int)(B * pl.groups_per_image);
    } else {
        pl.per_chunk = (B + kImageGroups - 1) / kImageGroups;
        pl.nchunks = (int)((B + pl.per_chunk - 1) / pl.per_chunk);
    }
    return pl;
}

int forward_host(const void* hq, const void* hk, const void* hv, void* hout, void* dq, void* dk, void* dv,
                 void* dout, int64_t B, int64_t N, int64_t H, int64_t D, float scale, int dtype,
                 cudaStream_t s) {
    if (!hq || !hk || !hv || !hout) return VITATTN_ERR_NULL;
    int rc = check_args(dq, dk, dv, dout, B, N, H, D, scale, dtype);
    if (rc) return rc;
    int num_sms = 0;
    rc = device_info(&num_sms);
    if (rc) return rc;
    rc = check_device_ptrs({dq, dk, dv, dout});
    if (rc) return rc;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    HostPipe* hp = nullptr;
    rc = host_pipe(dev, &hp);
    if (rc) return rc;

    const HostPlan pl = host_plan(B, H, D);
    const size_t token_bytes = (size_t)H * (size_t)D * 2u;
    const size_t image_bytes = (size_t)N * token_bytes;
    const void* hsrc[3] = {hq, hk, hv};
    uint8_t* ddst[3] = {static_cast<uint8_t*>(dq), static_cast<uint8_t*>(dk), static_cast<uint8_t*>(dv)};
    const int64_t ts[3] = {H * D, H * D, H * D};
    // the copies start once the caller's earlier work on `s` is done (it may still read dq..dout)
    e = cudaEventRecord(hp->start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->h2d, hp->start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->d2h, hp->start, 0);
    if (e != cudaSuccess) return cuda_fail(e);
    for (int c = 0; c < pl.nchunks; ++c) {
        // group c: images b0 .. b0 + nb - 1, heads h0 .. h0 + nh - 1
        const int G = pl.groups_per_image;
        const int64_t b0 = (G > 1) ? c / G : (int64_t)c * pl.per_chunk;
        const int64_t nb = (G > 1) ? 1 : std::min<int64_t>(pl.per_chunk, B - b0);
        const int64_t h0 = (G > 1) ? (c % G) * H / G : 0;
        const int64_t nh = (G > 1) ? (c % G + 1) * H / G - h0 : H;
        const size_t off = (size_t)b0 * image_bytes + (size_t)h0 * (size_t)D * 2u;
        const size_t width = (size_t)nh * (size_t)D * 2u;  // bytes of one token's heads in the group
        const size_t rows = (size_t)nb * (size_t)N;
        auto copy = [&](void* dst, const void* src, cudaMemcpyKind kind, cudaStream_t st) -> cudaError_t {
            if (nh == H) return cudaMemcpyAsync(dst, src, rows * width, kind, st);
            return cudaMemcpy2DAsync(dst, token_bytes, src, token_bytes, width, rows, kind, st);
        };
        for (int i = 0; i < 3 && e == cudaSuccess; ++i)
            e = copy(ddst[i] + off, static_cast<const uint8_t*>(hsrc[i]) + off, cudaMemcpyHostToDevice, hp->h2d);
        if (e == cudaSuccess) e = cudaEventRecord(hp->in[c], hp->h2d);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hp->in[c], 0);
        if (e != cudaSuccess) return cuda_fail(e);
        uint8_t* o = static_cast<uint8_t*>(dout) + off;
        if (nh == H) {
            rc = launch(ddst[0] + off, ddst[1] + off, ddst[2] + off, o, nb, N, H, D, scale, dtype, s, 0);
        } else {
            Ext ext;
            ext.ts = ts;
            ext.out_ts = H * D;
            rc = launch(ddst[0] + off, ddst[1] + off, ddst[2] + off, o, nb, N, nh, D, scale, dtype, s, 0, 0, ext);
        }
        if (rc) return rc;
        e = cudaEventRecord(hp->ran[c], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->d2h, hp->ran[c], 0);
        if (e == cudaSuccess) e = copy(static_cast<uint8_t*>(hout) + off, o, cudaMemcpyDeviceToHost, hp->d2h);
        if (e == cudaSuccess) e = cudaEventRecord(hp->out[c], hp->d2h);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    // work the caller enqueues on `s` afterwards (or a synchronisation of `s`) follows the last
    // output copy; the copy stream runs in order, so that covers every group
    e = cudaStreamWaitEvent(s, hp->out[pl.nchunks - 1], 0);
    if (e != cudaSuccess) return cuda_fail(e);
    return VITATTN_OK;
}

}  // namespace

extern "C" {

int vitattn_forward(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N,
                    int64_t H, int64_t D, float scale, int dtype, vitattn_stream_t stream) {
    return launch(q, k, v, out, B, N, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), 0);
}

int vitattn_forward_checked(const void* q, const void* k, const void* v, void* out, int64_t B,
                            int64_t N, int64_t H, int64_t D, float scale, int dtype,
                            vitattn_stream_t stream) {
    return forward_checked(q, k, v, out, B, N, H, D, scale, dtype,
                           reinterpret_cast<cudaStream_t>(stream), 0);
}

// Test hook, deliberately absent from the public header: the checked entry
// with test flags (bit 0: the producer withholds the first V block so that a
// bounded wait runs out and the timeout path is exercised; bit 1 / bit 2:
// force two / one query tiles per work item; bit 3: at most three CTAs, each
// looping over many work items).
VITATTN_API int vitattn_test_forward_flags(const void* q, const void* k, const void* v, void* out, int64_t B,
                               int64_t N, int64_t H, int64_t D, float scale, int dtype,
                               vitattn_stream_t stream, int flags) {
    return forward_checked(q, k, v, out, B, N, H, D, scale, dtype,
                           reinterpret_cast<cudaStream_t>(stream), flags);
}

int vitattn_forward_ext(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t Lq,
                        int64_t Lk, int64_t H, int64_t D, float scale, int causal, int dtype,
                        vitattn_stream_t stream) {
    Ext ext;
    ext.Nk = Lk < 1 ? -1 : Lk;  // a non-positive Lk is reported by the checks
    ext.causal = causal;
    ext.lse = lse;
    if (Lk < 1) return check_args_ext(q, k, v, out, lse, B, Lq, Lk, H, D, scale, dtype);
    return launch(q, k, v, out, B, Lq, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), 0, 0, ext);
}

int vitattn_forward_ext_checked(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B,
                                int64_t Lq, int64_t Lk, int64_t H, int64_t D, float scale, int causal, int dtype,
                                vitattn_stream_t stream) {
    if (Lk < 1) return check_args_ext(q, k, v, out, lse, B, Lq, Lk, H, D, scale, dtype);
    Ext ext;
    ext.Nk = Lk;
    ext.causal = causal;
    ext.lse = lse;
    return forward_checked(q, k, v, out, B, Lq, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), 0, 0,
                           ext);
}

// Test hook, deliberately absent from the public header: the checked
// cross-length / causal entry with the test flags of vitattn_test_forward_flags.
VITATTN_API int vitattn_test_forward_ext_flags(const void* q, const void* k, const void* v, void* out, float* lse,
                                               int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D,
                                               float scale, int causal, int dtype, vitattn_stream_t stream,
                                               int flags) {
    if (Lk < 1) return check_args_ext(q, k, v, out, lse, B, Lq, Lk, H, D, scale, dtype);
    Ext ext;
    ext.Nk = Lk;
    ext.causal = causal;
    ext.lse = lse;
    return forward_checked(q, k, v, out, B, Lq, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), flags,
                           0, ext);
}

int vitattn_check_args_ext(const void* q, const void* k, const void* v, const void* out, const float* lse,
                           int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D, float scale, int dtype) {
    return check_args_ext(q, k, v, out, lse, B, Lq, Lk, H, D, scale, dtype);
}

int vitattn_forward_gqa(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N, int64_t H,
                        int64_t Hkv, int64_t D, float scale, int dtype, vitattn_stream_t stream) {
    return launch(q, k, v, out, B, N, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), 0, Hkv);
}

int vitattn_forward_gqa_checked(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N,
                                int64_t H, int64_t Hkv, int64_t D, float scale, int dtype,
                                vitattn_stream_t stream) {
    return forward_checked(q, k, v, out, B, N, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), 0,
                           Hkv);
}

// Test hook, deliberately absent from the public header: the checked
// grouped-query entry with the test flags of vitattn_test_forward_flags.
VITATTN_API int vitattn_test_forward_gqa_flags(const void* q, const void* k, const void* v, void* out, int64_t B,
                                               int64_t N, int64_t H, int64_t Hkv, int64_t D, float scale,
                                               int dtype, vitattn_stream_t stream, int flags) {
    return forward_checked(q, k, v, out, B, N, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), flags,
                           Hkv);
}

int vitattn_check_args_gqa(const void* q, const void* k, const void* v, const void* out, int64_t B, int64_t N,
                           int64_t H, int64_t Hkv, int64_t D, float scale, int dtype) {
    return check_args_gqa(q, k, v, out, B, N, H, Hkv, D, scale, dtype);
}

int vitattn_forward_varlen(const void* q, const void* k, const void* v, void* out,
                           const int32_t* cu_seqlens, int64_t num_seqs, int64_t H, int64_t D, float scale,
                           int dtype, vitattn_stream_t stream) {
    return launch_varlen(q, k, v, out, cu_seqlens, num_seqs, H, D, scale, dtype,
                         reinterpret_cast<cudaStream_t>(stream), 0);
}

int vitattn_forward_varlen_checked(const void* q, const void* k, const void* v, void* out,
                                   const int32_t* cu_seqlens, int64_t num_seqs, int64_t H, int64_t D,
                                   float scale, int dtype, vitattn_stream_t stream) {
    return forward_varlen_checked(q, k, v, out, cu_seqlens, num_seqs, H, D, scale, dtype,
                                  reinterpret_cast<cudaStream_t>(stream), 0);
}

// Test hook, deliberately absent from the public header: the checked ragged
// entry with the test flags of vitattn_test_forward_flags.
VITATTN_API int vitattn_test_forward_varlen_flags(const void* q, const void* k, const void* v, void* out,
                                                  const int32_t* cu_seqlens, int64_t num_seqs, int64_t H,
                                                  int64_t D, float scale, int dtype, vitattn_stream_t stream,
                                                  int flags) {
    return forward_varlen_checked(q, k, v, out, cu_seqlens, num_seqs, H, D, scale, dtype,
                                  reinterpret_cast<cudaStream_t>(stream), flags);
}

int vitattn_check_args_varlen(const void* q, const void* k, const void* v, const void* out,
                              const int32_t* cu_seqlens, int64_t num_seqs, int64_t H, int64_t D,
                              float scale, int dtype) {
    return check_args_varlen(q, k, v, out, cu_seqlens, num_seqs, H, D, scale, dtype);
}

int vitattn_qkv_rope(const void* qkv, const float* cos_table, const float* sin_table, void* q, void* k, void* v,
                     int64_t T, int64_t H, int64_t D, int dtype, vitattn_stream_t stream) {
    return launch_rope(qkv, cos_table, sin_table, q, k, v, T, H, D, dtype, reinterpret_cast<cudaStream_t>(stream));
}

int vitattn_check_args_qkv_rope(const void* qkv, const float* cos_table, const float* sin_table, const void* q,
                                const void* k, const void* v, int64_t T, int64_t H, int64_t D, int dtype) {
    return check_args_rope(qkv, cos_table, sin_table, q, k, v, T, H, D, dtype);
}

int vitattn_qkv_norm_rope(const void* qkv, const float* cos_table, const float* sin_table,
                          const float* q_norm_w, const float* k_norm_w, float eps, void* q, void* k, void* v,
                          int64_t T, int64_t H, int64_t D, int dtype, vitattn_stream_t stream) {
    return launch_norm_rope(qkv, cos_table, sin_table, q_norm_w, k_norm_w, eps, q, k, v, T, H, D, dtype,
                            reinterpret_cast<cudaStream_t>(stream));
}

int vitattn_check_args_qkv_norm_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                     const float* q_norm_w, const float* k_norm_w, float eps, const void* q,
                                     const void* k, const void* v, int64_t T, int64_t H, int64_t D, int dtype) {
    return check_args_norm_rope(qkv, cos_table, sin_table, q_norm_w, k_norm_w, eps, q, k, v, T, H, D, dtype);
}

int vitattn_forward_strided(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N,
                            int64_t H, int64_t D, int64_t q_stride, int64_t k_stride, int64_t v_stride, float scale,
                            int dtype, vitattn_stream_t stream) {
    const int64_t ts[3] = {q_stride, k_stride, v_stride};
    Ext ext;
    ext.ts = ts;
    return launch(q, k, v, out, B, N, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), 0, 0, ext);
}

int vitattn_forward_strided_checked(const void* q, const void* k, const void* v, void* out, int64_t B,
                                    int64_t N, int64_t H, int64_t D, int64_t q_stride, int64_t k_stride,
                                    int64_t v_stride, float scale, int dtype, vitattn_stream_t stream) {
    const int64_t ts[3] = {q_stride, k_stride, v_stride};
    Ext ext;
    ext.ts = ts;
    return forward_checked(q, k, v, out, B, N, H, D, scale, dtype, reinterpret_cast<cudaStream_t>(stream), 0, 0,
                           ext);
}

int vitattn_check_args_strided(const void* q, const void* k, const void* v, const void* out, int64_t B, int64_t N,
                               int64_t H, int64_t D, int64_t q_stride, int64_t k_stride, int64_t v_stride,
                               float scale, int dtype) {
    const int64_t ts[3] = {q_stride, k_stride, v_stride};
    return check_args_strided(q, k, v, out, B, N, H, D, ts, scale, dtype);
}

int vitattn_qk_rope(const void* qkv, const float* cos_table, const float* sin_table, void* q, void* k, int64_t T,
                    int64_t H, int64_t D, int dtype, vitattn_stream_t stream) {
    return launch_rope(qkv, cos_table, sin_table, q, k, nullptr, T, H, D, dtype,
                       reinterpret_cast<cudaStream_t>(stream), false);
}

int vitattn_check_args_qk_rope(const void* qkv, const float* cos_table, const float* sin_table, const void* q,
                               const void* k, int64_t T, int64_t H, int64_t D, int dtype) {
    return check_args_rope(qkv, cos_table, sin_table, q, k, nullptr, T, H, D, dtype, false);
}

int vitattn_qk_norm_rope(const void* qkv, const float* cos_table, const float* sin_table, const float* q_norm_w,
                         const float* k_norm_w, float eps, void* q, void* k, int64_t T, int64_t H, int64_t D,
                         int dtype, vitattn_stream_t stream) {
    return launch_norm_rope(qkv, cos_table, sin_table, q_norm_w, k_norm_w, eps, q, k, nullptr, T, H, D, dtype,
                            reinterpret_cast<cudaStream_t>(stream), false);
}

int vitattn_check_args_qk_norm_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                    const float* q_norm_w, const float* k_norm_w, float eps, const void* q,
                                    const void* k, int64_t T, int64_t H, int64_t D, int dtype) {
    return check_args_norm_rope(qkv, cos_table, sin_table, q_norm_w, k_norm_w, eps, q, k, nullptr, T, H, D, dtype,
                                false);
}

int vitattn_forward_host(const void* hq, const void* hk, const void* hv, void* hout, void* dq,
                         void* dk, void* dv, void* dout, int64_t B, int64_t N, int64_t H,
                         int64_t D, float scale, int dtype, vitattn_stream_t stream) {
    return forward_host(hq, hk, hv, hout, dq, dk, dv, dout, B, N, H, D, scale, dtype,
                        reinterpret_cast<cudaStream_t>(stream));
}

int vitattn_check_args(const void* q, const void* k, const void* v, const void* out, int64_t B,
                       int64_t N, int64_t H, int64_t D, float scale, int dtype) {
    return check_args(q, k, v, out, B, N, H, D, scale, dtype);
}

const char* vitattn_strerror(int status) {
    switch (status) {
        case VITATTN_OK: return "ok";
        case VITATTN_ERR_NULL: return "a required pointer is NULL";
        case VITATTN_ERR_DIM: return "B, N, H must be >= 1 and the sizes must not overflow";
        case VITATTN_ERR_HEADDIM: return "unsupported head dimension (need 16 <= D <= 128, D % 8 == 0)";
        case VITATTN_ERR_DTYPE: return "dtype must be VITATTN_BF16 or VITATTN_F16";
        case VITATTN_ERR_ALIGN: return "tensor pointers must be 16-byte aligned";
        case VITATTN_ERR_ALIAS: return "out overlaps q, k or v";
        case VITATTN_ERR_CUDA: return "CUDA error (see vitattn_last_cuda_error)";
        case VITATTN_ERR_TIMEOUT: return "a bounded in-kernel wait ran out";
        case VITATTN_ERR_SCALE: return "scale must be finite (eps: finite and >= 0)";
        case VITATTN_ERR_DEVICE:
            return "the current device is not an sm_100 GPU, or a pointer is not memory its kernels can use";
        case VITATTN_ERR_SEQLENS: return "cu_seqlens must start at 0 and never decrease";
        case VITATTN_ERR_RANGE: return "a bf16 V value has magnitude >= 65536, outside the f16 P.V product's range";
        default: return "unknown status";
    }
}

int vitattn_last_cuda_error(void) { return t_last_cuda_error; }

int vitattn_version(void) { return kVersion; }

int vitattn_launches_per_call(void) { return 1; }

// Test hook, deliberately absent from the public header: how the host-buffer
// entry cuts a batch (out[0] images per group, out[1] groups per image, 1
// when heads are not cut, out[2] groups).  No CUDA call.
VITATTN_API int vitattn_test_host_plan(int64_t B, int64_t H, int64_t D, int64_t* out) {
    if (!out || B < 1 || H < 1 || D < 1) return VITATTN_ERR_DIM;
    const HostPlan pl = host_plan(B, H, D);
    out[0] = pl.per_chunk;
    out[1] = pl.groups_per_image;
    out[2] = pl.nchunks;
    return VITATTN_OK;
}

}  // extern "C"
