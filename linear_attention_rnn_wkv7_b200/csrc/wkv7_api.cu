// wkv7_api.cu -- the C ABI of libwkv7.so (declared in include/wkv7.h): host-side
// argument checks and kernel dispatch.  Everything the recurrence computes runs
// in the kernels included below; this file only validates and launches.
#include <cuda_runtime.h>

#include <atomic>

#include "wkv7.h"
#include "common.cuh"
#include "step.cuh"
#include "recurrent.cuh"
#include "chunked.cuh"
#include "backward.cuh"
#include "chunked_bwd.cuh"
#include "gdn_backward.cuh"

namespace {

constexpr int kVersion = 1 * 10000 + 0 * 100 + 0;

// Scratch of wkv7_bwd_noalloc: a file-scope device array, reserved when the library's
// module is loaded, so that entry point allocates nothing at call time.
constexpr size_t kStaticScratchBytes = WKV7_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The array's device address, looked up once per device with that device current (in
// host code the symbol is only a host-side stand-in, never a device address).
constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Address of the static scratch on the current device, or nullptr on a CUDA error.
void* static_scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_addr[dev].store(p, std::memory_order_release);
    return p;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

// Test hook of the chunked kernel's timeout path (wkv7_test_stall_next_chunked):
// consumed, and reset to -1, by the next chunked WKV7 launch.
std::atomic<int> g_stall_tid{-1};

// Head sizes with a kernel: K == V in {64, 128, 256} (the chunked form: 64 only).
inline bool head_size_ok(int K, int V) { return K == V && (K == 64 || K == 128 || K == 256); }

// Non-null and aligned to its element (g, beta are read one element at a time).
inline bool ok_scalar_ptr(const void* p, wkv7_dtype dtype) {
    const uintptr_t m = dtype == WKV7_BF16 ? 1u : 3u;
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & m) == 0;
}

}  // namespace

extern "C" {

const char* wkv7_status_string(wkv7_status s) {
    switch (s) {
        case WKV7_OK: return "WKV7_OK";
        case WKV7_ERR_INVALID_ARG: return "WKV7_ERR_INVALID_ARG";
        case WKV7_ERR_UNSUPPORTED: return "WKV7_ERR_UNSUPPORTED";
        case WKV7_ERR_CUDA: return "WKV7_ERR_CUDA";
        case WKV7_ERR_DEVICE_TIMEOUT: return "WKV7_ERR_DEVICE_TIMEOUT";
        case WKV7_ERR_DEVICE_BAD_SEQLENS: return "WKV7_ERR_DEVICE_BAD_SEQLENS";
    }
    return "WKV7_UNKNOWN_STATUS";
}

int wkv7_version(void) { return kVersion; }

wkv7_status wkv7_test_stall_next_chunked(int tid) {
    if (tid < -1 || tid >= wkv7::chunked::kThreads) return WKV7_ERR_INVALID_ARG;
    g_stall_tid.store(tid);
    return WKV7_OK;
}

wkv7_status wkv7_test_chunked_schedule(long long units, int len, int* resident, long long* ctas,
                                       long long* cmax) {
    using namespace wkv7::chunked;
    if (!resident || !ctas || !cmax || units < 0 || len < 0) return WKV7_ERR_INVALID_ARG;
    if (ensure_smem_attr<false, false, false>() != cudaSuccess) {
        (void)cudaGetLastError();
        return WKV7_ERR_CUDA;
    }
    const int slots = resident_ctas<false, false, false>();
    if (slots <= 0) return WKV7_ERR_CUDA;
    long long c = 0, m = 0;
    if (!balanced_geometry(units, len, slots, c, m)) c = m = 0;
    *resident = slots;
    *ctas = c;
    *cmax = m;
    return WKV7_OK;
}

wkv7_status wkv7_fwd(const void* r, const void* w, const void* k, const void* v,
                     const void* a, const void* b, const float* s0, const uint8_t* mask,
                     void* o, float* sT, int B, int T, int H, int K, int V,
                     const int32_t* cu_seqlens, int N, wkv7_layout layout, wkv7_dtype dtype,
                     wkv7_algo algo, void* stream_) {
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0 || N < 0) return WKV7_ERR_INVALID_ARG;
    if (layout != WKV7_LAYOUT_BTHK && layout != WKV7_LAYOUT_BHTK) return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (algo != WKV7_ALGO_AUTO && algo != WKV7_ALGO_RECURRENT && algo != WKV7_ALGO_CHUNKED)
        return WKV7_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1) return WKV7_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return WKV7_ERR_INVALID_ARG;
    } else if (N != B) {
        return WKV7_ERR_INVALID_ARG;
    }
    if (!head_size_ok(K, V)) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)N * H;
    const long long rows = (long long)B * T * H;
    if (units * (K / 64) > 0x7fffffffLL || rows > (1LL << 40) || (long long)B * T > 0x7fffffffLL)
        return WKV7_ERR_UNSUPPORTED;
    const bool tokens = rows > 0;
    if (tokens && (!ok_ptr(r) || !ok_ptr(w) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(a) ||
                   !ok_ptr(b) || !ok_ptr(o)))
        return WKV7_ERR_INVALID_ARG;
    if ((s0 && !aligned16(s0)) || (sT && !aligned16(sT))) return WKV7_ERR_INVALID_ARG;
    if (tokens && (o == r || o == w || o == k || o == v || o == a || o == b))
        return WKV7_ERR_INVALID_ARG;
    if (units == 0) return WKV7_OK;

    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int hf = layout == WKV7_LAYOUT_BHTK;
    // T == 0 (nothing but the state copy) always takes the recurrent kernel.
    const bool chunked = rows > 0 && (algo == WKV7_ALGO_CHUNKED ||
                         (algo == WKV7_ALGO_AUTO && dtype == WKV7_BF16 && K == 64 &&
                          wkv7::kChunkedBuilt));
    cudaError_t err;
    if (chunked) {
        if (dtype != WKV7_BF16 || K != 64 || !wkv7::kChunkedBuilt) return WKV7_ERR_UNSUPPORTED;
        err = wkv7::launch_chunked(r, w, k, v, a, b, s0, mask, o, sT, B, T, H, N, cu_seqlens,
                                   hf, g_stall_tid.exchange(-1), stream);
    } else if (dtype == WKV7_BF16) {
        err = wkv7::launch_recurrent<__nv_bfloat16>(r, w, k, v, a, b, s0, mask, o, sT, T, H, N,
                                                    cu_seqlens, hf, K, stream);
    } else {
        err = wkv7::launch_recurrent<float>(r, w, k, v, a, b, s0, mask, o, sT, T, H, N,
                                            cu_seqlens, hf, K, stream);
    }
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

wkv7_status wkv7_step(const void* r, const void* w, const void* k, const void* v,
                      const void* a, const void* b, float* state, void* o, int B, int H,
                      int K, int V, wkv7_dtype dtype, void* stream_) {
    if (B < 0 || H <= 0 || K <= 0 || V <= 0) return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (!head_size_ok(K, V)) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)B * H;
    if (units == 0) return WKV7_OK;
    if (units > (1LL << 33) || units * (K / 64) > 0x7fffffffLL) return WKV7_ERR_UNSUPPORTED;
    if (!ok_ptr(r) || !ok_ptr(w) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(a) || !ok_ptr(b) ||
        !ok_ptr(state) || !ok_ptr(o))
        return WKV7_ERR_INVALID_ARG;
    if (o == state || o == r || o == w || o == k || o == v || o == a || o == b)
        return WKV7_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const cudaError_t err =
        dtype == WKV7_BF16
            ? wkv7::launch_step<__nv_bfloat16>(r, w, k, v, a, b, state, o, units, K, stream)
            : wkv7::launch_step<float>(r, w, k, v, a, b, state, o, units, K, stream);
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

wkv7_status wkv7_gdn_fwd(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* s0, int s0_shared, void* o, float* sT,
                         int B, int T, int H, int K, int V, const int32_t* cu_seqlens, int N,
                         wkv7_layout layout, wkv7_dtype dtype, wkv7_algo algo, void* stream_) {
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0 || N < 0) return WKV7_ERR_INVALID_ARG;
    if (layout != WKV7_LAYOUT_BTHK && layout != WKV7_LAYOUT_BHTK) return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (algo != WKV7_ALGO_AUTO && algo != WKV7_ALGO_RECURRENT && algo != WKV7_ALGO_CHUNKED)
        return WKV7_ERR_INVALID_ARG;
    if (s0_shared != 0 && s0_shared != 1) return WKV7_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1) return WKV7_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return WKV7_ERR_INVALID_ARG;
    } else if (N != B) {
        return WKV7_ERR_INVALID_ARG;
    }
    if (!head_size_ok(K, V)) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)N * H;
    const long long rows = (long long)B * T * H;
    if (units * (K / 64) > 0x7fffffffLL || rows > (1LL << 40) || (long long)B * T > 0x7fffffffLL)
        return WKV7_ERR_UNSUPPORTED;
    const bool tokens = rows > 0;
    if (tokens && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) ||
                   !ok_scalar_ptr(g, dtype) || !ok_scalar_ptr(beta, dtype)))
        return WKV7_ERR_INVALID_ARG;
    if ((s0 && !aligned16(s0)) || (sT && !aligned16(sT))) return WKV7_ERR_INVALID_ARG;
    if (tokens && (o == q || o == k || o == v || o == g || o == beta))
        return WKV7_ERR_INVALID_ARG;
    if (s0_shared && sT && s0 == sT && N > 1) return WKV7_ERR_INVALID_ARG;
    if (units == 0) return WKV7_OK;
    if (!s0) s0_shared = 0;

    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int hf = layout == WKV7_LAYOUT_BHTK;
    const bool chunked = rows > 0 && (algo == WKV7_ALGO_CHUNKED ||
                         (algo == WKV7_ALGO_AUTO && dtype == WKV7_BF16 && K == 64 &&
                          wkv7::kChunkedBuilt));
    cudaError_t err;
    if (chunked) {
        if (dtype != WKV7_BF16 || K != 64 || !wkv7::kChunkedBuilt) return WKV7_ERR_UNSUPPORTED;
        err = wkv7::launch_chunked_gdn(q, k, v, g, beta, s0, s0_shared, o, sT, B, T, H, N,
                                       cu_seqlens, hf, stream);
    } else if (dtype == WKV7_BF16) {
        err = wkv7::launch_recurrent_gdn<__nv_bfloat16>(q, k, v, g, beta, s0, s0_shared, o, sT,
                                                        T, H, N, cu_seqlens, hf, K, stream);
    } else {
        err = wkv7::launch_recurrent_gdn<float>(q, k, v, g, beta, s0, s0_shared, o, sT, T, H,
                                                N, cu_seqlens, hf, K, stream);
    }
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

wkv7_status wkv7_gdn_step(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, float* state, void* o, int B, int H, int K, int V,
                          wkv7_dtype dtype, void* stream_) {
    if (B < 0 || H <= 0 || K <= 0 || V <= 0) return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (!head_size_ok(K, V)) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)B * H;
    if (units == 0) return WKV7_OK;
    if (units > (1LL << 33) || units * (K / 64) > 0x7fffffffLL) return WKV7_ERR_UNSUPPORTED;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(state) || !ok_ptr(o) ||
        !ok_scalar_ptr(g, dtype) || !ok_scalar_ptr(beta, dtype))
        return WKV7_ERR_INVALID_ARG;
    if (o == state || o == q || o == k || o == v || o == g || o == beta)
        return WKV7_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const cudaError_t err =
        dtype == WKV7_BF16
            ? wkv7::launch_step_gdn<__nv_bfloat16>(q, k, v, g, beta, state, o, units, K, stream)
            : wkv7::launch_step_gdn<float>(q, k, v, g, beta, state, o, units, K, stream);
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

wkv7_status wkv7_sane_fwd(const void* r, const void* w, const void* k, const void* v,
                          const void* a, const void* b, const float* tau,
                          const uint8_t* sane_mask, const float* s0, int s0_shared, void* o,
                          float* sT, int B, int T, int H, int K, int V, wkv7_layout layout,
                          wkv7_dtype dtype, void* stream_) {
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0) return WKV7_ERR_INVALID_ARG;
    if (layout != WKV7_LAYOUT_BTHK && layout != WKV7_LAYOUT_BHTK) return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (s0_shared != 0 && s0_shared != 1) return WKV7_ERR_INVALID_ARG;
    if (!head_size_ok(K, V)) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)B * H;
    const long long rows = (long long)B * T * H;
    if (units * (K / 64) > 0x7fffffffLL || rows > (1LL << 40) || (long long)B * T > 0x7fffffffLL)
        return WKV7_ERR_UNSUPPORTED;
    const bool tokens = rows > 0;
    if (tokens && (!ok_ptr(r) || !ok_ptr(w) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(a) ||
                   !ok_ptr(b) || !ok_ptr(o)))
        return WKV7_ERR_INVALID_ARG;
    if (T >= 16 && B > 0 && !ok_scalar_ptr(tau, WKV7_F32)) return WKV7_ERR_INVALID_ARG;
    if ((s0 && !aligned16(s0)) || (sT && !aligned16(sT))) return WKV7_ERR_INVALID_ARG;
    if (tokens && (o == r || o == w || o == k || o == v || o == a || o == b))
        return WKV7_ERR_INVALID_ARG;
    if (s0_shared && sT && s0 == sT && B > 1) return WKV7_ERR_INVALID_ARG;
    if (units == 0) return WKV7_OK;
    if (!s0) s0_shared = 0;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int hf = layout == WKV7_LAYOUT_BHTK;
    const cudaError_t err =
        dtype == WKV7_BF16
            ? wkv7::launch_recurrent_sane<__nv_bfloat16>(r, w, k, v, a, b, tau, sane_mask, s0,
                                                         s0_shared, o, sT, B, T, H, hf, K, stream)
            : wkv7::launch_recurrent_sane<float>(r, w, k, v, a, b, tau, sane_mask, s0, s0_shared,
                                                 o, sT, B, T, H, hf, K, stream);
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

wkv7_status wkv7_sane_step(const void* r, const void* w, const void* k, const void* v,
                           const void* a, const void* b, const float* tau,
                           const uint8_t* do_sane, int do_sane_all, float* state, void* o,
                           int B, int H, int K, int V, wkv7_dtype dtype, void* stream_) {
    if (B < 0 || H <= 0 || K <= 0 || V <= 0) return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (do_sane_all != 0 && do_sane_all != 1) return WKV7_ERR_INVALID_ARG;
    if (!head_size_ok(K, V)) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)B * H;
    if (units == 0) return WKV7_OK;
    if (units > (1LL << 33) || units * (K / 64) > 0x7fffffffLL) return WKV7_ERR_UNSUPPORTED;
    if (!ok_ptr(r) || !ok_ptr(w) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(a) || !ok_ptr(b) ||
        !ok_ptr(state) || !ok_ptr(o) || !ok_scalar_ptr(tau, WKV7_F32))
        return WKV7_ERR_INVALID_ARG;
    if (o == state || o == r || o == w || o == k || o == v || o == a || o == b)
        return WKV7_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const cudaError_t err =
        dtype == WKV7_BF16
            ? wkv7::launch_step_sane<__nv_bfloat16>(r, w, k, v, a, b, tau, do_sane, do_sane_all,
                                                    state, o, units, H, K, stream)
            : wkv7::launch_step_sane<float>(r, w, k, v, a, b, tau, do_sane, do_sane_all, state,
                                            o, units, H, K, stream);
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

size_t wkv7_bwd_workspace_bytes_algo(int B, int T, int H, int K, int V, int N, wkv7_dtype dtype,
                                     wkv7_algo algo) {
    if (B < 0 || T < 0 || H <= 0 || N < 0 || K != 64 || V != 64) return 0;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return 0;
    const long long rows = (long long)B * T;
    if (algo == WKV7_ALGO_CHUNKED || (algo == WKV7_ALGO_AUTO && dtype == WKV7_BF16))
        return dtype == WKV7_BF16 ? wkv7::bwd_chunked_workspace_bytes(rows, N, H) : 0;
    if (algo == WKV7_ALGO_RECURRENT || algo == WKV7_ALGO_AUTO)
        return wkv7::bwd::workspace_floats(rows, N, H) * sizeof(float);
    return 0;
}

size_t wkv7_bwd_workspace_bytes(int B, int T, int H, int K, int V, int N) {
    const size_t rec = wkv7_bwd_workspace_bytes_algo(B, T, H, K, V, N, WKV7_F32, WKV7_ALGO_RECURRENT);
    const size_t chk = wkv7_bwd_workspace_bytes_algo(B, T, H, K, V, N, WKV7_BF16, WKV7_ALGO_CHUNKED);
    return rec > chk ? rec : chk;
}

wkv7_status wkv7_bwd(const void* r, const void* w, const void* k, const void* v, const void* a,
                     const void* b, const float* s0, const uint8_t* mask, const void* dout,
                     const float* dsT, void* dr, void* dw, void* dk, void* dv, void* da,
                     void* db, float* ds0, int B, int T, int H, int K, int V,
                     const int32_t* cu_seqlens, int N, wkv7_layout layout, wkv7_dtype dtype,
                     void* workspace, size_t workspace_bytes, void* stream_) {
    return wkv7_bwd_with_algo(r, w, k, v, a, b, s0, mask, dout, dsT, dr, dw, dk, dv, da, db, ds0,
                              B, T, H, K, V, cu_seqlens, N, layout, dtype, WKV7_ALGO_AUTO,
                              workspace, workspace_bytes, stream_);
}

wkv7_status wkv7_bwd_with_algo(const void* r, const void* w, const void* k, const void* v,
                               const void* a, const void* b, const float* s0,
                               const uint8_t* mask, const void* dout, const float* dsT, void* dr,
                               void* dw, void* dk, void* dv, void* da, void* db, float* ds0,
                               int B, int T, int H, int K, int V, const int32_t* cu_seqlens,
                               int N, wkv7_layout layout, wkv7_dtype dtype, wkv7_algo algo,
                               void* workspace, size_t workspace_bytes, void* stream_) {
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0 || N < 0) return WKV7_ERR_INVALID_ARG;
    if (algo != WKV7_ALGO_AUTO && algo != WKV7_ALGO_RECURRENT && algo != WKV7_ALGO_CHUNKED)
        return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (layout != WKV7_LAYOUT_BTHK && layout != WKV7_LAYOUT_BHTK) return WKV7_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1) return WKV7_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return WKV7_ERR_INVALID_ARG;
    } else if (N != B) {
        return WKV7_ERR_INVALID_ARG;
    }
    if (K != 64 || V != 64) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)N * H;
    if (units > 0x7fffffffLL || (long long)B * T * H > (1LL << 40)) return WKV7_ERR_UNSUPPORTED;
    if (units == 0) return WKV7_OK;
    const bool tokens = (long long)B * T > 0;
    if (tokens && (!ok_ptr(r) || !ok_ptr(w) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(a) ||
                   !ok_ptr(b) || !ok_ptr(dout) || !ok_ptr(dr) || !ok_ptr(dw) || !ok_ptr(dk) ||
                   !ok_ptr(dv) || !ok_ptr(da) || !ok_ptr(db)))
        return WKV7_ERR_INVALID_ARG;
    if ((s0 && !aligned16(s0)) || (dsT && !aligned16(dsT)) || (ds0 && !aligned16(ds0)))
        return WKV7_ERR_INVALID_ARG;
    const void* ins[8] = {r, w, k, v, a, b, dout, s0};
    const void* outs[7] = {dr, dw, dk, dv, da, db, ds0};
    for (const void* x : outs)
        for (const void* y : ins)
            if (x && x == y) return WKV7_ERR_INVALID_ARG;
    if (!ok_ptr(workspace) ||
        workspace_bytes < wkv7_bwd_workspace_bytes_algo(B, T, H, K, V, N, dtype, algo))
        return WKV7_ERR_INVALID_ARG;
    if (algo == WKV7_ALGO_CHUNKED && dtype != WKV7_BF16) return WKV7_ERR_UNSUPPORTED;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int hf = layout == WKV7_LAYOUT_BHTK;
    if (dtype == WKV7_BF16 && algo != WKV7_ALGO_RECURRENT) {
        const cudaError_t err = wkv7::launch_bwd_chunked(r, w, k, v, a, b, s0, mask, dout, dsT,
                                                         dr, dw, dk, dv, da, db, ds0, B, T, H, N,
                                                         cu_seqlens, hf, workspace, stream);
        return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
    }
    const cudaError_t err =
        dtype == WKV7_BF16
            ? wkv7::launch_bwd<__nv_bfloat16>(r, w, k, v, a, b, s0, mask, dout, dsT, dr, dw, dk,
                                              dv, da, db, ds0, B, T, H, N, cu_seqlens, hf,
                                              static_cast<float*>(workspace), stream)
            : wkv7::launch_bwd<float>(r, w, k, v, a, b, s0, mask, dout, dsT, dr, dw, dk, dv, da,
                                      db, ds0, B, T, H, N, cu_seqlens, hf,
                                      static_cast<float*>(workspace), stream);
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

size_t wkv7_gdn_bwd_workspace_bytes(int B, int T, int H, int K, int V, int N, wkv7_dtype dtype,
                                     int s0_shared) {
    if (B < 0 || T < 0 || H <= 0 || N < 0 || K != 64 || V != 64) return 0;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return 0;
    return wkv7::gdnb::workspace_bytes((long long)B * T, N, H, s0_shared != 0);
}

wkv7_status wkv7_bwd_noalloc(const void* r, const void* w, const void* k, const void* v,
                             const void* a, const void* b, const float* s0,
                             const uint8_t* mask, const void* dout, const float* dsT, void* dr,
                             void* dw, void* dk, void* dv, void* da, void* db, float* ds0, int B,
                             int T, int H, int K, int V, const int32_t* cu_seqlens, int N,
                             wkv7_layout layout, wkv7_dtype dtype, void* stream) {
    const size_t need = wkv7_bwd_workspace_bytes_algo(B, T, H, K, V, N, dtype, WKV7_ALGO_AUTO);
    if (need > kStaticScratchBytes) return WKV7_ERR_UNSUPPORTED;
    void* scratch = static_scratch_on_current_device();
    if (!scratch) return WKV7_ERR_CUDA;
    // the chunked forward runs must not make a handoff area here (they use an existing one
    // or run one unit per CTA)
    bool& forbid = wkv7::chunked::handoff_alloc_forbidden();
    forbid = true;
    const wkv7_status st = wkv7_bwd(r, w, k, v, a, b, s0, mask, dout, dsT, dr, dw, dk, dv, da,
                                    db, ds0, B, T, H, K, V, cu_seqlens, N, layout, dtype, scratch,
                                    kStaticScratchBytes, stream);
    forbid = false;
    return st;
}

wkv7_status wkv7_gdn_bwd(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* s0, int s0_shared, const void* dout,
                         const float* dsT, void* dq, void* dk, void* dv, void* dg, void* dbeta,
                         float* ds0, int B, int T, int H, int K, int V,
                         const int32_t* cu_seqlens, int N, wkv7_layout layout,
                         wkv7_dtype dtype, void* workspace, size_t workspace_bytes,
                         void* stream_) {
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0 || N < 0) return WKV7_ERR_INVALID_ARG;
    if (dtype != WKV7_BF16 && dtype != WKV7_F32) return WKV7_ERR_INVALID_ARG;
    if (layout != WKV7_LAYOUT_BTHK && layout != WKV7_LAYOUT_BHTK) return WKV7_ERR_INVALID_ARG;
    if (s0_shared != 0 && s0_shared != 1) return WKV7_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1) return WKV7_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return WKV7_ERR_INVALID_ARG;
    } else if (N != B) {
        return WKV7_ERR_INVALID_ARG;
    }
    if (K != 64 || V != 64) return WKV7_ERR_UNSUPPORTED;
    const long long units = (long long)N * H;
    if (units > 0x7fffffffLL || (long long)B * T * H > (1LL << 40)) return WKV7_ERR_UNSUPPORTED;
    if (units == 0) return WKV7_OK;
    const bool tokens = (long long)B * T > 0;
    if (tokens && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(dout) || !ok_ptr(dq) ||
                   !ok_ptr(dk) || !ok_ptr(dv) || !ok_scalar_ptr(g, dtype) ||
                   !ok_scalar_ptr(beta, dtype) || !ok_scalar_ptr(dg, dtype) ||
                   !ok_scalar_ptr(dbeta, dtype)))
        return WKV7_ERR_INVALID_ARG;
    if ((s0 && !aligned16(s0)) || (dsT && !aligned16(dsT)) || (ds0 && !aligned16(ds0)))
        return WKV7_ERR_INVALID_ARG;
    const void* ins[7] = {q, k, v, g, beta, dout, s0};
    const void* outs[6] = {dq, dk, dv, dg, dbeta, ds0};
    for (const void* x : outs)
        for (const void* y : ins)
            if (x && x == y) return WKV7_ERR_INVALID_ARG;
    if (!s0) s0_shared = 0;
    if (!ok_ptr(workspace) ||
        workspace_bytes < wkv7_gdn_bwd_workspace_bytes(B, T, H, K, V, N, dtype, s0_shared))
        return WKV7_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int hf = layout == WKV7_LAYOUT_BHTK;
    const cudaError_t err =
        dtype == WKV7_BF16
            ? wkv7::launch_gdn_bwd<__nv_bfloat16>(q, k, v, g, beta, s0, s0_shared, dout, dsT, dq,
                                                  dk, dv, dg, dbeta, ds0, B, T, H, N, cu_seqlens,
                                                  hf, workspace, stream)
            : wkv7::launch_gdn_bwd<float>(q, k, v, g, beta, s0, s0_shared, dout, dsT, dq, dk, dv,
                                          dg, dbeta, ds0, B, T, H, N, cu_seqlens, hf, workspace,
                                          stream);
    return err == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

wkv7_status wkv7_get_last_error(void* stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    unsigned int flags = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return WKV7_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&flags, wkv7::g_error_flags, sizeof(flags)) != cudaSuccess)
        return WKV7_ERR_CUDA;
    if (flags) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(wkv7::g_error_flags, &zero, sizeof(zero)) != cudaSuccess)
            return WKV7_ERR_CUDA;
        if (flags & (1u << WKV7_ERR_DEVICE_TIMEOUT)) return WKV7_ERR_DEVICE_TIMEOUT;
        if (flags & (1u << WKV7_ERR_DEVICE_BAD_SEQLENS)) return WKV7_ERR_DEVICE_BAD_SEQLENS;
        return WKV7_ERR_CUDA;
    }
    return WKV7_OK;
}

}  // extern "C"
