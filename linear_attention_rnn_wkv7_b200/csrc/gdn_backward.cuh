// gdn_backward.cuh -- backward of the Gated DeltaNet forward (gated_delta_net_recurrent /
// gated_delta_net_chunk support backpropagation; rwkv-ops 0.9.0 README,
// "gdn_recurrent 使用方法" and "gdn_chunk 使用方法"), through the generalized-rule
// backward of backward.cuh.
//
// Gated DeltaNet is the generalized rule with r = qh, w = g on every channel, write key
// beta kh, a = kh and b = -e^g beta kh (qh = q/|q|, kh = k/|k|, a zero vector stays
// zero).  Three steps on the stream, all in fp32 whatever the input type (rounding
// the substituted vectors to bf16 would perturb every transition by 2^-9):
//   gdn_map_kernel    writes those five inputs and v, dL/do as fp32 (one warp per
//                     token-head);
//   the generalized backward (checkpointing forward + reverse pass) on them;
//   gdn_chain_kernel  applies the chain rule per token-head:
//       dkh = beta dk_w + da - e^g beta db;  dg = sum(dw) + db . b;
//       dbeta = kh . dk_w - e^g (kh . db);
//       dq = (dr - qh (qh . dr)) / |q|,  dk = (dkh - kh (kh . dkh)) / |k|  (0 for a zero q, k).
// A [1, H, K, V] initial state shared by every sequence is expanded before and its
// gradient summed over the sequences after.
#pragma once
#include <algorithm>

#include "common.cuh"
#include "backward.cuh"

namespace wkv7 {

namespace gdnb {

// Sum over the 32 lanes of a warp.
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

constexpr int kWarps = 8;  // token-heads per block

template <typename Tin>
__global__ void __launch_bounds__(kWarps * 32)
gdn_map_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ g,
               const Tin* __restrict__ beta, const Tin* __restrict__ v,
               const Tin* __restrict__ dout, float* __restrict__ r, float* __restrict__ w,
               float* __restrict__ kw, float* __restrict__ a, float* __restrict__ b,
               float* __restrict__ v32, float* __restrict__ do32, long long rows) {
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (row >= rows) return;  // warp-uniform
    const int lane = threadIdx.x & 31;
    const size_t e = (size_t)row * 64 + 2 * lane;
    const float2 qq = load2(q + e), kk = load2(k + e);
    const float sq = warp_sum(qq.x * qq.x + qq.y * qq.y);
    const float sk = warp_sum(kk.x * kk.x + kk.y * kk.y);
    const float nq = sq > 0.f ? rsqrtf(sq) : 0.f, nk = sk > 0.f ? rsqrtf(sk) : 0.f;
    const float gv = to_f32(g[row]), bt = to_f32(beta[row]);
    const float eb = -expf(gv) * bt;
    const float k0 = kk.x * nk, k1 = kk.y * nk;
    *reinterpret_cast<float2*>(r + e) = make_float2(qq.x * nq, qq.y * nq);
    *reinterpret_cast<float2*>(w + e) = make_float2(gv, gv);
    *reinterpret_cast<float2*>(kw + e) = make_float2(bt * k0, bt * k1);
    *reinterpret_cast<float2*>(a + e) = make_float2(k0, k1);
    *reinterpret_cast<float2*>(b + e) = make_float2(eb * k0, eb * k1);
    *reinterpret_cast<float2*>(v32 + e) = load2(v + e);
    *reinterpret_cast<float2*>(do32 + e) = load2(dout + e);
}

template <typename Tin>
__global__ void __launch_bounds__(kWarps * 32)
gdn_chain_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ g,
                 const Tin* __restrict__ beta, const float* __restrict__ dr,
                 const float* __restrict__ dw, const float* __restrict__ dkw,
                 const float* __restrict__ da, const float* __restrict__ db,
                 const float* __restrict__ dv32, Tin* __restrict__ dq, Tin* __restrict__ dk,
                 Tin* __restrict__ dv, Tin* __restrict__ dg, Tin* __restrict__ dbeta,
                 long long rows) {
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (row >= rows) return;  // warp-uniform
    const int lane = threadIdx.x & 31;
    const size_t e = (size_t)row * 64 + 2 * lane;
    const float2 qq = load2(q + e), kk = load2(k + e);
    const float nq2 = warp_sum(qq.x * qq.x + qq.y * qq.y);
    const float nk2 = warp_sum(kk.x * kk.x + kk.y * kk.y);
    const float iq = nq2 > 0.f ? rsqrtf(nq2) : 0.f, ik = nk2 > 0.f ? rsqrtf(nk2) : 0.f;
    const float gv = to_f32(g[row]), bt = to_f32(beta[row]);
    const float eg = expf(gv);
    const float2 xr = load2(dr + e), xw = load2(dw + e), xk = load2(dkw + e);
    const float2 xa = load2(da + e), xb = load2(db + e);
    const float q0 = qq.x * iq, q1 = qq.y * iq, k0 = kk.x * ik, k1 = kk.y * ik;
    // dkh = beta dk_w + da - e^g beta db
    const float h0 = bt * xk.x + xa.x - eg * bt * xb.x;
    const float h1 = bt * xk.y + xa.y - eg * bt * xb.y;
    const float qdr = warp_sum(q0 * xr.x + q1 * xr.y);
    const float kdh = warp_sum(k0 * h0 + k1 * h1);
    const float sdw = warp_sum(xw.x + xw.y);
    const float kdb = warp_sum(k0 * xb.x + k1 * xb.y);
    const float kdk = warp_sum(k0 * xk.x + k1 * xk.y);
    dq[e] = from_f32<Tin>((xr.x - q0 * qdr) * iq);
    dq[e + 1] = from_f32<Tin>((xr.y - q1 * qdr) * iq);
    dk[e] = from_f32<Tin>((h0 - k0 * kdh) * ik);
    dk[e + 1] = from_f32<Tin>((h1 - k1 * kdh) * ik);
    const float2 xv = load2(dv32 + e);
    dv[e] = from_f32<Tin>(xv.x);
    dv[e + 1] = from_f32<Tin>(xv.y);
    if (lane == 0) {
        dg[row] = from_f32<Tin>(sdw - eg * bt * kdb);
        dbeta[row] = from_f32<Tin>(kdk - eg * kdb);
    }
}

// dst[n][h] = src[h] for every sequence n (a shared initial state, expanded).
__global__ void expand_state_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                    long long per, long long total) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x)
        dst[i] = src[i % per];
}

// dst[h] = sum over n of src[n][h] (the gradient of a shared initial state).
__global__ void sum_states_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                  long long per, int N) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < per;
         i += (long long)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int n = 0; n < N; ++n) acc += src[(size_t)n * per + i];
        dst[i] = acc;
    }
}

// Workspace layout (bytes, every part 256-byte aligned): seven fp32 [rows * H, 64]
// inputs of the generalized backward (r, w, k_w, a, b, v, dL/do) and its six fp32
// gradients (dr, dw, dk_w, da, db, dv), the expanded initial state and its gradient
// ([N, H, 64, 64] fp32 each, when the state is shared), then the generalized backward's
// own workspace.
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline size_t workspace_bytes(long long rows, int N, int H, bool shared) {
    const size_t vec = align256((size_t)rows * H * 64 * sizeof(float));
    const size_t st = shared ? 2 * align256((size_t)N * H * 4096 * sizeof(float)) : 0;
    return 13 * vec + st + align256(bwd::workspace_floats(rows, N, H) * sizeof(float));
}

}  // namespace gdnb

template <typename Tin>
cudaError_t launch_gdn_bwd(const void* q, const void* k, const void* v, const void* g,
                           const void* beta, const float* s0, int s0_shared, const void* dout,
                           const float* dsT, void* dq, void* dk, void* dv, void* dg,
                           void* dbeta, float* ds0, int B, int T, int H, int N,
                           const int32_t* cu_seqlens, int head_first, void* ws,
                           cudaStream_t stream) {
    using namespace gdnb;
    const long long rows = (long long)B * T;
    const long long th = rows * H;  // token-heads
    const size_t vec = align256((size_t)th * 64 * sizeof(float));
    uint8_t* p = static_cast<uint8_t*>(ws);
    float* m[7];   // r, w, k_w, a, b, v, dL/do
    float* gr[6];  // dr, dw, dk_w, da, db, dv
    for (int i = 0; i < 7; ++i) m[i] = reinterpret_cast<float*>(p + i * vec);
    for (int i = 0; i < 6; ++i) gr[i] = reinterpret_cast<float*>(p + (7 + i) * vec);
    p += 13 * vec;
    const float* s0x = s0;
    float* ds0x = ds0;
    const long long per = (long long)H * 4096;
    if (s0_shared && s0) {
        const size_t st = align256((size_t)N * per * sizeof(float));
        float* e0 = reinterpret_cast<float*>(p);
        ds0x = ds0 ? reinterpret_cast<float*>(p + st) : nullptr;
        p += 2 * st;
        const long long total = (long long)N * per;
        expand_state_kernel<<<(unsigned)std::min<long long>((total + 255) / 256, 4096), 256, 0,
                              stream>>>(s0, e0, per, total);
        s0x = e0;
    }
    const unsigned blocks = (unsigned)((th + kWarps - 1) / kWarps);
    if (th > 0)
        gdn_map_kernel<Tin><<<blocks, kWarps * 32, 0, stream>>>(
            static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(g),
            static_cast<const Tin*>(beta), static_cast<const Tin*>(v),
            static_cast<const Tin*>(dout), m[0], m[1], m[2], m[3], m[4], m[5], m[6], th);
    cudaError_t err = launch_bwd<float>(m[0], m[1], m[2], m[5], m[3], m[4], s0x, nullptr, m[6],
                                        dsT, gr[0], gr[1], gr[2], gr[5], gr[3], gr[4], ds0x, B,
                                        T, H, N, cu_seqlens, head_first,
                                        reinterpret_cast<float*>(p), stream);
    if (err != cudaSuccess) return err;
    if (th > 0)
        gdn_chain_kernel<Tin><<<blocks, kWarps * 32, 0, stream>>>(
            static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(g),
            static_cast<const Tin*>(beta), gr[0], gr[1], gr[2], gr[3], gr[4], gr[5],
            static_cast<Tin*>(dq), static_cast<Tin*>(dk), static_cast<Tin*>(dv),
            static_cast<Tin*>(dg), static_cast<Tin*>(dbeta), th);
    if (s0_shared && s0 && ds0)
        sum_states_kernel<<<(unsigned)std::min<long long>((per + 255) / 256, 4096), 256, 0,
                            stream>>>(ds0x, ds0, per, N);
    return cudaGetLastError();
}

}  // namespace wkv7
