// recurrent.cuh -- token-by-token WKV7 forward on CUDA cores, fp32 throughout.
//
// The recurrence (rwkv-ops 0.9.0 README, "rwkv7op 使用方法"):
//     u_t = S_{t-1}^T a_t;  S_t = diag(exp w_t) S_{t-1} + b_t u_t^T + k_t v_t^T;  o_t = S_t^T r_t
// decouples over the V columns of the state: column j only needs u_t[j],
// which is the dot product of column j with a_t.  So one thread owns one state
// column (64 fp32 registers) and every reduction over K stays inside a thread;
// a block of 64 threads owns one (sequence, head).  Tokens are staged 16 at a
// time in shared memory (r, exp(w), k, a, b, v as fp32) so that each thread
// reads the shared vectors as float4 broadcasts.
//
// This is the fp32-input path (its accuracy is that of an fp32 recurrence)
// and the anchor the chunked tensor-core kernel is checked against; masks,
// packed varlen sequences and null s0 / sT are handled here exactly as in the
// chunked kernel.
//
// kGdn: Gated DeltaNet (rwkv-ops 0.9.0 README, "gdn_recurrent 使用方法").  The
// staging turns q, k, v, g, beta into the generalized rule's per-token vectors:
// r = qh, exp(w) = e^{g} on every channel, write key beta kh, a = kh and
// b = -e^{g} beta kh (qh, kh: q and k over their L2 norms), so the loop below
// applies e^{g} (I - beta kh kh^T) S + beta kh v^T.
#pragma once
#include "common.cuh"

namespace wkv7 {

constexpr int kRecTile = 16;

template <typename Tin, bool kGdn>
__global__ void __launch_bounds__(64)
recurrent_kernel(const Tin* __restrict__ r, const Tin* __restrict__ w, const Tin* __restrict__ k,
                 const Tin* __restrict__ v, const Tin* __restrict__ a, const Tin* __restrict__ b,
                 const float* s0, const uint8_t* __restrict__ mask, Tin* __restrict__ o,
                 float* sT, int T, int H, const int32_t* __restrict__ cu_seqlens,
                 const Tin* __restrict__ g, const Tin* __restrict__ beta, int s0_shared) {
    __shared__ __align__(16) float sm[6][kRecTile][64];  // r, d, k, a, b, v
    __shared__ uint8_t smask[kRecTile];
    __shared__ float sgb[4][kRecTile];  // Gated DeltaNet: g, beta, 1/|q|, 1/|k|

    const int h = blockIdx.x % H;
    const int n = blockIdx.x / H;
    const int j = threadIdx.x;
    int bb = n, bos = 0, eos = T;
    if (cu_seqlens) {
        bb = 0;
        bos = cu_seqlens[n];
        eos = cu_seqlens[n + 1];
        if (bos < 0 || eos < bos || eos > T) {  // block-uniform
            if (j == 0) raise_flag(5 /* WKV7_ERR_DEVICE_BAD_SEQLENS */);
            return;
        }
    }
    const size_t state_off = ((size_t)n * H + h) * 4096;
    const size_t init_off = s0_shared ? (size_t)h * 4096 : state_off;

    float S[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) S[i] = s0 ? s0[init_off + i * 64 + j] : 0.f;

    for (int t0 = bos; t0 < eos; t0 += kRecTile) {
        const int cnt = min(kRecTile, eos - t0);
        __syncthreads();
        if constexpr (kGdn) {
            for (int tt = 0; tt < cnt; ++tt) {
                const size_t row = (((size_t)bb * T + t0 + tt) * H + h) * 64;
                sm[0][tt][j] = to_f32(r[row + j]);  // q
                sm[3][tt][j] = to_f32(k[row + j]);
                sm[5][tt][j] = to_f32(v[row + j]);
            }
            if (j < cnt) {
                const size_t tok = ((size_t)bb * T + t0 + j) * H + h;
                sgb[0][j] = to_f32(g[tok]);
                sgb[1][j] = to_f32(beta[tok]);
                smask[j] = 1;
            }
            __syncthreads();
            if (j < 2 * cnt) {  // thread 2 tt + e: the inverse norm of q (e = 0) or k (e = 1)
                const float* x = sm[(j & 1) ? 3 : 0][j >> 1];
                float ss = 0.f;
                for (int i = 0; i < 64; ++i) ss = fmaf(x[i], x[i], ss);
                sgb[2 + (j & 1)][j >> 1] = ss > 0.f ? rsqrtf(ss) : 0.f;  // zero stays zero
            }
            __syncthreads();
            for (int tt = 0; tt < cnt; ++tt) {
                const float kn = sm[3][tt][j] * sgb[3][tt];
                const float alpha = expf(sgb[0][tt]), bt = sgb[1][tt];
                sm[0][tt][j] *= sgb[2][tt];
                sm[1][tt][j] = alpha;
                sm[2][tt][j] = bt * kn;
                sm[3][tt][j] = kn;
                sm[4][tt][j] = -alpha * bt * kn;
            }
        } else {
            for (int tt = 0; tt < cnt; ++tt) {
                const size_t row = (((size_t)bb * T + t0 + tt) * H + h) * 64;
                sm[0][tt][j] = to_f32(r[row + j]);
                sm[1][tt][j] = expf(to_f32(w[row + j]));
                sm[2][tt][j] = to_f32(k[row + j]);
                sm[3][tt][j] = to_f32(a[row + j]);
                sm[4][tt][j] = to_f32(b[row + j]);
                sm[5][tt][j] = to_f32(v[row + j]);
            }
            if (j < cnt) smask[j] = mask ? (mask[(size_t)bb * T + t0 + j] != 0) : 1;
        }
        __syncthreads();

        for (int tt = 0; tt < cnt; ++tt) {
            if (smask[tt]) {
                const float4* a4 = reinterpret_cast<const float4*>(sm[3][tt]);
                float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
#pragma unroll
                for (int i4 = 0; i4 < 16; ++i4) {
                    const float4 av = a4[i4];
                    u0 = fmaf(S[4 * i4 + 0], av.x, u0);
                    u1 = fmaf(S[4 * i4 + 1], av.y, u1);
                    u2 = fmaf(S[4 * i4 + 2], av.z, u2);
                    u3 = fmaf(S[4 * i4 + 3], av.w, u3);
                }
                const float u = (u0 + u1) + (u2 + u3);
                const float vj = sm[5][tt][j];
                const float4* d4 = reinterpret_cast<const float4*>(sm[1][tt]);
                const float4* k4 = reinterpret_cast<const float4*>(sm[2][tt]);
                const float4* b4 = reinterpret_cast<const float4*>(sm[4][tt]);
#pragma unroll
                for (int i4 = 0; i4 < 16; ++i4) {
                    const float4 dv = d4[i4], kv = k4[i4], bv = b4[i4];
                    S[4 * i4 + 0] = fmaf(S[4 * i4 + 0], dv.x, fmaf(bv.x, u, kv.x * vj));
                    S[4 * i4 + 1] = fmaf(S[4 * i4 + 1], dv.y, fmaf(bv.y, u, kv.y * vj));
                    S[4 * i4 + 2] = fmaf(S[4 * i4 + 2], dv.z, fmaf(bv.z, u, kv.z * vj));
                    S[4 * i4 + 3] = fmaf(S[4 * i4 + 3], dv.w, fmaf(bv.w, u, kv.w * vj));
                }
            }
            const float4* r4 = reinterpret_cast<const float4*>(sm[0][tt]);
            float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {
                const float4 rv = r4[i4];
                o0 = fmaf(S[4 * i4 + 0], rv.x, o0);
                o1 = fmaf(S[4 * i4 + 1], rv.y, o1);
                o2 = fmaf(S[4 * i4 + 2], rv.z, o2);
                o3 = fmaf(S[4 * i4 + 3], rv.w, o3);
            }
            const size_t row = (((size_t)bb * T + t0 + tt) * H + h) * 64;
            o[row + j] = from_f32<Tin>((o0 + o1) + (o2 + o3));
        }
    }
    if (sT) {
#pragma unroll
        for (int i = 0; i < 64; ++i) sT[state_off + i * 64 + j] = S[i];
    }
}

template <typename Tin>
cudaError_t launch_recurrent(const void* r, const void* w, const void* k, const void* v,
                             const void* a, const void* b, const float* s0,
                             const uint8_t* mask, void* o, float* sT, int T, int H, int N,
                             const int32_t* cu_seqlens, cudaStream_t stream) {
    const long long blocks = (long long)N * H;
    recurrent_kernel<Tin, false><<<(unsigned)blocks, 64, 0, stream>>>(
        static_cast<const Tin*>(r), static_cast<const Tin*>(w), static_cast<const Tin*>(k),
        static_cast<const Tin*>(v), static_cast<const Tin*>(a), static_cast<const Tin*>(b), s0,
        mask, static_cast<Tin*>(o), sT, T, H, cu_seqlens, nullptr, nullptr, 0);
    return cudaGetLastError();
}

// Gated DeltaNet: q, k [rows, H, 64], v [rows, H, 64], g, beta [rows, H].
template <typename Tin>
cudaError_t launch_recurrent_gdn(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* s0, int s0_shared, void* o,
                                 float* sT, int T, int H, int N, const int32_t* cu_seqlens,
                                 cudaStream_t stream) {
    const long long blocks = (long long)N * H;
    recurrent_kernel<Tin, true><<<(unsigned)blocks, 64, 0, stream>>>(
        static_cast<const Tin*>(q), nullptr, static_cast<const Tin*>(k),
        static_cast<const Tin*>(v), nullptr, nullptr, s0, nullptr, static_cast<Tin*>(o), sT, T,
        H, cu_seqlens, static_cast<const Tin*>(g), static_cast<const Tin*>(beta), s0_shared);
    return cudaGetLastError();
}

}  // namespace wkv7
