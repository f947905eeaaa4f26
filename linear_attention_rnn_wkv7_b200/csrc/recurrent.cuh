// recurrent.cuh -- token-by-token WKV7 forward on CUDA cores, fp32 throughout.
//
// The recurrence (rwkv-ops 0.9.0 README, "rwkv7op 使用方法"):
//     u_t = S_{t-1}^T a_t;  S_t = diag(exp w_t) S_{t-1} + b_t u_t^T + k_t v_t^T;  o_t = S_t^T r_t
// decouples over the V columns of the state: column j only needs u_t[j],
// which is the dot product of column j with a_t.  So a block owns a slab of 64
// state columns of one (sequence, head), and each column is held by P = K / 64
// threads of adjacent lanes, 64 rows (64 fp32 registers) each: the reductions over
// K are a thread's own sum plus log2(P) shuffles.  K = V = 64 is one block of 64
// threads per (sequence, head); the README's other head sizes (128, 256) take
// K / 64 column slabs of 64 x P threads, every slab reading the whole K-side vectors.
// (Four threads per column at every head size, i.e. more warps with shorter
// chains, measured slower: the extra shuffles sit on each token's dependency chain.)
//
// Tokens go through shared memory in tiles of 512 / K: while a tile is computed,
// cp.async copies the next tile's raw inputs (r, w, k, a, b rows and the slab's 64
// entries of v) into the other half of a double buffer, so the recurrence never
// waits for global memory.  Each tile is then converted once to fp32 (exp(w)
// included) in a layout whose 64-float parts are 68 floats apart, so the P parts a
// warp reads as float4 broadcasts sit in different banks.
//
// This is the fp32-input path (its accuracy is that of an fp32 recurrence)
// and the anchor the chunked tensor-core kernel is checked against; masks,
// packed varlen sequences and null s0 / sT are handled here exactly as in the
// chunked kernel.
//
// kSane: State Anomaly Neutralization (rwkv-ops 0.9.0 README, "rwkv7op_sane 使用方法"):
// after token 16 c + 15 of a sequence (c < T / 16, a full 16-token chunk) whose flag
// sane[b, c] is set (no flags: every chunk), each state entry is soft-clipped,
// S <- tau * tanh(S / tau) with tau = tau[b, c, h] > 0.  The token's output is read
// before the clip.  The README defers the clip function to its paper; tau * tanh(S /
// tau) is the reading taken (the state stays within (-tau, tau) and is unchanged to
// first order where |S| << tau).
//
// kGdn: Gated DeltaNet (rwkv-ops 0.9.0 README, "gdn_recurrent 使用方法").  The
// conversion turns q, k, v, g, beta into the generalized rule's per-token vectors:
// r = qh, exp(w) = e^{g} on every channel, write key beta kh, a = kh and
// b = -e^{g} beta kh (qh, kh: q and k over their L2 norms), so the loop below
// applies e^{g} (I - beta kh kh^T) S + beta kh v^T.
#pragma once
#include "common.cuh"

namespace wkv7 {

namespace rec {

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace rec

// K (= V): head size.  Block: 64 columns x P = K / 64 threads per column, 64 rows each.
template <typename Tin, bool kGdn, int K, bool kSane = false>
__global__ void __launch_bounds__(K)
recurrent_kernel(const Tin* __restrict__ r, const Tin* __restrict__ w, const Tin* __restrict__ k,
                 const Tin* __restrict__ v, const Tin* __restrict__ a, const Tin* __restrict__ b,
                 const float* s0, const uint8_t* __restrict__ mask, Tin* __restrict__ o,
                 float* sT, int T, int H, const int32_t* __restrict__ cu_seqlens,
                 const Tin* __restrict__ g, const Tin* __restrict__ beta, int s0_shared,
                 int head_first, const float* __restrict__ tau,
                 const uint8_t* __restrict__ sane_flags) {
    using namespace rec;
    constexpr int P = K / 64;        // threads per state column
    constexpr int R = 64;            // rows per thread
    constexpr int kSeg = R + 4;      // floats between the parts of a converted row
    constexpr int kThreads = K;
    constexpr int kTile = 512 / K;   // tokens per tile
    constexpr int kSlabs = K / 64;   // 64-column slabs per (sequence, head)
    constexpr int KP = P * kSeg;     // converted row length (padded parts)
    constexpr int EPC = 16 / (int)sizeof(Tin);  // elements per 16-byte copy
    constexpr int CR = K / EPC;      // copies per K-row
    constexpr int CV = 64 / EPC;     // copies per v slab row
    constexpr int NV = kGdn ? 2 : 5; // K-rows per token: q, k  or  r, w, k, a, b
    constexpr int PER_TOK = NV * CR + CV;
    __shared__ __align__(16) Tin raw[2][5][kTile][K];  // r (q), w, k, a, b as loaded
    __shared__ __align__(16) Tin rawv[2][kTile][64];
    __shared__ __align__(16) float sm[5][kTile][KP];   // r, d = exp(w), k, a, b (fp32)
    __shared__ __align__(16) float sv[kTile][64];      // this slab's v
    __shared__ uint8_t smask[kTile];
    __shared__ float sgb[4][kTile];  // Gated DeltaNet: g, beta, 1/|q|, 1/|k|

    const int slab = blockIdx.x % kSlabs;
    const int unit = blockIdx.x / kSlabs;
    const int h = unit % H;
    const int n = unit / H;
    const int tid = threadIdx.x;
    const int c = tid / P, part = tid % P;  // column of the slab, R-row part of it
    const int col = 64 * slab + c;          // state column
    int bb = n, bos = 0, eos = T;
    if (cu_seqlens) {
        bb = 0;
        bos = cu_seqlens[n];
        eos = cu_seqlens[n + 1];
        if (bos < 0 || eos < bos || eos > T) {  // block-uniform
            if (tid == 0 && slab == 0) raise_flag(5 /* WKV7_ERR_DEVICE_BAD_SEQLENS */);
            return;
        }
    }
    // token t of this unit is row tb + t * ts of the [*, K] inputs and outputs (and
    // element tb + t * ts of g and beta): [B, T, H, *] or, head first, [B, H, T, *]
    const size_t tb = head_first ? ((size_t)bb * H + h) * T : (size_t)bb * T * H + h;
    const size_t ts = head_first ? 1 : (size_t)H;
    const size_t state_off = ((size_t)n * H + h) * K * K;
    const size_t init_off = s0_shared ? (size_t)h * K * K : state_off;

    // Copies of tile [t0, t0 + cnt) into buffer buf; per-token scalars (mask or g,
    // beta) are read into registers here and stored at the tile's conversion.
    float pre_g = 0.f, pre_b = 0.f;
    uint8_t pre_m = 1;
    auto issue = [&](int buf, int t0, int cnt) {
        for (int idx = tid; idx < cnt * PER_TOK; idx += kThreads) {
            const int tt = idx / PER_TOK, rem = idx - tt * PER_TOK;
            const size_t row = (tb + (size_t)(t0 + tt) * ts) * K;
            if (rem < NV * CR) {
                const int vi = rem / CR, e = (rem - vi * CR) * EPC;
                const int slot = kGdn ? 2 * vi : vi;  // q -> slot 0, k -> slot 2
                const Tin* src = slot == 0 ? r : slot == 1 ? w : slot == 2 ? k : slot == 3 ? a : b;
                cp_async16(&raw[buf][slot][tt][e], src + row + e);
            } else {
                const int e = (rem - NV * CR) * EPC;
                cp_async16(&rawv[buf][tt][e], v + row + 64 * slab + e);
            }
        }
        if (tid < cnt) {
            const size_t tok = tb + (size_t)(t0 + tid) * ts;
            if constexpr (kGdn) {
                pre_g = to_f32(g[tok]);
                pre_b = to_f32(beta[tok]);
            } else {
                pre_m = mask ? (mask[(size_t)bb * T + t0 + tid] != 0) : 1;
            }
        }
    };

    float S[R];  // rows R part .. R part + R - 1 of column col
#pragma unroll
    for (int i = 0; i < R; ++i)
        S[i] = s0 ? s0[init_off + (size_t)(R * part + i) * K + col] : 0.f;

    if (bos < eos) issue(0, bos, min(kTile, eos - bos));
    cp_async_commit();
    const int pe = tid + (kSeg - R) * (tid / R);  // element tid, padded
    for (int t0 = bos, buf = 0; t0 < eos; t0 += kTile, buf ^= 1) {
        const int cnt = min(kTile, eos - t0);
        const float my_g = pre_g, my_b = pre_b;
        const uint8_t my_m = pre_m;
        if (t0 + kTile < eos) issue(buf ^ 1, t0 + kTile, min(kTile, eos - t0 - kTile));
        cp_async_commit();
        cp_async_wait<1>();  // this tile's copies (the next tile's may still be in flight)
        __syncthreads();     // every thread's copies visible; the last tile's reads done
        if constexpr (kGdn) {
            if (tid < cnt) {
                sgb[0][tid] = my_g;
                sgb[1][tid] = my_b;
                smask[tid] = 1;
            }
            if (tid < 2 * cnt) {  // thread 2 tt + e: the inverse norm of q (e = 0) or k (e = 1)
                const Tin* x = raw[buf][(tid & 1) ? 2 : 0][tid >> 1];
                float ss = 0.f;
                for (int i = 0; i < K; ++i) {
                    const float xi = to_f32(x[i]);
                    ss = fmaf(xi, xi, ss);
                }
                sgb[2 + (tid & 1)][tid >> 1] = ss > 0.f ? rsqrtf(ss) : 0.f;  // zero stays zero
            }
            __syncthreads();
            for (int tt = 0; tt < cnt; ++tt) {
                const float kn = to_f32(raw[buf][2][tt][tid]) * sgb[3][tt];
                const float alpha = expf(sgb[0][tt]), bt = sgb[1][tt];
                sm[0][tt][pe] = to_f32(raw[buf][0][tt][tid]) * sgb[2][tt];
                sm[1][tt][pe] = alpha;
                sm[2][tt][pe] = bt * kn;
                sm[3][tt][pe] = kn;
                sm[4][tt][pe] = -alpha * bt * kn;
                if (tid < 64) sv[tt][tid] = to_f32(rawv[buf][tt][tid]);
            }
        } else {
            for (int tt = 0; tt < cnt; ++tt) {
                sm[0][tt][pe] = to_f32(raw[buf][0][tt][tid]);
                sm[1][tt][pe] = expf(to_f32(raw[buf][1][tt][tid]));
                sm[2][tt][pe] = to_f32(raw[buf][2][tt][tid]);
                sm[3][tt][pe] = to_f32(raw[buf][3][tt][tid]);
                sm[4][tt][pe] = to_f32(raw[buf][4][tt][tid]);
                if (tid < 64) sv[tt][tid] = to_f32(rawv[buf][tt][tid]);
            }
            if (tid < cnt) smask[tid] = my_m;
        }
        __syncthreads();

        for (int tt = 0; tt < cnt; ++tt) {
            if (smask[tt]) {
                const float4* a4 = reinterpret_cast<const float4*>(sm[3][tt] + kSeg * part);
                float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
#pragma unroll
                for (int i4 = 0; i4 < R / 4; ++i4) {
                    const float4 av = a4[i4];
                    u0 = fmaf(S[4 * i4 + 0], av.x, u0);
                    u1 = fmaf(S[4 * i4 + 1], av.y, u1);
                    u2 = fmaf(S[4 * i4 + 2], av.z, u2);
                    u3 = fmaf(S[4 * i4 + 3], av.w, u3);
                }
                float u = (u0 + u1) + (u2 + u3);
#pragma unroll
                for (int m = 1; m < P; m *= 2) u += __shfl_xor_sync(0xffffffffu, u, m);
                const float vj = sv[tt][c];
                const float4* d4 = reinterpret_cast<const float4*>(sm[1][tt] + kSeg * part);
                const float4* k4 = reinterpret_cast<const float4*>(sm[2][tt] + kSeg * part);
                const float4* b4 = reinterpret_cast<const float4*>(sm[4][tt] + kSeg * part);
#pragma unroll
                for (int i4 = 0; i4 < R / 4; ++i4) {
                    const float4 dv = d4[i4], kv = k4[i4], bv = b4[i4];
                    S[4 * i4 + 0] = fmaf(S[4 * i4 + 0], dv.x, fmaf(bv.x, u, kv.x * vj));
                    S[4 * i4 + 1] = fmaf(S[4 * i4 + 1], dv.y, fmaf(bv.y, u, kv.y * vj));
                    S[4 * i4 + 2] = fmaf(S[4 * i4 + 2], dv.z, fmaf(bv.z, u, kv.z * vj));
                    S[4 * i4 + 3] = fmaf(S[4 * i4 + 3], dv.w, fmaf(bv.w, u, kv.w * vj));
                }
            }
            const float4* r4 = reinterpret_cast<const float4*>(sm[0][tt] + kSeg * part);
            float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
            for (int i4 = 0; i4 < R / 4; ++i4) {
                const float4 rv = r4[i4];
                o0 = fmaf(S[4 * i4 + 0], rv.x, o0);
                o1 = fmaf(S[4 * i4 + 1], rv.y, o1);
                o2 = fmaf(S[4 * i4 + 2], rv.z, o2);
                o3 = fmaf(S[4 * i4 + 3], rv.w, o3);
            }
            float ov = (o0 + o1) + (o2 + o3);
#pragma unroll
            for (int m = 1; m < P; m *= 2) ov += __shfl_xor_sync(0xffffffffu, ov, m);
            if (part == 0) {
                const size_t row = (tb + (size_t)(t0 + tt) * ts) * K;
                o[row + col] = from_f32<Tin>(ov);
            }
            if constexpr (kSane) {  // the output above was read before the clip
                const int tg = t0 + tt, ch = tg >> 4, C = T >> 4;  // no packed sequences here
                if ((tg & 15) == 15 && ch < C &&
                    (!sane_flags || sane_flags[(size_t)bb * C + ch] != 0)) {
                    const float tc = tau[((size_t)bb * C + ch) * H + h];
#pragma unroll
                    for (int i = 0; i < R; ++i) S[i] = tc * tanhf(S[i] / tc);
                }
            }
        }
    }
    cp_async_wait<0>();  // nothing is left in flight when the block exits
    if (sT) {
#pragma unroll
        for (int i = 0; i < R; ++i) sT[state_off + (size_t)(R * part + i) * K + col] = S[i];
    }
}

template <typename Tin, bool kGdn, int K, bool kSane = false>
cudaError_t launch_recurrent_k(const void* r, const void* w, const void* k, const void* v,
                               const void* a, const void* b, const float* s0,
                               const uint8_t* mask, void* o, float* sT, int T, int H, int N,
                               const int32_t* cu_seqlens, const void* g, const void* beta,
                               int s0_shared, int head_first, cudaStream_t stream,
                               const float* tau = nullptr, const uint8_t* sane_flags = nullptr) {
    const long long blocks = (long long)N * H * (K / 64);
    recurrent_kernel<Tin, kGdn, K, kSane><<<(unsigned)blocks, K, 0, stream>>>(
        static_cast<const Tin*>(r), static_cast<const Tin*>(w), static_cast<const Tin*>(k),
        static_cast<const Tin*>(v), static_cast<const Tin*>(a), static_cast<const Tin*>(b), s0,
        mask, static_cast<Tin*>(o), sT, T, H, cu_seqlens, static_cast<const Tin*>(g),
        static_cast<const Tin*>(beta), s0_shared, head_first, tau, sane_flags);
    return cudaGetLastError();
}

template <typename Tin, bool kGdn>
cudaError_t launch_recurrent_any(int K, const void* r, const void* w, const void* k,
                                 const void* v, const void* a, const void* b, const float* s0,
                                 const uint8_t* mask, void* o, float* sT, int T, int H, int N,
                                 const int32_t* cu_seqlens, const void* g, const void* beta,
                                 int s0_shared, int head_first, cudaStream_t stream) {
    switch (K) {
        case 64:
            return launch_recurrent_k<Tin, kGdn, 64>(r, w, k, v, a, b, s0, mask, o, sT, T, H, N,
                                                     cu_seqlens, g, beta, s0_shared, head_first,
                                                     stream);
        case 128:
            return launch_recurrent_k<Tin, kGdn, 128>(r, w, k, v, a, b, s0, mask, o, sT, T, H, N,
                                                      cu_seqlens, g, beta, s0_shared, head_first,
                                                      stream);
        case 256:
            return launch_recurrent_k<Tin, kGdn, 256>(r, w, k, v, a, b, s0, mask, o, sT, T, H, N,
                                                      cu_seqlens, g, beta, s0_shared, head_first,
                                                      stream);
    }
    return cudaErrorInvalidValue;
}

// WKV7: r, w, k, a, b [rows, H, K], v and o [rows, H, K] (K = V in {64, 128, 256}).
template <typename Tin>
cudaError_t launch_recurrent(const void* r, const void* w, const void* k, const void* v,
                             const void* a, const void* b, const float* s0,
                             const uint8_t* mask, void* o, float* sT, int T, int H, int N,
                             const int32_t* cu_seqlens, int head_first, int K,
                             cudaStream_t stream) {
    return launch_recurrent_any<Tin, false>(K, r, w, k, v, a, b, s0, mask, o, sT, T, H, N,
                                            cu_seqlens, nullptr, nullptr, 0, head_first, stream);
}

// Gated DeltaNet: q, k [rows, H, K], v [rows, H, K], g, beta [rows, H].
template <typename Tin>
cudaError_t launch_recurrent_gdn(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* s0, int s0_shared, void* o,
                                 float* sT, int T, int H, int N, const int32_t* cu_seqlens,
                                 int head_first, int K, cudaStream_t stream) {
    return launch_recurrent_any<Tin, true>(K, q, nullptr, k, v, nullptr, nullptr, s0, nullptr,
                                           o, sT, T, H, N, cu_seqlens, g, beta, s0_shared,
                                           head_first, stream);
}

// SANE forward: the WKV7 recurrence with the soft clip after every 16th token (kSane);
// tau [B, T / 16, H] fp32, sane_flags [B, T / 16] (or NULL: every full chunk); no mask and
// no packed sequences; s0 may be one [1, H, K, V] state shared by every batch row.
template <typename Tin>
cudaError_t launch_recurrent_sane(const void* r, const void* w, const void* k, const void* v,
                                  const void* a, const void* b, const float* tau,
                                  const uint8_t* sane_flags, const float* s0, int s0_shared,
                                  void* o, float* sT, int B, int T, int H, int head_first, int K,
                                  cudaStream_t stream) {
    switch (K) {
        case 64:
            return launch_recurrent_k<Tin, false, 64, true>(r, w, k, v, a, b, s0, nullptr, o, sT, T,
                                                            H, B, nullptr, nullptr, nullptr,
                                                            s0_shared, head_first, stream, tau,
                                                            sane_flags);
        case 128:
            return launch_recurrent_k<Tin, false, 128, true>(r, w, k, v, a, b, s0, nullptr, o, sT,
                                                             T, H, B, nullptr, nullptr, nullptr,
                                                             s0_shared, head_first, stream, tau,
                                                             sane_flags);
        case 256:
            return launch_recurrent_k<Tin, false, 256, true>(r, w, k, v, a, b, s0, nullptr, o, sT,
                                                             T, H, B, nullptr, nullptr, nullptr,
                                                             s0_shared, head_first, stream, tau,
                                                             sane_flags);
    }
    return cudaErrorInvalidValue;
}

}  // namespace wkv7
