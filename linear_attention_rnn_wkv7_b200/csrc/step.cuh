// step.cuh -- single-token WKV7 decode step (rwkv7_op_rnn, rwkv-ops 0.9.0
// README, "rwkv7_op_rnn 使用方法": the T = 1 case used for decoding).
//
// Per (batch, head) unit the 64 x 64 fp32 state is read from HBM once,
// updated and written back once:
//     u = S^T a;   S <- diag(exp w) S + b u^T + k v^T;   o = S^T r.
// The step is purely HBM-bound (32 KiB of state traffic per unit against
// ~9 flops per state element), so the kernel is organised around coalesced
// 128-bit state loads and stores and enough bytes in flight per SM:
//   - one warp owns one unit; lane l holds columns 4*(l%16) .. +3 of rows
//     32*(l/16) .. +31, i.e. 32 float4 registers;  one warp-wide load
//     instruction covers two full 256-byte state rows;
//   - the two K-halves of u = S^T a and o = S^T r are combined with one
//     shuffle (xor 16) per column;
//   - the per-token vectors (r, exp w, k, a, b) go through a 1.25 KiB per-warp
//     shared-memory stage so each lane reads its 32 rows as float4 broadcasts.
//
// kGdn: the Gated DeltaNet single step (rwkv-ops 0.9.0 README,
// gated_delta_net_recurrent_single_step).  The stage holds r = qh, exp(w) = e^{g},
// write key beta kh, a = kh, b = -e^{g} beta kh (qh, kh: q and k over their L2
// norms, reduced across the warp), so the same update applies
// e^{g} (I - beta kh kh^T) S + beta kh v^T.
//
// kSane: rwkv7_op_sane_rnn (rwkv-ops 0.9.0 README, "rwkv7_op_sane_rnn 使用方法"): when
// the unit's batch row is flagged (do_sane[b], or one flag for all), the state written
// back is soft-clipped, S <- tau * tanh(S / tau) with tau[b, h] > 0, while the output
// is read from the state before the clip (the reading of the clip function is the
// forward's, see recurrent.cuh).
//
// Head sizes 128 and 256 (step_kernel_wide): one block per (unit, 64-column slab)
// with K / 64 warps, warp p holding rows 64 p .. 64 p + 63 of the slab in the same
// lane layout as above; the K-reductions of u and o add the warps' partial sums
// through shared memory (two block barriers per step).
#pragma once
#include "common.cuh"

namespace wkv7 {

constexpr int kStepWarps = 4;  // units per block

// Soft clip of the SANE step (4 state entries).
__device__ __forceinline__ float4 sane_clip4(float4 s, float tc) {
    return make_float4(tc * tanhf(s.x / tc), tc * tanhf(s.y / tc), tc * tanhf(s.z / tc),
                       tc * tanhf(s.w / tc));
}

template <typename Tin, bool kGdn, bool kSane = false>
__global__ void __launch_bounds__(kStepWarps * 32)
step_kernel(const Tin* __restrict__ r, const Tin* __restrict__ w, const Tin* __restrict__ k,
            const Tin* __restrict__ v, const Tin* __restrict__ a, const Tin* __restrict__ b,
            float* __restrict__ state, Tin* __restrict__ o, long long units,
            const Tin* __restrict__ g, const Tin* __restrict__ beta,
            const float* __restrict__ tau, const uint8_t* __restrict__ do_sane,
            int do_sane_all, int H) {
    __shared__ __align__(16) float vec[kStepWarps][5][64];  // r, d = exp(w), k, a, b
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const long long unit = (long long)blockIdx.x * kStepWarps + warp;
    if (unit >= units) return;  // warp-uniform; only __syncwarp is used below

    const size_t voff = (size_t)unit * 64;
    float4* S_g = reinterpret_cast<float4*>(state + (size_t)unit * 64 * 64);
    const int c = lane & 15;  // float4 column group
    const int p = lane >> 4;  // row half
    bool clip = false;  // SANE: this unit's state is clipped after the step (warp-uniform)
    float tc = 1.f;
    if constexpr (kSane) {
        clip = do_sane ? do_sane[unit / H] != 0 : do_sane_all != 0;
        if (clip) tc = tau[unit];
    }

    // Issue the 16 KiB state read first so it overlaps the vector staging.
    float4 S[32];
#pragma unroll
    for (int m = 0; m < 32; ++m) S[m] = S_g[(32 * p + m) * 16 + c];

    if constexpr (kGdn) {
        const float2 qq = load2(r + voff + 2 * lane);
        const float2 kk = load2(k + voff + 2 * lane);
        float sq = qq.x * qq.x + qq.y * qq.y, sk = kk.x * kk.x + kk.y * kk.y;
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, m);
            sk += __shfl_xor_sync(0xffffffffu, sk, m);
        }
        const float nq = sq > 0.f ? rsqrtf(sq) : 0.f, nk = sk > 0.f ? rsqrtf(sk) : 0.f;
        const float alpha = expf(to_f32(g[unit])), bt = to_f32(beta[unit]);
        const float2 kn = make_float2(kk.x * nk, kk.y * nk);
        float* vv = &vec[warp][0][0];
        reinterpret_cast<float2*>(vv + 0 * 64)[lane] = make_float2(qq.x * nq, qq.y * nq);
        reinterpret_cast<float2*>(vv + 1 * 64)[lane] = make_float2(alpha, alpha);
        reinterpret_cast<float2*>(vv + 2 * 64)[lane] = make_float2(bt * kn.x, bt * kn.y);
        reinterpret_cast<float2*>(vv + 3 * 64)[lane] = kn;
        reinterpret_cast<float2*>(vv + 4 * 64)[lane] =
            make_float2(-alpha * bt * kn.x, -alpha * bt * kn.y);
    } else {
        const float2 rr = load2(r + voff + 2 * lane);
        const float2 ww = load2(w + voff + 2 * lane);
        const float2 kk = load2(k + voff + 2 * lane);
        const float2 aa = load2(a + voff + 2 * lane);
        const float2 bb = load2(b + voff + 2 * lane);
        float* vv = &vec[warp][0][0];
        reinterpret_cast<float2*>(vv + 0 * 64)[lane] = rr;
        reinterpret_cast<float2*>(vv + 1 * 64)[lane] = make_float2(expf(ww.x), expf(ww.y));
        reinterpret_cast<float2*>(vv + 2 * 64)[lane] = kk;
        reinterpret_cast<float2*>(vv + 3 * 64)[lane] = aa;
        reinterpret_cast<float2*>(vv + 4 * 64)[lane] = bb;
    }
    const float4 vcol = load4(v + voff + 4 * c);
    __syncwarp();

    const float* sr = &vec[warp][0][32 * p];
    const float* sd = &vec[warp][1][32 * p];
    const float* sk = &vec[warp][2][32 * p];
    const float* sa = &vec[warp][3][32 * p];
    const float* sb = &vec[warp][4][32 * p];

    // u = S^T a over this lane's 32 rows, then across the two row halves.
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m4 = 0; m4 < 8; ++m4) {
        const float4 a4 = reinterpret_cast<const float4*>(sa)[m4];
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 s = S[4 * m4 + q];
            u.x = fmaf(s.x, av[q], u.x);
            u.y = fmaf(s.y, av[q], u.y);
            u.z = fmaf(s.z, av[q], u.z);
            u.w = fmaf(s.w, av[q], u.w);
        }
    }
    u.x += __shfl_xor_sync(0xffffffffu, u.x, 16);
    u.y += __shfl_xor_sync(0xffffffffu, u.y, 16);
    u.z += __shfl_xor_sync(0xffffffffu, u.z, 16);
    u.w += __shfl_xor_sync(0xffffffffu, u.w, 16);

    // S <- diag(d) S + b u^T + k v^T;  o = S^T r;  store S.
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m4 = 0; m4 < 8; ++m4) {
        const float4 d4 = reinterpret_cast<const float4*>(sd)[m4];
        const float4 k4 = reinterpret_cast<const float4*>(sk)[m4];
        const float4 b4 = reinterpret_cast<const float4*>(sb)[m4];
        const float4 r4 = reinterpret_cast<const float4*>(sr)[m4];
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
        const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
        const float rv[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 s = S[4 * m4 + q];
            s.x = fmaf(s.x, dv[q], fmaf(bv[q], u.x, kv[q] * vcol.x));
            s.y = fmaf(s.y, dv[q], fmaf(bv[q], u.y, kv[q] * vcol.y));
            s.z = fmaf(s.z, dv[q], fmaf(bv[q], u.z, kv[q] * vcol.z));
            s.w = fmaf(s.w, dv[q], fmaf(bv[q], u.w, kv[q] * vcol.w));
            acc.x = fmaf(s.x, rv[q], acc.x);
            acc.y = fmaf(s.y, rv[q], acc.y);
            acc.z = fmaf(s.z, rv[q], acc.z);
            acc.w = fmaf(s.w, rv[q], acc.w);
            S_g[(32 * p + 4 * m4 + q) * 16 + c] = (kSane && clip) ? sane_clip4(s, tc) : s;
        }
    }
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
    if (p == 0) store4(o + voff + 4 * c, acc);
}

// K = V in {128, 256}: block = K / 64 warps on one 64-column slab of one unit.
template <typename Tin, bool kGdn, int K, bool kSane = false>
__global__ void __launch_bounds__(32 * (K / 64))
step_kernel_wide(const Tin* __restrict__ r, const Tin* __restrict__ w, const Tin* __restrict__ k,
                 const Tin* __restrict__ v, const Tin* __restrict__ a, const Tin* __restrict__ b,
                 float* __restrict__ state, Tin* __restrict__ o, const Tin* __restrict__ g,
                 const Tin* __restrict__ beta, const float* __restrict__ tau,
                 const uint8_t* __restrict__ do_sane, int do_sane_all, int H) {
    constexpr int P = K / 64;  // warps = row parts = column slabs per unit
    __shared__ __align__(16) float vec[5][K];  // r, d = exp(w), k, a, b
    __shared__ __align__(16) float part_u[P][64];
    __shared__ __align__(16) float part_o[P][64];
    __shared__ float nrm[2][P];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;  // row part
    const long long unit = blockIdx.x / P;
    const int slab = blockIdx.x % P;
    const size_t voff = (size_t)unit * K;
    float* Su = state + (size_t)unit * K * K;
    const int c = lane & 15;  // float4 column group of the slab
    const int ph = lane >> 4; // row half of the part
    const int row0 = 64 * warp + 32 * ph;
    const int col0 = 64 * slab + 4 * c;
    bool clip = false;  // SANE (block-uniform)
    float tc = 1.f;
    if constexpr (kSane) {
        clip = do_sane ? do_sane[unit / H] != 0 : do_sane_all != 0;
        if (clip) tc = tau[unit];
    }

    float4 S[32];
#pragma unroll
    for (int m = 0; m < 32; ++m)
        S[m] = *reinterpret_cast<const float4*>(Su + (size_t)(row0 + m) * K + col0);

    const int e0 = 64 * warp + 2 * lane;  // this lane's two vector entries
    if constexpr (kGdn) {
        const float2 qq = load2(r + voff + e0);
        const float2 kk = load2(k + voff + e0);
        float sq = qq.x * qq.x + qq.y * qq.y, sk = kk.x * kk.x + kk.y * kk.y;
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, m);
            sk += __shfl_xor_sync(0xffffffffu, sk, m);
        }
        if (lane == 0) {
            nrm[0][warp] = sq;
            nrm[1][warp] = sk;
        }
        __syncthreads();
        sq = 0.f;
        sk = 0.f;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            sq += nrm[0][p];
            sk += nrm[1][p];
        }
        const float nq = sq > 0.f ? rsqrtf(sq) : 0.f, nk = sk > 0.f ? rsqrtf(sk) : 0.f;
        const float alpha = expf(to_f32(g[unit])), bt = to_f32(beta[unit]);
        const float2 kn = make_float2(kk.x * nk, kk.y * nk);
        *reinterpret_cast<float2*>(&vec[0][e0]) = make_float2(qq.x * nq, qq.y * nq);
        *reinterpret_cast<float2*>(&vec[1][e0]) = make_float2(alpha, alpha);
        *reinterpret_cast<float2*>(&vec[2][e0]) = make_float2(bt * kn.x, bt * kn.y);
        *reinterpret_cast<float2*>(&vec[3][e0]) = kn;
        *reinterpret_cast<float2*>(&vec[4][e0]) = make_float2(-alpha * bt * kn.x, -alpha * bt * kn.y);
    } else {
        const float2 ww = load2(w + voff + e0);
        *reinterpret_cast<float2*>(&vec[0][e0]) = load2(r + voff + e0);
        *reinterpret_cast<float2*>(&vec[1][e0]) = make_float2(expf(ww.x), expf(ww.y));
        *reinterpret_cast<float2*>(&vec[2][e0]) = load2(k + voff + e0);
        *reinterpret_cast<float2*>(&vec[3][e0]) = load2(a + voff + e0);
        *reinterpret_cast<float2*>(&vec[4][e0]) = load2(b + voff + e0);
    }
    const float4 vcol = load4(v + voff + col0);
    __syncwarp();  // a warp reads only the rows its own lanes wrote

    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m4 = 0; m4 < 8; ++m4) {
        const float4 a4 = reinterpret_cast<const float4*>(&vec[3][row0])[m4];
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 s = S[4 * m4 + q];
            u.x = fmaf(s.x, av[q], u.x);
            u.y = fmaf(s.y, av[q], u.y);
            u.z = fmaf(s.z, av[q], u.z);
            u.w = fmaf(s.w, av[q], u.w);
        }
    }
    u.x += __shfl_xor_sync(0xffffffffu, u.x, 16);
    u.y += __shfl_xor_sync(0xffffffffu, u.y, 16);
    u.z += __shfl_xor_sync(0xffffffffu, u.z, 16);
    u.w += __shfl_xor_sync(0xffffffffu, u.w, 16);
    if (ph == 0) *reinterpret_cast<float4*>(&part_u[warp][4 * c]) = u;
    __syncthreads();
    u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const float4 x = *reinterpret_cast<const float4*>(&part_u[p][4 * c]);
        u.x += x.x;
        u.y += x.y;
        u.z += x.z;
        u.w += x.w;
    }

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m4 = 0; m4 < 8; ++m4) {
        const float4 d4 = reinterpret_cast<const float4*>(&vec[1][row0])[m4];
        const float4 k4 = reinterpret_cast<const float4*>(&vec[2][row0])[m4];
        const float4 b4 = reinterpret_cast<const float4*>(&vec[4][row0])[m4];
        const float4 r4 = reinterpret_cast<const float4*>(&vec[0][row0])[m4];
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
        const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
        const float rv[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 s = S[4 * m4 + q];
            s.x = fmaf(s.x, dv[q], fmaf(bv[q], u.x, kv[q] * vcol.x));
            s.y = fmaf(s.y, dv[q], fmaf(bv[q], u.y, kv[q] * vcol.y));
            s.z = fmaf(s.z, dv[q], fmaf(bv[q], u.z, kv[q] * vcol.z));
            s.w = fmaf(s.w, dv[q], fmaf(bv[q], u.w, kv[q] * vcol.w));
            acc.x = fmaf(s.x, rv[q], acc.x);
            acc.y = fmaf(s.y, rv[q], acc.y);
            acc.z = fmaf(s.z, rv[q], acc.z);
            acc.w = fmaf(s.w, rv[q], acc.w);
            *reinterpret_cast<float4*>(Su + (size_t)(row0 + 4 * m4 + q) * K + col0) =
                (kSane && clip) ? sane_clip4(s, tc) : s;
        }
    }
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
    if (ph == 0) *reinterpret_cast<float4*>(&part_o[warp][4 * c]) = acc;
    __syncthreads();
    if (warp == 0 && ph == 0) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const float4 y = *reinterpret_cast<const float4*>(&part_o[p][4 * c]);
            x.x += y.x;
            x.y += y.y;
            x.z += y.z;
            x.w += y.w;
        }
        store4(o + voff + col0, x);
    }
}

template <typename Tin, bool kGdn, bool kSane = false>
cudaError_t launch_step_any(int K, const void* r, const void* w, const void* k, const void* v,
                            const void* a, const void* b, float* state, void* o, long long units,
                            const void* g, const void* beta, cudaStream_t stream,
                            const float* tau = nullptr, const uint8_t* do_sane = nullptr,
                            int do_sane_all = 0, int H = 1) {
    const Tin *r_ = static_cast<const Tin*>(r), *w_ = static_cast<const Tin*>(w),
              *k_ = static_cast<const Tin*>(k), *v_ = static_cast<const Tin*>(v),
              *a_ = static_cast<const Tin*>(a), *b_ = static_cast<const Tin*>(b),
              *g_ = static_cast<const Tin*>(g), *be_ = static_cast<const Tin*>(beta);
    Tin* o_ = static_cast<Tin*>(o);
    if (K == 64) {
        const long long blocks = (units + kStepWarps - 1) / kStepWarps;
        step_kernel<Tin, kGdn, kSane><<<(unsigned)blocks, kStepWarps * 32, 0, stream>>>(
            r_, w_, k_, v_, a_, b_, state, o_, units, g_, be_, tau, do_sane, do_sane_all, H);
    } else if (K == 128) {
        step_kernel_wide<Tin, kGdn, 128, kSane><<<(unsigned)(units * 2), 64, 0, stream>>>(
            r_, w_, k_, v_, a_, b_, state, o_, g_, be_, tau, do_sane, do_sane_all, H);
    } else if (K == 256) {
        step_kernel_wide<Tin, kGdn, 256, kSane><<<(unsigned)(units * 4), 128, 0, stream>>>(
            r_, w_, k_, v_, a_, b_, state, o_, g_, be_, tau, do_sane, do_sane_all, H);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// WKV7 step: r, w, k, a, b, v, o [units, K]; state [units, K, K] (K in {64, 128, 256}).
template <typename Tin>
cudaError_t launch_step(const void* r, const void* w, const void* k, const void* v,
                        const void* a, const void* b, float* state, void* o, long long units,
                        int K, cudaStream_t stream) {
    return launch_step_any<Tin, false>(K, r, w, k, v, a, b, state, o, units, nullptr, nullptr,
                                       stream);
}

// Gated DeltaNet step: q, k, v, o [units, K], g, beta [units].
template <typename Tin>
cudaError_t launch_step_gdn(const void* q, const void* k, const void* v, const void* g,
                            const void* beta, float* state, void* o, long long units, int K,
                            cudaStream_t stream) {
    return launch_step_any<Tin, true>(K, q, nullptr, k, v, nullptr, nullptr, state, o, units, g,
                                      beta, stream);
}

// SANE step: the WKV7 step, then the soft clip of the written state for flagged batch
// rows; tau [units] = [B, H] fp32, do_sane [B] (or NULL: do_sane_all for every row).
template <typename Tin>
cudaError_t launch_step_sane(const void* r, const void* w, const void* k, const void* v,
                             const void* a, const void* b, const float* tau,
                             const uint8_t* do_sane, int do_sane_all, float* state, void* o,
                             long long units, int H, int K, cudaStream_t stream) {
    return launch_step_any<Tin, false, true>(K, r, w, k, v, a, b, state, o, units, nullptr,
                                             nullptr, stream, tau, do_sane, do_sane_all, H);
}

}  // namespace wkv7
