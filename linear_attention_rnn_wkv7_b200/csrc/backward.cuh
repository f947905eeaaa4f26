// backward.cuh -- backward of the WKV7 forward (the README's training entry,
// generalized_delta_rule, supports backpropagation; rwkv-ops 0.9.0 README,
// "rwkv7op 使用方法"), K = V = 64, fp32 on CUDA cores.
//
// Given dL/do and dL/dS_T, reverse-mode differentiation of
//     u_t = S_{t-1}^T a_t,  S_t = D_t S_{t-1} + b_t u_t^T + k_t v_t^T,  o_t = S_t^T r_t
// runs backwards with the adjoint G = dL/dS_t:
//     G += r_t do_t^T;  dr_t = S_t do_t;  dv_t = G^T k_t;  dk_t = G v_t;
//     du_t = G^T b_t;   db_t = G u_t;     da_t = S_{t-1} du_t;
//     dw_t = e^{w_t} * rowsum(G * S_{t-1});  G <- D_t G + a_t du_t^T
// and finally dL/ds0 = G.  Two kernels:
//   ckpt_kernel  re-runs the forward with one thread per state column (as the
//                recurrent forward) and writes the state before every kCkpt-th token
//                and the final state (the checkpoints), and every token's u_t;
//   bwd_kernel   walks the tokens backwards with one thread per state row: it holds
//                row i of S_t and of G, so dr, dk, db, da, dw are in-thread sums over
//                the row; dv and du (sums over rows) go through G written to shared
//                memory once per token.  S_{t-1} is rebuilt from S_t with the stored
//                u_t, S_{t-1} = D_t^{-1} (S_t - b_t u_t^T - k_t v_t^T), at most
//                kCkpt - 1 times in a row before the next checkpoint replaces it
//                (the rebuild scales errors by e^{-w} per step; with the checkpoint
//                interval of 8 that stays below e^{4.3} for per-step decays >= -0.607).
// A masked token passes G through unchanged and gets zero dw, dk, dv, da, db.
#pragma once
#include "common.cuh"

namespace wkv7 {

namespace bwd {

constexpr int kCkpt = 8;  // tokens between checkpoints (one reverse tile)
constexpr int kRow = 68;  // padded row length of the adjoint in shared memory
// Threads per state row in the reverse pass.  One: splitting rows over 2 or 4 lanes
// (shorter per-thread chains, but shuffle sums on every token's chain and twice or
// four times the warps at each barrier) measured 1.4x and 2.5x slower.
constexpr int kRowThreads = 1;

// Workspace, fp32: checkpoints [slots][H][64][64] (the heads of one slot side by
// side, so the blocks writing checkpoints at the same time write neighbouring 16 KB
// blocks), then u [H][B*T token rows][64].
// Sequence n (packed rows [bos_n, eos_n)) of head h keeps its ceil(L/kCkpt) + 1
// checkpoints from slot floor(bos_n / kCkpt) + 2 n on; these ranges never overlap
// (floor((bos + L) / 8) + 1 >= floor(bos / 8) + ceil(L / 8)), so
// slots = floor(B*T / kCkpt) + 2 N + 1 per head covers every layout and length mix.
inline long long ckpt_slots(long long rows, int N) { return rows / kCkpt + 2LL * N + 1; }
inline size_t workspace_floats(long long rows, int N, int H) {
    return (size_t)H * ckpt_slots(rows, N) * 4096 + (size_t)rows * H * 64;
}

// The unit's sequence: packed rows [bos, eos) of batch row bb, and its first slot.
struct Seq {
    int bb, bos, eos;
    long long slot0;
    bool ok;
};
__device__ __forceinline__ Seq unit_seq(int n, int T, const int32_t* cu_seqlens) {
    Seq q;
    if (cu_seqlens) {
        q.bb = 0;
        q.bos = cu_seqlens[n];
        q.eos = cu_seqlens[n + 1];
        q.ok = q.bos >= 0 && q.eos >= q.bos && q.eos <= T;
        q.slot0 = (long long)q.bos / kCkpt + 2LL * n;
    } else {
        q.bb = n;
        q.bos = 0;
        q.eos = T;
        q.ok = true;
        q.slot0 = (long long)n * T / kCkpt + 2LL * n;
    }
    return q;
}

template <typename Tin>
__global__ void __launch_bounds__(64)
ckpt_kernel(const Tin* __restrict__ w, const Tin* __restrict__ k, const Tin* __restrict__ v,
            const Tin* __restrict__ a, const Tin* __restrict__ b,
            const float* __restrict__ s0, const uint8_t* __restrict__ mask,
            float* __restrict__ ckpt, float* __restrict__ uws, int T, int H, int N,
            const int32_t* __restrict__ cu_seqlens, int head_first) {
    constexpr int kTile = 16;
    __shared__ __align__(16) float sm[4][kTile][64];  // d = exp(w), k, a, b
    __shared__ float sv[kTile][64];
    __shared__ uint8_t smask[kTile];
    const int unit = blockIdx.x;
    const int h = unit % H, n = unit / H;
    const int j = threadIdx.x;
    const Seq sq = unit_seq(n, T, cu_seqlens);
    if (!sq.ok) {  // block-uniform; reported by the reverse pass
        return;
    }
    const int L = sq.eos - sq.bos;
    const long long rows = cu_seqlens ? (long long)T : (long long)N * T;
    // token p of the unit: row tb + p * ts of the inputs; u row bb*T + bos + p of head h
    const size_t tb = head_first ? ((size_t)sq.bb * H + h) * T + sq.bos
                                 : ((size_t)sq.bb * T + sq.bos) * H + h;
    const size_t ts = head_first ? 1 : (size_t)H;
    float* ck = ckpt + ((size_t)sq.slot0 * H + h) * 4096;
    float* uu = uws + ((size_t)h * rows + (size_t)sq.bb * T + sq.bos) * 64;

    float S[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) S[i] = s0 ? s0[(size_t)unit * 4096 + i * 64 + j] : 0.f;

    for (int t0 = 0; t0 < L; t0 += kTile) {
        const int cnt = min(kTile, L - t0);
        __syncthreads();
        {  // 16-byte loads: EPL elements per thread, 64 / EPL threads per row; all of
           // the tile's loads are issued before the first store
            constexpr int EPL = 16 / (int)sizeof(Tin);  // elements per load
            constexpr int TPR = 64 / EPL;               // threads per row
            constexpr int RPS = 64 / TPR;               // rows (tokens) per sweep
            constexpr int SW = kTile / RPS;             // sweeps per tile
            const int e0 = (j % TPR) * EPL, rr = j / TPR;
            uint4 raw[5][SW];
#pragma unroll
            for (int s2 = 0; s2 < SW; ++s2) {
                const int tt = s2 * RPS + rr;
                if (tt < cnt) {
                    const size_t row = (tb + (size_t)(t0 + tt) * ts) * 64 + e0;
                    raw[0][s2] = *reinterpret_cast<const uint4*>(w + row);
                    raw[1][s2] = *reinterpret_cast<const uint4*>(k + row);
                    raw[2][s2] = *reinterpret_cast<const uint4*>(a + row);
                    raw[3][s2] = *reinterpret_cast<const uint4*>(b + row);
                    raw[4][s2] = *reinterpret_cast<const uint4*>(v + row);
                }
            }
#pragma unroll
            for (int s2 = 0; s2 < SW; ++s2) {
                const int tt = s2 * RPS + rr;
                if (tt < cnt) {
#pragma unroll
                    for (int q = 0; q < 5; ++q) {
                        const Tin* x = reinterpret_cast<const Tin*>(&raw[q][s2]);
                        float* dst = q == 4 ? &sv[tt][e0] : &sm[q][tt][e0];
#pragma unroll
                        for (int e = 0; e < EPL; ++e)
                            dst[e] = q == 0 ? expf(to_f32(x[e])) : to_f32(x[e]);
                    }
                }
            }
        }
        if (j < cnt) smask[j] = mask ? (mask[(size_t)sq.bb * T + sq.bos + t0 + j] != 0) : 1;
        __syncthreads();
        for (int tt = 0; tt < cnt; ++tt) {
            const int p = t0 + tt;
            if (p % kCkpt == 0) {  // the state before token p
                float* dst = ck + (size_t)(p / kCkpt) * H * 4096;
#pragma unroll
                for (int i = 0; i < 64; ++i) dst[i * 64 + j] = S[i];
            }
            if (!smask[tt]) {
                uu[(size_t)p * 64 + j] = 0.f;
                continue;
            }
            const float4* a4 = reinterpret_cast<const float4*>(sm[2][tt]);
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
            uu[(size_t)p * 64 + j] = u;
            const float vj = sv[tt][j];
            const float4* d4 = reinterpret_cast<const float4*>(sm[0][tt]);
            const float4* k4 = reinterpret_cast<const float4*>(sm[1][tt]);
            const float4* b4 = reinterpret_cast<const float4*>(sm[3][tt]);
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {
                const float4 dv = d4[i4], kv = k4[i4], bv = b4[i4];
                S[4 * i4 + 0] = fmaf(S[4 * i4 + 0], dv.x, fmaf(bv.x, u, kv.x * vj));
                S[4 * i4 + 1] = fmaf(S[4 * i4 + 1], dv.y, fmaf(bv.y, u, kv.y * vj));
                S[4 * i4 + 2] = fmaf(S[4 * i4 + 2], dv.z, fmaf(bv.z, u, kv.z * vj));
                S[4 * i4 + 3] = fmaf(S[4 * i4 + 3], dv.w, fmaf(bv.w, u, kv.w * vj));
            }
        }
    }
    float* dst = ck + (size_t)((L + kCkpt - 1) / kCkpt) * H * 4096;  // the final state
#pragma unroll
    for (int i = 0; i < 64; ++i) dst[i * 64 + j] = S[i];
}

// Sum of x over the P adjacent lanes that share a state row.
template <int P>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
    for (int m = 1; m < P; m *= 2) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// P threads per state row (adjacent lanes), 64 / P columns each.
template <typename Tin, int P>
__global__ void __launch_bounds__(64 * P)
bwd_kernel(const Tin* __restrict__ r, const Tin* __restrict__ w, const Tin* __restrict__ k,
           const Tin* __restrict__ v, const Tin* __restrict__ a, const Tin* __restrict__ b,
           const uint8_t* __restrict__ mask, const Tin* __restrict__ dout,
           const float* __restrict__ dsT, const float* __restrict__ ckpt,
           const float* __restrict__ uws, Tin* __restrict__ dr, Tin* __restrict__ dw,
           Tin* __restrict__ dk, Tin* __restrict__ dv, Tin* __restrict__ da,
           Tin* __restrict__ db, float* __restrict__ ds0, int T, int H, int N,
           const int32_t* __restrict__ cu_seqlens, int head_first) {
    constexpr int NC = 64 / P;  // columns (and, for the column sums, rows) per thread
    // per token of the tile: K-side r, e^{w}, e^{-w}, k, a, b; V-side v, do, u
    __shared__ __align__(16) float sK[6][kCkpt][64];
    __shared__ __align__(16) float sV[3][kCkpt][64];
    __shared__ __align__(16) float sG[64 * kRow];  // G rows (one token at a time)
    __shared__ __align__(16) float sdu[64];
    __shared__ uint8_t smask[kCkpt];
    const int unit = blockIdx.x;
    const int h = unit % H, n = unit / H;
    const int tid = threadIdx.x;
    const int i = tid / P, part = tid % P;  // state row; columns c0 .. c0 + NC - 1
    const int c0 = part * NC;
    const Seq sq = unit_seq(n, T, cu_seqlens);
    if (!sq.ok) {  // block-uniform: the sequence is skipped and reported
        if (tid == 0) raise_flag(5 /* WKV7_ERR_DEVICE_BAD_SEQLENS */);
        return;
    }
    const int L = sq.eos - sq.bos;
    const int nC = (L + kCkpt - 1) / kCkpt;
    const size_t tb = head_first ? ((size_t)sq.bb * H + h) * T + sq.bos
                                 : ((size_t)sq.bb * T + sq.bos) * H + h;
    const size_t ts = head_first ? 1 : (size_t)H;
    const float* ck = ckpt + ((size_t)sq.slot0 * H + h) * 4096;
    const long long rows = cu_seqlens ? (long long)T : (long long)N * T;
    const float* uu = uws + ((size_t)h * rows + (size_t)sq.bb * T + sq.bos) * 64;

    float S[NC], G[NC];
    auto load_state = [&](int slot) {
        const float4* src = reinterpret_cast<const float4*>(ck + (size_t)slot * H * 4096 + i * 64 + c0);
#pragma unroll
        for (int q = 0; q < NC / 4; ++q) {
            const float4 x = src[q];
            S[4 * q] = x.x; S[4 * q + 1] = x.y; S[4 * q + 2] = x.z; S[4 * q + 3] = x.w;
        }
    };
    load_state(nC);
#pragma unroll
    for (int jj = 0; jj < NC; ++jj)
        G[jj] = dsT ? dsT[(size_t)unit * 4096 + i * 64 + c0 + jj] : 0.f;

    for (int c = nC - 1; c >= 0; --c) {
        const int t0 = c * kCkpt, cnt = min(kCkpt, L - t0);
        __syncthreads();  // the previous tile's reads of the stage are done
        if (tid < 64) {  // 16-byte loads, all issued before the first store
            constexpr int EPL = 16 / (int)sizeof(Tin);  // input elements per load
            constexpr int TPR = 64 / EPL;               // threads per row
            constexpr int RPS = 64 / TPR;               // rows (tokens) per sweep
            constexpr int SW = (kCkpt + RPS - 1) / RPS; // sweeps per tile
            const int e0 = (tid % TPR) * EPL, rr = tid / TPR;
            uint4 raw[7][SW];
#pragma unroll
            for (int s2 = 0; s2 < SW; ++s2) {
                const int tt = s2 * RPS + rr;
                if (tt < cnt) {
                    const size_t row = (tb + (size_t)(t0 + tt) * ts) * 64 + e0;
                    raw[0][s2] = *reinterpret_cast<const uint4*>(r + row);
                    raw[1][s2] = *reinterpret_cast<const uint4*>(w + row);
                    raw[2][s2] = *reinterpret_cast<const uint4*>(k + row);
                    raw[3][s2] = *reinterpret_cast<const uint4*>(a + row);
                    raw[4][s2] = *reinterpret_cast<const uint4*>(b + row);
                    raw[5][s2] = *reinterpret_cast<const uint4*>(v + row);
                    raw[6][s2] = *reinterpret_cast<const uint4*>(dout + row);
                }
            }
            // u (fp32): 16 threads per row, 4 rows per sweep
            float4 ru[kCkpt / 4];
#pragma unroll
            for (int s2 = 0; s2 < kCkpt / 4; ++s2) {
                const int tt = s2 * 4 + tid / 16;
                if (tt < cnt)
                    ru[s2] = *reinterpret_cast<const float4*>(uu + (size_t)(t0 + tt) * 64 + (tid % 16) * 4);
            }
#pragma unroll
            for (int s2 = 0; s2 < SW; ++s2) {
                const int tt = s2 * RPS + rr;
                if (tt < cnt) {
                    const Tin* x[7];
#pragma unroll
                    for (int q = 0; q < 7; ++q) x[q] = reinterpret_cast<const Tin*>(&raw[q][s2]);
#pragma unroll
                    for (int e = 0; e < EPL; ++e) {
                        const float wv = to_f32(x[1][e]);
                        sK[0][tt][e0 + e] = to_f32(x[0][e]);
                        sK[1][tt][e0 + e] = expf(wv);
                        sK[2][tt][e0 + e] = expf(-wv);
                        sK[3][tt][e0 + e] = to_f32(x[2][e]);
                        sK[4][tt][e0 + e] = to_f32(x[3][e]);
                        sK[5][tt][e0 + e] = to_f32(x[4][e]);
                        sV[0][tt][e0 + e] = to_f32(x[5][e]);
                        sV[1][tt][e0 + e] = to_f32(x[6][e]);
                    }
                }
            }
#pragma unroll
            for (int s2 = 0; s2 < kCkpt / 4; ++s2) {
                const int tt = s2 * 4 + tid / 16;
                if (tt < cnt) *reinterpret_cast<float4*>(&sV[2][tt][(tid % 16) * 4]) = ru[s2];
            }
            if (tid < cnt) smask[tid] = mask ? (mask[(size_t)sq.bb * T + sq.bos + t0 + tid] != 0) : 1;
        }
        __syncthreads();

        for (int tt = cnt - 1; tt >= 0; --tt) {
            const size_t row = (tb + (size_t)(t0 + tt) * ts) * 64;
            const bool out = part == 0;  // the lane that writes row i's results
            const float ri = sK[0][tt][i];
            const float4* do4 = reinterpret_cast<const float4*>(sV[1][tt] + c0);
            float dri = 0.f;
#pragma unroll
            for (int q = 0; q < NC / 4; ++q) {  // G += r do^T;  dr = S_t do
                const float4 x = do4[q];
                G[4 * q] = fmaf(ri, x.x, G[4 * q]);
                G[4 * q + 1] = fmaf(ri, x.y, G[4 * q + 1]);
                G[4 * q + 2] = fmaf(ri, x.z, G[4 * q + 2]);
                G[4 * q + 3] = fmaf(ri, x.w, G[4 * q + 3]);
                dri = fmaf(S[4 * q], x.x, fmaf(S[4 * q + 1], x.y,
                      fmaf(S[4 * q + 2], x.z, fmaf(S[4 * q + 3], x.w, dri))));
            }
            dri = row_sum<P>(dri);
            if (out) dr[row + i] = from_f32<Tin>(dri);
            const bool upd = smask[tt] != 0;  // block-uniform
            if (!upd) {
                if (out) {
                    dw[row + i] = from_f32<Tin>(0.f);
                    dk[row + i] = from_f32<Tin>(0.f);
                    dv[row + i] = from_f32<Tin>(0.f);
                    da[row + i] = from_f32<Tin>(0.f);
                    db[row + i] = from_f32<Tin>(0.f);
                }
                if (tt == 0) load_state(c);  // the state before the tile (unchanged here)
                continue;
            }
            // dk = G v, db = G u (row sums); G row to shared memory for the column sums
            const float4* v4 = reinterpret_cast<const float4*>(sV[0][tt] + c0);
            const float4* u4 = reinterpret_cast<const float4*>(sV[2][tt] + c0);
            float dki = 0.f, dbi = 0.f;
            float4* gr = reinterpret_cast<float4*>(sG + i * kRow + c0);
#pragma unroll
            for (int q = 0; q < NC / 4; ++q) {
                const float4 xv = v4[q], xu = u4[q];
                dki = fmaf(G[4 * q], xv.x, fmaf(G[4 * q + 1], xv.y,
                      fmaf(G[4 * q + 2], xv.z, fmaf(G[4 * q + 3], xv.w, dki))));
                dbi = fmaf(G[4 * q], xu.x, fmaf(G[4 * q + 1], xu.y,
                      fmaf(G[4 * q + 2], xu.z, fmaf(G[4 * q + 3], xu.w, dbi))));
                gr[q] = make_float4(G[4 * q], G[4 * q + 1], G[4 * q + 2], G[4 * q + 3]);
            }
            dki = row_sum<P>(dki);
            dbi = row_sum<P>(dbi);
            if (out) {
                dk[row + i] = from_f32<Tin>(dki);
                db[row + i] = from_f32<Tin>(dbi);
            }
            __syncthreads();
            {  // as column i over rows c0 .. c0 + NC - 1: dv_i = sum_m G[m][i] k_m, du_i = G^T b
                const float* kk = sK[3][tt];
                const float* bbv = sK[5][tt];
                float sv0 = 0.f, sv1 = 0.f, su0 = 0.f, su1 = 0.f;
#pragma unroll
                for (int m = c0; m < c0 + NC; m += 2) {
                    const float g0 = sG[m * kRow + i], g1 = sG[(m + 1) * kRow + i];
                    sv0 = fmaf(g0, kk[m], sv0);
                    sv1 = fmaf(g1, kk[m + 1], sv1);
                    su0 = fmaf(g0, bbv[m], su0);
                    su1 = fmaf(g1, bbv[m + 1], su1);
                }
                const float dvi = row_sum<P>(sv0 + sv1), dui = row_sum<P>(su0 + su1);
                if (out) {
                    dv[row + i] = from_f32<Tin>(dvi);
                    sdu[i] = dui;
                }
            }
            __syncthreads();
            // S becomes S_{t-1}: the checkpoint at the tile start, else rebuilt from S_t
            if (tt == 0) {
                load_state(c);
            } else {
                const float ki = sK[3][tt][i], bi = sK[5][tt][i], dinv = sK[2][tt][i];
#pragma unroll
                for (int q = 0; q < NC / 4; ++q) {
                    const float4 xv = v4[q], xu = u4[q];
                    S[4 * q] = (S[4 * q] - fmaf(bi, xu.x, ki * xv.x)) * dinv;
                    S[4 * q + 1] = (S[4 * q + 1] - fmaf(bi, xu.y, ki * xv.y)) * dinv;
                    S[4 * q + 2] = (S[4 * q + 2] - fmaf(bi, xu.z, ki * xv.z)) * dinv;
                    S[4 * q + 3] = (S[4 * q + 3] - fmaf(bi, xu.w, ki * xv.w)) * dinv;
                }
            }
            const float4* du4 = reinterpret_cast<const float4*>(sdu + c0);
            const float di = sK[1][tt][i], ai = sK[4][tt][i];
            float dai = 0.f, dwi = 0.f;
#pragma unroll
            for (int q = 0; q < NC / 4; ++q) {
                const float4 x = du4[q];
                dai = fmaf(S[4 * q], x.x, fmaf(S[4 * q + 1], x.y,
                      fmaf(S[4 * q + 2], x.z, fmaf(S[4 * q + 3], x.w, dai))));
                dwi = fmaf(G[4 * q], S[4 * q], fmaf(G[4 * q + 1], S[4 * q + 1],
                      fmaf(G[4 * q + 2], S[4 * q + 2], fmaf(G[4 * q + 3], S[4 * q + 3], dwi))));
                G[4 * q] = fmaf(di, G[4 * q], ai * x.x);
                G[4 * q + 1] = fmaf(di, G[4 * q + 1], ai * x.y);
                G[4 * q + 2] = fmaf(di, G[4 * q + 2], ai * x.z);
                G[4 * q + 3] = fmaf(di, G[4 * q + 3], ai * x.w);
            }
            dai = row_sum<P>(dai);
            dwi = row_sum<P>(dwi);
            if (out) {
                da[row + i] = from_f32<Tin>(dai);
                dw[row + i] = from_f32<Tin>(di * dwi);
            }
        }
    }
    if (ds0) {
        float4* dst = reinterpret_cast<float4*>(ds0 + (size_t)unit * 4096 + i * 64 + c0);
#pragma unroll
        for (int q = 0; q < NC / 4; ++q)
            dst[q] = make_float4(G[4 * q], G[4 * q + 1], G[4 * q + 2], G[4 * q + 3]);
    }
}

}  // namespace bwd

template <typename Tin>
cudaError_t launch_bwd(const void* r, const void* w, const void* k, const void* v, const void* a,
                       const void* b, const float* s0, const uint8_t* mask, const void* dout,
                       const float* dsT, void* dr, void* dw, void* dk, void* dv, void* da,
                       void* db, float* ds0, int B, int T, int H, int N,
                       const int32_t* cu_seqlens, int head_first, float* ws,
                       cudaStream_t stream) {
    const long long units = (long long)N * H;
    const long long rows = (long long)B * T;
    const long long slots = bwd::ckpt_slots(rows, N);
    float* ckpt = ws;
    float* uws = ws + (size_t)H * slots * 4096;
    const Tin *r_ = static_cast<const Tin*>(r), *w_ = static_cast<const Tin*>(w),
              *k_ = static_cast<const Tin*>(k), *v_ = static_cast<const Tin*>(v),
              *a_ = static_cast<const Tin*>(a), *b_ = static_cast<const Tin*>(b);
    bwd::ckpt_kernel<Tin><<<(unsigned)units, 64, 0, stream>>>(w_, k_, v_, a_, b_, s0, mask, ckpt,
                                                              uws, T, H, N, cu_seqlens,
                                                              head_first);
    bwd::bwd_kernel<Tin, bwd::kRowThreads><<<(unsigned)units, 64 * bwd::kRowThreads, 0, stream>>>(
        r_, w_, k_, v_, a_, b_, mask, static_cast<const Tin*>(dout), dsT, ckpt, uws,
        static_cast<Tin*>(dr), static_cast<Tin*>(dw), static_cast<Tin*>(dk),
        static_cast<Tin*>(dv), static_cast<Tin*>(da), static_cast<Tin*>(db), ds0, T, H, N,
        cu_seqlens, head_first);
    return cudaGetLastError();
}

}  // namespace wkv7
