// chunked.cuh -- 64-token chunked WKV7 forward on tcgen05 tensor cores (bf16 in,
// fp32 state), one CTA per (sequence, head), two CTAs resident per SM.
//
// The recurrence (rwkv-ops 0.9.0 README, "rwkv7op 使用方法")
//     u_t = S_{t-1}^T a_t;  S_t = diag(exp w_t) S_{t-1} + b_t u_t^T + k_t v_t^T;  o_t = S_t^T r_t
// is rewritten exactly for a chunk of L = 64 tokens (t = 0..63, state S0 at the
// chunk start).  With g_t = sum_{j<=t} w_j (per channel, log space), a
// reference c = g_31 and E_t = exp(g_t - c):
//   r~ = r E_t, a~ = a E_{t-1}, k~ = k / E_t, b~ = b / E_t        (Gram operands)
//   A_rk[t][s] = r~_t.k~_s (s<=t), A_rb = r~.b~ (s<=t), A_ak = a~.k~ (s<t), A_ab = a~.b~ (s<t)
//   T = (I - A_ab)^-1 (the UT / WY representation of the chunk's rank-1 products)
//   Abar = a e^{g_{t-1}}, Rbar = r e^{g_t}, Bhat = b e^{g_L - g_t}, Khat = k e^{g_L - g_t}
//   W = T Abar, Z = T A_ak              (so the read vectors are U = W S0 + Z V)
//   S_L = diag(e^{g_L}) S0 + (Bhat^T W) S0 + (Khat^T + Bhat^T Z) V
//   O   = (Rbar + A_rb W) S0 + (A_rk + A_rb Z) V
// Only the last product depends on S0, so one chunk costs five tcgen05 MMA groups
// (Gram, W|Z, the two Bhat/A_rb products, final) with everything else on CUDA
// cores: the prefix sums and exps, the 64x64 triangular solve (fp32) and the
// TMEM -> shared-memory epilogues that re-layout each result as the next
// product's operand.  The write term Khat^T + Bhat^T Z enters the final MMA as a
// hi/lo pair of bf16 matrices (about 16 significant bits), which keeps the fp32
// final state within 1e-3 of the fp64 recurrence; all other operands are bf16.
//
// A masked or out-of-range token is folded into the loads as w = a = k = b = 0:
// its transition is then the identity and it writes nothing, and its output is
// read from the carried state.  Exps are clamped to [-40, 40] around c, so the
// factorisation is exact while |g_t - g_31| <= 40 inside a chunk (per-step log
// decay >= -1.2; the RWKV-7 parametrisation keeps it >= -0.607).
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace wkv7 {

constexpr bool kChunkedBuilt = true;

namespace chunked {

constexpr int kThreads = 256;
// Shared-memory map (bytes; every tile 1024-aligned, 64 rows x 128 B, 128B swizzle).
constexpr uint32_t OFF_R = 0;          // raw r -> r~        (Gram B rows 0..63)
constexpr uint32_t OFF_A = 8192;       // raw a -> a~        (Gram B rows 64..127)
constexpr uint32_t OFF_K = 16384;      // raw k -> k~        (Gram A rows 0..63)
constexpr uint32_t OFF_B = 24576;      // raw b -> b~        (Gram A rows 64..127)
constexpr uint32_t OFF_W = 32768;      // raw w -> Bhat      (MMA-3 A, MN-major atom 0)
constexpr uint32_t OFF_V = 40960;      // raw v              (final MMA B, MN-major)
constexpr uint32_t OFF_ABAR = 49152;   // Abar [s][k]        (MMA-2 A, MN-major atom 0)
constexpr uint32_t OFF_AAK = 57344;    // A_ak [s][s']       (MMA-2 A, MN-major atom 1)
constexpr uint32_t OFF_ARBT = 65536;   // A_rb^T [s][t]      (MMA-3 A, MN-major atom 1)
constexpr uint32_t OFF_ARKT = 73728;   // A_rk^T [s][t]      (epilogue 3); prologue scratch
constexpr uint32_t OFF_RBAR = 81920;   // Rbar [t][k]        (epilogue 3)
constexpr uint32_t OFF_S0 = 90112;     // S0 bf16 [k][v]     (final MMA B, MN-major)
constexpr uint32_t OFF_F0 = 98304;     // fp32 64x64: E_t, then Khat [s][k]
constexpr uint32_t OFF_MISC = 114688;  // mbarriers, TMEM address, abort flag
constexpr uint32_t kSmemBytes = OFF_MISC + 32;
// Aliases (lifetimes do not overlap).
constexpr uint32_t OFF_AAB = OFF_R;    // fp32 A_ab [t][s] (epilogue 1 -> solve), 16 KB
constexpr uint32_t OFF_TT = OFF_K;     // T^T [s][t]      (solve -> MMA-2 B, MN-major)
constexpr uint32_t OFF_WZT = OFF_K;    // [W^T; Z^T] [n][t] 128 rows (MMA-3 B, K-major)
constexpr uint32_t OFF_FIN0 = OFF_R;   // final A, K block 0: [M'; Rbar + A_rb W]
constexpr uint32_t OFF_FIN1 = OFF_ABAR;// final A, K block 1: [P_N hi; A_rk + A_rb Z]
constexpr uint32_t OFF_FIN2 = OFF_K;   // final A, K block 2: [P_N lo; 0]
// Tensor-memory columns (fp32 accumulators, 128 lanes).
constexpr uint32_t TM_D1 = 0;    // Gram, later MMA-3 (128 cols)
constexpr uint32_t TM_D2 = 128;  // [W^T; Z^T] (64 cols)
constexpr uint32_t TM_DF = 192;  // [S update; O] (64 cols)
constexpr uint32_t kTmemCols = 256;
constexpr float kExpClamp = 40.f;

// Byte offset of 16-byte chunk `c` of row `row` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw(uint32_t row, uint32_t c) {
    return row * 128u + ((c ^ (row & 7u)) << 4);
}
// Byte offset of bf16 element (row, col) in a 128B-swizzled 64-column tile.
__device__ __forceinline__ uint32_t swe(uint32_t row, uint32_t col) {
    return sw(row, col >> 3) + ((col & 7u) << 1);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float* v) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ float bf16_at(const uint8_t* tile, uint32_t row, uint32_t col) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + swe(row, col)));
}
__device__ __forceinline__ float clamped_exp(float x) {
    return __expf(fminf(fmaxf(x, -kExpClamp), kExpClamp));
}

// Load `n16` groups of 16 TMEM columns starting at column `col` for this warp's lanes.
template <int N16>
__device__ __forceinline__ void tmem_row(uint32_t tmem, int wq, uint32_t col, float* v) {
#pragma unroll
    for (int i = 0; i < N16; ++i) {
        float tmp[16];
        sm100::tmem_ld16(tmem + ((uint32_t)(32 * wq) << 16) + col + 16 * i, tmp);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[16 * i + j] = tmp[j];
    }
    sm100::tmem_ld_wait();
}

__device__ __forceinline__ void wait_or_abort(uint32_t bar, uint32_t parity, int* abort_flag) {
    if (!sm100::mbar_wait(bar, parity)) {
        raise_flag(4 /* WKV7_ERR_DEVICE_TIMEOUT */);
        *abort_flag = 1;
    }
}

__global__ void __launch_bounds__(kThreads, 2)
chunked_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const float* s0, const uint8_t* __restrict__ mask, __nv_bfloat16* __restrict__ o,
               float* sT, int T, int H, const int32_t* __restrict__ cu_seqlens) {
    extern __shared__ __align__(1024) uint8_t smem[];
    using namespace sm100;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;  // TMEM lane quarter, column half
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
        if (tid == 0) raise_flag(3 /* WKV7_ERR_CUDA */);
        return;
    }
    const int h = blockIdx.x % H;
    const int n = blockIdx.x / H;
    int bb = n, bos = 0, eos = T;
    if (cu_seqlens) {
        bb = 0;
        bos = cu_seqlens[n];
        eos = cu_seqlens[n + 1];
        if (bos < 0 || eos < bos || eos > T) {
            if (tid == 0) raise_flag(5 /* WKV7_ERR_DEVICE_BAD_SEQLENS */);
            return;
        }
    }
    const int len = eos - bos;
    const long long row0 = (long long)bb * T + bos;  // token row of the sequence start

    const uint32_t bar_tma = sbase + OFF_MISC, bar_mma = sbase + OFF_MISC + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC + 16);
    int* abort_flag = reinterpret_cast<int*>(smem + OFF_MISC + 20);
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // State rows: warps with lane quarter 0/1 own row m = 32*wq + lane, columns
    // [32*wh, 32*wh + 32), in fp32 registers for the whole sequence.
    const bool state_thread = wq < 2;
    const int m_row = 32 * wq + lane;
    const size_t state_off = ((size_t)n * H + h) * 4096;
    float S[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) S[j] = 0.f;
    if (state_thread) {
        if (s0) {
            const float4* src = reinterpret_cast<const float4*>(s0 + state_off + m_row * 64 + 32 * wh);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 f = src[j];
                S[4 * j] = f.x; S[4 * j + 1] = f.y; S[4 * j + 2] = f.z; S[4 * j + 3] = f.w;
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(smem + OFF_S0 + sw(m_row, 4 * wh + c)) = pack8(S + 8 * c);
    }
    float gamma = 1.f;  // e^{g_L} for this thread's channel (state threads)

    float* scratch = reinterpret_cast<float*>(smem + OFF_ARKT);  // prologue only
    uint8_t* validb = reinterpret_cast<uint8_t*>(scratch + 448);
    float* F0 = reinterpret_cast<float*>(smem + OFF_F0);
    uint32_t mma_phase = 0;
    int iter = 0;
    for (int c0 = 0; c0 < len; c0 += 64, ++iter) {
        const int nv = min(64, len - c0);
        // ---- 1. TMA: the chunk's six 64 x 64 bf16 tiles ------------------------------
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_tma, 6 * 8192);
            const int row = (int)(row0 + c0);
            tma_load_3d(sbase + OFF_R, &tm_r, bar_tma, 0, h, row);
            tma_load_3d(sbase + OFF_A, &tm_a, bar_tma, 0, h, row);
            tma_load_3d(sbase + OFF_K, &tm_k, bar_tma, 0, h, row);
            tma_load_3d(sbase + OFF_B, &tm_b, bar_tma, 0, h, row);
            tma_load_3d(sbase + OFF_W, &tm_w, bar_tma, 0, h, row);
            tma_load_3d(sbase + OFF_V, &tm_v, bar_tma, 0, h, row);
        }
        wait_or_abort(bar_tma, iter & 1, abort_flag);

        // ---- 2. prefix sums of w (mask folded), E_t = e^{g_t - c} ------------------------
        {
            const int kk = tid & 63, q = tid >> 6;
            float gl[16];
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = 16 * q + i;
                const bool val = t < nv && (!mask || mask[row0 + c0 + t] != 0);
                acc += val ? bf16_at(smem + OFF_W, t, kk) : 0.f;
                gl[i] = acc;
                if (kk == 0) validb[t] = val ? 1 : 0;
            }
            scratch[q * 64 + kk] = acc;
            __syncthreads();
            const float t0 = scratch[kk], t1 = scratch[64 + kk], t2 = scratch[128 + kk],
                        t3 = scratch[192 + kk];
            const float prefix = q == 0 ? 0.f : (q == 1 ? t0 : (q == 2 ? t0 + t1 : t0 + t1 + t2));
            const float c = t0 + t1;
            const float gL = (t0 + t1) + (t2 + t3);
#pragma unroll
            for (int i = 0; i < 16; ++i) F0[(16 * q + i) * 64 + kk] = clamped_exp(prefix + gl[i] - c);
            if (q == 0) {
                scratch[256 + kk] = clamped_exp(c);
                scratch[320 + kk] = clamped_exp(-c);
                scratch[384 + kk] = clamped_exp(gL - c);
            }
            gamma = __expf(gL);
            __syncthreads();
        }

        // ---- 3. scaled operands (two 8-channel pieces per thread) ------------------------
        {
            uint4 o_r[2], o_a[2], o_k[2], o_b[2], o_abar[2], o_bhat[2], o_rbar[2];
            float4 o_khat[2][2];
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int item = tid + 256 * it;
                const int t = item >> 3, j = item & 7;
                const bool val = validb[t] != 0;
                float rv[8], av[8], kv[8], bv[8];
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_R + sw(t, j)), rv);
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_A + sw(t, j)), av);
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_K + sw(t, j)), kv);
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_B + sw(t, j)), bv);
                float E[8], Em[8], ec[8], elc[8];
                const float* Erow = F0 + t * 64 + 8 * j;
                const float* Emrow = t > 0 ? F0 + (t - 1) * 64 + 8 * j : scratch + 320 + 8 * j;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    E[e] = Erow[e];
                    Em[e] = Emrow[e];
                    ec[e] = scratch[256 + 8 * j + e];
                    elc[e] = scratch[384 + 8 * j + e];
                }
                float rt[8], at[8], kt[8], btl[8], abar[8], bhat[8], khat[8], rbar[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float inv = __frcp_rn(E[e]);
                    const float a_ = val ? av[e] : 0.f, k_ = val ? kv[e] : 0.f,
                                b_ = val ? bv[e] : 0.f;
                    rt[e] = rv[e] * E[e];
                    at[e] = a_ * Em[e];
                    kt[e] = k_ * inv;
                    btl[e] = b_ * inv;
                    abar[e] = at[e] * ec[e];
                    bhat[e] = b_ * elc[e] * inv;
                    khat[e] = k_ * elc[e] * inv;
                    rbar[e] = rt[e] * ec[e];
                }
                o_r[it] = pack8(rt);
                o_a[it] = pack8(at);
                o_k[it] = pack8(kt);
                o_b[it] = pack8(btl);
                o_abar[it] = pack8(abar);
                o_bhat[it] = pack8(bhat);
                o_rbar[it] = pack8(rbar);
                o_khat[it][0] = make_float4(khat[0], khat[1], khat[2], khat[3]);
                o_khat[it][1] = make_float4(khat[4], khat[5], khat[6], khat[7]);
            }
            __syncthreads();  // every E_t read before F0 is overwritten by Khat
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int item = tid + 256 * it;
                const int t = item >> 3, j = item & 7;
                const uint32_t off = sw(t, j);
                *reinterpret_cast<uint4*>(smem + OFF_R + off) = o_r[it];
                *reinterpret_cast<uint4*>(smem + OFF_A + off) = o_a[it];
                *reinterpret_cast<uint4*>(smem + OFF_K + off) = o_k[it];
                *reinterpret_cast<uint4*>(smem + OFF_B + off) = o_b[it];
                *reinterpret_cast<uint4*>(smem + OFF_W + off) = o_bhat[it];
                *reinterpret_cast<uint4*>(smem + OFF_ABAR + off) = o_abar[it];
                *reinterpret_cast<uint4*>(smem + OFF_RBAR + off) = o_rbar[it];
                float4* kh = reinterpret_cast<float4*>(F0 + t * 64 + 8 * j);
                kh[0] = o_khat[it][0];
                kh[1] = o_khat[it][1];
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 4. Gram: D1 = [k~; b~] [r~; a~]^T  (128 x 128 x 64) ---------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 128, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_D1, smem_desc(sbase + OFF_K + 32 * kk, 16, 1024),
                          smem_desc(sbase + OFF_R + 32 * kk, 16, 1024), id, kk > 0);
            umma_commit(bar_mma);
        }
        wait_or_abort(bar_mma, mma_phase, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- 5. epilogue 1: masked A_rk^T, A_ak, A_rb^T (bf16), A_ab (fp32) ----------------
        {
            float v[64];
            tmem_row<4>(tmem + TM_D1, wq, 64 * wh, v);
            if (wq < 2) {
                const int s = m_row;  // row of k~
                if (wh == 0) {  // A_rk[t][s] = v[t], kept for s <= t -> A_rk^T row s
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = (s <= 8 * c + e) ? v[8 * c + e] : 0.f;
                        *reinterpret_cast<uint4*>(smem + OFF_ARKT + sw(s, c)) = pack8(x);
                    }
                } else {  // A_ak[t][s] = v[t], kept for s < t -> column s of the A_ak tile
#pragma unroll
                    for (int t = 0; t < 64; ++t)
                        *reinterpret_cast<__nv_bfloat16*>(smem + OFF_AAK + swe(t, s)) =
                            __float2bfloat16_rn(s < t ? v[t] : 0.f);
                }
            } else {
                const int s = m_row - 64;  // row of b~
                if (wh == 0) {  // A_rb[t][s], s <= t -> A_rb^T row s
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = (s <= 8 * c + e) ? v[8 * c + e] : 0.f;
                        *reinterpret_cast<uint4*>(smem + OFF_ARBT + sw(s, c)) = pack8(x);
                    }
                } else {  // A_ab[t][s], s < t -> fp32 [t][s]
                    float* aab = reinterpret_cast<float*>(smem + OFF_AAB);
#pragma unroll
                    for (int t = 0; t < 64; ++t) aab[t * 64 + s] = s < t ? v[t] : 0.f;
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 6. T = (I - A_ab)^-1 by forward substitution, 4 threads per column -----------
        {
            const int jj = lane >> 2, hq = lane & 3;
            const int j = 8 * warp + jj;
            const float* aab = reinterpret_cast<const float*>(smem + OFF_AAB);
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = 0.f;
#pragma unroll
            for (int t = 0; t < 64; ++t) {
                float acc = 0.f;
                if (t > 0) {
#pragma unroll
                    for (int i = 0; i <= (t - 1) / 16; ++i) {
                        const float4 arow =
                            *reinterpret_cast<const float4*>(aab + t * 64 + 16 * i + 4 * hq);
                        acc = fmaf(arow.x, x[4 * i + 0], acc);
                        acc = fmaf(arow.y, x[4 * i + 1], acc);
                        acc = fmaf(arow.z, x[4 * i + 2], acc);
                        acc = fmaf(arow.w, x[4 * i + 3], acc);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                const float val = (t == j) ? 1.f : acc;
                if (hq == ((t >> 2) & 3)) x[(t >> 4) * 4 + (t & 3)] = val;
            }
            // T^T row j (MN-major B of MMA-2): elements (j, t) = T[t][j]
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t0 = 16 * i + 4 * hq;
                uint2 u = make_uint2(pack2(x[4 * i], x[4 * i + 1]), pack2(x[4 * i + 2], x[4 * i + 3]));
                *reinterpret_cast<uint2*>(smem + OFF_TT + swe(j, t0)) = u;
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 7. MMA-2: [W^T; Z^T] = [Abar^T; A_ak^T] T^T  (128 x 64 x 64) -----------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_D2, smem_desc(sbase + OFF_ABAR + 2048 * kk, OFF_AAK - OFF_ABAR, 1024),
                          smem_desc(sbase + OFF_TT + 2048 * kk, 8192, 1024), id, kk > 0);
            umma_commit(bar_mma);
        }
        wait_or_abort(bar_mma, mma_phase, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- 8. epilogue 2: [W^T; Z^T] -> bf16 K-major B of MMA-3 ---------------------------
        {
            float v[32];
            tmem_row<2>(tmem + TM_D2, wq, 32 * wh, v);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(smem + OFF_WZT + sw(m_row, 4 * wh + c)) = pack8(v + 8 * c);
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 9. MMA-3: [Bhat^T; A_rb] [W | Z]  (128 x 128 x 64) ----------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 128, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_D1, smem_desc(sbase + OFF_W + 2048 * kk, OFF_ARBT - OFF_W, 1024),
                          smem_desc(sbase + OFF_WZT + 32 * kk, 16, 1024), id, kk > 0);
            umma_commit(bar_mma);
        }
        wait_or_abort(bar_mma, mma_phase, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- 10. epilogue 3: assemble the final A operand ---------------------------------
        {
            float v[64];
            tmem_row<4>(tmem + TM_D1, wq, 64 * wh, v);
            if (wq < 2) {
                const int k = m_row;
                if (wh == 0) {  // M' = Bhat^T W
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4*>(smem + OFF_FIN0 + sw(k, c)) = pack8(v + 8 * c);
                } else {  // P_N = Bhat^T Z + Khat^T, split into bf16 hi + lo
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float hi[8], lo[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = 8 * c + e;
                            const float p = v[s] + F0[s * 64 + k];
                            hi[e] = __bfloat162float(__float2bfloat16_rn(p));
                            lo[e] = p - hi[e];
                        }
                        *reinterpret_cast<uint4*>(smem + OFF_FIN1 + sw(k, c)) = pack8(hi);
                        *reinterpret_cast<uint4*>(smem + OFF_FIN2 + sw(k, c)) = pack8(lo);
                    }
                }
            } else {
                const int tp = m_row - 64;
                if (wh == 0) {  // Q = A_rb W + Rbar
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float rb[8];
                        unpack8(*reinterpret_cast<const uint4*>(smem + OFF_RBAR + sw(tp, c)), rb);
#pragma unroll
                        for (int e = 0; e < 8; ++e) rb[e] += v[8 * c + e];
                        *reinterpret_cast<uint4*>(smem + OFF_FIN0 + sw(m_row, c)) = pack8(rb);
                    }
                } else {  // P_O = A_rb Z + A_rk; the lo block is zero for these rows
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float po[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            po[e] = v[8 * c + e] + bf16_at(smem + OFF_ARKT, 8 * c + e, tp);
                        *reinterpret_cast<uint4*>(smem + OFF_FIN1 + sw(m_row, c)) = pack8(po);
                        *reinterpret_cast<uint4*>(smem + OFF_FIN2 + sw(m_row, c)) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 11. final MMA: [S upd; O] = A_fin [S0; V; V]  (128 x 64 x 192) --------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int blk = 0; blk < 3; ++blk) {
                const uint32_t aoff = blk == 0 ? OFF_FIN0 : (blk == 1 ? OFF_FIN1 : OFF_FIN2);
                const uint32_t boff = blk == 0 ? OFF_S0 : OFF_V;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_DF, smem_desc(sbase + aoff + 32 * kk, 16, 1024),
                              smem_desc(sbase + boff + 2048 * kk, 8192, 1024), id, (blk | kk) != 0);
            }
            umma_commit(bar_mma);
        }
        wait_or_abort(bar_mma, mma_phase, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- 12. epilogue 4: state carry (fp32) and the chunk's outputs ---------------------
        {
            float v[32];
            tmem_row<2>(tmem + TM_DF, wq, 32 * wh, v);
            if (state_thread) {
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = fmaf(gamma, S[j], v[j]);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(smem + OFF_S0 + sw(m_row, 4 * wh + c)) = pack8(S + 8 * c);
            } else {
                const int t = m_row - 64;
                if (t < nv) {
                    uint4* dst = reinterpret_cast<uint4*>(o + ((size_t)(row0 + c0 + t) * H + h) * 64 + 32 * wh);
#pragma unroll
                    for (int c = 0; c < 4; ++c) dst[c] = pack8(v + 8 * c);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }
        if (*abort_flag) break;
    }

    if (state_thread && sT && !*abort_flag) {
        float4* dst = reinterpret_cast<float4*>(sT + state_off + m_row * 64 + 32 * wh);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [rows, H, 64] bf16 tensor viewed as (64, H, rows); box = 64 tokens of one head.
inline bool make_map(CUtensorMap* map, const void* ptr, long long rows, int H) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {64 * 2, (cuuint64_t)H * 64 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace chunked

inline cudaError_t launch_chunked(const void* r, const void* w, const void* k, const void* v,
                                  const void* a, const void* b, const float* s0,
                                  const uint8_t* mask, void* o, float* sT, int B, int T, int H,
                                  int N, const int32_t* cu_seqlens, cudaStream_t stream) {
    using namespace chunked;
    const long long rows = (long long)B * T;
    CUtensorMap maps[6];
    const void* ptrs[6] = {r, w, k, v, a, b};
    for (int i = 0; i < 6; ++i)
        if (!make_map(&maps[i], ptrs[i], rows, H)) return cudaErrorInvalidValue;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunked_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    chunked_kernel<<<(unsigned)((long long)N * H), kThreads, kSmemBytes, stream>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], s0, mask,
        static_cast<__nv_bfloat16*>(o), sT, T, H, cu_seqlens);
    return cudaGetLastError();
}

}  // namespace wkv7
