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
constexpr uint32_t OFF_R = 0;          // raw r -> r~        (Gram A rows 0..63)
constexpr uint32_t OFF_A = 8192;       // raw a -> a~        (Gram A rows 64..127)
constexpr uint32_t OFF_K = 16384;      // raw k -> k~        (Gram B rows 0..63)
constexpr uint32_t OFF_B = 24576;      // raw b -> b~        (Gram B rows 64..127)
constexpr uint32_t OFF_W = 32768;      // raw w -> Bhat      (MMA-3 A, MN-major atom 0)
constexpr uint32_t OFF_V = 40960;      // raw v              (final MMA B, MN-major)
constexpr uint32_t OFF_ABAR = 49152;   // Abar [s][k]        (MMA-2 A, MN-major atom 0)
constexpr uint32_t OFF_AAK = 57344;    // A_ak [s][s']       (MMA-2 A, MN-major atom 1)
constexpr uint32_t OFF_ARBT = 65536;   // A_rb^T [s][t]      (MMA-3 A, MN-major atom 1)
constexpr uint32_t OFF_ARK = 73728;    // A_rk [t][s]        (epilogue 3); prologue scratch
constexpr uint32_t OFF_RBAR = 81920;   // Rbar [t][k]        (epilogue 3)
constexpr uint32_t OFF_S0 = 90112;     // S0 bf16 [k][v]     (final MMA B, MN-major)
constexpr uint32_t OFF_F0 = 98304;     // fp32 64x64: E_t, then Khat [s][k]
constexpr uint32_t OFF_MISC = 114688;  // mbarriers, TMEM address, abort flag
constexpr uint32_t OFF_GAMMA = OFF_MISC + 64;  // e^{g_L} per channel (64 fp32)
constexpr uint32_t kSmemBytes = OFF_GAMMA + 256;
// Aliases (lifetimes do not overlap).
constexpr uint32_t OFF_AAB = OFF_R;    // fp32 A_ab [t][s] (epilogue 1 -> solve), 16 KB
constexpr uint32_t OFF_TF = OFF_K;     // fp32 T [t][s]    (solve), 16 KB
constexpr uint32_t OFF_TT = OFF_R;     // T^T [s][t]      (solve -> MMA-2 B, MN-major)
constexpr uint32_t OFF_WZT = OFF_K;    // [W^T; Z^T] [n][t] 128 rows (MMA-3 B, K-major)
constexpr uint32_t OFF_FIN0 = OFF_R;   // final A, K block 0: [M'; Rbar + A_rb W]
constexpr uint32_t OFF_FIN1 = OFF_ABAR;// final A, K block 1: [P_N hi; A_rk + A_rb Z]
constexpr uint32_t OFF_FIN2 = OFF_K;   // final A, K block 2: [P_N lo; 0]
// Prologue scratch inside the A_rk tile (free until epilogue 1), in floats.
constexpr int SCR_TOT = 0, SCR_EC = 512, SCR_EMC = 576, SCR_ELC = 640, SCR_VALID = 704;
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

// Float index of (row, col) in a 64x64 fp32 tile whose 16-byte chunks are permuted
// within each 64-byte group by bits 2..3 of the row, so that four rows 4 apart
// read with float4 loads hit different banks.
__device__ __forceinline__ int fidx(int row, int col) {
    return row * 64 + ((((col >> 2) ^ ((row >> 2) & 3)) << 2) | (col & 3));
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

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// Warp-level D += A * B, m16n8k8, tf32 operands, fp32 accumulate.  Fragment
// ownership (g = lane / 4, q = lane % 4): A (g|g+8, q|q+4), B (k = q|q+4, n = g),
// C/D (g|g+8, 2q|2q+1).
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16x16x16 product of fp32 blocks in an fidx tile: acc += X[xr.., xc..] * Y[yr.., yc..].
__device__ __forceinline__ void block_mma(float (&acc)[2][4], const float* X, int xr, int xc,
                                          const float* Y, int yr, int yc, int lane) {
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = to_tf32(X[fidx(xr + g, xc + 8 * ks + q)]);
        const uint32_t a1 = to_tf32(X[fidx(xr + g + 8, xc + 8 * ks + q)]);
        const uint32_t a2 = to_tf32(X[fidx(xr + g, xc + 8 * ks + q + 4)]);
        const uint32_t a3 = to_tf32(X[fidx(xr + g + 8, xc + 8 * ks + q + 4)]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(Y[fidx(yr + 8 * ks + q, yc + 8 * nt + g)]);
            const uint32_t b1 = to_tf32(Y[fidx(yr + 8 * ks + q + 4, yc + 8 * nt + g)]);
            mma_tf32(acc[nt], a0, a1, a2, a3, b0, b1);
        }
    }
}

__device__ __forceinline__ void store_block(float* Tf, int r0, int c0, const float (&acc)[2][4],
                                            int lane) {
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        Tf[fidx(r0 + g, c0 + 8 * nt + 2 * q)] = acc[nt][0];
        Tf[fidx(r0 + g, c0 + 8 * nt + 2 * q + 1)] = acc[nt][1];
        Tf[fidx(r0 + g + 8, c0 + 8 * nt + 2 * q)] = acc[nt][2];
        Tf[fidx(r0 + g + 8, c0 + 8 * nt + 2 * q + 1)] = acc[nt][3];
    }
}

// Level L of the blocked inverse on warp-level tensor-core MMAs (tf32 operands,
// fp32 accumulation): warp j computes block (i, j), i = j + L, as
// T_ij = T_ii * sum_{m=j}^{i-1} A_im T_mj, staging the sum in block (i, j) itself.
template <int L>
__device__ __forceinline__ void solve_level_mma(const float* A, float* Tf, int warp, int lane) {
    if (warp >= 4 - L) return;
    const int j = warp, i = j + L;
    float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int d = 0; d < L; ++d) block_mma(y, A, 16 * i, 16 * (j + d), Tf, 16 * (j + d), 16 * j, lane);
    store_block(Tf, 16 * i, 16 * j, y, lane);
    __syncwarp();
    float z[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    block_mma(z, Tf, 16 * i, 16 * i, Tf, 16 * i, 16 * j, lane);
    __syncwarp();
    store_block(Tf, 16 * i, 16 * j, z, lane);
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
    float* scratch = reinterpret_cast<float*>(smem + OFF_ARK);  // prologue only
    uint8_t* validb = reinterpret_cast<uint8_t*>(scratch + SCR_VALID);
    float* F0 = reinterpret_cast<float*>(smem + OFF_F0);
    float* gamma_s = reinterpret_cast<float*>(smem + OFF_GAMMA);
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
            const int p = tid & 31, q = tid >> 5;  // channels 2p, 2p+1; tokens 8q .. 8q+7
            float2 gl[8];
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = 8 * q + i;
                const bool val = t < nv && (!mask || mask[row0 + c0 + t] != 0);
                const float2 wv = __bfloat1622float2(
                    *reinterpret_cast<const __nv_bfloat162*>(smem + OFF_W + swe(t, 2 * p)));
                acc.x += val ? wv.x : 0.f;
                acc.y += val ? wv.y : 0.f;
                gl[i] = acc;
                if (p == 0) validb[t] = val ? 1 : 0;
            }
            reinterpret_cast<float2*>(scratch + SCR_TOT + q * 64)[p] = acc;
            __syncthreads();
            float2 prefix = make_float2(0.f, 0.f), c = prefix, gL = prefix;
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                const float2 tq = reinterpret_cast<const float2*>(scratch + SCR_TOT + qq * 64)[p];
                if (qq < q) { prefix.x += tq.x; prefix.y += tq.y; }
                if (qq < 4) { c.x += tq.x; c.y += tq.y; }
                gL.x += tq.x; gL.y += tq.y;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                reinterpret_cast<float2*>(F0 + (8 * q + i) * 64)[p] =
                    make_float2(clamped_exp(prefix.x + gl[i].x - c.x),
                                clamped_exp(prefix.y + gl[i].y - c.y));
            if (q == 0) {
                reinterpret_cast<float2*>(scratch + SCR_EC)[p] =
                    make_float2(clamped_exp(c.x), clamped_exp(c.y));
                reinterpret_cast<float2*>(scratch + SCR_EMC)[p] =
                    make_float2(clamped_exp(-c.x), clamped_exp(-c.y));
                reinterpret_cast<float2*>(scratch + SCR_ELC)[p] =
                    make_float2(clamped_exp(gL.x - c.x), clamped_exp(gL.y - c.y));
                reinterpret_cast<float2*>(gamma_s)[p] = make_float2(__expf(gL.x), __expf(gL.y));
            }
            __syncthreads();
        }

        // ---- 3. scaled operands (two 8-channel pieces per thread); each thread rewrites
        //         only the chunks it read, and Khat waits until every E_t read is done ----
        {
            float4 o_khat[2][2];
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int item = tid + 256 * it;
                const int t = item >> 3, j = item & 7;
                const bool val = validb[t] != 0;
                const uint32_t off = sw(t, j);
                float rv[8], av[8], kv[8], bv[8];
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_R + off), rv);
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_A + off), av);
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_K + off), kv);
                unpack8(*reinterpret_cast<const uint4*>(smem + OFF_B + off), bv);
                float E[8], Em[8], ec[8], elc[8];
                const float* Erow = F0 + t * 64 + 8 * j;
                const float* Emrow = t > 0 ? F0 + (t - 1) * 64 + 8 * j : scratch + SCR_EMC + 8 * j;
                *reinterpret_cast<float4*>(E) = reinterpret_cast<const float4*>(Erow)[0];
                *reinterpret_cast<float4*>(E + 4) = reinterpret_cast<const float4*>(Erow)[1];
                *reinterpret_cast<float4*>(Em) = reinterpret_cast<const float4*>(Emrow)[0];
                *reinterpret_cast<float4*>(Em + 4) = reinterpret_cast<const float4*>(Emrow)[1];
                *reinterpret_cast<float4*>(ec) = reinterpret_cast<const float4*>(scratch + SCR_EC + 8 * j)[0];
                *reinterpret_cast<float4*>(ec + 4) = reinterpret_cast<const float4*>(scratch + SCR_EC + 8 * j)[1];
                *reinterpret_cast<float4*>(elc) = reinterpret_cast<const float4*>(scratch + SCR_ELC + 8 * j)[0];
                *reinterpret_cast<float4*>(elc + 4) = reinterpret_cast<const float4*>(scratch + SCR_ELC + 8 * j)[1];
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
                *reinterpret_cast<uint4*>(smem + OFF_R + off) = pack8(rt);
                *reinterpret_cast<uint4*>(smem + OFF_A + off) = pack8(at);
                *reinterpret_cast<uint4*>(smem + OFF_K + off) = pack8(kt);
                *reinterpret_cast<uint4*>(smem + OFF_B + off) = pack8(btl);
                *reinterpret_cast<uint4*>(smem + OFF_W + off) = pack8(bhat);
                *reinterpret_cast<uint4*>(smem + OFF_ABAR + off) = pack8(abar);
                *reinterpret_cast<uint4*>(smem + OFF_RBAR + off) = pack8(rbar);
                o_khat[it][0] = make_float4(khat[0], khat[1], khat[2], khat[3]);
                o_khat[it][1] = make_float4(khat[4], khat[5], khat[6], khat[7]);
            }
            __syncthreads();  // every E_t read before F0 is overwritten by Khat
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int item = tid + 256 * it;
                const int t = item >> 3, j = item & 7;
                float4* kh = reinterpret_cast<float4*>(F0 + t * 64 + 8 * j);
                kh[0] = o_khat[it][0];
                kh[1] = o_khat[it][1];
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 4. Gram: D1 = [r~; a~] [k~; b~]^T  (128 x 128 x 64) ---------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 128, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_D1, smem_desc(sbase + OFF_R + 32 * kk, 16, 1024),
                          smem_desc(sbase + OFF_K + 32 * kk, 16, 1024), id, kk > 0);
            umma_commit(bar_mma);
        }
        wait_or_abort(bar_mma, mma_phase, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- 5. epilogue 1: rows t of D1 -> masked A_rk, A_rb^T, A_ak (bf16), A_ab (fp32) --
        {
            float v[64];
            tmem_row<4>(tmem + TM_D1, wq, 64 * wh, v);
            if (wq < 2) {
                const int t = m_row;  // row of r~
                if (wh == 0) {  // A_rk[t][s] = v[s], kept for s <= t -> row t
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = (8 * c + e <= t) ? v[8 * c + e] : 0.f;
                        *reinterpret_cast<uint4*>(smem + OFF_ARK + sw(t, c)) = pack8(x);
                    }
                } else {  // A_rb[t][s] = v[s], kept for s <= t -> column t of A_rb^T
#pragma unroll
                    for (int s_ = 0; s_ < 64; ++s_)
                        *reinterpret_cast<__nv_bfloat16*>(smem + OFF_ARBT + swe(s_, t)) =
                            __float2bfloat16_rn(s_ <= t ? v[s_] : 0.f);
                }
            } else {
                const int t = m_row - 64;  // row of a~
                if (wh == 0) {  // A_ak[t][s] = v[s], kept for s < t -> row t
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = (8 * c + e < t) ? v[8 * c + e] : 0.f;
                        *reinterpret_cast<uint4*>(smem + OFF_AAK + sw(t, c)) = pack8(x);
                    }
                } else {  // A_ab[t][s], kept for s < t -> fp32 row t
                    float* aab = reinterpret_cast<float*>(smem + OFF_AAB);
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4) {
                        float4 x;
                        x.x = (4 * c4 + 0 < t) ? v[4 * c4 + 0] : 0.f;
                        x.y = (4 * c4 + 1 < t) ? v[4 * c4 + 1] : 0.f;
                        x.z = (4 * c4 + 2 < t) ? v[4 * c4 + 2] : 0.f;
                        x.w = (4 * c4 + 3 < t) ? v[4 * c4 + 3] : 0.f;
                        *reinterpret_cast<float4*>(aab + fidx(t, 4 * c4)) = x;
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 6. T = (I - A_ab)^-1: 16x16 diagonal blocks by fp32 forward substitution,
        //         then the off-diagonal blocks level by level on warp MMAs,
        //         T_ij = T_ii * sum_{m=j}^{i-1} A_im T_mj ------------------------------------
        {
            const float* A = reinterpret_cast<const float*>(smem + OFF_AAB);
            float* Tf = reinterpret_cast<float*>(smem + OFF_TF);
            if (tid < 64) {  // diagonal block b, column c
                const int b = tid >> 4, c = tid & 15, base = 16 * b;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = 0.f;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                    for (int s4 = 0; s4 < t; s4 += 4) {
                        const float4 a4 =
                            *reinterpret_cast<const float4*>(A + fidx(base + t, base + s4));
                        acc0 = fmaf(a4.x, x[s4 + 0], acc0);
                        acc1 = fmaf(a4.y, x[s4 + 1], acc1);
                        acc0 = fmaf(a4.z, x[s4 + 2], acc0);
                        acc1 = fmaf(a4.w, x[s4 + 3], acc1);
                    }
                    x[t] = (t == c) ? 1.f : acc0 + acc1;
                }
#pragma unroll
                for (int t = 0; t < 16; ++t) Tf[fidx(base + t, base + c)] = x[t];
            }
            __syncthreads();
            solve_level_mma<1>(A, Tf, warp, lane);
            __syncthreads();
            solve_level_mma<2>(A, Tf, warp, lane);
            __syncthreads();
            solve_level_mma<3>(A, Tf, warp, lane);
            __syncthreads();
            // T^T row j (MN-major B of MMA-2): elements (j, t) = T[t][j]; zero above the
            // diagonal blocks
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int item = tid + 256 * it;
                const int j = item >> 3, hc = item & 7;
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = 8 * hc + e;
                    x[e] = ((t >> 4) < (j >> 4)) ? 0.f : Tf[fidx(t, j)];
                }
                *reinterpret_cast<uint4*>(smem + OFF_TT + sw(j, hc)) = pack8(x);
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
                        unpack8(*reinterpret_cast<const uint4*>(smem + OFF_ARK + sw(tp, c)), po);
#pragma unroll
                        for (int e = 0; e < 8; ++e) po[e] += v[8 * c + e];
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
                const float gamma = gamma_s[m_row];  // e^{g_L} of this state row's channel
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
