// chunked_bwd.cuh -- backward of the WKV7 forward in the chunked (WY) form on tcgen05
// tensor cores, bf16, K = V = 64 (the README's training entry, generalized_delta_rule,
// supports backpropagation; rwkv-ops 0.9.0 README, "rwkv7op 使用方法").
//
// For L = sum(o * dout) + sum(S_T * dsT), with G_t = dL/dS_t,
//     G_t = r_t do_t^T + (diag(e^{w_{t+1}}) + a_{t+1} b_{t+1}^T) G_{t+1},   G_{T-1} = r do^T + dsT,
// and ds0 = (diag(e^{w_0}) + a_0 b_0^T) G_0.  Read backwards in time, that is itself a
// WKV7 recurrence: with X_tau = G_{L-1-tau},
//     X_tau = (diag(e^{w'_tau}) + b'_tau a'_tau^T) X_{tau-1} + k'_tau v'_tau^T
// where w'_tau = w_{L-tau}, b' = a_{L-tau}, a' = b_{L-tau} (tau >= 1; the identity at
// tau = 0) and k'_tau = r_{L-1-tau}, v'_tau = do_{L-1-tau} (tau < L), started from dsT;
// one more transition (tau = L, no input) gives ds0.  So the backward is four launches:
//   1. prep:     offsets of the reversed sequences (each padded at its start to a
//                multiple of 64 tokens: p = 63 - L % 64 identity steps, then L + 1 steps);
//   2. forward:  the chunked forward with per-chunk fp16 checkpoints of the state
//                S0 at every chunk start, and no outputs;
//   3. reversed: the same kernel over the reversed sequences from dsT, reading the
//                original tensors itself (a masked token's transition is the identity,
//                its output still feeds G; r' = k, so its outputs X_tau^T k_{L-1-tau} =
//                G_t^T k_t are dv, written in place, zero for a masked token): its final
//                state is ds0 and its per-chunk checkpoints hold G at the last token of
//                every chunk of the original sequence (the padding puts chunk boundaries
//                there);
//   4. grad:     the chunks in parallel (persistent, one CTA per SM): each chunk's
//                gradients from its inputs, S0 and dSL = G_e - r_e do_e^T (e its last
//                token; dSL = dsT for a partial last chunk), on tcgen05.
//
// The per-chunk adjoint (grad kernel), with the forward's chunk algebra (chunked.cuh):
//   X = Abar S0 + A_ak V,  U = T X                     (U = W S0 + Z V)
//   dU = A_rb^T dO + Bhat dSL,  dX = T^T dU,  dT = dU X^T
//   dA_rk = (dO V^T)_{s<=t}, dA_rb = (dO U^T)_{s<=t}, dA_ak = (dX V^T)_{s<t},
//   dA_ab = (T^T dT T^T)_{s<t}
//   acc_r = dA_rk k~ + dA_rb b~,  dRbar = dO S0^T       dr = E acc_r + e^{g_t} dRbar
//   acc_a = dA_ak k~ + dA_ab b~,  dAbar = dX S0^T       da = E_{t-1} acc_a + e^{g_{t-1}} dAbar
//   acc_k = dA_rk^T r~ + dA_ak^T a~ + V dSL^T            dk = acc_k / E
//   acc_b = dA_rb^T r~ + dA_ab^T a~ + U dSL^T            db = acc_b / E
//   dw_t = R - a_t da_t - sum_{t' < t} (r dr - k dk - b db + a da)_{t'}
//   R = rowsum(S0 * (Rbar^T dO + Abar^T dX + e^{g_L} dSL))        (per channel)
// (the adjoint of the E_t, E_{t-1} and e^{g_L} factors, summed back over the in-chunk
// prefix of w).  e^{g_t} = E_t e^{g_L} is applied in fp32 in the last step: folded into
// an fp16 operand (e^{g_L} S0) it would underflow once a chunk's decay is strong.  A masked token has zero dw, dk, da, db (its fold w = 0, a = k = b = 0
// has no derivative); dv comes from the reversed run.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "chunked.cuh"

namespace wkv7 {
namespace cbwd {

using namespace chunked;
using namespace sm100;

constexpr int kThreads = 512;  // the gradient kernel: 16 warps

// ---------------------------------------------------------------------------------
// Workspace layout (bytes, each region 256-aligned).
// ---------------------------------------------------------------------------------
struct Ws {
    long long rows, rowsR;   // token rows of the inputs; bound on the reversed rows
    long long slotsF, slotsR;  // checkpoint slots per head (forward, reversed)
    size_t off_cu, off_ckF, off_ckR, total;
};
inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
inline Ws ws_layout(long long rows, int N, int H) {
    Ws w;
    w.rows = rows;
    w.rowsR = rows + 64LL * N;
    w.slotsF = rows / 64 + N + 1;
    w.slotsR = w.rowsR / 64 + N + 1;
    w.off_cu = 0;
    w.off_ckF = al256((size_t)(N + 1) * 4);
    w.off_ckR = al256(w.off_ckF + (size_t)H * w.slotsF * 8192);
    w.total = al256(w.off_ckR + (size_t)H * w.slotsR * 8192);
    return w;
}

// Sequence n: first token row in the [B*T] row space and length.
__device__ __forceinline__ void seq_of(int n, int T, const int32_t* cu, long long& row0, int& L,
                                       bool& ok) {
    if (cu) {
        const int bos = cu[n], eos = cu[n + 1];
        ok = bos >= 0 && eos >= bos && eos <= T;
        row0 = bos;
        L = eos - bos;
    } else {
        ok = true;
        row0 = (long long)n * T;
        L = T;
    }
}

// ---------------------------------------------------------------------------------
// 1. prep: cu'[n] = sum_{m<n} 64 (floor(L_m / 64) + 1), one CTA.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) prep_kernel(const int32_t* __restrict__ cu, int T, int N,
                                                    int32_t* __restrict__ cur) {
    __shared__ int32_t tot[32];
    __shared__ int32_t carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int n = base + tid;
        int lr = 0;
        if (n < N) {
            long long row0;
            int L;
            bool ok;
            seq_of(n, T, cu, row0, L, ok);
            if (!ok) {
                raise_flag(5 /* WKV7_ERR_DEVICE_BAD_SEQLENS */);
                L = 0;
            }
            lr = 64 * (L / 64 + 1);
        }
        int incl = lr;
#pragma unroll
        for (int d = 1; d < 32; d *= 2) {
            const int up = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += up;
        }
        if (lane == 31) tot[warp] = incl;
        __syncthreads();
        int pre = carry;
        for (int w2 = 0; w2 < warp; ++w2) pre += tot[w2];
        if (n < N) cur[n] = pre + incl - lr;
        __syncthreads();
        if (tid == 1023) carry = pre + incl;
        __syncthreads();
    }
    if (tid == 0) cur[N] = carry;
}

// ---------------------------------------------------------------------------------
// 5. grad: the per-chunk adjoint on tcgen05.
// ---------------------------------------------------------------------------------
// Shared-memory tiles (8 KB, 64 rows x 128 B, 128B swizzle).
enum : uint32_t {
    G_R = 0, G_A, G_K, G_B,  // r, a, k, b -> r~, a~, k~, b~ (bf16)
    G_W,                     // w -> Abar (fp16)
    G_V, G_DO,               // v, dO -> fp16 in place (dO rows past the chunk zeroed)
    G_S0, G_DS,              // S0 (fp16 checkpoint), G -> dSL (fp16)
    G_BH, G_RB, G_SPARE,     // Bhat, Rbar (fp16); a spare tile
    G_E, G_E2,               // E (fp32, two tiles)
    G_SP,                    // prologue scratch -> A_ab's diagonal blocks and T_ii; reloaded r
    G_AB,                    // A_ab's blocks left of the diagonal (fp16); reloaded k
    G_AAK, G_ARB,            // A_ak, A_rb (fp16, masked); reloaded a, b
    G_T,                     // T = (I - A_ab)^-1 (fp16)
    G_X, G_DU, G_DT,         // X -> U;  dU -> dX;  T_ii A_im scratch -> dT -> Y (fp16)
    G_DARK, G_DAAK, G_DARB, G_DAAB,  // dA_rk, dA_ak, dA_rb, dA_ab (bf16); then staging
    kNumTiles
};
constexpr uint32_t gt(uint32_t i) { return i * kTile; }
constexpr uint32_t GOFF_MISC = kNumTiles * kTile;
// misc: mbarriers (tma, mma, reload) at +0, +8, +16; TMEM address at +32;
constexpr uint32_t GOFF_GAMMA = GOFF_MISC + 64;      // e^{g_L} (64 fp32, plain order)
constexpr uint32_t GOFF_R = GOFF_GAMMA + 256;        // R per channel (64 fp32)
constexpr uint32_t GOFF_EM0 = GOFF_R + 256;          // E_{-1} per channel (64 fp32)
constexpr uint32_t GOFF_RAW = GOFF_EM0 + 256;        // raw r and dO of token 63 (2 x 64 fp32)
constexpr uint32_t GOFF_TOT = GOFF_RAW + 512;        // scan totals [4 quadrants][64]
constexpr uint32_t GOFF_NEXT = GOFF_TOT + 1024;      // the CTA's next work item (and index)
constexpr uint32_t GOFF_RP = GOFF_NEXT + 128;        // rowsum(S0 P) quarters [4][64] (fixed order)
constexpr uint32_t kGSmemBytes = GOFF_RP + 1024;
static_assert(kGSmemBytes <= 232448, "fits one CTA per SM");
constexpr uint32_t kGTmemCols = 512;
// TMEM columns (every accumulator M = 64): C0..C2 hold each phase's products for its
// epilogue; dRbar, dAbar, acc_k, acc_b and P have their own columns; acc_r and acc_a
// take C2 and C1 once phase C's epilogue has read them.
constexpr uint32_t C0 = 0, C1 = 64, C2 = 128, C_DRB = 192, C_DAB = 256, C_AK = 320, C_AB = 384,
                   C_P = 448, C_AR = 128, C_AA = 64;

// E tile index (fp32 [t][c], groups of 8 channels XOR-swizzled by row).
__device__ __forceinline__ int eidx(int t, int c) { return t * 64 + (c ^ ((t & 7) << 3)); }

// Store one warp's share (rows 16 wq.., columns 32 wh..) of the M = 64 accumulator at
// TMEM column `col` as a 16-bit tile; mode 1 keeps s <= t, mode 2 keeps s < t.
template <typename Pack>
__device__ __forceinline__ void acc_to_tile(uint32_t tmem, uint32_t col, uint32_t tile, int wq,
                                            int wh, int lane, int mode, Pack pk) {
    float v[16];
    tmem_frag(tmem + col, wq, 32 * wh, v);
    if (mode) {
        const int g = lane >> 2, q = lane & 3;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = 16 * wq + g + 8 * hr, s = 32 * wh + 8 * j + 2 * q + e;
                    if (mode == 1 ? s > t : s >= t) v[4 * j + 2 * hr + e] = 0.f;
                }
    }
    frag_to_tile(tile, 16 * wq, 4 * wh, v, lane, pk);
}

// One 16 x 16 block in fragment layout (sm100::tmem_ld16x16) to a 128B-swizzled tile:
// rows row0 .. row0 + 15, 16-byte chunks chunk0, chunk0 + 1 (one stmatrix.x4).
template <typename Pack>
__device__ __forceinline__ void frag8_to_tile(uint32_t tile, int row0, int chunk0, const float (&v)[8],
                                              int lane, Pack pk) {
    const int mi = lane >> 3;
    const uint32_t addr = tile + sw(row0 + 8 * (mi & 1) + (lane & 7), chunk0 + (mi >> 1));
    stsm_x4(addr, pk(v[0], v[1]), pk(v[2], v[3]), pk(v[4], v[5]), pk(v[6], v[7]));
}
// One warp's 16 x 16 block (rows 16 wq .., columns 16 wc ..) of the M = 64 accumulator at
// TMEM column `col` as a 16-bit tile; mode 1 keeps s <= t, mode 2 keeps s < t.
template <typename Pack>
__device__ __forceinline__ void acc16_to_tile(uint32_t tmem, uint32_t col, uint32_t tile, int wq,
                                              int wc, int lane, int mode, Pack pk) {
    float v[8];
    sm100::tmem_ld16x16(tmem + ((uint32_t)(32 * wq) << 16) + col + 16 * wc, v);
    sm100::tmem_ld_wait();
    if (mode) {
        const int g = lane >> 2, q = lane & 3;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = 16 * wq + g + 8 * hr, s = 16 * wc + 8 * j + 2 * q + e;
                    if (mode == 1 ? s > t : s >= t) v[4 * j + 2 * hr + e] = 0.f;
                }
    }
    frag8_to_tile(tile, 16 * wq, 2 * wc, v, lane, pk);
}

// D (+)= A B over K = 64 (four K16 steps) from 64-row tiles; a_mn / b_mn: the tile is
// stored MN-major for that operand (rows = the K index), else K-major (rows = M / N).
__device__ __forceinline__ void mma64(uint32_t tmem_d, uint32_t a, bool a_mn, uint32_t b, bool b_mn,
                                      bool bf16, bool acc) {
    const uint32_t id = bf16 ? idesc_bf16(64, 64, a_mn, b_mn) : idesc_f16(64, 64, a_mn, b_mn);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = a_mn ? smem_desc(a + 2048 * kk, 8192, 1024) : smem_desc(a + 32 * kk, 16, 1024);
        const uint64_t db = b_mn ? smem_desc(b + 2048 * kk, 8192, 1024) : smem_desc(b + 32 * kk, 16, 1024);
        umma_bf16(tmem_d, da, db, id, (acc || kk > 0) ? 1u : 0u);
    }
}

// Work item `it` (slot fastest, then head) -> the chunk: sequence n with
// floor(row0_n / 64) + n <= slot, its chunk c; false for a slot that no chunk maps to.
struct Item {
    int n, c, h, L, nv, slot, rslot;
    long long row0, crow;
};
__device__ __forceinline__ bool item_of(int it, int slotsF, int T, int N, const int32_t* cu,
                                        Item& I) {
    I.h = it / slotsF;
    I.slot = it - I.h * slotsF;
    if (!cu && (T & 63) == 0) {  // equal lengths, a multiple of 64: T / 64 + 1 slots each
        const int per = T / 64 + 1;
        I.n = I.slot / per;
        I.c = I.slot - I.n * per;
        I.L = T;
        I.row0 = (long long)I.n * T;
        if (I.n >= N || I.c >= T / 64) return false;
        I.nv = 64;
        I.crow = I.row0 + 64LL * I.c;
        return true;
    }
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const long long r0 = cu ? (long long)cu[mid] : (long long)mid * T;
        if ((r0 >> 6) + mid <= I.slot) lo = mid; else hi = mid - 1;
    }
    I.n = lo;
    bool ok;
    seq_of(I.n, T, cu, I.row0, I.L, ok);
    if (!ok) return false;  // flagged by prep
    I.c = I.slot - (int)((I.row0 >> 6) + I.n);
    if (I.c < 0 || 64 * I.c >= I.L) return false;
    I.nv = min(64, I.L - 64 * I.c);
    I.crow = I.row0 + 64LL * I.c;
    return true;
}
// The first item with a chunk among it, it + gridDim.x, ..., or -1; with the slot of its
// state-gradient checkpoint (reversed sequence n starts at cur[n]).
__device__ __forceinline__ int next_item(int it, int total, int slotsF, int T, int N,
                                         const int32_t* cu, const int32_t* cur, Item& I) {
    for (; it < total; it += gridDim.x)
        if (item_of(it, slotsF, T, N, cu, I)) {
            // reversed sequences are 64 (floor(L / 64) + 1) rows each: closed form for
            // equal lengths
            const int c0r = cu ? cur[I.n] / 64 : I.n * (T / 64 + 1);
            I.rslot = c0r + I.n + I.L / 64 - I.c;
            return it;
        }
    return -1;
}

// Persistent: CTA b takes work items b, b + gridDim.x, ... (one CTA per SM); each
// chunk's nine input tiles are loaded while the previous chunk's final epilogue runs.
template <bool kHf>
__global__ void __launch_bounds__(kThreads, 1)
grad_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_w,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
            const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_ckf,
            const __grid_constant__ CUtensorMap tm_ckr, const __grid_constant__ CUtensorMap tm_dr,
            const __grid_constant__ CUtensorMap tm_dw, const __grid_constant__ CUtensorMap tm_dk,
            const __grid_constant__ CUtensorMap tm_da, const __grid_constant__ CUtensorMap tm_db,
            const uint8_t* __restrict__ mask, const int32_t* __restrict__ cu,
            const int32_t* __restrict__ cur, int T, int H, int N, int slotsF, int slotsR,
            __nv_bfloat16* __restrict__ dr, __nv_bfloat16* __restrict__ dw,
            __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ da,
            __nv_bfloat16* __restrict__ db) {
    extern __shared__ __align__(1024) uint8_t smem[];
    using namespace sm100;
    // 16 warps: wq = TMEM lane quadrant (rows 16 wq .. of an M = 64 accumulator), wc =
    // 16-column quarter of it in the epilogues; warps 0..7 keep the single-thread and
    // warp roles (MMA issue, T, the A_ab inverses, TMA issue)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wq = warp & 3, wc = warp >> 2;
    const int g = lane >> 2, q = lane & 3;
    const int total = slotsF * H;  // below 2^31 (checked on the host)

    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_tma = sbase + GOFF_MISC, bar_mma = sbase + GOFF_MISC + 8,
                   bar_rl = sbase + GOFF_MISC + 16;
    float* gam = reinterpret_cast<float*>(smem + GOFF_GAMMA);
    float* Rc = reinterpret_cast<float*>(smem + GOFF_R);
    float* em0 = reinterpret_cast<float*>(smem + GOFF_EM0);
    float* raw = reinterpret_cast<float*>(smem + GOFF_RAW);
    float* tot = reinterpret_cast<float*>(smem + GOFF_TOT);
    float* Ef = reinterpret_cast<float*>(smem + gt(G_E));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + GOFF_MISC + 32);
    int timed_out = 0;
    uint32_t mph = 0, tph = 0, rph = 0;

    Item I, In;
    int it = next_item(blockIdx.x, total, slotsF, T, N, cu, cur, I);
    if (it < 0) return;

    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kGTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_rl, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == 1 && lane < 14) {
        const CUtensorMap* maps[14] = {&tm_r, &tm_w, &tm_k, &tm_v, &tm_a, &tm_b, &tm_do,
                                       &tm_ckf, &tm_ckr, &tm_dr, &tm_dw, &tm_dk, &tm_da, &tm_db};
        prefetch_tensormap(maps[lane]);
    }

    // Input tile i (0..8) of item J: r, a, k, b, w, v, dO by the input maps (token-major:
    // (channel, head, token row); head first: (channel, token, b*H + h)), S0 and G from
    // the two checkpoint arrays.  Each TMA instruction takes a few hundred cycles to
    // issue, so the nine are spread over the warps.
    auto load_in = [&](const Item& J, int i) {
        const int jy = kHf ? (int)(J.crow % T) : J.h;
        const int jz = kHf ? (int)((J.crow / T) * H + J.h) : (int)J.crow;
        const CUtensorMap* map = i == 0 ? &tm_r : i == 1 ? &tm_a : i == 2 ? &tm_k
                               : i == 3 ? &tm_b : i == 4 ? &tm_w : i == 5 ? &tm_v
                               : i == 6 ? &tm_do : i == 7 ? &tm_ckf : &tm_ckr;
        const uint32_t dst = i == 0 ? G_R : i == 1 ? G_A : i == 2 ? G_K : i == 3 ? G_B
                           : i == 4 ? G_W : i == 5 ? G_V : i == 6 ? G_DO : i == 7 ? G_S0 : G_DS;
        if (i < 7)
            tma_load_3d(sbase + gt(dst), map, bar_tma, 0, jy, jz);
        else
            tma_load_3d(sbase + gt(dst), map, bar_tma, 0, 0,
                        i == 7 ? J.h * slotsF + J.slot : J.h * slotsR + J.rslot);
    };
    if (warp == 0) {
        if (lane == 0) mbar_arrive_expect_tx(bar_tma, 9 * kTile);
        __syncwarp();
        if (lane < 9) load_in(I, lane);
    }
    // rowsum(S0 P) partials, one per 16-column quarter (added in a fixed order)
    float* Rq = reinterpret_cast<float*>(smem + GOFF_RP);

    // The previous chunk's outputs (dr dw dk da db), staged in the dA tiles and X: five
    // TMA tile stores (one per warp), or the rows < nv copied for a partial chunk (the
    // rows after belong to another sequence).  Called by every thread after a barrier.
    int p_nv = 0, p_h = 0, p_cy = 0, p_cz = 0;
    long long p_crow = 0;
    auto flush = [&]() {
        if (p_nv == 0) return;
        const uint32_t stg[5] = {G_DARK, G_X, G_DAAK, G_DAAB, G_DARB};  // dr dw dk da db
        if (p_nv == 64) {
            if (lane == 0 && warp >= 8 && warp < 13) {  // warps 8..12 (warp 0 scans next)
                const int ws = warp - 8;
                const CUtensorMap* map = ws == 0 ? &tm_dr : ws == 1 ? &tm_dw : ws == 2 ? &tm_dk
                                       : ws == 3 ? &tm_da : &tm_db;
                tma_store_3d(map, sbase + gt(stg[ws]), 0, p_cy, p_cz);
                bulk_commit();
            }
        } else {
            __nv_bfloat16* outs[5] = {dr, dw, dk, da, db};
            for (int i = tid; i < 5 * 64 * 8; i += kThreads) {
                const int which = i / 512, rem = i % 512, t = rem >> 3, chk = rem & 7;
                if (t >= p_nv) continue;
                const long long e = kHf ? (((p_crow / T) * H + p_h) * (long long)T + (p_crow % T) + t) * 64
                                        : ((p_crow + t) * H + p_h) * 64;
                *reinterpret_cast<uint4*>(outs[which] + e + 8 * chk) =
                    *reinterpret_cast<const uint4*>(smem + gt(stg[which]) + sw(t, chk));
            }
        }
        p_nv = 0;
    };

    while (it >= 0) {
    const int h = I.h, nv = I.nv;
    const long long crow = I.crow;
    const int cy = kHf ? (int)(crow % T) : h;
    const int cz = kHf ? (int)((crow / T) * H + h) : (int)crow;
    wait_or_abort(bar_tma, tph, timed_out);
    tph ^= 1;

    // ---- prologue: prefix sums of w (mask folded), E, and the operands; thread = one
    //      token t of the chunk, channels 8 j .. 8 j + 7 -------------------------------
    {
        float* scr = reinterpret_cast<float*>(smem + gt(G_SP));  // warp totals [16][64], g_L
        float* pre_s = reinterpret_cast<float*>(smem + gt(G_DT));  // exclusive prefixes [16][64]
        const int j = tid & 7, t = tid >> 3;
        const bool in = t < nv, val = in && (!mask || mask[crow + t] != 0);
        const uint32_t off = sw(t, j);
        const int h0 = cswz(8 * j), h1 = cswz(8 * j + 4);
        float wv[8], incl[8];
        {
            uint4 qa = *reinterpret_cast<const uint4*>(smem + gt(G_W) + off);
            if (!val) qa = make_uint4(0, 0, 0, 0);  // a masked token's w is zero
            unpack8(qa, wv);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            wv[e] *= kLog2e;  // log decays in log2 units from here on
            incl[e] = wv[e];
        }
#pragma unroll
        for (int d = 8; d < 32; d *= 2) {  // the warp's four tokens
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float up = __shfl_up_sync(0xffffffffu, incl[e], d);
                if (lane >= d) incl[e] += up;
            }
        }
        if (lane >= 24) {
            *reinterpret_cast<float4*>(scr + warp * 64 + h0) = make_float4(incl[0], incl[1], incl[2], incl[3]);
            *reinterpret_cast<float4*>(scr + warp * 64 + h1) = make_float4(incl[4], incl[5], incl[6], incl[7]);
        }
        if (__syncthreads_or(timed_out)) goto teardown;
        flush();  // the previous chunk's outputs
        if (warp == 0) {  // per channel pair: exclusive prefixes over the warps, g_L, e^{g_L}
            const int ch = cswz(2 * lane);
            float2 gL = make_float2(0.f, 0.f);
#pragma unroll
            for (int w2 = 0; w2 < kThreads / 32; ++w2) {
                const float2 x = *reinterpret_cast<const float2*>(scr + w2 * 64 + ch);
                *reinterpret_cast<float2*>(pre_s + w2 * 64 + ch) = gL;
                gL.x += x.x;
                gL.y += x.y;
            }
            *reinterpret_cast<float2*>(scr + 1024 + ch) = gL;
            gam[2 * lane] = ex2(gL.x);  // plain channel order (cswz keeps pairs together)
            gam[2 * lane + 1] = ex2(gL.y);
        }
        __syncthreads();
        float ga[8], cc[8], ec[8];
        {
            const float4 x0 = *reinterpret_cast<const float4*>(pre_s + warp * 64 + h0);
            const float4 x1 = *reinterpret_cast<const float4*>(pre_s + warp * 64 + h1);
            const float pre[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) ga[e] = pre[e] + incl[e];  // g at token t
        }
        *reinterpret_cast<float4*>(cc) = *reinterpret_cast<const float4*>(scr + 1024 + h0);
        *reinterpret_cast<float4*>(cc + 4) = *reinterpret_cast<const float4*>(scr + 1024 + h1);
#pragma unroll
        for (int e = 0; e < 8; ++e) ec[e] = gam[8 * j + e];
        float rv[8], av[8], kv[8], bv[8], vv[8], dv[8];
        unpack8(*reinterpret_cast<const uint4*>(smem + gt(G_R) + off), rv);
        unpack8(*reinterpret_cast<const uint4*>(smem + gt(G_A) + off), av);
        unpack8(*reinterpret_cast<const uint4*>(smem + gt(G_K) + off), kv);
        unpack8(*reinterpret_cast<const uint4*>(smem + gt(G_B) + off), bv);
        unpack8(*reinterpret_cast<const uint4*>(smem + gt(G_V) + off), vv);
        unpack8(*reinterpret_cast<const uint4*>(smem + gt(G_DO) + off), dv);
        if (t == 63) {  // raw r and dO of the last token (dSL = G - r do^T)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                raw[8 * j + e] = rv[e];
                raw[64 + 8 * j + e] = dv[e];
            }
        }
        float Ev[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float d = clamp2(ga[e] - cc[e]);
            const float E = ex2(d);                              // e^{g_t - g_L}
            const float Ep = ex2(clamp2(ga[e] - wv[e] - cc[e]));  // e^{g_{t-1} - g_L}
            if (t == 0) em0[8 * j + e] = Ep;
            const float inv = val ? ex2(-d) : 0.f;
            const float ep = val ? Ep : 0.f;
            rv[e] = in ? rv[e] * E : 0.f;  // r~
            av[e] = av[e] * ep;            // a~
            kv[e] = kv[e] * inv;           // k~
            bv[e] = bv[e] * inv;           // b~
            Ev[e] = E;
            if (!in) dv[e] = 0.f;
        }
        float ab[8], rb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            ab[e] = av[e] * ec[e];  // Abar = a~ e^{g_L}
            rb[e] = rv[e] * ec[e];  // Rbar = r~ e^{g_L}
        }
        *reinterpret_cast<uint4*>(smem + gt(G_R) + off) = pack8(rv);
        *reinterpret_cast<uint4*>(smem + gt(G_A) + off) = pack8(av);
        *reinterpret_cast<uint4*>(smem + gt(G_K) + off) = pack8(kv);
        *reinterpret_cast<uint4*>(smem + gt(G_B) + off) = pack8(bv);
        *reinterpret_cast<uint4*>(smem + gt(G_W) + off) = pack8h(ab);
        *reinterpret_cast<uint4*>(smem + gt(G_RB) + off) = pack8h(rb);
        *reinterpret_cast<uint4*>(smem + gt(G_BH) + off) = pack8h(bv);
        *reinterpret_cast<uint4*>(smem + gt(G_V) + off) = pack8h(vv);
        *reinterpret_cast<uint4*>(smem + gt(G_DO) + off) = pack8h(dv);
        *reinterpret_cast<float4*>(Ef + eidx(t, 8 * j)) = make_float4(Ev[0], Ev[1], Ev[2], Ev[3]);
        *reinterpret_cast<float4*>(Ef + eidx(t, 8 * j + 4)) = make_float4(Ev[4], Ev[5], Ev[6], Ev[7]);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
    }

    // ---- Gram: [A_ak | A_ab] = a~ [k~ | b~]^T, A_rb = r~ b~^T (bf16) ----------------
    if (tid == 0) {
        tc_fence_after();
        mma64(tmem + C0, sbase + gt(G_A), false, sbase + gt(G_K), false, true, false);
        mma64(tmem + C1, sbase + gt(G_A), false, sbase + gt(G_B), false, true, false);
        mma64(tmem + C2, sbase + gt(G_R), false, sbase + gt(G_B), false, true, false);
        umma_commit(bar_mma);
    }
    // While it runs: dSL (fp16) and R = e^{g_L} rowsum(S0 dSL); thread = state row c,
    // 8 of its columns.
    {
        const int row = tid >> 3, chk = tid & 7;
        const float gm = gam[row];
        const float rr = nv == 64 ? raw[row] : 0.f;
        const uint32_t off = sw(row, chk);
        const uint4 s4 = *reinterpret_cast<const uint4*>(smem + gt(G_S0) + off);
        const uint4 g4 = *reinterpret_cast<const uint4*>(smem + gt(G_DS) + off);
        const uint32_t sw4[4] = {s4.x, s4.y, s4.z, s4.w}, gw4[4] = {g4.x, g4.y, g4.z, g4.w};
        uint32_t go[4];
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sw4[i]));
            float2 gf = __half22float2(*reinterpret_cast<const __half2*>(&gw4[i]));
            const int v0 = 8 * chk + 2 * i;
            gf.x -= rr * raw[64 + v0];
            gf.y -= rr * raw[64 + v0 + 1];
            part = fmaf(sf.x, gf.x, fmaf(sf.y, gf.y, part));
            go[i] = pack2h(gf.x, gf.y);
        }
        *reinterpret_cast<uint4*>(smem + gt(G_DS) + off) = make_uint4(go[0], go[1], go[2], go[3]);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        part += __shfl_xor_sync(0xffffffffu, part, 4);
        if (chk == 0) Rc[row] = gm * part;
        fence_proxy_async();
    }
    wait_or_abort(bar_mma, mph, timed_out);
    mph ^= 1;
    tc_fence_after();

    // ---- Gram epilogue: warps 4..7 A_ab's diagonal inverses and left blocks; warps
    //      8..11 masked A_ak, 12..15 masked A_rb ------------------------------------------
    if (warp >= 4 && warp < 8) {
        float v[2][16];
        tmem_frag(tmem + C1, wq, 0, v[0]);
        tmem_frag(tmem + C1, wq, 32, v[1]);
        float* dg = reinterpret_cast<float*>(smem + gt(G_SP));
        {
            const bool hi = wq >= 2, odd = wq & 1;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int s2 = 8 * jj + 2 * q + e;
                    const int i0 = 4 * jj + e, i1 = 4 * (2 + jj) + e;
                    const float lo0 = odd ? v[0][i1] : v[0][i0], hi0 = odd ? v[1][i1] : v[1][i0];
                    const float lo1 = odd ? v[0][i1 + 2] : v[0][i0 + 2];
                    const float hi1 = odd ? v[1][i1 + 2] : v[1][i0 + 2];
                    dg[dtidx(wq, s2, g)] = (s2 < g) ? (hi ? hi0 : lo0) : 0.f;
                    dg[dtidx(wq, s2, g + 8)] = (s2 < g + 8) ? (hi ? hi1 : lo1) : 0.f;
                }
        }
        __syncwarp();
        if (lane < 16) {
            const int bb = wq, cidx = lane;
            const float* nt = dg + dtidx(bb, 0, 0);
            float x[16];
#pragma unroll
            for (int t2 = 0; t2 < 16; ++t2) x[t2] = (t2 == cidx) ? 1.f : 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 15; ++s2) {
                const float xs = x[s2];
#pragma unroll
                for (int t4 = ((s2 + 1) >> 2) << 2; t4 < 16; t4 += 4) {
                    const float4 n4 = *reinterpret_cast<const float4*>(nt + s2 * kDgRow + t4);
                    const float nvv[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (t4 + e > s2) x[t4 + e] = fmaf(nvv[e], xs, x[t4 + e]);
                }
            }
            uint8_t* Tb = smem + gt(G_SP) + kDiagBytes;
#pragma unroll
            for (int t2 = 0; t2 < 16; t2 += 2) {
                const uint32_t hp = pack2h(x[t2], x[t2 + 1]);
                *reinterpret_cast<uint16_t*>(Tb + bb * 768 + t2 * 48 + 2 * cidx) = (uint16_t)(hp & 0xFFFFu);
                *reinterpret_cast<uint16_t*>(Tb + bb * 768 + (t2 + 1) * 48 + 2 * cidx) = (uint16_t)(hp >> 16);
            }
        }
        if (wq > 0) frag_half_to_tile(sbase + gt(G_AB), 16 * wq, 0, 0, v[0], lane, PackH{});
        if (wq > 1) frag_half_to_tile(sbase + gt(G_AB), 16 * wq, 0, 1, v[0], lane, PackH{});
        if (wq > 2) frag_half_to_tile(sbase + gt(G_AB), 16 * wq, 4, 0, v[1], lane, PackH{});
    } else if (warp >= 8 && warp < 12) {
        acc_to_tile(tmem, C0, sbase + gt(G_AAK), wq, 0, lane, 2, PackH{});
        acc_to_tile(tmem, C0, sbase + gt(G_AAK), wq, 1, lane, 2, PackH{});
    } else if (warp >= 12) {
        acc_to_tile(tmem, C2, sbase + gt(G_ARB), wq, 0, lane, 1, PackH{});
        acc_to_tile(tmem, C2, sbase + gt(G_ARB), wq, 1, lane, 1, PackH{});
    }
    // the previous chunk's output stores have read the staging tiles before phase A's
    // epilogue writes them
    if (lane == 0 && warp >= 8 && warp < 13) bulk_wait_read0();
    tc_fence_before();
    if (__syncthreads_or(timed_out)) goto teardown;

    // ---- A: X = Abar S0 + A_ak V;  dU = A_rb^T dO + Bhat dSL;  dA_rk = dO V^T ---------
    if (tid == 0) {
        tc_fence_after();
        mma64(tmem + C0, sbase + gt(G_W), false, sbase + gt(G_S0), true, false, false);
        mma64(tmem + C0, sbase + gt(G_AAK), false, sbase + gt(G_V), true, false, true);
        mma64(tmem + C1, sbase + gt(G_ARB), true, sbase + gt(G_DO), true, false, false);
        mma64(tmem + C1, sbase + gt(G_BH), false, sbase + gt(G_DS), true, false, true);
        mma64(tmem + C2, sbase + gt(G_DO), false, sbase + gt(G_V), false, false, false);
        umma_commit(bar_mma);
        // background (read after later commits): dRbar = dO S0^T, acc_k = V dSL^T,
        // P = Rbar^T dO
        mma64(tmem + C_DRB, sbase + gt(G_DO), false, sbase + gt(G_S0), false, false, false);
        mma64(tmem + C_AK, sbase + gt(G_V), false, sbase + gt(G_DS), false, false, false);
        mma64(tmem + C_P, sbase + gt(G_RB), true, sbase + gt(G_DO), true, false, false);
    }
    // ---- T = (I - A_ab)^-1 by block forward substitution (warp-level fp16 MMAs) on
    //      warps 0..7: warps 0..5 form the six products T_ii A_im (m < i); then warp w
    //      builds columns 8 w .. 8 w + 7 (column block w / 2, MMA n-tile w % 2):
    //      X_b = T_bb, X_i = sum_{b<=m<i} (T_ii A_im) X_m.  Meanwhile warps 8..15 store
    //      phase A's products (issued above; they do not need T). ------------------------
    if (warp < 8) {
        uint8_t* Tb = smem + gt(G_SP) + kDiagBytes;
        uint8_t* Tab = smem + gt(G_DT);
        const int lr = (lane & 7) + 8 * ((lane >> 3) & 1), lc = 8 * (lane >> 4);
        const uint32_t a_lane = lr * 48 + 2 * lc;
        auto a_frag = [&](const uint8_t* blk, uint32_t (&af)[4]) {
            ldsm_x4(smem_u32(blk) + a_lane, af[0], af[1], af[2], af[3]);
        };
        if (warp < 6) {
            const int blk = warp;
            const int i = blk < 1 ? 1 : (blk < 3 ? 2 : 3);
            const int m = blk < 1 ? 0 : (blk < 3 ? blk - 1 : blk - 3);
            uint32_t af[4];
            a_frag(Tb + i * 768, af);
            float z[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            uint32_t bfa[4];
            ldsm_x4_t(sbase + gt(G_AB) + sw(16 * i + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * m + (lane >> 4)),
                      bfa[0], bfa[1], bfa[2], bfa[3]);
            mma_f16_16816(z[0], af[0], af[1], af[2], af[3], bfa[0], bfa[1]);
            mma_f16_16816(z[1], af[0], af[1], af[2], af[3], bfa[2], bfa[3]);
            uint8_t* dst = Tab + blk * 768;  // blocks (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                *reinterpret_cast<uint32_t*>(dst + g * 48 + 2 * (8 * nt + 2 * q)) = pack2h(z[nt][0], z[nt][1]);
                *reinterpret_cast<uint32_t*>(dst + (g + 8) * 48 + 2 * (8 * nt + 2 * q)) = pack2h(z[nt][2], z[nt][3]);
            }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");  // warps 0..7: T_ii A_im visible
        {
            const int cb = warp >> 1, nt = warp & 1;  // column block, n-tile
            uint8_t* tt = smem + gt(G_T);
            uint32_t xb[3][2];  // B fragments of X_0..X_2 in this n-tile
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t top, bot;
                if (i < cb) {
                    top = bot = 0u;
                } else if (i == cb) {
                    top = *reinterpret_cast<const uint32_t*>(Tb + i * 768 + g * 48 + 2 * (8 * nt + 2 * q));
                    bot = *reinterpret_cast<const uint32_t*>(Tb + i * 768 + (g + 8) * 48 + 2 * (8 * nt + 2 * q));
                } else {
                    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < 3; ++m) {
                        if (m < cb || m >= i) continue;
                        const int blk = (i == 1) ? 0 : (i == 2 ? 1 + m : 3 + m);
                        uint32_t af[4];
                        a_frag(Tab + blk * 768, af);
                        mma_f16_16816(y, af[0], af[1], af[2], af[3], xb[m][0], xb[m][1]);
                    }
                    top = pack2h(y[0], y[1]);
                    bot = pack2h(y[2], y[3]);
                }
                const int col = 16 * cb + 8 * nt + 2 * q;
                *reinterpret_cast<uint32_t*>(tt + swe(16 * i + g, col)) = top;
                *reinterpret_cast<uint32_t*>(tt + swe(16 * i + g + 8, col)) = bot;
                if (i < 3) {
                    xb[i][0] = movmatrix_t(top);
                    xb[i][1] = movmatrix_t(bot);
                }
            }
        }
    } else {
        wait_or_abort(bar_mma, mph, timed_out);
        tc_fence_after();
        if (warp < 12) {  // X, and dA_rk's first half
            acc_to_tile(tmem, C0, sbase + gt(G_X), wq, 0, lane, 0, PackH{});
            acc_to_tile(tmem, C0, sbase + gt(G_X), wq, 1, lane, 0, PackH{});
            acc_to_tile(tmem, C2, sbase + gt(G_DARK), wq, 0, lane, 1, PackB{});
        } else {          // dU, and dA_rk's second half
            acc_to_tile(tmem, C1, sbase + gt(G_DU), wq, 0, lane, 0, PackH{});
            acc_to_tile(tmem, C1, sbase + gt(G_DU), wq, 1, lane, 0, PackH{});
            acc_to_tile(tmem, C2, sbase + gt(G_DARK), wq, 1, lane, 1, PackB{});
        }
    }
    mph ^= 1;
    fence_proxy_async();
    tc_fence_before();
    if (__syncthreads_or(timed_out)) goto teardown;

    // ---- B: U = T X;  dX = T^T dU;  dT = dU X^T ------------------------------------
    //      (and the original r, k, a, b again, for dw, into tiles that are dead now:
    //      armed here, issued by warps 4..7 below)
    if (tid == 0) {
        tc_fence_after();
        mbar_arrive_expect_tx(bar_rl, 4 * kTile);
        mma64(tmem + C0, sbase + gt(G_T), false, sbase + gt(G_X), true, false, false);
        mma64(tmem + C1, sbase + gt(G_T), true, sbase + gt(G_DU), true, false, false);
        mma64(tmem + C2, sbase + gt(G_DU), false, sbase + gt(G_X), false, false, false);
        umma_commit(bar_mma);
    }
    wait_or_abort(bar_mma, mph, timed_out);
    mph ^= 1;
    tc_fence_after();
    if (warp >= 4 && warp < 8 && lane == 0) {
        const int i = warp - 4;
        tma_load_3d(sbase + gt(i == 0 ? G_SP : i == 1 ? G_AB : i == 2 ? G_AAK : G_ARB),
                    i == 0 ? &tm_r : i == 1 ? &tm_k : i == 2 ? &tm_a : &tm_b, bar_rl, 0, cy, cz);
    }
    acc16_to_tile(tmem, C0, sbase + gt(G_X), wq, wc, lane, 0, PackH{});   // U
    acc16_to_tile(tmem, C1, sbase + gt(G_DU), wq, wc, lane, 0, PackH{});  // dX
    acc16_to_tile(tmem, C2, sbase + gt(G_DT), wq, wc, lane, 0, PackH{});  // dT
    fence_proxy_async();
    tc_fence_before();
    if (__syncthreads_or(timed_out)) goto teardown;

    // ---- C: dA_rb = dO U^T; dA_ak = dX V^T; Y = dT T^T;
    //      background: dAbar = dX S0^T, acc_b = U dSL^T, P += Abar^T dX
    if (tid == 0) {
        tc_fence_after();
        mma64(tmem + C0, sbase + gt(G_DO), false, sbase + gt(G_X), false, false, false);
        mma64(tmem + C1, sbase + gt(G_DU), false, sbase + gt(G_V), false, false, false);
        mma64(tmem + C2, sbase + gt(G_DT), false, sbase + gt(G_T), false, false, false);
        umma_commit(bar_mma);
        mma64(tmem + C_DAB, sbase + gt(G_DU), false, sbase + gt(G_S0), false, false, false);
        mma64(tmem + C_AB, sbase + gt(G_X), false, sbase + gt(G_DS), false, false, false);
        mma64(tmem + C_P, sbase + gt(G_W), true, sbase + gt(G_DU), true, false, true);
    }
    wait_or_abort(bar_mma, mph, timed_out);
    mph ^= 1;
    tc_fence_after();
    acc16_to_tile(tmem, C0, sbase + gt(G_DARB), wq, wc, lane, 1, PackB{});
    acc16_to_tile(tmem, C1, sbase + gt(G_DAAK), wq, wc, lane, 2, PackB{});
    acc16_to_tile(tmem, C2, sbase + gt(G_DT), wq, wc, lane, 0, PackH{});  // Y
    fence_proxy_async();
    tc_fence_before();
    if (__syncthreads_or(timed_out)) goto teardown;

    // ---- D: dA_ab = T^T Y (the commit also covers P, finished in the background of C);
    //      background: every gradient-accumulator term that does not need dA_ab
    //      (bf16 against the Gram operands)
    if (tid == 0) {
        tc_fence_after();
        mma64(tmem + C0, sbase + gt(G_T), true, sbase + gt(G_DT), true, false, false);
        umma_commit(bar_mma);
        mma64(tmem + C_AR, sbase + gt(G_DARK), false, sbase + gt(G_K), true, true, false);
        mma64(tmem + C_AR, sbase + gt(G_DARB), false, sbase + gt(G_B), true, true, true);
        mma64(tmem + C_AA, sbase + gt(G_DAAK), false, sbase + gt(G_K), true, true, false);
        mma64(tmem + C_AK, sbase + gt(G_DARK), true, sbase + gt(G_R), true, true, true);
        mma64(tmem + C_AK, sbase + gt(G_DAAK), true, sbase + gt(G_A), true, true, true);
        mma64(tmem + C_AB, sbase + gt(G_DARB), true, sbase + gt(G_R), true, true, true);
    }
    if (warp == 4) {  // the next chunk of this CTA: shared, and its load barrier armed
        const int itn = next_item(it + gridDim.x, total, slotsF, T, N, cu, cur, In);
        if (lane == 0) {
            *reinterpret_cast<Item*>(smem + GOFF_NEXT) = In;
            *reinterpret_cast<int*>(smem + GOFF_NEXT + 64) = itn;
            if (itn >= 0) mbar_arrive_expect_tx(bar_tma, 9 * kTile);
        }
    }
    wait_or_abort(bar_mma, mph, timed_out);
    mph ^= 1;
    tc_fence_after();
    acc16_to_tile(tmem, C0, sbase + gt(G_DAAB), wq, wc, lane, 2, PackB{});
    {  // rowsum(S0 * P) over this warp's 16 columns (added to R in the final epilogue)
        float v[8];
        tmem_ld16x16(tmem + ((uint32_t)(32 * wq) << 16) + C_P + 16 * wc, v);
        tmem_ld_wait();
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int row = 16 * wq + g + 8 * hr;
            float part = 0.f;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(
                    smem + gt(G_S0) + swe(row, 16 * wc + 8 * j + 2 * q)));
                part = fmaf(s2.x, v[4 * j + 2 * hr], fmaf(s2.y, v[4 * j + 2 * hr + 1], part));
            }
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (q == 0) Rq[64 * wc + row] = part;
        }
    }
    fence_proxy_async();
    tc_fence_before();
    if (__syncthreads_or(timed_out)) goto teardown;

    // ---- E: the dA_ab terms of acc_a and acc_b ---------------------------------------
    if (tid == 0) {
        tc_fence_after();
        mma64(tmem + C_AA, sbase + gt(G_DAAB), false, sbase + gt(G_B), true, true, true);
        mma64(tmem + C_AB, sbase + gt(G_DAAB), true, sbase + gt(G_A), true, true, true);
        umma_commit(bar_mma);
    }
    wait_or_abort(bar_mma, mph, timed_out);
    mph ^= 1;
    tc_fence_after();
    // Every input tile is dead now: the next chunk's nine loads (one per warp) overlap
    // the final epilogue.
    it = *reinterpret_cast<const volatile int*>(smem + GOFF_NEXT + 64);
    if (it >= 0) {
        I = *reinterpret_cast<const Item*>(smem + GOFF_NEXT);
        if (lane == 0 && warp < 9) load_in(I, warp);
    }
    wait_or_abort(bar_rl, rph, timed_out);
    rph ^= 1;

    // ---- final epilogue: dr, da, dk, db, and dw by an exclusive prefix over tokens;
    //      thread = rows 16 wq + g (+8) x columns 16 wc + 8 j + 2 q (+1), j = 0, 1 ------
    {
        float ar[8], aa[8], ak[8], abv[8], drb[8], dab[8];
        {
            const uint32_t ta = tmem + ((uint32_t)(32 * wq) << 16) + 16 * wc;
            tmem_ld16x16(ta + C_AR, ar);
            tmem_ld16x16(ta + C_AA, aa);
            tmem_ld16x16(ta + C_AK, ak);
            tmem_ld16x16(ta + C_AB, abv);
            tmem_ld16x16(ta + C_DRB, drb);
            tmem_ld16x16(ta + C_DAB, dab);
            tmem_ld_wait();
        }
        // the original r, k, a, b at this thread's fragment positions (ldmatrix of the
        // 16 x 16 block: register 2 j + hr = rows g + 8 hr, columns 8 j + 2 q, +1)
        uint32_t fr_r[4], fr_k[4], fr_a[4], fr_b[4];
        {
            const uint32_t o = sw(16 * wq + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * wc + (lane >> 4));
            ldsm_x4(sbase + gt(G_SP) + o, fr_r[0], fr_r[1], fr_r[2], fr_r[3]);
            ldsm_x4(sbase + gt(G_AB) + o, fr_k[0], fr_k[1], fr_k[2], fr_k[3]);
            ldsm_x4(sbase + gt(G_AAK) + o, fr_a[0], fr_a[1], fr_a[2], fr_a[3]);
            ldsm_x4(sbase + gt(G_ARB) + o, fr_b[0], fr_b[1], fr_b[2], fr_b[3]);
        }
        // a bf16 pair (low half first) as two floats: bf16 is the top half of an fp32
        auto bf2 = [](uint32_t u) { return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u)); };
        float hv[8], fv[8];
        // kPlain: a full chunk without a mask (every row in and valid, known at compile time)
        auto elem = [&](auto plain_c) {
        constexpr bool kPlain = decltype(plain_c)::value;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int t = 16 * wq + g + 8 * hr;
            const bool in = kPlain || t < nv;
            const bool val = kPlain || (in && (!mask || mask[crow + t] != 0));
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int cidx = 16 * wc + 8 * j + 2 * q;
                const float2 E2 = *reinterpret_cast<const float2*>(Ef + eidx(t, cidx));
                const float2 Em = t > 0 ? *reinterpret_cast<const float2*>(Ef + eidx(t - 1, cidx))
                                        : make_float2(em0[cidx], em0[cidx + 1]);
                const int fi = 2 * j + hr;
                const float2 r2 = bf2(fr_r[fi]), k2 = bf2(fr_k[fi]), a2 = bf2(fr_a[fi]),
                             b2 = bf2(fr_b[fi]);
                const float Ee[2] = {E2.x, E2.y}, Eme[2] = {Em.x, Em.y};
                const float re[2] = {r2.x, r2.y}, ke[2] = {k2.x, k2.y}, ae[2] = {a2.x, a2.y},
                            be[2] = {b2.x, b2.y};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int ix = 4 * j + 2 * hr + e;
                    const float gm = gam[cidx + e];
                    const float vdr = in ? fmaf(Ee[e], ar[ix], (Ee[e] * gm) * drb[ix]) : 0.f;
                    const float vdk = val ? __fdividef(ak[ix], Ee[e]) : 0.f;
                    const float vdb = val ? __fdividef(abv[ix], Ee[e]) : 0.f;
                    const float vda = val ? fmaf(Eme[e], aa[ix], (Eme[e] * gm) * dab[ix]) : 0.f;
                    ar[ix] = vdr;
                    ak[ix] = vdk;
                    abv[ix] = vdb;
                    aa[ix] = vda;
                    fv[ix] = ae[e] * vda;
                    hv[ix] = in ? re[e] * vdr - ke[e] * vdk - be[e] * vdb + fv[ix] : 0.f;
                }
            }
        }
        };
        if (nv == 64 && !mask)
            elem(std::true_type{});
        else
            elem(std::false_type{});
        // stage dr, dk, db, da (bf16) in the dA tiles (read by MMA-E, done)
        frag8_to_tile(sbase + gt(G_DARK), 16 * wq, 2 * wc, ar, lane, PackB{});
        frag8_to_tile(sbase + gt(G_DAAK), 16 * wq, 2 * wc, ak, lane, PackB{});
        frag8_to_tile(sbase + gt(G_DARB), 16 * wq, 2 * wc, abv, lane, PackB{});
        frag8_to_tile(sbase + gt(G_DAAB), 16 * wq, 2 * wc, aa, lane, PackB{});
        // exclusive prefix of h over the tokens: rows g (lanes 4 g + q) within the warp,
        // then rows g + 8, then the quadrants before this one
        float ex[8];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i0 = 4 * j + e, i1 = 4 * j + 2 + e;
                float s0v = hv[i0], s1v = hv[i1];
#pragma unroll
                for (int d = 4; d < 32; d *= 2) {
                    const float u0 = __shfl_up_sync(0xffffffffu, s0v, d);
                    const float u1 = __shfl_up_sync(0xffffffffu, s1v, d);
                    if (lane >= d) {
                        s0v += u0;
                        s1v += u1;
                    }
                }
                const float tot0 = __shfl_sync(0xffffffffu, s0v, 28 + q);
                const float tot1 = __shfl_sync(0xffffffffu, s1v, 28 + q);
                ex[i0] = s0v - hv[i0];
                ex[i1] = tot0 + s1v - hv[i1];
                if (g == 0) tot[wq * 64 + 16 * wc + 8 * j + 2 * q + e] = tot0 + tot1;
            }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int cidx = 16 * wc + 8 * j + 2 * q + e;
                float pre = 0.f;
                for (int w2 = 0; w2 < wq; ++w2) pre += tot[w2 * 64 + cidx];
                const float R = Rc[cidx] + Rq[cidx] + Rq[64 + cidx] + Rq[128 + cidx] + Rq[192 + cidx];
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int ix = 4 * j + 2 * hr + e;
                    const int t = 16 * wq + g + 8 * hr;
                    const bool val = t < nv && (!mask || mask[crow + t] != 0);
                    hv[ix] = val ? R - fv[ix] - (pre + ex[ix]) : 0.f;
                }
            }
        frag8_to_tile(sbase + gt(G_X), 16 * wq, 2 * wc, hv, lane, PackB{});  // dw
        fence_proxy_async();
        // The stores leave after the next CTA barrier (the next chunk's first, or the
        // one after the loop), which orders them after every thread's staging writes.
        p_nv = nv;
        p_h = h;
        p_cy = cy;
        p_cz = cz;
        p_crow = crow;
    }

    }  // chunks
    __syncthreads();
    flush();
    if (lane == 0 && warp >= 8 && warp < 13) bulk_wait0();  // the last output stores are complete

teardown:
    if (timed_out) {
        // bounded drains of what may still be in flight, then free the tensor memory
        if (tid == 0) {
            (void)mbar_wait(bar_tma, tph);
            (void)mbar_wait(bar_mma, mph ^ 1u);
            (void)mbar_wait(bar_rl, rph);
        }
        if (lane == 0 && warp >= 8 && warp < 13) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kGTmemCols);
    }
}

// ---------------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------------
template <bool kHf>
inline cudaError_t launch_grad(const void* r, const void* w, const void* k, const void* v,
                               const void* a, const void* b, const void* dout,
                               const uint8_t* mask, void* dr, void* dw, void* dk, void* da,
                               void* db, int B, int T, int H, int N, const int32_t* cu,
                               const int32_t* cur, const void* ckF, const void* ckR,
                               const Ws& lay, cudaStream_t stream) {
    CUtensorMap m[14];
    const void* ins[7] = {r, w, k, v, a, b, dout};
    for (int i = 0; i < 7; ++i)
        if (!make_map(&m[i], ins[i], B, T, H, kHf)) return cudaErrorInvalidValue;
    if (!make_ck_map(&m[7], ckF, (long long)H * lay.slotsF)) return cudaErrorInvalidValue;
    if (!make_ck_map(&m[8], ckR, (long long)H * lay.slotsR)) return cudaErrorInvalidValue;
    void* outs[5] = {dr, dw, dk, da, db};
    for (int i = 0; i < 5; ++i)
        if (!make_map(&m[9 + i], outs[i], B, T, H, kHf)) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidValue;
    constexpr int kMaxDev = 64;  // the dynamic shared-memory size, set once per device
    static bool attr_set[kMaxDev] = {};
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(grad_kernel<kHf>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kGSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const long long items = lay.slotsF * H;
    if (items > 0x7fffffffLL - 4096) return cudaErrorInvalidValue;  // item + grid stays an int
    const unsigned grid = (unsigned)(items < sms ? items : sms);
    grad_kernel<kHf><<<grid, kThreads, kGSmemBytes, stream>>>(
        m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], m[8], m[9], m[10], m[11], m[12], m[13],
        mask, cu, cur, T, H, N, (int)lay.slotsF, (int)lay.slotsR,
        static_cast<__nv_bfloat16*>(dr), static_cast<__nv_bfloat16*>(dw),
        static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(da),
        static_cast<__nv_bfloat16*>(db));
    return cudaGetLastError();
}

}  // namespace cbwd

// A second stream and two events per (host thread, device): the checkpointing forward
// and the reversed run are independent, and run side by side so that each one's last
// partial wave of CTAs overlaps the other.
struct ForkJoin {
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
inline cudaError_t fork_join_for_current_device(ForkJoin*& out) {
    constexpr int kMaxDev = 64;
    thread_local ForkJoin fj[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    ForkJoin& f = fj[dev];
    if (!f.side) {
        if ((e = cudaStreamCreateWithFlags(&f.side, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&f.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&f.join, cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    out = &f;
    return cudaSuccess;
}

inline size_t bwd_chunked_workspace_bytes(long long rows, int N, int H) {
    return cbwd::ws_layout(rows, N, H).total;
}

// The whole chunked backward (bf16, K = V = 64) on `stream`.
inline cudaError_t launch_bwd_chunked(const void* r, const void* w, const void* k, const void* v,
                                      const void* a, const void* b, const float* s0,
                                      const uint8_t* mask, const void* dout, const float* dsT,
                                      void* dr, void* dw, void* dk, void* dv, void* da, void* db,
                                      float* ds0, int B, int T, int H, int N,
                                      const int32_t* cu_seqlens, int head_first, void* workspace,
                                      cudaStream_t stream) {
    using namespace cbwd;
    const long long rows = (long long)B * T;
    const Ws lay = ws_layout(rows, N, H);
    if (lay.slotsF > 0x7fffffffLL || lay.slotsR > 0x7fffffffLL ||
        (long long)H * lay.slotsR > 0x7fffffffLL || lay.rowsR > 0x7fffffffLL)
        return cudaErrorInvalidValue;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* cur = reinterpret_cast<int32_t*>(ws + lay.off_cu);
    void* ckF = ws + lay.off_ckF;
    void* ckR = ws + lay.off_ckR;
    cudaError_t e;
    // 1. reversed sequence offsets
    prep_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, T, N, cur);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 2. forward with per-chunk checkpoints, no outputs, and 3. (below) the reversed run,
    //    side by side: the reversed run goes to a second stream forked after prep
    ForkJoin* fj = nullptr;
    if ((e = fork_join_for_current_device(fj)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(fj->fork, stream)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(fj->side, fj->fork, 0)) != cudaSuccess) return e;
    chunked::Extras exF;
    exF.ck = ckF;
    exF.ck_slots = (int)lay.slotsF;
    if ((e = launch_chunked(r, w, k, v, a, b, s0, mask, nullptr, nullptr, B, T, H, N, cu_seqlens,
                            head_first, -1, stream, exF)) != cudaSuccess)
        return e;
    // 3. the state gradient as a forward run over the reversed sequences, from dsT
    chunked::RevIn rin;
    rin.w = static_cast<const __nv_bfloat16*>(w);
    rin.a = static_cast<const __nv_bfloat16*>(a);
    rin.b = static_cast<const __nv_bfloat16*>(b);
    rin.r = static_cast<const __nv_bfloat16*>(r);
    rin.dout = static_cast<const __nv_bfloat16*>(dout);
    rin.k = static_cast<const __nv_bfloat16*>(k);
    rin.mask = mask;
    rin.cu = cu_seqlens;
    rin.T = T;
    rin.hf = head_first;
    rin.dv = static_cast<__nv_bfloat16*>(dv);
    chunked::Extras exR;
    exR.ck = ckR;
    exR.ck_slots = (int)lay.slotsR;
    if ((e = launch_chunked_rev(rin, B, dsT, ds0, (int)lay.rowsR, H, N, cur, exR, fj->side)) !=
        cudaSuccess)
        return e;
    if ((e = cudaEventRecord(fj->join, fj->side)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(stream, fj->join, 0)) != cudaSuccess) return e;
    // 4. per-chunk gradients
    e = head_first ? launch_grad<true>(r, w, k, v, a, b, dout, mask, dr, dw, dk, da, db, B, T, H,
                                       N, cu_seqlens, cur, ckF, ckR, lay, stream)
                   : launch_grad<false>(r, w, k, v, a, b, dout, mask, dr, dw, dk, da, db, B, T,
                                        H, N, cu_seqlens, cur, ckF, ckR, lay, stream);
    if (e != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace wkv7
