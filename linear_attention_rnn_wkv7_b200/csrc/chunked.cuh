// chunked.cuh -- 64-token chunked WKV7 forward on tcgen05 tensor cores (bf16 in,
// fp32 state), two CTAs resident per SM, each running one (sequence, head) unit or,
// for units of one length, an equal run of the units' chunks (Sched).
//
// The recurrence (rwkv-ops 0.9.0 README, "rwkv7op 使用方法")
//     u_t = S_{t-1}^T a_t;  S_t = diag(exp w_t) S_{t-1} + b_t u_t^T + k_t v_t^T;  o_t = S_t^T r_t
// is rewritten exactly for a chunk of L = 64 tokens (t = 0..63, state S0 at the
// chunk start).  With g_t = sum_{j<=t} w_j (per channel, log space), the chunk's
// last prefix g_L = g_63 as reference and E_t = exp(g_t - g_L) (>= 1):
//   r~ = r E_t, a~ = a E_{t-1}, k~ = k / E_t, b~ = b / E_t        (Gram operands)
//   A_rk[t][s] = r~_t.k~_s (s<=t), A_rb = r~.b~ (s<=t), A_ak = a~.k~ (s<t), A_ab = a~.b~ (s<t)
//   T = (I - A_ab)^-1 (the UT / WY representation of the chunk's rank-1 products)
//   Abar = a e^{g_{t-1}} = a~ e^{g_L}, Rbar = r e^{g_t} = r~ e^{g_L},
//   Bhat = b e^{g_L - g_t} = b~, Khat = k e^{g_L - g_t} = k~
//   W = T Abar, Z = T A_ak,  U = W S0 + Z V   (U: the chunk's read vectors u_t)
//   S_L = diag(e^{g_L}) S0 + Bhat^T U + Khat^T V
//   O   = Rbar S0 + A_rb U + A_rk V
// Only U and what follows depend on S0.  One chunk costs three rounds of tcgen05
// MMAs with fp32 accumulators in tensor memory: the Gram matrices (two commit
// groups), MMA-U (U = [W | Z] [S0; V], M = 64, K = 128), and the final products (the
// state accumulating onto itself scaled by e^{g_L}, and O).  [W | Z] = T [Abar | A_ak]
// comes from a block forward substitution on warp-level MMAs (each warp owns 16 of
// its 128 columns), after the 16x16 diagonal blocks of T by fp32 forward
// substitution.  CUDA cores do the prefix sums and exps and the tensor-memory ->
// shared-memory epilogues that re-layout each result as the next product's operand;
// the M = 64 accumulators are read 16 lanes x 32 columns at a time in the warp-MMA
// fragment layout (all 32 threads busy) and written back with stmatrix.
// Precision: the Gram operands need bf16's exponent range (E_t spans e^{+-40}).  Every
// later operand (the substitution, MMA-U, the final products, the fp16 copies of S0,
// V and U) stays near 1 in magnitude and is fp16, with three more significant bits than
// bf16; that keeps the fp32 final state within 1e-3 of the fp64 recurrence (measured
// over every unit of the B=8, T=4096, H=64 workload: 4.8e-4 of max |S|).
//
// A masked or out-of-range token is folded into the loads as w = 0 and zero a, k, b
// scales: its transition is then the identity and it writes nothing, and its output
// is read from the carried state.  Exps are clamped to [-80, 80] (every operand and
// Gram entry stays finite in fp32 and bf16), so the factorisation is exact while
// g_t - g_L <= 80 inside a chunk (per-step log decay >= -1.26; the RWKV-7
// parametrisation keeps it >= -0.607).
//
// Gated DeltaNet (rwkv-ops 0.9.0 README, "gdn_recurrent 使用方法" / "gdn_chunk
// 使用方法") runs through the same kernel (template flag kGdn): its transition
// e^{g} (I - beta kh kh^T) and write beta kh v^T are the generalized rule with one
// log decay per token on every channel (w_t = g_t), a = kh, b = -e^{g} beta kh and
// write key beta kh, where qh and kh are q and k L2-normalised over K.  Only the
// loads (q, k, v by TMA; g and beta per token) and the prologue differ: the scan is
// over one scalar per token, and the operands are built from qh and kh in registers.
#pragma once
#include <cuda.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "sm100.cuh"

namespace wkv7 {

constexpr bool kChunkedBuilt = true;

namespace chunked {

constexpr int kThreads = 256;
constexpr int kMinCtasPerSm = 2;  // registers (128 per thread) and shared memory allow two
constexpr int kStoreTid = 64;  // issues the output tile stores (an output warp's lane 0)
// Shared-memory map.  Fourteen 8 KB tiles (64 rows x 128 B, 1024-aligned, 128B
// swizzle) plus a small control block.  Consecutive chunks alternate between two
// layouts of the same tiles: the next chunk's six input tiles are exactly the tiles
// this chunk no longer needs once its MMA-U has read W and Z, so their TMA loads
// overlap this chunk's last epilogue and final products.
constexpr uint32_t kTile = 8192;
constexpr uint32_t OFF_S0 = 12 * kTile;    // S0 fp16 [k][v] (MMA-U and O's B operand), then
                                           // the output staging; both layouts
constexpr uint32_t OFF_MISC = 14 * kTile;  // mbarriers, TMEM address, unit index
constexpr uint32_t OFF_GAMMA = OFF_MISC + 64;  // e^{g_L}, channel c at cswz(c) (64 fp32)
constexpr uint32_t kSmemBytes = OFF_GAMMA + 256;

// Tile roles of one chunk (byte offsets):
//   R     raw r -> r~ (B of A_rk^T / A_rb^T) -> A_ab's blocks left of the diagonal
//   A     raw a -> a~ (A of the Gram) -> U fp16 [t][v] (B of the final products)
//   K, B  raw k, b -> k~, b~ (B of the Gram, and together [k~; b~] the A of A_rk^T /
//         A_rb^T); K then holds T_ii A_im during [W|Z]
//   W     raw w -> Bhat fp16 [s][k] (A of S's U block, MN-major)
//   V     raw v -> fp16 in place [s][v] (B of the V blocks)
//   KHAT  Khat fp16 [s][k] (A of S's V block)     RBAR  Rbar fp16 [t][k] (A of O's S0 block)
//   ARKT  A_rk^T fp16 [s][t], ARBT A_rb^T fp16 [s][t] (A of O's V and U blocks)
//   ABAR  Abar fp16 [t][k] -> W [t][k];  AAK  A_ak [t][s] -> Z [t][s]  (A of MMA-U)
//   SP    prologue scratch, then A_ab's fp32 diagonal blocks and T_ii (epilogue 1 -> [W|Z])
struct LayR {
    uint32_t R, A, K, B, W, V, KHAT, ARKT, ARBT, RBAR, ABAR, AAK, SP;
};
// Even chunks (tiles 0..13, 12 is S0) and odd chunks: each layout's inputs
// {R, A, K, B, W, V} are the other's {R, K, B, ABAR, AAK, SP}, all dead once that
// chunk's MMA-U is done; K and B are adjacent in both ([k~; b~] is one 128-row operand).
__device__ __forceinline__ LayR lay_of(int par) {
    return par ? LayR{0 * kTile, 13 * kTile, 2 * kTile, 3 * kTile, 10 * kTile, 11 * kTile,
                      6 * kTile, 7 * kTile,  8 * kTile, 9 * kTile, 1 * kTile,  4 * kTile,
                      5 * kTile}
               : LayR{0 * kTile, 1 * kTile,  2 * kTile, 3 * kTile, 4 * kTile,  5 * kTile,
                      6 * kTile, 7 * kTile,  8 * kTile, 9 * kTile, 10 * kTile, 11 * kTile,
                      13 * kTile};
}
// Prologue scratch in the SP tile, in floats.
constexpr int SCR_TOT = 0, SCR_C = 512, SCR_PRE = 576;  // floats (SCR_PRE: 8 x 64)
// Tensor-memory columns.  An M = 64 accumulator holds row m in lane (m % 16) +
// 32 (m / 16): lanes 0..15 of each 32-lane quadrant; M = 128 uses all 128 lanes.
constexpr uint32_t TM_D1 = 0;    // [A_ak | A_ab] = a~ [k~; b~]^T, M = 64 (128 cols); then U
constexpr uint32_t TM_DU = 0;    // U = [W | Z] [S0; V], M = 64 (64 cols)
constexpr uint32_t TM_D1B = 128; // [A_rk^T; A_rb^T] = [k~; b~] r~^T, M = 128 (64 cols); then O
constexpr uint32_t TM_DFO = 128; // O, M = 64 (64 cols)
constexpr uint32_t TM_DFS = 192; // the fp32 state S, M = 64 (64 cols), for the whole sequence
constexpr uint32_t kTmemCols = 256;
constexpr float kExpClamp = 80.f;

// Byte offset of 16-byte chunk `c` of row `row` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw(uint32_t row, uint32_t c) {
    return row * 128u + ((c ^ (row & 7u)) << 4);
}
// Byte offset of bf16 element (row, col) in a 128B-swizzled 64-column tile.
__device__ __forceinline__ uint32_t swe(uint32_t row, uint32_t col) {
    return sw(row, col >> 3) + ((col & 7u) << 1);
}

// Float index of element (row t, column s) of diagonal 16x16 block bb of A_ab, kept in
// fp32 and stored transposed (s-major rows of 16 floats padded to 20, so that the
// fragment-layout writes of rows s = 2q + e, q = 0..3, fall in four different 8-bank
// groups).  They and the fp16 inverses T_bb (48-byte rows) live in the SP tile, free
// once the prologue is done.
constexpr int kDgRow = 20;
__device__ __forceinline__ int dtidx(int bb, int s, int t) {
    return bb * 16 * kDgRow + s * kDgRow + t;
}
constexpr uint32_t kDiagBytes = 4 * 16 * kDgRow * 4;  // the four fp32 diagonal blocks, then T_bb
static_assert(kDiagBytes + 4 * 768 <= kTile, "diagonal blocks and T_bb fit one tile");

// Position of channel c in a 64-float per-channel row (prologue scratch, e^{g_L},
// Khat rows): the two 16-byte halves of each 32-byte group swap places in the upper
// half of the row, so that lanes j and j + 4 of a thread's eight 32-byte strided
// float4 accesses land in different banks.
__device__ __forceinline__ int cswz(int c) { return c ^ ((c & 32) >> 3); }

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
}
// fp16 pairs, rounded to nearest and saturated at +-65504 (never inf).  fp16 keeps
// three more significant bits than bf16; it carries the operands of the [W | Z]
// substitution and of MMA-3, whose magnitudes stay near 1.
__device__ __forceinline__ uint32_t pack2h(float a, float b) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}
__device__ __forceinline__ uint4 pack8h(const float* v) {
    return make_uint4(pack2h(v[0], v[1]), pack2h(v[2], v[3]), pack2h(v[4], v[5]), pack2h(v[6], v[7]));
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
// 2^x by the hardware approximation (relative error about 2^-22, subnormal results
// flushed to zero); the prologue keeps
// log decays in log2 units so that every exponential is one such instruction.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kClamp2 = kExpClamp * kLog2e;  // the exponent clamp in log2 units
__device__ __forceinline__ float clamp2(float x) { return fminf(fmaxf(x, -kClamp2), kClamp2); }

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

// Store 32 fp32 columns [col, col + 32) of this warp's lanes.
__device__ __forceinline__ void tmem_row_st32(uint32_t tmem, int wq, uint32_t col, const float* v) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float tmp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) tmp[j] = v[16 * i + j];
        sm100::tmem_st16(tmem + ((uint32_t)(32 * wq) << 16) + col + 16 * i, tmp);
    }
}

// Warp-level D += A * B, m16n8k16, fp16 operands, fp32 accumulate.  Fragment
// ownership (g = lane / 4, q = lane % 4): A (g|g+8, 2q..2q+1 | 2q+8..2q+9),
// B (k = 2q..2q+1 | 2q+8..2q+9, n = g), C/D (g|g+8, 2q|2q+1).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Four 8x8 b16 matrices; lane l gives the address of row (l % 8) of matrix l / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// Four 8x8 b16 matrices from warp-MMA fragment registers (lane l: row l / 4, columns
// 2 (l % 4), +1 of each) to shared memory; lane l gives the address of row l % 8 of
// matrix l / 8 (16 bytes per row).
__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2,
                                        uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// Half h (columns 16h .. 16h + 15) of a 16-row x 32-column block held in fragment
// layout (sm100::tmem_ld16x32) to a 128B-swizzled tile: rows row0 .. row0 + 15, 16-byte
// chunks chunk0 + 2h, +1; each element pair packed by `pk` (fp16 or bf16).  One
// stmatrix.x4, whose matrices are (chunk 2h, rows +0), (2h, +8), (2h + 1, +0), (2h + 1, +8).
template <typename Pack>
__device__ __forceinline__ void frag_half_to_tile(uint32_t tile, int row0, int chunk0, int h,
                                                  const float (&v)[16], int lane, Pack pk) {
    const int mi = lane >> 3;  // the matrix this lane addresses
    const uint32_t addr = tile + sw(row0 + 8 * (mi & 1) + (lane & 7), chunk0 + 2 * h + (mi >> 1));
    stsm_x4(addr, pk(v[8 * h + 0], v[8 * h + 1]), pk(v[8 * h + 2], v[8 * h + 3]),
            pk(v[8 * h + 4], v[8 * h + 5]), pk(v[8 * h + 6], v[8 * h + 7]));
}
template <typename Pack>
__device__ __forceinline__ void frag_to_tile(uint32_t tile, int row0, int chunk0, const float (&v)[16],
                                             int lane, Pack pk) {
    frag_half_to_tile(tile, row0, chunk0, 0, v, lane, pk);
    frag_half_to_tile(tile, row0, chunk0, 1, v, lane, pk);
}
struct PackH {
    __device__ __forceinline__ uint32_t operator()(float a, float b) const { return pack2h(a, b); }
};
struct PackB {
    __device__ __forceinline__ uint32_t operator()(float a, float b) const { return pack2(a, b); }
};

// The 16 rows of an M = 64 accumulator that warp quadrant wq owns (rows 16 wq .. 16 wq + 15,
// lanes 0..15 of the quadrant), columns col .. col + 31, in fragment layout.
__device__ __forceinline__ void tmem_frag(uint32_t tmem, int wq, uint32_t col, float (&v)[16]) {
    sm100::tmem_ld16x32(tmem + ((uint32_t)(32 * wq) << 16) + col, v);
    sm100::tmem_ld_wait();
}

// Transpose of an 8x8 b16 matrix held one 32-bit pair per lane (lane l: row l / 4,
// columns 2 (l % 4), +1), returned in the same layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}


// Bounded wait on an mbarrier phase.  A thread that gives up raises the timeout flag
// and records it in `timed_out`; it then carries on to the next CTA barrier, where
// __syncthreads_or makes the decision to abandon the sequence the same for every
// thread (no thread leaves while others wait at a barrier).
__device__ __forceinline__ void wait_or_abort(uint32_t bar, uint32_t parity, int& timed_out) {
    if (!sm100::mbar_wait(bar, parity)) {
        raise_flag(4 /* WKV7_ERR_DEVICE_TIMEOUT */);
        timed_out = 1;
    }
}

// The reversed run (kRev) of the backward's state gradient reads the original tensors
// itself: reversed sequence n is p = 63 - L % 64 identity steps, then step tau = 0..L with
// transition w, b, a of token L - tau (tau >= 1; identity for a masked token) and write
// pair r, dO of token L - 1 - tau (tau < L); its read vector is k of token L - 1 - tau,
// so the outputs are dv of that token (zero for a masked token), written in place.
struct RevIn {
    const __nv_bfloat16 *w, *a, *b, *r, *dout, *k;  // original tensors
    const uint8_t* mask;                             // [B, T] or nullptr
    const int32_t* cu;                               // original cu_seqlens or nullptr
    int T, hf;                                       // original T and layout
    __nv_bfloat16* dv;                               // dv, the original layout
};

// Everything one CTA keeps for its (sequence, head) between chunks.
struct Ctx {
    uint8_t* smem;
    uint32_t sbase, tmem, bar_tma, bar_mma, mma_phase;
    uint32_t bar_g2, g2_phase;  // the Gram's second commit group (see the Gram issue)
    int tid, warp, lane, wq, wh;
    long long row0;  // token row of the sequence start in the [B*T] token space (mask)
    int len;
    const uint8_t* mask;
    __nv_bfloat16* o;  // this unit's first output row; rows o_ts elements apart
    long long o_ts;
    long long gb0;     // Gated DeltaNet: index of the first token's g / beta; gbs apart
    int gbs;
    int tma_y, tma_z;  // tile coordinates of the sequence start (dims 1 and 2 of the maps)
    int timed_out;     // this thread gave up on a wait (agreed on at the next CTA barrier)
    uint32_t tma_par_last;  // parity of the last input load issued (drained on abort)
    // Test hook of the timeout path: thread `stall_tid` of CTA 0 waits, with a short
    // limit, on an mbarrier nothing arrives at (after chunk 0's inputs have landed, with
    // no copy or MMA in flight).  -1 (every normal launch): off.
    int stall_tid;
    uint32_t bar_never;
    float* gamma_s;
    const CUtensorMap *tm_r, *tm_w, *tm_k, *tm_v, *tm_a, *tm_b, *tm_o;
    // State checkpoints (the backward's): when `ck` is set, each chunk's fp16 starting
    // state (the S0 operand tile) is stored to checkpoint slice ck_z0 + chunk index.
    const CUtensorMap* tm_ck;
    bool ck;
    int ck_z0;
    // kRev: the original sequence (length, padding, first token's element offset and
    // token stride in the inputs, row in the mask, and its dv tile coordinates)
    const RevIn* ri;
    int rv_L, rv_p, rv_y0, rv_z0;
    long long rv_base, rv_ts, rv_row0;
    const __nv_bfloat16 *g, *beta;  // Gated DeltaNet only: [rows, H]
};

// Lanes 0..5 of the calling warp: request the six 64 x 64 bf16 input tiles of the chunk
// starting at token c0 into layout `par` (lane 0 arms the barrier first; the
// six copies are issued in parallel).  Gated DeltaNet loads three (q, k, v into the
// r, k, v tiles).
template <bool kGdn, bool kHf>
__device__ __forceinline__ void issue_loads(const Ctx& cx, int c0, int par) {
    const LayR L = lay_of(par);
    using namespace sm100;
    const int lane = cx.lane;
    if (lane == 0) mbar_arrive_expect_tx(cx.bar_tma, (kGdn ? 3 : 6) * kTile);
    __syncwarp();
    // token-major maps are (channel, head, token row); head-first maps (channel, token,
    // batch x head): the chunk start advances dimension 2 or dimension 1
    const int cy = kHf ? cx.tma_y + c0 : cx.tma_y;
    const int cz = kHf ? cx.tma_z : cx.tma_z + c0;
    if constexpr (kGdn) {
        if (lane < 3) {
            const CUtensorMap* map = lane == 0 ? cx.tm_r : lane == 1 ? cx.tm_k : cx.tm_v;
            const uint32_t dst = lane == 0 ? L.R : lane == 1 ? L.K : L.V;
            tma_load_3d(cx.sbase + dst, map, cx.bar_tma, 0, cy, cz);
        }
    } else if (lane < 6) {
        const CUtensorMap* map = lane == 0 ? cx.tm_r : lane == 1 ? cx.tm_a : lane == 2 ? cx.tm_k
                               : lane == 3 ? cx.tm_b : lane == 4 ? cx.tm_w : cx.tm_v;
        const uint32_t dst = lane == 0 ? L.R : lane == 1 ? L.A : lane == 2 ? L.K
                           : lane == 3 ? L.B : lane == 4 ? L.W : L.V;
        tma_load_3d(cx.sbase + dst, map, cx.bar_tma, 0, cy, cz);
    }
}

// Input tile i (0..5: r, a, k, b, w, v; Gated DeltaNet 0..2: q, k, v) of the chunk at
// token c0 into layout `par`, by the calling thread (the barrier is armed elsewhere).
// Each TMA instruction takes a few hundred cycles to issue, so a chunk's loads come
// from one thread of each of several warps.
template <bool kGdn, bool kHf>
__device__ __forceinline__ void issue_load_one(const Ctx& cx, int c0, int par, int i) {
    const LayR L = lay_of(par);
    const int cy = kHf ? cx.tma_y + c0 : cx.tma_y;
    const int cz = kHf ? cx.tma_z : cx.tma_z + c0;
    const CUtensorMap* map;
    uint32_t dst;
    if constexpr (kGdn) {
        map = i == 0 ? cx.tm_r : i == 1 ? cx.tm_k : cx.tm_v;
        dst = i == 0 ? L.R : i == 1 ? L.K : L.V;
    } else {
        map = i == 0 ? cx.tm_r : i == 1 ? cx.tm_a : i == 2 ? cx.tm_k : i == 3 ? cx.tm_b
            : i == 4 ? cx.tm_w : cx.tm_v;
        dst = i == 0 ? L.R : i == 1 ? L.A : i == 2 ? L.K : i == 3 ? L.B : i == 4 ? L.W : L.V;
    }
    sm100::tma_load_3d(cx.sbase + dst, map, cx.bar_tma, 0, cy, cz);
}

// kRev, every thread: 12 of the chunk's 6 x 64 x 8 16-byte pieces by cp.async, each
// from its original token (zero-filled where the step has no transition or no write),
// then the mbarrier tracks this thread's copies (one plain arrive after the next CTA
// barrier completes the count).
__device__ __forceinline__ void issue_loads_rev(const Ctx& cx, int c0, int par) {
    const LayR L = lay_of(par);
    const RevIn& ri = *cx.ri;
    const int cc = cx.tid & 7;
#pragma unroll
    for (int half = 0; half < 2; ++half) {  // rows j and j + 32, 16-byte piece cc of each
        const int j = (cx.tid >> 3) + 32 * half;
        const int tau = c0 + j - cx.rv_p;
        const int t1 = cx.rv_L - tau, t2 = t1 - 1;  // transition token, write-pair token
        const bool ok1 = tau >= 1 && tau <= cx.rv_L && (!ri.mask || ri.mask[cx.rv_row0 + t1] != 0);
        const bool ok2 = tau >= 0 && tau < cx.rv_L;
        const long long o1 = ok1 ? cx.rv_base + (long long)t1 * cx.rv_ts + 8 * cc : 0;
        const long long o2 = ok2 ? cx.rv_base + (long long)t2 * cx.rv_ts + 8 * cc : 0;
        const uint32_t n1 = ok1 ? 16u : 0u, n2 = ok2 ? 16u : 0u, d = cx.sbase + sw(j, cc);
        // w', a', b' = w, b, a of token t1;  k', v', r' = r, dO, k of token t2
        sm100::cp_async_16(d + L.W, ri.w + o1, n1);
        sm100::cp_async_16(d + L.A, ri.b + o1, n1);
        sm100::cp_async_16(d + L.B, ri.a + o1, n1);
        sm100::cp_async_16(d + L.K, ri.r + o2, n2);
        sm100::cp_async_16(d + L.V, ri.dout + o2, n2);
        sm100::cp_async_16(d + L.R, ri.k + o2, n2);
    }
    sm100::cp_async_mbar_arrive(cx.bar_tma);
}

// Work of one CTA.  When every unit (sequence, head) has the same length, the units'
// chunks, laid end to end unit by unit, are cut into equal runs of `cmax` >= C chunks
// (C per unit), one run per CTA, with no more CTAs than fit on the GPU at once
// (McNaughton's wrap-around rule for preemptive scheduling on identical machines).  A
// unit cut between CTAs m and m + 1 still runs in order: m + 1 takes the unit's first
// chunks at the start of its run, m the unit's last chunks at the end of its run, and
// the fp32 state passes between them through handoff slot m.  Because cmax >= C, the
// later part starts (no earlier than cmax minus its length) after the earlier part has
// ended (no later than C minus the later part's length), so the wait is normally nil;
// it is bounded all the same.  Otherwise (packed sequences of different lengths) each
// CTA runs one unit.
struct Sched {
    int Lu;              // the common unit length in tokens; 0: one unit per CTA
    long long cmax;      // chunks per CTA
    float* ho_state;     // [slots][64][64] fp32 handoff states
    unsigned* ho_flag;   // [slots]: equals `epoch` once the slot's state is written
    unsigned epoch;      // this launch's (nonzero) flag value
};

// Bounded wait (one second of device time) until *f == want, with acquire ordering.
__device__ __forceinline__ bool wait_flag(const unsigned* f, unsigned want) {
    const uint64_t t0 = sm100::globaltimer_ns();
    for (uint32_t i = 0; i < (1u << 30); ++i) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        if (v == want) return true;
        __nanosleep(128);
        if ((i & 15u) == 15u && sm100::globaltimer_ns() - t0 > 1000000000ull) return false;
    }
    return false;
}
__device__ __forceinline__ void st_release(unsigned* f, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}

// One 64-token chunk starting at token c0, in layout P (its inputs already requested).
// Returns false, the same in every thread, when a bounded wait ran out: the caller then
// abandons the sequence.
template <bool kGdn, bool kHf, bool kRev>
__device__ __forceinline__ bool chunk(Ctx& cx, int c0, bool has_next, int par) {
    const LayR L = lay_of(par);
    using namespace sm100;
    uint8_t* smem = cx.smem;
    const uint32_t sbase = cx.sbase, tmem = cx.tmem, bar_mma = cx.bar_mma;
    const int tid = cx.tid, warp = cx.warp, lane = cx.lane, wq = cx.wq, wh = cx.wh;
    const long long row0 = cx.row0;
    const uint8_t* mask = cx.mask;
    __nv_bfloat16* o = cx.o;
    // a state-only run (no outputs): the work that only feeds O is skipped
    const bool so = !kRev && o == nullptr;
    float* gamma_s = cx.gamma_s;
    uint32_t& mma_phase = cx.mma_phase;
    float* scratch = reinterpret_cast<float*>(smem + L.SP);  // prologue only
    const int nv = min(64, cx.len - c0);
    // The previous chunk's output store has read the S0 tile before this chunk's
    // epilogue 3 writes it (ordered by the barriers in between).
    if (tid == kStoreTid) sm100::bulk_wait_read0();
    float gq[2] = {0.f, 0.f}, bq[2] = {0.f, 0.f};  // Gated DeltaNet: g, beta of tokens t0, t0+1
    if constexpr (kGdn) {  // issued before the tile wait, so their latency overlaps it
        const int t0 = 2 * (tid >> 3);
        const long long gbs = kHf ? 1 : cx.gbs;
        const long long tok = cx.gb0 + (long long)(c0 + t0) * gbs;
        if (t0 < nv) {
            gq[0] = __bfloat162float(cx.g[tok]);
            bq[0] = __bfloat162float(cx.beta[tok]);
        }
        if (t0 + 1 < nv) {
            gq[1] = __bfloat162float(cx.g[tok + gbs]);
            bq[1] = __bfloat162float(cx.beta[tok + gbs]);
        }
    }
    wait_or_abort(cx.bar_tma, par, cx.timed_out);
    if (c0 == 0 && tid == cx.stall_tid && !sm100::mbar_wait_short(cx.bar_never, 0)) {
        raise_flag(4 /* WKV7_ERR_DEVICE_TIMEOUT */);
        cx.timed_out = 1;
    }

        // ---- 2. prefix sums of w (mask folded) and every scaled operand, in one pass.
        //         Thread (q, j) owns tokens 2q, 2q+1 and channels 8j..8j+7: a shuffle
        //         scan over the warp's four token pairs, warp totals exchanged through
        //         shared memory, each warp's exclusive prefix and the per-channel
        //         constants from warp 0, then E_t and the operands, written in
        //         place. ----------------------------------------------------------------
        {
            const int j = tid & 7, t0 = 2 * (tid >> 3);
            const bool va = t0 < nv && (!mask || mask[row0 + c0 + t0] != 0);
            const bool vb = t0 + 1 < nv && (!mask || mask[row0 + c0 + t0 + 1] != 0);
            const uint32_t offa = sw(t0, j), offb = sw(t0 + 1, j);
            const int h0 = cswz(8 * j), h1 = cswz(8 * j + 4);  // this thread's channel halves
            float rts[2][8], ats[2][8], ec[8];  // fp32 r~ and a~, kept for Rbar and Abar; e^{g_L}
            // The token's operands to shared memory: r~, a~, k~ (bf16), b~ (bf16 and fp16
            // as Bhat), Khat (fp16).
            auto put = [&](int it, const float* kt, const float* btl) {
                const uint32_t off = it ? offb : offa;
                *reinterpret_cast<uint4*>(smem + L.R + off) = pack8(rts[it]);
                *reinterpret_cast<uint4*>(smem + L.A + off) = pack8(ats[it]);
                const uint4 kq = pack8(kt);
                *reinterpret_cast<uint4*>(smem + L.K + off) = kq;
                *reinterpret_cast<uint4*>(smem + L.B + off) = pack8(btl);
                *reinterpret_cast<uint4*>(smem + L.W + off) = pack8h(btl);  // Bhat (fp16)
                *reinterpret_cast<uint4*>(smem + L.KHAT + off) = pack8h(kt);  // Khat (fp16)
            };
            if constexpr (kGdn) {
                // Gated DeltaNet: one log decay per token, so the scan runs on one value per
                // token pair; qh, kh from the tiles with norms reduced over the pair's 8 lanes.
                const float wa = va ? gq[0] * kLog2e : 0.f, wb = vb ? gq[1] * kLog2e : 0.f;
                float incl = wa + wb;
#pragma unroll
                for (int d = 8; d < 32; d *= 2) {
                    const float up = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += up;
                }
                if (lane == 24) scratch[SCR_TOT + warp] = incl;  // the warp's 8-token sum
                float qv[2][8], kv[2][8], nq[2], nk[2];
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const uint32_t off = it ? offb : offa;
                    unpack8(*reinterpret_cast<const uint4*>(smem + L.R + off), qv[it]);
                    unpack8(*reinterpret_cast<const uint4*>(smem + L.K + off), kv[it]);
                    float sq = 0.f, sk = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        sq = fmaf(qv[it][e], qv[it][e], sq);
                        sk = fmaf(kv[it][e], kv[it][e], sk);
                    }
#pragma unroll
                    for (int m = 1; m < 8; m *= 2) {
                        sq += __shfl_xor_sync(0xffffffffu, sq, m);
                        sk += __shfl_xor_sync(0xffffffffu, sk, m);
                    }
                    nq[it] = sq > 0.f ? rsqrtf(sq) : 0.f;  // a zero vector stays zero
                    nk[it] = sk > 0.f ? rsqrtf(sk) : 0.f;
                }
                if (__syncthreads_or(cx.timed_out)) return false;  // a wait ran out: stop
                float pre = 0.f, gL = 0.f;  // earlier warps' sum; g_L (log2 units)
#pragma unroll
                for (int w2 = 0; w2 < 8; ++w2) {
                    const float x = scratch[SCR_TOT + w2];
                    pre += (w2 < warp) ? x : 0.f;
                    gL += x;
                }
                const float eg = ex2(gL);
                if (tid < 64) gamma_s[tid] = eg;
#pragma unroll
                for (int e = 0; e < 8; ++e) ec[e] = eg;
                const float ga = pre + (incl - wb);  // g at token t0
                float Ep = ex2(clamp2(ga - wa - gL));   // E_{t0-1}
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const bool val = it ? vb : va;
                    const float d = clamp2((it ? ga + wb : ga) - gL);
                    const float E = ex2(d);
                    const float inv = val ? ex2(-d) : 0.f;  // a masked token writes nothing
                    const float ep = val ? Ep : 0.f;
                    const float bw = bq[it] * inv;                   // beta / E
                    const float bb = -ex2(it ? wb : wa) * bw;       // -e^{g} beta / E
                    const float rq = nq[it] * E, ak = nk[it] * ep;
                    float kt[8], btl[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float kn = kv[it][e] * nk[it];
                        rts[it][e] = qv[it][e] * rq;
                        ats[it][e] = kv[it][e] * ak;
                        kt[e] = kn * bw;
                        btl[e] = kn * bb;
                    }
                    Ep = E;
                    put(it, kt, btl);
                }
            } else {
                float wa[8], wb[8], incl[8];
                {  // a masked token's w is zero (cleared on the packed words)
                    const uint32_t ma = va ? 0xFFFFFFFFu : 0u, mb = vb ? 0xFFFFFFFFu : 0u;
                    uint4 qa = *reinterpret_cast<const uint4*>(smem + L.W + offa);
                    uint4 qb = *reinterpret_cast<const uint4*>(smem + L.W + offb);
                    qa.x &= ma; qa.y &= ma; qa.z &= ma; qa.w &= ma;
                    qb.x &= mb; qb.y &= mb; qb.z &= mb; qb.w &= mb;
                    unpack8(qa, wa);
                    unpack8(qb, wb);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {  // log decays in log2 units from here on
                    wa[e] *= kLog2e;
                    wb[e] *= kLog2e;
                    incl[e] = wa[e] + wb[e];
                }
#pragma unroll
                for (int d = 8; d < 32; d *= 2) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float up = __shfl_up_sync(0xffffffffu, incl[e], d);
                        if (lane >= d) incl[e] += up;
                    }
                }
                float* wt = scratch + SCR_TOT;  // [warp][channel] sums of w over the warp's 8 tokens
                if (lane >= 24) {
                    *reinterpret_cast<float4*>(wt + warp * 64 + h0) =
                        make_float4(incl[0], incl[1], incl[2], incl[3]);
                    *reinterpret_cast<float4*>(wt + warp * 64 + h1) =
                        make_float4(incl[4], incl[5], incl[6], incl[7]);
                }
                if (__syncthreads_or(cx.timed_out)) return false;  // a wait ran out: stop
                if (warp == 0) {  // per channel: exclusive prefixes over the warps, c = g_L, e^{g_L}
                    const int ch = cswz(2 * lane);  // channels 2 lane, 2 lane + 1
                    float2 gL = make_float2(0.f, 0.f);
#pragma unroll
                    for (int w2 = 0; w2 < 8; ++w2) {
                        const float2 x = *reinterpret_cast<const float2*>(wt + w2 * 64 + ch);
                        *reinterpret_cast<float2*>(scratch + SCR_PRE + w2 * 64 + ch) = gL;
                        gL.x += x.x; gL.y += x.y;
                    }
                    *reinterpret_cast<float2*>(scratch + SCR_C + ch) = gL;
                    *reinterpret_cast<float2*>(gamma_s + ch) = make_float2(ex2(gL.x), ex2(gL.y));
                }
                __syncthreads();  // per-channel constants ready
                float ga[8];  // g at token t0: earlier warps + this warp's pairs up to t0
                {
                    const float4 x0 = *reinterpret_cast<const float4*>(scratch + SCR_PRE + warp * 64 + h0);
                    const float4 x1 = *reinterpret_cast<const float4*>(scratch + SCR_PRE + warp * 64 + h1);
                    const float pre[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) ga[e] = pre[e] + (incl[e] - wb[e]);
                }
                float cc[8];  // c = g_L (log2 units)
                *reinterpret_cast<float4*>(cc) = *reinterpret_cast<const float4*>(scratch + SCR_C + h0);
                *reinterpret_cast<float4*>(cc + 4) = *reinterpret_cast<const float4*>(scratch + SCR_C + h1);
                *reinterpret_cast<float4*>(ec) = *reinterpret_cast<const float4*>(gamma_s + h0);
                *reinterpret_cast<float4*>(ec + 4) = *reinterpret_cast<const float4*>(gamma_s + h1);
                float Ep[8];  // E at token t0 - 1 (g_{t0-1} = g_{t0} - w_{t0})
#pragma unroll
                for (int e = 0; e < 8; ++e) Ep[e] = ex2(clamp2(ga[e] - wa[e] - cc[e]));
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const uint32_t off = it ? offb : offa;
                    const bool val = it ? vb : va;
                    float rv[8], av[8], kv[8], bv[8];
                    unpack8(*reinterpret_cast<const uint4*>(smem + L.R + off), rv);
                    unpack8(*reinterpret_cast<const uint4*>(smem + L.A + off), av);
                    unpack8(*reinterpret_cast<const uint4*>(smem + L.K + off), kv);
                    unpack8(*reinterpret_cast<const uint4*>(smem + L.B + off), bv);
                    float kt[8], btl[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float g = it ? ga[e] + wb[e] : ga[e];
                        const float d = clamp2(g - cc[e]);
                        const float E = ex2(d);  // e^{g_t - g_L}
                        // A masked token writes nothing: its a, k, b scales are zero.
                        const float inv = val ? ex2(-d) : 0.f;
                        const float ep = val ? Ep[e] : 0.f;
                        rts[it][e] = rv[e] * E;
                        ats[it][e] = av[e] * ep;
                        kt[e] = kv[e] * inv;   // = Khat (fp32)
                        btl[e] = bv[e] * inv;  // = Bhat
                        Ep[e] = E;  // E_{t-1} of the next token
                    }
                    put(it, kt, btl);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();

            // Gram on the tensor cores, in two commit groups: first A_ab = a~ b~^T (M = 64),
            // so that the warps holding it start on its diagonal inverses while the second
            // group runs: A_ak = a~ k~^T (M = 64) and [A_rk^T; A_rb^T] = [k~; b~] r~^T
            // (M = 128), the transposes the output product takes as MN-major operands.
            if (tid == 0) {
                tc_fence_after();
                // the next chunk's input barrier, armed now (its loads are issued after
                // MMA-U, several CTA barriers later)
                if (!kRev && has_next) mbar_arrive_expect_tx(cx.bar_tma, (kGdn ? 3 : 6) * kTile);
                constexpr uint32_t id64 = idesc_bf16(64, 64, false, false);
                constexpr uint32_t id128 = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_D1 + 64, smem_desc(sbase + L.A + 32 * kk, 16, 1024),
                              smem_desc(sbase + L.B + 32 * kk, 16, 1024), id64, kk > 0);
                umma_commit(bar_mma);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_D1, smem_desc(sbase + L.A + 32 * kk, 16, 1024),
                              smem_desc(sbase + L.K + 32 * kk, 16, 1024), id64, kk > 0);
                if (!so) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + TM_D1B, smem_desc(sbase + L.K + 32 * kk, 16, 1024),
                                  smem_desc(sbase + L.R + 32 * kk, 16, 1024), id128, kk > 0);
                }
                umma_commit(cx.bar_g2);
            }
            // While it runs: Abar = a~ e^{g_L} and Rbar = r~ e^{g_L} (fp16), V to fp16 in
            // place (tiles the Gram does not read).
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const uint32_t off = it ? offb : offa;
                float abar[8], rbar[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    abar[e] = ats[it][e] * ec[e];
                    rbar[e] = rts[it][e] * ec[e];
                }
                *reinterpret_cast<uint4*>(smem + L.ABAR + off) = pack8h(abar);
                if (!so) *reinterpret_cast<uint4*>(smem + L.RBAR + off) = pack8h(rbar);
                float vf[8];
                unpack8(*reinterpret_cast<const uint4*>(smem + L.V + off), vf);
                *reinterpret_cast<uint4*>(smem + L.V + off) = pack8h(vf);
            }
            // And the state this chunk starts from (rows k = 16 wq + lane of the M = 64
            // accumulator, lanes 0..15): its fp16 copy, the B operand of MMA-U and of O's S0
            // block, and the state itself scaled by e^{g_L} in tensor memory, where the
            // final product S_L += Bhat^T U + Khat^T V accumulates onto it.
            {
                float sv[16];
                tmem_frag(tmem + TM_DFS, wq, 32 * wh, sv);
                frag_to_tile(sbase + OFF_S0, 16 * wq, 4 * wh, sv, lane, PackH{});
                const float g0 = gamma_s[cswz(16 * wq + (lane >> 2))];
                const float g1 = gamma_s[cswz(16 * wq + (lane >> 2) + 8)];
#pragma unroll
                for (int j2 = 0; j2 < 4; ++j2) {
                    sv[4 * j2 + 0] *= g0;
                    sv[4 * j2 + 1] *= g0;
                    sv[4 * j2 + 2] *= g1;
                    sv[4 * j2 + 3] *= g1;
                }
                sm100::tmem_st16x32(tmem + TM_DFS + ((uint32_t)(32 * wq) << 16) + 32 * wh, sv);
                tmem_st_wait();
            }
        }

        // ---- 4. Gram waits: the warps holding A_ab need only the first group ------------
        const bool ab_warp = wh == 1;
        wait_or_abort(ab_warp ? bar_mma : cx.bar_g2, ab_warp ? mma_phase : cx.g2_phase,
                      cx.timed_out);
        tc_fence_after();

        // ---- 5. epilogue 1.  M = 64 rows t = 16 wq + lane (lanes 0..15) of [A_ak | A_ab]:
        //         warps 4..7 hold A_ab's block row wq, write its diagonal block (fp32,
        //         transposed) and invert it at once, then, once the second group has read
        //         r~, store the blocks left of it (fp16) over r~; warps 0..3 store masked
        //         A_ak and all of [A_rk^T; A_rb^T] (M = 128, rows s = 32 wq + lane),
        //         masked s <= t, as fp16 [s][t]. ------------------------------------------
        {
            const int g = lane >> 2, q = lane & 3;
            const int t0 = 16 * wq + g;  // fragment rows t0 and t0 + 8 of a~
            if (ab_warp) {
                float v[2][16];  // A_ab columns 0..31, 32..63
                tmem_frag(tmem + TM_D1 + 64, wq, 0, v[0]);
                tmem_frag(tmem + TM_D1 + 64, wq, 32, v[1]);
                float* dg = reinterpret_cast<float*>(smem + L.SP);
                {   // the diagonal block (columns 16 wq ..), transposed, strictly lower
                    const bool hi = wq >= 2, odd = wq & 1;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int s2 = 8 * jj + 2 * q + e;  // column within the block
                            const int i0 = 4 * jj + e, i1 = 4 * (2 + jj) + e;
                            const float lo0 = odd ? v[0][i1] : v[0][i0], hi0 = odd ? v[1][i1] : v[1][i0];
                            const float lo1 = odd ? v[0][i1 + 2] : v[0][i0 + 2];
                            const float hi1 = odd ? v[1][i1 + 2] : v[1][i0 + 2];
                            dg[dtidx(wq, s2, g)] = (s2 < g) ? (hi ? hi0 : lo0) : 0.f;
                            dg[dtidx(wq, s2, g + 8)] = (s2 < g + 8) ? (hi ? hi1 : lo1) : 0.f;
                        }
                }
                // T_bb = (I - N_bb)^-1 with N_bb strictly lower, for this warp's block:
                // lane c < 16 solves (I - N) x = e_c column-wise; once x[s] is final it is
                // added into every later x[t], so the dependent chain is one FMA per row.
                // T_bb goes out as fp16.
                __syncwarp();
                if (lane < 16) {
                    const int bb = wq, c = lane;
                    const float* nt = dg + dtidx(bb, 0, 0);
                    float x[16];
#pragma unroll
                    for (int t2 = 0; t2 < 16; ++t2) x[t2] = (t2 == c) ? 1.f : 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < 15; ++s2) {
                        const float xs = x[s2];
#pragma unroll
                        for (int t4 = ((s2 + 1) >> 2) << 2; t4 < 16; t4 += 4) {
                            const float4 n4 = *reinterpret_cast<const float4*>(nt + s2 * kDgRow + t4);
                            const float nv[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if (t4 + e > s2) x[t4 + e] = fmaf(nv[e], xs, x[t4 + e]);
                        }
                    }
                    uint8_t* Tb = smem + L.SP + kDiagBytes;  // fp16 16x16 blocks, 48-byte rows
#pragma unroll
                    for (int t2 = 0; t2 < 16; t2 += 2) {  // column c: rows t2 and t2 + 1
                        const uint32_t hp = pack2h(x[t2], x[t2 + 1]);
                        *reinterpret_cast<uint16_t*>(Tb + bb * 768 + t2 * 48 + 2 * c) = (uint16_t)(hp & 0xFFFFu);
                        *reinterpret_cast<uint16_t*>(Tb + bb * 768 + (t2 + 1) * 48 + 2 * c) = (uint16_t)(hp >> 16);
                    }
                }
                wait_or_abort(cx.bar_g2, cx.g2_phase, cx.timed_out);  // r~ has been read
                tc_fence_after();
                // A_ab[t][s] over r~: the 16-column blocks left of the diagonal
                if (wq > 0) frag_half_to_tile(sbase + L.R, 16 * wq, 0, 0, v[0], lane, PackH{});
                if (wq > 1) frag_half_to_tile(sbase + L.R, 16 * wq, 0, 1, v[0], lane, PackH{});
                if (wq > 2) frag_half_to_tile(sbase + L.R, 16 * wq, 4, 0, v[1], lane, PackH{});
            } else {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {  // A_ak[t][s], kept for s < t
                    float v[16];
                    tmem_frag(tmem + TM_D1, wq, 32 * h2, v);
#pragma unroll
                    for (int j2 = 0; j2 < 4; ++j2)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int s2 = 32 * h2 + 8 * j2 + 2 * q + e;
                            if (s2 >= t0) v[4 * j2 + e] = 0.f;
                            if (s2 >= t0 + 8) v[4 * j2 + 2 + e] = 0.f;
                        }
                    frag_to_tile(sbase + L.AAK, 16 * wq, 4 * h2, v, lane, PackH{});
                }
                // row s of A_rk^T (wq 0, 1) or A_rb^T (wq 2, 3): A_x[t][s] = v[t], kept s <= t
                const int s_ = 32 * (wq & 1) + lane;
                const uint32_t dst = wq < 2 ? L.ARKT : L.ARBT;
#pragma unroll
                for (int h2 = 0; h2 < (so ? 0 : 2); ++h2) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        float tmp[16];
                        tmem_ld16(tmem + ((uint32_t)(32 * wq) << 16) + TM_D1B + 32 * h2 + 16 * i, tmp);
#pragma unroll
                        for (int j2 = 0; j2 < 16; ++j2) v[16 * i + j2] = tmp[j2];
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            x[e] = (s_ <= 32 * h2 + 8 * c + e) ? v[8 * c + e] : 0.f;
                        *reinterpret_cast<uint4*>(smem + dst + sw(s_, 4 * h2 + c)) = pack8h(x);
                    }
                }
            }
            mma_phase ^= 1;
            cx.g2_phase ^= 1;
            fence_proxy_async();
            tc_fence_before();
            if (__syncthreads_or(cx.timed_out)) return false;
            // The chunk's fp16 starting state (written in the Gram window) to its
            // checkpoint slice; the tile is next overwritten by epilogue 4's staging, and
            // the same thread waits for this store's reads before that (epilogue U).
            if (cx.ck && tid == kStoreTid) {
                tma_store_3d(cx.tm_ck, sbase + OFF_S0, 0, 0, cx.ck_z0 + (c0 >> 6));
                bulk_commit();
            }
        }

        // ---- 6. [W | Z] = T [Abar | A_ak], T = (I - A_ab)^-1, by block forward
        //         substitution over four 16-row blocks:
        //             X_i = T_ii RHS_i + sum_{m<i} (T_ii A_im) X_m.
        //         The 16x16 diagonal inverses T_ii come from fp32 forward substitution;
        //         the products T_ii A_im and T_ii RHS_i are independent and run in
        //         parallel on warp-level fp16 MMAs (fp32 accumulate); then each warp
        //         finishes its own 16 of the 128 right-hand-side columns, writing X in
        //         place over the right-hand side (fp16), where MMA-3 reads it as its
        //         MN-major B operand. ------------------------------------------------
        {
            // fp16 16x16 blocks with rows of 48 bytes: T_ii (4, from epilogue 1) and
            // T_ii A_im (6, in the dead k~ tile).
            uint8_t* Tb = smem + L.SP + kDiagBytes;
            uint8_t* Tab = smem + L.K;
            const int g = lane >> 2, q = lane & 3;
            uint8_t* xt = smem + (warp < 4 ? L.ABAR : L.AAK);  // tile of this warp's columns
            const int nb = 2 * (warp & 3);                     // first 16-byte chunk of them
            const uint32_t xs = smem_u32(xt);
            // ldmatrix row addresses of this lane: A blocks (48-byte rows) and the
            // transposed B fragments of rows kb..kb+15 of this warp's 16 columns.
            const int lr = (lane & 7) + 8 * ((lane >> 3) & 1), lc = 8 * (lane >> 4);
            const uint32_t a_lane = lr * 48 + 2 * lc;
            auto b_addr = [&](int kb) -> uint32_t {
                const int row = kb + (lane & 7) + 8 * ((lane >> 3) & 1);
                return xs + sw(row, nb + (lane >> 4));
            };
            auto a_frag = [&](const uint8_t* blk, uint32_t (&af)[4]) {
                ldsm_x4(smem_u32(blk) + a_lane, af[0], af[1], af[2], af[3]);
            };
            // (a) warps 0..5: T_ii A_im, one block each, stored bf16.
            if (warp < 6) {
                const int i = warp < 1 ? 1 : (warp < 3 ? 2 : 3);
                const int m = warp < 1 ? 0 : (warp < 3 ? warp - 1 : warp - 3);
                uint32_t af[4];
                a_frag(Tb + i * 768, af);
                float z[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                uint32_t bfa[4];  // B = A_im (fp16 rows 16i.., columns 16m..), transposed fragments
                ldsm_x4_t(smem_u32(smem + L.R) +
                              sw(16 * i + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * m + (lane >> 4)),
                          bfa[0], bfa[1], bfa[2], bfa[3]);
                mma_f16_16816(z[0], af[0], af[1], af[2], af[3], bfa[0], bfa[1]);
                mma_f16_16816(z[1], af[0], af[1], af[2], af[3], bfa[2], bfa[3]);
                uint8_t* dst = Tab + warp * 768;  // blocks (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    *reinterpret_cast<uint32_t*>(dst + g * 48 + 2 * (8 * nt + 2 * q)) = pack2h(z[nt][0], z[nt][1]);
                    *reinterpret_cast<uint32_t*>(dst + (g + 8) * 48 + 2 * (8 * nt + 2 * q)) = pack2h(z[nt][2], z[nt][3]);
                }
            }
            // (b) every warp, its 16 columns: Y_i = T_ii RHS_i for the four block rows.
            float y[4][2][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) y[i][nt][e] = 0.f;
                uint32_t af[4], bf[4];
                a_frag(Tb + i * 768, af);
                ldsm_x4_t(b_addr(16 * i), bf[0], bf[1], bf[2], bf[3]);
                mma_f16_16816(y[i][0], af[0], af[1], af[2], af[3], bf[0], bf[1]);
                mma_f16_16816(y[i][1], af[0], af[1], af[2], af[3], bf[2], bf[3]);
            }
            __syncthreads();  // T_ii A_im visible; every warp has read its right-hand side
            // (c) X_i = Y_i + sum_{m<i} (T_ii A_im) X_m, written in place over the right-hand
            //     side in bf16 for MMA-3.  Later block rows take X_m as their B operand
            //     straight from registers: the bf16 C fragments, transposed 8x8 at a time.
            uint32_t xb[3][4];  // B fragments of X_0..X_2 (n-tile 0: b0 b1, n-tile 1: b0 b1)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int m = 0; m < i; ++m) {
                    const int blk = (i == 1) ? 0 : (i == 2 ? 1 + m : 3 + m);
                    uint32_t af[4];
                    a_frag(Tab + blk * 768, af);
                    mma_f16_16816(y[i][0], af[0], af[1], af[2], af[3], xb[m][0], xb[m][1]);
                    mma_f16_16816(y[i][1], af[0], af[1], af[2], af[3], xb[m][2], xb[m][3]);
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int col = 8 * (nb + nt) + 2 * q;
                    const uint32_t top = pack2h(y[i][nt][0], y[i][nt][1]);
                    const uint32_t bot = pack2h(y[i][nt][2], y[i][nt][3]);
                    *reinterpret_cast<uint32_t*>(xt + swe(16 * i + g, col)) = top;
                    *reinterpret_cast<uint32_t*>(xt + swe(16 * i + g + 8, col)) = bot;
                    if (i < 3) {
                        xb[i][2 * nt] = movmatrix_t(top);
                        xb[i][2 * nt + 1] = movmatrix_t(bot);
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
        }

        // ---- 7. MMA-U: U = [W | Z] [S0; V], the chunk's read vectors u_t = S_{t-1}^T a_t
        //         (M = 64, K = 128, fp16). ---------------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idu = idesc_f16(64, 64, false, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_DU, smem_desc(sbase + L.ABAR + 32 * kk, 16, 1024),
                          smem_desc(sbase + OFF_S0 + 2048 * kk, 8192, 1024), idu, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_DU, smem_desc(sbase + L.AAK + 32 * kk, 16, 1024),
                          smem_desc(sbase + L.V + 2048 * kk, 8192, 1024), idu, 1u);
            umma_commit(bar_mma);
        }
        wait_or_abort(bar_mma, mma_phase, cx.timed_out);
        mma_phase ^= 1;
        tc_fence_after();

        // W and Z have been read: every tile the next chunk loads into is dead now.
        if (has_next) {
            if constexpr (kRev)
                issue_loads_rev(cx, c0 + 64, par ^ 1);
            else if (lane == 0 && warp >= 1 && warp <= (kGdn ? 3 : 6))
                issue_load_one<kGdn, kHf>(cx, c0 + 64, par ^ 1, warp - 1);
            cx.tma_par_last = par ^ 1;
        }

        // ---- 8. epilogue U: U (rows t = 16 wq + lane, lanes 0..15) to fp16 [t][v] over a~,
        //         the B operand of both final products. -------------------------------------
        {
            float v[16];
            tmem_frag(tmem + TM_DU, wq, 32 * wh, v);
            frag_to_tile(sbase + L.A, 16 * wq, 4 * wh, v, lane, PackH{});
            if (cx.ck && tid == kStoreTid) sm100::bulk_wait_read0();  // the S0 tile is read
            fence_proxy_async();
            tc_fence_before();
            if (__syncthreads_or(cx.timed_out)) return false;
            // every thread's copies are tracked by now: complete the arrival count
            if (kRev && has_next && tid == 0) sm100::mbar_arrive(cx.bar_tma);
        }

        // ---- 9. the final products (M = 64, fp16):
        //         S_L += Bhat^T U + Khat^T V   (onto the state scaled by e^{g_L})
        //         O    = A_rb U + A_rk V + Rbar S0 ------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idmm = idesc_f16(64, 64, true, true);   // A and B MN-major
            constexpr uint32_t idkm = idesc_f16(64, 64, false, true);  // A K-major
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_DFS, smem_desc(sbase + L.W + 2048 * kk, 8192, 1024),
                          smem_desc(sbase + L.A + 2048 * kk, 8192, 1024), idmm, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_DFS, smem_desc(sbase + L.KHAT + 2048 * kk, 8192, 1024),
                          smem_desc(sbase + L.V + 2048 * kk, 8192, 1024), idmm, 1u);
            if (!so) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_DFO, smem_desc(sbase + L.ARBT + 2048 * kk, 8192, 1024),
                              smem_desc(sbase + L.A + 2048 * kk, 8192, 1024), idmm, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_DFO, smem_desc(sbase + L.ARKT + 2048 * kk, 8192, 1024),
                              smem_desc(sbase + L.V + 2048 * kk, 8192, 1024), idmm, 1u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_DFO, smem_desc(sbase + L.RBAR + 32 * kk, 16, 1024),
                              smem_desc(sbase + OFF_S0 + 2048 * kk, 8192, 1024), idkm, 1u);
            }
            umma_commit(bar_mma);
        }
        wait_or_abort(bar_mma, mma_phase, cx.timed_out);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- 10. epilogue 4: the chunk's outputs (rows t = 16 wq + lane of O); the new fp32
        //          state stays in tensor memory. ---------------------------------------------
        if constexpr (kRev) {
            // row j is dv of original token tb - j (zero for a masked one); rows staged
            // reversed, so the tile is tokens tb - 63 .. tb in order
            float v[16];
            tmem_frag(tmem + TM_DFO, wq, 32 * wh, v);
            const RevIn& ri = *cx.ri;
            const int tb = cx.rv_L - 1 - (c0 - cx.rv_p);
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int t = tb - (16 * wq + (lane >> 2) + 8 * hr);
                const bool keep = t >= 0 && t < cx.rv_L && (!ri.mask || ri.mask[cx.rv_row0 + t] != 0);
                if (!keep) {
#pragma unroll
                    for (int j2 = 0; j2 < 4; ++j2) v[4 * j2 + 2 * hr] = v[4 * j2 + 2 * hr + 1] = 0.f;
                }
            }
            {
                const int mi = lane >> 3;
                const int row = 16 * wq + 8 * (mi & 1) + (lane & 7);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    stsm_x4(sbase + OFF_S0 + sw(63 - row, 4 * wh + 2 * hh + (mi >> 1)),
                            pack2(v[8 * hh + 0], v[8 * hh + 1]), pack2(v[8 * hh + 2], v[8 * hh + 3]),
                            pack2(v[8 * hh + 4], v[8 * hh + 5]), pack2(v[8 * hh + 6], v[8 * hh + 7]));
            }
            fence_proxy_async();
            __syncthreads();
            const int t0s = tb - 63;  // token of staging row 0
            if (t0s >= 0 && t0s + 63 < cx.rv_L) {
                if (tid == kStoreTid) {
                    tma_store_3d(cx.tm_o, sbase + OFF_S0, 0, ri.hf ? cx.rv_y0 + t0s : cx.rv_y0,
                                 ri.hf ? cx.rv_z0 : cx.rv_z0 + t0s);
                    bulk_commit();
                }
            } else {
                for (int i = tid; i < 512; i += kThreads) {
                    const int r = i >> 3, cc = i & 7, t = t0s + r;
                    if (t >= 0 && t < cx.rv_L)
                        *reinterpret_cast<uint4*>(ri.dv + cx.rv_base + (long long)t * cx.rv_ts + 8 * cc) =
                            *reinterpret_cast<const uint4*>(smem + OFF_S0 + sw(r, cc));
                }
            }
        } else if (o != nullptr) {  // (no outputs: a state-only run)
            float v[16];
            tmem_frag(tmem + TM_DFO, wq, 32 * wh, v);
            if (nv == 64) {
                // A full chunk: the bf16 rows are staged in the (now dead) S0 tile in the
                // inputs' swizzled layout and leave as one TMA tile store, so each output
                // row is written by whole lines instead of 16-byte pieces of many rows.
                frag_to_tile(sbase + OFF_S0, 16 * wq, 4 * wh, v, lane, PackB{});
                fence_proxy_async();
                __syncthreads();
                if (tid == kStoreTid) {
                    const int cy = kHf ? cx.tma_y + c0 : cx.tma_y;
                    const int cz = kHf ? cx.tma_z : cx.tma_z + c0;
                    tma_store_3d(cx.tm_o, sbase + OFF_S0, 0, cy, cz);
                    bulk_commit();
                }
            } else {  // a partial last chunk: the sequence's own rows, element pairs
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int t = 16 * wq + (lane >> 2) + 8 * hr;
                    if (t < nv) {
                        uint32_t* dst = reinterpret_cast<uint32_t*>(
                            o + (c0 + t) * (kHf ? 64 : cx.o_ts) + 32 * wh + 2 * (lane & 3));
#pragma unroll
                        for (int j2 = 0; j2 < 4; ++j2)
                            dst[4 * j2] = pack2(v[4 * j2 + 2 * hr], v[4 * j2 + 2 * hr + 1]);
                    }
                }
            }
        }
        // No barrier: the next chunk reads and writes nothing this epilogue touches before
        // its own first barrier (its prologue waits for the output store's reads).
        tc_fence_before();
        return true;
}

// Piece k of CTA blockIdx.x's run under the balanced schedule (Sched): unit (n, h),
// its chunks [cb, ce), and the handoff slots its first and final states come from and
// go to (-1: s0 and sT).  False past the run's end.
struct Piece {
    int n, h, cb, ce, in_slot, out_slot;
};
__device__ __forceinline__ bool piece_of(int k, const Sched& sc, int N, int H, Piece& pc) {
    const long long C = (sc.Lu + 63) / 64;
    const long long p0 = (long long)blockIdx.x * sc.cmax;
    const long long pe = min(p0 + sc.cmax, (long long)N * H * C);
    const long long u = p0 / C + k;  // piece 0 starts at p0, piece k > 0 at unit u's start
    const long long p = k == 0 ? p0 : u * C;
    if (p >= pe) return false;
    const long long uend = (u + 1) * C;
    pc.n = (int)(u / H);
    pc.h = (int)(u - (long long)pc.n * H);
    pc.cb = 0;
    pc.ce = (int)C;
    pc.in_slot = pc.out_slot = -1;
    if (p != u * C) {  // list part [p, uend): the unit's first uend - p chunks
        pc.ce = (int)(uend - p);
        pc.out_slot = blockIdx.x - 1;
    } else if (uend > pe) {  // list part [p, pe): the unit's last pe - p chunks
        pc.cb = (int)(C - (pe - p));
        pc.in_slot = blockIdx.x;
    }
    return true;
}

// The per-unit fields of cx for unit (sequence n, head h): the sequence's token rows,
// output, gate and checkpoint offsets, its TMA coordinates and, for kRev, the original
// sequence.  Packed offsets are valid here (checked by the caller or built by the
// backward's preparation kernel).
template <bool kHf, bool kRev>
__device__ __forceinline__ void set_unit(Ctx& cx, int n, int h, int T, int H,
                                         const int32_t* cu_seqlens, __nv_bfloat16* o,
                                         int ck_slots, const RevIn& rin) {
    int bb = n, bos = 0, eos = T;
    if (cu_seqlens) {
        bb = 0;
        bos = cu_seqlens[n];
        eos = cu_seqlens[n + 1];
    }
    cx.row0 = (long long)bb * T + bos;
    cx.len = eos - bos;
    if (kHf) {
        const long long u0 = ((long long)bb * H + h) * T + bos;  // [B, H, T] token index
        cx.o = o ? o + u0 * 64 : nullptr;
        cx.o_ts = 64;
        cx.gb0 = u0;
        cx.gbs = 1;
        cx.tma_y = bos;
        cx.tma_z = bb * H + h;
    } else {
        cx.o = o ? o + (cx.row0 * H + h) * 64 : nullptr;
        cx.o_ts = (long long)H * 64;
        cx.gb0 = cx.row0 * H + h;
        cx.gbs = H;
        cx.tma_y = h;
        cx.tma_z = (int)cx.row0;
    }
    if constexpr (kRev) {
        int bb_o = n, bos_o = 0, L_o = rin.T;
        if (rin.cu) {
            bb_o = 0;
            bos_o = rin.cu[n];
            L_o = rin.cu[n + 1] - bos_o;
            if (bos_o < 0 || L_o < 0 || bos_o + L_o > rin.T) bos_o = L_o = 0;  // flagged by prep
        }
        cx.rv_L = L_o;
        cx.rv_p = 63 - (L_o & 63);
        cx.rv_row0 = (long long)bb_o * rin.T + bos_o;
        if (rin.hf) {
            cx.rv_base = (((long long)bb_o * H + h) * rin.T + bos_o) * 64;
            cx.rv_ts = 64;
            cx.rv_y0 = bos_o;
            cx.rv_z0 = bb_o * H + h;
        } else {
            cx.rv_base = (cx.rv_row0 * H + h) * 64;
            cx.rv_ts = (long long)H * 64;
            cx.rv_y0 = h;
            cx.rv_z0 = (int)cx.rv_row0;
        }
    }
    cx.ck_z0 = h * ck_slots + (int)(cx.row0 >> 6) + n;  // slot: floor(row0 / 64) + n + chunk
}

// kGdn: Gated DeltaNet (tm_r, tm_k, tm_v map q, k, v; g and beta per token; s0 may be
// one state per head shared by every sequence, s0_shared != 0).  kHf (head first):
// inputs, o (and g, beta) are [B, H, T, *] instead of [B, T, H, *]; the maps follow.
template <bool kGdn, bool kHf, bool kRev>
__global__ void __launch_bounds__(kThreads, kMinCtasPerSm)
chunked_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ CUtensorMap tm_ck,
               const float* s0, const uint8_t* __restrict__ mask, __nv_bfloat16* __restrict__ o,
               float* sT, int T, int H, int N, const int32_t* __restrict__ cu_seqlens,
               const __nv_bfloat16* __restrict__ g, const __nv_bfloat16* __restrict__ beta,
               int s0_shared, int stall_tid, int ck_slots, const __grid_constant__ RevIn rin,
               const __grid_constant__ Sched sc) {
    extern __shared__ __align__(1024) uint8_t smem[];
    using namespace sm100;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;  // TMEM lane quarter, column half
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
        if (tid == 0) raise_flag(3 /* WKV7_ERR_CUDA */);
        return;
    }
    const bool bal = sc.Lu > 0;
    int n = blockIdx.x / H;
    if (!bal && cu_seqlens && N <= kThreads) {
        // Packed sequences are taken longest first (ties by index): blocks start in
        // index order, so the long sequences do not end up in the last wave.  Each CTA
        // ranks the lengths itself, in a tile that is free until the first chunk.
        int* lens = reinterpret_cast<int*>(smem + 9 * kTile);
        int* pick = lens + kThreads;
        if (tid < N) lens[tid] = cu_seqlens[tid + 1] - cu_seqlens[tid];
        __syncthreads();
        if (tid < N) {
            const int mine = lens[tid];
            int rank = 0;
            for (int j = 0; j < N; ++j) {
                const int lj = lens[j];
                rank += (lj > mine) || (lj == mine && j < tid);
            }
            if (rank == n) *pick = tid;
        }
        __syncthreads();
        n = *pick;
        __syncthreads();  // the tile is reused later
    }
    if (!bal && cu_seqlens) {
        const int bos = cu_seqlens[n], eos = cu_seqlens[n + 1];
        if (bos < 0 || eos < bos || eos > T) {
            if (tid == 0) raise_flag(5 /* WKV7_ERR_DEVICE_BAD_SEQLENS */);
            return;
        }
    }

    Ctx cx;
    cx.smem = smem;
    cx.sbase = sbase;
    cx.bar_tma = sbase + OFF_MISC;
    cx.bar_mma = sbase + OFF_MISC + 8;
    cx.bar_g2 = sbase + OFF_MISC + 32;
    cx.g2_phase = 0;
    cx.mma_phase = 0;
    cx.tid = tid;
    cx.warp = warp;
    cx.lane = lane;
    cx.wq = wq;
    cx.wh = wh;
    cx.mask = mask;
    cx.timed_out = 0;
    cx.tma_par_last = 0;
    cx.stall_tid = blockIdx.x == 0 ? stall_tid : -1;
    cx.bar_never = sbase + OFF_MISC + 24;
    cx.gamma_s = reinterpret_cast<float*>(smem + OFF_GAMMA);
    cx.tm_r = &tm_r;
    cx.tm_w = &tm_w;
    cx.tm_k = &tm_k;
    cx.tm_v = &tm_v;
    cx.tm_a = &tm_a;
    cx.tm_b = &tm_b;
    cx.tm_o = &tm_o;
    cx.tm_ck = &tm_ck;
    cx.ri = &rin;
    cx.ck = ck_slots > 0;
    cx.g = g;
    cx.beta = beta;

    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC + 16);
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        *reinterpret_cast<int*>(smem + OFF_MISC + 40) = n;  // the unit of a one-unit CTA
        mbar_init(cx.bar_tma, 1);
        mbar_init(cx.bar_mma, 1);
        mbar_init(cx.bar_g2, 1);
        mbar_init(cx.bar_never, 1);  // nothing ever arrives (the timeout test hook)
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cx.tmem = *tmem_slot;
    if (warp == 0 && lane < 7)
        prefetch_tensormap(lane == 0 ? &tm_r : lane == 1 ? &tm_a : lane == 2 ? &tm_k
                           : lane == 3 ? &tm_b : lane == 4 ? &tm_w : lane == 5 ? &tm_v : &tm_o);

    // The fp32 state lives in tensor memory as an M = 64 accumulator: row k in lane
    // (k % 16) + 32 (k / 16), so lanes 0..15 of warp w hold rows 16 (w % 4) + lane,
    // columns [32 (w / 4), 32 (w / 4) + 32).  The other lanes of those columns stay unused.
    const int srow = 16 * wq + lane;  // state row of this thread (lanes 0..15)

    // This CTA's pieces, in time order (see Sched): with the balanced schedule, piece k
    // of its run of the unit-major chunk list (recomputed where needed, so that nothing
    // of it stays live across the chunks); otherwise the one unit n, h.
    bool ok = true;
    int par = 0;  // layout of the next chunk (chunks alternate between the two)
    for (int piece = 0; ok; ++piece) {
        Piece pc;
        if (bal) {
            if (!piece_of(piece, sc, N, H, pc)) break;
        } else {
            if (piece > 0) break;
            pc = Piece{*reinterpret_cast<const int*>(smem + OFF_MISC + 40), (int)(blockIdx.x % H),
                       0, INT_MAX, -1, -1};
        }
        const int cb = pc.cb, ce = pc.ce, in_slot = pc.in_slot, h = pc.h;
        set_unit<kHf, kRev>(cx, pc.n, h, T, H, cu_seqlens, o, ck_slots, rin);
        const int tb = 64 * cb;
        const int te = ce == INT_MAX ? cx.len : min(cx.len, 64 * ce);

        // the piece's first loads (they do not depend on the state)
        if (tb < te) {
            if constexpr (kRev) {
                issue_loads_rev(cx, tb, par);
                __syncthreads();  // every thread's copies are tracked: complete the count
                if (tid == 0) mbar_arrive(cx.bar_tma);
            } else if (warp == 0) {
                issue_loads<kGdn, kHf>(cx, tb, par);
            }
            cx.tma_par_last = par;
        }

        // the starting state: s0 (or zeros) at a unit's start, else the handoff slot
        {
            const float* src = nullptr;
            if (in_slot >= 0) {
                int late = 0;
                if (tid == 0 && !wait_flag(sc.ho_flag + in_slot, sc.epoch)) {
                    raise_flag(4 /* WKV7_ERR_DEVICE_TIMEOUT */);
                    late = 1;
                }
                if (__syncthreads_or(late)) {
                    ok = false;
                    break;
                }
                src = sc.ho_state + (size_t)in_slot * 4096;
            } else if (s0 && cb == 0) {
                src = s0 + (s0_shared ? (size_t)h : (size_t)pc.n * H + h) * 4096;
            }
            float sv[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] = 0.f;
            if (src && lane < 16) {
                const float4* s4 = reinterpret_cast<const float4*>(src + srow * 64 + 32 * wh);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 f = in_slot >= 0 ? __ldcg(s4 + j) : s4[j];
                    sv[4 * j] = f.x;
                    sv[4 * j + 1] = f.y;
                    sv[4 * j + 2] = f.z;
                    sv[4 * j + 3] = f.w;
                }
            }
            tmem_row_st32(cx.tmem + TM_DFS, wq, 32 * wh, sv);
            tmem_st_wait();
            if (in_slot >= 0) {  // consumed: clear the flag for the next launch
                __syncthreads();
                if (tid == 0) *reinterpret_cast<volatile unsigned*>(sc.ho_flag + in_slot) = 0u;
            }
        }
        tc_fence_before();

        for (int c0 = tb; c0 < te && ok; c0 += 64, par ^= 1)
            ok = chunk<kGdn, kHf, kRev>(cx, c0, c0 + 64 < te, par);
        // The last chunk's final-MMA wait is agreed on here (it has no barrier of its own).
        if (ok && __syncthreads_or(cx.timed_out)) ok = false;
        tc_fence_after();
        if (!ok) break;

        // the final state: to sT at a unit's end, else to the handoff slot
        int out_slot = -1, un, uh;
        if (bal) {
            (void)piece_of(piece, sc, N, H, pc);
            out_slot = pc.out_slot;
            un = pc.n;
            uh = pc.h;
        } else {
            un = *reinterpret_cast<const int*>(smem + OFF_MISC + 40);
            uh = (int)(blockIdx.x % H);
        }
        const size_t state_off = ((size_t)un * H + uh) * 4096;
        float* dst = out_slot >= 0 ? sc.ho_state + (size_t)out_slot * 4096
                                   : (sT ? sT + state_off : nullptr);
        if (dst) {
            float sv[32];
            tmem_row<2>(cx.tmem + TM_DFS, wq, 32 * wh, sv);
            if (lane < 16) {
                float4* d4 = reinterpret_cast<float4*>(dst + srow * 64 + 32 * wh);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    d4[j] = make_float4(sv[4 * j], sv[4 * j + 1], sv[4 * j + 2], sv[4 * j + 3]);
            }
        }
        if (out_slot >= 0) {
            __syncthreads();  // every thread's part of the state is written
            if (tid == 0) {
                __threadfence();
                st_release(sc.ho_flag + out_slot, sc.epoch);
            }
        }
        tc_fence_before();
    }

    tc_fence_after();
    if (!ok) {
        // Abandoned: before the tensor memory is freed, wait (bounded again) for the
        // last issued input copy and MMA, so that neither lands in memory this CTA no
        // longer owns.  Waiting on a phase that has already completed returns at once.
        if (tid == 0) {
            (void)mbar_wait(cx.bar_tma, cx.tma_par_last);
            (void)mbar_wait(cx.bar_mma, cx.mma_phase ^ 1u);
            (void)mbar_wait(cx.bar_g2, cx.g2_phase ^ 1u);
        }
    }
    if (tid == kStoreTid) bulk_wait0();  // the output stores are complete
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(cx.tmem, kTmemCols);
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

// [B*T, H, 64] bf16 tensor viewed as (64, H, B*T), box = 64 tokens of one head; or,
// head first, [B*H, T, 64] viewed as (64, T, B*H), box = 64 tokens of one (b, h).  Both
// boxes land as 64 rows of 128 bytes, token-major.  L2 fetches are promoted to 256 bytes
// (a token-major row and the next head's, which the CTA of that head, running at the
// same time, reads) unless `wide_l2` is false (128 bytes: when the CTAs running at once
// do not hold neighbouring heads, the other half would be fetched for nobody).
inline bool make_map(CUtensorMap* map, const void* ptr, int B, int T, int H, int head_first,
                     bool wide_l2 = true) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t rows = (cuuint64_t)B * T;
    cuuint64_t dims[3] = {64, (cuuint64_t)H, rows};
    cuuint64_t strides[2] = {64 * 2, (cuuint64_t)H * 64 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    if (head_first) {
        dims[1] = (cuuint64_t)T;
        dims[2] = (cuuint64_t)B * H;
        strides[1] = (cuuint64_t)T * 64 * 2;
        box[1] = 64;
        box[2] = 1;
    }
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               wide_l2 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// State checkpoints: [H * slots][64][64] 16-bit (fp16) tiles, viewed as (64, 64,
// H * slots), box = one whole tile.
inline bool make_ck_map(CUtensorMap* map, const void* ptr, long long slices) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || slices <= 0 || slices > 0x7fffffffLL) return false;
    cuuint64_t dims[3] = {64, 64, (cuuint64_t)slices};
    cuuint64_t strides[2] = {64 * 2, 64 * 64 * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace chunked

namespace chunked {
// Optional extras of a launch: per-chunk state checkpoints (ck != nullptr: H * ck_slots
// fp16 tiles; chunk c of unit (n, h) goes to slice h * ck_slots + floor(row0 / 64) + n + c,
// row0 the sequence's first token row); o may be nullptr (no outputs).
struct Extras {
    void* ck = nullptr;
    int ck_slots = 0;
};

// The kernel's dynamic shared-memory size (above the default limit) and the largest
// shared-memory carveout (two CTAs per SM need all of it), set once per device.
template <bool kGdn, bool kHf, bool kRev>
inline cudaError_t ensure_smem_attr() {
    constexpr int kMaxDev = 64;
    static bool attr_set[kMaxDev] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(chunked_kernel<kGdn, kHf, kRev>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(chunked_kernel<kGdn, kHf, kRev>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    return cudaSuccess;
}

// Launch geometry of the balanced schedule (Sched) for `units` units of Lu tokens with
// `slots` CTAs resident at once: `ctas` runs of `cmax` chunks.  False (one unit per
// CTA) unless there are more units than slots.
inline bool balanced_geometry(long long units, int Lu, long long slots, long long& ctas,
                              long long& cmax) {
    if (Lu <= 0 || slots <= 0 || units <= slots) return false;
    const long long C = (Lu + 63) / 64, total = units * C;
    cmax = std::max(C, (total + slots - 1) / slots);
    ctas = (total + cmax - 1) / cmax;
    return true;
}

// CTAs of chunked_kernel<kGdn, kHf, kRev> resident on the current device at once (its
// dynamic shared-memory size already set), 0 if unknown.
template <bool kGdn, bool kHf, bool kRev>
inline int resident_ctas() {
    constexpr int kMaxDev = 64;
    static int cached[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        (void)cudaGetLastError();
        return 0;
    }
    if (cached[dev] == 0) {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunked_kernel<kGdn, kHf, kRev>,
                                                          kThreads, kSmemBytes) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            (void)cudaGetLastError();
            return 0;
        }
        // The occupancy query answers one per SM for this kernel, while it runs two
        // (its registers and shared memory are sized for two; the launch list shows
        // it): take the design's two unless the query allows more.
        cached[dev] = std::max(per_sm, kMinCtasPerSm) * sms;
    }
    return cached[dev];
}

// The handoff slots of the balanced schedule (Sched): one area per (host thread, device,
// stream), so launches that may run at the same time never share one.  It is made on
// first use (outside stream capture: a launch being captured with no area yet runs one
// unit per CTA) and kept for the life of the process; a captured launch keeps the area
// and epoch it was captured with, and each consumer clears its flag, so replays work.
// Set (per host thread) while an entry point that promises no allocation runs: the
// balanced schedule then takes an existing handoff area or none.
inline bool& handoff_alloc_forbidden() {
    thread_local bool forbidden = false;
    return forbidden;
}
struct Handoff {
    int dev = -1;
    cudaStream_t stream = nullptr;
    int slots = 0;
    float* state = nullptr;
    unsigned* flag = nullptr;
    unsigned epoch = 0;
};
inline Handoff* handoff_for(cudaStream_t stream, int slots) {
    constexpr int kMax = 16;
    thread_local Handoff cache[kMax];
    thread_local int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev && cache[i].stream == stream && cache[i].slots >= slots)
            return &cache[i];
    if (used == kMax || handoff_alloc_forbidden()) return nullptr;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    if (cs != cudaStreamCaptureStatusNone) return nullptr;
    const size_t state_bytes = (size_t)slots * 4096 * sizeof(float);
    void* mem = nullptr;
    // relaxed capture mode for this thread: the allocation must not disturb a capture
    // that another thread may have open
    cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
    (void)cudaThreadExchangeStreamCaptureMode(&mode);
    const cudaError_t e = cudaMalloc(&mem, state_bytes + (size_t)slots * sizeof(unsigned));
    (void)cudaThreadExchangeStreamCaptureMode(&mode);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    unsigned* flag = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(mem) + state_bytes);
    if (cudaMemsetAsync(flag, 0, (size_t)slots * sizeof(unsigned), stream) != cudaSuccess) {
        (void)cudaGetLastError();
        (void)cudaFree(mem);
        return nullptr;
    }
    Handoff& hb = cache[used++];
    hb.dev = dev;
    hb.stream = stream;
    hb.slots = slots;
    hb.state = static_cast<float*>(mem);
    hb.flag = flag;
    hb.epoch = 0;
    return &hb;
}
template <bool kGdn, bool kHf, bool kRev = false>
inline cudaError_t launch_layout(const void* const* ptrs, int nmaps, const float* s0,
                          const uint8_t* mask, void* o, float* sT, int B, int T, int H, int N,
                          const int32_t* cu_seqlens, const void* g, const void* beta,
                          int s0_shared, int stall_tid, const Extras& ex,
                          cudaStream_t stream, const RevIn* rin = nullptr,
                          int B_o = 0, int T_o = 0) {
    if (const cudaError_t e = ensure_smem_attr<kGdn, kHf, kRev>(); e != cudaSuccess) return e;
    // Units of one length (no packed sequences; for kRev, reversed sequences of an
    // unpacked problem) take the balanced schedule when there are more units than
    // resident CTAs (and a handoff area is at hand).
    long long grid = (long long)N * H, ctas = 0, cmax = 0;
    const int Lu = kRev ? (rin && !rin->cu ? 64 * (T_o / 64 + 1) : 0) : (cu_seqlens ? 0 : T);
    Handoff* hb = nullptr;
    if (Lu > 0 && balanced_geometry(grid, Lu, resident_ctas<kGdn, kHf, kRev>(), ctas, cmax))
        hb = handoff_for(stream, (int)ctas);
    const bool wide_l2 = hb == nullptr;  // neighbouring heads run at once only without it

    CUtensorMap maps[8];
    if (kRev) {  // the output is dv in the original layout; no input maps (cp.async loads)
        if (!make_map(&maps[6], rin->dv, B_o, T_o, H, rin->hf, wide_l2)) return cudaErrorInvalidValue;
        for (int i = 0; i < 6; ++i) maps[i] = maps[6];  // unused by the kernel
    }
    for (int i = 0; i < nmaps; ++i)
        if (!make_map(&maps[i], ptrs[i], B, T, H, kHf, wide_l2)) return cudaErrorInvalidValue;
    for (int i = nmaps; i < 6 && !kRev; ++i) maps[i] = maps[0];  // unused by the kernel
    if (kRev) {
    } else if (o) {
        if (!make_map(&maps[6], o, B, T, H, kHf, wide_l2)) return cudaErrorInvalidValue;  // the output
    } else {
        maps[6] = maps[0];  // unused: no outputs
    }
    if (ex.ck) {
        if (ex.ck_slots <= 0 || !make_ck_map(&maps[7], ex.ck, (long long)H * ex.ck_slots))
            return cudaErrorInvalidValue;
    } else {
        maps[7] = maps[0];  // unused: no checkpoints
    }
    const RevIn rv = rin ? *rin : RevIn{};
    Sched sc{};
    if (hb) {
        if (++hb->epoch == 0) hb->epoch = 1;
        sc.Lu = Lu;
        sc.cmax = cmax;
        sc.ho_state = hb->state;
        sc.ho_flag = hb->flag;
        sc.epoch = hb->epoch;
        grid = ctas;
    }
    chunked_kernel<kGdn, kHf, kRev><<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], maps[7], s0, mask,
        static_cast<__nv_bfloat16*>(o), sT, T, H, N, cu_seqlens,
        static_cast<const __nv_bfloat16*>(g), static_cast<const __nv_bfloat16*>(beta), s0_shared,
        stall_tid, ex.ck ? ex.ck_slots : 0, rv, sc);
    return cudaGetLastError();
}
template <bool kGdn>
inline cudaError_t launch(const void* const* ptrs, int nmaps, const float* s0,
                          const uint8_t* mask, void* o, float* sT, int B, int T, int H, int N,
                          const int32_t* cu_seqlens, const void* g, const void* beta,
                          int s0_shared, int head_first, int stall_tid, const Extras& ex,
                          cudaStream_t stream) {
    return head_first
               ? launch_layout<kGdn, true>(ptrs, nmaps, s0, mask, o, sT, B, T, H, N, cu_seqlens,
                                           g, beta, s0_shared, stall_tid, ex, stream)
               : launch_layout<kGdn, false>(ptrs, nmaps, s0, mask, o, sT, B, T, H, N, cu_seqlens,
                                            g, beta, s0_shared, stall_tid, ex, stream);
}
}  // namespace chunked

inline cudaError_t launch_chunked(const void* r, const void* w, const void* k, const void* v,
                                  const void* a, const void* b, const float* s0,
                                  const uint8_t* mask, void* o, float* sT, int B, int T, int H,
                                  int N, const int32_t* cu_seqlens, int head_first,
                                  int stall_tid, cudaStream_t stream,
                                  const chunked::Extras& ex = chunked::Extras{}) {
    const void* ptrs[6] = {r, w, k, v, a, b};
    return chunked::launch<false>(ptrs, 6, s0, mask, o, sT, B, T, H, N, cu_seqlens, nullptr,
                                  nullptr, 0, head_first, stall_tid, ex, stream);
}

// The backward's reversed run of the state gradient (see RevIn): unit n of the packed
// reversed sequences `cur` ([N + 1], multiples of 64, rows_r in all) for every head, from
// the state dsT (or zero) to ds0, with per-chunk checkpoints and dv written in the
// original layout ([B_o, T_o, H, 64] or head first).  The input maps are not read.
inline cudaError_t launch_chunked_rev(const chunked::RevIn& rin, int B_o, const float* dsT, float* ds0,
                                      int rows_r, int H, int N, const int32_t* cur,
                                      const chunked::Extras& ex, cudaStream_t stream) {
    return chunked::launch_layout<false, false, true>(nullptr, 0, dsT, nullptr, nullptr, ds0, 1,
                                                      rows_r, H, N, cur, nullptr, nullptr, 0, -1,
                                                      ex, stream, &rin, B_o, rin.T);
}

// Gated DeltaNet: q, k, v [B*T, H, 64] bf16 through the r, k, v maps; g, beta [B*T, H]
// (head first: [B*H, T, 64] and [B*H, T]).
inline cudaError_t launch_chunked_gdn(const void* q, const void* k, const void* v,
                                      const void* g, const void* beta, const float* s0,
                                      int s0_shared, void* o, float* sT, int B, int T, int H,
                                      int N, const int32_t* cu_seqlens, int head_first,
                                      cudaStream_t stream) {
    // map order r, w, k, v: the unused w slot repeats q
    const void* ptrs[4] = {q, q, k, v};
    return chunked::launch<true>(ptrs, 4, s0, nullptr, o, sT, B, T, H, N, cu_seqlens, g, beta,
                                 s0_shared, head_first, -1, chunked::Extras{}, stream);
}

}  // namespace wkv7
