/*
 * wkv7.h -- C ABI of the B200 (sm_100a) WKV7 library (libwkv7.so).
 *
 * WKV7 is the RWKV-7 "generalized delta rule" recurrence behind
 * generalized_delta_rule(r, w, k, v, a, b, initial_state, output_final_state,
 * head_first, mask) and its length-one decode form rwkv7_op_rnn (rwkv-ops
 * 0.9.0 README, sections "rwkv7op 使用方法" and "rwkv7_op_rnn 使用方法";
 * rwkv-ops 0.7.4 README, same sections).  Per (sequence, head) a K x V fp32
 * state S, stored row-major [k][v], evolves token by token:
 *
 *     u_t = S_{t-1}^T a_t                      (a reads the old state)
 *     S_t = diag(exp(w_t)) S_{t-1} + b_t u_t^T + k_t v_t^T
 *     o_t = S_t^T r_t
 *
 * w is the per-channel decay in log space (the README's docstring: "decay
 * term in log space"); q in the docstring is r here, gk is w.  mask[b,t] = 0
 * means the state is not updated at that token (docstring: 1 update, 0 no
 * update); the output there is read from the unchanged state,
 * o_t = S_{t-1}^T r_t.
 *
 * Conventions shared by every entry point:
 *  - All pointers are DEVICE pointers of the current CUDA device, dense,
 *    row-major and 16-byte aligned.  The caller owns and allocates every
 *    buffer; the library frees nothing and allocates one thing of its own: the
 *    chunked kernel's handoff area (about 4.9 MB per host thread, device and
 *    stream, made by the first launch on that stream that splits sequences
 *    between CTAs, outside stream capture; see wkv7_fwd).
 *  - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *    stream).  A non-OK return means either nothing was launched (argument
 *    check on the host) or the launch itself failed (WKV7_ERR_CUDA).
 *  - Problems only the device can see (a cu_seqlens entry out of order or out
 *    of range) are recorded in a device-side flag; the affected sequence is
 *    skipped (its outputs are left unwritten) and wkv7_get_last_error reports
 *    it.  No kernel traps, asserts or spins without a bound.
 *  - Inputs r, w, k, a, b are [B, T, H, K]; v is [B, T, H, V]; the output o is
 *    [B, T, H, V]; all of them share one element type (wkv7_dtype).  With
 *    WKV7_LAYOUT_BHTK (the README's head_first=True) they are [B, H, T, K] /
 *    [B, H, T, V] instead.  States are fp32 [N, H, K, V] in both layouts (the
 *    README's initial_state / final_state layout).
 *  - Supported head sizes: K == V in {64, 128, 256} (the README's head_size,
 *    default 64).  The chunked tensor-core kernel takes 64 only; other sizes
 *    run on the fp32 CUDA-core kernels.  Anything else returns
 *    WKV7_ERR_UNSUPPORTED.
 */
#ifndef WKV7_H
#define WKV7_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WKV7_OK = 0,
    WKV7_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, bad size, bad combination   */
    WKV7_ERR_UNSUPPORTED = 2,    /* valid request outside the supported set (e.g. K != 64) */
    WKV7_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed                    */
    WKV7_ERR_DEVICE_TIMEOUT = 4, /* a bounded device-side wait gave up (reported later)    */
    WKV7_ERR_DEVICE_BAD_SEQLENS = 5 /* a kernel found cu_seqlens out of order / range       */
} wkv7_status;

typedef enum {
    WKV7_BF16 = 0, /* r, w, k, v, a, b and o are bfloat16 */
    WKV7_F32 = 1   /* r, w, k, v, a, b and o are float32  */
} wkv7_dtype;

typedef enum {
    WKV7_LAYOUT_BTHK = 0, /* [B, T, H, *]: token-major (README default, head_first=False) */
    WKV7_LAYOUT_BHTK = 1  /* [B, H, T, *]: head-first (README head_first=True)            */
} wkv7_layout;

typedef enum {
    WKV7_ALGO_AUTO = 0,      /* library's choice (chunked tensor-core form for bf16, K = 64)   */
    WKV7_ALGO_RECURRENT = 1, /* token-by-token fp32 recurrence on CUDA cores                  */
    WKV7_ALGO_CHUNKED = 2    /* 64-token chunks, WY form, tcgen05 tensor cores (bf16 only)    */
} wkv7_algo;

/*
 * wkv7_fwd -- forward over whole sequences (generalized_delta_rule /
 * generalized_delta_rule_inference; forward only, no autograd state kept).
 *
 *   r, w, k, a, b  [B, T, H, K]  dtype   receptance, log decay, key, a (read), b (write)
 *   v              [B, T, H, V]  dtype
 *   s0             [N, H, K, V]  fp32    initial states, or NULL for zeros
 *                                        (README: initial_state=None)
 *   mask           [B, T]        uint8   nonzero = update, 0 = keep the state; NULL = all 1;
 *                                        with cu_seqlens it is [1, T] over the packed rows
 *   o              [B, T, H, V]  dtype   output, fully written (must not alias an input)
 *   sT             [N, H, K, V]  fp32    final states, or NULL to skip
 *                                        (README: output_final_state=False); may equal s0
 *   cu_seqlens     [N + 1]       int32   packed variable-length form, or NULL.  When given,
 *                                        B must be 1, sequence n is rows
 *                                        [cu_seqlens[n], cu_seqlens[n+1]) of the packed T,
 *                                        cu_seqlens[0] = 0, cu_seqlens[N] = T, non-decreasing.
 *                                        When NULL, N must equal B.
 *   layout         wkv7_layout           token-major or head-first inputs and o (mask stays
 *                                        [B, T], states [N, H, K, V])
 *   algo           wkv7_algo             kernel family (WKV7_ALGO_AUTO unless testing)
 *
 * Returns WKV7_OK after enqueueing the kernel(s) on `stream`.
 * B, T or N may be 0 (nothing to compute; with T == 0, sT receives s0 or zeros).
 *
 * Range of the chunked form (WKV7_ALGO_CHUNKED, and AUTO for bf16): exact while a
 * 64-token chunk's decay stays within e^{-80} (per-step log decay >= -1.26 on
 * average); the state and v enter its last tensor-core product as fp16 operands,
 * so their magnitudes must stay below 65504 (larger values saturate).  The
 * recurrent form has neither limit.
 *
 * Scheduling of the chunked form: an unpacked problem (cu_seqlens == NULL) with more
 * (sequence, head) units than the GPU holds CTAs at once (two per SM) is cut into
 * equal runs of chunks, one per CTA, a sequence split between two CTAs passing its
 * fp32 state through the library's handoff area (see the conventions above); the
 * results are bit-identical to one CTA per unit.  Packed problems, smaller ones, and a
 * launch being captured on a stream that has no handoff area yet run one CTA per
 * unit (packed sequences longest first).
 */
wkv7_status wkv7_fwd(const void* r, const void* w, const void* k, const void* v,
                     const void* a, const void* b, const float* s0, const uint8_t* mask,
                     void* o, float* sT, int B, int T, int H, int K, int V,
                     const int32_t* cu_seqlens, int N, wkv7_layout layout, wkv7_dtype dtype,
                     wkv7_algo algo, void* stream);

/*
 * wkv7_step -- one decode token for B independent states (rwkv7_op_rnn with
 * T = 1; README: inputs (B, 1, H, K), state (B, H, K, K)).
 *
 *   r, w, k, a, b  [B, H, K]     dtype
 *   v              [B, H, V]     dtype
 *   state          [B, H, K, V]  fp32    read and updated IN PLACE (S_{t-1} -> S_t)
 *   o              [B, H, V]     dtype   o = S_t^T r (must not alias state or inputs)
 *
 * Each state is streamed from HBM once and written back once.
 */
wkv7_status wkv7_step(const void* r, const void* w, const void* k, const void* v,
                      const void* a, const void* b, float* state, void* o, int B, int H,
                      int K, int V, wkv7_dtype dtype, void* stream);

/*
 * wkv7_bwd -- backward of wkv7_fwd (the README's training entry,
 * generalized_delta_rule, supports backpropagation; rwkv-ops 0.9.0 README,
 * "rwkv7op 使用方法").  For the loss L = sum(o * dout) + sum(S_T * dsT) it writes
 * the gradients of every forward input, by reverse-mode differentiation of the
 * recurrence:
 *
 *     G = dL/dS_t;  G += r_t do_t^T;  dr_t = S_t do_t;  dv_t = G^T k_t;  dk_t = G v_t;
 *     du_t = G^T b_t;  db_t = G u_t;  da_t = S_{t-1} du_t;
 *     dw_t = e^{w_t} * rowsum(G * S_{t-1});  G <- diag(e^{w_t}) G + a_t du_t^T;
 *     ds0 = G after the first token.
 *
 *   r, w, k, v, a, b, s0, mask, cu_seqlens, N, layout   as for wkv7_fwd (K = V = 64)
 *   dout           shaped like v dtype   dL/do (required)
 *   dsT            [N, H, K, V]  fp32    dL/dS_T, or NULL for zero
 *   dr, dw, dk, da, db (shaped like r), dv (like v)   dtype   outputs (fully written;
 *                                        must not alias an input)
 *   ds0            [N, H, K, V]  fp32    dL/ds0, or NULL to skip
 *   workspace      device buffer of at least wkv7_bwd_workspace_bytes(B, T, H, K, V, N)
 *                  bytes, or of wkv7_bwd_workspace_bytes_algo for the family that runs
 *                  (16-byte aligned; the caller owns it; contents on return are scratch)
 *
 * K = V = 64 only.  A masked token passes the state gradient through and has zero
 * dw, dk, dv, da, db.  Two kernel families (wkv7_bwd picks as AUTO does):
 *   - bf16 (AUTO, WKV7_ALGO_CHUNKED): the chunked form on tcgen05 tensor cores.  The
 *     state gradient G_t = dL/dS_t obeys G_t = r_t do_t^T + (diag(e^{w_{t+1}}) +
 *     a_{t+1} b_{t+1}^T) G_{t+1}: a WKV7 recurrence read backwards in time (a and b
 *     swapped, r and do as the write pair), so it runs on the chunked forward kernel
 *     over reversed copies of the inputs, from dsT; its final state is ds0 and its
 *     outputs (with k as the read vector) are dv.  A forward pass stores the fp16 state
 *     at every 64-token chunk start, the reversed pass the state gradient at every
 *     chunk end, and one kernel then forms every chunk's dr, dw, dk, da, db in
 *     parallel from the chunk's inputs and those two 64 x 64 checkpoints (the adjoint
 *     of the chunk's WY products).  Six launches on `stream`.
 *   - fp32 (AUTO, WKV7_ALGO_RECURRENT): fp32 recurrences on CUDA cores: a forward that
 *     stores the states every 8 tokens and every token's u = S_{t-1}^T a, then the
 *     reverse pass.  Two launches on `stream`.
 * The workspace bound covers both.
 */
size_t wkv7_bwd_workspace_bytes(int B, int T, int H, int K, int V, int N);

/*
 * wkv7_bwd_workspace_bytes_algo -- the workspace one kernel family needs (what
 * wkv7_bwd_with_algo checks): the chunked form (dtype bf16 with WKV7_ALGO_CHUNKED or
 * WKV7_ALGO_AUTO) needs the reversed-sequence offsets and the fp16 state checkpoints of
 * its two passes, about 2 x 8 KiB per 64-token chunk and head; the fp32 recurrences
 * (WKV7_ALGO_RECURRENT, or AUTO with fp32) the states every 8 tokens and every token's
 * u.  Returns 0 for unsupported arguments (K != 64, fp32 with WKV7_ALGO_CHUNKED).
 * wkv7_bwd_workspace_bytes is the larger of the two.
 */
size_t wkv7_bwd_workspace_bytes_algo(int B, int T, int H, int K, int V, int N, wkv7_dtype dtype,
                                     wkv7_algo algo);

wkv7_status wkv7_bwd(const void* r, const void* w, const void* k, const void* v, const void* a,
                     const void* b, const float* s0, const uint8_t* mask, const void* dout,
                     const float* dsT, void* dr, void* dw, void* dk, void* dv, void* da,
                     void* db, float* ds0, int B, int T, int H, int K, int V,
                     const int32_t* cu_seqlens, int N, wkv7_layout layout, wkv7_dtype dtype,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * wkv7_bwd_with_algo -- wkv7_bwd with the kernel family chosen by the caller:
 * WKV7_ALGO_AUTO (as wkv7_bwd), WKV7_ALGO_RECURRENT (the fp32 CUDA-core recurrences,
 * bf16 or fp32 inputs) or WKV7_ALGO_CHUNKED (bf16 only; fp32 returns
 * WKV7_ERR_UNSUPPORTED).  Arguments and results are otherwise those of wkv7_bwd.
 */
wkv7_status wkv7_bwd_with_algo(const void* r, const void* w, const void* k, const void* v,
                               const void* a, const void* b, const float* s0,
                               const uint8_t* mask, const void* dout, const float* dsT, void* dr,
                               void* dw, void* dk, void* dv, void* da, void* db, float* ds0,
                               int B, int T, int H, int K, int V, const int32_t* cu_seqlens,
                               int N, wkv7_layout layout, wkv7_dtype dtype, wkv7_algo algo,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * wkv7_bwd_noalloc -- wkv7_bwd with the library's own scratch instead of a caller
 * workspace.  The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory (code that runs where cudaMalloc is forbidden or
 * unavailable, such as a host framework that owns every allocation, or a path that
 * must not call into the allocator).  The scratch is a file-scope device array of
 * WKV7_STATIC_SCRATCH_BYTES that every GPU which loads the library keeps until exit.
 * Problems whose wkv7_bwd_workspace_bytes exceed it return WKV7_ERR_UNSUPPORTED before
 * anything is launched.  The call allocates nothing itself (its chunked forward runs
 * take the balanced schedule only on a stream that already has a handoff area, else
 * one CTA per unit, with the same results); it runs on the CURRENT
 * device, which must be the device of every pointer and of the stream.  Its first call
 * on a device looks up the array's address there (cudaGetSymbolAddress, cached per
 * device); with CUDA's lazy module loading that first call may also load the library's
 * device code, which is when the array is reserved -- make a first call (or any other
 * call into the library) on each device before capturing a stream.  Every call shares
 * the one array: calls that overlap on the GPU race (issue them on one stream, or
 * synchronise between streams).  Arguments and results are those of wkv7_bwd.
 */
#define WKV7_STATIC_SCRATCH_BYTES (64u << 20)

wkv7_status wkv7_bwd_noalloc(const void* r, const void* w, const void* k, const void* v,
                             const void* a, const void* b, const float* s0,
                             const uint8_t* mask, const void* dout, const float* dsT, void* dr,
                             void* dw, void* dk, void* dv, void* da, void* db, float* ds0, int B,
                             int T, int H, int K, int V, const int32_t* cu_seqlens, int N,
                             wkv7_layout layout, wkv7_dtype dtype, void* stream);

/*
 * wkv7_sane_fwd -- the WKV7 forward with State Anomaly Neutralization
 * (generalized_delta_rule_sane / generalized_delta_rule_sane_inference; rwkv-ops 0.9.0
 * README, "rwkv7op_sane 使用方法").  The recurrence of wkv7_fwd, and after the last
 * token of every full 16-token chunk c (tokens 16 c .. 16 c + 15, c < T / 16) whose
 * flag is set, the state is soft-clipped elementwise with that chunk's tau:
 *
 *     S <- tau[b, c, h] * tanh(S / tau[b, c, h])
 *
 * The output of token 16 c + 15 is read from the state before the clip (README: the
 * output is based on the state before SANE).  A partial last chunk is not clipped
 * (tau holds T / 16 chunks; README: the inference kernel reads tau per chunk, so T
 * need not be a multiple of 16).  The README defers the clip function to the SANE
 * paper; tau * tanh(S / tau) is the reading implemented (parity for the function
 * itself is unpinned by the pages).
 *
 *   r, w, k, v, a, b  as for wkv7_fwd ([B, T, H, *], or [B, H, T, *] with
 *                     WKV7_LAYOUT_BHTK); no token mask and no packed sequences
 *   tau            [B, T / 16, H]  fp32  > 0 (README: softplus(param) + 1); may be NULL
 *                                        only when T < 16
 *   sane_mask      [B, T / 16]   uint8   nonzero = clip after that chunk, 0 = skip (README:
 *                                        per-chunk 0/1 shared by all heads); NULL = every chunk
 *   s0             [B, H, K, V]  fp32    initial states or NULL; with s0_shared = 1 a single
 *                                        [1, H, K, V] state used by every batch row
 *   o              [B, T, H, V]  dtype   output; sT [B, H, K, V] fp32 or NULL (may equal s0
 *                                        unless s0_shared with B > 1)
 *   K = V in {64, 128, 256}; dtype bf16 or fp32 (fp32 state and arithmetic throughout).
 *
 * Runs on the fp32 CUDA-core recurrent kernel.  Returns WKV7_ERR_INVALID_ARG /
 * WKV7_ERR_UNSUPPORTED before any launch on bad arguments, WKV7_ERR_CUDA if the
 * launch fails.  The caller owns every buffer.
 */
wkv7_status wkv7_sane_fwd(const void* r, const void* w, const void* k, const void* v,
                          const void* a, const void* b, const float* tau,
                          const uint8_t* sane_mask, const float* s0, int s0_shared, void* o,
                          float* sT, int B, int T, int H, int K, int V, wkv7_layout layout,
                          wkv7_dtype dtype, void* stream);

/*
 * wkv7_sane_step -- one decode token with State Anomaly Neutralization
 * (rwkv7_op_sane_rnn; rwkv-ops 0.9.0 README, "rwkv7_op_sane_rnn 使用方法").  The step
 * of wkv7_step; then, for the batch rows whose flag is set, the state written back is
 * soft-clipped with tau[b, h] as in wkv7_sane_fwd.  o is read from the state before
 * the clip.  The README's loop calls it with do_sane = (step % 16 == 15).
 *
 *   r, w, k, v, a, b, state, o   as for wkv7_step ([B, H, K], state [B, H, K, V] in place)
 *   tau            [B, H]        fp32    > 0
 *   do_sane        [B]           uint8   nonzero = clip that row; NULL = do_sane_all (0 or 1)
 *                                        for every row (README: do_sane is a bool or [B])
 *
 * Errors and ownership as for wkv7_step.
 */
wkv7_status wkv7_sane_step(const void* r, const void* w, const void* k, const void* v,
                           const void* a, const void* b, const float* tau,
                           const uint8_t* do_sane, int do_sane_all, float* state, void* o,
                           int B, int H, int K, int V, wkv7_dtype dtype, void* stream);

/*
 * wkv7_gdn_fwd -- Gated DeltaNet forward over whole sequences
 * (gated_delta_net_recurrent / gated_delta_net_recurrent_inference /
 * gated_delta_net_chunk; rwkv-ops 0.9.0 README, "gdn_recurrent 使用方法" and
 * "gdn_chunk 使用方法"), computed by the same kernels as wkv7_fwd.  Per
 * (sequence, head) and token, with qh = q / |q| and kh = k / |k| over K (the
 * README: q and k are L2-normalised inside; a zero vector stays zero):
 *
 *     S_t = exp(g_t) (I - beta_t kh_t kh_t^T) S_{t-1} + beta_t kh_t v_t^T
 *     o_t = S_t^T qh_t
 *
 * i.e. the generalized rule above with w_t = g_t on every channel, a_t = kh_t,
 * b_t = -exp(g_t) beta_t kh_t and write key beta_t kh_t.  q is not scaled
 * further (the README states no scale).
 *
 *   q, k           [B, T, H, K]  dtype   query and key (normalised inside)
 *   v              [B, T, H, V]  dtype
 *   g              [B, T, H]     dtype   log-space decay gate (exp(g) multiplies the state)
 *   beta           [B, T, H]     dtype   write strength, expected in (0, 1) (README: already
 *                                        passed through a sigmoid; not checked)
 *   s0             [N, H, K, V]  fp32    initial states, or NULL for zeros; with s0_shared = 1
 *                                        a single [1, H, K, V] state used by every sequence
 *   o              [B, T, H, V]  dtype   output (must not alias an input)
 *   sT             [N, H, K, V]  fp32    final states, or NULL; may equal s0 unless s0_shared
 *                                        and N > 1
 *   cu_seqlens, N, layout, algo, stream  as for wkv7_fwd (no mask: the README's operator has
 *                                        none); head-first g and beta are [B, H, T]
 *
 * q, k, v, o, s0, sT must be 16-byte aligned; g and beta only aligned to their element.
 * The chunked form has the range stated for wkv7_fwd: a chunk's summed gate within
 * -80, and state / v magnitudes below 65504.
 */
wkv7_status wkv7_gdn_fwd(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* s0, int s0_shared, void* o, float* sT,
                         int B, int T, int H, int K, int V, const int32_t* cu_seqlens, int N,
                         wkv7_layout layout, wkv7_dtype dtype, wkv7_algo algo, void* stream);

/*
 * wkv7_gdn_step -- one Gated DeltaNet decode token for B independent states
 * (gated_delta_net_recurrent_single_step; README: q, k (B, H, K), v (B, H, V),
 * g, beta (B, H), state (B, H, K, V)).
 *
 *   q, k           [B, H, K]     dtype
 *   v              [B, H, V]     dtype
 *   g, beta        [B, H]        dtype   (element-aligned)
 *   state          [B, H, K, V]  fp32    read and updated IN PLACE
 *   o              [B, H, V]     dtype   o = S_t^T qh (must not alias state or inputs)
 */
wkv7_status wkv7_gdn_step(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, float* state, void* o, int B, int H, int K, int V,
                          wkv7_dtype dtype, void* stream);

/*
 * wkv7_gdn_bwd -- backward of wkv7_gdn_fwd (the README's gated_delta_net_recurrent
 * and gated_delta_net_chunk support backpropagation), for
 * L = sum(o * dout) + sum(S_T * dsT): the generalized-rule backward (wkv7_bwd) on the
 * substituted inputs r = qh, w = g, write key beta kh, a = kh, b = -e^g beta kh, then
 * the chain rule through the substitution and the L2 normalisation of q and k (the
 * gradient of a zero q or k is zero).
 *
 *   q, k, v, g, beta, s0, s0_shared, cu_seqlens, N, layout   as for wkv7_gdn_fwd (K = V = 64)
 *   dout           shaped like v dtype   dL/do (required)
 *   dsT            [N, H, K, V]  fp32    dL/dS_T, or NULL
 *   dq, dk (like q), dv (like v), dg, dbeta (like g)   dtype   outputs
 *   ds0            fp32, shaped like s0 ([1, H, K, V] when shared: summed over the
 *                  sequences), or NULL
 *   workspace      at least wkv7_gdn_bwd_workspace_bytes(B, T, H, K, V, N, dtype,
 *                  s0_shared) bytes of device memory (16-byte aligned)
 */
size_t wkv7_gdn_bwd_workspace_bytes(int B, int T, int H, int K, int V, int N, wkv7_dtype dtype,
                                     int s0_shared);

wkv7_status wkv7_gdn_bwd(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* s0, int s0_shared, const void* dout,
                         const float* dsT, void* dq, void* dk, void* dv, void* dg, void* dbeta,
                         float* ds0, int B, int T, int H, int K, int V,
                         const int32_t* cu_seqlens, int N, wkv7_layout layout,
                         wkv7_dtype dtype, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * wkv7_get_last_error -- synchronises `stream`, returns and clears the sticky
 * device-side flag (WKV7_ERR_DEVICE_TIMEOUT / WKV7_ERR_DEVICE_BAD_SEQLENS) of
 * the current device, or WKV7_ERR_CUDA if the stream reports a CUDA error,
 * else WKV7_OK.
 */
wkv7_status wkv7_get_last_error(void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* wkv7_status_string(wkv7_status s);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int wkv7_version(void);

/*
 * wkv7_test_stall_next_chunked -- test hook of the failure path (no counterpart on the
 * pages).  Every wait of the chunked kernel on an asynchronous copy or MMA is bounded
 * (one second of device time); a thread that gives up raises WKV7_ERR_DEVICE_TIMEOUT,
 * the CTA agrees on abandoning its sequence at its next barrier, waits (bounded) for
 * the copies and MMAs it issued, frees its tensor memory and returns, so the context
 * stays usable.  This call makes the NEXT chunked wkv7_fwd launch exercise that path
 * without any fault: thread `tid` of the first CTA waits, with a 2 ms limit, on an
 * mbarrier that nothing arrives at, right after its first chunk's inputs have landed
 * (no copy or MMA in flight).  That sequence's outputs and final state are then not
 * written; wkv7_get_last_error reports WKV7_ERR_DEVICE_TIMEOUT.  tid = -1 cancels;
 * the hook is consumed by one launch.  Returns WKV7_ERR_INVALID_ARG for tid outside
 * [-1, 256).
 */
wkv7_status wkv7_test_stall_next_chunked(int tid);

/*
 * wkv7_test_chunked_schedule -- test hook (no counterpart on the pages): the launch
 * geometry the chunked kernel takes for `units` (sequence, head) units all `len` tokens
 * long (unpacked problems) on the current device.  *resident receives the CTAs of the
 * token-major WKV7 kernel resident at once; when units > *resident the balanced
 * schedule cuts the units' chunks, laid end to end, into *ctas runs of *cmax chunks (one
 * CTA each; a unit cut between CTAs m and m+1 runs its first chunks on m+1 and its last
 * ones on m), else *ctas = *cmax = 0 (one unit per CTA).  Host memory pointers, written
 * only on success.  Returns WKV7_ERR_INVALID_ARG for a null pointer, units < 0 or
 * len < 0, WKV7_ERR_CUDA when the device cannot be queried.  Launches nothing.
 */
wkv7_status wkv7_test_chunked_schedule(long long units, int len, int* resident, long long* ctas,
                                       long long* cmax);

#ifdef __cplusplus
}
#endif

#endif /* WKV7_H */
