/*
 * rwkv_wkv.h -- C ABI of libwkv.so: the WKV time-mixing recurrences of RWKV-4 and
 * Eagle/Finch (RWKV-5/6) on NVIDIA B200 (sm_100a).
 *
 * Sources (page title, section):
 *  [R4]   "RWKV: Reinventing RNNs for the Transformer Era" (Chinese translation):
 *         section "类 Transformer 的并行化" (time-parallel mode: the WKV update is a
 *         serial scan of cost O(BTd)); section "梯度稳定性和层堆叠" (single-step
 *         time-dependent softmax); section "利用时间结构进行时序数据处理" (time decay
 *         e^{-w} and bonus e^{u} of eq. 14); section "类 RNN 的序列解码" (RNN-mode
 *         decoding with constant memory per token).
 *  [E412] "RWKV-5/6 (Eagle and Finch)", section 4.1.2 (Eagle time mixing): matrix-valued
 *         state s = sum of k^T v, decayed per key channel by w, gain u on the current
 *         token, receptance as a query; w = exp(-exp(omega)) in (0,1).  Section 4 fixes
 *         row vectors with matrices acting on the right.
 *  [F422] same page, section 4.2.2 (Finch time mixing): w_t varies per token and channel.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller, dense and row-major
 *    with the channel index innermost.  The library never allocates, frees or retains
 *    them; it reads inputs and writes outputs asynchronously on the calling thread's
 *    stream (rwkv_set_stream) and returns before the GPU has finished.
 *  - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16, round-to-nearest-
 *    even on output).  Accumulation is fp32 throughout.
 *  - Every tensor pointer must be 16-byte aligned (RWKV_ERR_ALIGN otherwise).
 *  - Sizes are int64_t and must be >= 0 (RWKV_ERR_SHAPE otherwise).  A call with no
 *    output element to produce returns RWKV_OK without launching; for T == 0 the final
 *    state is still written (a copy of s0, or the empty state).
 *  - A pointer may be NULL only where stated, or when the tensor it names is empty.
 *  - Outputs must not overlap any input (RWKV_ERR_ALIAS), except that a state output
 *    may be the very same pointer as the state input (in-place state update).
 *  - Return value: RWKV_OK (0) or a negative rwkv_status.  Argument errors are found
 *    on the host before any CUDA call.  RWKV_ERR_CUDA means a launch or CUDA runtime
 *    call failed; rwkv_last_error() has the text.  Faults inside a kernel that the
 *    kernel itself detects (e.g. a bounded wait that ran out) are reported through the
 *    device status word, read with rwkv_get_device_status().
 *  - The library keeps no device memory of its own beyond its status word and the fixed
 *    scratch array of rwkv_wkv6_forward_bf16_noalloc (statically allocated __device__
 *    variables).  The only per-call allocation is the stream-ordered scratch of a split
 *    chunked WKV-6 call (see rwkv_set_wkv6_segments); the backward pass takes its
 *    workspace from the caller.
 */
#ifndef RWKV_WKV_H
#define RWKV_WKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RWKV_ABI_VERSION 1

typedef enum rwkv_status {
    RWKV_OK = 0,
    RWKV_ERR_NULL = -1,        /* a required pointer is NULL                          */
    RWKV_ERR_SHAPE = -2,       /* a negative size, or a size product overflows        */
    RWKV_ERR_UNSUPPORTED = -3, /* e.g. WKV-6 head size N != 64                        */
    RWKV_ERR_ALIAS = -4,       /* an output overlaps an input                         */
    RWKV_ERR_CUDA = -5,        /* a CUDA runtime call or kernel launch failed         */
    RWKV_ERR_TIMEOUT = -6,     /* a bounded device-side wait ran out (device status)  */
    RWKV_ERR_ALIGN = -7,       /* a tensor pointer is not 16-byte aligned             */
    RWKV_ERR_ARG = -8,         /* another invalid argument (e.g. unknown option)      */
    RWKV_ERR_BOUNDS = -9       /* debug build only: a kernel's index check failed and
                                  the access was skipped (device status)              */
} rwkv_status;

/* ------------------------------------------------------------------ RWKV-4 WKV [R4]
 * Per batch row b and channel c, with keys k_t, values v_t:
 *   y_t = ( sum_{i<t} e^{-(t-1-i) w_c + k_i} v_i + e^{u_c + k_t} v_t )
 *       / ( sum_{i<t} e^{-(t-1-i) w_c + k_i}     + e^{u_c + k_t}     )
 * evaluated in the running-maximum (time-dependent softmax) form, so k may be large.
 *   w, u : [C] fp32.  w is the positive decay RATE (per-step factor e^{-w}); the
 *          library does not exponentiate a learned parameter for you.
 *   k, v : [B, T, C];  y : [B, T, C] (same dtype as k).
 */
int rwkv_wkv4_forward(int64_t B, int64_t T, int64_t C,
                      const float *w, const float *u,
                      const float *k, const float *v, float *y);
int rwkv_wkv4_forward_bf16(int64_t B, int64_t T, int64_t C,
                           const float *w, const float *u,
                           const uint16_t *k, const uint16_t *v, uint16_t *y);

/* RWKV-4 WKV with state carry, so a sequence can be split across calls exactly
 * ([R4] RNN-mode decoding).  State layout s0/sT: [B, 3, C] fp32 = (a, b, p) per
 * channel, meaning numerator = a e^p and denominator = b e^p of the decayed past sums
 * after the last token processed.  An empty state has a = b = 0 (p is then ignored;
 * the library writes p = -1e30 for it).  s0 NULL = empty state; sT NULL = not written;
 * sT may equal s0.  The (a, b, p) triple is not unique: compare states through
 * a e^{p-P}, b e^{p-P} at a common P. */
int rwkv_wkv4_forward_state(int64_t B, int64_t T, int64_t C,
                            const float *w, const float *u,
                            const float *k, const float *v,
                            const float *s0, float *y, float *sT);
int rwkv_wkv4_forward_state_bf16(int64_t B, int64_t T, int64_t C,
                                 const float *w, const float *u,
                                 const uint16_t *k, const uint16_t *v,
                                 const float *s0, uint16_t *y, float *sT);

/* ------------------------------------------------------- Eagle/Finch WKV-6 [E412][F422]
 * Per batch row b and head h, state S (N x N, row i = key channel, column j = value
 * channel), for t = 0..T-1:
 *   y_t[j] = sum_i r_t[i] ( S[i][j] + u[i] k_t[i] v_t[j] )
 *   S[i][j] <- w_t[i] S[i][j] + k_t[i] v_t[j]
 * with S = s0 before the first token and sT = S after the last.
 *   r, k, v, w, y : [B, T, H, N]; w_t in (0, 1] (Eagle: constant over t; Finch: per
 *                   token).  w outside (0, 1] is outside the contract: results are then
 *                   unspecified but the call never faults.
 *   u             : [H, N] fp32.
 *   s0, sT        : [B, H, N, N] fp32.  s0 NULL = zero state; sT NULL = not written;
 *                   sT may equal s0 (in-place).
 *   N must be 64 (RWKV_ERR_UNSUPPORTED otherwise).
 * fp32 inputs run a serial fp32 kernel (SIMT).  bf16 inputs with T > 1 run the chunked
 * tensor-core kernel (64-token chunks, bf16 operands, fp32 accumulation, state in fp32);
 * T == 1 runs the bandwidth-bound decode kernel.
 */
int rwkv_wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t N,
                      const float *r, const float *k, const float *v, const float *w,
                      const float *u, const float *s0, float *y, float *sT);
int rwkv_wkv6_forward_bf16(int64_t B, int64_t T, int64_t H, int64_t N,
                           const uint16_t *r, const uint16_t *k, const uint16_t *v,
                           const uint16_t *w, const float *u, const float *s0,
                           uint16_t *y, float *sT);

/* WKV-6 with the time-mixing output stage fused into the epilogue ([E412]: LayerNorm on
 * each head, i.e. GroupNorm over the H heads, then the SiLU attention gate):
 *   o = the rwkv_wkv6_forward_bf16 output (fp32 before rounding),
 *   y[b,t,h,:] = SiLU(g[b,t,h,:]) * ( ln_w[h,:] * (o - mean) / sqrt(var + eps) + ln_b[h,:] )
 * with mean and var (mean of squared deviations) over the N channels of o[b,t,h,:] and
 * SiLU(x) = x / (1 + e^-x).  y is written once, in bf16; the state is as in
 * rwkv_wkv6_forward_bf16.
 *   g             : [B, T, H, N] bf16, the gate before its activation; must not overlap y.
 *   ln_w, ln_b    : [H, N] fp32, the per-channel scale and shift (not NULL).
 *   eps           : >= 0 (RWKV_ERR_ARG otherwise).
 * T > 1 runs the chunked kernel, T == 1 the decode kernel, each with the fused epilogue
 * (the rwkv_set_wkv6_algo choice does not apply).  Other arguments, layouts, aliasing
 * rules and errors are those of rwkv_wkv6_forward_bf16. */
int rwkv_wkv6_forward_gated_bf16(int64_t B, int64_t T, int64_t H, int64_t N,
                                 const uint16_t *r, const uint16_t *k, const uint16_t *v,
                                 const uint16_t *w, const float *u, const float *s0,
                                 const uint16_t *g, const float *ln_w, const float *ln_b, float eps,
                                 uint16_t *y, float *sT);

/* WKV-6 fed the decay LOGIT instead of the decay ([E412]: w = exp(-exp(omega)) with omega
 * the trainable per-head parameter; [F422]: omega_t per token, the learned omega plus the
 * data-dependent LoRA offset of the Finch token shift, section 4.2.1).  The kernels form
 *   w_t[i] = exp(-exp(omega_t[i]))
 * in fp32 as they load each tile and then run the recurrence of rwkv_wkv6_forward_bf16.
 * Passing omega_t saves the caller a separate elementwise pass over [B, T, H, N], and a decay
 * close to 1 keeps its distance from 1: a bf16 w cannot hold one (the largest bf16 value
 * below 1 is 1 - 2^-8), so slowly decaying channels of a bf16 w round to w = 1 or to
 * 1 - 2^-8.  Any omega, +-inf included, gives w in [0, 1]; NaN is outside the contract.
 *   omega         : [B, T, H, N] bf16 (in place of w).
 *   g, ln_w, ln_b : all NULL = plain output (as rwkv_wkv6_forward_bf16);  all non-NULL =
 *                   the fused head LayerNorm + SiLU gate of rwkv_wkv6_forward_gated_bf16,
 *                   with eps as there.  Some but not all NULL: RWKV_ERR_NULL.  eps is
 *                   ignored without the gate.
 * Kernels, the rwkv_set_wkv6_algo choice (plain output only), layouts, aliasing rules and
 * errors are those of rwkv_wkv6_forward_bf16 / rwkv_wkv6_forward_gated_bf16.  The chunked
 * kernel forms w_t with the hardware's approximate base-2 exponential (relative error of
 * order 1e-7 on w_t); the serial and decode kernels with the accurate one. */
int rwkv_wkv6_forward_omega_bf16(int64_t B, int64_t T, int64_t H, int64_t N,
                                 const uint16_t *r, const uint16_t *k, const uint16_t *v,
                                 const uint16_t *omega, const float *u, const float *s0,
                                 const uint16_t *g, const float *ln_w, const float *ln_b, float eps,
                                 uint16_t *y, float *sT);

/* WKV-6 backward pass, for training ([E412], [F422]; the gradients of the recurrence of
 * rwkv_wkv6_forward by the chain rule, walked backwards in time).  Given the gradients of a
 * loss L with respect to the forward's outputs,
 *   dy  = dL/dy  [B, T, H, N] (dtype of r),   dsT = dL/dsT [B, H, N, N] fp32 (NULL = 0),
 * it writes, all fp32:
 *   dr, dk, dv, dw : [B, T, H, N]   dL/dr, dL/dk, dL/dv, dL/dw per token and channel
 *                    (rwkv_wkv6_backward_omega_bf16: domega = dL/domega_t in place of dw);
 *   du             : [H, N]         dL/du, summed over the batch rows in a fixed order
 *                                   (deterministic);
 *   ds0            : [B, H, N, N]   dL/ds0, or NULL = not written.  ds0 may be the very
 *                                   same array as dsT (in place).
 * With L_t = dL/d(state after token t), L_{T-1} = dsT and S = the state before token t:
 *   dr_t[i] = sum_j dy_t[j] (S[i][j] + u[i] k_t[i] v_t[j])
 *   dk_t[i] = sum_j L_t[i][j] v_t[j] + u[i] r_t[i] (dy_t . v_t)
 *   dv_t[j] = sum_i L_t[i][j] k_t[i] + (sum_i r_t[i] u[i] k_t[i]) dy_t[j]
 *   dw_t[i] = sum_j L_t[i][j] S[i][j]           domega_t[i] = -dw_t[i] exp(omega_t[i]) w_t[i]
 *   du[i]   = sum_{b,t} r_t[i] k_t[i] (dy_t . v_t)
 *   L_{t-1} = diag(w_t) L_t + r_t^T dy_t,       ds0 = L_{-1}.
 * Inputs r, k, v, w (or omega), u, s0 are those of the forward call; the forward states
 * are recomputed, not read.
 *   workspace : device scratch owned by the caller, 16-byte aligned, of at least the size
 *               rwkv_wkv6_backward_workspace_bytes reports (about B*H*ceil(T/8)*N*N*4 bytes:
 *               room for an fp32 checkpoint of the state every 8 tokens, which the exact
 *               walks below use; the chunked path needs about an eighth of it); it must not
 *               overlap any tensor.  A smaller workspace_bytes is refused with RWKV_ERR_ARG
 *               before any launch.  Its contents need no initialisation and are undefined
 *               after the call.
 * Two paths (rwkv_set_wkv6_algo on the calling thread chooses):
 *   - bf16 inputs (default, and RWKV_WKV6_AUTO / RWKV_WKV6_CHUNKED): the chunked tensor-core
 *     path in 64-token chunks -- a pass over the chunks for the state entering each chunk
 *     (kept in bf16), a reverse pass for the state gradient leaving each chunk, and one
 *     kernel over all (b, h, chunk) at once for the gradients, with bf16 MMA operands and
 *     fp32 accumulation (results within the bf16 tolerance of the exact gradient).  A (b, h)
 *     sequence with a channel whose 64-token decay product falls below 2^-100, or (w input)
 *     with a w below 2^-5, is served by the exact walks instead, inside the same call.
 *   - fp32 inputs, or RWKV_WKV6_SERIAL: the exact walks on CUDA cores in fp32 (a forward
 *     pass for dr, du and the checkpoints; a backward pass over state rows for dk, dw; one
 *     over state columns for dv, ds0).
 * du is summed over the batch rows (and chunks) in a fixed order: results are deterministic.
 * N must be 64.  T = 0 writes du = 0 and ds0 = dsT.  Aliasing: no output may overlap an
 * input, the workspace or another output (except ds0 == dsT).  Other rules and errors as
 * rwkv_wkv6_forward. */
int rwkv_wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N, size_t *bytes);
int rwkv_wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t N,
                       const float *r, const float *k, const float *v, const float *w,
                       const float *u, const float *s0, const float *dy, const float *dsT,
                       float *dr, float *dk, float *dv, float *dw, float *du, float *ds0,
                       void *workspace, size_t workspace_bytes);
int rwkv_wkv6_backward_bf16(int64_t B, int64_t T, int64_t H, int64_t N,
                            const uint16_t *r, const uint16_t *k, const uint16_t *v,
                            const uint16_t *w, const float *u, const float *s0,
                            const uint16_t *dy, const float *dsT,
                            float *dr, float *dk, float *dv, float *dw, float *du, float *ds0,
                            void *workspace, size_t workspace_bytes);
int rwkv_wkv6_backward_omega_bf16(int64_t B, int64_t T, int64_t H, int64_t N,
                                  const uint16_t *r, const uint16_t *k, const uint16_t *v,
                                  const uint16_t *omega, const float *u, const float *s0,
                                  const uint16_t *dy, const float *dsT,
                                  float *dr, float *dk, float *dv, float *domega, float *du,
                                  float *ds0, void *workspace, size_t workspace_bytes);

/* Kernel choice for WKV-6 on the calling thread: RWKV_WKV6_AUTO (default, as above),
 * RWKV_WKV6_SERIAL (always the serial kernel; the backward takes the exact fp32 walks),
 * RWKV_WKV6_CHUNKED (the chunked kernel for bf16 whatever T; ignored for fp32).  Returns
 * RWKV_OK or RWKV_ERR_ARG. */
#define RWKV_WKV6_AUTO 0
#define RWKV_WKV6_SERIAL 1
#define RWKV_WKV6_CHUNKED 2
int rwkv_set_wkv6_algo(int algo);
int rwkv_get_wkv6_algo(void);

/* Sequence split of the chunked WKV-6 kernel on the calling thread.  Each (b, h) sequence
 * is walked by one CTA; when there are fewer sequences than two per SM the library cuts
 * every sequence into G segments (of at least four 64-token chunks) that run side by
 * side: a first pass gives the end state (from zero) and decay product of P pieces of each
 * segment but the last (P = 1, 2, 4 ...: halves while the pieces keep at least four chunks
 * and the first pass fits on the GPU at once), and each segment then starts from its exact
 * incoming state.  The result equals the unsplit evaluation up to fp32 rounding order.  The
 * split needs B*H*(G-1)*P*(N*N+N)*4 bytes of scratch, plus B*H*N*N*4 bytes for a copy of s0
 * when the state is updated in place
 * (sT == s0: the copy is taken before any segment runs, so no segment can read an s0 that
 * the last segment has already overwritten).  The scratch is taken stream-ordered (on the
 * calling thread's stream, within the call) from a memory pool the library keeps per
 * device, which holds up to 64 MB between calls.
 *   segments = 0 (default): choose G;  1: never split;  n >= 2: split into at most n.
 * Returns RWKV_OK or RWKV_ERR_ARG. */
int rwkv_set_wkv6_segments(int segments);
int rwkv_get_wkv6_segments(void);

/* Allocation-free variant of rwkv_wkv6_forward_bf16 (the paper has no counterpart: it is
 * a service of this library).  Some callers may not allocate device memory at all -- a
 * serving process that has handed its whole HBM budget to its own pool, code that must
 * not touch the allocator while other work is in flight, or a runtime that forbids
 * allocation outside its own set-up phase.  For them this call runs the chunked kernel with
 * the same sequence split as the default entry point, but keeps the split's scratch in a
 * fixed array inside the library (RWKV_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU
 * that loads the library until the process exits) and never allocates or frees memory.
 *   segments: 0 = choose the split as rwkv_wkv6_forward_bf16 does, capped to what the
 *             array holds; n >= 1 = split into at most n segments.  The first pass uses
 *             P pieces per segment as the default entry point does, fewer (down to 1) when
 *             their entries would not fit.  A split needing more than
 *             RWKV_NOALLOC_SCRATCH_BYTES (B*H*(G-1)*P*(N*N+N)*4 bytes for G segments,
 *             plus B*H*N*N*4 bytes for the copy of s0 when sT == s0) is rejected with
 *             RWKV_ERR_SHAPE before any launch; rwkv_last_error() says why.
 * Arguments, layouts and the result are otherwise those of rwkv_wkv6_forward_bf16 (always
 * the chunked kernel, whatever T).
 *   - The first call on each device looks up the array's device address (a CUDA runtime
 *     query, no allocation); make that first call before capturing a stream into a graph.
 *   - Every call shares the one array and it keeps what the last call left; the kernels
 *     write every scratch entry before reading it, so nothing has to be cleared.  Calls
 *     whose GPU work overlaps (different streams, or host threads without ordering) race
 *     on the array: order them on one stream. */
#define RWKV_NOALLOC_SCRATCH_BYTES (4u << 20)
int rwkv_wkv6_forward_bf16_noalloc(int64_t B, int64_t T, int64_t H, int64_t N,
                                   const uint16_t *r, const uint16_t *k, const uint16_t *v,
                                   const uint16_t *w, const float *u, const float *s0,
                                   uint16_t *y, float *sT, int segments);

/* Test hook for the failure path (process-wide).  While enabled, every chunked WKV-6
 * launch first waits on a barrier that nothing signals, with a short bound; the wait
 * runs out, the kernel records RWKV_ERR_TIMEOUT in the device status word, releases its
 * resources and returns without computing (outputs are then unspecified).  No fault or
 * hang is involved.  Returns the previous setting. */
int rwkv_debug_inject_timeout(int enable);

/* ------------------------------------------------------------------ runtime plumbing */
/* Stream used by launches from the calling thread (a cudaStream_t; NULL = legacy
 * default stream).  Thread-local; the caller keeps the stream alive. */
void rwkv_set_stream(void *cuda_stream);
void *rwkv_get_stream(void);

/* Synchronises the calling thread's stream, then returns and clears the device status
 * word of the current device: RWKV_OK, or the first error a kernel recorded since the
 * last call (e.g. RWKV_ERR_TIMEOUT).  Returns RWKV_ERR_CUDA if the synchronisation
 * itself fails. */
int rwkv_get_device_status(void);

/* Static description of a status code. */
const char *rwkv_status_string(int status);

/* Thread-local text of the last failing call's error ("" if none). */
const char *rwkv_last_error(void);

/* RWKV_ABI_VERSION of the loaded library. */
int rwkv_abi_version(void);

/* 1 if the loaded library is the bounds-checked debug build (compiled with
 * WKV_DEBUG_BOUNDS), else 0.  In that build every kernel checks its global, shared-memory and
 * tensor-memory indices and TMA coordinates; a failed check skips the access and records
 * RWKV_ERR_BOUNDS in the device status word (rwkv_get_device_status) -- nothing traps.  It
 * is meant for tests on new shapes; it runs slower. */
int rwkv_debug_bounds(void);

#ifdef __cplusplus
}
#endif

#endif /* RWKV_WKV_H */
