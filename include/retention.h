/*
 * retention.h -- C ABI of libretention, the B200 (sm_100a) implementation of the
 * retention contraction of Multi-Scale Retention (RetNet).
 *
 * The operation (page "Retentive Networks -- Microsoft Propone l'Alternativa
 * Architetturale ai Transformer", aimpact.prandi.net, section "Il meccanismo:
 * Multi-Scale Retention"), per batch row b and head h with decay gamma_h:
 *
 *     y_n = sum_{m <= n} gamma_h^(n-m) (q_n . k_m) v_m  +  gamma_h^(n+1) q_n S_in
 *
 * computed in three equivalent forms named by the same section: parallel
 * (the whole decayed score matrix at once), chunkwise (blocks of length C:
 * parallel inside a block, recurrence between blocks) and recurrent
 * (S_n = gamma S_{n-1} + k_n^T v_n, y_n = q_n S_n; one token per call).
 * gamma^0 is taken as 1, also for gamma = 0.  There is no normalisation and no
 * denominator (author responses on paperhub.cn, "Retentive Network: A
 * Successor to Transformer ...", reply comparing Eq. (1) with RFA-Gate).
 *
 * Layouts (all row-major and contiguous, element = the call's dtype unless
 * stated):
 *     q, k   [B][H][L][dk]          v, y   [B][H][L][dv]
 *     state  [B][H][dk][dv]  always fp32 (the "h x d" state shape from the
 *                            paperhub.cn author responses, reply on inference cost)
 *     gamma  [H]             HOST array of fp32, each finite and in [0, 1]
 * Ownership: the caller owns every buffer.  q, k, v, y, state and workspace are
 * DEVICE pointers (from cudaMalloc, torch, ...); gamma is a HOST pointer read
 * during the call.  Every call is asynchronous on `stream` (a cudaStream_t;
 * NULL = legacy default stream) and allocates nothing.
 *
 * Precision: RET_BF16 runs the tensor-core path (bf16 operands, fp32
 * accumulation, fp32 state, y rounded to bf16).  RET_F32 runs fp32 CUDA-core
 * kernels (fp32 throughout).
 *
 * Errors: every argument is validated before anything is launched; a call that
 * returns anything but RET_OK has launched nothing.  RET_EUNSUPPORTED marks a
 * shape/dtype combination this library does not implement (there is no
 * fallback).  Kernels never trap: a wait that runs out of time sets a device
 * status word instead, read with retention_get_device_status().
 */
#ifndef RETENTION_H
#define RETENTION_H

#include <stddef.h>

#if defined(__GNUC__)
#define RET_API __attribute__((visibility("default")))
#else
#define RET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RET_OK = 0,
  RET_EINVAL = 1,        /* null pointer, bad size, gamma outside [0,1], misalignment */
  RET_EUNSUPPORTED = 2,  /* valid request that this library does not implement */
  RET_ECUDA = 3,         /* a CUDA runtime call failed (launch, attribute, copy) */
  RET_ETIMEOUT = 4,      /* a kernel's bounded wait expired (device status) */
  RET_EBOUNDS = 5        /* bounds-checked builds only (-DRET_BOUNDS_CHECK): an index
                            check in a kernel failed and its access was skipped */
} ret_status;

typedef enum { RET_F32 = 0, RET_BF16 = 1 } ret_dtype;

/* L is ignored by retention_recurrent_step (one token per call). */
typedef struct {
  int B, H, L, dk, dv;
} ret_shape;

/* Largest head count one call accepts (per-head decay travels in the launch). */
#define RET_MAX_HEADS 1024

/*
 * Parallel form: y = (Q K^T (.) D) V per (b, h), D[n][m] = gamma_h^(n-m) for
 * m <= n and 0 above the diagonal.  Same page and section, "forma parallela";
 * it is Eq. (5) / Fig. 2a in the paperhub.cn author responses (reply on why the
 * two forms of Fig. 2 are equivalent).  No state in or out.
 * Supported: RET_F32 with dk <= 256; RET_BF16 with dk in {64, 128, 256} and
 * dv a multiple of 64.  Pointers must be 16-byte aligned.
 */
RET_API ret_status retention_parallel(const void* q, const void* k, const void* v, const float* gamma,
                              void* y, ret_shape s, ret_dtype dt, void* stream);

/*
 * Chunkwise form with block length `chunk` (C): inside a block of length l
 * (C, or the remainder for the last block) starting at t0, for i < l,
 *     y_{t0+i} = sum_{j<=i} gamma^(i-j) (q_i . k_j) v_j + gamma^(i+1) q_i S_prev
 *     S_new    = gamma^l S_prev + sum_{j<l} gamma^(l-1-j) k_j^T v_j
 * (same page and section, "forma chunkwise"; the equations are the split of the
 * definition's sum at each block start).
 * state_in  : device fp32 [B][H][dk][dv], or NULL for a zero initial state.
 * state_out : device fp32, or NULL; receives S after the last token.  It may be
 *             the same buffer as state_in (in-place carry between calls).
 * workspace : optional device scratch of workspace_bytes bytes (>= 256-byte
 *             aligned).  With enough of it (see the query below) the sequence is
 *             also split across CTAs for parallelism; with less, or NULL, the
 *             call still runs, with fewer CTAs.  Results do not depend on it
 *             beyond fp32 rounding.
 * Supported: RET_F32 with 1 <= chunk <= 128, dk <= 256; RET_BF16 with dk in
 * {64, 128, 256}, dv a multiple of 128 and chunk a multiple of 16 in
 * [16, 128], or in [16, 256] when dk <= 128.
 */
RET_API ret_status retention_chunkwise(const void* q, const void* k, const void* v, const float* gamma,
                               void* y, const float* state_in, float* state_out, int chunk,
                               ret_shape s, ret_dtype dt, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Workspace size that lets retention_chunkwise use its full sequence split for
 * this shape (0 when the shape needs none). */
RET_API size_t retention_chunkwise_workspace_bytes(int chunk, ret_shape s, ret_dtype dt);

/*
 * One recurrent (decode) step, in place on the state:
 *     S <- gamma_h S + k^T v ;  y = q S        (same page and section, "forma ricorrente")
 * q, k [B][H][1][dk], v, y [B][H][1][dv] in the call's dtype; state fp32
 * [B][H][dk][dv], read and written in place.  Supported for both dtypes with
 * dk <= 1024; state must be 16-byte aligned.
 */
RET_API ret_status retention_recurrent_step(const void* q, const void* k, const void* v,
                                    const float* gamma, void* y, float* state, ret_shape s,
                                    ret_dtype dt, void* stream);

/*
 * Chunkwise form for callers that cannot allocate device memory -- for
 * example code that must not touch the allocator while a CUDA graph is being
 * captured, runtimes that fix every device buffer at start-up, or plugin hosts
 * that own all device memory.  Same arguments and results as
 * retention_chunkwise, without the workspace pair: the scratch for the
 * sequence split comes from a fixed 16 MiB array inside this library's device
 * memory, held on every GPU that loads the library until the process exits.  The pages have no counterpart; this
 * is a property of the library, not of the method.
 *   - Shapes whose split needs more scratch than the array holds
 *     (retention_chunkwise_workspace_bytes() > 16 MiB) return
 *     RET_EUNSUPPORTED before anything is launched; shapes that need no split
 *     never touch the array.
 *   - The first call on a device, whatever its shape, looks up the array's
 *     device address (once per device, with that device current); make that
 *     first call before any stream capture.
 *   - Every call uses the same array and leaves its contents behind.  Nothing
 *     in it has to start at zero (each call writes every slot it reads), but
 *     calls that can run at the same time on the GPU -- different streams, or
 *     different host threads -- race on it: serialise them.
 *   - No cudaMalloc, cudaFree or other allocating call is made.
 */
RET_API ret_status retention_chunkwise_static_ws(const void* q, const void* k, const void* v,
                                                 const float* gamma, void* y, const float* state_in,
                                                 float* state_out, int chunk, ret_shape s,
                                                 ret_dtype dt, void* stream);

/*
 * The state_out of retention_chunkwise without y: for the L tokens of the call,
 *     state_out = gamma^L state_in + sum_t gamma^(L-1-t) k_t^T v_t
 * (the recurrence of the page "Retentive Networks -- Microsoft ...", section
 * "Il meccanismo", unrolled over the call).  It reads only k and v, so it costs
 * about a third of the full call.  Uses: a prompt whose outputs are not needed
 * before decoding, and the first pass of a sequence cut across GPUs (each
 * rank's run summed from a zero state, then retention_state_fold).
 * k : device [B][H][L][dk], v : device [B][H][L][dv], the call's dtype, 16-byte
 *     aligned.  state_in : device fp32 [B][H][dk][dv] or NULL (zero).
 * state_out : device fp32 [B][H][dk][dv], required; may alias state_in.
 * bf16: shapes and chunks of the tensor-core chunkwise path; workspace of
 *     retention_chunkwise_state_workspace_bytes() bytes (256-byte aligned), at
 *     least two states per (b, h): the run is cut into segments summed in
 *     parallel, fewer when the workspace is smaller.  fp32: as retention_chunkwise
 *     (no workspace).
 * L = 0 copies state_in (or zeros) to state_out.
 */
RET_API ret_status retention_chunkwise_state(const void* k, const void* v, const float* gamma,
                                             const float* state_in, float* state_out, int chunk, ret_shape s,
                                             ret_dtype dt, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace size of retention_chunkwise_state (0 for fp32 or L = 0). */
RET_API size_t retention_chunkwise_state_workspace_bytes(int chunk, ret_shape s, ret_dtype dt);

/*
 * The state at the end of consecutive runs of tokens, from each run's own sum:
 * with D_i the state of run i from a zero state (retention_chunkwise_state) and
 * len_i its length,
 *     S = state_in;  for i = 0 .. n-1:  S = gamma^len_i S + D_i;  state_out = S.
 * The same page and section: the state after a run is the decayed state before
 * it plus the run's own sum.  On a sequence cut across ranks, rank r folds the
 * parts of ranks 0 .. r-1 to get the state its own run starts from.
 * parts : device fp32 [n][B][H][dk][dv] (the D_i), 16-byte aligned; a
 *         state_out that overlaps them is RET_EINVAL.
 * lens  : host int [n], each >= 0.  n in [0, 256].
 * state_in : device fp32 [B][H][dk][dv] or NULL (zero); state_out : device fp32,
 *         may alias state_in.  s.L is ignored.  Runs on `stream`.
 */
RET_API ret_status retention_state_fold(const float* parts, const int* lens, int n, const float* gamma,
                                        const float* state_in, float* state_out, ret_shape s, void* stream);

/*
 * Chunkwise form on host buffers: q, k, v are copied from host memory, the
 * chunkwise form runs on the device, and y is copied back to host memory, all
 * inside this call's work on `stream` (the same results as
 * retention_chunkwise on device copies of the inputs).  The (b, h) rows are
 * processed in groups of consecutive heads of one batch row.  Each group's
 * host-to-device copy, its kernels and its device-to-host copy run on
 * separate streams, ordered by events, so the two copy directions and the
 * kernels of different groups overlap.  This is a property of the library, not
 * of the method.
 * q_host, k_host, v_host, y_host : host buffers, [B][H][L][d] in the call's
 *             dtype; page-locked memory lets the copies run asynchronously.
 *             They must stay valid, and y_host unread, until `stream` completes.
 * q_dev, k_dev, v_dev, y_dev : device buffers of the same sizes, owned by the
 *             caller (the library allocates no device memory).
 * state_in, state_out, chunk, workspace : as for retention_chunkwise (device
 *             pointers; the workspace serves one group at a time, see the query
 *             below).
 * n_groups  : requested number of groups (<= 0: 8).  Groups never span batch
 *             rows, so the call may use more.
 * The copy streams and events are created on first use on each device and
 * kept until the process exits.  Returns before the work completes; errors in
 * the arguments are reported before anything is enqueued.
 */
RET_API ret_status retention_chunkwise_host(const void* q_host, const void* k_host, const void* v_host,
                                            const float* gamma, void* y_host, void* q_dev, void* k_dev,
                                            void* v_dev, void* y_dev, const float* state_in, float* state_out,
                                            int chunk, ret_shape s, ret_dtype dt, void* workspace,
                                            size_t workspace_bytes, int n_groups, void* stream);

/* Workspace size that lets every group of retention_chunkwise_host use its full
 * sequence split. */
RET_API size_t retention_chunkwise_host_workspace_bytes(int chunk, ret_shape s, ret_dtype dt, int n_groups);

/*
 * Per-head group normalisation of a retention output (the layer that follows
 * the contraction; author responses on paperhub.cn, "Retentive Network: A
 * Successor to Transformer for Large Language Models", reply on GroupNorm vs
 * LayerNorm: one group per head, since heads carry different statistics).
 * For each (b, h, n) the dv values of y_n form one group:
 *     out_c = (y_c - mean) / sqrt(var + eps) * weight[h*dv + c] + bias[h*dv + c]
 * with the biased variance (the page gives no formula, eps or affine; these
 * are the readings taken).
 * y, out   : device [B][H][L][dv] in the call's dtype (s.dk is ignored); out may
 *            be y.  16-byte aligned when dv % 128 == 0.
 * weight, bias : device fp32 [H*dv], or NULL for 1 and 0.
 * eps      : finite, >= 0.  Supported: dv <= 1024.
 */
RET_API ret_status retention_groupnorm(const void* y, void* out, float eps, const float* weight,
                                       const float* bias, ret_shape s, ret_dtype dt, void* stream);

/* Activations of the output gate. */
typedef enum { RET_GATE_NONE = 0, RET_GATE_SWISH = 1, RET_GATE_SIGMOID = 2 } ret_gate_act;

/*
 * retention_groupnorm followed by the output gate of gated multi-scale
 * retention (named next to GroupNorm in the same author responses, reply on
 * the "transformer without softmax" remark, with no formula).  Reading taken:
 *     out_c = GroupNorm(y)_c * act(gate_c)
 * with act(x) = x (RET_GATE_NONE), x / (1 + e^-x) (RET_GATE_SWISH) or
 * 1 / (1 + e^-x) (RET_GATE_SIGMOID), in one pass over y and gate.
 * gate : device [B][H][L][dv] in the call's dtype (the gate input, e.g. the
 *        caller's projection of the layer input), or NULL for no gate; same
 *        alignment rule as y.  out may be y (not gate).
 * act  : a ret_gate_act; anything else is RET_EINVAL.
 * Other arguments and limits as retention_groupnorm.
 */
RET_API ret_status retention_groupnorm_gated(const void* y, const void* gate, void* out, float eps,
                                             const float* weight, const float* bias, int act, ret_shape s,
                                             ret_dtype dt, void* stream);

/*
 * Chunkwise form followed by retention_groupnorm on its output, in place: y
 * receives the normalised output.  The other arguments are as for
 * retention_chunkwise.  With bf16, dv = 128 (one head = one 128-column slice),
 * dk <= 128, chunk <= 128 and weight and bias 16-byte aligned (or NULL) the
 * chunkwise kernel normalises each row in its epilogue, before y is stored
 * (one launch, no extra pass over y); otherwise the normalisation runs as a
 * second kernel on the stream.
 */
RET_API ret_status retention_chunkwise_gn(const void* q, const void* k, const void* v, const float* gamma,
                                          void* y, const float* state_in, float* state_out, int chunk,
                                          ret_shape s, ret_dtype dt, float eps, const float* weight,
                                          const float* bias, void* workspace, size_t workspace_bytes,
                                          void* stream);

/* Workspace size for retention_chunkwise_gn (that of the chunkwise call). */
RET_API size_t retention_chunkwise_gn_workspace_bytes(int chunk, ret_shape s, ret_dtype dt);

/*
 * retention_chunkwise_gn with the output gate: y receives
 * GroupNorm(y) * act(gate) (see retention_groupnorm_gated), in place; with a
 * gate the normalisation and gate always run as a second kernel.  gate:
 * device [B][H][L][dv] in the call's dtype, 16-byte aligned, sharing no byte
 * with y (RET_EINVAL otherwise: y is normalised in place while the gate is
 * read); NULL for no gate.  act: a ret_gate_act.  Workspace:
 * retention_chunkwise_gn_workspace_bytes().
 */
RET_API ret_status retention_chunkwise_gn_gated(const void* q, const void* k, const void* v, const float* gamma,
                                                void* y, const float* state_in, float* state_out, int chunk,
                                                ret_shape s, ret_dtype dt, float eps, const float* weight,
                                                const float* bias, const void* gate, int act, void* workspace,
                                                size_t workspace_bytes, void* stream);

/*
 * Backward pass of retention_parallel: for the upstream gradient dy of
 * y = retention_parallel(q, k, v), writes
 *     dq_n = sum_{m<=n} gamma^(n-m) (dy_n . v_m) k_m
 *     dk_m = sum_{n>=m} gamma^(n-m) (dy_n . v_m) q_n
 *     dv_m = sum_{n>=m} gamma^(n-m) (q_n . k_m) dy_n
 * (the derivative of the retention sum of the page "Retentive Networks --
 * Microsoft ...", section "Il meccanismo"; the pages give no backward pass).
 * Each is a retention sum itself: dq on (dy, v, k), and dk, dv the
 * anti-causal sums (n >= m) on (v, dy, q) and (k, q, dy), which the kernels
 * walk from the end of the sequence; the call runs three parallel-form
 * launches on `stream` and copies nothing.
 * q, k, dq, dk : device [B][H][L][dk]; v, dy, dv : device [B][H][L][dv]; all in
 *             the call's dtype, 16-byte aligned.
 * workspace : not used (retention_parallel_backward_workspace_bytes() is 0);
 *             NULL is accepted.
 * Supported: bf16 with dk and dv in {64, 128, 256}; fp32 with dk, dv <= 256.
 */
RET_API ret_status retention_parallel_backward(const void* q, const void* k, const void* v, const float* gamma,
                                               const void* dy, void* dq, void* dk, void* dv, ret_shape s,
                                               ret_dtype dt, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace size of retention_parallel_backward: 0 (kept for callers that size
 * a workspace before the call). */
RET_API size_t retention_parallel_backward_workspace_bytes(ret_shape s, ret_dtype dt);

/*
 * The same gradients through the chunkwise form (blocks of `chunk`, zero
 * initial state): the three retention sums of retention_parallel_backward
 * computed by retention_chunkwise, so the cost grows linearly with L.  No
 * state gradient: the forward call it differentiates starts from a zero state
 * and its state_out is not used.
 * dk and dv are the anti-causal sums, walked from the end of the sequence
 * (their blocks are of min(chunk, 128) rows; the result does not depend on the
 * block length beyond rounding).  Nothing is copied.
 * Supported: bf16 with dk and dv in {128, 256} (each is the value width of one
 * of the three calls) and a chunk the chunkwise path takes for both; fp32 with
 * dk, dv <= 256 and chunk <= 128.  Workspace: the chunkwise calls'
 * sequence-split scratch, retention_chunkwise_backward_workspace_bytes() bytes
 * (0 when no call splits; NULL is then accepted), 256-byte aligned.
 */
RET_API ret_status retention_chunkwise_backward(const void* q, const void* k, const void* v, const float* gamma,
                                                const void* dy, void* dq, void* dk, void* dv, int chunk, ret_shape s,
                                                ret_dtype dt, void* workspace, size_t workspace_bytes,
                                                void* stream);

/* Workspace size of retention_chunkwise_backward. */
RET_API size_t retention_chunkwise_backward_workspace_bytes(int chunk, ret_shape s, ret_dtype dt);

/*
 * Backward pass of a retention_chunkwise call that carries a state: the
 * gradients of y and state_out with respect to q, k, v and state_in.  With
 * state_in S0 the forward gives y_n += gamma^(n+1) q_n S0 and
 * state_out = gamma^L S0 + sum_m gamma^(L-1-m) k_m^T v_m (the recurrence of
 * the page "Retentive Networks -- Microsoft ...", section "Il meccanismo",
 * started from S0), so for upstream gradients dy and dS_out this call adds to
 * the sums of retention_chunkwise_backward
 *     dq_n += gamma^(n+1) dy_n S0^T
 *     dk_m += gamma^(L-1-m) v_m dS_out^T,   dv_m += gamma^(L-1-m) k_m dS_out
 * and writes dS0 = gamma^L dS_out + sum_n gamma^(n+1) q_n^T dy_n.  Each extra
 * term is the initial-state term of one of the three chunkwise sums, so the
 * cost is that of retention_chunkwise_backward plus a transpose of the states.
 * state_in   : device fp32 [B][H][dk][dv] the forward call started from, or
 *              NULL (zero state).
 * dstate_out : device fp32 [B][H][dk][dv] gradient of state_out, or NULL
 *              (state_out unused).
 * dstate_in  : device fp32 [B][H][dk][dv] receives dS0, or NULL (not wanted).
 *              May alias state_in or dstate_out (both are consumed first), so a
 *              caller walking a long sequence backwards call by call can keep
 *              one state-gradient buffer.
 * All three 16-byte aligned.  With L = 0 the call writes dS0 = dS_out (zero
 * when dstate_out is NULL) and nothing else.
 * Heads with gamma below 2^-60 drop the dS_out terms of rows m < L-1 of dk and
 * dv, whose factor gamma^(L-1-m) is below 2^-60; every other term is kept.
 * Supported shapes, dtypes and chunks: those of retention_chunkwise_backward.
 * workspace : retention_chunkwise_backward_state_workspace_bytes() bytes,
 *             256-byte aligned (that of retention_chunkwise_backward plus
 *             three fp32 states, needed when any state pointer is given).
 */
RET_API ret_status retention_chunkwise_backward_state(const void* q, const void* k, const void* v,
                                                      const float* gamma, const void* dy, const float* state_in,
                                                      const float* dstate_out, void* dq, void* dk, void* dv,
                                                      float* dstate_in, int chunk, ret_shape s, ret_dtype dt,
                                                      void* workspace, size_t workspace_bytes, void* stream);

/* Workspace size of retention_chunkwise_backward_state (any state pointer given). */
RET_API size_t retention_chunkwise_backward_state_workspace_bytes(int chunk, ret_shape s, ret_dtype dt);

/* Synchronises `stream`, then returns and clears the device status word:
 * RET_OK, RET_ETIMEOUT if a kernel's bounded wait expired since the last
 * query, RET_EBOUNDS if a bounds-checked build found an index out of range,
 * or RET_ECUDA if the stream reported an error. */
RET_API ret_status retention_get_device_status(void* stream);

/* Static, NUL-terminated name of a status code. */
RET_API const char* retention_status_str(ret_status st);

/* ABI version of this header (major * 100 + minor). */
RET_API int retention_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RETENTION_H */
