/*
 * mlstm.h -- C ABI of the chunkwise-parallel (TFLA) mLSTM forward and backward
 * kernels for NVIDIA B200 (sm_100a).
 *
 * What is computed.  "Tiled Flash Linear Attention: More Efficient Linear RNN
 * and xLSTM Kernels" (TFLA summary page, sections Problem and Approach; arXiv
 * abstract page, Abstract) describes the mLSTM, a gated linear RNN with a
 * matrix memory, in two variants: mLSTMexp (exponential input gate, normaliser
 * state n_t and max state m_t) and mLSTMsig (sigmoid input gate, no normaliser
 * and no max state).  Both use a sigmoid forget gate and scale q by
 * 1/sqrt(d_qk).  Per (batch, head), with C_0 = 0, n_0 = 0:
 *
 *   C_t = f_t C_{t-1} + i_t k_t v_t^T        n_t = f_t n_{t-1} + i_t k_t
 *   mLSTMsig: h_t = C_t^T q'_t
 *   mLSTMexp: h_t = C_t^T q'_t / max(|n_t . q'_t|, 1)        q'_t = q_t / sqrt(d_qk)
 *
 * with f_t = sigmoid(fgate_pre_t), and i_t = exp(igate_pre_t) (EXP) or
 * sigmoid(igate_pre_t) (SIG).  The pages print no formula; this is the plainest
 * reading of what they state.  The library evaluates it chunkwise, as the pages
 * describe: the sequence is split into chunks of `chunk` tokens, the state
 * entering each chunk is materialised in memory, and the outputs of all chunks
 * are computed in parallel with the intra-chunk matmuls tiled along the
 * sequence (the second level of TFLA), so the chunk size is not bounded by
 * shared memory.
 *
 * Layout.  Row-major, contiguous, head-major:
 *   q, k, dq, dk : [B, NH, T, d_qk]      v, h, dh, dv : [B, NH, T, d_hv]
 *   igate_pre, fgate_pre, digate_pre, dfgate_pre : [B, NH, T]
 * Every tensor uses the one I/O dtype (MLSTM_BF16 or MLSTM_FP32); arithmetic
 * is fp32 (bf16 tensor-core operands with fp32 accumulation on the bf16 path).
 * All pointers are device pointers, 16-byte aligned.
 *
 * Supported sizes.  B, NH >= 0; T >= 0 (T need not be a multiple of `chunk`:
 * the last chunk is then shorter); chunk a power of two in [64, 4096];
 * d_qk in {64, 128, 256}; d_hv in {64, 128, 256, 512}; B*NH*T < 2^31.
 * Other values return MLSTM_ERR_UNSUPPORTED.  B*NH*T == 0 is a no-op.
 *
 * Ownership.  The caller allocates every buffer.  The library never
 * allocates or frees device memory, never synchronises the stream and keeps
 * no per-call state; all work is enqueued on `stream` (a cudaStream_t passed
 * as void*, NULL = legacy default stream) and the call returns at once.
 *
 * Errors.  Argument errors are detected on the host before any launch and
 * return MLSTM_ERR_INVALID / MLSTM_ERR_UNSUPPORTED / MLSTM_ERR_WORKSPACE with
 * nothing enqueued.  A failed launch returns MLSTM_ERR_CUDA; an earlier sticky
 * CUDA error in the context is reported the same way and is not cleared.
 */
#ifndef MLSTM_H
#define MLSTM_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MLSTM_SIG = 0, MLSTM_EXP = 1 } mlstm_variant_t;
typedef enum { MLSTM_BF16 = 0, MLSTM_FP32 = 1 } mlstm_dtype_t;

typedef enum {
  MLSTM_OK = 0,
  MLSTM_ERR_INVALID = 1,      /* null pointer, negative size, bad enum       */
  MLSTM_ERR_UNSUPPORTED = 2,  /* valid but outside the supported sizes       */
  MLSTM_ERR_WORKSPACE = 3,    /* workspace / saved buffer too small          */
  MLSTM_ERR_CUDA = 4,         /* a CUDA launch or the context failed         */
  MLSTM_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up          */
} mlstm_status_t;

/* Regions of the `saved` buffer that mlstm_fwd fills and mlstm_bwd reads.
 * Offsets are in bytes from the start of the buffer, 256-byte aligned.
 * NC = ceil(T / chunk); BH = B * NH.  Regions absent for a variant have
 * size 0.
 *   gate_b   float [BH, T]    in-chunk inclusive cumulative sum of log f
 *   gate_li  float [BH, T]    log input gate (i~ for EXP, logsigmoid(i~) for SIG)
 *   gate_m   float [BH, T]    EXP: max state m_t of the recurrence
 *   norm     float [BH, T]    EXP: stabilised normaliser  n~_t . q'_t
 *   state_c  [BH, NC, d_qk, d_hv]  state entering each chunk (EXP: scaled
 *            by exp(-m) of the chunk's previous row).  fp32 path: one float
 *            plane.  bf16 path: two bf16 planes back to back, hi = bf16(C)
 *            then lo = bf16(C - hi), so hi + lo keeps about 16 mantissa bits
 *            for the backward pass
 *   state_n  float [BH, NC, d_qk]  EXP: normaliser state entering each chunk
 *   tile_table  float [BH, NC, 5 chunk + max(32, chunk / 32)]  bf16 with
 *            chunk >= 256 only: per-chunk gate factors of the large-chunk
 *            output kernel (row exponents, inter-chunk row factors, the
 *            normaliser floor exp(-m_t), key exponents, per-32-key column
 *            factors and their block maxima).  Forward scratch; the backward
 *            does not read it. */
typedef struct {
  size_t gate_b, gate_li, gate_m, norm, state_c, state_n, tile_table;
  size_t gate_b_bytes, gate_li_bytes, gate_m_bytes, norm_bytes, state_c_bytes, state_n_bytes,
      tile_table_bytes;
  size_t total;
} mlstm_saved_layout_t;

/* Fill *layout for the given problem.  Returns MLSTM_OK or an argument error. */
int mlstm_saved_layout(int B, int NH, int T, int d_qk, int d_hv, int chunk,
                       int variant, int dtype, mlstm_saved_layout_t* layout);

/* Bytes of the `saved` buffer (0 on an argument error). */
size_t mlstm_saved_size(int B, int NH, int T, int d_qk, int d_hv, int chunk,
                        int variant, int dtype);

/* Bytes of workspace mlstm_fwd needs when `saved` is NULL (the saved regions
 * then live in the workspace); with a non-NULL `saved` it needs none. */
size_t mlstm_fwd_workspace_size(int B, int NH, int T, int d_qk, int d_hv,
                                int chunk, int variant, int dtype);

/* Bytes of workspace mlstm_bwd needs (0 on an argument error). */
size_t mlstm_bwd_workspace_size(int B, int NH, int T, int d_qk, int d_hv,
                                int chunk, int variant, int dtype);

/* Forward pass.  Reads q, k, v, igate_pre, fgate_pre; writes h and, when
 * `saved` is non-NULL, the saved regions for mlstm_bwd (mlstm_saved_size
 * bytes).  `workspace` may be NULL when `saved` is non-NULL.  The steps are
 * those of the chunkwise form: gate preprocessing, the inter-chunk state
 * recurrence, then the tiled intra-chunk outputs fused with the inter-chunk
 * term q' C_prev and the normaliser (TFLA summary page, Approach; arXiv
 * abstract page, Abstract).  On the bf16 path with chunk 128 and d_qk = d_hv
 * = 128 the recurrence and the outputs run in one kernel that carries each
 * head's state through its chunks on chip; the saved regions are the same. */
int mlstm_fwd(const void* q, const void* k, const void* v,
              const void* igate_pre, const void* fgate_pre,
              void* h, void* saved,
              void* workspace, size_t workspace_bytes,
              int B, int NH, int T, int d_qk, int d_hv, int chunk,
              int variant, int dtype, void* stream);

/* Backward pass of sum(dh * h).  Reads q, k, v, the gate preactivations, the
 * forward output h, the upstream gradient dh and `saved` as filled by
 * mlstm_fwd on the same inputs (required, not NULL).  Writes dq, dk, dv and
 * the preactivation gradients digate_pre, dfgate_pre.  The timed training
 * kernels of the TFLA summary page (Key results) are this forward plus this
 * backward.  On the bf16 path with chunk 128 and d_qk = d_hv = 128 one kernel
 * runs on a high-priority stream of the calling thread, forked from `stream`
 * after the kernels before it and joined back before the last one, so that
 * dq can use the SMs it leaves idle; all work is ordered after what `stream`
 * held at the call and before what it receives later.  That stream and its two
 * events are created on the thread's first such call on a device (make it
 * before any stream capture) and kept until the process exits. */
int mlstm_bwd(const void* q, const void* k, const void* v,
              const void* igate_pre, const void* fgate_pre,
              const void* h, const void* dh, const void* saved,
              void* dq, void* dk, void* dv, void* digate_pre, void* dfgate_pre,
              void* workspace, size_t workspace_bytes,
              int B, int NH, int T, int d_qk, int d_hv, int chunk,
              int variant, int dtype, void* stream);

/* Allocation-free forward, for callers that cannot call cudaMalloc when they
 * run the op (a framework that owns every device allocation, a plugin behind
 * a custom allocator, a launch path where allocating would synchronise).  The
 * pages have no counterpart: this is a deployment convenience.  It computes
 * exactly what mlstm_fwd computes with saved == NULL, but its scratch (gate
 * sums, max states, chunk states) lives in a 32 MiB array compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  The caller passes the inputs and the output h, device pointers as
 * for mlstm_fwd.  Problems whose scratch (mlstm_fwd_workspace_size) exceeds
 * 32 MiB return MLSTM_ERR_WORKSPACE before any launch; no saved state is kept,
 * so there is no backward from this entry point.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) with that device
 * current.  Under CUDA's default lazy module loading, that lookup is what
 * places the 32 MiB array on the device, and the first launch of each kernel
 * loads that kernel's code; either may allocate device memory and synchronise.
 * So make one warm-up call with the same sizes, variant and dtype on each
 * device before any region that must not allocate and before any stream
 * capture.  After it, calls of that configuration allocate nothing: the entry
 * point calls no cudaMalloc, cudaFree or allocating library routine.  The
 * cached address is per device ordinal and is not refreshed after
 * cudaDeviceReset.  All calls share the one array, so calls whose
 * kernels overlap on the GPU (different streams, or different host threads)
 * race on it: serialise them. */
int mlstm_fwd_noalloc(const void* q, const void* k, const void* v,
                      const void* igate_pre, const void* fgate_pre, void* h,
                      int B, int NH, int T, int d_qk, int d_hv, int chunk,
                      int variant, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * Recurrent form: one token at a time, and the hand-off from a chunkwise
 * forward to it.  "flash-linear-attention" README, the FusedRecurrent form
 * (O(T), states on chip); "Tiled Flash Linear Attention", TFLA summary page,
 * Approach (the mLSTM recurrence, exponential or sigmoid input gate, sigmoid
 * forget gate, normaliser and max state for mLSTMexp).
 *
 * State buffer (device memory owned by the caller), per head, fp32, 256-byte
 * aligned regions of size mlstm_state_size():
 *   C [B*NH, d_qk, d_hv]  at offset 0; for EXP scaled by exp(-m)
 *   n [B*NH, d_qk]        EXP only, next 256-byte boundary after C
 *   m [B*NH]              EXP only, next 256-byte boundary after n
 * The zero state (no token seen) is C = 0, n = 0, m = -inf.
 * ------------------------------------------------------------------------- */

/* Bytes of a state buffer (0 on an argument error). */
size_t mlstm_state_size(int B, int NH, int d_qk, int d_hv, int variant);

/* Write the zero state into `state` (enqueued on `stream`).  Errors:
 * MLSTM_ERR_INVALID (NULL or misaligned state), MLSTM_ERR_UNSUPPORTED,
 * MLSTM_ERR_CUDA. */
int mlstm_state_zero(void* state, int B, int NH, int d_qk, int d_hv, int variant, void* stream);

/* State after the last token of a sequence that mlstm_fwd processed with
 * the same sizes, from its `saved` buffer (the state entering the last
 * chunk, gate cumsums and max states) and its k, v: C_T = beta C_enter +
 * sum_s w_s k_s v_s^T over the last chunk, n likewise, m_T the last max
 * state.  Writes `state` (layout above); reads k, v, saved.  T = 0 writes
 * the zero state.  Errors as mlstm_fwd. */
int mlstm_final_state(const void* k, const void* v, const void* saved, void* state,
                      int B, int NH, int T, int d_qk, int d_hv, int chunk,
                      int variant, int dtype, void* stream);

/* One token of the recurrence for every head.  q, k [B, NH, d_qk] and
 * v [B, NH, d_hv] in the I/O dtype; igate_pre, fgate_pre [B, NH] in the I/O
 * dtype; h [B, NH, d_hv] out in the I/O dtype.  Reads state_in, writes
 * state_out; the two must not overlap (MLSTM_ERR_INVALID), callers
 * alternate two buffers.
 *   SIG: C' = f C + i k v^T, h = C'^T q / sqrt(d_qk)
 *   EXP: m' = max(log f + m, i~), C' = exp(log f + m - m') C + exp(i~ - m') k v^T,
 *        n' likewise, h = C'^T q' / max(|n' . q'|, exp(-m'))
 * with f = sigmoid(f~), i = sigmoid(i~) (SIG).  Arithmetic in fp32.
 * Errors: MLSTM_ERR_INVALID (NULL, misaligned or overlapping buffers),
 * MLSTM_ERR_UNSUPPORTED (sizes outside the chunkwise path's), MLSTM_ERR_CUDA. */
int mlstm_step(const void* q, const void* k, const void* v, const void* igate_pre,
               const void* fgate_pre, void* h, const void* state_in, void* state_out,
               int B, int NH, int d_qk, int d_hv, int variant, int dtype, void* stream);

/* The chunkwise forward of a sequence that continues from a state, for
 * chaining calls (a long prompt in pieces, or a prompt after generated
 * tokens).  Same arguments, layouts, ownership and errors as mlstm_fwd, plus:
 *   state_in   the state before the first token (layout above), read; NULL:
 *              the zero state, which makes this call mlstm_fwd.
 *   state_out  the state after the last token, written; NULL: not wanted.
 * With the recurrence above started from state_in, h is the same as for the
 * whole sequence: inside, the state enters the first chunk like any chunk's
 * state (its C and n, and m as the first chunk's m_{c-1}), and state_out is
 * mlstm_final_state's result.  state_in and state_out must not overlap
 * (MLSTM_ERR_INVALID).  T = 0 copies state_in (or the zero state) to
 * state_out.  h may be NULL when state_out is not: the state-only pass (gate
 * preprocessing, chunk states and the final state, no output kernel).  The
 * saved buffer of such a call is for mlstm_bwd_state with the same state_in. */
int mlstm_fwd_state(const void* q, const void* k, const void* v, const void* igate_pre,
                    const void* fgate_pre, void* h, void* saved, void* workspace,
                    size_t workspace_bytes, const void* state_in, void* state_out, int B, int NH,
                    int T, int d_qk, int d_hv, int chunk, int variant, int dtype, void* stream);

/* The backward of mlstm_fwd_state, with the initial state held constant (its
 * max state m, like every max state, carries no gradient).  Same arguments,
 * layouts and errors as mlstm_bwd, plus:
 *   state_in   the state the forward started from (NULL: the zero state).
 *   dstate_in  gradient of the loss with respect to state_in's C and (EXP) n,
 *              written into those regions of a state-layout buffer (its m
 *              region is not written); NULL: not wanted.  It is one more step
 *              of the state-gradient recurrence: beta_0 dC_0 + Q_0^T diag(u)
 *              dH_0 over the first chunk.
 *   dstate_out gradient of the loss with respect to the final state's C and
 *              (EXP) n (state layout, read; its m region is ignored), for a loss
 *              that also reads state_out, e.g. through a later call's
 *              dstate_in; NULL: none.  It starts the state-gradient recurrence
 *              (the gradient of the state leaving the last chunk), gives dk and
 *              dv an inter-chunk term in the last chunk, and adds
 *              <dC_T, C_T> + <dn_T, n_T> to every forget-gate gradient (the
 *              final state reads every key before it); the final state is
 *              rebuilt from `saved` in the workspace.
 * dstate_in must not overlap state_in or dstate_out (MLSTM_ERR_INVALID).
 * With T = 0 the gradient with respect to the initial state is dstate_out.
 * dq, dk, dv, digate_pre and dfgate_pre may all be NULL when dstate_in is not:
 * the state-gradient-only pass (per-token normaliser terms and the state
 * recurrence, no intra-chunk or gate kernels). */
int mlstm_bwd_state(const void* q, const void* k, const void* v, const void* igate_pre,
                    const void* fgate_pre, const void* h, const void* dh, const void* saved,
                    const void* state_in, void* dstate_in, const void* dstate_out, void* dq,
                    void* dk, void* dv, void* digate_pre, void* dfgate_pre, void* workspace,
                    size_t workspace_bytes, int B, int NH, int T, int d_qk, int d_hv, int chunk,
                    int variant, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * Sequence segments.  A sequence split into consecutive segments (one per
 * GPU, say) is processed exactly by: the state-only pass of every segment from
 * the zero state (mlstm_fwd_state with h = NULL), each segment's total log
 * forget gate (mlstm_log_decay), an exchange of both, the state entering every
 * segment by chaining the earlier segments' states (mlstm_state_chain), and a
 * forward of every segment from that state.  "Tiled Flash Linear Attention",
 * TFLA summary page, Problem and Approach (states at chunk boundaries carry
 * everything a later chunk needs, so they can cross a device boundary too).
 * ------------------------------------------------------------------------- */

/* log_decay [B*NH] (fp32, written) = sum over the T tokens of
 * log sigmoid(fgate_pre) for every head; fgate_pre [B, NH, T] in the I/O
 * dtype.  T = 0 writes zeros.  Errors: MLSTM_ERR_INVALID (NULL or misaligned
 * pointer), MLSTM_ERR_UNSUPPORTED, MLSTM_ERR_CUDA. */
int mlstm_log_decay(const void* fgate_pre, float* log_decay, int B, int NH, int T, int dtype,
                    void* stream);

/* state_out = the state after segment b when b starts from state_a, given
 * state_b (b's final state from the zero state) and b's log_decay:
 * unstabilised, exp(G_b) (state a) + (state b); for mLSTMexp the stabilised
 * form with m = max(G_b + m_a, m_b) (the max-state recurrence unrolled over
 * the segment).  All three buffers in the state layout above, fp32;
 * state_out must not overlap state_a or state_b (MLSTM_ERR_INVALID). */
int mlstm_state_chain(const void* state_a, const void* state_b, const float* log_decay_b,
                      void* state_out, int B, int NH, int d_qk, int d_hv, int variant,
                      void* stream);

/* The backward of chained segments.  For segment b, given
 *   dstate_local  the gradient with respect to b's initial state from b's own
 *                 outputs (mlstm_bwd_state with dstate_in and the five
 *                 gradient outputs NULL: the state-gradient-only pass),
 *   dstate_out    the gradient with respect to b's final state,
 *   state_in, state_out  the states entering and leaving b (their m), and b's
 *                 log_decay,
 * dstate_in = dstate_local + f dstate_out with f = exp(G_b + m_in - m_out)
 * (exp(G_b) for mLSTMsig): the state map through b is S_out = f S_in + (b's
 * own state) in the stabilised form, the max states held constant.  C and
 * (EXP) n regions of state-layout buffers; dstate_in must not overlap
 * dstate_local or dstate_out (MLSTM_ERR_INVALID). */
int mlstm_dstate_chain(const void* dstate_local, const void* dstate_out, const void* state_in,
                       const void* state_out, const float* log_decay, void* dstate_in, int B,
                       int NH, int d_qk, int d_hv, int variant, void* stream);


/* Synchronise `stream` and report what the kernels of this device found:
 * MLSTM_ERR_TIMEOUT if a tensor-core kernel launched on the current device
 * gave up a bounded wait (2 s) since the previous mlstm_device_status call on
 * that device (the outputs of that launch are invalid), MLSTM_ERR_CUDA on a
 * CUDA error, else MLSTM_OK.  Each failure is reported once.  A failure stays
 * within its own launch: each launch carries its own abort epoch, so the
 * launches after a failed one run normally whether or not this call is made
 * in between.  The call reads the kernels' failure flags without clearing
 * them, so it does not disturb kernels running on other streams; a failure of
 * a launch on another stream of the same device is reported too.  This is the
 * one call that blocks. */
int mlstm_device_status(void* stream);

/* Self-test of the failure report: enqueue one tiny kernel whose bounded wait
 * (on a barrier that nothing completes) runs out after 2 s, as a tensor-core
 * kernel's wait would if a hand-over never came.  The kernel then raises its
 * launch's failure flag and returns; it faults nothing and the context stays
 * usable.  The next mlstm_device_status on this device returns
 * MLSTM_ERR_TIMEOUT.  Not part of the mLSTM computation (the pages have no
 * counterpart); for tests of the error path. */
int mlstm_selftest_timeout(void* stream);

/* Static text for a status code. */
const char* mlstm_status_string(int status);

/* Text of the CUDA error behind the calling thread's last MLSTM_ERR_CUDA
 * ("" if none).  Valid until the thread's next call into the library. */
const char* mlstm_last_error(void);

/* Number of kernels mlstm_fwd / mlstm_bwd enqueue for this problem (0 on an
 * argument error or an empty problem). */
int mlstm_fwd_launch_count(int B, int NH, int T, int d_qk, int d_hv, int chunk,
                           int variant, int dtype);
int mlstm_bwd_launch_count(int B, int NH, int T, int d_qk, int d_hv, int chunk,
                           int variant, int dtype);

/* Static name of the index-th kernel that mlstm_fwd (pass 0) or mlstm_bwd
 * (pass 1) enqueues for this problem ("" when out of range). */
const char* mlstm_launch_name(int pass, int index, int B, int NH, int T, int d_qk,
                              int d_hv, int chunk, int variant, int dtype);

/* Run every kernel of the calling thread's later calls on their own stream
 * (serial != 0), or let mlstm_bwd run one kernel on its side stream again
 * (0, the default).  The results are the same either way; the serial order
 * times each kernel alone.  Returns MLSTM_OK. */
int mlstm_set_serial_launches(int serial);

/* Per-kernel timing hook for the calling thread.  While set (count > 0),
 * every mlstm_fwd / mlstm_bwd call records events[2i] (a cudaEvent_t passed
 * as void*) on the stream its i-th kernel runs on just before that kernel and
 * events[2i+1] just after it, for i < count/2; kernels beyond that are not
 * bracketed.  The
 * array is borrowed, not copied: it must stay valid until the hook is
 * cleared with (NULL, 0).  Returns MLSTM_ERR_INVALID for count < 0 or a NULL
 * array with count > 0. */
int mlstm_set_timing_events(void* const* events, int count);

#ifdef __cplusplus
}
#endif

#endif /* MLSTM_H */
