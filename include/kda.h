/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) library
 * (libkda.so).
 *
 * The recurrence (per batch b and value head hv, for t = 0 .. T-1):
 *
 *     S_dec = exp(g_t) (.) S_{t-1}            decay, exp(g_t) broadcast along V
 *     r_t   = v_t - k_t^T S_dec               delta-rule residual
 *     S_t   = S_dec + (beta_t k_t) (x) r_t    rank-1 write
 *     o_t   = (scale q_t)^T S_t               readout after the write
 *
 * Defined by "K3/kda/ops/reference/recurrent.py" (naive_kda_fwd and the
 * module docstring), restated step by step in "K3/notes/sections/sec-01.tex"
 * (section "KDA recurrence core", the four-step update), and for one decode
 * token by "kimi_k3_host/kda.rs" (kda_recurrent_step).  Value head hv reads
 * query/key head hv / (HV / H) (repeat-interleave of the head axis).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are caller-owned DEVICE pointers to dense row-major
 *     arrays with the stated shapes, in the memory of the calling thread's
 *     current CUDA device (the one the kernels launch on; stream must belong
 *     to it too).  The library never frees or retains them.
 *   - dtype selects the element type of q, k, v, o, dO, dq, dk, dv:
 *     KDA_DTYPE_FP32 (float) or KDA_DTYPE_BF16 (bfloat16).  g, beta, states
 *     and their gradients are always float.
 *   - g is the log-space per-channel decay (both gates of the host model give
 *     g <= 0); beta is the write strength after the sigmoid, in (0, 1).
 *   - scale multiplies q; it must be finite and > 0 (the usual 1/sqrt(K) is
 *     the caller's choice).
 *   - K and V must each be 32, 64 or 128; HV must be a multiple of H.
 *   - stream is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on it and returns; results are ready when the
 *     stream reaches that point.
 *   - Return value: KDA_OK (0) or one of the KDA_ERR_* codes below; the
 *     arguments are validated before anything is enqueued, so a non-zero
 *     return from validation leaves all buffers untouched.  kda_last_error()
 *     returns a message for the calling thread's most recent failure.
 *   - The library makes no device allocation when it is called: scratch
 *     comes from the caller's workspace.  Its module does hold one fixed
 *     array of KDA_NOALLOC_SCRATCH_BYTES on every GPU that loads it (the
 *     scratch of kda_bwd_noalloc), from load until the process exits.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  KDA_OK = 0,
  KDA_ERR_NULL = 1,        /* a required pointer is NULL */
  KDA_ERR_SHAPE = 2,       /* a size is < 1, HV % H != 0, or a grid limit is exceeded */
  KDA_ERR_DTYPE = 3,       /* dtype is not KDA_DTYPE_FP32 / KDA_DTYPE_BF16 */
  KDA_ERR_UNSUPPORTED = 4, /* K or V not in {32, 64, 128} */
  KDA_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required */
  KDA_ERR_CUDA = 6,        /* a CUDA call failed (launch or attribute) */
  KDA_ERR_ARG = 7,         /* scale not finite/positive, misaligned pointer, bad flags */
};

enum { KDA_DTYPE_FP32 = 0, KDA_DTYPE_BF16 = 1 };

/* Flags of kda_bwd. */
enum {
  /* The workspace was given to a kda_fwd on the same inputs (same q, k, v,
   * g, beta, S0, scale and sizes) with at least kda_fwd_workspace_bytes()
   * bytes, and still holds the chunk states and interaction records that it
   * stored at its start; kda_bwd then skips its own forward pass. */
  KDA_BWD_STATES_FROM_FWD = 1,
};

/* Message for the calling thread's most recent non-zero return ("" if none).
 * The pointer stays valid until the next call from the same thread. */
const char* kda_last_error(void);

/* Reads and clears the device-side error bits of the library's kernels on the
 * current device, synchronising it first.  Bit 0: a tensor-core kernel gave
 * up waiting for its own tensor-core work (a bounded wait ran out) and
 * skipped the rest of its launch; its outputs are then undefined.  Bit 1: a
 * kernel of the chunked tensor-core forward found its shared memory not
 * 1024-byte aligned (its TMA tiles need it) and skipped its launch.  Returns
 * KDA_OK or KDA_ERR_CUDA; *flags receives the bits (0 = none). */
int kda_device_status(unsigned* flags);

/* Test hook for the failure path of the bounded waits.  Every wait of the
 * chunked tensor-core forward (the two kernels that kda_fwd, kda_fwd_varlen
 * and kda_fwd_prep run when given their workspace) and of the tensor-core
 * backward's state-gradient pass probes its mbarrier at most `polls` times
 * (0 restores the default, 2^24) before it gives up.  A
 * kernel that gives up first waits, under the default bound, for every copy
 * and tensor-core product it has already issued, then frees its tensor
 * memory, sets bit 0 of kda_device_status() and returns; its outputs are
 * undefined.  With polls = 1 the first wait of each such kernel gives up.
 * The value is per device (the current one) and persists until changed.
 * Returns KDA_OK or KDA_ERR_CUDA. */
int kda_set_wait_polls(unsigned polls);

/* Bytes of the training workspace of kda_fwd: the fp32 state entering every
 * 32 steps [B, HV, ceil(T / 32), K, V], then (K = V = 128) the per-64-step
 * interaction records (P^T, T, T^T operand images and Ah, 64 KB per chunk)
 * and the scratch of kda_fwd_scratch_bytes(); 0 if a size is invalid. */
size_t kda_fwd_workspace_bytes(int B, int T, int HV, int K, int V);

/* Bytes of the optional scratch that lets kda_fwd run as two kernels: a
 * chunk-parallel pass that leaves every chunk's operands of the state
 * products there, then the sequential state pass.  On the tensor-core path
 * (K = V = 128, bf16) the chunk-parallel pass leaves the T and P operand
 * images (32,768 bytes per 64-step chunk) and the state pass rebuilds the
 * other operands from the inputs;
 * on the CUDA-core path (fp32 inputs, or other K and V) the chunk records take
 * 4 (2 C^2 + 3 C K + K) bytes per 32-step chunk (C = 32); for K = V = 128 the
 * larger of the two, as the dtype is not an argument.  For other K and V the
 * CUDA-core path also keeps the state entering every chunk and its residual
 * solution U (4 (K V + C V) bytes per chunk), and a third, chunk-parallel
 * kernel forms the outputs.  0 if a size is invalid. */
size_t kda_fwd_scratch_bytes(int B, int T, int HV, int K, int V);

/* Bytes kda_bwd needs: the chunk states and interaction records (as
 * kda_fwd_workspace_bytes lays them out), then the larger of the forward's
 * scratch and [gradients of the state leaving every 32 steps (state layout);
 * when HV > H fp32 per-value-head partials of dq and dk [B, T, HV, K] each;
 * per-chunk gradient records (K = V = 128; 66,368 bytes per 64-step chunk:
 * the chunk's C x C and C x K adjoints in fp16 with a power-of-two scale
 * per 64 rows and 32 columns, its per-row and per-channel terms in fp32)];
 * 0 if a size is invalid.  This is
 * at least kda_fwd_workspace_bytes(), so one buffer serves both calls. */
size_t kda_bwd_workspace_bytes(int B, int T, int H, int HV, int K, int V);

/* Chunk-parallel prefill forward ("recurrent.py", naive_kda_fwd; the chunk
 * form is the triangular-solve algebra of "research_layers.py",
 * delta_recurrence).
 *   q, k  [B, T, H, K]   dtype      v   [B, T, HV, V] dtype
 *   g     [B, T, HV, K]  float      beta [B, T, HV]   float
 *   S0    [B, HV, K, V]  float, or NULL for a zero initial state
 *   o     [B, T, HV, V]  dtype (output)
 *   S_T   [B, HV, K, V]  float (output), or NULL to skip the final state
 *   workspace: NULL; or, 16-byte aligned, at least
 *     kda_fwd_workspace_bytes(B, T, HV, K, V) bytes: the states and records
 *     for a later kda_bwd with KDA_BWD_STATES_FROM_FWD are stored there; or
 *     at least kda_fwd_scratch_bytes() (but fewer than the former): used as
 *     scratch only.  A workspace of neither size is KDA_ERR_WORKSPACE.  With
 *     either, the forward runs as two kernels (chunk-parallel pass, then the
 *     state pass: tensor-core shapes; CUDA-core shapes when v is 16-byte
 *     aligned); without one, one kernel carries each state slice through
 *     its chunks.
 * With a training workspace, bf16 K = V = 128 and 16-byte aligned q, k, v, g
 * (the inputs of the tensor-core backward), o must be 16-byte aligned too
 * (KDA_ERR_ARG otherwise), so that the stored states and records are the
 * tensor-core path's.
 * o and S_T must not alias any input.  S_T may alias S0 only if S0 is not
 * needed afterwards (S0 is read before S_T is written, per value column). */
int kda_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
            const float* S0, float scale, int B, int T, int H, int HV, int K, int V, int dtype,
            void* o, float* S_T, void* workspace, size_t workspace_bytes, void* stream);

/* Packed variable-length prefill: N sequences of lengths cu_seqlens[s+1] -
 * cu_seqlens[s] laid back to back on one time axis of T = cu_seqlens[N] steps,
 * each run as kda_fwd runs one batch row (its own initial and final state;
 * the state passing of "recurrent.py", naive_kda_fwd, initial_state and
 * output_final_state, per sequence).
 *   q, k [T, H, K] dtype; v [T, HV, V] dtype; g [T, HV, K] float; beta [T, HV] float
 *   cu_seqlens: HOST int32 [N + 1], cu_seqlens[0] = 0, non-decreasing (empty
 *     sequences allowed: their final state is their initial state)
 *   S0 [N, HV, K, V] float or NULL; o [T, HV, V] dtype; S_T [N, HV, K, V] float or NULL
 *   workspace: required, 16-byte aligned; at least
 *     kda_fwd_varlen_workspace_bytes() bytes for the two-kernel forward, else at
 *     least its chunk table (then one kernel per (sequence, value head)).
 * Runs on the tensor-core path only: bf16, K = V = 128, 16-byte aligned q, k,
 * v, g and o (KDA_ERR_ARG otherwise).  The chunk table is uploaded from the
 * host with one copy on `stream`.  A workspace of at least
 * kda_bwd_varlen_workspace_bytes() bytes also receives the states and
 * interaction records for a later kda_bwd_varlen with KDA_BWD_STATES_FROM_FWD. */
size_t kda_fwd_varlen_workspace_bytes(const int* cu_seqlens, int N, int HV, int K, int V);
int kda_fwd_varlen(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const float* S0, float scale, const int* cu_seqlens, int N, int H, int HV, int K, int V,
                   int dtype, void* o, float* S_T, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of kda_fwd_varlen (per sequence the backward of kda_bwd, from its
 * own dS_T to its own dS0).
 *   inputs and cu_seqlens as kda_fwd_varlen; dO [T, HV, V] dtype; dS_T
 *   [N, HV, K, V] float or NULL
 *   dq, dk [T, H, K] dtype; dv [T, HV, V] dtype; dg [T, HV, K] float;
 *   dbeta [T, HV] float; dS0 [N, HV, K, V] float or NULL
 *   workspace: at least kda_bwd_varlen_workspace_bytes() bytes, 16-byte aligned
 *   flags: 0 (the forward pass runs first) or KDA_BWD_STATES_FROM_FWD (the
 *     workspace went through kda_fwd_varlen on the same inputs)
 * Tensor-core path only (bf16, K = V = 128, 16-byte aligned q, k, v, dO, g, dq, dv). */
size_t kda_bwd_varlen_workspace_bytes(const int* cu_seqlens, int N, int H, int HV, int K, int V);
int kda_bwd_varlen(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const float* S0, const void* dO, const float* dS_T, float scale, const int* cu_seqlens, int N,
                   int H, int HV, int K, int V, int dtype, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                   float* dS0, void* workspace, size_t workspace_bytes, int flags, void* stream);

/* One decode token on a state updated IN PLACE ("kimi_k3_host/kda.rs",
 * kda_recurrent_step, with the q/k L2 normalisation and the sigmoid of beta
 * left to the caller).
 *   q, k  [B, H, K]   dtype      v    [B, HV, V] dtype
 *   g     [B, HV, K]  float      beta [B, HV]    float
 *   S     [B, HV, K, V] float, read and overwritten with the new state;
 *         16-byte aligned
 *   o     [B, HV, V]  dtype (output) */
int kda_decode_step(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, float* S, float scale, int B, int H, int HV, int K, int V,
                    int dtype, void* o, void* stream);

/* Backward of kda_fwd ("recurrent.py", KDAFunction.backward), returning
 * also the gradient of the initial state.
 *   inputs as kda_fwd; dO [B, T, HV, V] dtype; dS_T [B, HV, K, V] float or
 *   NULL (zero upstream gradient of the final state)
 *   dq, dk [B, T, H, K] dtype; dv [B, T, HV, V] dtype (grouped heads summed)
 *   dg [B, T, HV, K] float; dbeta [B, T, HV] float
 *   dS0 [B, HV, K, V] float, or NULL to skip it
 *   workspace: at least kda_bwd_workspace_bytes(B, T, H, HV, K, V) bytes,
 *     16-byte aligned, reused as scratch (contents on return are unspecified
 *     except that the chunk states stay valid).
 *   flags: 0 or KDA_BWD_STATES_FROM_FWD. */
int kda_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
            const float* S0, const void* dO, const float* dS_T, float scale, int B, int T, int H,
            int HV, int K, int V, int dtype, void* dq, void* dk, void* dv, float* dg,
            float* dbeta, float* dS0, void* workspace, size_t workspace_bytes, int flags,
            void* stream);

/* ---- The preparation around the recurrence ("kimi_k3_host/kda.rs").
 * L2 normalisation of a q or k row: x / sqrt(sum x^2 + KDA_L2_EPS)
 * (l2norm_rows, KDA_L2_EPS).  Decay gate from its pre-activation z
 * (bounded_gate), x = z + dt_bias[hv], d = exp(A_log[hv]):
 *     g = gate_lower_bound * sigmoid(d x)      gate_lower_bound < 0
 *     g = -d * softplus(x)                     gate_lower_bound = 0 (no bound)
 * beta = sigmoid(beta_logit) (kda_recurrent_step).  Output gate
 * (full_rank_output_gate), per (step, value head) row of V values:
 *     o <- sigmoid(out_gate) * o / sqrt(mean(o^2) + out_eps).
 * Short convolution (conv_update): depthwise over the channels q | k | v
 * (2 H K + HV V channels: the H K query channels, the H K key channels, then
 * the HV V value channels, each tensor's own row-major order), weights
 * w [channels, W] and window [B, channels, W] (oldest input first, newest in
 * slot W - 1), y = SiLU(sum_j w[c][j] window[j]) after the window takes the
 * new input; 1 <= W <= 8. */
#define KDA_L2_EPS 1e-6f

/* Prefill from the raw projections: kda_fwd with the preparation fused into
 * its kernels (q, k normalised per row, g from z, beta from its logit) and
 * the optional output gate applied to o before it is stored.
 *   q, k [B, T, H, K] dtype (before normalisation); v [B, T, HV, V] dtype
 *   z [B, T, HV, K] dtype; A_log [HV] float; dt_bias [HV, K] float
 *   beta_logit [B, T, HV] float
 *   out_gate [B, T, HV, V] dtype, or NULL for no output gate; out_eps >= 0
 *   S0, S_T, o as kda_fwd (o is gated when out_gate is given)
 *   workspace: NULL, or 16-byte aligned scratch; with at least
 *     kda_fwd_prep_workspace_bytes() bytes every path runs (the two-kernel
 *     tensor-core forward, and the CUDA-core forward's fp32 output for the
 *     gate pass); with NULL the tensor-core path runs as one kernel per
 *     (b, hv), and a CUDA-core bf16 shape with an output gate returns
 *     KDA_ERR_WORKSPACE.
 * No chunk states are stored (there is no backward of the preparation). */
size_t kda_fwd_prep_workspace_bytes(int B, int T, int H, int HV, int K, int V, int dtype);
int kda_fwd_prep(const void* q, const void* k, const void* v, const void* z, const float* A_log,
                 const float* dt_bias, float gate_lower_bound, const float* beta_logit, const void* out_gate,
                 float out_eps, const float* S0, float scale, int B, int T, int H, int HV, int K, int V, int dtype,
                 void* o, float* S_T, void* workspace, size_t workspace_bytes, void* stream);

/* The short convolution with SiLU over whole sequences (the prefill form of
 * conv_update, applied to every step in order).
 *   xq, xk [B, T, H, K] dtype; xv [B, T, HV, V] dtype (the projections)
 *   w [2 H K + HV V, W] float; state_in [B, 2 H K + HV V, W] float or NULL
 *   (zero window); state_out the same shape (the window after the last step)
 *   or NULL; state_out must not overlap state_in
 *   q, k, v outputs in the shapes and dtype of xq, xk, xv (the convolved
 *   activations, rounded to dtype); they must not alias the inputs.
 *   T <= 2097120 (65535 blocks of 32 steps; KDA_ERR_SHAPE above). */
int kda_short_conv(const void* xq, const void* xk, const void* xv, const float* w, const float* state_in,
                   float* state_out, int B, int T, int H, int HV, int K, int V, int W, int dtype, void* q,
                   void* k, void* v, void* stream);

/* One decode token from the raw projections ("kimi_k3_host/kda.rs",
 * kda_decode_token, with bounded_gate and full_rank_output_gate): the
 * convolution step, the preparation, the recurrence step on S IN PLACE and
 * the optional output gate, in one launch.
 *   xq, xk [B, H, K] dtype; xv [B, HV, V] dtype
 *   conv_w [2 H K + HV V, W] float; conv_in [B, 2 H K + HV V, W] float or NULL
 *   (zero window); conv_out the same shape, receives the new window; it may
 *   equal conv_in only when H == HV (grouped heads share the q/k windows)
 *   z [B, HV, K] dtype; A_log, dt_bias, gate_lower_bound as kda_fwd_prep
 *   beta_logit [B, HV] float; out_gate [B, HV, V] dtype or NULL
 *   S [B, HV, K, V] float, 16-byte aligned, read and overwritten
 *   o [B, HV, V] dtype (output) */
int kda_decode_token(const void* xq, const void* xk, const void* xv, const float* conv_w, const float* conv_in,
                     float* conv_out, int W, const void* z, const float* A_log, const float* dt_bias,
                     float gate_lower_bound, const float* beta_logit, const void* out_gate, float out_eps, float* S,
                     float scale, int B, int H, int HV, int K, int V, int dtype, void* o, void* stream);

/* Prefill of the asymmetric erase/write delta recurrence ("research_layers.py",
 * delta_recurrence and delta_token_reference), per state head hv:
 *     S_bar = exp(g_t) (.) S_{t-1}
 *     S_t   = S_bar + k_t (z_t - e_t^T S_bar)^T     (erase along e, write along k)
 *     o_t   = (scale q_t)^T S_t                     per query head, after the write
 * KDA is the case e = beta k, z = beta v.  Heads follow the page's layer:
 * query head hq reads state head hq / (HQ / HV).
 *   q [B, T, HQ, K] dtype; k, e [B, T, HV, K] dtype; z [B, T, HV, V] dtype;
 *   g [B, T, HV, K] float; S0 [B, HV, K, V] float or NULL
 *   o [B, T, HQ, V] dtype (output); S_T [B, HV, K, V] float or NULL
 * HQ must be a multiple of HV.  Runs on the CUDA-core chunk kernels; see
 * kda_fwd_erase_workspace_bytes for the workspace. */
int kda_fwd_erase(const void* q, const void* k, const void* e, const void* z, const float* g, const float* S0,
                  float scale, int B, int T, int HQ, int HV, int K, int V, int dtype, void* o, float* S_T,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the optional workspace of kda_fwd_erase (16-byte aligned, with a
 * 16-byte aligned z): with it the variant runs as three kernels, a
 * chunk-parallel pass that leaves every 32-step chunk's operands there
 * (4 (2 C^2 + 3 C K + K + (HQ / HV - 1)(C^2 + C K)) bytes per chunk and state
 * head, C = 32: the inverse times diag(beta), the residual and carry
 * operands, and P and the decayed queries of every query head), a state pass
 * per state head and 32 value columns that carries the state once and stores
 * the state entering every chunk and the chunk's residual solution U
 * (4 (K V + C V) bytes per chunk and state head), and a chunk-parallel
 * read-out of every query head.  Without a workspace (NULL) one kernel per
 * query head carries a copy of its state head.  A non-NULL workspace smaller
 * than this is KDA_ERR_WORKSPACE.  0 if a size is invalid. */
size_t kda_fwd_erase_workspace_bytes(int B, int T, int HQ, int HV, int K, int V);

/* Size in bytes of the fixed device array that kda_bwd_noalloc uses as its
 * scratch (64 MiB, held on every GPU that loads the library until exit). */
#define KDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* kda_bwd for callers that cannot allocate device memory: a plugin whose host
 * framework owns all device memory and gives it no workspace, or a running
 * loop that forbids allocator calls (cudaMalloc/cudaFree synchronise the
 * device and fail once another allocator has reserved the memory).  Nothing
 * in the method's definition corresponds to this entry point; it is a
 * deployment convenience.
 *   Arguments, layouts and results are those of kda_bwd (flags = 0); the
 *   caller still owns every input and output.  The scratch is a file-scope
 *   __device__ array of KDA_NOALLOC_SCRATCH_BYTES; a problem whose
 *   kda_bwd_workspace_bytes() exceeds it returns KDA_ERR_WORKSPACE with a
 *   message and enqueues nothing.  Nothing is allocated: the first call on a
 *   device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current and caches it, so make that first call before any
 *   stream capture.  A cudaDeviceReset() on that device invalidates the
 *   cached address: do not call kda_bwd_noalloc again in such a process.  All calls share the one array: calls whose work overlaps
 *   on the GPU (other streams or threads on the same device) race and must be
 *   ordered by the caller.  Each call writes every scratch byte it reads, so
 *   stale contents from an earlier call are never used. */
int kda_bwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, const float* S0, const void* dO, const float* dS_T,
                    float scale, int B, int T, int H, int HV, int K, int V, int dtype, void* dq,
                    void* dk, void* dv, float* dg, float* dbeta, float* dS0, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
