// Internal declarations shared by the KDA library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace kda {

constexpr int FWD_CHUNK = 32;    // chunk length of the chunked kernels
constexpr int FWD_VBLOCK = 32;   // V columns per CTA in the chunked kernels

// Per-(b, hv, 64-step chunk) record of the tensor-core backward: three fp16
// matrices, row-major with the 4-element groups of row r XOR-swizzled by
// r % 8 (element (r, c) of a row of n at rec_off(r, c, n)): [dP; dA] as [i'][j]
// (128 x 64, i' < 64 dP) at half offset GH_PA, [dQE; dKE'] as [i'][f] (128 x
// 128, i' < 64 dQE) at GH_QK, dKEd as [i][f] (64 x 128) at GH_KED; then fp32
// dbeta_R [64] and dEl [128] at float offsets G_DBR, G_DEL; then 16 fp32
// power-of-two scales of the fp16 values (value = half * scale), one per
// 64-row half and group of 32 columns: [dP; dA] as [half][2] at G_SC,
// [dQE; dKE'] as [half][4] at G_SC + 4, dKEd as [4] at G_SC + 12; GREC floats
// per chunk.  (The scale puts each block's largest magnitude in [2^14,
// 2^15): fp16 keeps 11 significant bits down to 2^-29 of it, about 3e-4
// relative RMS added to the gradients against their 2e-3 bar, whatever the
// gradients' range.)
constexpr int GH_PA = 0, GH_QK = 8192, GH_KED = 24576, G_DBR = 16384, G_DEL = 16448, G_SC = 16576, GREC = 16592;
// Per-(b, hv, 64-step chunk) interaction record that the tensor-core forward
// stores with a workspace (floats).  Three 64 x 64 tf32 operand images in the
// K-major canonical layout of the tensor-core kernels (element (r, k) at
// float (r / 8) * 512 + (k / 4) * 32 + (r % 8) * 4 + k % 4), so that the
// backward copies them into shared memory unchanged:
//   [0, INTER_T)         P^T image:  (r, k) = P[k][r]
//   [INTER_T, INTER_AH)  T image:    (r, k) = T[r][k]
//   [INTER_TT, +4096)    T^T image:  (r, k) = T[k][r]
// and Ah row-major at INTER_AH.  The backward reads it instead of recomputing
// the interaction products and the inverse.
constexpr int INTER_T = 4096, INTER_AH = 8192, INTER_TT = 12288, INTER_REC = 16384;
// Per-(b, hv, 64-step chunk) record of the chunked tensor-core forward
// (bytes): the T and P operand images that the chunk-parallel kernel leaves
// for the state pass (64 x 64 tf32 each, K-major canonical layout,
// (r, k) = T[r][k] and P[r][k]).
constexpr unsigned FWR_T = 0, FWR_P = 16384, FWI_BYTES = 32768;

// Chunk geometry of the tensor-core kernels (Args: FwdArgs or BwdArgs).
// Uniform batches: sequence s = batch row, NT = ceil(T / 64) chunks each, the
// state workspace in the 32-step layout [B, HV, ceil(T / 32), K, V].  Packed
// sequences: the chunk table; one state slot per (value head, chunk).  gc is
// the global index of a (sequence, value head, chunk) for the per-chunk
// records, images and buffers.
template <class Args>
__device__ __forceinline__ int chunk_begin(const Args& a, int s) { return a.ctab ? a.seq0[s] : 0; }
template <class Args>
__device__ __forceinline__ int chunk_end(const Args& a, int s) { return a.ctab ? a.seq0[s + 1] : (a.T + 63) / 64; }
template <class Args>
__device__ __forceinline__ int row_of(const Args& a, int s) { return a.ctab ? 0 : s; }  // batch row of the tokens
template <class Args>
__device__ __forceinline__ int2 chunk_span(const Args& a, int c) {  // (first step, steps)
  if (a.ctab) return make_int2(a.ctab[2 * c], a.ctab[2 * c + 1]);
  return make_int2(c * 64, min(64, a.T - c * 64));
}
template <class Args>
__device__ __forceinline__ size_t chunk_gc(const Args& a, int s, int hv, int c) {
  return a.ctab ? (size_t)hv * a.NC + c : ((size_t)s * a.HV + hv) * ((a.T + 63) / 64) + c;
}
template <class Args>  // slot of the state entering chunk c
__device__ __forceinline__ size_t state_slot(const Args& a, int s, int hv, int c) {
  return a.ctab ? (size_t)hv * a.NC + c : ((size_t)s * a.HV + hv) * ((a.T + 31) / 32) + 2 * c;
}
template <class Args>  // slot of the gradient of the state leaving chunk c
__device__ __forceinline__ size_t dstate_slot(const Args& a, int s, int hv, int c) {
  if (a.ctab) return (size_t)hv * a.NC + c;
  const int nt32 = (a.T + 31) / 32;
  return ((size_t)s * a.HV + hv) * nt32 + (2 * c + 1 < nt32 ? 2 * c + 1 : 2 * c);
}

__host__ __device__ constexpr int rec_off(int r, int c, int n) {
  return r * n + ((((c >> 2) ^ (r & 7))) << 2) + (c & 3);
}

// Fused input preparation ("kimi_k3_host/kda.rs": l2norm_rows, bounded_gate,
// and the sigmoid kda_recurrent_step applies to its beta input).  With z set:
// q and k rows are L2-normalised (eps KDA_L2_EPS inside the root), g is
// computed from z (the gate pre-activation, [rows, HV, K] in the input dtype)
// as gate_lb * sigmoid(e^{A_log[hv]} (z + dt_bias[hv])) for gate_lb < 0 or
// -e^{A_log[hv]} softplus(z + dt_bias[hv]) for gate_lb = 0, and beta holds
// logits.
struct PrepArgs {
  const void* z;
  const float* A_log;    // [HV]
  const float* dt_bias;  // [HV, K]
  float gate_lb;
};

struct FwdArgs {
  const void *q, *k, *v;
  const float *g, *beta, *S0;
  void* o;          // may be null (state pass only)
  float* S_T;       // may be null
  float* states;    // may be null; [B, HV, NT, K, V] state entering each chunk
  float* inter;     // may be null; per-chunk interaction records (K = V = 128)
  unsigned char* img;  // may be null; per-chunk operand images of the two-kernel forward (K = V = 128)
  float scale;
  int B, T, H, HV, K, V;
  // Packed sequences (null ctab: B uniform batch rows of T steps).  Then B is
  // the number of sequences, T the packed length, rows index the packed axis;
  // chunk c covers steps ctab[2c] .. ctab[2c] + ctab[2c+1] - 1, and sequence
  // s owns chunks seq0[s] .. seq0[s+1] - 1 (NC chunks in all).
  const int* ctab;
  const int* seq0;
  int NC;
  PrepArgs prep;      // fused input preparation (prep.z null: inputs used as given)
  const void* og;     // output-gate pre-activation [rows, HV, V] in the input dtype, or null
  float og_eps;
  float* o32;         // CUDA-core path with og: fp32 output scratch [rows, HV, V] for the gate pass
  // Asymmetric erase/write variant ("research_layers.py", delta_recurrence):
  // erase [rows, HV, K] in the input dtype; then H counts QUERY heads (a
  // multiple of HV: query head hq reads state head hq / (H / HV)), k, g and
  // erase have HV heads, v holds z [rows, HV, V], beta is unused and o is
  // [rows, H, V].
  const void* erase;
};

struct BwdArgs {
  const void *q, *k, *v, *dO;
  const float *g, *beta, *dS_T;
  const float* states;   // [B, HV, NT, K, V]
  const float* inter;    // per-chunk interaction records of the forward (K = V = 128), else null
  float* dstates;        // [B, HV, NT, K, V] gradient of the state leaving each chunk
  void *dq, *dk, *dv;    // dtype of q/k/v
  float *dg, *dbeta, *dS0;
  float *dq_part, *dk_part;  // fp32 [B, T, HV, K] per value head when HV > H, else null
  float* gws;                // per-chunk records of the tensor-core backward (K = V = 128), else null
  float scale;
  int B, T, H, HV, K, V;
  const int* ctab;  // packed sequences, as in FwdArgs (null: uniform batch rows)
  const int* seq0;
  int NC;
  // tensor-core launches over part of the problem: the state-gradient pass
  // covers heads (sequence * HV + hv) head0 .. head0 + its grid - 1, the
  // gradient kernel items item0 .. item1 - 1 (item1 <= 0: all)
  int head0, item0, item1;
  // assembly: CTA i prefetches to L2 what CTA i + pf_items (a multiple of 4,
  // the CTAs resident at once: most likely its successor on the SM) reads
  // (0: none)
  int pf_items;
};

struct DecodeArgs {
  const void *q, *k, *v;
  const float *g, *beta;
  float* S;
  void* o;
  float scale;
  int B, H, HV;
};

// One decode token from the raw projections ("kimi_k3_host/kda.rs",
// kda_decode_token): the short-convolution step on the q | k | v channels,
// then the prepared recurrence step and the optional output gate.
struct DecodeTokenArgs {
  const void *xq, *xk, *xv;     // [B, H, K], [B, H, K], [B, HV, V]
  const float* conv_w;          // [Cn, W], Cn = 2 H K + HV V
  const float* conv_in;         // [B, Cn, W]
  float* conv_out;              // [B, Cn, W] (may equal conv_in when H == HV)
  PrepArgs prep;                // z [B, HV, K]
  const float* beta;            // logits [B, HV]
  const void* og;               // [B, HV, V] or null
  float og_eps;
  float* S;                     // [B, HV, K, V] in place
  void* o;                      // [B, HV, V]
  float scale;
  int B, H, HV, W;
};

// The short causal convolution with SiLU over whole sequences
// ("kimi_k3_host/kda.rs", conv_update applied to every step in order).
struct ConvArgs {
  const void *xq, *xk, *xv;     // [B, T, H, K], [B, T, H, K], [B, T, HV, V]
  const float* w;               // [Cn, W]
  const float* state_in;        // [B, Cn, W] or null (zeros)
  float* state_out;             // [B, Cn, W] or null
  void *q, *k, *v;              // outputs, shapes of the inputs, input dtype
  int B, T, H, HV, K, V, W;
};

// error reporting (thread-local message; returns the code)
int set_error(int code, const char* msg);
int set_cuda_error(const char* where, cudaError_t e);

int launch_fwd(const FwdArgs& a, int dtype, cudaStream_t stream);
// the CUDA-core forward whatever the shape (stores all 32-step states)
int launch_fwd_ffma(const FwdArgs& a, int dtype, cudaStream_t stream);
bool fwd_tc_eligible(const FwdArgs& a, int dtype);
int launch_fwd_erase(const FwdArgs& a, int dtype, cudaStream_t stream);
// two-kernel CUDA-core forward (chunk preparation into `prep`, then the state
// pass); erase: the asymmetric erase/write variant
bool fwd_fma2_eligible(const FwdArgs& a, const void* workspace);
size_t fma_prep_bytes(int B, int T, int HV, int K, int QG);
size_t fma_split_bytes(int B, int T, int HQ, int HV, int K, int V);
bool fma_kda_split(int K, int V);
int launch_fwd_fma2(const FwdArgs& a, int dtype, bool erase, float* prep, cudaStream_t stream);
int launch_fwd_tc(const FwdArgs& a, cudaStream_t stream);
// the chunked tensor-core forward (a.img: FWI_BYTES per chunk): chunk-parallel
// interaction and inverse, then the state pass
int launch_fwd_chunked(const FwdArgs& a, cudaStream_t stream);
int take_fwd_chunked_error(unsigned* out);
// the gate of the fused preparation into g (fp32 [rows, HV, 128]) from the bf16 z
int launch_prep_gate(const void* z, const float* A_log, const float* dt_bias, float lb, float* g, size_t rows, int HV,
                     cudaStream_t stream);
// probes of every bounded wait in the chunked forward (0: the default)
int set_wait_polls(unsigned polls);
int set_bwd_wait_polls(unsigned polls);
// 4-D TMA tensor maps [rows, T, heads, 128] (rows = B, or 1 for packed
// sequences; CUtensorMap, 128 bytes each) of raw rows: q and k over the
// query/key heads, x (dO) and v over the value heads as bf16 with 64-channel
// boxes, g as fp32 with 32-channel boxes; 64 steps x one head per box,
// 128-byte swizzle, zero fill past the tensor.  (v may be null: no map.)
struct alignas(64) RawMaps {
  unsigned char q[128], k[128], x[128], g[128], v[128];
};
int make_raw_maps(RawMaps* m, const void* q, const void* k, const void* x, const float* g, const void* v, int rows,
                  int T, int H, int HV);
int take_device_error(unsigned* out);
int take_bwd_device_error(unsigned* out);
int launch_bwd(const BwdArgs& a, int dtype, cudaStream_t stream);
bool bwd_tc_eligible(const BwdArgs& a, int dtype);
// the tensor-core backward: state-gradient pass, gradient products and the
// assembly (launched through `assemble` for a range of heads)
typedef int (*AssembleLaunch)(const BwdArgs& a, int head0, int nheads, cudaStream_t stream);
int launch_bwd_tc_passes(const BwdArgs& a, cudaStream_t stream, AssembleLaunch assemble);
int launch_decode(const DecodeArgs& a, int K, int V, int dtype, cudaStream_t stream);
int launch_decode_token(const DecodeTokenArgs& a, int K, int V, int dtype, cudaStream_t stream);
int launch_short_conv(const ConvArgs& a, int dtype, cudaStream_t stream);
// the output-gate pass of the CUDA-core forward: o = gate(o32, og)
int launch_out_gate(const float* o32, const void* og, float eps, size_t rows, int V, int dtype, void* o,
                    cudaStream_t stream);

}  // namespace kda
