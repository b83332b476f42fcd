// C ABI of the KDA library: argument validation, workspace carving and
// dispatch to the kernels.  See include/kda.h for the contract.
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace kda {

static thread_local char g_err[512] = "";

int set_error(int code, const char* msg) {
  snprintf(g_err, sizeof(g_err), "%s", msg);
  return code;
}

int set_cuda_error(const char* where, cudaError_t e) {
  snprintf(g_err, sizeof(g_err), "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
  return KDA_ERR_CUDA;
}

static bool supported_dim(int d) { return d == 32 || d == 64 || d == 128; }

static int check_common(const char* fn, int B, int T, int H, int HV, int K, int V, int dtype,
                        float scale) {
  char buf[256];
  if (B < 1 || T < 1 || H < 1 || HV < 1 || K < 1 || V < 1) {
    snprintf(buf, sizeof(buf), "%s: sizes must be >= 1 (B=%d T=%d H=%d HV=%d K=%d V=%d)", fn, B, T, H,
             HV, K, V);
    return set_error(KDA_ERR_SHAPE, buf);
  }
  if (HV % H != 0) {
    snprintf(buf, sizeof(buf), "%s: HV=%d is not a multiple of H=%d", fn, HV, H);
    return set_error(KDA_ERR_SHAPE, buf);
  }
  if (B > 65535 || HV > 65535) {
    snprintf(buf, sizeof(buf), "%s: B=%d or HV=%d exceeds 65535", fn, B, HV);
    return set_error(KDA_ERR_SHAPE, buf);
  }
  if (!supported_dim(K) || !supported_dim(V)) {
    snprintf(buf, sizeof(buf), "%s: K=%d, V=%d; each must be 32, 64 or 128", fn, K, V);
    return set_error(KDA_ERR_UNSUPPORTED, buf);
  }
  if (dtype != KDA_DTYPE_FP32 && dtype != KDA_DTYPE_BF16) {
    snprintf(buf, sizeof(buf), "%s: dtype=%d is not KDA_DTYPE_FP32 (0) or KDA_DTYPE_BF16 (1)", fn, dtype);
    return set_error(KDA_ERR_DTYPE, buf);
  }
  if (!(scale > 0.f) || !isfinite(scale)) {
    snprintf(buf, sizeof(buf), "%s: scale=%g must be finite and > 0", fn, (double)scale);
    return set_error(KDA_ERR_ARG, buf);
  }
  return KDA_OK;
}

static size_t states_bytes(int B, int T, int HV, int K, int V) {
  const size_t NT = (size_t)(T + FWD_CHUNK - 1) / FWD_CHUNK;
  return (size_t)B * HV * NT * K * V * sizeof(float);
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// interaction records stored by the tensor-core forward (K = V = 128)
static size_t inter_bytes(int B, int T, int HV, int K, int V) {
  if (K != 128 || V != 128) return 0;
  const size_t NT64 = (size_t)(T + 63) / 64;
  return (size_t)B * HV * NT64 * INTER_REC * sizeof(float);
}

// per-chunk T and P images of the chunked tensor-core forward (K = V = 128)
static size_t img_bytes(int B, int T, int HV, int K, int V) {
  if (K != 128 || V != 128) return 0;
  const size_t NT64 = (size_t)(T + 63) / 64;
  return (size_t)B * HV * NT64 * FWI_BYTES;
}

// scratch of the two-kernel forwards: for K = V = 128 the chunk images of the
// tensor-core path or the CUDA-core path's chunk records (fp32 inputs),
// whichever is larger (the dtype is not an argument here); for other K and V
// the CUDA-core records, then the state entering and U of every chunk for the
// separate read-out kernel
static size_t scratch_bytes(int B, int T, int HV, int K, int V) {
  if (K != 32 && K != 64 && K != 128) return 0;
  if (fma_kda_split(K, V)) return fma_split_bytes(B, T, HV, HV, K, V);
  const size_t img = img_bytes(B, T, HV, K, V), prep = fma_prep_bytes(B, T, HV, K, 1);
  return img > prep ? img : prep;
}

// training forward: [states | interaction records | scratch]
static size_t fwd_ws_bytes(int B, int T, int HV, int K, int V) {
  return states_bytes(B, T, HV, K, V) + inter_bytes(B, T, HV, K, V) + scratch_bytes(B, T, HV, K, V);
}

// Packed sequences: the chunk table (t0, L per chunk of at most 64 steps,
// sequence by sequence) and each sequence's first chunk, from the host
// cu_seqlens.  Returns the number of chunks, or -1 if cu_seqlens is invalid.
static long varlen_chunks(const int* cu, int N, std::vector<int>* tab, std::vector<int>* seq0) {
  if (!cu || N < 1 || cu[0] != 0) return -1;
  long nc = 0;
  for (int s = 0; s < N; ++s) {
    if (cu[s + 1] < cu[s]) return -1;
    if (seq0) seq0->push_back((int)nc);
    for (int t0 = cu[s]; t0 < cu[s + 1]; t0 += 64, ++nc)
      if (tab) {
        tab->push_back(t0);
        tab->push_back(cu[s + 1] - t0 < 64 ? cu[s + 1] - t0 : 64);
      }
  }
  if (seq0) seq0->push_back((int)nc);
  return nc;
}

// workspace of kda_fwd_varlen: [chunk table | sequence starts] (256-byte
// aligned), then the chunk images of the two-kernel forward
static size_t varlen_table_bytes(long nc, int N) {
  return ((size_t)(2 * nc + N + 1) * sizeof(int) + 255) / 256 * 256;
}

// training workspace of packed sequences (K = V = 128): [table | states (one
// per value head and chunk) | interaction records | the chunk images, which
// the backward overwrites with [state gradients | dq/dk partials | records]]
struct VarlenLayout {
  size_t table, states, inter, img, tail, total;
  VarlenLayout(long nc, int N, int T, int H, int HV) {
    table = varlen_table_bytes(nc, N);
    states = (size_t)HV * nc * 128 * 128 * sizeof(float);
    inter = (size_t)HV * nc * INTER_REC * sizeof(float);
    img = (size_t)HV * nc * FWI_BYTES;
    tail = states + (HV > H ? 2 * (size_t)T * HV * 128 * sizeof(float) : 0) + (size_t)HV * nc * GREC * sizeof(float);
    total = table + states + inter + (tail > img ? tail : img);
  }
};

}  // namespace kda

using namespace kda;

extern "C" {

const char* kda_last_error(void) { return g_err; }

int kda_device_status(unsigned* flags) {
  if (!flags) return set_error(KDA_ERR_NULL, "kda_device_status: flags must be non-NULL");
  unsigned f1 = 0, f2 = 0, f3 = 0;
  int rc = take_device_error(&f1);
  if (!rc) rc = take_bwd_device_error(&f2);
  if (!rc) rc = take_fwd_chunked_error(&f3);
  *flags = f1 | f2 | f3;
  return rc;
}

int kda_set_wait_polls(unsigned polls) {
  g_err[0] = 0;
  const int rc = set_wait_polls(polls);
  return rc ? rc : set_bwd_wait_polls(polls);
}

size_t kda_fwd_workspace_bytes(int B, int T, int HV, int K, int V) {
  if (B < 1 || T < 1 || HV < 1 || K < 1 || V < 1) return 0;
  return fwd_ws_bytes(B, T, HV, K, V);
}

size_t kda_fwd_scratch_bytes(int B, int T, int HV, int K, int V) {
  if (B < 1 || T < 1 || HV < 1 || K < 1 || V < 1) return 0;
  return scratch_bytes(B, T, HV, K, V);
}

static size_t grads_record_bytes(int B, int T, int HV, int K, int V) {
  if (K != 128 || V != 128) return 0;
  const size_t NT64 = (size_t)(T + 63) / 64;
  return (size_t)B * HV * NT64 * GREC * sizeof(float);
}

// the part of the backward workspace after [states | interaction records]:
// the forward's chunk images, which the backward then overwrites with
// [state gradients | dq/dk partials | gradient records]
static size_t bwd_tail_bytes(int B, int T, int H, int HV, int K, int V) {
  size_t bytes = states_bytes(B, T, HV, K, V);
  if (HV > H) bytes += 2 * (size_t)B * T * HV * K * sizeof(float);
  return bytes + grads_record_bytes(B, T, HV, K, V);
}

size_t kda_bwd_workspace_bytes(int B, int T, int H, int HV, int K, int V) {
  if (B < 1 || T < 1 || H < 1 || HV < 1 || K < 1 || V < 1 || HV % H) return 0;
  const size_t tail = bwd_tail_bytes(B, T, H, HV, K, V), img = scratch_bytes(B, T, HV, K, V);
  return states_bytes(B, T, HV, K, V) + inter_bytes(B, T, HV, K, V) + (tail > img ? tail : img);
}

int kda_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
            const float* S0, float scale, int B, int T, int H, int HV, int K, int V, int dtype,
            void* o, float* S_T, void* workspace, size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  int rc = check_common("kda_fwd", B, T, H, HV, K, V, dtype, scale);
  if (rc) return rc;
  if (!q || !k || !v || !g || !beta || !o)
    return set_error(KDA_ERR_NULL, "kda_fwd: q, k, v, g, beta and o must be non-NULL");
  float *states = nullptr, *inter = nullptr;
  unsigned char* img = nullptr;
  if (workspace) {
    if (!aligned16(workspace)) return set_error(KDA_ERR_ARG, "kda_fwd: workspace must be 16-byte aligned");
    char* ws = static_cast<char*>(workspace);
    const size_t sb = states_bytes(B, T, HV, K, V), ib = inter_bytes(B, T, HV, K, V);
    const size_t gb = scratch_bytes(B, T, HV, K, V);
    if (workspace_bytes >= fwd_ws_bytes(B, T, HV, K, V)) {  // training: states for the backward
      states = reinterpret_cast<float*>(ws);
      inter = ib ? reinterpret_cast<float*>(ws + sb) : nullptr;
      img = gb ? reinterpret_cast<unsigned char*>(ws + sb + ib) : nullptr;
    } else if (gb && workspace_bytes >= gb) {  // scratch only
      img = reinterpret_cast<unsigned char*>(ws);
    } else {
      return set_error(KDA_ERR_WORKSPACE,
                       "kda_fwd: workspace smaller than kda_fwd_scratch_bytes() and kda_fwd_workspace_bytes()");
    }
  }
  FwdArgs a{q, k, v, g, beta, S0, o, S_T, states, inter, img, scale, B, T, H, HV, K, V};
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (states && dtype == KDA_DTYPE_BF16 && K == 128 && V == 128 && aligned16(q) && aligned16(k) && aligned16(v) &&
      aligned16(g) && !aligned16(o))  // (a tensor-core backward on these inputs reads tensor-core records)
    return set_error(KDA_ERR_ARG, "kda_fwd: the training forward of this shape needs a 16-byte aligned o");
  if (fwd_tc_eligible(a, dtype)) return launch_fwd_tc(a, st);
  if (img && fwd_fma2_eligible(a, img)) {  // the scratch holds the CUDA-core path's chunk records
    a.img = nullptr;
    return launch_fwd_fma2(a, dtype, false, reinterpret_cast<float*>(img), st);
  }
  a.img = nullptr;
  return launch_fwd_ffma(a, dtype, st);
}

size_t kda_fwd_varlen_workspace_bytes(const int* cu_seqlens, int N, int HV, int K, int V) {
  const long nc = varlen_chunks(cu_seqlens, N, nullptr, nullptr);
  if (nc < 0 || HV < 1 || K != 128 || V != 128) return 0;
  return varlen_table_bytes(nc, N) + (size_t)nc * HV * FWI_BYTES;
}

int kda_fwd_varlen(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const float* S0, float scale, const int* cu_seqlens, int N, int H, int HV, int K, int V,
                   int dtype, void* o, float* S_T, void* workspace, size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  std::vector<int> tab, seq0;
  const long nc = varlen_chunks(cu_seqlens, N, &tab, &seq0);
  if (nc < 0)
    return set_error(KDA_ERR_ARG, "kda_fwd_varlen: cu_seqlens must start at 0 and be non-decreasing (N >= 1)");
  const int T = cu_seqlens[N];
  int rc = check_common("kda_fwd_varlen", N, T > 0 ? T : 1, H, HV, K, V, dtype, scale);
  if (rc) return rc;
  if (T > 0 && (!q || !k || !v || !g || !beta || !o))
    return set_error(KDA_ERR_NULL, "kda_fwd_varlen: q, k, v, g, beta and o must be non-NULL");
  if (!workspace) return set_error(KDA_ERR_WORKSPACE, "kda_fwd_varlen: workspace is required");
  if (!aligned16(workspace)) return set_error(KDA_ERR_ARG, "kda_fwd_varlen: workspace must be 16-byte aligned");
  const size_t tb = varlen_table_bytes(nc, N), full = tb + (size_t)nc * HV * FWI_BYTES;
  if (workspace_bytes < tb)
    return set_error(KDA_ERR_WORKSPACE, "kda_fwd_varlen: workspace smaller than its chunk table");
  char* ws = static_cast<char*>(workspace);
  float *states = nullptr, *inter = nullptr;
  unsigned char* img = workspace_bytes >= full ? reinterpret_cast<unsigned char*>(ws + tb) : nullptr;
  const VarlenLayout lay(nc, N, T, H, HV);
  if (K == 128 && V == 128 && workspace_bytes >= lay.total) {  // training: states and records for kda_bwd_varlen
    states = reinterpret_cast<float*>(ws + tb);
    inter = reinterpret_cast<float*>(ws + tb + lay.states);
    img = reinterpret_cast<unsigned char*>(ws + tb + lay.states + lay.inter);
  }
  FwdArgs a{q, k, v, g, beta, S0, o, S_T, states, inter, img, scale, N, T, H, HV, K,
            V, reinterpret_cast<const int*>(ws), reinterpret_cast<const int*>(ws) + 2 * nc, (int)nc};
  if (!fwd_tc_eligible(a, dtype))
    return set_error(KDA_ERR_ARG,
                     "kda_fwd_varlen: packed sequences run on the tensor-core path only (bf16, K = V = 128, "
                     "16-byte aligned q, k, v, g, o)");
  std::vector<int> host(tab);
  host.insert(host.end(), seq0.begin(), seq0.end());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(ws, host.data(), host.size() * sizeof(int), cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return set_cuda_error("kda_fwd_varlen: chunk table upload", e);
  return launch_fwd_tc(a, st);
}

size_t kda_bwd_varlen_workspace_bytes(const int* cu_seqlens, int N, int H, int HV, int K, int V) {
  const long nc = varlen_chunks(cu_seqlens, N, nullptr, nullptr);
  if (nc < 0 || H < 1 || HV < 1 || HV % H || K != 128 || V != 128) return 0;
  return VarlenLayout(nc, N, cu_seqlens[N], H, HV).total;
}

int kda_bwd_varlen(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const float* S0, const void* dO, const float* dS_T, float scale, const int* cu_seqlens, int N,
                   int H, int HV, int K, int V, int dtype, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                   float* dS0, void* workspace, size_t workspace_bytes, int flags, void* stream) {
  g_err[0] = 0;
  std::vector<int> tab, seq0;
  const long nc = varlen_chunks(cu_seqlens, N, &tab, &seq0);
  if (nc < 0)
    return set_error(KDA_ERR_ARG, "kda_bwd_varlen: cu_seqlens must start at 0 and be non-decreasing (N >= 1)");
  const int T = cu_seqlens[N];
  int rc = check_common("kda_bwd_varlen", N, T > 0 ? T : 1, H, HV, K, V, dtype, scale);
  if (rc) return rc;
  if (T > 0 && (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta))
    return set_error(KDA_ERR_NULL,
                     "kda_bwd_varlen: q, k, v, g, beta, dO, dq, dk, dv, dg and dbeta must be non-NULL");
  if (flags & ~KDA_BWD_STATES_FROM_FWD) return set_error(KDA_ERR_ARG, "kda_bwd_varlen: unknown flags");
  if (K != 128 || V != 128 || dtype != KDA_DTYPE_BF16)
    return set_error(KDA_ERR_ARG, "kda_bwd_varlen: packed sequences run on the tensor-core path only (bf16, K = V = 128)");
  const VarlenLayout lay(nc, N, T, H, HV);
  if (!workspace || workspace_bytes < lay.total)
    return set_error(KDA_ERR_WORKSPACE, "kda_bwd_varlen: workspace smaller than kda_bwd_varlen_workspace_bytes()");
  if (!aligned16(workspace)) return set_error(KDA_ERR_ARG, "kda_bwd_varlen: workspace must be 16-byte aligned");
  char* ws = static_cast<char*>(workspace);
  const int* ctab = reinterpret_cast<const int*>(ws);
  float* states = reinterpret_cast<float*>(ws + lay.table);
  float* inter = reinterpret_cast<float*>(ws + lay.table + lay.states);
  char* x = ws + lay.table + lay.states + lay.inter;
  float* dstates = reinterpret_cast<float*>(x);
  float *dq_part = nullptr, *dk_part = nullptr;
  size_t off = lay.states;
  if (HV > H) {
    dq_part = reinterpret_cast<float*>(x + off);
    dk_part = dq_part + (size_t)T * HV * K;
    off += 2 * (size_t)T * HV * K * sizeof(float);
  }
  float* gws = reinterpret_cast<float*>(x + off);
  BwdArgs a{q, k, v, dO, g, beta, dS_T, states, inter, dstates, dq, dk, dv, dg, dbeta, dS0,
            dq_part, dk_part, gws, scale, N, T, H, HV, K, V, ctab, ctab + 2 * nc, (int)nc};
  FwdArgs fa{q, k, v, g, beta, S0, nullptr, nullptr, states, inter, reinterpret_cast<unsigned char*>(x), scale,
             N, T, H, HV, K, V, ctab, ctab + 2 * nc, (int)nc};
  if (!bwd_tc_eligible(a, dtype) || !fwd_tc_eligible(fa, dtype))
    return set_error(KDA_ERR_ARG, "kda_bwd_varlen: the tensor-core path needs 16-byte aligned q, k, v, dO, g, dq, dv");
  std::vector<int> host(tab);
  host.insert(host.end(), seq0.begin(), seq0.end());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(ws, host.data(), host.size() * sizeof(int), cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return set_cuda_error("kda_bwd_varlen: chunk table upload", e);
  if (!(flags & KDA_BWD_STATES_FROM_FWD)) {
    rc = launch_fwd_tc(fa, st);
    if (rc) return rc;
  }
  return launch_bwd(a, dtype, st);
}

int kda_decode_step(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, float* S, float scale, int B, int H, int HV, int K, int V,
                    int dtype, void* o, void* stream) {
  g_err[0] = 0;
  int rc = check_common("kda_decode_step", B, 1, H, HV, K, V, dtype, scale);
  if (rc) return rc;
  if (!q || !k || !v || !g || !beta || !S || !o)
    return set_error(KDA_ERR_NULL, "kda_decode_step: q, k, v, g, beta, S and o must be non-NULL");
  if (!aligned16(S)) return set_error(KDA_ERR_ARG, "kda_decode_step: S must be 16-byte aligned");
  DecodeArgs a{q, k, v, g, beta, S, o, scale, B, H, HV};
  return launch_decode(a, K, V, dtype, static_cast<cudaStream_t>(stream));
}

size_t kda_fwd_erase_workspace_bytes(int B, int T, int HQ, int HV, int K, int V) {
  if (B < 1 || T < 1 || HQ < 1 || HV < 1 || HQ % HV || V < 1 || (K != 32 && K != 64 && K != 128)) return 0;
  return fma_split_bytes(B, T, HQ, HV, K, V);
}

int kda_fwd_erase(const void* q, const void* k, const void* e, const void* z, const float* g, const float* S0,
                  float scale, int B, int T, int HQ, int HV, int K, int V, int dtype, void* o, float* S_T,
                  void* workspace, size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  char buf[256];
  int rc = check_common("kda_fwd_erase", B, T, 1, 1, K, V, dtype, scale);
  if (rc) return rc;
  if (HQ < 1 || HV < 1 || HQ % HV || HQ > 65535) {
    snprintf(buf, sizeof(buf), "kda_fwd_erase: HQ=%d must be a positive multiple of HV=%d (<= 65535)", HQ, HV);
    return set_error(KDA_ERR_SHAPE, buf);
  }
  if (!q || !k || !e || !z || !g || !o)
    return set_error(KDA_ERR_NULL, "kda_fwd_erase: q, k, e, z, g and o must be non-NULL");
  FwdArgs a{q, k, z, g, nullptr, S0, o, S_T, nullptr, nullptr, nullptr, scale, B, T, HQ, HV, K, V};
  a.erase = e;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (workspace) {
    if (workspace_bytes < kda_fwd_erase_workspace_bytes(B, T, HQ, HV, K, V))
      return set_error(KDA_ERR_WORKSPACE, "kda_fwd_erase: workspace smaller than kda_fwd_erase_workspace_bytes()");
    if (fwd_fma2_eligible(a, workspace)) return launch_fwd_fma2(a, dtype, true, static_cast<float*>(workspace), st);
  }
  return launch_fwd_erase(a, dtype, st);
}

static int check_gate(const char* fn, const void* z, const float* A_log, const float* dt_bias, float lb,
                      const float* beta_logit) {
  char buf[256];
  if (!z || !A_log || !dt_bias || !beta_logit) {
    snprintf(buf, sizeof(buf), "%s: z, A_log, dt_bias and beta_logit must be non-NULL", fn);
    return set_error(KDA_ERR_NULL, buf);
  }
  if (!(lb <= 0.f) || !isfinite(lb)) {
    snprintf(buf, sizeof(buf), "%s: gate_lower_bound=%g must be finite and <= 0 (0: no bound)", fn, (double)lb);
    return set_error(KDA_ERR_ARG, buf);
  }
  return KDA_OK;
}

static bool ranges_overlap(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return a && b && x < y + bn && y < x + an;
}

// the tensor-core path of kda_fwd_prep: [T and P images | g (fp32) | fp32 rows for the output gate]
static size_t prep_tc_bytes(int B, int T, int HV, int K, int V) {
  return img_bytes(B, T, HV, K, V) + (size_t)B * T * HV * K * sizeof(float) + (size_t)B * T * HV * V * sizeof(float);
}

size_t kda_fwd_prep_workspace_bytes(int B, int T, int H, int HV, int K, int V, int dtype) {
  if (B < 1 || T < 1 || H < 1 || HV < 1 || K < 1 || V < 1 || HV % H) return 0;
  const size_t tc = (dtype == KDA_DTYPE_BF16 && K == 128 && V == 128) ? prep_tc_bytes(B, T, HV, K, V) : 0;
  const size_t o32 = dtype == KDA_DTYPE_BF16 ? (size_t)B * T * HV * V * sizeof(float) : 0;
  return tc > o32 ? tc : o32;
}

int kda_fwd_prep(const void* q, const void* k, const void* v, const void* z, const float* A_log,
                 const float* dt_bias, float gate_lower_bound, const float* beta_logit, const void* out_gate,
                 float out_eps, const float* S0, float scale, int B, int T, int H, int HV, int K, int V, int dtype,
                 void* o, float* S_T, void* workspace, size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  int rc = check_common("kda_fwd_prep", B, T, H, HV, K, V, dtype, scale);
  if (rc) return rc;
  if (!q || !k || !v || !o) return set_error(KDA_ERR_NULL, "kda_fwd_prep: q, k, v and o must be non-NULL");
  if ((rc = check_gate("kda_fwd_prep", z, A_log, dt_bias, gate_lower_bound, beta_logit))) return rc;
  if (out_gate && (!(out_eps >= 0.f) || !isfinite(out_eps)))
    return set_error(KDA_ERR_ARG, "kda_fwd_prep: out_eps must be finite and >= 0");
  if (workspace && !aligned16(workspace))
    return set_error(KDA_ERR_ARG, "kda_fwd_prep: workspace must be 16-byte aligned");
  FwdArgs a{q, k, v, nullptr, beta_logit, S0, o, S_T, nullptr, nullptr, nullptr, scale, B, T, H, HV, K, V};
  a.prep = PrepArgs{z, A_log, dt_bias, gate_lower_bound};
  a.og = out_gate;
  a.og_eps = out_eps;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fwd_tc_eligible(a, dtype)) {
    if (!workspace || workspace_bytes < prep_tc_bytes(B, T, HV, K, V))
      return launch_fwd_tc(a, st);  // one kernel per (b, hv) carrying the whole pipeline
    // chunk-parallel kernel and state pass: the gate first (element-wise), then the
    // two kernels on g, then the output gate over the fp32 rows
    char* ws = static_cast<char*>(workspace);
    const size_t ib = img_bytes(B, T, HV, K, V), gb = (size_t)B * T * HV * K * sizeof(float);
    float* gbuf = reinterpret_cast<float*>(ws + ib);
    a.img = reinterpret_cast<unsigned char*>(ws);
    a.g = gbuf;
    if (out_gate) a.o32 = reinterpret_cast<float*>(ws + ib + gb);
    rc = launch_prep_gate(z, A_log, dt_bias, gate_lower_bound, gbuf, (size_t)B * T, HV, st);
    if (!rc) rc = launch_fwd_tc(a, st);
    if (!rc && out_gate) rc = launch_out_gate(a.o32, out_gate, out_eps, (size_t)B * T * HV, V, dtype, o, st);
    return rc;
  }
  if (out_gate) {  // the CUDA-core forward stores fp32 o for the gate pass (in place for fp32)
    if (dtype == KDA_DTYPE_FP32) {
      a.o32 = static_cast<float*>(o);
    } else {
      if (!workspace || workspace_bytes < (size_t)B * T * HV * V * sizeof(float))
        return set_error(KDA_ERR_WORKSPACE, "kda_fwd_prep: the output gate of this shape needs "
                                            "kda_fwd_prep_workspace_bytes() of workspace");
      a.o32 = static_cast<float*>(workspace);
    }
  }
  return launch_fwd_ffma(a, dtype, st);
}

int kda_short_conv(const void* xq, const void* xk, const void* xv, const float* w, const float* state_in,
                   float* state_out, int B, int T, int H, int HV, int K, int V, int W, int dtype, void* q,
                   void* k, void* v, void* stream) {
  g_err[0] = 0;
  int rc = check_common("kda_short_conv", B, T, H, HV, K, V, dtype, 1.f);
  if (rc) return rc;
  if (!xq || !xk || !xv || !w || !q || !k || !v)
    return set_error(KDA_ERR_NULL, "kda_short_conv: xq, xk, xv, w, q, k and v must be non-NULL");
  if (W < 1 || W > 8) return set_error(KDA_ERR_ARG, "kda_short_conv: W must be in 1..8");
  if ((long long)T > 65535LL * 32)  // blocks of 32 steps on gridDim.y
    return set_error(KDA_ERR_SHAPE, "kda_short_conv: T above 2097120 steps exceeds the launch grid");
  const size_t cn = (size_t)2 * H * K + (size_t)HV * V, win = (size_t)B * cn * W * sizeof(float);
  if (ranges_overlap(state_in, win, state_out, win))
    return set_error(KDA_ERR_ARG, "kda_short_conv: state_out must not overlap state_in");
  const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4, nqk = (size_t)B * T * H * K * es, nv = (size_t)B * T * HV * V * es;
  const void* ins[3] = {xq, xk, xv};
  const void* outs[3] = {q, k, v};
  const size_t ns[3] = {nqk, nqk, nv};
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j)
      if (ranges_overlap(ins[i], ns[i], outs[j], ns[j]))
        return set_error(KDA_ERR_ARG, "kda_short_conv: the outputs must not alias the inputs");
  ConvArgs a{xq, xk, xv, w, state_in, state_out, q, k, v, B, T, H, HV, K, V, W};
  return launch_short_conv(a, dtype, static_cast<cudaStream_t>(stream));
}

int kda_decode_token(const void* xq, const void* xk, const void* xv, const float* conv_w, const float* conv_in,
                     float* conv_out, int W, const void* z, const float* A_log, const float* dt_bias,
                     float gate_lower_bound, const float* beta_logit, const void* out_gate, float out_eps, float* S,
                     float scale, int B, int H, int HV, int K, int V, int dtype, void* o, void* stream) {
  g_err[0] = 0;
  int rc = check_common("kda_decode_token", B, 1, H, HV, K, V, dtype, scale);
  if (rc) return rc;
  if (!xq || !xk || !xv || !conv_w || !conv_out || !S || !o)
    return set_error(KDA_ERR_NULL, "kda_decode_token: xq, xk, xv, conv_w, conv_out, S and o must be non-NULL");
  if ((rc = check_gate("kda_decode_token", z, A_log, dt_bias, gate_lower_bound, beta_logit))) return rc;
  if (W < 1 || W > 8) return set_error(KDA_ERR_ARG, "kda_decode_token: W must be in 1..8");
  if (out_gate && (!(out_eps >= 0.f) || !isfinite(out_eps)))
    return set_error(KDA_ERR_ARG, "kda_decode_token: out_eps must be finite and >= 0");
  if (!aligned16(S)) return set_error(KDA_ERR_ARG, "kda_decode_token: S must be 16-byte aligned");
  const size_t win = (size_t)B * (2 * (size_t)H * K + (size_t)HV * V) * W * sizeof(float);
  if (H != HV && ranges_overlap(conv_in, win, conv_out, win))
    return set_error(KDA_ERR_ARG, "kda_decode_token: conv_out may overlap conv_in only when H == HV");
  if (conv_in && conv_in != conv_out && ranges_overlap(conv_in, win, conv_out, win))
    return set_error(KDA_ERR_ARG, "kda_decode_token: conv_out must equal conv_in or not overlap it");
  DecodeTokenArgs a{xq, xk, xv, conv_w, conv_in, conv_out, PrepArgs{z, A_log, dt_bias, gate_lower_bound},
                    beta_logit, out_gate, out_eps, S, o, scale, B, H, HV, W};
  return launch_decode_token(a, K, V, dtype, static_cast<cudaStream_t>(stream));
}

int kda_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
            const float* S0, const void* dO, const float* dS_T, float scale, int B, int T, int H,
            int HV, int K, int V, int dtype, void* dq, void* dk, void* dv, float* dg,
            float* dbeta, float* dS0, void* workspace, size_t workspace_bytes, int flags,
            void* stream) {
  g_err[0] = 0;
  int rc = check_common("kda_bwd", B, T, H, HV, K, V, dtype, scale);
  if (rc) return rc;
  if (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta)
    return set_error(KDA_ERR_NULL,
                     "kda_bwd: q, k, v, g, beta, dO, dq, dk, dv, dg and dbeta must be non-NULL");
  if (flags & ~KDA_BWD_STATES_FROM_FWD) return set_error(KDA_ERR_ARG, "kda_bwd: unknown flags");
  if (!workspace) return set_error(KDA_ERR_WORKSPACE, "kda_bwd: workspace is required");
  if (workspace_bytes < kda_bwd_workspace_bytes(B, T, H, HV, K, V))
    return set_error(KDA_ERR_WORKSPACE, "kda_bwd: workspace smaller than kda_bwd_workspace_bytes()");
  if (!aligned16(workspace)) return set_error(KDA_ERR_ARG, "kda_bwd: workspace must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t sb = states_bytes(B, T, HV, K, V);
  char* ws = static_cast<char*>(workspace);
  float* states = reinterpret_cast<float*>(ws);
  const size_t ib = inter_bytes(B, T, HV, K, V);
  float* inter = ib ? reinterpret_cast<float*>(ws + sb) : nullptr;
  unsigned char* img = img_bytes(B, T, HV, K, V) ? reinterpret_cast<unsigned char*>(ws + sb + ib) : nullptr;
  float* dstates = reinterpret_cast<float*>(ws + sb + ib);  // over the forward's chunk images
  float *dq_part = nullptr, *dk_part = nullptr;
  size_t off = sb + ib + sb;
  if (HV > H) {
    dq_part = reinterpret_cast<float*>(ws + off);
    dk_part = dq_part + (size_t)B * T * HV * K;
    off += 2 * (size_t)B * T * HV * K * sizeof(float);
  }
  float* gws = grads_record_bytes(B, T, HV, K, V) ? reinterpret_cast<float*>(ws + off) : nullptr;
  BwdArgs a{q, k, v, dO, g, beta, dS_T, states, inter, dstates, dq, dk, dv, dg, dbeta, dS0,
            dq_part, dk_part, gws, scale, B, T, H, HV, K, V};
  FwdArgs fa{q, k, v, g, beta, S0, nullptr, nullptr, states, inter, img, scale, B, T, H, HV, K, V};
  // The tensor-core forward keeps only the state entering each 64-step chunk,
  // which is all the tensor-core backward reads; the CUDA-core backward needs
  // every 32-step state, so it gets them from the CUDA-core forward.
  const bool tc_bwd = bwd_tc_eligible(a, dtype);
  if (!(flags & KDA_BWD_STATES_FROM_FWD) || (!tc_bwd && fwd_tc_eligible(fa, dtype))) {
    rc = tc_bwd ? launch_fwd(fa, dtype, st) : launch_fwd_ffma(fa, dtype, st);
    if (rc) return rc;
  }
  return launch_bwd(a, dtype, st);
}

}  // extern "C"
