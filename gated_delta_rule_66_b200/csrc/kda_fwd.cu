// Chunk-parallel KDA prefill forward.
//
// One CTA owns one (batch b, value head hv, 32-column slice of V).  The
// columns of the state evolve independently of one another (every step of
// "K3/kda/ops/reference/recurrent.py", naive_kda_fwd, reads and writes a
// state column only through k, q, g and beta of its own row), so a V slice
// carries its own K x VB fp32 state through the whole sequence in shared
// memory and needs nothing from the other slices.  Per chunk of C steps the
// CTA forms the decayed interactions, inverts the unit lower-triangular
// system, and applies the three state contractions (residual, readout,
// state carry) with fp32 FMA on a 16 x 16 thread grid.
#include "kda_chunk.cuh"
#include "kda_internal.h"

namespace kda {

template <int K, int C, int VB, bool ERASE = false>
struct FwdSmem {
  static constexpr int LDK = K + 1, LDC = C + 1, LDV = VB + 1;
  static constexpr int oK = 0, oQ = oK + C * LDK, oC = oQ + C * LDK, oE1 = oC + C * LDK,
                       oE2o = oE1 + C * LDK, oE2d = oE2o + BS * LDK, oAh = oE2d + BS * LDK,
                       oT = oAh + C * LDC, oP = oT + C * LDC, oW = oP + C * LDC, oV = oW + BS * LDC,
                       oM = oV + C * LDV, oBeta = oM + K * LDV, oEl = oBeta + C, oFlag = oEl + K,
                       oR = oFlag + 4, total = oR + (ERASE ? C * LDK : 0);
  static constexpr size_t bytes = (size_t)total * sizeof(float);
};

// The chunk of the asymmetric erase/write variant: q~ = scale q of query head
// hq, the write keys k, erase rows e and decay g of state head hv (rows past
// the sequence end zero), beta = 1; then g is replaced by its cumulative sum.
template <int K, int C, typename TIn>
__device__ __forceinline__ void load_chunk_erase(const FwdArgs& a, int b, int t0, int L, int hq, int hv, float* sQ,
                                                 float* sK, float* sR, float* sC, float* sBeta) {
  constexpr int LDK = K + 1;
  const TIn* q = static_cast<const TIn*>(a.q);
  const TIn* k = static_cast<const TIn*>(a.k);
  const TIn* e = static_cast<const TIn*>(a.erase);
  for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K;
    float qv = 0.f, kv = 0.f, ev = 0.f, gv = 0.f;
    if (i < L) {
      const size_t t = (size_t)b * a.T + t0 + i;
      qv = to_f(q[(t * a.H + hq) * K + f]) * a.scale;
      kv = to_f(k[(t * a.HV + hv) * K + f]);
      ev = to_f(e[(t * a.HV + hv) * K + f]);
      gv = a.g[(t * a.HV + hv) * K + f];
    }
    sQ[i * LDK + f] = qv;
    sK[i * LDK + f] = kv;
    sR[i * LDK + f] = ev;
    sC[i * LDK + f] = gv;
  }
  for (int i = threadIdx.x; i < C; i += NTHREADS) sBeta[i] = 1.f;
  __syncthreads();
  for (int f = threadIdx.x; f < K; f += NTHREADS) {
    float run = 0.f;
    for (int i = 0; i < C; ++i) {
      run += sC[i * LDK + f];
      sC[i * LDK + f] = run;
    }
  }
  __syncthreads();
}

// ERASE: the asymmetric erase/write variant ("research_layers.py",
// delta_recurrence): blockIdx.y is the query head hq, which carries (a copy
// of) the recurrence of state head hv = hq / (H / HV) and reads it out; the
// erase rows take k's place in the interaction Ah and in the residual.
template <int K, int C, int VB, typename TIn, bool ERASE = false>
__global__ void __launch_bounds__(NTHREADS, 1)
    kda_fwd_chunk_kernel(FwdArgs a) {
  using S = FwdSmem<K, C, VB, ERASE>;
  constexpr bool PRECISE = sizeof(TIn) == 4;
  constexpr int LDK = S::LDK, LDC = S::LDC, LDV = S::LDV;
  extern __shared__ float smem[];
  float *sK = smem + S::oK, *sQ = smem + S::oQ, *sC = smem + S::oC, *sE1 = smem + S::oE1,
        *sE2o = smem + S::oE2o, *sE2d = smem + S::oE2d, *sAh = smem + S::oAh, *sT = smem + S::oT,
        *sP = smem + S::oP, *sW = smem + S::oW, *sV = smem + S::oV, *sM = smem + S::oM,
        *sBeta = smem + S::oBeta, *sEl = smem + S::oEl, *sR = ERASE ? smem + S::oR : nullptr;
  int* sFlag = reinterpret_cast<int*>(smem + S::oFlag);

  const TIn* __restrict__ q = static_cast<const TIn*>(a.q);
  const TIn* __restrict__ k = static_cast<const TIn*>(a.k);
  const TIn* __restrict__ v = static_cast<const TIn*>(a.v);
  TIn* __restrict__ o = static_cast<TIn*>(a.o);
  const int v0 = blockIdx.x * VB, b = blockIdx.z;
  const int hq = blockIdx.y, hv = ERASE ? hq / (a.H / a.HV) : hq;  // (query head = value head for KDA)
  const int h = ERASE ? 0 : hv / (a.HV / a.H);
  const int T = a.T, V = a.V, NT = (T + C - 1) / C;
  const size_t head = (size_t)b * a.HV + hv;
  const int HO = ERASE ? a.H : a.HV, ho = hq;  // heads of o, this CTA's head in o
  const bool writes_state = !ERASE || hq % (a.H / a.HV) == 0;

  // entering state
  for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
    const int f = idx / VB, n = idx % VB;
    sM[f * LDV + n] = a.S0 ? a.S0[(head * K + f) * V + v0 + n] : 0.f;
  }

  for (int ch = 0; ch < NT; ++ch) {
    const int t0 = ch * C, L = min(C, T - t0);
    __syncthreads();
    if (a.states) {
      float* dst = a.states + ((head * NT + ch) * K) * V;
      for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
        const int f = idx / VB, n = idx % VB;
        dst[(size_t)f * V + v0 + n] = sM[f * LDV + n];
      }
    }
    if constexpr (ERASE)
      load_chunk_erase<K, C, TIn>(a, b, t0, L, hq, hv, sQ, sK, sR, sC, sBeta);
    else
      load_chunk_qkgb<K, C, TIn>(q, k, a.g, a.beta, a.scale, b, t0, L, T, a.H, a.HV, h, hv, sQ, sK,
                                 sC, sBeta, static_cast<const TIn*>(a.prep.z), a.prep.A_log, a.prep.dt_bias,
                                 a.prep.gate_lb);
    for (int idx = threadIdx.x; idx < C * VB; idx += NTHREADS) {
      const int i = idx / VB, n = idx % VB;
      sV[i * LDV + n] = (i < L) ? to_f(v[(((size_t)b * T + t0 + i) * a.HV + hv) * V + v0 + n]) : 0.f;
    }
    build_interaction<K, C, PRECISE>(sK, sQ, sC, sE1, sE2o, sE2d, sFlag, sAh, sP, sR);
    invert_unit_lower<C>(sAh, sBeta, sT, sW);

    // decayed operands: sE1 <- k o e^{c_last - c}, sK <- k o e^c, sQ <- q~ o e^c
    for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
      const int i = idx / K, f = idx % K;
      const float c = sC[i * LDK + f], cl = sC[(C - 1) * LDK + f];
      const float e = kexp<PRECISE>(c), ed = kexp<PRECISE>(cl - c);
      const float kk = sK[i * LDK + f];
      sE1[i * LDK + f] = kk * ed;
      if constexpr (ERASE) sR[i * LDK + f] *= e;  // the residual reads the erase rows
      else sK[i * LDK + f] = kk * e;
      sQ[i * LDK + f] *= e;
    }
    for (int f = threadIdx.x; f < K; f += NTHREADS) sEl[f] = kexp<PRECISE>(sC[(C - 1) * LDK + f]);
    __syncthreads();

    constexpr int TMC = C / 16, TNV = VB / 16, TMK = K / 16;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    {  // R = diag(beta) (V - (K o e^c) M), in place in sV
      float acc[TMC][TNV];
      zero(acc);
      const float* sRes = ERASE ? sR : sK;
      mm(acc, K, [&](int i, int f) { return sRes[i * LDK + f]; },
         [&](int f, int n) { return sM[f * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const int i = ty + 16 * x, n = tx + 16 * y;
          sV[i * LDV + n] = sBeta[i] * (sV[i * LDV + n] - acc[x][y]);
        }
    }
    __syncthreads();
    {  // U = T R, in place
      float acc[TMC][TNV];
      zero(acc);
      mm(acc, C, [&](int i, int j) { return sT[i * LDC + j]; },
         [&](int j, int n) { return sV[j * LDV + n]; });
      __syncthreads();
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) sV[(ty + 16 * x) * LDV + tx + 16 * y] = acc[x][y];
    }
    __syncthreads();
    if (a.o) {  // O = (Q~ o e^c) M + P U
      float acc[TMC][TNV];
      zero(acc);
      mm(acc, K, [&](int i, int f) { return sQ[i * LDK + f]; },
         [&](int f, int n) { return sM[f * LDV + n]; });
      mm(acc, C, [&](int i, int j) { return sP[i * LDC + j]; },
         [&](int j, int n) { return sV[j * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const int i = ty + 16 * x, n = tx + 16 * y;
          if (i < L) {
            const size_t at = (((size_t)b * T + t0 + i) * HO + ho) * V + v0 + n;
            if (a.o32) a.o32[at] = acc[x][y];  // fp32 for the output-gate pass
            else o[at] = from_f<TIn>(acc[x][y]);
          }
        }
    }
    {  // M' = diag(e^{c_last}) M + (K o e^{c_last - c})^T U
      float acc[TMK][TNV];
#pragma unroll
      for (int x = 0; x < TMK; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const int f = ty + 16 * x, n = tx + 16 * y;
          acc[x][y] = sEl[f] * sM[f * LDV + n];
        }
      mm(acc, C, [&](int f, int i) { return sE1[i * LDK + f]; },
         [&](int i, int n) { return sV[i * LDV + n]; });
      __syncthreads();
#pragma unroll
      for (int x = 0; x < TMK; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) sM[(ty + 16 * x) * LDV + tx + 16 * y] = acc[x][y];
    }
  }
  __syncthreads();
  if (a.S_T && writes_state) {
    for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
      const int f = idx / VB, n = idx % VB;
      a.S_T[(head * K + f) * V + v0 + n] = sM[f * LDV + n];
    }
  }
}

template <int K, typename TIn>
static int launch_fwd_t(const FwdArgs& a, cudaStream_t stream) {
  constexpr int C = FWD_CHUNK, VB = FWD_VBLOCK;
  using S = FwdSmem<K, C, VB>;
  auto kern = kda_fwd_chunk_kernel<K, C, VB, TIn>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::bytes);
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: cudaFuncSetAttribute", e);
  dim3 grid(a.V / VB, a.HV, a.B);
  kern<<<grid, NTHREADS, S::bytes, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: launch", e);
  return 0;
}

template <int K, typename TIn>
static int launch_fwd_erase_t(const FwdArgs& a, cudaStream_t stream) {
  constexpr int C = FWD_CHUNK, VB = FWD_VBLOCK;
  using S = FwdSmem<K, C, VB, true>;
  auto kern = kda_fwd_chunk_kernel<K, C, VB, TIn, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::bytes);
  if (e != cudaSuccess) return set_cuda_error("kda_fwd_erase: cudaFuncSetAttribute", e);
  kern<<<dim3(a.V / VB, a.H, a.B), NTHREADS, S::bytes, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_fwd_erase: launch", e);
  return 0;
}

int launch_fwd_erase(const FwdArgs& a, int dtype, cudaStream_t stream) {
  const bool bf = dtype == 1;
  switch (a.K) {
    case 32: return bf ? launch_fwd_erase_t<32, __nv_bfloat16>(a, stream) : launch_fwd_erase_t<32, float>(a, stream);
    case 64: return bf ? launch_fwd_erase_t<64, __nv_bfloat16>(a, stream) : launch_fwd_erase_t<64, float>(a, stream);
    case 128: return bf ? launch_fwd_erase_t<128, __nv_bfloat16>(a, stream) : launch_fwd_erase_t<128, float>(a, stream);
  }
  return set_error(4, "kda_fwd_erase: unsupported K");
}

int launch_fwd(const FwdArgs& a, int dtype, cudaStream_t stream) {
  if (fwd_tc_eligible(a, dtype)) return launch_fwd_tc(a, stream);
  return launch_fwd_ffma(a, dtype, stream);
}

int launch_fwd_ffma(const FwdArgs& a, int dtype, cudaStream_t stream) {
  const bool bf = dtype == 1;
  int rc = 4;
  switch (a.K) {
    case 32: rc = bf ? launch_fwd_t<32, __nv_bfloat16>(a, stream) : launch_fwd_t<32, float>(a, stream); break;
    case 64: rc = bf ? launch_fwd_t<64, __nv_bfloat16>(a, stream) : launch_fwd_t<64, float>(a, stream); break;
    case 128: rc = bf ? launch_fwd_t<128, __nv_bfloat16>(a, stream) : launch_fwd_t<128, float>(a, stream); break;
    default: return set_error(4, "kda_fwd: unsupported K");
  }
  if (rc || !a.o || !a.o32) return rc;
  // the output gate needs whole rows of V; the chunk kernel's CTAs own V slices
  return launch_out_gate(a.o32, a.og, a.og_eps, (size_t)a.B * a.T * a.HV, a.V, dtype, a.o, stream);
}

// "kimi_k3_host/kda.rs", full_rank_output_gate: one warp per (step, value
// head) row of V values: o = sigmoid(og) o32 / sqrt(mean(o32^2) + eps).
template <typename TIn>
__global__ void __launch_bounds__(256) kda_out_gate_kernel(const float* __restrict__ o32,
                                                           const TIn* __restrict__ og, float eps, size_t rows,
                                                           int V, TIn* __restrict__ o) {
  const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* src = o32 + row * V;
  float x[4], s = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int n = lane + 32 * u;
    x[u] = n < V ? src[n] : 0.f;
    s = fmaf(x[u], x[u], s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float inv = rsqrtf(s / (float)V + eps);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int n = lane + 32 * u;
    if (n < V) o[row * V + n] = from_f<TIn>(x[u] * inv * prep_sigmoid(to_f(og[row * V + n])));
  }
}

int launch_out_gate(const float* o32, const void* og, float eps, size_t rows, int V, int dtype, void* o,
                    cudaStream_t stream) {
  if (rows == 0) return 0;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (dtype == 1)
    kda_out_gate_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
        o32, static_cast<const __nv_bfloat16*>(og), eps, rows, V, static_cast<__nv_bfloat16*>(o));
  else
    kda_out_gate_kernel<float><<<blocks, 256, 0, stream>>>(o32, static_cast<const float*>(og), eps, rows, V,
                                                           static_cast<float*>(o));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: output-gate launch", e);
  return 0;
}

size_t fwd_smem_bytes(int K) {
  switch (K) {
    case 32: return FwdSmem<32, FWD_CHUNK, FWD_VBLOCK>::bytes;
    case 64: return FwdSmem<64, FWD_CHUNK, FWD_VBLOCK>::bytes;
    case 128: return FwdSmem<128, FWD_CHUNK, FWD_VBLOCK>::bytes;
  }
  return 0;
}

}  // namespace kda
