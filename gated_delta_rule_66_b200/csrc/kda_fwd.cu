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

template <int K, int C, int VB>
struct FwdSmem {
  static constexpr int LDK = K + 1, LDC = C + 1, LDV = VB + 1;
  static constexpr int oK = 0, oQ = oK + C * LDK, oC = oQ + C * LDK, oE1 = oC + C * LDK,
                       oE2o = oE1 + C * LDK, oE2d = oE2o + BS * LDK, oAh = oE2d + BS * LDK,
                       oT = oAh + C * LDC, oP = oT + C * LDC, oW = oP + C * LDC, oV = oW + BS * LDC,
                       oM = oV + C * LDV, oBeta = oM + K * LDV, oEl = oBeta + C, oFlag = oEl + K,
                       total = oFlag + 4;
  static constexpr size_t bytes = (size_t)total * sizeof(float);
};

template <int K, int C, int VB, typename TIn>
__global__ void __launch_bounds__(NTHREADS, 1)
    kda_fwd_chunk_kernel(FwdArgs a) {
  using S = FwdSmem<K, C, VB>;
  constexpr bool PRECISE = sizeof(TIn) == 4;
  constexpr int LDK = S::LDK, LDC = S::LDC, LDV = S::LDV;
  extern __shared__ float smem[];
  float *sK = smem + S::oK, *sQ = smem + S::oQ, *sC = smem + S::oC, *sE1 = smem + S::oE1,
        *sE2o = smem + S::oE2o, *sE2d = smem + S::oE2d, *sAh = smem + S::oAh, *sT = smem + S::oT,
        *sP = smem + S::oP, *sW = smem + S::oW, *sV = smem + S::oV, *sM = smem + S::oM,
        *sBeta = smem + S::oBeta, *sEl = smem + S::oEl;
  int* sFlag = reinterpret_cast<int*>(smem + S::oFlag);

  const TIn* __restrict__ q = static_cast<const TIn*>(a.q);
  const TIn* __restrict__ k = static_cast<const TIn*>(a.k);
  const TIn* __restrict__ v = static_cast<const TIn*>(a.v);
  TIn* __restrict__ o = static_cast<TIn*>(a.o);
  const int v0 = blockIdx.x * VB, hv = blockIdx.y, b = blockIdx.z;
  const int h = hv / (a.HV / a.H);
  const int T = a.T, V = a.V, NT = (T + C - 1) / C;
  const size_t head = (size_t)b * a.HV + hv;

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
    load_chunk_qkgb<K, C, TIn>(q, k, a.g, a.beta, a.scale, b, t0, L, T, a.H, a.HV, h, hv, sQ, sK,
                               sC, sBeta);
    for (int idx = threadIdx.x; idx < C * VB; idx += NTHREADS) {
      const int i = idx / VB, n = idx % VB;
      sV[i * LDV + n] = (i < L) ? to_f(v[(((size_t)b * T + t0 + i) * a.HV + hv) * V + v0 + n]) : 0.f;
    }
    build_interaction<K, C, PRECISE>(sK, sQ, sC, sE1, sE2o, sE2d, sFlag, sAh, sP);
    invert_unit_lower<C>(sAh, sBeta, sT, sW);

    // decayed operands: sE1 <- k o e^{c_last - c}, sK <- k o e^c, sQ <- q~ o e^c
    for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
      const int i = idx / K, f = idx % K;
      const float c = sC[i * LDK + f], cl = sC[(C - 1) * LDK + f];
      const float e = kexp<PRECISE>(c), ed = kexp<PRECISE>(cl - c);
      const float kk = sK[i * LDK + f];
      sE1[i * LDK + f] = kk * ed;
      sK[i * LDK + f] = kk * e;
      sQ[i * LDK + f] *= e;
    }
    for (int f = threadIdx.x; f < K; f += NTHREADS) sEl[f] = kexp<PRECISE>(sC[(C - 1) * LDK + f]);
    __syncthreads();

    constexpr int TMC = C / 16, TNV = VB / 16, TMK = K / 16;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    {  // R = diag(beta) (V - (K o e^c) M), in place in sV
      float acc[TMC][TNV];
      zero(acc);
      mm(acc, K, [&](int i, int f) { return sK[i * LDK + f]; },
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
          if (i < L) o[(((size_t)b * T + t0 + i) * a.HV + hv) * V + v0 + n] = from_f<TIn>(acc[x][y]);
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
  if (a.S_T) {
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

int launch_fwd(const FwdArgs& a, int dtype, cudaStream_t stream) {
  if (fwd_tc_eligible(a, dtype)) return launch_fwd_tc(a, stream);
  return launch_fwd_ffma(a, dtype, stream);
}

int launch_fwd_ffma(const FwdArgs& a, int dtype, cudaStream_t stream) {
  const bool bf = dtype == 1;
  switch (a.K) {
    case 32: return bf ? launch_fwd_t<32, __nv_bfloat16>(a, stream) : launch_fwd_t<32, float>(a, stream);
    case 64: return bf ? launch_fwd_t<64, __nv_bfloat16>(a, stream) : launch_fwd_t<64, float>(a, stream);
    case 128: return bf ? launch_fwd_t<128, __nv_bfloat16>(a, stream) : launch_fwd_t<128, float>(a, stream);
  }
  return set_error(4, "kda_fwd: unsupported K");
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
