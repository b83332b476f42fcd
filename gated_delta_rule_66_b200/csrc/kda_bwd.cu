// Chunked KDA backward.
//
// Definition: the BPTT of "K3/kda/ops/reference/recurrent.py",
// KDAFunction.backward (dS += q~ (x) do; dq~ = S_t do; da = dS r; dr = a^T dS;
// dbeta = k . da; dk = beta da - S_dec dr; dv = dr; dS_dec = dS - k (x) dr;
// dg = sum_v S_dec o dS_dec; dS <- e^g o dS_dec), grouped-head sums for dq/dk
// and the scale on dq, plus dS0 (the accumulator after t = 0).
//
// The same gradients are taken here chunk by chunk from the chunk algebra
// of kda_chunk.cuh, in three launches:
//   1. state pass: the forward kernel stores the state entering every chunk
//      (skipped when the caller's kda_fwd already wrote them);
//   2. state-gradient pass (this file, one CTA per (b, hv, 32 V columns),
//      chunks in reverse): dM_in = diag(e^{c_last}) dM_out + (Q~ o e^c)^T dO
//      - (K o e^c)^T diag(beta) T^T (P^T dO + (K o e^{c_last-c}) dM_out).
//      It needs no forward state; it stores dM_out of every chunk and
//      returns dS0 = dM_in of chunk 0;
//   3. per-chunk gradients (this file, one CTA per (b, hv, chunk), all
//      chunks in parallel): recompute U from the stored entering state, form
//      dU, dR, dv, dbeta, the C x C adjoints dP and dA, the adjoints of the
//      decayed operands, map them back to dq, dk and the in-chunk decay
//      adjoint dc, and reverse-cumsum dc into dg.
#include "kda_asm.cuh"
#include "kda_chunk.cuh"
#include "kda_internal.h"

namespace kda {

template <int K, int C, int VB>
struct DstSmem {
  static constexpr int LDK = K + 1, LDC = C + 1, LDV = VB + 1;
  static constexpr int oK = 0, oQ = oK + C * LDK, oC = oQ + C * LDK, oE1 = oC + C * LDK,
                       oE2o = oE1 + C * LDK, oE2d = oE2o + BS * LDK, oAh = oE2d + BS * LDK,
                       oT = oAh + C * LDC, oP = oT + C * LDC, oW = oP + C * LDC,
                       odO = oW + BS * LDC, odU = odO + C * LDV, odM = odU + C * LDV,
                       oBeta = odM + K * LDV, oEl = oBeta + C, oFlag = oEl + K, total = oFlag + 4;
  static constexpr size_t bytes = (size_t)total * sizeof(float);
};

template <int K, int C, int VB, typename TIn>
__global__ void __launch_bounds__(NTHREADS, 1) kda_bwd_dstate_kernel(BwdArgs a) {
  using S = DstSmem<K, C, VB>;
  constexpr bool PRECISE = sizeof(TIn) == 4;
  constexpr int LDK = S::LDK, LDC = S::LDC, LDV = S::LDV;
  extern __shared__ float smem[];
  float *sK = smem + S::oK, *sQ = smem + S::oQ, *sC = smem + S::oC, *sE1 = smem + S::oE1,
        *sE2o = smem + S::oE2o, *sE2d = smem + S::oE2d, *sAh = smem + S::oAh, *sT = smem + S::oT,
        *sP = smem + S::oP, *sW = smem + S::oW, *sdO = smem + S::odO, *sdU = smem + S::odU,
        *sdM = smem + S::odM, *sBeta = smem + S::oBeta, *sEl = smem + S::oEl;
  int* sFlag = reinterpret_cast<int*>(smem + S::oFlag);
  const TIn* __restrict__ q = static_cast<const TIn*>(a.q);
  const TIn* __restrict__ k = static_cast<const TIn*>(a.k);
  const TIn* __restrict__ dO = static_cast<const TIn*>(a.dO);
  const int v0 = blockIdx.x * VB, hv = blockIdx.y, b = blockIdx.z;
  const int h = hv / (a.HV / a.H);
  const int T = a.T, V = a.V, NT = (T + C - 1) / C;
  const size_t head = (size_t)b * a.HV + hv;

  for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
    const int f = idx / VB, n = idx % VB;
    sdM[f * LDV + n] = a.dS_T ? a.dS_T[(head * K + f) * V + v0 + n] : 0.f;
  }
  for (int ch = NT - 1; ch >= 0; --ch) {
    const int t0 = ch * C, L = min(C, T - t0);
    __syncthreads();
    {
      float* dst = a.dstates + ((head * NT + ch) * K) * V;
      for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
        const int f = idx / VB, n = idx % VB;
        dst[(size_t)f * V + v0 + n] = sdM[f * LDV + n];
      }
    }
    load_chunk_qkgb<K, C, TIn>(q, k, a.g, a.beta, a.scale, b, t0, L, T, a.H, a.HV, h, hv, sQ, sK,
                               sC, sBeta);
    for (int idx = threadIdx.x; idx < C * VB; idx += NTHREADS) {
      const int i = idx / VB, n = idx % VB;
      sdO[i * LDV + n] = (i < L) ? to_f(dO[(((size_t)b * T + t0 + i) * a.HV + hv) * V + v0 + n]) : 0.f;
    }
    build_interaction<K, C, PRECISE>(sK, sQ, sC, sE1, sE2o, sE2d, sFlag, sAh, sP);
    invert_unit_lower<C>(sAh, sBeta, sT, sW);
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
    {  // dU = P^T dO + (K o e^{c_last-c}) dM_out
      float acc[TMC][TNV];
      zero(acc);
      mm(acc, C, [&](int i, int j) { return sP[j * LDC + i]; },
         [&](int j, int n) { return sdO[j * LDV + n]; });
      mm(acc, K, [&](int i, int f) { return sE1[i * LDK + f]; },
         [&](int f, int n) { return sdM[f * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) sdU[(ty + 16 * x) * LDV + tx + 16 * y] = acc[x][y];
    }
    __syncthreads();
    {  // dX = diag(beta) T^T dU, in place
      float acc[TMC][TNV];
      zero(acc);
      mm(acc, C, [&](int i, int j) { return sT[j * LDC + i]; },
         [&](int j, int n) { return sdU[j * LDV + n]; });
      __syncthreads();
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const int i = ty + 16 * x;
          sdU[i * LDV + tx + 16 * y] = sBeta[i] * acc[x][y];
        }
    }
    __syncthreads();
    {  // dM_in = diag(e^{c_last}) dM_out + (Q~ o e^c)^T dO - (K o e^c)^T dX
      float acc[TMK][TNV];
#pragma unroll
      for (int x = 0; x < TMK; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const int f = ty + 16 * x, n = tx + 16 * y;
          acc[x][y] = sEl[f] * sdM[f * LDV + n];
        }
      mm(acc, C, [&](int f, int i) { return sQ[i * LDK + f]; },
         [&](int i, int n) { return sdO[i * LDV + n]; });
      mm(acc, C, [&](int f, int i) { return -sK[i * LDK + f]; },
         [&](int i, int n) { return sdU[i * LDV + n]; });
      __syncthreads();
#pragma unroll
      for (int x = 0; x < TMK; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) sdM[(ty + 16 * x) * LDV + tx + 16 * y] = acc[x][y];
    }
  }
  __syncthreads();
  if (a.dS0) {
    for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
      const int f = idx / VB, n = idx % VB;
      a.dS0[(head * K + f) * V + v0 + n] = sdM[f * LDV + n];
    }
  }
}

template <int K, int C, int VB>
struct GradSmem {
  static constexpr int LDK = K + 1, LDC = C + 1, LDV = VB + 1;
  static constexpr int oK = 0, oQ = oK + C * LDK, oC = oQ + C * LDK, oE = oC + C * LDK,
                       oEd = oE + C * LDK, oAh = oEd + C * LDK, oT = oAh + C * LDC,
                       oP = oT + C * LDC, odA = oP + C * LDC, odP = odA + C * LDC,
                       oW = odP + C * LDC, odQE = oW + BS * LDC, odKE = odQE + C * LDK,
                       odKEd = odKE + C * LDK, oBeta = odKEd + C * LDK, oEl = oBeta + C,
                       odEl = oEl + K, odb = odEl + K, oLast = odb + C, oFlag = oLast + K,
                       oR = oFlag + 4;
  // region R: either the V-block operands or the decay-factor scratch
  static constexpr int rM = 0, rdM = rM + K * LDV, rX = rdM + K * LDV, rdO = rX + C * LDV,
                       rU = rdO + C * LDV, rdU = rU + C * LDV, rEnd1 = rdU + C * LDV;
  static constexpr int rE1 = 0, rE2o = rE1 + C * LDK, rE2d = rE2o + BS * LDK, rEnd2 = rE2d + BS * LDK;
  static constexpr int total = oR + (rEnd1 > rEnd2 ? rEnd1 : rEnd2);
  static constexpr size_t bytes = (size_t)total * sizeof(float);
};

template <int K, int C, int VB, typename TIn>
__global__ void __launch_bounds__(NTHREADS, 1) kda_bwd_grads_kernel(BwdArgs a) {
  using S = GradSmem<K, C, VB>;
  constexpr bool PRECISE = sizeof(TIn) == 4;
  constexpr int LDK = S::LDK, LDC = S::LDC, LDV = S::LDV;
  extern __shared__ float smem[];
  float *sK = smem + S::oK, *sQ = smem + S::oQ, *sC = smem + S::oC, *sE = smem + S::oE,
        *sEd = smem + S::oEd, *sAh = smem + S::oAh, *sT = smem + S::oT, *sP = smem + S::oP,
        *sdA = smem + S::odA, *sdP = smem + S::odP, *sW = smem + S::oW, *sdQE = smem + S::odQE,
        *sdKE = smem + S::odKE, *sdKEd = smem + S::odKEd, *sBeta = smem + S::oBeta,
        *sEl = smem + S::oEl, *sdEl = smem + S::odEl, *sdb = smem + S::odb, *sLast = smem + S::oLast;
  int* sFlag = reinterpret_cast<int*>(smem + S::oFlag);
  float* R = smem + S::oR;
  float *sM = R + S::rM, *sdM = R + S::rdM, *sX = R + S::rX, *sdO = R + S::rdO, *sU = R + S::rU,
        *sdU = R + S::rdU;
  float *sE1 = R + S::rE1, *sE2o = R + S::rE2o, *sE2d = R + S::rE2d;

  const TIn* __restrict__ q = static_cast<const TIn*>(a.q);
  const TIn* __restrict__ k = static_cast<const TIn*>(a.k);
  const TIn* __restrict__ v = static_cast<const TIn*>(a.v);
  const TIn* __restrict__ dO = static_cast<const TIn*>(a.dO);
  const int ch = blockIdx.x, hv = blockIdx.y, b = blockIdx.z;
  const int G = a.HV / a.H, h = hv / G;
  const int T = a.T, V = a.V, NT = (T + C - 1) / C;
  const int t0 = ch * C, L = min(C, T - t0);
  const size_t head = (size_t)b * a.HV + hv;

  load_chunk_qkgb<K, C, TIn>(q, k, a.g, a.beta, a.scale, b, t0, L, T, a.H, a.HV, h, hv, sQ, sK, sC,
                             sBeta);
  build_interaction<K, C, PRECISE>(sK, sQ, sC, sE1, sE2o, sE2d, sFlag, sAh, sP);
  invert_unit_lower<C>(sAh, sBeta, sT, sW);
  for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K;
    const float c = sC[i * LDK + f], cl = sC[(C - 1) * LDK + f];
    sE[i * LDK + f] = kexp<PRECISE>(c);
    sEd[i * LDK + f] = kexp<PRECISE>(cl - c);
    sdQE[i * LDK + f] = 0.f;
    sdKE[i * LDK + f] = 0.f;
    sdKEd[i * LDK + f] = 0.f;
  }
  for (int idx = threadIdx.x; idx < C * C; idx += NTHREADS) {
    const int i = idx / C, j = idx % C;
    sdA[i * LDC + j] = 0.f;
    sdP[i * LDC + j] = 0.f;
  }
  for (int f = threadIdx.x; f < K; f += NTHREADS) {
    sEl[f] = kexp<PRECISE>(sC[(C - 1) * LDK + f]);
    sdEl[f] = 0.f;
  }
  for (int i = threadIdx.x; i < C; i += NTHREADS) sdb[i] = 0.f;

  constexpr int TMC = C / 16, TNV = VB / 16, TNC = C / 16, TNK = K / 16;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* Mg = a.states + ((head * NT + ch) * K) * V;
  const float* dMg = a.dstates + ((head * NT + ch) * K) * V;

  for (int v0 = 0; v0 < V; v0 += VB) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
      const int f = idx / VB, n = idx % VB;
      sM[f * LDV + n] = Mg[(size_t)f * V + v0 + n];
      sdM[f * LDV + n] = dMg[(size_t)f * V + v0 + n];
    }
    for (int idx = threadIdx.x; idx < C * VB; idx += NTHREADS) {
      const int i = idx / VB, n = idx % VB;
      const size_t off = (((size_t)b * T + t0 + i) * a.HV + hv) * V + v0 + n;
      sX[i * LDV + n] = (i < L) ? to_f(v[off]) : 0.f;
      sdO[i * LDV + n] = (i < L) ? to_f(dO[off]) : 0.f;
    }
    __syncthreads();
    {  // X = V - (K o e^c) M, in place
      float acc[TMC][TNV];
      zero(acc);
      mm(acc, K, [&](int i, int f) { return sK[i * LDK + f] * sE[i * LDK + f]; },
         [&](int f, int n) { return sM[f * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) sX[(ty + 16 * x) * LDV + tx + 16 * y] -= acc[x][y];
    }
    __syncthreads();
    {  // U = T diag(beta) X ; dU = P^T dO + (K o e^{c_last-c}) dM_out
      float acc[TMC][TNV], acc2[TMC][TNV];
      zero(acc);
      zero(acc2);
      mm(acc, C, [&](int i, int j) { return sT[i * LDC + j]; },
         [&](int j, int n) { return sBeta[j] * sX[j * LDV + n]; });
      mm(acc2, C, [&](int i, int j) { return sP[j * LDC + i]; },
         [&](int j, int n) { return sdO[j * LDV + n]; });
      mm(acc2, K, [&](int i, int f) { return sK[i * LDK + f] * sEd[i * LDK + f]; },
         [&](int f, int n) { return sdM[f * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          sU[(ty + 16 * x) * LDV + tx + 16 * y] = acc[x][y];
          sdU[(ty + 16 * x) * LDV + tx + 16 * y] = acc2[x][y];
        }
    }
    __syncthreads();
    {  // dR = T^T dU, in place; dv = diag(beta) dR
      float acc[TMC][TNV];
      zero(acc);
      mm(acc, C, [&](int i, int j) { return sT[j * LDC + i]; },
         [&](int j, int n) { return sdU[j * LDV + n]; });
      __syncthreads();
      TIn* dv = static_cast<TIn*>(a.dv);
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const int i = ty + 16 * x, n = tx + 16 * y;
          sdU[i * LDV + n] = acc[x][y];
          if (i < L) dv[(((size_t)b * T + t0 + i) * a.HV + hv) * V + v0 + n] = from_f<TIn>(sBeta[i] * acc[x][y]);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < C; i += NTHREADS) {  // dbeta from the residual
      float s = 0.f;
      for (int n = 0; n < VB; ++n) s = fmaf(sdU[i * LDV + n], sX[i * LDV + n], s);
      sdb[i] += s;
    }
    for (int f = threadIdx.x; f < K; f += NTHREADS) {  // d e^{c_last}
      float s = 0.f;
      for (int n = 0; n < VB; ++n) s = fmaf(sM[f * LDV + n], sdM[f * LDV + n], s);
      sdEl[f] += s;
    }
    {  // dP += dO U^T ; dA -= dR U^T
      float accP[TMC][TNC], accA[TMC][TNC];
      zero(accP);
      zero(accA);
      mm(accP, VB, [&](int i, int n) { return sdO[i * LDV + n]; },
         [&](int n, int j) { return sU[j * LDV + n]; });
      mm(accA, VB, [&](int i, int n) { return sdU[i * LDV + n]; },
         [&](int n, int j) { return sU[j * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNC; ++y) {
          const int i = ty + 16 * x, j = tx + 16 * y;
          sdP[i * LDC + j] += accP[x][y];
          sdA[i * LDC + j] -= accA[x][y];
        }
    }
    {  // dQE += dO M^T ; dKE -= diag(beta) dR M^T ; dKEd += U dM_out^T
      float a1[TMC][TNK], a2[TMC][TNK], a3[TMC][TNK];
      zero(a1);
      zero(a2);
      zero(a3);
      mm(a1, VB, [&](int i, int n) { return sdO[i * LDV + n]; },
         [&](int n, int f) { return sM[f * LDV + n]; });
      mm(a2, VB, [&](int i, int n) { return sdU[i * LDV + n]; },
         [&](int n, int f) { return sM[f * LDV + n]; });
      mm(a3, VB, [&](int i, int n) { return sU[i * LDV + n]; },
         [&](int n, int f) { return sdM[f * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNK; ++y) {
          const int i = ty + 16 * x, f = tx + 16 * y;
          sdQE[i * LDK + f] += a1[x][y];
          sdKE[i * LDK + f] -= sBeta[i] * a2[x][y];
          sdKEd[i * LDK + f] += a3[x][y];
        }
    }
  }
  __syncthreads();

  // dbeta from A; dA_hat = beta_i dA (strict lower); e^{c_last} terms of dc
  for (int i = threadIdx.x; i < C; i += NTHREADS) {
    float s = sdb[i];
    for (int j = 0; j < i; ++j) s = fmaf(sdA[i * LDC + j], sAh[i * LDC + j], s);
    sdb[i] = s;
  }
  for (int f = threadIdx.x; f < K; f += NTHREADS) {
    float s = sdEl[f] * sEl[f];
    for (int i = 0; i < C; ++i) s = fmaf(sdKEd[i * LDK + f], sK[i * LDK + f] * sEd[i * LDK + f], s);
    sLast[f] = s;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < C * C; idx += NTHREADS) {
    const int i = idx / C, j = idx % C;
    sdA[i * LDC + j] = (j < i) ? sdA[i * LDC + j] * sBeta[i] : 0.f;
    if (j > i) sdP[i * LDC + j] = 0.f;
  }
  // elementwise parts: sdQE <- dq~, sdKE <- dk, sdKEd <- dc
  for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K, o = i * LDK + f;
    const float e = sE[o], ed = sEd[o], kk = sK[o], qq = sQ[o];
    const float dqe = sdQE[o], dke = sdKE[o], dked = sdKEd[o];
    sdQE[o] = dqe * e;
    sdKE[o] = dke * e + dked * ed;
    sdKEd[o] = (dqe * qq + dke * kk) * e - dked * kk * ed;
  }
  __syncthreads();
  float *sDq = sdQE, *sDk = sdKE, *sDc = sdKEd;

  factored_terms<K, C, PRECISE, false>(sK, sQ, sC, sdA, sdP, sE1, sE2o, sE2d, sFlag, sDq, sDk, sDc);

  // dg = reverse cumulative sum of dc over the chunk (plus the chunk-end terms)
  for (int f = threadIdx.x; f < K; f += NTHREADS) {
    float run = sLast[f];
    for (int i = C - 1; i >= 0; --i) {
      run += sDc[i * LDK + f];
      sDc[i * LDK + f] = run;
    }
  }
  __syncthreads();
  TIn* dq = static_cast<TIn*>(a.dq);
  TIn* dk = static_cast<TIn*>(a.dk);
  for (int idx = threadIdx.x; idx < L * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K, o = i * LDK + f;
    const size_t row_v = ((size_t)b * T + t0 + i) * a.HV + hv;
    a.dg[row_v * K + f] = sDc[o];
    if (G == 1) {
      const size_t row_h = ((size_t)b * T + t0 + i) * a.H + h;
      dq[row_h * K + f] = from_f<TIn>(a.scale * sDq[o]);
      dk[row_h * K + f] = from_f<TIn>(sDk[o]);
    } else {
      a.dq_part[row_v * K + f] = a.scale * sDq[o];
      a.dk_part[row_v * K + f] = sDk[o];
    }
  }
  for (int i = threadIdx.x; i < L; i += NTHREADS) a.dbeta[((size_t)b * T + t0 + i) * a.HV + hv] = sdb[i];
}

// dq[b,t,h,:] = sum over the G value heads of the group, converted to dtype.
template <typename TIn>
__global__ void kda_group_sum_kernel(const float* __restrict__ part, TIn* __restrict__ out,
                                     size_t rows_h, int H, int G, int K) {
  const size_t n = rows_h * K;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n;
       idx += (size_t)gridDim.x * blockDim.x) {
    const size_t row = idx / K;  // (b*T + t)*H + h
    const int f = (int)(idx % K);
    const size_t bt = row / H;
    const int h = (int)(row % H);
    float s = 0.f;
    for (int j = 0; j < G; ++j) s += part[((bt * H + h) * G + j) * K + f];
    out[idx] = from_f<TIn>(s);
  }
}


template <typename TIn>
__global__ void __launch_bounds__(NTHREADS, 2) kda_bwd_assemble_kernel(BwdArgs a) {
  extern __shared__ float smem[];
  const int head = a.head0 + blockIdx.y;  // (sequence or batch row) * HV + hv
  if (a.pf_items > 0 && (blockIdx.x & 3) == 0) {
    // CTAs start in linear order, so the CTA that follows this one on its SM is
    // about pf_items (a multiple of 4: all CTAs resident at once) further on:
    // the chunk it and its three neighbours assemble goes into L2 now
    const long long nx = (long long)blockIdx.y * gridDim.x + blockIdx.x + a.pf_items;
    if (nx < (long long)gridDim.x * gridDim.y) {
      const int hn = a.head0 + (int)(nx / gridDim.x);
      prefetch_assembly<TIn>(a, (int)(nx % gridDim.x) >> 2, hn % a.HV, hn / a.HV);
    }
  }
  assemble_quarter<TIn>(a, smem, blockIdx.x >> 2, blockIdx.x & 3, head % a.HV, head / a.HV);
}

// The assembly of heads (sequence * HV + hv) head0 .. head0 + nheads - 1.
template <typename TIn>
static int launch_assemble(const BwdArgs& a0, int head0, int nheads, cudaStream_t stream) {
  auto kern = kda_bwd_assemble_kernel<TIn>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AsmSmem::bytes);
  if (e != cudaSuccess) return set_cuda_error("kda_bwd: cudaFuncSetAttribute", e);
  const int NT = a0.ctab ? a0.NC : (a0.T + 63) / 64;
  if (NT == 0 || nheads <= 0) return 0;  // (packed batches of empty sequences)
  BwdArgs a = a0;
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTHREADS, AsmSmem::bytes) != cudaSuccess)
    per_sm = 1;
  a.pf_items = (sms * (per_sm > 0 ? per_sm : 1)) & ~3;
  for (int done = 0; done < nheads; done += 65535) {  // gridDim.y is at most 65535
    a.head0 = head0 + done;
    kern<<<dim3(NT * 4, min(nheads - done, 65535)), NTHREADS, AsmSmem::bytes, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("kda_bwd: assemble launch", e);
  }
  return 0;
}

template <int K, typename TIn>
static int launch_bwd_t(const BwdArgs& a, cudaStream_t stream) {
  constexpr int C = FWD_CHUNK, VB = FWD_VBLOCK;
  const int NT = (a.T + C - 1) / C;
  const bool tc = bwd_tc_eligible(a, sizeof(TIn) == 2 ? 1 : 0);
  if (tc) {
    int rc = launch_bwd_tc_passes(a, stream, launch_assemble<TIn>);
    if (rc) return rc;
  } else {
    using S = DstSmem<K, C, VB>;
    auto kern = kda_bwd_dstate_kernel<K, C, VB, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::bytes);
    if (e != cudaSuccess) return set_cuda_error("kda_bwd: cudaFuncSetAttribute", e);
    kern<<<dim3(a.V / VB, a.HV, a.B), NTHREADS, S::bytes, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("kda_bwd: state-gradient launch", e);
    using S2 = GradSmem<K, C, VB>;
    auto kern2 = kda_bwd_grads_kernel<K, C, VB, TIn>;
    e = cudaFuncSetAttribute(kern2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S2::bytes);
    if (e != cudaSuccess) return set_cuda_error("kda_bwd: cudaFuncSetAttribute", e);
    kern2<<<dim3(NT, a.HV, a.B), NTHREADS, S2::bytes, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("kda_bwd: gradient launch", e);
  }
  if (a.HV > a.H) {
    const int G = a.HV / a.H;
    const size_t rows_h = (size_t)(a.ctab ? 1 : a.B) * a.T * a.H;
    const size_t n = rows_h * a.K;
    if (n == 0) return 0;
    const int blocks = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
    kda_group_sum_kernel<TIn><<<blocks, 256, 0, stream>>>(a.dq_part, static_cast<TIn*>(a.dq), rows_h, a.H, G, a.K);
    kda_group_sum_kernel<TIn><<<blocks, 256, 0, stream>>>(a.dk_part, static_cast<TIn*>(a.dk), rows_h, a.H, G, a.K);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("kda_bwd: group-sum launch", e);
  }
  return 0;
}

int launch_bwd(const BwdArgs& a, int dtype, cudaStream_t stream) {
  const bool bf = dtype == 1;
  switch (a.K) {
    case 32: return bf ? launch_bwd_t<32, __nv_bfloat16>(a, stream) : launch_bwd_t<32, float>(a, stream);
    case 64: return bf ? launch_bwd_t<64, __nv_bfloat16>(a, stream) : launch_bwd_t<64, float>(a, stream);
    case 128: return bf ? launch_bwd_t<128, __nv_bfloat16>(a, stream) : launch_bwd_t<128, float>(a, stream);
  }
  return set_error(4, "kda_bwd: unsupported K");
}

}  // namespace kda
