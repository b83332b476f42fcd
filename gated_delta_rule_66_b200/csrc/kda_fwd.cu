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
#include "kda_tc.cuh"

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

// ============================================================================
// Two-kernel CUDA-core forward (chunk-parallel preparation + sequential state
// pass), used when the caller gives a workspace of kda_fwd_scratch_bytes()
// (or kda_fwd_erase_workspace_bytes()).
//
// The state-independent part of every chunk (interactions, inverse, decayed
// operands) runs first for all chunks at once, one CTA per (b, state head,
// chunk), and leaves per chunk in the workspace (FmaRec):
//   Tb   = T diag(beta)                  C x C
//   Rt   = Tb (R o e^c)                  C x K  (R = k; the erase rows e)
//   KEd  = k o e^{c_last - c}            C x K
//   El   = e^{c_last}                    K
//   per query head: P (C x C) and Q~ o e^c (C x K)
// so that the state pass only applies, per chunk and V slice,
//   U = Tb V - Rt M,   O = (Q~ o e^c) M + P U,   M' = diag(El) M + KEd^T U
// (the same chunk algebra as the single-kernel path, with the residual's two
// terms multiplied through by Tb ahead of time).  For the erase/write variant
// one state pass carries a state head once and reads it out for all its
// query heads.
// ============================================================================
__host__ __device__ constexpr int fma_rec_floats(int K, int C, int QG) {
  return C * C + 2 * C * K + K + QG * (C * C + C * K);
}

template <int K, int C, bool ERASE>
struct PrepSmem {
  static constexpr int LDK = K + 1, LDC = C + 1;
  static constexpr int oK = 0, oQ = oK + C * LDK, oC = oQ + C * LDK, oE1 = oC + C * LDK,
                       oE2o = oE1 + C * LDK, oE2d = oE2o + BS * LDK, oAh = oE2d + BS * LDK,
                       oT = oAh + C * LDC, oP = oT + C * LDC, oW = oP + C * LDC, oBeta = oW + BS * LDC,
                       oFlag = oBeta + C, oR = oFlag + 4, total = oR + (ERASE ? C * LDK : 0);
  static constexpr size_t bytes = (size_t)total * sizeof(float);
};

// q~ = scale q of query head hq for one chunk (rows past the end zero)
template <int K, int C, typename TIn>
__device__ __forceinline__ void load_chunk_q(const FwdArgs& a, int b, int t0, int L, int hq, float* sQ) {
  constexpr int LDK = K + 1;
  const TIn* q = static_cast<const TIn*>(a.q);
  for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K;
    sQ[i * LDK + f] = (i < L) ? to_f(q[(((size_t)b * a.T + t0 + i) * a.H + hq) * K + f]) * a.scale : 0.f;
  }
  __syncthreads();
}

template <int K, int C, typename TIn, bool ERASE>
__global__ void __launch_bounds__(NTHREADS) kda_fwd_chunkprep_kernel(FwdArgs a, float* __restrict__ prep) {
  using S = PrepSmem<K, C, ERASE>;
  constexpr bool PRECISE = sizeof(TIn) == 4;
  constexpr int LDK = S::LDK, LDC = S::LDC;
  extern __shared__ float smem[];
  float *sK = smem + S::oK, *sQ = smem + S::oQ, *sC = smem + S::oC, *sE1 = smem + S::oE1,
        *sE2o = smem + S::oE2o, *sE2d = smem + S::oE2d, *sAh = smem + S::oAh, *sT = smem + S::oT,
        *sP = smem + S::oP, *sW = smem + S::oW, *sBeta = smem + S::oBeta, *sR = ERASE ? smem + S::oR : nullptr;
  int* sFlag = reinterpret_cast<int*>(smem + S::oFlag);
  const int ch = blockIdx.x, hv = blockIdx.y, b = blockIdx.z;
  const int T = a.T, NT = (T + C - 1) / C, t0 = ch * C, L = min(C, T - t0);
  const int QG = ERASE ? a.H / a.HV : 1;
  float* rec = prep + (((size_t)b * a.HV + hv) * NT + ch) * fma_rec_floats(K, C, QG);
  float *gTb = rec, *gRt = gTb + C * C, *gKEd = gRt + C * K, *gEl = gKEd + C * K, *gQ0 = gEl + K;

  if constexpr (ERASE)
    load_chunk_erase<K, C, TIn>(a, b, t0, L, hv * QG, hv, sQ, sK, sR, sC, sBeta);
  else
    load_chunk_qkgb<K, C, TIn>(static_cast<const TIn*>(a.q), static_cast<const TIn*>(a.k), a.g, a.beta, a.scale,
                               b, t0, L, T, a.H, a.HV, hv / (a.HV / a.H), hv, sQ, sK, sC, sBeta);
  for (int qi = 0; qi < QG; ++qi) {
    if (qi > 0) load_chunk_q<K, C, TIn>(a, b, t0, L, hv * QG + qi, sQ);
    // Ah (erase or key rows against keys) and P (queries against keys); the
    // inverse below needs the first Ah only (later query heads overwrite it)
    build_interaction<K, C, PRECISE>(sK, sQ, sC, sE1, sE2o, sE2d, sFlag, sAh, sP, sR);
    float* gP = gQ0 + (size_t)qi * (C * C + C * K);
    float* gQE = gP + C * C;
    for (int idx = threadIdx.x; idx < C * C; idx += NTHREADS) gP[idx] = sP[(idx / C) * LDC + idx % C];
    for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
      const int i = idx / K, f = idx % K;
      gQE[idx] = sQ[i * LDK + f] * kexp<PRECISE>(sC[i * LDK + f]);
    }
    if (qi == 0) invert_unit_lower<C>(sAh, sBeta, sT, sW);
    __syncthreads();
  }
  // decayed operands: KEd (global), R o e^c (in place), e^{c_last}; Tb = T diag(beta)
  float* sRe = ERASE ? sR : sK;
  for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K;
    const float c = sC[i * LDK + f], cl = sC[(C - 1) * LDK + f];
    gKEd[idx] = sK[i * LDK + f] * kexp<PRECISE>(cl - c);
    if constexpr (ERASE) sRe[i * LDK + f] *= kexp<PRECISE>(c);
  }
  __syncthreads();
  if constexpr (!ERASE) {  // (k's rows are read above before they are scaled)
    for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
      const int i = idx / K, f = idx % K;
      sRe[i * LDK + f] *= kexp<PRECISE>(sC[i * LDK + f]);
    }
  }
  for (int f = threadIdx.x; f < K; f += NTHREADS) gEl[f] = kexp<PRECISE>(sC[(C - 1) * LDK + f]);
  for (int idx = threadIdx.x; idx < C * C; idx += NTHREADS) {
    const int i = idx / C, j = idx % C;
    const float v = sT[i * LDC + j] * sBeta[j];
    sT[i * LDC + j] = v;
    gTb[idx] = v;
  }
  __syncthreads();
  {  // Rt = Tb (R o e^c)
    constexpr int TMC = C / 16, TNK = K / 16;
    float acc[TMC][TNK];
    zero(acc);
    mm(acc, C, [&](int i, int j) { return sT[i * LDC + j]; }, [&](int j, int f) { return sRe[j * LDK + f]; });
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int x = 0; x < TMC; ++x)
#pragma unroll
      for (int y = 0; y < TNK; ++y) gRt[(ty + 16 * x) * K + tx + 16 * y] = acc[x][y];
  }
}

// The state pass: one CTA per (b, state head, V slice of VB columns) carries
// the K x VB state through the chunks; each chunk's operands (FmaRec) and V
// rows come in by 16-byte cp.async, one chunk ahead when two buffers fit.
template <int K, int C, int VB, typename TIn>
struct StateSmem {
  static constexpr int LDV = VB + 1;
  static constexpr int oM = 0, oU = oM + K * LDV, oBuf = oU + C * LDV;
  // a buffer: the chunk's record, then its V rows (TIn, C x VB)
  __host__ __device__ static constexpr int vfloats(int) { return (C * VB * (int)sizeof(TIn) + 15) / 16 * 4; }
  // (with the read-out split the pass reads only the first part of a record:
  // T diag(beta), Rt, KEd, e^{c_last})
  __host__ __device__ static int rec_load(int QG, bool split) {
    return split ? C * C + 2 * C * K + K : fma_rec_floats(K, C, QG);
  }
  __host__ __device__ static int buf_floats(int QG, bool split) { return rec_load(QG, split) + vfloats(0); }
  static size_t bytes(int QG, bool split, int nbuf) {
    return (size_t)(oBuf + nbuf * buf_floats(QG, split)) * sizeof(float);
  }
};

// (With mst and ust (always for ERASE) the read-out is left to
// kda_fwd_readout_kernel: the pass stores the state entering every chunk into
// mst [B, HV, NT, K, V] and U into ust [B, HV, NT, C, V] instead.)
template <int K, int C, int VB, typename TIn, bool ERASE>
__global__ void __launch_bounds__(NTHREADS, 1)
    kda_fwd_statepass_kernel(FwdArgs a, const float* __restrict__ prep, int nbuf, float* __restrict__ mst,
                             float* __restrict__ ust) {
  const bool split = ust != nullptr;
  using S = StateSmem<K, C, VB, TIn>;
  constexpr int LDV = S::LDV, TMC = C / 16, TNV = VB / 16, TMK = K / 16;
  extern __shared__ __align__(16) float smem[];
  float *sM = smem + S::oM, *sU = smem + S::oU;
  const int QG = ERASE ? a.H / a.HV : 1, REC = fma_rec_floats(K, C, QG), LREC = S::rec_load(QG, split),
            BUF = S::buf_floats(QG, split);
  const int v0 = blockIdx.x * VB, hv = blockIdx.y, b = blockIdx.z;
  const int T = a.T, V = a.V, NT = (T + C - 1) / C;
  const size_t head = (size_t)b * a.HV + hv;
  const int HO = ERASE ? a.H : a.HV;
  const TIn* __restrict__ v = static_cast<const TIn*>(a.v);
  TIn* __restrict__ o = static_cast<TIn*>(a.o);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* recs = prep + head * NT * (size_t)REC;

  const auto issue = [&](int ch, float* buf) {  // the chunk's record and V rows into buf
    const float* src = recs + (size_t)ch * REC;
    const uint32_t sb = (uint32_t)__cvta_generic_to_shared(buf);
    for (int x = threadIdx.x; x < LREC / 4; x += NTHREADS) tc::cp_async16(sb + x * 16, src + x * 4, true);
    constexpr int PR = VB * (int)sizeof(TIn) / 16;  // 16-byte pieces per V row
    const int t0 = ch * C, L = min(C, T - t0);
    const uint32_t vb = sb + LREC * 4;
    for (int x = threadIdx.x; x < C * PR; x += NTHREADS) {
      const int i = x / PR, pc = x % PR;
      const bool ok = i < L;
      const TIn* row = v + (((size_t)b * T + t0 + (ok ? i : 0)) * a.HV + hv) * V + v0;
      tc::cp_async16(vb + x * 16, reinterpret_cast<const unsigned char*>(row) + pc * 16, ok);
    }
    tc::cp_async_commit();
  };

  for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
    const int f = idx / VB, n = idx % VB;
    sM[f * LDV + n] = a.S0 ? a.S0[(head * K + f) * V + v0 + n] : 0.f;
  }
  float* buf0 = smem + S::oBuf;
  issue(0, buf0);
  for (int ch = 0; ch < NT; ++ch) {
    const int t0 = ch * C, L = min(C, T - t0);
    float* cur = buf0 + (nbuf == 2 ? (ch & 1) * BUF : 0);
    if (nbuf == 2 && ch + 1 < NT) {  // (the other buffer's last readers passed the previous chunk's end barrier)
      issue(ch + 1, buf0 + ((ch + 1) & 1) * BUF);
      tc::cp_async_wait_group<1>();
    } else {
      tc::cp_async_wait_group<0>();
    }
    __syncthreads();
    const float *cTb = cur, *cRt = cTb + C * C, *cKEd = cRt + C * K, *cEl = cKEd + C * K, *cQ0 = cEl + K;
    const TIn* cV = reinterpret_cast<const TIn*>(cur + LREC);
    float* const mdst = split ? mst : a.states;  // (mst is the state store when the call keeps states)
    if (mdst) {
      float* dst = mdst + ((head * NT + ch) * K) * V;
      for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
        const int f = idx / VB, n = idx % VB;
        dst[(size_t)f * V + v0 + n] = sM[f * LDV + n];
      }
    }
    {  // U = Tb V - Rt M
      float acc[TMC][TNV], neg[TMC][TNV];
      zero(acc);
      zero(neg);
      mmk<C>(acc, [&](int i, int j) { return cTb[i * C + j]; }, [&](int j, int n) { return to_f(cV[j * VB + n]); });
      mmk<K>(neg, [&](int i, int f) { return cRt[i * K + f]; }, [&](int f, int n) { return sM[f * LDV + n]; });
#pragma unroll
      for (int x = 0; x < TMC; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const float u = acc[x][y] - neg[x][y];
          sU[(ty + 16 * x) * LDV + tx + 16 * y] = u;
          if (split) ust[((head * NT + ch) * C + ty + 16 * x) * V + v0 + tx + 16 * y] = u;
        }
    }
    __syncthreads();
    if (!split && a.o) {
      for (int qi = 0; qi < QG; ++qi) {  // O = (Q~ o e^c) M + P U for each query head of this state head
        const float* cP = cQ0 + (size_t)qi * (C * C + C * K);
        const float* cQE = cP + C * C;
        float acc[TMC][TNV];
        zero(acc);
        mmk<K>(acc, [&](int i, int f) { return cQE[i * K + f]; }, [&](int f, int n) { return sM[f * LDV + n]; });
        mmk<C>(acc, [&](int i, int j) { return cP[i * C + j]; }, [&](int j, int n) { return sU[j * LDV + n]; });
        const int ho = ERASE ? hv * QG + qi : hv;
#pragma unroll
        for (int x = 0; x < TMC; ++x)
#pragma unroll
          for (int y = 0; y < TNV; ++y) {
            const int i = ty + 16 * x, n = tx + 16 * y;
            if (i < L) o[(((size_t)b * T + t0 + i) * HO + ho) * V + v0 + n] = from_f<TIn>(acc[x][y]);
          }
      }
    }
    {  // M' = diag(El) M + KEd^T U
      float acc[TMK][TNV];
#pragma unroll
      for (int x = 0; x < TMK; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) {
          const int f = ty + 16 * x, n = tx + 16 * y;
          acc[x][y] = cEl[f] * sM[f * LDV + n];
        }
      mmk<C>(acc, [&](int f, int i) { return cKEd[i * K + f]; }, [&](int i, int n) { return sU[i * LDV + n]; });
      __syncthreads();
#pragma unroll
      for (int x = 0; x < TMK; ++x)
#pragma unroll
        for (int y = 0; y < TNV; ++y) sM[(ty + 16 * x) * LDV + tx + 16 * y] = acc[x][y];
    }
    if (nbuf == 1 && ch + 1 < NT) {
      __syncthreads();  // every read of this chunk's buffer is done
      issue(ch + 1, buf0);
    }
    __syncthreads();
  }
  if (a.S_T) {
    for (int idx = threadIdx.x; idx < K * VB; idx += NTHREADS) {
      const int f = idx / VB, n = idx % VB;
      a.S_T[(head * K + f) * V + v0 + n] = sM[f * LDV + n];
    }
  }
}

// Read-out, one CTA per (b, query head, chunk): O = (Q~ o e^c) M + P U over
// all V columns, from the chunk record and the state and U the state pass
// stored (KDA: the query head is the value head).
template <int K, int C, int V, typename TIn, bool ERASE>
__global__ void __launch_bounds__(NTHREADS) kda_fwd_readout_kernel(FwdArgs a, const float* __restrict__ prep,
                                                                    const float* __restrict__ mst,
                                                                    const float* __restrict__ ust) {
  constexpr int TMC = C / 16, TNV = V / 16, LDV = V + 4;
  extern __shared__ __align__(16) float smem[];
  float *sQE = smem, *sP = sQE + C * K, *sM = sP + C * C, *sU = sM + K * LDV;
  const int ch = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int QG = ERASE ? a.H / a.HV : 1, hv = hq / QG, qi = hq % QG, HO = ERASE ? a.H : a.HV;
  const int T = a.T, NT = (T + C - 1) / C, t0 = ch * C, L = min(C, T - t0);
  const size_t hc = ((size_t)b * a.HV + hv) * NT + ch;
  const float* rec = prep + hc * fma_rec_floats(K, C, QG);
  const float* gP = rec + C * C + 2 * C * K + K + (size_t)qi * (C * C + C * K);
  const float* gQE = gP + C * C;
  const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(smem);
  for (int x = threadIdx.x; x < C * K / 4; x += NTHREADS) tc::cp_async16(s0 + x * 16, gQE + x * 4, true);
  for (int x = threadIdx.x; x < C * C / 4; x += NTHREADS) tc::cp_async16(s0 + (C * K + x * 4) * 4, gP + x * 4, true);
  const float* gM = mst + hc * K * V;
  const float* gU = ust + hc * C * V;
  for (int x = threadIdx.x; x < K * V / 4; x += NTHREADS) {
    const int f = x / (V / 4), n4 = (x % (V / 4)) * 4;
    tc::cp_async16(s0 + (uint32_t)(sM - smem + f * LDV + n4) * 4, gM + f * V + n4, true);
  }
  for (int x = threadIdx.x; x < C * V / 4; x += NTHREADS) {
    const int i = x / (V / 4), n4 = (x % (V / 4)) * 4;
    tc::cp_async16(s0 + (uint32_t)(sU - smem + i * LDV + n4) * 4, gU + i * V + n4, true);
  }
  tc::cp_async_wait_all();
  __syncthreads();
  float acc[TMC][TNV];
  zero(acc);
  mmk<K>(acc, [&](int i, int f) { return sQE[i * K + f]; }, [&](int f, int n) { return sM[f * LDV + n]; });
  mmk<C>(acc, [&](int i, int j) { return sP[i * C + j]; }, [&](int j, int n) { return sU[j * LDV + n]; });
  TIn* o = static_cast<TIn*>(a.o);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int x = 0; x < TMC; ++x)
#pragma unroll
    for (int y = 0; y < TNV; ++y) {
      const int i = ty + 16 * x, n = tx + 16 * y;
      if (i < L) o[(((size_t)b * T + t0 + i) * HO + hq) * V + n] = from_f<TIn>(acc[x][y]);
    }
}

size_t fma_prep_bytes(int B, int T, int HV, int K, int QG) {
  const size_t NT = (size_t)(T + FWD_CHUNK - 1) / FWD_CHUNK;
  return (size_t)B * HV * NT * fma_rec_floats(K, FWD_CHUNK, QG) * sizeof(float);
}

// The workspace of the read-out split: the chunk records, then the state
// entering every chunk and U of every chunk for the read-out kernel.
size_t fma_split_bytes(int B, int T, int HQ, int HV, int K, int V) {
  const size_t NT = (size_t)(T + FWD_CHUNK - 1) / FWD_CHUNK;
  return fma_prep_bytes(B, T, HV, K, HQ / HV) + (size_t)B * HV * NT * ((size_t)K * V + (size_t)FWD_CHUNK * V) * 4;
}
// KDA shapes other than K = V = 128 run the read-out split (their scratch is
// sized for it); K = V = 128 keeps the read-out in the state pass, so that
// its scratch stays within the tensor-core path's chunk images.
bool fma_kda_split(int K, int V) { return !(K == 128 && V == 128); }

// Whether the two-kernel CUDA-core forward takes this call: plain inputs (no
// fused preparation or output gate), 16-byte aligned v (its rows come in by
// 16-byte copies) and workspace.
bool fwd_fma2_eligible(const FwdArgs& a, const void* workspace) {
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  return !a.ctab && !a.prep.z && !a.og && workspace && al16(workspace) && al16(a.v) && a.V % 16 == 0;
}

// state slices of 16 value columns (twice the CTAs of 32-column slices: the
// pass is latency-bound, measured 0.134 vs 0.147 ms on the fp32 twin workload)
constexpr int FMA2_VB = 16;

template <int K, typename TIn, bool ERASE>
static int launch_fwd_fma2_t(const FwdArgs& a, float* prep, cudaStream_t stream) {
  constexpr int C = FWD_CHUNK, VB = FMA2_VB;
  const char* who = ERASE ? "kda_fwd_erase" : "kda_fwd";
  const int NT = (a.T + C - 1) / C, QG = ERASE ? a.H / a.HV : 1;
  auto k1 = kda_fwd_chunkprep_kernel<K, C, TIn, ERASE>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PrepSmem<K, C, ERASE>::bytes);
  if (e != cudaSuccess) return set_cuda_error(who, e);
  k1<<<dim3(NT, a.HV, a.B), NTHREADS, PrepSmem<K, C, ERASE>::bytes, stream>>>(a, prep);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error(who, e);
  using SS = StateSmem<K, C, VB, TIn>;
  const bool split = ERASE || fma_kda_split(K, a.V);
  const int nbuf = SS::bytes(QG, split, 2) <= 200 * 1024 ? 2 : 1;
  if (SS::bytes(QG, split, nbuf) > 227 * 1024)
    return set_error(4, "two-kernel CUDA-core forward: too many query heads per state head");
  auto k2 = kda_fwd_statepass_kernel<K, C, VB, TIn, ERASE>;
  e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SS::bytes(QG, split, nbuf));
  if (e != cudaSuccess) return set_cuda_error(who, e);
  float* mst = nullptr;
  float* ust = nullptr;
  if (split) {  // (a kept state store doubles as the read-out's state)
    float* region = prep + fma_prep_bytes(a.B, a.T, a.HV, K, QG) / sizeof(float);
    mst = (!ERASE && a.states) ? a.states : region;
    ust = region + (size_t)a.B * a.HV * NT * K * a.V;
  }
  k2<<<dim3(a.V / VB, a.HV, a.B), NTHREADS, SS::bytes(QG, split, nbuf), stream>>>(a, prep, nbuf, mst, ust);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error(who, e);
  if (split) {
    if (!a.o) return 0;
    const size_t sb = (size_t)(C * K + C * C + (K + C) * (a.V + 4)) * sizeof(float);
    const auto k3 = a.V == 32 ? kda_fwd_readout_kernel<K, C, 32, TIn, ERASE>
                  : a.V == 64 ? kda_fwd_readout_kernel<K, C, 64, TIn, ERASE>
                              : kda_fwd_readout_kernel<K, C, 128, TIn, ERASE>;
    e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
    if (e != cudaSuccess) return set_cuda_error(who, e);
    k3<<<dim3(NT, ERASE ? a.H : a.HV, a.B), NTHREADS, sb, stream>>>(a, prep, mst, ust);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(who, e);
  }
  return 0;
}

int launch_fwd_fma2(const FwdArgs& a, int dtype, bool erase, float* prep, cudaStream_t stream) {
  const bool bf = dtype == 1;
#define KDA_FMA2(KK)                                                                                     \
  case KK:                                                                                               \
    if (erase)                                                                                           \
      return bf ? launch_fwd_fma2_t<KK, __nv_bfloat16, true>(a, prep, stream)                           \
                : launch_fwd_fma2_t<KK, float, true>(a, prep, stream);                                   \
    return bf ? launch_fwd_fma2_t<KK, __nv_bfloat16, false>(a, prep, stream)                            \
              : launch_fwd_fma2_t<KK, float, false>(a, prep, stream);
  switch (a.K) {
    KDA_FMA2(32)
    KDA_FMA2(64)
    KDA_FMA2(128)
  }
#undef KDA_FMA2
  return set_error(4, "kda_fwd: unsupported K");
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

// The same for V = 128 with four consecutive values per lane: one 16-byte
// load of o32 and one 8-byte (bf16) or 16-byte (fp32) load of og and store
// of o per lane and row.
template <typename TIn>
__global__ void __launch_bounds__(256) kda_out_gate4_kernel(const float* __restrict__ o32,
                                                            const TIn* __restrict__ og, float eps, size_t rows,
                                                            TIn* __restrict__ o) {
  const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const size_t e0 = row * 128 + 4 * lane;
  const float4 x = *reinterpret_cast<const float4*>(o32 + e0);
  float gv[4];
  if constexpr (sizeof(TIn) == 2) {
    const uint2 r = *reinterpret_cast<const uint2*>(og + e0);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&r.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&r.y);
    gv[0] = __low2float(lo); gv[1] = __high2float(lo); gv[2] = __low2float(hi); gv[3] = __high2float(hi);
  } else {
    const float4 r = *reinterpret_cast<const float4*>(og + e0);
    gv[0] = r.x; gv[1] = r.y; gv[2] = r.z; gv[3] = r.w;
  }
  float s = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, x.w * x.w)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float inv = rsqrtf(s / 128.f + eps);
  const float y[4] = {x.x * inv * prep_sigmoid(gv[0]), x.y * inv * prep_sigmoid(gv[1]),
                      x.z * inv * prep_sigmoid(gv[2]), x.w * inv * prep_sigmoid(gv[3])};
  if constexpr (sizeof(TIn) == 2) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(y[0], y[1]), hi = __floats2bfloat162_rn(y[2], y[3]);
    uint2 r;
    r.x = *reinterpret_cast<const uint32_t*>(&lo);
    r.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(o + e0) = r;
  } else {
    *reinterpret_cast<float4*>(o + e0) = make_float4(y[0], y[1], y[2], y[3]);
  }
}

int launch_out_gate(const float* o32, const void* og, float eps, size_t rows, int V, int dtype, void* o,
                    cudaStream_t stream) {
  if (rows == 0) return 0;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  const size_t al = (size_t)o32 | (size_t)og | (size_t)o;
  if (V == 128 && (al & 15) == 0) {
    if (dtype == 1)
      kda_out_gate4_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
          o32, static_cast<const __nv_bfloat16*>(og), eps, rows, static_cast<__nv_bfloat16*>(o));
    else
      kda_out_gate4_kernel<float><<<blocks, 256, 0, stream>>>(o32, static_cast<const float*>(og), eps, rows,
                                                              static_cast<float*>(o));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("kda_fwd: output-gate launch", e);
    return 0;
  }
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

}  // namespace kda
