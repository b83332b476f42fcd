// Shared device code of the chunked KDA kernels (forward, state-gradient
// pass, per-chunk gradients).
//
// Chunk algebra ("research_layers.py", delta_recurrence, with erase = write
// = k and the write strength beta folded into the residual; the per-step
// recurrence itself is the one of "K3/kda/ops/reference/recurrent.py",
// naive_kda_fwd).  Inside a chunk of C steps with entering state M (K x V)
// and in-chunk cumulative decay c_i = sum_{s<=i} g_s (a K-vector per row):
//
//   Ah[i][j] = sum_f k_if k_jf exp(c_if - c_jf)          j <  i
//   P [i][j] = sum_f q~_if k_jf exp(c_if - c_jf)         j <= i   (q~ = scale q)
//   T        = (I + diag(beta) Ah)^-1                    unit lower triangular
//   U        = T diag(beta) (V - (K o e^c) M)            U_i = beta_i r_i
//   O        = (Q~ o e^c) M + P U
//   M'       = diag(e^{c_last}) M + (K o e^{c_last - c})^T U
//
// The page's own factoring k / exp(c) overflows once the in-chunk decay
// passes ~88 in log space (the production gate reaches -5 per step).  Here
// every exp(c_i - c_j) in Ah and P is split at a reference row rho inside the
// 16-row sub-block structure: for a column block J and a row i in a later
// block, rho is the last row of J, so both exp(c_i - c_rho) and
// exp(c_rho - c_j) are <= 1; on a diagonal block rho is the block's middle
// row and both factors stay within exp(+-span) where span is the block's
// largest in-block decay.  A diagonal block whose span exceeds 80 (possible
// only for an unbounded gate) is formed pair by pair instead.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int NTHREADS = 256;   // every chunked kernel runs 256 threads
constexpr int BS = 16;          // sub-block rows for the decay reference points
constexpr float DIAG_SPAN_MAX = 80.f;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

template <bool PRECISE>
__device__ __forceinline__ float kexp(float x) {
  if constexpr (PRECISE) return expf(x); else return __expf(x);
}

// Register-tiled product on a 16 x 16 thread grid: thread (ty, tx) owns the
// outputs (ty + 16 a, tx + 16 b), a < TM, b < TN; acc += sum_kk fa(row, kk) * fb(kk, col).
template <int TM, int TN, typename FA, typename FB>
__device__ __forceinline__ void mm(float (&acc)[TM][TN], int kd, FA fa, FB fb) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 2
  for (int kk = 0; kk < kd; ++kk) {
    float a[TM], b[TN];
#pragma unroll
    for (int i = 0; i < TM; ++i) a[i] = fa(ty + 16 * i, kk);
#pragma unroll
    for (int j = 0; j < TN; ++j) b[j] = fb(kk, tx + 16 * j);
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

template <int TM, int TN>
__device__ __forceinline__ void zero(float (&acc)[TM][TN]) {
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

// Loads one chunk of q (times scale), k, g and beta for head (b, hv) into
// shared memory as fp32; rows past the sequence end are zero (a zero row has
// no decay, no write and no read, so it leaves the state untouched).
// Then replaces g by its in-chunk cumulative sum c.
template <int K, int C, typename TIn>
__device__ __forceinline__ void load_chunk_qkgb(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                const float* __restrict__ g,
                                                const float* __restrict__ beta, float scale, int b,
                                                int t0, int L, int T, int H, int HV, int h, int hv,
                                                float* sQ, float* sK, float* sC, float* sBeta) {
  constexpr int LDK = K + 1;
  for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K;
    float qv = 0.f, kv = 0.f, gv = 0.f;
    if (i < L) {
      const size_t rq = ((size_t)b * T + t0 + i) * H + h;
      const size_t rg = ((size_t)b * T + t0 + i) * HV + hv;
      qv = to_f(q[rq * K + f]) * scale;
      kv = to_f(k[rq * K + f]);
      gv = g[rg * K + f];
    }
    sQ[i * LDK + f] = qv;
    sK[i * LDK + f] = kv;
    sC[i * LDK + f] = gv;
  }
  for (int i = threadIdx.x; i < C; i += NTHREADS)
    sBeta[i] = (i < L) ? beta[((size_t)b * T + t0 + i) * HV + hv] : 0.f;
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

// Per column block J: the exp factors of the split products.
//   sE1[i][f]  = exp(c_if - c_ref(i),f)  for rows i >= 16 J, ref = middle of J
//                for rows inside J and the last row of J below it
//   sE2o[j][f] = exp(c_last(J),f - c_jf) for j in J (off-diagonal columns)
//   sE2d[j][f] = exp(c_mid(J),f  - c_jf) for j in J (diagonal block columns)
// Returns (block-uniformly) whether the diagonal block must be formed pair
// by pair because its decay span exceeds DIAG_SPAN_MAX.
template <int K, int C, bool PRECISE>
__device__ __forceinline__ bool block_factors(int J, const float* sC, float* sE1, float* sE2o,
                                              float* sE2d, int* sFlag) {
  constexpr int LDK = K + 1;
  const int r0 = J * BS, rho_off = r0 + BS - 1, rho_diag = r0 + BS / 2 - 1;
  if (threadIdx.x == 0) *sFlag = 0;
  __syncthreads();
  for (int f = threadIdx.x; f < K; f += NTHREADS) {
    if (sC[r0 * LDK + f] - sC[rho_off * LDK + f] > DIAG_SPAN_MAX) atomicOr(sFlag, 1);
  }
  for (int idx = threadIdx.x; idx < (C - r0) * K; idx += NTHREADS) {
    const int i = r0 + idx / K, f = idx % K;
    const int ref = (i < r0 + BS) ? rho_diag : rho_off;
    sE1[i * LDK + f] = kexp<PRECISE>(sC[i * LDK + f] - sC[ref * LDK + f]);
  }
  for (int idx = threadIdx.x; idx < BS * K; idx += NTHREADS) {
    const int jj = idx / K, f = idx % K, j = r0 + jj;
    sE2o[jj * LDK + f] = kexp<PRECISE>(sC[rho_off * LDK + f] - sC[j * LDK + f]);
    sE2d[jj * LDK + f] = kexp<PRECISE>(sC[rho_diag * LDK + f] - sC[j * LDK + f]);
  }
  __syncthreads();
  return *sFlag != 0;
}

// Builds Ah (strict lower) and P (lower incl. diagonal), C x C, row stride C+1.
template <int K, int C, bool PRECISE>
__device__ void build_interaction(const float* sK, const float* sQ, const float* sC, float* sE1,
                                  float* sE2o, float* sE2d, int* sFlag, float* sAh, float* sP) {
  constexpr int LDK = K + 1, LDC = C + 1, NB = C / BS;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  for (int J = 0; J < NB; ++J) {
    const bool pairwise = block_factors<K, C, PRECISE>(J, sC, sE1, sE2o, sE2d, sFlag);
    const int j = J * BS + tx;
#pragma unroll
    for (int a = 0; a < NB; ++a) {
      const int i = a * BS + ty;
      if (a < J) {  // above the diagonal: structurally zero
        sAh[i * LDC + j] = 0.f;
        sP[i * LDC + j] = 0.f;
        continue;
      }
      float accA = 0.f, accP = 0.f;
      if (a == J && pairwise) {
        for (int f = 0; f < K; ++f) {
          const float e = kexp<PRECISE>(sC[i * LDK + f] - sC[j * LDK + f]);
          const float kj = sK[j * LDK + f] * e;
          accA = fmaf(sK[i * LDK + f], kj, accA);
          accP = fmaf(sQ[i * LDK + f], kj, accP);
        }
      } else {
        const float* e2 = (a == J) ? sE2d : sE2o;
#pragma unroll 4
        for (int f = 0; f < K; ++f) {
          const float kj = sK[j * LDK + f] * e2[tx * LDK + f];
          const float e1 = sE1[i * LDK + f];
          accA = fmaf(sK[i * LDK + f] * e1, kj, accA);
          accP = fmaf(sQ[i * LDK + f] * e1, kj, accP);
        }
      }
      sAh[i * LDC + j] = (j < i) ? accA : 0.f;
      sP[i * LDC + j] = (j <= i) ? accP : 0.f;
    }
    __syncthreads();
  }
}

// T = (I + diag(beta) Ah)^-1 for the unit lower-triangular system, by
// forward substitution on the 16 x 16 diagonal blocks and block
// substitution T_IJ = -T_II sum_{J<=L<I} A_IL T_LJ for the rest.
// sW is scratch of BS x (C+1).
template <int C>
__device__ void invert_unit_lower(const float* sAh, const float* sBeta, float* sT, float* sW) {
  constexpr int LDC = C + 1, NB = C / BS;
  for (int idx = threadIdx.x; idx < C * C; idx += NTHREADS) {
    const int i = idx / C, j = idx % C;
    sT[i * LDC + j] = (i == j) ? 1.f : 0.f;
  }
  __syncthreads();
  // diagonal blocks: one half-warp per block, lane = column inside the block
  if (threadIdx.x < NB * BS) {
    const int blk = threadIdx.x / BS, c = threadIdx.x % BS, o = blk * BS;
    for (int r = 1; r < BS; ++r) {
      const int i = o + r;
      float acc = 0.f;
      if (c < r) {
        acc = sAh[i * LDC + o + c];
        for (int m = c + 1; m < r; ++m) acc = fmaf(sAh[i * LDC + o + m], sT[(o + m) * LDC + o + c], acc);
        acc = -sBeta[i] * acc;
      }
      __syncwarp();
      if (c < r) sT[i * LDC + o + c] = acc;
      __syncwarp();
    }
  }
  __syncthreads();
  for (int I = 1; I < NB; ++I) {
    const int o = I * BS, ncol = o;
    // W[r][c] = sum_{l=c}^{o-1} beta_{o+r} Ah[o+r][l] T[l][c]
    for (int idx = threadIdx.x; idx < BS * ncol; idx += NTHREADS) {
      const int r = idx / ncol, c = idx % ncol;
      float acc = 0.f;
      for (int l = c; l < o; ++l) acc = fmaf(sAh[(o + r) * LDC + l], sT[l * LDC + c], acc);
      sW[r * LDC + c] = sBeta[o + r] * acc;
    }
    __syncthreads();
    // T[o+r][c] = -sum_{m<=r} T[o+r][o+m] W[m][c]
    for (int idx = threadIdx.x; idx < BS * ncol; idx += NTHREADS) {
      const int r = idx / ncol, c = idx % ncol;
      float acc = 0.f;
      for (int m = 0; m <= r; ++m) acc = fmaf(sT[(o + r) * LDC + o + m], sW[m * LDC + c], acc);
      sT[(o + r) * LDC + c] = -acc;
    }
    __syncthreads();
  }
}

}  // namespace kda
