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

// ---- preparation math ("kimi_k3_host/kda.rs")
constexpr float KDA_L2_EPS_F = 1e-6f;  // l2norm_rows: eps added to the sum of squares
__device__ __forceinline__ float prep_sigmoid(float x) { return 1.f / (1.f + expf(-x)); }
// bounded_gate: lb sigmoid(dec x) (lb < 0) or -dec softplus(x) (lb = 0), x = z + dt_bias, dec = e^{A_log}
__device__ __forceinline__ float prep_gate(float x, float dec, float lb) {
  if (lb != 0.f) return lb * prep_sigmoid(dec * x);
  return -dec * (fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));
}

// The same with the fast exp / reciprocal / log (absolute error of g ~1e-7;
// the bf16 tensor-core paths, whose bar is 2e-3)
__device__ __forceinline__ float rcp_approx(float x) {  // hardware reciprocal; rcp(+inf) = +0
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float prep_sigmoid_fast(float x) { return rcp_approx(1.f + __expf(-x)); }
__device__ __forceinline__ float prep_gate_fast(float x, float dec, float lb) {
  if (lb != 0.f) return lb * prep_sigmoid_fast(dec * x);
  return -dec * (fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))));
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

// The same with a compile-time depth, fully unrolled (the loads of later
// steps are issued ahead: for short, latency-bound products).
template <int KD, int TM, int TN, typename FA, typename FB>
__device__ __forceinline__ void mmk(float (&acc)[TM][TN], FA fa, FB fb) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int kk = 0; kk < KD; ++kk) {
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
// With z (fused preparation, "kimi_k3_host/kda.rs"): q and k rows are
// L2-normalised (l2norm_rows), g = prep_gate(z + dt_bias) (bounded_gate) and
// beta = sigmoid(beta) (kda_recurrent_step takes the logit).
template <int K, int C, typename TIn>
__device__ __forceinline__ void load_chunk_qkgb(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                const float* __restrict__ g,
                                                const float* __restrict__ beta, float scale, int b,
                                                int t0, int L, int T, int H, int HV, int h, int hv,
                                                float* sQ, float* sK, float* sC, float* sBeta,
                                                const TIn* __restrict__ z = nullptr,
                                                const float* __restrict__ A_log = nullptr,
                                                const float* __restrict__ dt_bias = nullptr, float lb = 0.f) {
  constexpr int LDK = K + 1;
  const bool prep = z != nullptr;
  const float dec = prep ? expf(A_log[hv]) : 0.f;
  for (int idx = threadIdx.x; idx < C * K; idx += NTHREADS) {
    const int i = idx / K, f = idx % K;
    float qv = 0.f, kv = 0.f, gv = 0.f;
    if (i < L) {
      const size_t rq = ((size_t)b * T + t0 + i) * H + h;
      const size_t rg = ((size_t)b * T + t0 + i) * HV + hv;
      qv = to_f(q[rq * K + f]) * (prep ? 1.f : scale);
      kv = to_f(k[rq * K + f]);
      gv = prep ? prep_gate(to_f(z[rg * K + f]) + dt_bias[(size_t)hv * K + f], dec, lb) : g[rg * K + f];
    }
    sQ[i * LDK + f] = qv;
    sK[i * LDK + f] = kv;
    sC[i * LDK + f] = gv;
  }
  for (int i = threadIdx.x; i < C; i += NTHREADS) {
    float bv = 0.f;
    if (i < L) {
      bv = beta[((size_t)b * T + t0 + i) * HV + hv];
      if (prep) bv = prep_sigmoid(bv);
    }
    sBeta[i] = bv;
  }
  __syncthreads();
  if (prep) {  // row norms: one warp per row at a time, then q~ = scale q_hat
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < 2 * C; r += NTHREADS / 32) {
      float* row = (r < C ? sQ : sK) + (r % C) * LDK;
      float s = 0.f;
      for (int f = lane; f < K; f += 32) s = fmaf(row[f], row[f], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      const float mul = rsqrtf(s + KDA_L2_EPS_F) * (r < C ? scale : 1.f);
      for (int f = lane; f < K; f += 32) row[f] *= mul;
    }
  }
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
template <int K, int C, bool PRECISE, int LDK_ = K + 1>
__device__ __forceinline__ bool block_factors(int J, const float* sC, float* sE1, float* sE2o,
                                              float* sE2d, int* sFlag) {
  constexpr int LDK = LDK_;
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
// With sR (the erase rows of the asymmetric variant, "research_layers.py",
// delta_recurrence: read = erase * decay) Ah[i][j] = sum_f r_if k_jf e^{c_i - c_j}
// instead of k_if.
template <int K, int C, bool PRECISE>
__device__ void build_interaction(const float* sK, const float* sQ, const float* sC, float* sE1,
                                  float* sE2o, float* sE2d, int* sFlag, float* sAh, float* sP,
                                  const float* sR = nullptr) {
  constexpr int LDK = K + 1, LDC = C + 1, NB = C / BS;
  if (!sR) sR = sK;
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
          accA = fmaf(sR[i * LDK + f], kj, accA);
          accP = fmaf(sQ[i * LDK + f], kj, accP);
        }
      } else {
        const float* e2 = (a == J) ? sE2d : sE2o;
#pragma unroll 4
        for (int f = 0; f < K; ++f) {
          const float kj = sK[j * LDK + f] * e2[tx * LDK + f];
          const float e1 = sE1[i * LDK + f];
          accA = fmaf(sR[i * LDK + f] * e1, kj, accA);
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


// Adds to dq~, dk and the decay adjoint dc the terms that flow through the
// interaction matrices (dA_hat = beta_i dA, strict lower; dP, lower incl.
// diagonal; both C x C with row stride C+1):
//   row terms    rowA_i = sum_j dA_hat_ij (k_j o e^{c_i - c_j}),  rowP_i likewise with dP
//   column terms colA_j = sum_i dA_hat_ij (k_i o e^{c_i - c_j}),  colP_j with q~_i
//   dk += rowA + colA + colP,  dq~ += rowP,
//   dc += k o rowA + q~ o rowP - k o (colA + colP)
// with every exp(c_i - c_j) split at the 16-row sub-block references of
// block_factors (pair by pair for a diagonal block whose span is too wide).
// sK, sQ, sC, sDq, sDk, sDc are C x K with row stride K+1; sE1 / sE2o / sE2d
// are the scratch of block_factors.  One column block J at a time:
// factored_block_scalar with fp32 FMA (any block), factored_block_mma with
// 3xTF32 warp MMAs (blocks whose exponents split, K a multiple of 8).
template <int K, int C, bool PRECISE, int LDK_ = K + 1, int LDC_ = C + 1>
__device__ void factored_block_scalar(int J, bool pairwise, const float* sK, const float* sQ, const float* sC,
                                      const float* sdA, const float* sdP, const float* sE1, const float* sE2o,
                                      const float* sE2d, float* sDq, float* sDk, float* sDc) {
  constexpr int LDK = LDK_, LDC = LDC_;
    const int r0 = J * BS;
    // row terms: rows i >= r0 against the columns of block J
    for (int idx = threadIdx.x; idx < (C - r0) * K; idx += NTHREADS) {
      const int i = r0 + idx / K, f = idx % K;
      const bool diag = i < r0 + BS;
      const int jmax = diag ? i : r0 + BS - 1;   // j <= i
      float rA = 0.f, rP = 0.f;
      if (diag && pairwise) {
        for (int j = r0; j <= jmax; ++j) {
          const float w = sK[j * LDK + f] * kexp<PRECISE>(sC[i * LDK + f] - sC[j * LDK + f]);
          rA = fmaf(sdA[i * LDC + j], w, rA);
          rP = fmaf(sdP[i * LDC + j], w, rP);
        }
      } else {
        const float* e2 = diag ? sE2d : sE2o;
        for (int j = r0; j <= jmax; ++j) {
          const float w = sK[j * LDK + f] * e2[(j - r0) * LDK + f];
          rA = fmaf(sdA[i * LDC + j], w, rA);
          rP = fmaf(sdP[i * LDC + j], w, rP);
        }
        const float e1 = sE1[i * LDK + f];
        rA *= e1;
        rP *= e1;
      }
      const int o = i * LDK + f;
      sDk[o] += rA;
      sDq[o] += rP;
      sDc[o] += sK[o] * rA + sQ[o] * rP;
    }
    __syncthreads();
    // column terms: columns j of block J against rows i >= j
    for (int idx = threadIdx.x; idx < BS * K; idx += NTHREADS) {
      const int jj = idx / K, f = idx % K, j = r0 + jj;
      float cAd = 0.f, cPd = 0.f, cAo = 0.f, cPo = 0.f;
      for (int i = j; i < r0 + BS; ++i) {
        const int o = i * LDK + f;
        const float x = (pairwise) ? kexp<PRECISE>(sC[o] - sC[j * LDK + f]) : sE1[o];
        cAd = fmaf(sdA[i * LDC + j], sK[o] * x, cAd);
        cPd = fmaf(sdP[i * LDC + j], sQ[o] * x, cPd);
      }
      for (int i = r0 + BS; i < C; ++i) {
        const int o = i * LDK + f;
        const float x = sE1[o];
        cAo = fmaf(sdA[i * LDC + j], sK[o] * x, cAo);
        cPo = fmaf(sdP[i * LDC + j], sQ[o] * x, cPo);
      }
      const float e2d = pairwise ? 1.f : sE2d[jj * LDK + f], e2o = sE2o[jj * LDK + f];
      const float col = (cAd + cPd) * e2d + (cAo + cPo) * e2o;
      const int o = j * LDK + f;
      sDk[o] += col;
      sDc[o] -= sK[o] * col;
    }
    __syncthreads();
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// d += a (16 x 8, row-major) * b (8 x 8), tf32 inputs, fp32 accumulate.
// Fragments (g = lane / 4, t = lane % 4): a0 (g, t), a1 (g+8, t), a2 (g, t+4),
// a3 (g+8, t+4); b0 (k = t, n = g), b1 (k = t+4, n = g); d0 (g, 2t),
// d1 (g, 2t+1), d2 (g+8, 2t), d3 (g+8, 2t+1).
__device__ __forceinline__ void mma_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// x = hi + lo with both halves exactly representable in tf32; three tf32
// products hi*hi + hi*lo + lo*hi carry ~fp32 accuracy (the lo*lo term is
// below fp32 rounding).
struct Split {
  uint32_t hi, lo;
};
__device__ __forceinline__ Split split_tf32(float x) {
  const uint32_t h = to_tf32(x);
  return {h, to_tf32(x - __uint_as_float(h))};
}
__device__ __forceinline__ void mma3(float (&d)[4], const Split (&a)[4], const Split (&b)[2]) {
  const uint32_t ah[4] = {a[0].hi, a[1].hi, a[2].hi, a[3].hi}, al[4] = {a[0].lo, a[1].lo, a[2].lo, a[3].lo};
  const uint32_t bh[2] = {b[0].hi, b[1].hi}, bl[2] = {b[0].lo, b[1].lo};
  mma_16x8x8(d, al, bh);
  mma_16x8x8(d, ah, bl);
  mma_16x8x8(d, ah, bh);
}

template <int K, int C, int LDK_ = K + 1, int LDC_ = C + 1>
__device__ void factored_block_mma(int J, const float* sK, const float* sQ, const float* sdA, const float* sdP,
                                   const float* sE1, const float* sE2o, const float* sE2d, float* sDq, float* sDk,
                                   float* sDc) {
  constexpr int LDK = LDK_, LDC = LDC_, NB = C / BS, NTL = K / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int r0 = J * BS;
  // row terms: row block I >= J, 8 key channels per tile
  for (int x = warp; x < (NB - J) * NTL; x += NTHREADS / 32) {
    const int I = J + x / NTL, f0 = (x % NTL) * 8, i0 = I * BS;
    const float* e2 = (I == J) ? sE2d : sE2o;
    float accA[4] = {0.f, 0.f, 0.f, 0.f}, accP[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int j = r0 + ks * 8 + t;
      Split aA[4], aP[4], bw[2];
      aA[0] = split_tf32(sdA[(i0 + g) * LDC + j]);
      aA[1] = split_tf32(sdA[(i0 + g + 8) * LDC + j]);
      aA[2] = split_tf32(sdA[(i0 + g) * LDC + j + 4]);
      aA[3] = split_tf32(sdA[(i0 + g + 8) * LDC + j + 4]);
      aP[0] = split_tf32(sdP[(i0 + g) * LDC + j]);
      aP[1] = split_tf32(sdP[(i0 + g + 8) * LDC + j]);
      aP[2] = split_tf32(sdP[(i0 + g) * LDC + j + 4]);
      aP[3] = split_tf32(sdP[(i0 + g + 8) * LDC + j + 4]);
      bw[0] = split_tf32(sK[j * LDK + f0 + g] * e2[(j - r0) * LDK + f0 + g]);
      bw[1] = split_tf32(sK[(j + 4) * LDK + f0 + g] * e2[(j + 4 - r0) * LDK + f0 + g]);
      mma3(accA, aA, bw);
      mma3(accP, aP, bw);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + g + ((e & 2) ? 8 : 0), f = f0 + 2 * t + (e & 1), o = i * LDK + f;
      const float e1 = sE1[o], rA = accA[e] * e1, rP = accP[e] * e1;
      sDk[o] += rA;
      sDq[o] += rP;
      sDc[o] += sK[o] * rA + sQ[o] * rP;
    }
  }
  __syncthreads();
  // column terms: columns of block J against rows i of J (diagonal) and below
  for (int x = warp; x < NTL; x += NTHREADS / 32) {
    const int f0 = x * 8;
    float accD[4] = {0.f, 0.f, 0.f, 0.f}, accO[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ks = 0; ks < (C - r0) / 8; ++ks) {
      const int i = r0 + ks * 8 + t;
      Split aA[4], aP[4], bk[2], bq[2];
      aA[0] = split_tf32(sdA[i * LDC + r0 + g]);
      aA[1] = split_tf32(sdA[i * LDC + r0 + g + 8]);
      aA[2] = split_tf32(sdA[(i + 4) * LDC + r0 + g]);
      aA[3] = split_tf32(sdA[(i + 4) * LDC + r0 + g + 8]);
      aP[0] = split_tf32(sdP[i * LDC + r0 + g]);
      aP[1] = split_tf32(sdP[i * LDC + r0 + g + 8]);
      aP[2] = split_tf32(sdP[(i + 4) * LDC + r0 + g]);
      aP[3] = split_tf32(sdP[(i + 4) * LDC + r0 + g + 8]);
      const int o0 = i * LDK + f0 + g, o1 = (i + 4) * LDK + f0 + g;
      bk[0] = split_tf32(sK[o0] * sE1[o0]);
      bk[1] = split_tf32(sK[o1] * sE1[o1]);
      bq[0] = split_tf32(sQ[o0] * sE1[o0]);
      bq[1] = split_tf32(sQ[o1] * sE1[o1]);
      if (ks < 2) {
        mma3(accD, aA, bk);
        mma3(accD, aP, bq);
      } else {
        mma3(accO, aA, bk);
        mma3(accO, aP, bq);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int jj = g + ((e & 2) ? 8 : 0), j = r0 + jj, f = f0 + 2 * t + (e & 1), o = j * LDK + f;
      const float col = accD[e] * sE2d[jj * LDK + f] + accO[e] * sE2o[jj * LDK + f];
      sDk[o] += col;
      sDc[o] -= sK[o] * col;
    }
  }
  __syncthreads();
}

// The interaction terms of factored_terms for C = 64 on tf32 warp MMAs, one
// pass, no shared scratch and no barriers: warp w owns the 16 x 16 output
// tile of row block I = w / 2 and channels 16 (w % 2) .. + 15 (K = 32) and
// accumulates in registers, over every column block J <= I, the row terms of
// its rows and the column terms of the same rows (columns of block I); each
// A fragment feeds both 8-channel halves.  The split-exponent factors are
// formed on the fly from c (natural units).  Requires every 16-row block's
// decay span to be at most 80 (checked by the caller).
// Each product rounds its operands to tf32 once.  Every pair (i, j) enters
// dc twice, as a row term of i and as a column term of j, and the reverse
// cumulative sum of dc cancels the pairs that do not straddle the row; so
// that this cancellation is exact, both entries of a pair are formed from
// the same rounded factors: the row term multiplies its product by the
// rounded operand that the column term of the pair feeds to the MMA (and the
// other way round), and both use the same reference row of the split
// exponent.  dq and dk keep the fp32 factors.  (Splitting the operands into
// tf32 hi/lo pairs instead, with three products each, costs twice the time.)
__device__ __forceinline__ float tf32f(float x) { return __uint_as_float(to_tf32(x)); }

template <int K, int LDK_ = K + 1, int LDC_ = 65>
__device__ void factored_terms_tf32(const float* sK, const float* sQ, const float* sC, const float* sdA,
                                    const float* sdP, float* sDq, float* sDk, float* sDc) {
  constexpr int C = 64, LDK = LDK_, LDC = LDC_, NH = K / 16;
  static_assert(4 * NH == NTHREADS / 32, "one 16 x 16 tile per warp");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int I = warp / NH, fb = (warp % NH) * 16, i0 = I * BS;
  float totA[2][4] = {}, totP[2][4] = {}, dcr[2][4] = {};
  // row terms: rows of block I against the columns of every block J <= I
  for (int J = 0; J <= I; ++J) {
    const int r0 = J * BS, ref = (I == J) ? r0 + BS / 2 - 1 : r0 + BS - 1;
    float accA[2][4] = {}, accP[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int j = r0 + ks * 8 + t;
      const uint32_t aA[4] = {to_tf32(sdA[(i0 + g) * LDC + j]), to_tf32(sdA[(i0 + g + 8) * LDC + j]),
                              to_tf32(sdA[(i0 + g) * LDC + j + 4]), to_tf32(sdA[(i0 + g + 8) * LDC + j + 4])};
      const uint32_t aP[4] = {to_tf32(sdP[(i0 + g) * LDC + j]), to_tf32(sdP[(i0 + g + 8) * LDC + j]),
                              to_tf32(sdP[(i0 + g) * LDC + j + 4]), to_tf32(sdP[(i0 + g + 8) * LDC + j + 4])};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int fa = fb + 8 * h + g;
        const float cr = sC[ref * LDK + fa];
        const uint32_t bw[2] = {to_tf32(sK[j * LDK + fa] * __expf(cr - sC[j * LDK + fa])),
                                to_tf32(sK[(j + 4) * LDK + fa] * __expf(cr - sC[(j + 4) * LDK + fa]))};
        mma_16x8x8(accA[h], aA, bw);
        mma_16x8x8(accP[h], aP, bw);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + g + ((e & 2) ? 8 : 0), f = fb + 8 * h + 2 * t + (e & 1);
        const float e1 = __expf(sC[i * LDK + f] - sC[ref * LDK + f]);
        totA[h][e] = fmaf(accA[h][e], e1, totA[h][e]);
        totP[h][e] = fmaf(accP[h][e], e1, totP[h][e]);
        const float ak = tf32f(sK[i * LDK + f] * e1), aq = tf32f(sQ[i * LDK + f] * e1);
        dcr[h][e] = fmaf(accA[h][e], ak, fmaf(accP[h][e], aq, dcr[h][e]));
      }
  }
  // column terms: the columns of block I against its own rows and all rows below
  float accD[2][4] = {}, accO[2][4] = {};
  const int rd = i0 + BS / 2 - 1, ro = i0 + BS - 1;
  for (int ks = 0; ks < (C - i0) / 8; ++ks) {
    const int i = i0 + ks * 8 + t, ref = (ks < 2) ? rd : ro;
    const uint32_t aA[4] = {to_tf32(sdA[i * LDC + i0 + g]), to_tf32(sdA[i * LDC + i0 + g + 8]),
                            to_tf32(sdA[(i + 4) * LDC + i0 + g]), to_tf32(sdA[(i + 4) * LDC + i0 + g + 8])};
    const uint32_t aP[4] = {to_tf32(sdP[i * LDC + i0 + g]), to_tf32(sdP[i * LDC + i0 + g + 8]),
                            to_tf32(sdP[(i + 4) * LDC + i0 + g]), to_tf32(sdP[(i + 4) * LDC + i0 + g + 8])};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int fa = fb + 8 * h + g;
      const float cr = sC[ref * LDK + fa];
      const float x0 = __expf(sC[i * LDK + fa] - cr), x1 = __expf(sC[(i + 4) * LDK + fa] - cr);
      const uint32_t bk[2] = {to_tf32(sK[i * LDK + fa] * x0), to_tf32(sK[(i + 4) * LDK + fa] * x1)};
      const uint32_t bq[2] = {to_tf32(sQ[i * LDK + fa] * x0), to_tf32(sQ[(i + 4) * LDK + fa] * x1)};
      if (ks < 2) {
        mma_16x8x8(accD[h], aA, bk);
        mma_16x8x8(accD[h], aP, bq);
      } else {
        mma_16x8x8(accO[h], aA, bk);
        mma_16x8x8(accO[h], aP, bq);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + g + ((e & 2) ? 8 : 0), f = fb + 8 * h + 2 * t + (e & 1), o = i * LDK + f;
      const float ci = sC[o], kk = sK[o];
      const float yd = __expf(sC[rd * LDK + f] - ci), yo = __expf(sC[ro * LDK + f] - ci);
      const float col = accD[h][e] * yd + accO[h][e] * yo;
      const float dcc = accD[h][e] * tf32f(kk * yd) + accO[h][e] * tf32f(kk * yo);
      sDk[o] += totA[h][e] + col;
      sDq[o] += totP[h][e];
      sDc[o] += dcr[h][e] - dcc;
    }
  __syncthreads();
}

template <int K, int C, bool PRECISE, bool USE_MMA, int LDK_ = K + 1, int LDC_ = C + 1>
__device__ void factored_terms(const float* sK, const float* sQ, const float* sC, const float* sdA,
                               const float* sdP, float* sE1, float* sE2o, float* sE2d, int* sFlag,
                               float* sDq, float* sDk, float* sDc) {
  constexpr int NB = C / BS;
  for (int J = 0; J < NB; ++J) {
    const bool pairwise = block_factors<K, C, PRECISE, LDK_>(J, sC, sE1, sE2o, sE2d, sFlag);
    if (USE_MMA && !pairwise)
      factored_block_mma<K, C, LDK_, LDC_>(J, sK, sQ, sdA, sdP, sE1, sE2o, sE2d, sDq, sDk, sDc);
    else
      factored_block_scalar<K, C, PRECISE, LDK_, LDC_>(J, pairwise, sK, sQ, sC, sdA, sdP, sE1, sE2o, sE2d, sDq,
                                                       sDk, sDc);
  }
}

}  // namespace kda
