// Tensor-core (tcgen05) chunked KDA prefill forward for K = V = 128, bf16
// q/k/v/o, fp32 g/beta/state.
//
// One CTA per (b, hv) carries the whole K x V fp32 state through the
// sequence in tensor memory (TMEM), transposed (lane = value column n,
// column = key channel f), so that it feeds the next products directly as
// their A operand.  Per chunk of C = 64 steps (chunk algebra of
// "research_layers.py", delta_recurrence, with erase = write = k and beta
// folded into the residual; the interaction products are in
// kda_tc_chunk.cuh):
//
//   T         = (I + diag(beta) Ah)^-1                     (CUDA cores)
//   W^T       = (diag(beta) K o e^c)^T T^T,  U0^T = (diag(beta) V)^T T^T
//   X^T       = M^T W^T,   O^T = M^T (Q~ o e^c)^T          (A = state in TMEM)
//   U^T       = U0^T - X^T
//   M'^T      = M^T diag(e^{c_last}) + U^T (K o e^{c_last - c})
//   O^T      += U^T P^T
//
// All products are tcgen05.mma kind::tf32 with fp32 accumulation in TMEM;
// the CUDA cores write the operands into shared memory in the K-major
// no-swizzle canonical layout (kda_tc.cuh), rounded to tf32.  With a state
// workspace the kernel also stores the state entering every 32 steps (the
// chunk start, and the mid-chunk state
// M_mid^T = M^T diag(e^{c_31}) + U^T[:, :32] (K o e^{c_31 - c})[:32]) for the
// backward.
#include <cuda_bf16.h>

#include "kda_internal.h"
#include "kda_tc_chunk.cuh"

namespace kda {

__device__ unsigned int g_kda_device_error;

namespace tcf {
using namespace tcc;
constexpr uint32_t OP_BKET = OP, OP_BVT = OP + 32768, OP_QE = OP + 65536, OP_KEDT = OP + 98304,
                   OP_KMID = OP + 131072;
// TMEM columns
constexpr uint32_t TM_S = 0, TM_X = 128, TM_O = 192, TM_U = 256, TM_W = 320, TM_APA = 384, TM_APB = 448,
                   TM_MID = 320;  // mid-chunk state (after the W and interaction tiles are read)
}  // namespace tcf

__global__ void __launch_bounds__(256, 1) kda_fwd_tc_kernel(FwdArgs a) {
  using namespace tcf;
  using namespace tc;
  extern __shared__ __align__(1024) unsigned char sm[];
  Ctx cx;
  cx.sm = sm;
  cx.sb = smem_u32(sm);
  cx.tid = threadIdx.x;
  cx.warp = cx.tid >> 5;
  cx.lane = cx.tid & 31;
  cx.sub = cx.warp & 3;
  cx.hcol = cx.warp >> 2;
  cx.Lr = cx.sub * 32 + cx.lane;
  cx.lo = (uint32_t)(cx.sub * 32) << 16;
  const int tid = cx.tid, hcol = cx.hcol, Lr = cx.Lr;
  const uint32_t lo = cx.lo, sb = cx.sb;

  const int hv = blockIdx.x, b = blockIdx.y;
  const int G = a.HV / a.H, h = hv / G, T = a.T, NT = (T + C - 1) / C;
  const int NT32 = (T + 31) / 32;  // the state workspace holds the state entering every 32 steps
  const size_t head = (size_t)b * a.HV + hv;
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
  __nv_bfloat16* og = static_cast<__nv_bfloat16*>(a.o);
  float* sBeta = cx.beta();
  float* sEl = reinterpret_cast<float*>(sm + S_EL);
  float* sE31 = reinterpret_cast<float*>(sm + S_EMID);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S_BAR);
  uint32_t* sTm = reinterpret_cast<uint32_t*>(sm + S_TMEM);
  const float* sC = cx.c();

  if (cx.warp == 0) tmem_alloc(sTm, 512);
  if (tid == 0) mbar_init(bar, 1);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = *sTm;
  cx.tm = tm;
  uint32_t phase = 0;
  bool failed = false;

  {  // entering state, transposed: lane n, column f
    for (int cb = 0; cb < 2; ++cb) {
      const int f0 = hcol * 64 + cb * 32;
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        r[j] = __float_as_uint(a.S0 ? a.S0[(head * KD + f0 + j) * VD + Lr] : 0.f);
      tmem_st32(tm + lo + TM_S + f0, r);
    }
    tmem_wait_st();
  }
  fence_before();
  __syncthreads();

  for (int ch = 0; ch < NT; ++ch) {
    const int t0 = ch * C, L = min(C, T - t0);
    load_raw_issue(cx, qg, kg, vg, a.g, a.beta, b, T, t0, L, a.H, a.HV, h, hv);
    if (ch + 1 < NT) prefetch_chunk(cx, qg, kg, vg, a.g, b, T, t0 + C, min(C, T - t0 - C), a.H, a.HV, h, hv);
    load_raw_wait();
    const bool wide = cumsum_span(cx);
    build_op1_and_issue(cx, a.scale, tm + TM_APA, tm + TM_APB, bar);
    if (!wait_mma(bar, phase)) { failed = true; break; }

    // ---------------------------------------------------------------- state-product operands
    {  // Q~ o e^c as [i][f]: thread items of 4 channels, 16-byte stores
      const int fq = item_f(cx);
      for (int m = 0; m < 8; ++m) {
        const int i = item_row(cx, m);
        const float4 c4 = ld4(sC + i * LDCF + fq);
        float qf[4];
        bf16x4(sm + RAW_Q + i * 256 + fq * 2, qf);
        st_tf32x4(sm, OP_QE + kmaj(i, fq, 128), a.scale * qf[0] * ex2(c4.x), a.scale * qf[1] * ex2(c4.y),
                  a.scale * qf[2] * ex2(c4.z), a.scale * qf[3] * ex2(c4.w));
      }
    }
    {  // transposed operands [f][i]: thread items of one channel x 4 rows, 16-byte stores
      const int f = tid & 127;
      const float c63 = sC[63 * LDCF + f], c31 = sC[31 * LDCF + f];
      const __nv_bfloat16* kcol = reinterpret_cast<const __nv_bfloat16*>(sm + RAW_K) + f;
      const __nv_bfloat16* vcol = reinterpret_cast<const __nv_bfloat16*>(sm + RAW_X) + f;
      for (int m = 0; m < 8; ++m) {
        const int i0 = ((tid >> 7) + 2 * m) * 4;
        float bke[4], ked[4], bv[4], kmid[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u;
          const float c = sC[i * LDCF + f], kk = __bfloat162float(kcol[i * 128]), bi = sBeta[i];
          bke[u] = bi * kk * ex2(c);
          ked[u] = kk * ex2(c63 - c);
          bv[u] = bi * __bfloat162float(vcol[i * 128]);
          if (a.states && i0 < 32) kmid[u] = kk * ex2(c31 - c);
        }
        st_tf32x4(sm, OP_BKET + kmaj(f, i0, 64), bke[0], bke[1], bke[2], bke[3]);
        st_tf32x4(sm, OP_KEDT + kmaj(f, i0, 64), ked[0], ked[1], ked[2], ked[3]);
        st_tf32x4(sm, OP_BVT + kmaj(f, i0, 64), bv[0], bv[1], bv[2], bv[3]);
        if (a.states && i0 < 32) st_tf32x4(sm, OP_KMID + kmaj(f, i0, 32), kmid[0], kmid[1], kmid[2], kmid[3]);
      }
      if (tid < KD) {
        sEl[tid] = ex2(c63);
        sE31[tid] = ex2(c31);
      }
    }
    Pairwise pw;
    if (wide) pairwise_compute(cx, a.scale, pw);
    __syncthreads();  // raw inputs consumed; the raw region is reused below

    float* irec = a.inter ? a.inter + (head * NT + ch) * INTER_REC : nullptr;
    readout_ap(cx, tm + TM_APA, tm + TM_APB, false, wide, pw, irec);
    invert(cx);
    {  // T as the operand image (rows i, K = j); with a record also its T, T^T images and Ah
      const float* tr = reinterpret_cast<const float*>(sm + R_TROW);
      for (int x = tid; x < C * 16; x += NTH) {  // 16-byte piece x of the image: x * 16 = kmaj(i, j4, 64)
        const int i = ((x >> 7) << 3) | (x & 7), j4 = ((x >> 3) & 15) * 4;
        const float* p = tr + i * 65 + j4;
        const uint4 t = make_uint4(tf32_rna(p[0]), tf32_rna(p[1]), tf32_rna(p[2]), tf32_rna(p[3]));
        *reinterpret_cast<uint4*>(sm + R_T + x * 16) = t;
        if (irec) {
          const float* pc = tr + j4 * 65 + i;
          *reinterpret_cast<uint4*>(irec + INTER_T + x * 4) = t;
          *reinterpret_cast<uint4*>(irec + INTER_TT + x * 4) =
              make_uint4(tf32_rna(pc[0]), tf32_rna(pc[65]), tf32_rna(pc[130]), tf32_rna(pc[195]));
        }
      }
      if (irec) {
        const float* ah = reinterpret_cast<const float*>(sm + R_AH);
        for (int x = tid; x < C * C; x += NTH) irec[INTER_AH + x] = ah[(x >> 6) * 65 + (x & 63)];
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      fence_after();
      const uint32_t id = idesc_tf32(128, 64);
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t bT = desc(sb + R_T + ks * 256, 2048);
        mma_ss(tm + TM_W, desc(sb + OP_BKET + ks * 256, 2048), bT, id, ks > 0);
        mma_ss(tm + TM_U, desc(sb + OP_BVT + ks * 256, 2048), bT, id, ks > 0);
      }
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }

    // ---------------------------------------------------------------- W into shared memory
    {
      float v[32];
      tmem_ld32(tm + lo + TM_W + hcol * 32, v);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) st_tf32(sm, R_WOP + kmaj_pad(hcol * 32 + jj, Lr, 128), v[jj]);
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      fence_after();
      const uint32_t id = idesc_tf32(128, 64);
      for (int ks = 0; ks < 16; ++ks) {
        mma_ts(tm + TM_X, tm + TM_S + ks * 8, desc(sb + R_WOP + ks * 288, 4608, 144), id, ks > 0);
        mma_ts(tm + TM_O, tm + TM_S + ks * 8, desc(sb + OP_QE + ks * 256, 4096), id, ks > 0);
      }
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }

    // ---------------------------------------------------------------- U^T = U0^T - X^T ; M^T <- M^T diag(e^{c_last})
    {
      float u0[32], x[32];
      uint32_t r[32];
      tmem_ld32(tm + lo + TM_U + hcol * 32, u0);
      tmem_ld32(tm + lo + TM_X + hcol * 32, x);
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = tf32_rna(u0[j] - x[j]);
      tmem_st32(tm + lo + TM_U + hcol * 32, r);
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hcol * 64 + cb * 32;
        float s[32];
        tmem_ld32(tm + lo + TM_S + f0, s);
        if (a.states) {  // the state entering this chunk, and e^{c_31} M^T to start the mid state
          float* dst = a.states + ((head * NT32 + 2 * ch) * KD + f0) * VD + Lr;
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[(size_t)j * VD] = s[j];
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(s[j] * sE31[f0 + j]);
          tmem_st32(tm + lo + TM_MID + f0, r);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(s[j] * sEl[f0 + j]);
        tmem_st32(tm + lo + TM_S + f0, r);
      }
      tmem_wait_st();
    }
    fence_before();
    __syncthreads();
    if (tid == 0) {
      fence_after();
      const uint32_t idS = idesc_tf32(128, 128), idO = idesc_tf32(128, 64);
      for (int ks = 0; ks < 8; ++ks) {
        mma_ts(tm + TM_S, tm + TM_U + ks * 8, desc(sb + OP_KEDT + ks * 256, 2048), idS, 1);
        mma_ts(tm + TM_O, tm + TM_U + ks * 8, desc(sb + R_P + ks * 256, 2048), idO, 1);
      }
      if (a.states)
        for (int ks = 0; ks < 4; ++ks)
          mma_ts(tm + TM_MID, tm + TM_U + ks * 8, desc(sb + OP_KMID + ks * 256, 1024), idS, 1);
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }

    // ---------------------------------------------------------------- O out (and the mid-chunk state)
    if (a.states && 2 * ch + 1 < NT32) {
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hcol * 64 + cb * 32;
        float s[32];
        tmem_ld32(tm + lo + TM_MID + f0, s);
        float* dst = a.states + ((head * NT32 + 2 * ch + 1) * KD + f0) * VD + Lr;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[(size_t)j * VD] = s[j];
      }
    }
    if (a.o) {
      float v[32];
      tmem_ld32(tm + lo + TM_O + hcol * 32, v);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const int i = hcol * 32 + jj;
        if (i < L) og[(((size_t)b * T + t0 + i) * a.HV + hv) * VD + Lr] = __float2bfloat16_rn(v[jj]);
      }
    }
    fence_before();
    __syncthreads();
  }

  if (!failed && a.S_T) {
    fence_after();
    for (int cb = 0; cb < 2; ++cb) {
      const int f0 = hcol * 64 + cb * 32;
      float s[32];
      tmem_ld32(tm + lo + TM_S + f0, s);
#pragma unroll
      for (int j = 0; j < 32; ++j) a.S_T[(head * KD + f0 + j) * VD + Lr] = s[j];
    }
  }
  fence_before();
  __syncthreads();
  if (cx.warp == 0) tmem_dealloc(tm, 512);
  if (failed && tid == 0) atomicOr(&g_kda_device_error, 1u);
}

bool fwd_tc_eligible(const FwdArgs& a, int dtype) {
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  return dtype == 1 && a.K == 128 && a.V == 128 && al16(a.q) && al16(a.k) && al16(a.v) && al16(a.g);
}

int launch_fwd_tc(const FwdArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kda_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tcc::SMEM_BYTES);
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: cudaFuncSetAttribute", e);
  kda_fwd_tc_kernel<<<dim3(a.HV, a.B), tcc::NTH, tcc::SMEM_BYTES, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: tensor-core launch", e);
  return 0;
}

int take_device_error(unsigned* out) {
  unsigned v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_kda_device_error, sizeof(v));
  if (e != cudaSuccess) return set_cuda_error("kda_device_status", e);
  e = cudaMemcpyToSymbol(g_kda_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return set_cuda_error("kda_device_status", e);
  *out = v;
  return 0;
}

}  // namespace kda
