// Tensor-core (tcgen05) reverse pass of the KDA backward for K = V = 128,
// bf16 q/k/dO, fp32 g/beta: the gradient of the state leaving every 64-step
// chunk, and dS0.
//
// From the chunk algebra (kda_tc_chunk.cuh) the gradient of the state entering
// a chunk, given the gradient dM of the state leaving it, is
//   dU  = P^T dO + (K o e^{c_last - c}) dM
//   dR  = T^T dU
//   dM_in = diag(e^{c_last}) dM + (Q~ o e^c)^T dO - (diag(beta) K o e^c)^T dR
// ("recurrent.py", KDAFunction.backward, taken a chunk at a time; dM needs no
// forward state).  One CTA per (b, hv) walks the chunks in reverse with dM^T
// held in TMEM (lane = value column n, column = key channel f):
//   dU^T  = dO^T P + dM^T (K o e^{c_last-c})^T      (A = dO^T or dM^T, both in TMEM)
//   dR^T  = dU^T T
//   dM_in^T = dM^T diag(e^{c_last}) + dO^T (Q~ o e^c) - dR^T (diag(beta) K o e^c)
// P and T come from the forward's interaction record as ready operand images.
// The gradient of the state leaving every chunk is stored (at the chunk's odd
// index of the 32-step state layout, or its even one when the sequence ends in
// the chunk's first half); the per-chunk gradient kernel reads it there.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "kda_internal.h"
#include "kda_tc_chunk.cuh"

namespace kda {

__device__ unsigned int g_kda_bwd_device_error;  // this file's kernels (one flag per translation unit)

namespace tcb {
using namespace tcc;
constexpr uint32_t OP_KED = OP, OP_QET = OP + 32768, OP_NKET = OP + 65536;
// the chunk's P^T and T^T images, above the operands (the raw region then
// takes the next chunk's rows while this chunk's products run)
constexpr uint32_t IMG_PT = OP + 98304, IMG_TT = OP + 114688;
static_assert(IMG_TT + 16384 <= SMALL, "state-gradient shared-memory map");
constexpr uint32_t TM_S = 0, TM_DU = 128, TM_DR = 192, TM_DOT = 256;
}  // namespace tcb

// four fp32 values rounded to fp16 into 8 bytes of shared memory
__device__ __forceinline__ void st4h(__half* p, const float* v) {
  const __half2 lo = __floats2half2_rn(v[0], v[1]), hi = __floats2half2_rn(v[2], v[3]);
  uint2 u;
  u.x = *reinterpret_cast<const unsigned*>(&lo);
  u.y = *reinterpret_cast<const unsigned*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}
__global__ void __launch_bounds__(256, 1) kda_bwd_dstate_tc_kernel(BwdArgs a) {
  using namespace tcb;
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

  const int head_ = a.head0 + blockIdx.x;
  const int hv = head_ % a.HV, sq = head_ / a.HV;  // batch row, or sequence of a packed batch
  const int b = row_of(a, sq), c0 = chunk_begin(a, sq), c1 = chunk_end(a, sq);
  const int G = a.HV / a.H, h = hv / G, T = a.T;
  const size_t head = (size_t)sq * a.HV + hv;
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* dog = static_cast<const __nv_bfloat16*>(a.dO);
  float* sBeta = cx.beta();
  float* sEl = reinterpret_cast<float*>(sm + S_EL);
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

  {  // gradient of the final state, transposed
    for (int cb = 0; cb < 2; ++cb) {
      const int f0 = hcol * 64 + cb * 32;
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        r[j] = __float_as_uint(a.dS_T ? a.dS_T[(head * KD + f0 + j) * VD + Lr] : 0.f);
      tmem_st32(tm + lo + TM_S + f0, r);
    }
    tmem_wait_st();
  }
  fence_before();
  __syncthreads();

  // Copies run one chunk ahead, in cp.async groups committed in the order
  // raw(c1-1), images(c1-1), raw(c1-2), images(c1-2), ...: a chunk's raw rows
  // are requested once the previous chunk's rows are consumed, its images
  // once the previous chunk's products have read theirs.
  if (c1 > c0) {
    const int2 sp = chunk_span(a, c1 - 1);
    load_raw_issue<NTH, true>(cx, qg, kg, dog, a.g, a.beta, b, T, sp.x, sp.y, a.H, a.HV, h, hv);
    cp_async_commit();
    const float* irec = a.inter + chunk_gc(a, sq, hv, c1 - 1) * INTER_REC;
    copy_image(cx, IMG_PT, irec);             // P^T: (row i, K j) = P[j][i]
    copy_image(cx, IMG_TT, irec + INTER_TT);  // T^T: (row i, K j) = T[j][i]
    cp_async_commit();
  }
  for (int ch = c1 - 1; ch >= c0; --ch) {
    cp_async_wait_group<1>();  // this chunk's raw rows (its images may still be in flight)
    __syncthreads();
    cumsum_span(cx);

    // ---------------------------------------------------------------- operands of the gradient products
    {
      {  // K o e^{c_last-c} as [i][f]: thread items of 4 channels, 16-byte stores
        const int fq = item_f(cx);
        const float4 c63v = ld4(sC + 63 * LDCF + fq);
        const float c63[4] = {c63v.x, c63v.y, c63v.z, c63v.w};
        for (int m = 0; m < 8; ++m) {
          const int i = item_row(cx, m);
          const float4 c4 = ld4(sC + i * LDCF + fq);
          float kf[4];
          bf16x4(sm + RAW_K + raw_off(i, fq), kf);
          st_tf32x4(sm, OP_KED + kmaj(i, fq, 128), kf[0] * ex2(c63[0] - c4.x), kf[1] * ex2(c63[1] - c4.y),
                    kf[2] * ex2(c63[2] - c4.z), kf[3] * ex2(c63[3] - c4.w));
        }
      }
      {  // (Q~ o e^c)^T and -(diag(beta) K o e^c)^T as [f][i]: one channel x 4 rows, 16-byte stores
        const int f = tid & 127;
        for (int m = 0; m < 8; ++m) {
          const int i0 = ((tid >> 7) + 2 * m) * 4;
          float qe[4], nke[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            const float e = ex2(sC[i * LDCF + f]);
            const uint32_t o = raw_off(i, f);
            qe[u] = a.scale * __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + RAW_Q + o)) * e;
            nke[u] = -sBeta[i] * __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + RAW_K + o)) * e;
          }
          st_tf32x4(sm, OP_QET + kmaj(f, i0, 64), qe[0], qe[1], qe[2], qe[3]);
          st_tf32x4(sm, OP_NKET + kmaj(f, i0, 64), nke[0], nke[1], nke[2], nke[3]);
        }
      }
      if (tid < KD) sEl[tid] = ex2(sC[63 * LDCF + tid]);
      // dO^T into TMEM: lane n, columns j
      {
        uint32_t r[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
          r[jj] = tf32_rna(__bfloat162float(
              *reinterpret_cast<const __nv_bfloat16*>(sm + RAW_X + raw_off(hcol * 32 + jj, Lr))));
        tmem_st32(tm + lo + TM_DOT + hcol * 32, r);
        tmem_wait_st();
      }
    }
    fence_before();
    __syncthreads();  // this chunk's raw rows are consumed: the next chunk's may come in
    if (ch > c0) {
      const int2 sp = chunk_span(a, ch - 1);
      load_raw_issue<NTH, true>(cx, qg, kg, dog, a.g, a.beta, b, T, sp.x, sp.y, a.H, a.HV, h, hv);
    }
    cp_async_commit();           // (an empty group on the last chunk keeps the count uniform)
    cp_async_wait_group<1>();    // this chunk's images
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {  // dU^T = dO^T P + dM^T (K o e^{c_last-c})^T
      fence_after();
      const uint32_t id = idesc_tf32(128, 64);
      for (int ks = 0; ks < 8; ++ks)
        mma_ts(tm + TM_DU, tm + TM_DOT + ks * 8, desc(sb + IMG_PT + ks * 256, 2048), id, ks > 0);
      for (int ks = 0; ks < 16; ++ks)
        mma_ts(tm + TM_DU, tm + TM_S + ks * 8, desc(sb + OP_KED + ks * 256, 4096), id, 1);
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }
    if (tid == 0) {  // dR^T = dU^T T
      const uint32_t id = idesc_tf32(128, 64);
      for (int ks = 0; ks < 8; ++ks)
        mma_ts(tm + TM_DR, tm + TM_DU + ks * 8, desc(sb + IMG_TT + ks * 256, 2048), id, ks > 0);
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }
    if (ch > c0) {  // the products have read this chunk's images: the next chunk's may come in
      const float* irec = a.inter + chunk_gc(a, sq, hv, ch - 1) * INTER_REC;
      copy_image(cx, IMG_PT, irec);
      copy_image(cx, IMG_TT, irec + INTER_TT);
    }
    cp_async_commit();

    // ---------------------------------------------------------------- store dM (leaving this chunk); start dM_in
    float sv[2][32];  // dM leaving this chunk (this thread's lane, 64 channels), stored once
                      // the products below are under way
    {
      uint32_t r[32];
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hcol * 64 + cb * 32;
        tmem_ld32(tm + lo + TM_S + f0, sv[cb]);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(sv[cb][j] * sEl[f0 + j]);
        tmem_st32(tm + lo + TM_S + f0, r);
      }
      tmem_wait_st();
    }
    fence_before();
    __syncthreads();
    if (tid == 0) {
      fence_after();
      const uint32_t id = idesc_tf32(128, 128);
      for (int ks = 0; ks < 8; ++ks) {
        mma_ts(tm + TM_S, tm + TM_DOT + ks * 8, desc(sb + OP_QET + ks * 256, 2048), id, 1);
        mma_ts(tm + TM_S, tm + TM_DR + ks * 8, desc(sb + OP_NKET + ks * 256, 2048), id, 1);
      }
      commit(bar);
    }
    {
      float* slot = a.dstates + dstate_slot(a, sq, hv, ch) * (KD * VD);
      store_slot32(slot, hcol * 2, Lr, sv[0]);
      store_slot32(slot, hcol * 2 + 1, Lr, sv[1]);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }
    fence_before();
    __syncthreads();
  }

  cp_async_wait_all();  // (copies still in flight after an early exit)
  if (!failed && a.dS0) {
    fence_after();
    for (int cb = 0; cb < 2; ++cb) {
      const int f0 = hcol * 64 + cb * 32;
      float s[32];
      tmem_ld32(tm + lo + TM_S + f0, s);
#pragma unroll
      for (int j = 0; j < 32; ++j) a.dS0[(head * KD + f0 + j) * VD + Lr] = s[j];
    }
  }
  fence_before();
  __syncthreads();
  if (cx.warp == 0) tmem_dealloc(tm, 512);
  if (failed && tid == 0) atomicOr(&g_kda_bwd_device_error, 1u);
}

bool bwd_tc_eligible(const BwdArgs& a, int dtype) {
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  return dtype == 1 && a.K == 128 && a.V == 128 && a.gws != nullptr && a.inter != nullptr && al16(a.q) &&
         al16(a.k) && al16(a.v) && al16(a.dO) && al16(a.g) && al16(a.dq) && al16(a.dv);
}

static int launch_bwd_dstate_tc(const BwdArgs& a, int nheads, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kda_bwd_dstate_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tcc::SMEM_BYTES);
  if (e != cudaSuccess) return set_cuda_error("kda_bwd: cudaFuncSetAttribute", e);
  kda_bwd_dstate_tc_kernel<<<nheads, tcc::NTH, tcc::SMEM_BYTES, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_bwd: tensor-core state-gradient launch", e);
  return 0;
}


// ============================================================================
// Per-chunk gradient products on the tensor cores (K = V = 128, C = 64).
//
// One CTA per (b, hv, chunk), all chunks in parallel.  With M the state
// entering the chunk and dM the gradient of the state leaving it (both from
// the workspace), it recomputes
//   X = V - (K o e^c) M,  U = T diag(beta) X,  dU = P^T dO + (K o e^{c_last-c}) dM,
//   dR = T^T dU,  dv = diag(beta) dR,
// and forms every product that sums over the value columns n:
//   dP = dO U^T,  dA = -dR U^T,  dQE = dO M^T,  dKE' = -dR M^T (dKE = diag(beta) dKE'),
//   dKEd = U dM^T,  dbeta_R_i = sum_n dR_in X_in,  dEl_f = sum_n M_fn dM_fn,
// writing them (with Ah) to a per-chunk record that kda_bwd_assemble_kernel
// turns into dq, dk, dg and dbeta.  Lane-n products use the transposed forms
// (A operands M^T, dM^T, dO^T, X^T, dU^T in TMEM); the sums over n contract
// [dO; -dR] against U, M and dM staged in shared memory.
// ============================================================================
namespace tcg {
using namespace tcc;
// Shared memory: K o e^c and K o e^{c_last-c} until the first products, then U
// over them; [dO; -dR] at the top of the operand region; the T^T, P^T and T
// images in the raw region once the raw chunk is consumed; M or dM staged as
// [f][n] over the raw region after the second products (written from their
// transposed TMEM copies).  U, [dO; -dR], M and dM use the padded layout
// (LBO 144), which their lane-per-column stores need.
constexpr uint32_t OP_KE = OP, OP_KED = OP + 32768, OP_U = OP, OP_PBR = OP + 36864, OP_DO = OP + 73728;
// the V rows (bf16 [i][n], 16 KB) wait in the -dR half of [dO; -dR] until X is formed
constexpr uint32_t OP_V = OP_DO + 64 * 128 * 36 / 8;
// dv rows (bf16 [i][n], 16 KB) are staged in the dead K o e^{c_last-c} operand
// (after the first products, clear of U, the dbeta_R partials and the record)
constexpr uint32_t OP_DV = OP + 48128;
static_assert(OP_DV >= OP_PBR + 1024 && OP_DV + 16384 <= OP_KED + 32768 && OP_DV >= 4 * 32768,
              "dv staging");
constexpr uint32_t R_TT = 16384, R_MB = 0;
constexpr uint32_t PAD_SBO = 128 * 36;  // bytes per 8 rows of a padded 128-wide K tile
static_assert(OP_DO + 2 * 64 * PAD_SBO / 8 <= SMALL && OP_PBR + 1024 <= OP_DO && R_MB + 16 * PAD_SBO <= OP &&
                  R_TT + 16384 <= R_P,
              "gradient-kernel shared-memory map");
// TMEM columns: M^T and dM^T stay until they are staged as [f][n] operands
// for the third and fourth products (U at 448, dR over the spent dO^T)
constexpr uint32_t TM_M = 0, TM_U = 448, TM_QK = 0, TM_DM = 128, TM_DR = 256, TM_KED = 128, TM_DOT = 256,
                   TM_PA = 256, TM_X = 320, TM_DU = 384;
}  // namespace tcg

// A K x V state held transposed in TMEM (lane n, column f; columns tmc ..
// tmc + 127) written to R_MB as the [f][n] operand (padded K-major layout):
// each thread its lane n and the 64 channels of its column half.
__device__ __forceinline__ void stage_fn(const tcc::Ctx& cx, uint32_t tmc) {
  using namespace tcg;
#pragma unroll
  for (int cb = 0; cb < 2; ++cb) {
    const int f0 = cx.hcol * 64 + cb * 32;
    float v[32];
    tc::tmem_ld32(cx.tm + cx.lo + tmc + f0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) *reinterpret_cast<float*>(cx.sm + R_MB + tc::kmaj_pad(f0 + j, cx.Lr, 128)) = v[j];
  }
}

__global__ void __launch_bounds__(256, 1) kda_bwd_grads_tc_kernel(BwdArgs a) {
  using namespace tcg;
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
  const int tid = cx.tid, hcol = cx.hcol, Lr = cx.Lr, lane = cx.lane;
  const uint32_t lo = cx.lo, sb = cx.sb;

  const int G = a.HV / a.H, T = a.T;
  const int NT = a.ctab ? a.NC : (T + C - 1) / C;
  const int items = a.item1 > 0 ? a.item1 : NT * a.HV * (a.ctab ? 1 : a.B);
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
  const __nv_bfloat16* dog = static_cast<const __nv_bfloat16*>(a.dO);
  __nv_bfloat16* dvg = static_cast<__nv_bfloat16*>(a.dv);
  float* sBeta = cx.beta();
  float* sDEl = reinterpret_cast<float*>(sm + S_EL);    // 128 floats
  float* sDbR = reinterpret_cast<float*>(sm + S_EMID);  // 64 floats
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S_BAR);
  uint32_t* sTm = reinterpret_cast<uint32_t*>(sm + S_TMEM);
  const float* sC = cx.c();
  // per-subpartition partial sums, added in a fixed order (deterministic)
  float* partEl = reinterpret_cast<float*>(sm + R_AH);   // [4][128], once Ah is in the record
  float* partBr = reinterpret_cast<float*>(sm + OP_PBR);  // [4][64], once K o e^{c_last-c} is consumed

  if (cx.warp == 0) tmem_alloc(sTm, 512);
  if (tid == 0) mbar_init(bar, 1);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = *sTm;
  cx.tm = tm;
  uint32_t phase = 0;
  bool failed = false;

  // one item per CTA: chunk ch of batch row sq (packed sequences: chunk ch of
  // the table, sq = 0); items run chunk fastest, then value head, then batch row
  for (int item = a.item0 + blockIdx.x; item < items && !failed; item += gridDim.x) {
    const int ch = item % NT, hv = (item / NT) % a.HV, sq = item / (NT * a.HV);
    const int h = hv / G, b = row_of(a, sq);
    const int2 sp = chunk_span(a, ch);
    const int t0 = sp.x, L = sp.y;
    const size_t gc = chunk_gc(a, sq, hv, ch);
    float* rec = a.gws + gc * GREC;
    // ---------------------------------------------------------------- loads
    const float* irec = a.inter + gc * INTER_REC;  // P^T, T, T^T images of this chunk (forward)
    const float* mst = a.states + state_slot(a, sq, hv, ch) * (KD * VD);     // M: state entering the chunk
    const float* dmst = a.dstates + dstate_slot(a, sq, hv, ch) * (KD * VD);  // dM: gradient of the leaving state
    load_raw_issue(cx, qg, kg, dog, a.g, a.beta, b, T, t0, L, a.H, a.HV, h, hv);
    for (int x = tid; x < C * 16; x += NTH) {  // V rows [i][n] (bf16) into the -dR half of [dO; -dR]
      const int i = x >> 4, c16 = x & 15;
      cp_async16(sb + OP_V + x * 16, vg + (((size_t)b * T + t0 + (i < L ? i : 0)) * a.HV + hv) * VD + c16 * 8, i < L);
    }
    if (tid < 9) prefetch_l2(mst + tid * 1024, tid < 8 ? 4096 : 2048);  // (fp16 values and their scales)
    else if (tid >= 16 && tid < 25) prefetch_l2(dmst + (tid - 16) * 1024, tid < 24 ? 4096 : 2048);
    else if (tid == 32) prefetch_l2(irec, 2 * 16384);
    else if (tid == 33) prefetch_l2(irec + INTER_TT, 16384);
    if (!load_raw_wait(cx)) { failed = true; break; }
    cumsum_span(cx);

    // ---------------------------------------------------------------- K o e^c, K o e^{c_last-c}, dO, dO^T
    {
      const int fq = item_f(cx);
      const float4 c63v = ld4(sC + 63 * LDCF + fq);
      const float c63[4] = {c63v.x, c63v.y, c63v.z, c63v.w};
      for (int m = 0; m < 8; ++m) {
        const int i = item_row(cx, m);
        const float4 c4 = ld4(sC + i * LDCF + fq);
        const float c[4] = {c4.x, c4.y, c4.z, c4.w};
        float kf[4], df[4];
        bf16x4(sm + RAW_K + raw_off(i, fq), kf);
        bf16x4(sm + RAW_X + raw_off(i, fq), df);
        float e[4], ed[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          e[u] = ex2(c[u]);
          ed[u] = ex2(c63[u] - c[u]);
        }
        st_tf32x4(sm, OP_KE + kmaj(i, fq, 128), kf[0] * e[0], kf[1] * e[1], kf[2] * e[2], kf[3] * e[3]);
        st_tf32x4(sm, OP_KED + kmaj(i, fq, 128), kf[0] * ed[0], kf[1] * ed[1], kf[2] * ed[2], kf[3] * ed[3]);
        st_tf32x4(sm, OP_DO + kmaj_pad(i, fq, 128), df[0], df[1], df[2], df[3]);
      }
      uint32_t r[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj)
        r[jj] = tf32_rna(__bfloat162float(
              *reinterpret_cast<const __nv_bfloat16*>(sm + RAW_X + raw_off(hcol * 32 + jj, Lr))));
      tmem_st32(tm + lo + TM_DOT + hcol * 32, r);
      tmem_wait_st();
    }
    fence_async_smem();
    fence_before();
    __syncthreads();  // raw inputs consumed
    copy_image(cx, R_P, irec);               // P^T: (row i, K j) = P[j][i]
    copy_image(cx, R_T, irec + INTER_T);     // T:   (row i, K j) = T[i][j]
    copy_image(cx, R_TT, irec + INTER_TT);   // T^T: (row i, K j) = T[j][i]

    // ---------------------------------------------------------------- M^T, dM^T into TMEM; dEl
    {
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hcol * 64 + cb * 32;
        uint32_t rm[32], rd[32];
        float pr[32], mv[32], dv[32];
        load_slot32(mst, f0 / 32, Lr, mv);
        load_slot32(dmst, f0 / 32, Lr, dv);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          rm[j] = __float_as_uint(mv[j]);
          rd[j] = __float_as_uint(dv[j]);
          pr[j] = mv[j] * dv[j];
        }
        tmem_st32(tm + lo + TM_M + f0, rm);
        tmem_st32(tm + lo + TM_DM + f0, rd);
        partEl[cx.sub * KD + f0 + lane] = warp_sum32(pr, lane);
      }
      tmem_wait_st();
    }
    cp_async_wait_all();
    fence_async_smem();
    fence_before();
    __syncthreads();
    if (tid < KD) sDEl[tid] = ((partEl[tid] + partEl[KD + tid]) + partEl[2 * KD + tid]) + partEl[3 * KD + tid];
    if (tid == 0) {  // X'^T = M^T (K o e^c)^T ; dU^T = dO^T P + dM^T (K o e^{c_last-c})^T
      fence_after();
      const uint32_t id = idesc_tf32(128, 64);
      for (int ks = 0; ks < 16; ++ks)
        mma_ts(tm + TM_X, tm + TM_M + ks * 8, desc(sb + OP_KE + ks * 256, 4096), id, ks > 0);
      for (int ks = 0; ks < 8; ++ks)
        mma_ts(tm + TM_DU, tm + TM_DOT + ks * 8, desc(sb + R_P + ks * 256, 2048), id, ks > 0);
      for (int ks = 0; ks < 16; ++ks)
        mma_ts(tm + TM_DU, tm + TM_DM + ks * 8, desc(sb + OP_KED + ks * 256, 4096), id, 1);
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }
    float xs[32];  // X^T = V^T - X'^T (lane n, rows i of this warp half), kept for dbeta_R
    {
      float x[32];
      uint32_t r[32];
      tmem_ld32(tm + lo + TM_X + hcol * 32, x);
#pragma unroll
      const __nv_bfloat16* sV = reinterpret_cast<const __nv_bfloat16*>(sm + OP_V);
      for (int jj = 0; jj < 32; ++jj) {
        xs[jj] = __bfloat162float(sV[(hcol * 32 + jj) * VD + Lr]) - x[jj];
        r[jj] = tf32_rna(sBeta[hcol * 32 + jj] * xs[jj]);
      }
      tmem_st32(tm + lo + TM_X + hcol * 32, r);
      tmem_wait_st();
    }
    fence_before();
    __syncthreads();
    if (tid == 0) {  // U^T = (X^T diag(beta)) T^T ; dR^T = dU^T T
      fence_after();
      const uint32_t id = idesc_tf32(128, 64);
      for (int ks = 0; ks < 8; ++ks) {
        mma_ts(tm + TM_U, tm + TM_X + ks * 8, desc(sb + R_T + ks * 256, 2048), id, ks > 0);
        mma_ts(tm + TM_DR, tm + TM_DU + ks * 8, desc(sb + R_TT + ks * 256, 2048), id, ks > 0);
      }
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }

    // ---------------------------------------------------------------- dv, dbeta_R; U and -dR as [i][n] operands
    {
      float u[32], dr[32];
      tmem_ld32(tm + lo + TM_U + hcol * 32, u);
      tmem_ld32(tm + lo + TM_DR + hcol * 32, dr);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const int i = hcol * 32 + jj;
        reinterpret_cast<__nv_bfloat16*>(sm + OP_DV)[i * VD + Lr] = __float2bfloat16_rn(sBeta[i] * dr[jj]);
        st_tf32(sm, OP_U + kmaj_pad(i, Lr, 128), u[jj]);
        st_tf32(sm, OP_DO + kmaj_pad(64 + i, Lr, 128), -dr[jj]);
        xs[jj] *= dr[jj];
      }
      partBr[cx.sub * C + hcol * 32 + lane] = warp_sum32(xs, lane);
    }
    stage_fn(cx, TM_M);  // M as [f][n] for the sums over n (from M^T in TMEM)
    fence_before();
    fence_async_smem();
    __syncthreads();
    for (int x = tid; x < L * 16; x += NTH) {  // dv rows as 16-byte pieces
      const int i = x >> 4, c16 = x & 15;
      *reinterpret_cast<uint4*>(dvg + (((size_t)b * T + t0 + i) * a.HV + hv) * VD + c16 * 8) =
          *reinterpret_cast<const uint4*>(sm + OP_DV + x * 16);
    }
    if (tid < C) sDbR[tid] = ((partBr[tid] + partBr[C + tid]) + partBr[2 * C + tid]) + partBr[3 * C + tid];
    if (tid == 0) {  // [dP; dA] = [dO; -dR] U^T ; [dQE; dKE'] = [dO; -dR] M^T
      fence_after();
      for (int ks = 0; ks < 16; ++ks) {
        const uint64_t aD = desc(sb + OP_DO + ks * 288, PAD_SBO, 144);
        mma_ss(tm + TM_PA, aD, desc(sb + OP_U + ks * 288, PAD_SBO, 144), idesc_tf32(128, 64), ks > 0);
        mma_ss(tm + TM_QK, aD, desc(sb + R_MB + ks * 288, PAD_SBO, 144), idesc_tf32(128, 128), ks > 0);
      }
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }
    stage_fn(cx, TM_DM);  // dM as [f][n] (from dM^T in TMEM)
    fence_before();
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {  // dKEd = U dM^T
      fence_after();
      for (int ks = 0; ks < 16; ++ks)
        mma_ss(tm + TM_KED, desc(sb + OP_U + ks * 288, PAD_SBO, 144), desc(sb + R_MB + ks * 288, PAD_SBO, 144),
               idesc_tf32(64, 128), ks > 0);
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }

    // ---------------------------------------------------------------- record
    {  // the record staged in shared memory (now free) in its global layout, then bulk-stored
      __half* st = reinterpret_cast<__half*>(sm);  // fp16 [dP; dA] | [dQE; dKE'] | dKEd, as in the record
      static_assert(2 * (GH_KED + 8192) <= OP_DO, "record staging below [dO; -dR]");
      static_assert(2 * (GH_KED + 8192) == 4 * G_DBR, "fp32 tail follows the fp16 matrices");
      float v[32];
      tmem_ld32(tm + lo + TM_PA + hcol * 32, v);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) st4h(st + GH_PA + rec_off(Lr, hcol * 32 + 4 * q4, 64), v + 4 * q4);
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hcol * 64 + cb * 32;
        tmem_ld32(tm + lo + TM_QK + f0, v);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) st4h(st + GH_QK + rec_off(Lr, f0 + 4 * q4, 128), v + 4 * q4);
        tmem_ld32(tm + lo + TM_KED + f0, v);
        if (lane < 16) {
          const int r = cx.sub * 16 + lane;  // M = 64 accumulator layout
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) st4h(st + GH_KED + rec_off(r, f0 + 4 * q4, 128), v + 4 * q4);
        }
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        bulk_s2g(rec, sb, 32768);
        bulk_s2g(rec + 8192, sb + 32768, 32768);
        bulk_s2g(rec + G_DBR, sb + S_EMID, 256);
        bulk_s2g(rec + G_DEL, sb + S_EL, 512);
        bulk_commit();
        bulk_wait_read();
      }
    }
    // the record's shared-memory sources are read and every TMEM read-out is
    // complete before the next item overwrites them
    fence_before();
    __syncthreads();
  }

  fence_before();
  __syncthreads();
  if (cx.warp == 0) tmem_dealloc(tm, 512);
  if (failed && tid == 0) atomicOr(&g_kda_bwd_device_error, 1u);
}

static int launch_bwd_grads_tc(const BwdArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kda_bwd_grads_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tcc::SMEM_BYTES);
  if (e != cudaSuccess) return set_cuda_error("kda_bwd: cudaFuncSetAttribute", e);
  const int NT = a.ctab ? a.NC : (a.T + tcc::C - 1) / tcc::C;
  if (NT == 0) return 0;  // (packed batches of empty sequences)
  const long long items = (a.item1 > 0 ? a.item1 : (long long)NT * a.HV * (a.ctab ? 1 : a.B)) - a.item0;
  if (items <= 0) return 0;
  // one CTA per item (not persistent): when the kernel shares the GPU with the
  // state-gradient pass, the SMs that pass frees take the remaining items.
  // (An L2 prefetch of the inputs of the item one SM count further on, as
  // the assembly does, measured 0.36 ms slower per fwd+bwd step at B = 2,
  // H = 96, T = 4096.)
  kda_bwd_grads_tc_kernel<<<(int)items, tcc::NTH, tcc::SMEM_BYTES, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_bwd: tensor-core gradient launch", e);
  return 0;
}

// A non-blocking stream of the highest priority on the current device, made
// on first use and kept until exit (null if it cannot be made).
static cudaStream_t side_stream() {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    int lo = 0, hi = 0;
    cudaStream_t s = nullptr;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) == cudaSuccess &&
        cudaStreamCreateWithPriority(&s, cudaStreamNonBlocking, hi) == cudaSuccess)
      streams[dev] = s;
    else
      cudaGetLastError();
  }
  return streams[dev];
}

// The reverse state-gradient pass, the per-chunk gradient products and the
// assembly.  The pass has one CTA per (sequence, value head) and one CTA per
// SM; when the heads fill some waves of SMs and leave a partial last wave
// (heads A, then B), that wave runs on a high-priority side stream while the
// gradient products of heads A start in the SMs it leaves idle; then the
// assembly of heads A follows on the side stream while the gradient products
// of heads B run on the caller's stream (the two kernels load and compute in
// different phases), and the assembly of heads B ends the call.
int launch_bwd_tc_passes(const BwdArgs& a, cudaStream_t stream, AssembleLaunch assemble) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nheads = a.B * a.HV, NT = (a.T + tcc::C - 1) / tcc::C;
  const int nA = (nheads / sms) * sms;
  cudaStream_t side = (!a.ctab && nA > 0 && nA < nheads) ? side_stream() : nullptr;
  if (!side) {
    int rc = launch_bwd_dstate_tc(a, nheads, stream);
    if (!rc) rc = launch_bwd_grads_tc(a, stream);
    return rc ? rc : assemble(a, 0, nheads, stream);
  }
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};  // dstate(A) done, grads(A) done, side work done
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 3 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
  int rc = 0;
  BwdArgs aA = a, aB = a;
  aA.item0 = 0;
  aA.item1 = nA * NT;
  aB.head0 = nA;
  aB.item0 = nA * NT;
  aB.item1 = nheads * NT;
  if (e == cudaSuccess) rc = launch_bwd_dstate_tc(aA, nA, stream);
  if (e == cudaSuccess && !rc) e = cudaEventRecord(ev[0], stream);
  if (e == cudaSuccess && !rc) e = cudaStreamWaitEvent(side, ev[0], 0);
  if (e == cudaSuccess && !rc) {  // the side stream's work, joined back into the caller's stream
    rc = launch_bwd_dstate_tc(aB, nheads - nA, side);
    cudaEvent_t evB = nullptr;
    if (!rc) e = cudaEventCreateWithFlags(&evB, cudaEventDisableTiming);
    if (e == cudaSuccess && !rc) e = cudaEventRecord(evB, side);
    if (e == cudaSuccess && !rc) rc = launch_bwd_grads_tc(aA, stream);
    if (e == cudaSuccess && !rc) e = cudaEventRecord(ev[1], stream);
    if (e == cudaSuccess && !rc) e = cudaStreamWaitEvent(side, ev[1], 0);
    if (e == cudaSuccess && !rc) rc = assemble(a, 0, nA, side);
    const cudaError_t e2 = cudaEventRecord(ev[2], side);
    if (e == cudaSuccess) e = e2;
    if (e == cudaSuccess && !rc) e = cudaStreamWaitEvent(stream, evB, 0);
    if (e == cudaSuccess && !rc) rc = launch_bwd_grads_tc(aB, stream);
    if (e == cudaSuccess && !rc) rc = assemble(a, nA, nheads - nA, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, ev[2], 0);
    if (evB) cudaEventDestroy(evB);
  }
  for (int i = 0; i < 3; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);
  if (e != cudaSuccess) return set_cuda_error("kda_bwd: side-stream ordering", e);
  return rc;
}

}  // namespace kda

namespace kda {
int take_bwd_device_error(unsigned* out) {
  unsigned v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_kda_bwd_device_error, sizeof(v));
  if (e != cudaSuccess) return set_cuda_error("kda_device_status", e);
  e = cudaMemcpyToSymbol(g_kda_bwd_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return set_cuda_error("kda_device_status", e);
  *out = v;
  return 0;
}
}  // namespace kda
