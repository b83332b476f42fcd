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
// workspace the kernel also stores the state entering every chunk (at even
// indices of the 32-step state layout) and the chunk's interaction record for
// the backward.
#include <cuda_bf16.h>

#include "kda_internal.h"
#include "kda_tc_chunk.cuh"

namespace kda {

__device__ unsigned int g_kda_device_error;

namespace tcf {
using namespace tcc;
constexpr uint32_t OP_BKET = OP, OP_BVT = OP + 32768, OP_QE = OP + 65536, OP_KEDT = OP + 98304;
// TMEM columns
constexpr uint32_t TM_S = 0, TM_X = 128, TM_O = 192, TM_U = 256, TM_W = 320, TM_APA = 384, TM_APB = 448;
}  // namespace tcf

// The chunks of the sequence s that a CTA carries: [c0, c1), chunk c at steps
// span(c).x .. + span(c).y - 1 of batch row `row` (uniform batches: sequence
// = batch row, chunk c at 64 c; packed sequences: the chunk table, row 0).
struct SeqChunks {
  int c0, c1, row;
  __device__ SeqChunks(const FwdArgs& a, int s) {
    if (a.ctab) {
      c0 = a.seq0[s];
      c1 = a.seq0[s + 1];
      row = 0;
    } else {
      c0 = 0;
      c1 = (a.T + tcc::C - 1) / tcc::C;
      row = s;
    }
  }
  __device__ int2 span(const FwdArgs& a, int c) const {
    if (a.ctab) return make_int2(a.ctab[2 * c], a.ctab[2 * c + 1]);
    return make_int2(c * tcc::C, min(tcc::C, a.T - c * tcc::C));
  }
};

// The state-independent part of one chunk: load, cumulative decay, the
// interaction products and their read-out, the inverse T, the operands of the
// state products (Q~ o e^c, (K o e^{c_last-c})^T in shared memory; e^{c_last}
// per channel) and
// W^T = (diag(beta) K o e^c)^T T^T, U0^T = (diag(beta) V)^T T^T in TMEM.  With
// `irec` it stores the chunk's interaction record.
// The chunk covers steps t0 .. t0 + L - 1 of batch row b (packed sequences:
// b = 0 and t0 on the packed axis); with Ln > 0 the next chunk of the same
// sequence (Ln steps from t0 + 64) is prefetched into L2.
// Returns false, block-uniformly, if a tensor-core wait ran out.
// With PREP the fused input preparation runs on the loaded chunk (FwdArgs::prep):
// q, k rows L2-normalised, g from z, beta from its logit.
template <int NTHR, bool PREP = false>
__device__ __forceinline__ bool fwd_chunk_head(const tcc::Ctx& cx, const FwdArgs& a, int b, int hv, int h,
                                               int t0, int L, int Ln, float* irec, uint64_t* bar,
                                               uint32_t& phase) {
  using namespace tcf;
  using namespace tc;
  unsigned char* sm = cx.sm;
  const uint32_t sb = cx.sb, tm = cx.tm;
  const int tid = cx.tid;
  const int T = a.T;
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
  const float* sBeta = cx.beta();
  float* sEl = reinterpret_cast<float*>(sm + S_EL);
  const float* sC = cx.c();
  const __nv_bfloat16* zg = static_cast<const __nv_bfloat16*>(a.prep.z);
  float dtb = 0.f, dec = 0.f;  // gate constants, loaded while the chunk's copies are in flight
  if constexpr (PREP) {
    load_raw_issue_prep<NTHR>(cx, qg, kg, vg, zg, a.beta, b, T, t0, L, a.H, a.HV, h, hv);
    dtb = a.prep.dt_bias[(size_t)hv * KD + (tid & 127)];
    dec = a.prep.A_log[hv];
    if (Ln > 0) prefetch_chunk(cx, qg, kg, vg, zg, b, T, t0 + C, Ln, a.H, a.HV, h, hv, 2);
  } else {
    load_raw_issue<NTHR>(cx, qg, kg, vg, a.g, a.beta, b, T, t0, L, a.H, a.HV, h, hv);
    if (Ln > 0) prefetch_chunk(cx, qg, kg, vg, a.g, b, T, t0 + C, Ln, a.H, a.HV, h, hv);
  }
  if (!load_raw_wait(cx)) return false;
  bool wide;
  if constexpr (PREP) {
    row_norms<NTHR>(cx, a.scale);
    wide = cumsum_span<true, NTHR>(cx, dtb, expf(dec), a.prep.gate_lb, L);
  } else {
    wide = cumsum_span(cx);
  }
  build_op1_and_issue<NTHR, PREP>(cx, a.scale, tm + TM_APA, tm + TM_APB, bar);
  if (!wait_mma(bar, phase)) return false;

  // ---------------------------------------------------------------- state-product operands
  {  // Q~ o e^c as [i][f]: thread items of 4 channels, 16-byte stores
    const int fq = item_f<NTHR>(cx);
    for (int m = 0; m < 2048 / NTHR; ++m) {
      const int i = item_row<NTHR>(cx, m);
      const float4 c4 = ld4(sC + i * LDCF + fq);
      const float qs = PREP ? sC[i * LDCF + NORM_Q] : a.scale;
      float qf[4];
      bf16x4(sm + RAW_Q + raw_off(i, fq), qf);
      st_tf32x4(sm, OP_QE + kmaj(i, fq, 128), qs * qf[0] * ex2(c4.x), qs * qf[1] * ex2(c4.y),
                qs * qf[2] * ex2(c4.z), qs * qf[3] * ex2(c4.w));
    }
  }
  {  // transposed operands [f][i]: thread items of one channel x 4 rows, 16-byte stores
    const int f = tid & 127;
    const float c63 = sC[63 * LDCF + f];

    for (int m = 0; m < 2048 / NTHR; ++m) {
      const int i0 = ((tid >> 7) + (NTHR / 128) * m) * 4;
      float bke[4], ked[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u;
        const float c = sC[i * LDCF + f], bi = sBeta[i];
        float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + RAW_K + raw_off(i, f)));
        if (PREP) kk *= sC[i * LDCF + NORM_K];
        bke[u] = bi * kk * ex2(c);
        ked[u] = kk * ex2(c63 - c);
        bv[u] = bi * __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + RAW_X + raw_off(i, f)));
      }
      st_tf32x4(sm, OP_BKET + kmaj(f, i0, 64), bke[0], bke[1], bke[2], bke[3]);
      st_tf32x4(sm, OP_KEDT + kmaj(f, i0, 64), ked[0], ked[1], ked[2], ked[3]);
      st_tf32x4(sm, OP_BVT + kmaj(f, i0, 64), bv[0], bv[1], bv[2], bv[3]);
    }
    if (tid < KD) sEl[tid] = ex2(c63);
  }
  Pairwise pw;
  if (wide) pairwise_compute<PREP>(cx, a.scale, pw);
  __syncthreads();  // raw inputs consumed; the raw region is reused below

  readout_ap<NTHR>(cx, tm + TM_APA, tm + TM_APB, wide, pw, nullptr);
  if (irec) {  // the P^T image of the record from the P image (16-byte pieces; piece x holds
               // P^T(r, k .. k + 3) = P[k .. k + 3][r], r = 8 (x / 128) + x % 8, k = 4 ((x % 128) / 8))
    for (int x = tid; x < C * C / 4; x += NTHR) {
      const int r = (x >> 7) * 8 + (x & 7), k = ((x & 127) >> 3) * 4;
      uint4 w;
      w.x = *reinterpret_cast<const uint32_t*>(sm + p_off(k, r));
      w.y = *reinterpret_cast<const uint32_t*>(sm + p_off(k + 1, r));
      w.z = *reinterpret_cast<const uint32_t*>(sm + p_off(k + 2, r));
      w.w = *reinterpret_cast<const uint32_t*>(sm + p_off(k + 3, r));
      *reinterpret_cast<uint4*>(irec + x * 4) = w;
    }
  }
  invert<NTHR>(cx);
  {  // T as the operand image (rows i, K = j); with a record also its T, T^T images and Ah
    const float* tr = reinterpret_cast<const float*>(sm + R_TROW);
    for (int x = tid; x < C * 16; x += NTHR) {  // 16-byte piece x of the image: x * 16 = kmaj(i, j4, 64)
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
      for (int x = tid; x < C * C; x += NTHR) irec[INTER_AH + x] = ah[(x >> 6) * 65 + (x & 63)];
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
  return wait_mma(bar, phase);
}

template <bool PREP>
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

  const int hv = blockIdx.x, sq = blockIdx.y;  // batch row, or sequence of a packed batch
  const SeqChunks sc(a, sq);
  const int b = sc.row;
  const int G = a.HV / a.H, h = hv / G, T = a.T, NT = (T + C - 1) / C;
  const size_t head = (size_t)sq * a.HV + hv;
  __nv_bfloat16* og = static_cast<__nv_bfloat16*>(a.o);
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

  for (int c = sc.c0; c < sc.c1; ++c) {
    const int2 sp = sc.span(a, c);
    const int t0 = sp.x, L = sp.y, ch = c - sc.c0;
    const int Ln = c + 1 < sc.c1 ? sc.span(a, c + 1).y : 0;
    float* irec = a.inter ? a.inter + chunk_gc(a, sq, hv, c) * INTER_REC : nullptr;
    if (!fwd_chunk_head<NTH, PREP>(cx, a, b, hv, h, t0, L, Ln, irec, bar, phase)) {
      failed = true;
      break;
    }

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
        if (a.states)  // the state entering this chunk
          store_slot32(a.states + state_slot(a, sq, hv, sc.c0 + ch) * (KD * VD), f0 / 32, Lr, s);
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
      commit(bar);
    }
    if (!wait_mma(bar, phase)) { failed = true; break; }

    // ---------------------------------------------------------------- O out
    if (a.o) {
      float v[32];
      tmem_ld32(tm + lo + TM_O + hcol * 32, v);
      if (a.og) {  // output gate; the raw region is free here (W and P are consumed)
        const __nv_bfloat16* gate = static_cast<const __nv_bfloat16*>(a.og);
        out_gate_rows(v, reinterpret_cast<float*>(sm + R_AH), cx.warp, cx.lane, a.og_eps);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int i = hcol * 32 + jj;
          if (i < L) v[jj] *= prep_sigmoid_fast(__bfloat162float(gate[(((size_t)b * T + t0 + i) * a.HV + hv) * VD + Lr]));
        }
      }
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
  return dtype == 1 && a.K == 128 && a.V == 128 && al16(a.q) && al16(a.k) && al16(a.v) && al16(a.g) &&
         al16(a.o) && al16(a.prep.z) && al16(a.og);
}

template <bool PREP>
static int launch_fwd_tc_t(const FwdArgs& a, cudaStream_t stream) {
  if (a.img) return launch_fwd_chunked(a, stream);  // chunk-parallel kernel + state pass
  cudaError_t e = cudaFuncSetAttribute(kda_fwd_tc_kernel<PREP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tcc::SMEM_BYTES);
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: cudaFuncSetAttribute", e);
  kda_fwd_tc_kernel<PREP><<<dim3(a.HV, a.B), tcc::NTH, tcc::SMEM_BYTES, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: tensor-core launch", e);
  return 0;
}

int launch_fwd_tc(const FwdArgs& a, cudaStream_t stream) {
  return a.prep.z ? launch_fwd_tc_t<true>(a, stream) : launch_fwd_tc_t<false>(a, stream);
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
