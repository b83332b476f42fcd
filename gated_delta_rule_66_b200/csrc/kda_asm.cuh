// Assembly of dq, dk, dg and dbeta for one quarter of the key channels of a
// 64-step chunk from the per-chunk gradient record, with tf32 warp MMAs for
// the interaction terms (any decay span: pair by pair, with 3xTF32 products,
// where the split exponents would leave fp32 range).
#pragma once

#include <cuda_fp16.h>

#include "kda_chunk.cuh"
#include "kda_internal.h"

namespace kda {

// Assembles dq, dk, dg and dbeta of one 64-step chunk from the record that
// kda_bwd_grads_tc_kernel wrote (Ah, [dP; dA], [dQE; dKE'], dKEd, dbeta_R,
// dEl): dbeta = dbeta_R + sum_j dA_ij Ah_ij; dq~ = dQE o e^c; dk = dKE o e^c +
// dKEd o e^{c_last-c}; dc = (dQE o q~ + dKE o k) o e^c - dKEd o k o e^{c_last-c};
// then the interaction terms (factored_terms) and dg = reverse cumsum of dc.
// Everything here is independent across key channels, so one CTA handles one
// (b, hv, chunk, quarter of the 128 key channels); two CTAs fit on an SM.
// Row strides (words): LDK = 40 (8 mod 32) puts the warp-MMA fragment loads of
// K, Q and c (lanes: row t, channel g) in 32 distinct banks; LDC = 68 (4 mod
// 32) does the same for the row-term fragments of dP and dA (lanes: row g,
// column t).  Accesses with the lanes along a row are conflict-free anyway.
struct AsmSmem {
  static constexpr int C = 64, KQ = 32, LDK = 40, LDC = 68;
  static constexpr int oK = 0, oQ = oK + C * LDK, oC = oQ + C * LDK, oDq = oC + C * LDK, oDk = oDq + C * LDK,
                       oDc = oDk + C * LDK, oE1 = oDc + C * LDK, oE2o = oE1 + C * LDK, oE2d = oE2o + BS * LDK,
                       odA = oE2d + BS * LDK, odP = odA + C * LDC, oBeta = odP + C * LDC, oSeg = oBeta + C,
                       oLast = oSeg + 8 * KQ, oFlag = oLast + KQ, total = oFlag + 4;
  static constexpr size_t bytes = (size_t)total * sizeof(float);
};

// Four consecutive q or k values (16-byte aligned fp32 or 8-byte aligned bf16)
__device__ __forceinline__ void load4(const float* p, float (&o)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&o)[4]) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&r.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&r.y);
  o[0] = __low2float(lo); o[1] = __high2float(lo); o[2] = __low2float(hi); o[3] = __high2float(hi);
}

__device__ __forceinline__ void store4(float* p, float x, float y, float z, float w) {
  *reinterpret_cast<float4*>(p) = make_float4(x, y, z, w);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, float x, float y, float z, float w) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(x, y), hi = __floats2bfloat162_rn(z, w);
  uint2 r;
  r.x = *reinterpret_cast<const uint32_t*>(&lo);
  r.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = r;
}

// Inclusive (forward) or reverse cumulative sum over the C = 64 rows of each
// of the KQ = 32 columns of a [64][LDK] array, by 8 segments of 8 rows
// (256 threads; seg is 8 x KQ scratch; `base` is added to every element of a
// reverse sum).  Ends with a barrier.

// four consecutive fp16 record elements (8-byte aligned) as floats, times their group's scale
__device__ __forceinline__ float4 ld4h(const __half* p, float sc) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  return make_float4(lo.x * sc, lo.y * sc, hi.x * sc, hi.y * sc);
}
template <bool REVERSE>
__device__ __forceinline__ void cumsum64(float* a, float* seg, const float* base) {
  constexpr int LDK = AsmSmem::LDK, KQ = AsmSmem::KQ;
  const int f = threadIdx.x % KQ, sg = threadIdx.x / KQ;  // 8 segments
  float v[8], run = 0.f;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int i = REVERSE ? (63 - (sg * 8 + r)) : (sg * 8 + r);
    run += a[i * LDK + f];
    v[r] = run;
  }
  seg[sg * KQ + f] = run;
  __syncthreads();
  float carry = REVERSE && base ? base[f] : 0.f;
  for (int s2 = 0; s2 < sg; ++s2) carry += seg[s2 * KQ + f];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int i = REVERSE ? (63 - (sg * 8 + r)) : (sg * 8 + r);
    a[i * LDK + f] = v[r] + carry;
  }
  __syncthreads();
}

// One (chunk, quarter) with the CTA's 256 threads, shared memory at `smem`
// (AsmSmem::bytes): chunk ch of batch row sq (packed sequences: chunk ch of
// the table, sq = 0).  Ends with a barrier.
// L2 prefetch of everything the four quarters of chunk ch of (sq, hv) read:
// its gradient record, q and k rows of its key head, g rows, and Ah.
template <typename TIn>
__device__ __forceinline__ void prefetch_assembly(const BwdArgs& a, int ch, int hv, int sq) {
  constexpr int KD = 128;
  const int tid = threadIdx.x, G = a.HV / a.H, h = hv / G, b = row_of(a, sq);
  const int2 sp = chunk_span(a, ch);
  const size_t gc = chunk_gc(a, sq, hv, ch);
  if (tid < 17) {  // GREC floats = 16 pieces of 4096 bytes + the rest
    static_assert(GREC * 4 > 16 * 4096 && GREC * 4 - 16 * 4096 <= 4096 && GREC * 4 % 16 == 0, "record pieces");
    const uint32_t bytes = tid < 16 ? 4096u : (uint32_t)(GREC * 4 - 16 * 4096);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.gws + gc * GREC + tid * 1024), "r"(bytes)
                 : "memory");
    return;
  }
  if (tid >= 20 && tid < 24) {  // (Ah: 4 pieces)
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.inter + gc * INTER_REC + INTER_AH +
                                                                    (tid - 20) * 1024),
                 "r"(4096u)
                 : "memory");
    return;
  }
  const int i = tid & 63, which = tid >> 6;  // which 1: q, 2: k, 3: g
  if (which == 0 || i >= sp.y) return;
  const size_t t = (size_t)b * a.T + sp.x + i;
  const void* p = which == 1   ? static_cast<const void*>(static_cast<const TIn*>(a.q) + (t * a.H + h) * KD)
                  : which == 2 ? static_cast<const void*>(static_cast<const TIn*>(a.k) + (t * a.H + h) * KD)
                               : static_cast<const void*>(a.g + (t * a.HV + hv) * KD);
  const uint32_t bytes = which == 3 ? KD * 4 : KD * (uint32_t)sizeof(TIn);
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

template <typename TIn>
__device__ __forceinline__ void assemble_quarter(const BwdArgs& a, float* smem, int ch, int fq4, int hv, int sq) {
  using S = AsmSmem;
  constexpr int C = S::C, KQ = S::KQ, LDK = S::LDK, LDC = S::LDC, KD = 128;
  float *sK = smem + S::oK, *sQ = smem + S::oQ, *sC = smem + S::oC, *sDq = smem + S::oDq,
        *sDk = smem + S::oDk, *sDc = smem + S::oDc, *sE1 = smem + S::oE1, *sE2o = smem + S::oE2o,
        *sE2d = smem + S::oE2d, *sdA = smem + S::odA, *sdP = smem + S::odP, *sBeta = smem + S::oBeta,
        *sSeg = smem + S::oSeg, *sLast = smem + S::oLast;
  int* sFlag = reinterpret_cast<int*>(smem + S::oFlag);
  const int G = a.HV / a.H, h = hv / G, T = a.T, b = row_of(a, sq);
  const int2 sp = chunk_span(a, ch);
  const int t0 = sp.x, L = sp.y, f0 = fq4 * KQ;
  const size_t gc = chunk_gc(a, sq, hv, ch);
  const float* rec = a.gws + gc * GREC;
  const __half* rech = reinterpret_cast<const __half*>(rec);
  const TIn* q = static_cast<const TIn*>(a.q);
  const TIn* k = static_cast<const TIn*>(a.k);
  const int tid = threadIdx.x;

  // [dQE; dKE'] and dKEd of this quarter, consumed further down: lane = channel f,
  // warp w = rows 8w .. 8w + 7 (each row a 128-byte run of the row-major record)
  const int ef = tid & 31, ei = (tid >> 5) * 8;
  // Ah of row 16 fq4 + tid / 16, columns 4 (tid % 16) .. + 3 (for dbeta; rows past L are zero)
  const float4 ah4 = (16 * fq4 + (tid >> 4) < L)
                         ? *reinterpret_cast<const float4*>(a.inter + gc * INTER_REC + INTER_AH +
                                                            (16 * fq4 + (tid >> 4)) * 64 + (tid & 15) * 4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
  float qe[8], ke[8], kd[8];
  // the fp16 record's block scales: [dQE; dKE'] and dKEd of this quarter, [dP; dA] of both column groups
  const float sq_e = rec[G_SC + 4 + fq4], sk_e = rec[G_SC + 8 + fq4], sd_e = rec[G_SC + 12 + fq4];
  const float sp_0 = rec[G_SC + 0], sp_1 = rec[G_SC + 1], sa_0 = rec[G_SC + 2], sa_1 = rec[G_SC + 3];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    qe[u] = __half2float(rech[GH_QK + rec_off(ei + u, f0 + ef, 128)]) * sq_e;
    ke[u] = __half2float(rech[GH_QK + rec_off(64 + ei + u, f0 + ef, 128)]) * sk_e;
    kd[u] = __half2float(rech[GH_KED + rec_off(ei + u, f0 + ef, 128)]) * sd_e;
  }
  {  // inputs of this channel quarter (4 channels per item) and the C x C adjoints; loads first
    float4 gv[2], dp[4], da[4];
    float qv[2][4], kv[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int idx = tid + m * NTHREADS, i = idx >> 3, f4 = (idx & 7) * 4;
      gv[m] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) qv[m][u] = kv[m][u] = 0.f;
      if (i < L) {
        const size_t rq = (((size_t)b * T + t0 + i) * a.H + h) * KD + f0 + f4;
        gv[m] = *reinterpret_cast<const float4*>(a.g + (((size_t)b * T + t0 + i) * a.HV + hv) * KD + f0 + f4);
        load4(q + rq, qv[m]);
        load4(k + rq, kv[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {  // row i of [dP; dA], four columns j per item
      const int idx = tid + m * NTHREADS, i = idx >> 4, j4 = (idx & 15) * 4;
      // only the lower triangle is used (dP: j <= i, dA: j < i): wholly upper pieces are not read
      const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
      dp[m] = (j4 <= i) ? ld4h(rech + GH_PA + rec_off(i, j4, 64), j4 < 32 ? sp_0 : sp_1) : z4;
      da[m] = (j4 <= i) ? ld4h(rech + GH_PA + rec_off(64 + i, j4, 64), j4 < 32 ? sa_0 : sa_1) : z4;
    }
    float bt[4];  // beta of the rows of the [dA] items
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int i = (tid >> 4) + 16 * m;
      bt[m] = (i < L) ? a.beta[((size_t)b * T + t0 + i) * a.HV + hv] : 0.f;
    }
    if (tid < C) sBeta[tid] = (tid < L) ? a.beta[((size_t)b * T + t0 + tid) * a.HV + hv] : 0.f;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int idx = tid + m * NTHREADS, i = idx >> 3, f4 = (idx & 7) * 4;
      const float gg[4] = {gv[m].x, gv[m].y, gv[m].z, gv[m].w};
      // (LDK = 40: rows 16-byte aligned)
      *reinterpret_cast<float4*>(sQ + i * LDK + f4) =
          make_float4(qv[m][0] * a.scale, qv[m][1] * a.scale, qv[m][2] * a.scale, qv[m][3] * a.scale);
      *reinterpret_cast<float4*>(sK + i * LDK + f4) = make_float4(kv[m][0], kv[m][1], kv[m][2], kv[m][3]);
      *reinterpret_cast<float4*>(sC + i * LDK + f4) = make_float4(gg[0], gg[1], gg[2], gg[3]);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int idx = tid + m * NTHREADS, i = idx >> 4, j4 = (idx & 15) * 4;
      const float vdp[4] = {dp[m].x, dp[m].y, dp[m].z, dp[m].w}, vda[4] = {da[m].x, da[m].y, da[m].z, da[m].w};
      float4 wp, wa;
      wp.x = (j4 <= i) ? vdp[0] : 0.f;
      wp.y = (j4 + 1 <= i) ? vdp[1] : 0.f;
      wp.z = (j4 + 2 <= i) ? vdp[2] : 0.f;
      wp.w = (j4 + 3 <= i) ? vdp[3] : 0.f;
      wa.x = (j4 < i) ? vda[0] : 0.f;
      wa.y = (j4 + 1 < i) ? vda[1] : 0.f;
      wa.z = (j4 + 2 < i) ? vda[2] : 0.f;
      wa.w = (j4 + 3 < i) ? vda[3] : 0.f;
      if (m == fq4) {  // dbeta = dbeta_R + sum_{j<i} dA_ij Ah_ij for this quarter's 16 rows (16 threads per row)
        float sb = fmaf(wa.x, ah4.x, fmaf(wa.y, ah4.y, fmaf(wa.z, ah4.z, wa.w * ah4.w)));
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) sb += __shfl_xor_sync(0xffffffffu, sb, off);
        if ((tid & 15) == 0 && i < L) a.dbeta[((size_t)b * T + t0 + i) * a.HV + hv] = rec[G_DBR + i] + sb;
      }
      wa.x *= bt[m];  // the interaction terms take diag(beta) dA
      wa.y *= bt[m];
      wa.z *= bt[m];
      wa.w *= bt[m];
      *reinterpret_cast<float4*>(sdP + i * LDC + j4) = wp;  // LDC = 68: rows 16-byte aligned
      *reinterpret_cast<float4*>(sdA + i * LDC + j4) = wa;
    }
  }
  __syncthreads();
  cumsum64<false>(sC, sSeg, nullptr);
  {  // element-wise terms; the chunk-end sum of dKEd o k o e^{c_last-c} over this warp's
     // 8 rows goes to sSeg (warp w = rows 8w .. 8w + 7, lane = channel)
    float send = 0.f;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int f = ef, i4 = ei + 4 * m;
      const float vq[4] = {qe[4 * m], qe[4 * m + 1], qe[4 * m + 2], qe[4 * m + 3]},
                  vk[4] = {ke[4 * m], ke[4 * m + 1], ke[4 * m + 2], ke[4 * m + 3]},
                  vd[4] = {kd[4 * m], kd[4 * m + 1], kd[4 * m + 2], kd[4 * m + 3]};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i4 + u, o = i * LDK + f;
        const float c = sC[o], e = __expf(c), ed = __expf(sC[(C - 1) * LDK + f] - c);
        const float dqe = vq[u], dke = sBeta[i] * vk[u], dked = vd[u];
        const float kk = sK[o], qq = sQ[o];
        sDq[o] = dqe * e;
        sDk[o] = dke * e + dked * ed;
        sDc[o] = (dqe * qq + dke * kk) * e - dked * kk * ed;
        send += dked * kk * ed;
      }
    }
    sSeg[(ei >> 3) * KQ + ef] = send;
  }
  __syncthreads();
  {  // chunk-end terms: dEl o e^{c_last} + sum_i dKEd o k o e^{c_last - c}
    if (tid < KQ) {
      float t = rec[G_DEL + f0 + tid] * __expf(sC[(C - 1) * LDK + tid]);
      for (int s2 = 0; s2 < 8; ++s2) t += sSeg[s2 * KQ + tid];
      sLast[tid] = t;
    }
    __syncthreads();
  }
  {  // split exponents hold when every 16-row block's decay span is at most 80
    bool wide = false;
    if (tid < 4 * KQ) {
      const int J = tid / KQ, f = tid % KQ;
      wide = sC[(16 * J) * LDK + f] - sC[(16 * J + 15) * LDK + f] > DIAG_SPAN_MAX;
    }
    if (__syncthreads_or(wide))
      factored_terms<KQ, C, false, false, LDK, LDC>(sK, sQ, sC, sdA, sdP, sE1, sE2o, sE2d, sFlag, sDq, sDk, sDc);
    else
      factored_terms_tf32<KQ, LDK, LDC>(sK, sQ, sC, sdA, sdP, sDq, sDk, sDc);
  }
  cumsum64<true>(sDc, sSeg, sLast);
  TIn* dq = static_cast<TIn*>(a.dq);
  TIn* dk = static_cast<TIn*>(a.dk);
  const uintptr_t al = (uintptr_t)a.dg | (G == 1 ? ((uintptr_t)dq | (uintptr_t)dk)
                                                 : ((uintptr_t)a.dq_part | (uintptr_t)a.dk_part));
  if ((al & 15u) == 0) {  // four channels per item, 16-byte (fp32) and 8-byte (bf16) stores
    for (int idx = tid; idx < L * (KQ / 4); idx += NTHREADS) {
      const int i = idx / (KQ / 4), f = (idx % (KQ / 4)) * 4, o = i * LDK + f;
      const size_t row_v = ((size_t)b * T + t0 + i) * a.HV + hv;
      const float4 c4 = *reinterpret_cast<const float4*>(sDc + o), q4 = *reinterpret_cast<const float4*>(sDq + o),
                   k4 = *reinterpret_cast<const float4*>(sDk + o);
      *reinterpret_cast<float4*>(a.dg + row_v * KD + f0 + f) = c4;
      const float sc = a.scale;
      if (G == 1) {
        const size_t row_h = ((size_t)b * T + t0 + i) * a.H + h;
        store4(dq + row_h * KD + f0 + f, sc * q4.x, sc * q4.y, sc * q4.z, sc * q4.w);
        store4(dk + row_h * KD + f0 + f, k4.x, k4.y, k4.z, k4.w);
      } else {
        *reinterpret_cast<float4*>(a.dq_part + row_v * KD + f0 + f) = make_float4(sc * q4.x, sc * q4.y, sc * q4.z, sc * q4.w);
        *reinterpret_cast<float4*>(a.dk_part + row_v * KD + f0 + f) = k4;
      }
    }
    __syncthreads();
    return;
  }
  for (int idx = tid; idx < L * KQ; idx += NTHREADS) {
    const int i = idx / KQ, f = idx % KQ, o = i * LDK + f;
    const size_t row_v = ((size_t)b * T + t0 + i) * a.HV + hv;
    a.dg[row_v * KD + f0 + f] = sDc[o];
    if (G == 1) {
      const size_t row_h = ((size_t)b * T + t0 + i) * a.H + h;
      dq[row_h * KD + f0 + f] = from_f<TIn>(a.scale * sDq[o]);
      dk[row_h * KD + f0 + f] = from_f<TIn>(sDk[o]);
    } else {
      a.dq_part[row_v * KD + f0 + f] = a.scale * sDq[o];
      a.dk_part[row_v * KD + f0 + f] = sDk[o];
    }
  }
  __syncthreads();
}

}  // namespace kda
