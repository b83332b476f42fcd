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

// four fp32 values times `up`, rounded to fp16, into 8 bytes of shared memory
__device__ __forceinline__ void st4h(__half* p, const float* v, float up) {
  const __half2 lo = __floats2half2_rn(v[0] * up, v[1] * up), hi = __floats2half2_rn(v[2] * up, v[3] * up);
  uint2 u;
  u.x = *reinterpret_cast<const unsigned*>(&lo);
  u.y = *reinterpret_cast<const unsigned*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}
// The largest magnitude of v[0..31] over the warp's lanes (lanes < n), as float bits
__device__ __forceinline__ unsigned warp_absmax32(const float (&v)[32], int lane, int n = 32) {
  float m = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
  return __reduce_max_sync(0xffffffffu, lane < n ? __float_as_uint(m) : 0u);  // (non-negative floats order as ints)
}
// The power-of-two factor that puts magnitude m (float bits) in [2^14, 2^15)
// (the fp16 record's block scale is its inverse, written to *inv)
__device__ __forceinline__ float block_up(unsigned mbits, float* inv) {
  const int ex = (int)((mbits >> 23) & 0xff) - 126;
  const int e = min(126, max(-126, 15 - ex));
  if (inv) *inv = __int_as_float((127 - e) << 23);
  return __int_as_float((127 + e) << 23);
}
// Warp-specialised, 544 threads (17 warps), one CTA per (sequence, value head):
//   issuer warp 0 (lane 0): the three products of every chunk and the P^T,
//     T^T image copies (a tcgen05.mma issue holds its thread for about the
//     product's duration, so this warp does nothing else);
//   chain warps 1-8 (TMEM lanes 32 (w % 4) .., lane = value column n; column
//     half (w - 1) / 4): the operands of the state product, (Q~ o e^c)^T and
//     -(diag(beta) K o e^c)^T as [f][i], and e^{c_last}; the state gradient's
//     decay in TMEM, storing the gradient leaving every chunk on the way;
//   builder warps 9-16: the decay and the operands K o e^{c_last-c} as
//     [i][f] and dO^T (into one of two TMEM buffers), the next chunk's while
//     this chunk's products run;
//   loader warp 17 (lane 0): the next chunk's q, k, dO and g tiles by TMA
//     once the builders are done with the current ones, and the chunk after
//     next into L2 (a TMA issue can hold its thread for a while).
// Per chunk (in reverse): dU^T (waits for the previous chunk's state
// product), dR^T = dU^T T, then dM^T <- dM^T diag(e^{c_last}) + dO^T (Q~ o
// e^c) - dR^T (diag(beta) K o e^c) once the chain has decayed dM^T.  Every wait
// is bounded (g_kda_bwd_wait_polls probes); one that gives up sets the
// shared abort word, which ends the other roles' waits too.
namespace tcd {
using namespace tcc;
constexpr int D_THREADS = 576, D_CH = 256, D_BU0 = 288, D_BU = 256, D_LD0 = 544;
constexpr uint32_t D_KED = OP, D_QET = OP + 32768, D_NKET = OP + 65536, D_PT = OP + 98304, D_TT = OP + 114688,
                   D_BAR = OP + 131072, D_CNT = D_BAR + 128;
static_assert(D_CNT + 64 <= SMALL, "state-gradient shared-memory map");
// TMEM columns: dM^T, dU^T, dR^T, two dO^T buffers (chunks alternate), and the
// chain's copy of the gradient leaving the chunk (stored after the decay is released)
constexpr uint32_t DT_S = 0, DT_DU = 128, DT_DR = 192, DT_DOT = 256, DT_COPY = 384;
enum { DB_RAW, DB_P, DB_T, DB_DU, DB_DR, DB_S, DNB_ASYNC, DB_KED = DNB_ASYNC, DB_C, DB_QN, DB_RS, DNB_ALL };
// named barriers: 1 the chain warps, 2 the builder warps, 3 the issuer warp with the chain warps
constexpr int DBAR_CH = 1, DBAR_BU = 2, DBAR_S0 = 3;
}  // namespace tcd

__device__ unsigned int g_kda_bwd_wait_polls = 1u << 24;

__global__ void __launch_bounds__(tcd::D_THREADS, 1) kda_bwd_dstate_tc_kernel(const __grid_constant__ RawMaps maps,
                                                                              BwdArgs a) {
  using namespace tcd;
  using namespace tc;
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  if (sb & 1023u) {  // the 128-byte swizzle of the TMA tiles needs a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(&g_kda_bwd_device_error, 2u);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int head_ = a.head0 + blockIdx.x;
  const int hv = head_ % a.HV, sq = head_ / a.HV;  // batch row, or sequence of a packed batch
  const int b = row_of(a, sq), c0 = chunk_begin(a, sq), c1 = chunk_end(a, sq), nch = c1 - c0;
  const int G = a.HV / a.H, h = hv / G, T = a.T;
  const size_t head = (size_t)sq * a.HV + hv;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + D_BAR);
  int* cnt = reinterpret_cast<int*>(sm + D_CNT);  // issued phases per async barrier; [15]: abort
  volatile int* abort = cnt + 15;
  uint32_t* sTm = reinterpret_cast<uint32_t*>(sm + S_TMEM);
  float* sEl = reinterpret_cast<float*>(sm + S_EL);
  float* sBeta = reinterpret_cast<float*>(sm + S_BETA);
  unsigned char* tC = sm + RAW_C;  // g, then the cumulative decay (fp32 TMA tile)
  const uint32_t polls = g_kda_bwd_wait_polls;

  if (warp == 0) tmem_alloc(sTm, 512);
  if (tid == 0) {
    for (int i = 0; i < DNB_ALL; ++i)
      mbar_init(bars + i, i < DNB_ASYNC ? 1 : (i == DB_RS || i == DB_QN ? D_CH : D_BU));
    for (int i = 0; i < 16; ++i) cnt[i] = 0;
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = *sTm;
  const auto irec = [&](int ch) { return a.inter + chunk_gc(a, sq, hv, ch) * INTER_REC; };

  if (warp == 0) {
    // ======================================================================== issuer warp
    named_sync(DBAR_S0, 32 + D_CH);  // the final state's gradient is in TMEM
    if (lane == 0 && nch > 0) {
      const auto issue_img = [&](int which, uint32_t dst, const float* src) {
        mbar_expect_tx(bars + which, 16384);
        bulk_g2s(dst, src, 16384, bars + which);
        ++cnt[which];
      };
      const auto commit_to = [&](int which) {
        commit(bars + which);
        ++cnt[which];
      };
      issue_img(DB_P, sb + D_PT, irec(c1 - 1));             // P^T: (row i, K j) = P[j][i]
      issue_img(DB_T, sb + D_TT, irec(c1 - 1) + INTER_TT);  // T^T: (row i, K j) = T[j][i]
      for (int k = 0; k < nch; ++k) {
        const int ch = c1 - 1 - k;
        const uint32_t par = k & 1, dot = DT_DOT + (k & 1) * 64;
        // dU^T = dO^T P + dM^T (K o e^{c_last-c})^T, dM^T the gradient leaving this chunk
        if (!wait_one(bars + DB_KED, par, polls, abort)) break;
        if (!wait_one(bars + DB_P, par, polls, abort)) break;
        if (k > 0 && !wait_one(bars + DB_S, par ^ 1, polls, abort)) break;
        fence_after();
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(tm + DT_DU, tm + dot + ks * 8, desc(sb + D_PT + ks * 256, 2048), idesc_tf32(128, 64), ks > 0);
        for (int ks = 0; ks < 16; ++ks)
          mma_ts(tm + DT_DU, tm + DT_S + ks * 8, desc(sb + D_KED + ks * 256, 4096), idesc_tf32(128, 64), 1);
        commit_to(DB_DU);
        if (!wait_one(bars + DB_DU, par, polls, abort)) break;
        if (k + 1 < nch) issue_img(DB_P, sb + D_PT, irec(ch - 1));  // this chunk's P^T is consumed
        // dR^T = dU^T T
        if (!wait_one(bars + DB_T, par, polls, abort)) break;
        fence_after();
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(tm + DT_DR, tm + DT_DU + ks * 8, desc(sb + D_TT + ks * 256, 2048), idesc_tf32(128, 64), ks > 0);
        commit_to(DB_DR);
        if (!wait_one(bars + DB_DR, par, polls, abort)) break;
        if (k + 1 < nch) issue_img(DB_T, sb + D_TT, irec(ch - 1) + INTER_TT);
        // dM^T += dO^T (Q~ o e^c) - dR^T (diag(beta) K o e^c) once the chain has decayed dM^T
        if (!wait_one(bars + DB_QN, par, polls, abort)) break;
        if (!wait_one(bars + DB_RS, par, polls, abort)) break;
        fence_after();
        for (int ks = 0; ks < 8; ++ks) {
          mma_ts(tm + DT_S, tm + dot + ks * 8, desc(sb + D_QET + ks * 256, 2048), idesc_tf32(128, 128), 1);
          mma_ts(tm + DT_S, tm + DT_DR + ks * 8, desc(sb + D_NKET + ks * 256, 2048), idesc_tf32(128, 128), 1);
        }
        commit_to(DB_S);
      }
    }
    __syncwarp();
  } else if (warp <= 8) {
    // ======================================================================== chain warps
    const int n = (warp & 3) * 32 + lane, hc = (warp - 1) >> 2;  // TMEM lane (value column), column half
    const uint32_t lo = (uint32_t)((warp & 3) * 32) << 16;
    for (int cb = 0; cb < 2; ++cb) {  // gradient of the final state, transposed
      const int f0 = hc * 64 + cb * 32;
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(a.dS_T ? a.dS_T[(head * KD + f0 + j) * VD + n] : 0.f);
      tmem_st32(tm + lo + DT_S + f0, r);
    }
    tmem_wait_st();
    fence_before();
    named_sync(DBAR_S0, 32 + D_CH);
    bool ok = true;
    const int ct = tid - 32;  // 0 .. 255
    for (int k = 0; k < nch; ++k) {
      const int ch = c1 - 1 - k;
      const uint32_t par = k & 1;
      // (Q~ o e^c)^T, -(diag(beta) K o e^c)^T as [f][i] and e^{c_last}: once this chunk's decay is
      // formed and the previous chunk's state product (which read them) is done
      if (!(ok = role_wait(bars + DB_C, par, polls, abort, DBAR_CH, D_CH))) break;
      if (k > 0 && !(ok = role_wait(bars + DB_S, par ^ 1, polls, abort, DBAR_CH, D_CH))) break;
      {
        const int f = ct & 127;
        for (int m = 0; m < 8; ++m) {
          const int i0 = ((ct >> 7) + 2 * m) * 4;
          float qe[4], nke[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            const float e = ex2(ldf(tC, i, f));
            qe[u] = a.scale * ldb(sm + RAW_Q, i, f) * e;
            nke[u] = -sBeta[i] * ldb(sm + RAW_K, i, f) * e;
          }
          st_tf32x4(sm, D_QET + kmaj(f, i0, 64), qe[0], qe[1], qe[2], qe[3]);
          st_tf32x4(sm, D_NKET + kmaj(f, i0, 64), nke[0], nke[1], nke[2], nke[3]);
        }
        if (ct < KD) sEl[ct] = ex2(ldf(tC, 63, ct));
      }
      fence_async_smem();
      mbar_arrive(bars + DB_QN);  // (also: the chain is done with this chunk's raw rows)
      // the gradient leaving this chunk: stored, then decayed by e^{c_last} once dU^T has read it
      // (the wait is also the chain's barrier for e^{c_last})
      if (!(ok = role_wait(bars + DB_DU, par, polls, abort, DBAR_CH, D_CH))) break;
      fence_after();
#pragma unroll 1
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hc * 64 + cb * 32;
        float sv[32];
        uint32_t r[32];
        tmem_ld32(tm + lo + DT_S + f0, sv);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(sv[j]);
        tmem_st32(tm + lo + DT_COPY + f0, r);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(sv[j] * sEl[f0 + j]);
        tmem_st32(tm + lo + DT_S + f0, r);
      }
      tmem_wait_st();
      fence_before();
      mbar_arrive(bars + DB_RS);
      // the gradient leaving this chunk to the workspace, while the state product runs
      float* slot = a.dstates + dstate_slot(a, sq, hv, ch) * (KD * VD);
#pragma unroll 1
      for (int cb = 0; cb < 2; ++cb) {
        float sv[32];
        tmem_ld32(tm + lo + DT_COPY + hc * 64 + cb * 32, sv);
        store_slot32(slot, hc * 2 + cb, n, sv);
      }
    }
    if (ok && a.dS0 && (nch == 0 || role_wait(bars + DB_S, (nch - 1) & 1, polls, abort, DBAR_CH, D_CH))) {
      fence_after();
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hc * 64 + cb * 32;
        float sv[32];
        tmem_ld32(tm + lo + DT_S + f0, sv);
#pragma unroll
        for (int j = 0; j < 32; ++j) a.dS0[(head * KD + f0 + j) * VD + n] = sv[j];
      }
    }
  } else if (warp < D_LD0 / 32) {
    // ======================================================================== builder warps
    const int bt = tid - D_BU0;  // 0 .. 255
    Ctx cx;  // the builders' view: thread index bt
    cx.sm = sm;
    cx.sb = sb;
    cx.tid = bt;
    float* sCarry = reinterpret_cast<float*>(sm + S_CARRY);
    const int n = (warp & 3) * 32 + lane, hb = (warp - 9) >> 2;  // dO^T: TMEM lane n, columns 32 hb ..
    const uint32_t lo = (uint32_t)((warp & 3) * 32) << 16;
    // beta (HV floats apart per step, which no tensor map addresses) goes through the
    // registers of 64 threads
    const auto beta_of = [&](int ch) {
      const int2 sp = chunk_span(a, ch);
      return bt < sp.y ? a.beta[((size_t)b * T + sp.x + bt) * a.HV + hv] : 0.f;
    };
    float bval = 0.f;
    if (nch > 0 && bt < C) bval = beta_of(c1 - 1);
    for (int k = 0; k < nch; ++k) {
      const int ch = c1 - 1 - k, L = chunk_span(a, ch).y;
      const uint32_t par = k & 1, dot = DT_DOT + (k & 1) * 64;
      if (!role_wait(bars + DB_RAW, par, polls, abort, DBAR_BU, D_BU)) break;
      if (bt < C) sBeta[bt] = bval;
      if (L < C) {  // rows past the sequence (a packed batch's next sequence) count as zero
        for (int x = bt; x < (C - L) * 16; x += D_BU) {  // 16-byte pieces of the bf16 rows
          const int i = L + (x >> 4), p = x & 15;
          const uint32_t o = (uint32_t)((p >> 3) * 8192 + i * 128 + (((p & 7) ^ (i & 7)) << 4));
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(sm + RAW_Q + o) = z;
          *reinterpret_cast<uint4*>(sm + RAW_K + o) = z;
          *reinterpret_cast<uint4*>(sm + RAW_X + o) = z;
        }
        for (int x = bt; x < (C - L) * 32; x += D_BU) {  // and of the fp32 g rows
          const int i = L + (x >> 5), p = x & 31;
          *reinterpret_cast<uint4*>(tC + (p >> 3) * 8192 + i * 128 + (((p & 7) ^ (i & 7)) << 4)) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      named_sync(DBAR_BU, D_BU);
      {  // cumulative decay (times log2 e) in place: channel bt % 128, rows 32 (bt / 128) ..
        const int f = bt & 127, hh = bt >> 7;
        float v[32], run = 0.f;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          run += ldf(tC, hh * 32 + r, f);
          v[r] = run;
        }
        if (hh == 0) sCarry[f] = run;
        named_sync(DBAR_BU, D_BU);
        const float carry = hh ? sCarry[f] : 0.f;
#pragma unroll
        for (int r = 0; r < 32; ++r) *reinterpret_cast<float*>(tC + ft_off(hh * 32 + r, f)) = (v[r] + carry) * LOG2E;
        named_sync(DBAR_BU, D_BU);
      }
      mbar_arrive(bars + DB_C);  // the decay (and beta) of this chunk for the chain's operands
      // K o e^{c_last-c} as [i][f] and dO^T: free once the previous chunk's dU^T is done
      if (k > 0 && !role_wait(bars + DB_DU, par ^ 1, polls, abort, DBAR_BU, D_BU)) break;
      {
        const int fq = item_f<D_BU>(cx);
        const float4 c63v = *reinterpret_cast<const float4*>(tC + ft_off(63, fq));
        const float c63[4] = {c63v.x, c63v.y, c63v.z, c63v.w};
        for (int m = 0; m < 8; ++m) {
          const int i = item_row<D_BU>(cx, m);
          const float4 c4 = *reinterpret_cast<const float4*>(tC + ft_off(i, fq));
          float kf[4];
          bf16x4(sm + RAW_K + bt_off(i, fq), kf);
          st_tf32x4(sm, D_KED + kmaj(i, fq, 128), kf[0] * ex2(c63[0] - c4.x), kf[1] * ex2(c63[1] - c4.y),
                    kf[2] * ex2(c63[2] - c4.z), kf[3] * ex2(c63[3] - c4.w));
        }
        uint32_t r[32];  // dO^T: lane n, columns j = 32 hb ..
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) r[jj] = tf32_rna(ldb(sm + RAW_X, hb * 32 + jj, n));
        tmem_st32(tm + lo + dot + hb * 32, r);
        tmem_wait_st();
      }
      fence_async_smem();
      fence_before();
      mbar_arrive(bars + DB_KED);  // (also: the builders are done with this chunk's raw rows)
      if (k + 1 < nch && bt < C) bval = beta_of(ch - 1);
    }
  } else {
    // ======================================================================== loader warp
    if (lane == 0 && nch > 0) {
      const auto raw = [&](int ch) {
        const int t0 = chunk_span(a, ch).x;
        mbar_expect_tx(bars + DB_RAW, 3 * TILE_BF16 + TILE_F32);
        for (int j = 0; j < 2; ++j) {
          tma_load_4d(sb + RAW_Q + j * 8192, maps.q, 64 * j, h, t0, b, bars + DB_RAW);
          tma_load_4d(sb + RAW_K + j * 8192, maps.k, 64 * j, h, t0, b, bars + DB_RAW);
          tma_load_4d(sb + RAW_X + j * 8192, maps.x, 64 * j, hv, t0, b, bars + DB_RAW);
        }
        for (int j = 0; j < 4; ++j) tma_load_4d(sb + RAW_C + j * 8192, maps.g, 32 * j, hv, t0, b, bars + DB_RAW);
        ++cnt[DB_RAW];
      };
      const auto prefetch = [&](int ch) {
        const int t2 = chunk_span(a, ch).x;
        for (int j = 0; j < 2; ++j) {
          tma_prefetch_4d(maps.q, 64 * j, h, t2, b);
          tma_prefetch_4d(maps.k, 64 * j, h, t2, b);
          tma_prefetch_4d(maps.x, 64 * j, hv, t2, b);
        }
        for (int j = 0; j < 4; ++j) tma_prefetch_4d(maps.g, 32 * j, hv, t2, b);
      };
      raw(c1 - 1);
      if (nch > 1) prefetch(c1 - 2);
      for (int k = 0; k + 1 < nch; ++k) {  // chunk k + 1's tiles once builders and chain are done with chunk k's
        if (!wait_one(bars + DB_KED, k & 1, polls, abort)) break;
        if (!wait_one(bars + DB_QN, k & 1, polls, abort)) break;
        raw(c1 - 2 - k);
        if (k + 2 < nch) prefetch(c1 - 3 - k);
      }
    }
    __syncwarp();
  }

  cp_async_wait_all();  // (the builders' copies still in flight after an early exit)
  __syncthreads();
  if (tid == 0) {  // every issued copy and product (the last state product too) ends before the memory goes
    for (int i = 0; i < DNB_ASYNC; ++i)
      if (cnt[i] > 0) mbar_wait_lim(bars + i, (cnt[i] - 1) & 1, 1u << 24);
  }
  fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
  if (*abort && tid == 0) atomicOr(&g_kda_bwd_device_error, 1u);
}

bool bwd_tc_eligible(const BwdArgs& a, int dtype) {
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  return dtype == 1 && a.K == 128 && a.V == 128 && a.gws != nullptr && a.inter != nullptr && al16(a.q) &&
         al16(a.k) && al16(a.v) && al16(a.dO) && al16(a.g) && al16(a.dq) && al16(a.dv);
}

static int launch_bwd_dstate_tc(const BwdArgs& a, int nheads, cudaStream_t stream) {
  RawMaps maps;
  const int rc = make_raw_maps(&maps, a.q, a.k, a.dO, a.g, nullptr, a.ctab ? 1 : a.B, a.T, a.H, a.HV);
  if (rc) return rc;
  cudaError_t e = cudaFuncSetAttribute(kda_bwd_dstate_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tcc::SMEM_BYTES);
  if (e != cudaSuccess) return set_cuda_error("kda_bwd: cudaFuncSetAttribute", e);
  kda_bwd_dstate_tc_kernel<<<nheads, tcd::D_THREADS, tcc::SMEM_BYTES, stream>>>(maps, a);
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
// the record's scales are staged over the spent T image (above the fp16 record staging)
constexpr uint32_t SC_STAGE = 65536;
static_assert(SC_STAGE >= 65536 && SC_STAGE + 64 + 160 <= OP, "record scale staging");
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

__global__ void __launch_bounds__(256, 1) kda_bwd_grads_tc_kernel(const __grid_constant__ RawMaps maps,
                                                                   BwdArgs a) {
  using namespace tcg;
  using namespace tc;
  extern __shared__ __align__(1024) unsigned char sm[];
  if (smem_u32(sm) & 1023u) {  // the 128-byte swizzle of the TMA tiles needs a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(&g_kda_bwd_device_error, 2u);
    return;
  }
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
  __nv_bfloat16* dvg = static_cast<__nv_bfloat16*>(a.dv);
  float* sBeta = cx.beta();
  float* sDEl = reinterpret_cast<float*>(sm + S_EL);    // 128 floats
  float* sDbR = reinterpret_cast<float*>(sm + S_EMID);  // 64 floats
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S_BAR);
  uint64_t* bar_raw = reinterpret_cast<uint64_t*>(sm + S_TMEM + 8);  // the raw tiles' TMA
  uint32_t* sTm = reinterpret_cast<uint32_t*>(sm + S_TMEM);
  unsigned char* tC = sm + RAW_C;  // g, then the cumulative decay (fp32 TMA tile)
  float* sCarry = reinterpret_cast<float*>(sm + S_CARRY);
  const uint32_t polls = g_kda_bwd_wait_polls;
  uint32_t n_raw = 0, w_raw = 0;
  // per-subpartition partial sums, added in a fixed order (deterministic)
  float* partEl = reinterpret_cast<float*>(sm + R_AH);   // [4][128], once Ah is in the record
  float* partBr = reinterpret_cast<float*>(sm + OP_PBR);  // [4][64], once K o e^{c_last-c} is consumed

  if (cx.warp == 0) tmem_alloc(sTm, 512);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_raw, 1);
  }
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
    // q, k, dO, g tiles into the raw region and the v tile into the -dR half of [dO; -dR], by
    // TMA from one thread; beta (HV floats apart per step) by 64 threads
    if (tid == 0) {
      mbar_expect_tx(bar_raw, 4 * TILE_BF16 + TILE_F32);
      for (int j = 0; j < 2; ++j) {
        tma_load_4d(sb + RAW_Q + j * 8192, maps.q, 64 * j, h, t0, b, bar_raw);
        tma_load_4d(sb + RAW_K + j * 8192, maps.k, 64 * j, h, t0, b, bar_raw);
        tma_load_4d(sb + RAW_X + j * 8192, maps.x, 64 * j, hv, t0, b, bar_raw);
        tma_load_4d(sb + OP_V + j * 8192, maps.v, 64 * j, hv, t0, b, bar_raw);
      }
      for (int j = 0; j < 4; ++j) tma_load_4d(sb + RAW_C + j * 8192, maps.g, 32 * j, hv, t0, b, bar_raw);
    }
    ++n_raw;
    if (tid < C) sBeta[tid] = tid < L ? a.beta[((size_t)b * T + t0 + tid) * a.HV + hv] : 0.f;
    if (tid < 9) prefetch_l2(mst + tid * 1024, tid < 8 ? 4096 : 2048);  // (fp16 values and their scales)
    else if (tid >= 16 && tid < 25) prefetch_l2(dmst + (tid - 16) * 1024, tid < 24 ? 4096 : 2048);
    else if (tid == 32) prefetch_l2(irec, 2 * 16384);
    else if (tid == 33) prefetch_l2(irec + INTER_TT, 16384);
    if (__syncthreads_or(!mbar_wait_lim(bar_raw, w_raw & 1, polls))) { failed = true; break; }
    ++w_raw;
    if (L < C) {  // rows past the sequence (a packed batch's next sequence) count as zero
      for (int x = tid; x < (C - L) * 16; x += NTH) {  // 16-byte pieces of the bf16 rows
        const int i = L + (x >> 4), p = x & 15;
        const uint32_t o = (uint32_t)((p >> 3) * 8192 + i * 128 + (((p & 7) ^ (i & 7)) << 4));
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(sm + RAW_Q + o) = z;
        *reinterpret_cast<uint4*>(sm + RAW_K + o) = z;
        *reinterpret_cast<uint4*>(sm + RAW_X + o) = z;
        *reinterpret_cast<uint4*>(sm + OP_V + o) = z;
      }
      for (int x = tid; x < (C - L) * 32; x += NTH) {  // and of the fp32 g rows
        const int i = L + (x >> 5), p = x & 31;
        *reinterpret_cast<uint4*>(tC + (p >> 3) * 8192 + i * 128 + (((p & 7) ^ (i & 7)) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      __syncthreads();
    }
    {  // cumulative decay (times log2 e) in place: channel tid % 128, rows 32 (tid / 128) ..
      const int f = tid & 127, hh = tid >> 7;
      float v[32], run = 0.f;
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        run += ldf(tC, hh * 32 + r, f);
        v[r] = run;
      }
      if (hh == 0) sCarry[f] = run;
      __syncthreads();
      const float carry = hh ? sCarry[f] : 0.f;
#pragma unroll
      for (int r = 0; r < 32; ++r) *reinterpret_cast<float*>(tC + ft_off(hh * 32 + r, f)) = (v[r] + carry) * LOG2E;
      __syncthreads();
    }

    // ---------------------------------------------------------------- K o e^c, K o e^{c_last-c}, dO, dO^T
    {
      const int fq = item_f(cx);
      const float4 c63v = *reinterpret_cast<const float4*>(tC + ft_off(63, fq));
      const float c63[4] = {c63v.x, c63v.y, c63v.z, c63v.w};
      for (int m = 0; m < 8; ++m) {
        const int i = item_row(cx, m);
        const float4 c4 = *reinterpret_cast<const float4*>(tC + ft_off(i, fq));
        const float c[4] = {c4.x, c4.y, c4.z, c4.w};
        float kf[4], df[4];
        bf16x4(sm + RAW_K + bt_off(i, fq), kf);
        bf16x4(sm + RAW_X + bt_off(i, fq), df);
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
      for (int jj = 0; jj < 32; ++jj) r[jj] = tf32_rna(ldb(sm + RAW_X, hcol * 32 + jj, Lr));
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
      for (int jj = 0; jj < 32; ++jj) {
        xs[jj] = ldb(sm + OP_V, hcol * 32 + jj, Lr) - x[jj];
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
      // their 16 block scales, as in the record, and the per-warp maxima they come from
      float* ssc = reinterpret_cast<float*>(sm + SC_STAGE);
      unsigned* wmax = reinterpret_cast<unsigned*>(sm + SC_STAGE + 64);  // [warp][5]
      static_assert(2 * (GH_KED + 8192) <= OP_DO, "record staging below [dO; -dR]");
      static_assert(2 * (GH_KED + 8192) == 4 * G_DBR, "fp32 tail follows the fp16 matrices");
      static_assert(GREC == G_SC + 16, "record scales");
      const int warp = cx.warp, half = cx.sub >> 1;  // rows 64 half .. of [dP; dA] and [dQE; dKE']
      float v[32];
      {  // block maxima: [dP; dA] (half, hcol), [dQE; dKE'] (half, 2 hcol + cb), dKEd (2 hcol + cb)
        tmem_ld32(tm + lo + TM_PA + hcol * 32, v);
        unsigned m0 = warp_absmax32(v, lane);
        unsigned mq[2], mk[2];
        for (int cb = 0; cb < 2; ++cb) {
          tmem_ld32(tm + lo + TM_QK + hcol * 64 + cb * 32, v);
          mq[cb] = warp_absmax32(v, lane);
          tmem_ld32(tm + lo + TM_KED + hcol * 64 + cb * 32, v);
          mk[cb] = warp_absmax32(v, lane, 16);  // (M = 64 accumulator: lanes < 16)
        }
        if (lane == 0) {
          wmax[warp * 5 + 0] = m0;
          wmax[warp * 5 + 1] = mq[0];
          wmax[warp * 5 + 2] = mq[1];
          wmax[warp * 5 + 3] = mk[0];
          wmax[warp * 5 + 4] = mk[1];
        }
      }
      __syncthreads();
      // warp w = 4 hcol + sub: the blocks of rows half (sub / 2) come from warps 4 hcol + 2 half + {0, 1};
      // dKEd's from the four warps 4 hcol + {0 .. 3}
      const int w0 = 4 * hcol + 2 * half, wk = 4 * hcol;
      float inv;
      float up = block_up(max(wmax[w0 * 5 + 0], wmax[(w0 + 1) * 5 + 0]), &inv);
      if (cx.sub == 2 * half && lane == 0) ssc[half * 2 + hcol] = inv;
      tmem_ld32(tm + lo + TM_PA + hcol * 32, v);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) st4h(st + GH_PA + rec_off(Lr, hcol * 32 + 4 * q4, 64), v + 4 * q4, up);
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hcol * 64 + cb * 32;
        up = block_up(max(wmax[w0 * 5 + 1 + cb], wmax[(w0 + 1) * 5 + 1 + cb]), &inv);
        if (cx.sub == 2 * half && lane == 0) ssc[4 + half * 4 + f0 / 32] = inv;
        tmem_ld32(tm + lo + TM_QK + f0, v);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) st4h(st + GH_QK + rec_off(Lr, f0 + 4 * q4, 128), v + 4 * q4, up);
        const unsigned mk = max(max(wmax[wk * 5 + 3 + cb], wmax[(wk + 1) * 5 + 3 + cb]),
                                max(wmax[(wk + 2) * 5 + 3 + cb], wmax[(wk + 3) * 5 + 3 + cb]));
        up = block_up(mk, &inv);
        if (cx.sub == 0 && lane == 0) ssc[12 + f0 / 32] = inv;
        tmem_ld32(tm + lo + TM_KED + f0, v);
        if (lane < 16) {
          const int r = cx.sub * 16 + lane;  // M = 64 accumulator layout
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) st4h(st + GH_KED + rec_off(r, f0 + 4 * q4, 128), v + 4 * q4, up);
        }
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        bulk_s2g(rec, sb, 32768);
        bulk_s2g(rec + 8192, sb + 32768, 32768);
        bulk_s2g(rec + G_DBR, sb + S_EMID, 256);
        bulk_s2g(rec + G_DEL, sb + S_EL, 512);
        bulk_s2g(rec + G_SC, sb + SC_STAGE, 64);
        bulk_commit();
        bulk_wait_read();
      }
    }
    // the record's shared-memory sources are read and every TMEM read-out is
    // complete before the next item overwrites them (its tiles by TMA)
    fence_before();
    fence_async_smem();
    __syncthreads();
  }

  if (failed && tid == 0) {  // the raw tiles and the products still in flight end before the memory goes
    while (w_raw < n_raw) mbar_wait_lim(bar_raw, (w_raw++) & 1, 1u << 24);
    mbar_wait_lim(bar, (phase ^ 1) & 1, 1u << 24);  // (wait_mma flips the phase even when it gives up)
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
  RawMaps maps;
  const int rc = make_raw_maps(&maps, a.q, a.k, a.dO, a.g, a.v, a.ctab ? 1 : a.B, a.T, a.H, a.HV);
  if (rc) return rc;
  kda_bwd_grads_tc_kernel<<<(int)items, tcc::NTH, tcc::SMEM_BYTES, stream>>>(maps, a);
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
int set_bwd_wait_polls(unsigned polls) {
  const unsigned v = polls ? polls : (1u << 24);
  const cudaError_t e = cudaMemcpyToSymbol(g_kda_bwd_wait_polls, &v, sizeof(v));
  if (e != cudaSuccess) return set_cuda_error("kda_set_wait_polls", e);
  return 0;
}

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
