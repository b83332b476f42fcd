// Chunked tensor-core (tcgen05) KDA prefill forward for K = V = 128, bf16
// q/k/v/o, fp32 g/beta/state, as two kernels:
//
//   kda_fwd_intra_tc_kernel  (chunk-parallel, every (sequence, value head,
//       64-step chunk) at once, two CTAs per SM): the in-chunk cumulative
//       decay, the interaction products Ah and P (split exponents, see
//       kda_tc_chunk.cuh), and the inverse T = (I + diag(beta) Ah)^-1.  It
//       leaves only the T and P operand images (32 KB per chunk) in the
//       workspace, plus, for a training forward, the backward's record.
//   kda_fwd_state_tc_kernel  (one CTA per (sequence, value head)): carries
//       the K x V state through the chunks in tensor memory.  It rebuilds the
//       cheap per-chunk operands itself from the raw rows, so that nothing of
//       size C x K crosses HBM twice:
//         [Y^T | O^T] = M^T [K o e^c ; Q~ o e^c]^T       (state in TMEM as A)
//         Z^T         = (V^T - Y^T) diag(beta)
//         U^T         = Z^T T^T                          (U = T diag(beta)(V - (K o e^c) M))
//         M'^T        = M^T diag(e^{c_last}) + U^T (K o e^{c_last - c})
//         O^T        += U^T P^T
//       (the chunk algebra of "research_layers.py", delta_recurrence, with
//       erase = write = k and beta folded into the residual).  The loop is
//       software-pipelined: the next chunk's raw rows arrive by TMA and its
//       decay and [K o e^c ; Q~ o e^c] operand are built while this chunk's
//       last state products run, and the previous chunk's output leaves while
//       the next chunk's first products run.
//
// With the fused preparation (PREP) the gate g = gate(z + dt_bias) comes from
// kda_prep_gate_kernel (an element-wise pass over z), the kernels form the
// q and k row factors scale / |q_i| and 1 / |k_i| from the raw rows and the
// beta sigmoid themselves, and with an output gate the state pass writes fp32
// rows that the row kernel of the output gate finishes.
//
// q, k, v and g are staged by TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast)
// from 4-D tensor maps [B, T, heads, 128]; the T and P images by 1-D bulk
// copies.  beta is HV floats apart per step, which no tensor map can address
// (its row stride need not be a multiple of 16 bytes): 64 threads load it.
//
// Bounded waits: every mbarrier wait gives up after g_kda_wait_polls probes
// (kda_set_wait_polls; a test sets it to 1).  A kernel that gives up waits
// for every copy and tensor-core product it has issued (with the default
// bound), frees its tensor memory, sets bit 0 of the device error word and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"
#include "kda_tc_chunk.cuh"

namespace kda {

__device__ unsigned int g_kda_fwd_chunked_error;
constexpr unsigned DEFAULT_WAIT_POLLS = 1u << 24;
__device__ unsigned int g_kda_wait_polls = DEFAULT_WAIT_POLLS;

namespace fc {
using namespace tcc;

// 4-D tensor maps [rows, T, heads, 128] of the raw inputs (rows = B, or 1 for
// packed sequences); box 64 steps x one head x one 128-byte column block.
struct FwdMaps {
  CUtensorMap q, k, v, g;
};


// Barrier of the threads that run a per-chunk preparation: the whole CTA, or
// one role of a warp-specialised kernel (named barrier `id` over `n` threads).
struct SyncAll {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct SyncNamed {
  int id, n;
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
};

// One thread issues the TMA loads of a chunk's q, k rows (query/key head h)
// and g rows (value head hv) on `bar`.
__device__ __forceinline__ void issue_qkg(const FwdMaps& m, uint32_t sQ, uint32_t sK, uint32_t sG, uint64_t* bar,
                                          int b, int t0, int h, int hv) {
  using namespace tc;
  mbar_expect_tx(bar, 2 * TILE_BF16 + TILE_F32);
  tma_load_4d(sQ, &m.q, 0, h, t0, b, bar);
  tma_load_4d(sQ + 8192, &m.q, 64, h, t0, b, bar);
  tma_load_4d(sK, &m.k, 0, h, t0, b, bar);
  tma_load_4d(sK + 8192, &m.k, 64, h, t0, b, bar);
#pragma unroll
  for (int j = 0; j < 4; ++j) tma_load_4d(sG + j * 8192, &m.g, 32 * j, hv, t0, b, bar);
}
__device__ __forceinline__ void prefetch_qkg(const FwdMaps& m, int b, int t0, int h, int hv) {
  using namespace tc;
  tma_prefetch_4d(&m.q, 0, h, t0, b);
  tma_prefetch_4d(&m.q, 64, h, t0, b);
  tma_prefetch_4d(&m.k, 0, h, t0, b);
  tma_prefetch_4d(&m.k, 64, h, t0, b);
#pragma unroll
  for (int j = 0; j < 4; ++j) tma_prefetch_4d(&m.g, 32 * j, hv, t0, b);
}

// Per-chunk input preparation on the landed raw tiles (256 threads): the g
// rows at or past L are cleared (packed sequences: they belong to the next
// sequence), so that c_63 = c_{L-1}; with PREP the row factors scale / |q_i|
// and 1 / |k_i| ("kimi_k3_host/kda.rs", l2norm_rows) go to sNq, sNk.  Ends
// with a barrier of the 256 threads that run it (`sync`; tid counts from 0
// among them).
template <bool PREP, class Sync>
__device__ __forceinline__ void prep_tile(unsigned char* sQ, unsigned char* sK, unsigned char* sG, float* sNq,
                                          float* sNk, int tid, int L, float scale, Sync sync) {
  if constexpr (PREP) {  // 2 threads per row, rows 0..63 of q then of k
    const int r = tid >> 1, part = tid & 1, i = r & 63;
    const unsigned char* t = r < 64 ? sQ : sK;
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      float x[4];
      bf16x4(t + bt_off(i, part * 64 + 4 * u), x);
      s = fmaf(x[0], x[0], fmaf(x[1], x[1], fmaf(x[2], x[2], fmaf(x[3], x[3], s))));
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    if (part == 0) {
      const float nrm = rsqrtf(s + KDA_L2_EPS_F);
      if (r < 64) sNq[i] = nrm * scale;
      else sNk[i] = nrm;
    }
  }
  if (L < C)
    for (int x = tid; x < (C - L) * KD; x += NTH) *reinterpret_cast<float*>(sG + ft_off(L + x / KD, x % KD)) = 0.f;
  sync();
}

// In-chunk cumulative decay in place over the fp32 tile: natural-log g in,
// c_i = sum_{s<=i} g_s times log2(e) out.  Thread t: channel t % 128, rows
// 32 (t / 128) .. + 31, then the carry of the first half.  Returns,
// block-uniformly with WIDE, whether some 32-row half's decay from its middle
// row to either end exceeds 80 (the split exponents would leave fp32 range).
// (WIDE needs the whole CTA: its answer is a block-wide vote)
template <bool WIDE, class Sync>
__device__ __forceinline__ bool cumsum_tile(unsigned char* sG, float* sCarry, int tid, Sync sync) {
  const int f = tid & 127, hh = tid >> 7;
  float v[32], run = 0.f;
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    run += ldf(sG, hh * 32 + r, f);
    v[r] = run;
  }
  if (hh == 0) sCarry[f] = run;
  sync();
  const float carry = hh ? sCarry[f] : 0.f;
#pragma unroll
  for (int r = 0; r < 32; ++r) *reinterpret_cast<float*>(sG + ft_off(hh * 32 + r, f)) = (v[r] + carry) * LOG2E;
  sync();
  if constexpr (!WIDE) {
    return false;
  } else {
    bool w = false;
    if (tid < KD) {
      const float lim = DIAG_SPAN_MAX * LOG2E;
      const float c0 = ldf(sG, 0, tid), c15 = ldf(sG, 15, tid), c31 = ldf(sG, 31, tid);
      const float c32 = ldf(sG, 32, tid), c47 = ldf(sG, 47, tid), c63 = ldf(sG, 63, tid);
      w = fabsf(c0 - c15) > lim || fabsf(c15 - c31) > lim || fabsf(c32 - c47) > lim || fabsf(c47 - c63) > lim;
    }
    return __syncthreads_or(w);
  }
}

__device__ __forceinline__ float4 ld4f(const unsigned char* t, int i, int f) {
  return *reinterpret_cast<const float4*>(t + ft_off(i, f));
}

// ============================================================================
// kda_fwd_intra_tc_kernel
// ============================================================================
// Shared memory (bytes): the raw q, k tiles and the g / decay tile; the
// interaction operands of one quarter of the key channels (32 channels:
// [K o x; Q~ o x] 128 x 32, K o y 64 x 32, the lower-left block's 64 x 32 and
// 32 x 32), K-major with K extent 32; then beta, the row factors, the decay
// carry, the barriers and the TMEM base.  After the last quarter the raw
// region holds Ah, T (row-major) and the inverse's scratch (kda_tc_chunk.cuh
// R_AH, R_TROW, R_SW) and the operand region the T and P images.
constexpr uint32_t K1_Q = 0, K1_K = 16384, K1_C = 32768, K1_OP = 65536;
constexpr uint32_t Q_XA = 0, Q_YA = 16384, Q_XB = 24576, Q_YB = 32768, Q_BYTES = 36864;
constexpr uint32_t K1_TIMG = K1_OP, K1_PIMG = K1_OP + 16384;
constexpr uint32_t K1_BETA = K1_OP + Q_BYTES, K1_NQ = K1_BETA + 256, K1_NK = K1_NQ + 256, K1_CARRY = K1_NK + 256,
                   K1_BAR = K1_CARRY + 512, K1_TMEM = K1_BAR + 32, K1_BYTES = K1_TMEM + 16;
static_assert(R_SW + 3072 <= K1_OP && R_TROW + 16640 <= R_SW, "inverse scratch inside the raw region");
static_assert(K1_PIMG + 16384 <= K1_OP + Q_BYTES, "T and P images inside the operand region");
static_assert(2 * (K1_BYTES + 1024) <= 233472, "two CTAs per SM");

// Operands of key channels 32p .. 32p + 31 (see the split exponents in
// kda_tc_chunk.cuh): thread t builds rows 8 (t / 64) + t % 8 (+ 32) of the
// four channels 32p + 4 ((t / 8) % 8) .. + 3; eight consecutive lanes hold
// eight rows, so their 16-byte stores fall in distinct bank groups.
template <bool NORM>
__device__ __forceinline__ void build_quarter(unsigned char* sm, int tid, int p, float scale) {
  using namespace tc;
  const unsigned char* sC = sm + K1_C;
  const float* sNq = reinterpret_cast<const float*>(sm + K1_NQ);
  const float* sNk = reinterpret_cast<const float*>(sm + K1_NK);
  unsigned char* op = sm + K1_OP;
  const int rl = tid & 7, fg = (tid >> 3) & 7, rb = tid >> 6, kq = 4 * fg, f = 32 * p + kq;
  const float4 r15 = ld4f(sC, 15, f), r47 = ld4f(sC, 47, f), r31 = ld4f(sC, 31, f);
  const float c31[4] = {r31.x, r31.y, r31.z, r31.w};
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int i = 32 * m + 8 * rb + rl;
    const float4 c4 = ld4f(sC, i, f);
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
    const float4 rr = m ? r47 : r15;
    const float cr[4] = {rr.x, rr.y, rr.z, rr.w};
    float kf[4], qf[4];
    bf16x4(sm + K1_K + bt_off(i, f), kf);
    bf16x4(sm + K1_Q + bt_off(i, f), qf);
    const float qm = NORM ? sNq[i] : scale, km = NORM ? sNk[i] : 1.f;
    float xa[4], ya[4], xb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      kf[u] *= km;
      qf[u] *= qm;
      xa[u] = ex2(cc[u] - cr[u]);
      ya[u] = ex2(cr[u] - cc[u]);
      xb[u] = m ? ex2(cc[u] - c31[u]) : ex2(c31[u] - cc[u]);
    }
    st_tf32x4(op, Q_XA + kmaj(i, kq, 32), kf[0] * xa[0], kf[1] * xa[1], kf[2] * xa[2], kf[3] * xa[3]);
    st_tf32x4(op, Q_XA + kmaj(64 + i, kq, 32), qf[0] * xa[0], qf[1] * xa[1], qf[2] * xa[2], qf[3] * xa[3]);
    st_tf32x4(op, Q_YA + kmaj(i, kq, 32), kf[0] * ya[0], kf[1] * ya[1], kf[2] * ya[2], kf[3] * ya[3]);
    if (m) {
      st_tf32x4(op, Q_XB + kmaj(i - 32, kq, 32), kf[0] * xb[0], kf[1] * xb[1], kf[2] * xb[2], kf[3] * xb[3]);
      st_tf32x4(op, Q_XB + kmaj(i, kq, 32), qf[0] * xb[0], qf[1] * xb[1], qf[2] * xb[2], qf[3] * xb[3]);
    } else {
      st_tf32x4(op, Q_YB + kmaj(i, kq, 32), kf[0] * xb[0], kf[1] * xb[1], kf[2] * xb[2], kf[3] * xb[3]);
    }
  }
}

// Same-half Ah / P entries pair by pair over all 128 channels (only when
// cumsum_tile reported a span beyond the split-exponent range); the same
// thread split as tcc::pairwise_compute, which readout_ap consumes.
template <bool NORM>
__device__ __forceinline__ void pairwise_tile(const unsigned char* sm, int tid, float scale, Pairwise& pw) {
  const unsigned char* sC = sm + K1_C;
  const float* sNq = reinterpret_cast<const float*>(sm + K1_NQ);
  const float* sNk = reinterpret_cast<const float*>(sm + K1_NK);
  pw.kind = tid >> 7;
  pw.i = (tid >> 1) & 63;
  pw.j0 = (pw.i & 32) + (tid & 1) * 16;
  const unsigned char* xi = sm + (pw.kind ? K1_Q : K1_K);
  for (int jj = 0; jj < 16; ++jj) {
    const int j = pw.j0 + jj;
    float acc = 0.f;
    if (pw.kind ? (j <= pw.i) : (j < pw.i)) {
      for (int f = 0; f < KD; ++f)
        acc = fmaf(ldb(xi, pw.i, f) * ldb(sm + K1_K, j, f), tc::ex2(ldf(sC, pw.i, f) - ldf(sC, j, f)), acc);
      if (NORM)
        acc *= (pw.kind ? sNq[pw.i] : sNk[pw.i]) * sNk[j];
      else if (pw.kind)
        acc *= scale;
    }
    pw.v[jj] = acc;
  }
}

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, uint32_t polls) {
  return !__syncthreads_or(!tc::mbar_wait_lim(bar, parity, polls));
}

template <bool PREP>
__global__ void __launch_bounds__(NTH, 2) kda_fwd_intra_tc_kernel(const __grid_constant__ FwdMaps maps, FwdArgs a) {
  using namespace tc;
  extern __shared__ __align__(1024) unsigned char sm[];
  if (smem_u32(sm) & 1023u) {  // the 128-byte swizzle of the TMA tiles needs a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(&g_kda_fwd_chunked_error, 2u);
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
  const int tid = cx.tid;
  const uint32_t sb = cx.sb;
  const int G = a.HV / a.H, NTc = (a.T + C - 1) / C;
  const int items = a.ctab ? a.NC * a.HV : NTc * a.HV * a.B;
  float* sBeta = reinterpret_cast<float*>(sm + K1_BETA);
  uint64_t* bar_raw = reinterpret_cast<uint64_t*>(sm + K1_BAR);
  uint64_t* bar_mma = bar_raw + 1;
  uint32_t* sTm = reinterpret_cast<uint32_t*>(sm + K1_TMEM);
  const uint32_t polls = g_kda_wait_polls;

  if (cx.warp == 0) tmem_alloc(sTm, 128);
  if (tid == 0) {
    mbar_init(bar_raw, 1);
    mbar_init(bar_mma, 1);
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = *sTm;
  cx.tm = tm;
  constexpr uint32_t TM_A = 0, TM_B = 64;
  uint32_t n_raw = 0, w_raw = 0, n_mma = 0, w_mma = 0;
  bool failed = false;

  // item = the chunk's global index (chunk fastest, then value head, then batch row)
  const auto span_of = [&](int item, int& hv, int& b, int& t0, int& L) {
    if (a.ctab) {
      const int c = item % a.NC;
      hv = item / a.NC;
      b = 0;
      t0 = a.ctab[2 * c];
      L = a.ctab[2 * c + 1];
    } else {
      const int ch = item % NTc;
      hv = (item / NTc) % a.HV;
      b = item / (NTc * a.HV);
      t0 = ch * C;
      L = min(C, a.T - t0);
    }
  };
  const auto issue = [&](int item) {
    int hv, b, t0, L;
    span_of(item, hv, b, t0, L);
    issue_qkg(maps, sb + K1_Q, sb + K1_K, sb + K1_C, bar_raw, b, t0, hv / G, hv);
  };
  if (blockIdx.x < items) {
    if (tid == 0) issue(blockIdx.x);
    ++n_raw;
  }
  bool first = true;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    int hv, b, t0, L;
    span_of(item, hv, b, t0, L);
    float bval = 0.f;
    if (tid < C && tid < L) {
      bval = a.beta[((size_t)b * a.T + t0 + tid) * a.HV + hv];
      if (PREP) bval = prep_sigmoid_fast(bval);
    }
    if (!wait_all(bar_raw, w_raw & 1, polls)) { failed = true; break; }
    ++w_raw;
    if (tid < C) sBeta[tid] = bval;
    if (tid == 0 && item + 2 * (int)gridDim.x < items) {  // the item after next into L2
      int hv2, b2, t2, L2;
      span_of(item + 2 * gridDim.x, hv2, b2, t2, L2);
      prefetch_qkg(maps, b2, t2, hv2 / G, hv2);
    }
    prep_tile<PREP>(sm + K1_Q, sm + K1_K, sm + K1_C, reinterpret_cast<float*>(sm + K1_NQ),
                    reinterpret_cast<float*>(sm + K1_NK), tid, L, a.scale, SyncAll());
    const bool wide = cumsum_tile<true>(sm + K1_C, reinterpret_cast<float*>(sm + K1_CARRY), tid, SyncAll());

    for (int p = 0; p < 4; ++p) {
      if (p == 0) {  // the previous item's T and P images have left the operand region
        if (!first && tid == 0) bulk_wait_read();
        __syncthreads();
      } else {
        if (!wait_all(bar_mma, w_mma & 1, polls)) { failed = true; break; }
        ++w_mma;
      }
      build_quarter<PREP>(sm, tid, p, a.scale);
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        fence_after();
        const uint32_t idA = idesc_tf32(128, 64), idB = idesc_tf32(64, 32);
        for (int ks = 0; ks < 4; ++ks)
          mma_ss(tm + TM_A, desc(sb + K1_OP + Q_XA + ks * 256, 1024), desc(sb + K1_OP + Q_YA + ks * 256, 1024),
                 idA, (p | ks) != 0);
        for (int ks = 0; ks < 4; ++ks)
          mma_ss(tm + TM_B, desc(sb + K1_OP + Q_XB + ks * 256, 1024), desc(sb + K1_OP + Q_YB + ks * 256, 1024),
                 idB, (p | ks) != 0);
        commit(bar_mma);
      }
      ++n_mma;
    }
    if (failed) break;
    first = false;
    Pairwise pw;
    pw.kind = -1;
    pw.i = pw.j0 = 0;
    if (wide) pairwise_tile<PREP>(sm, tid, a.scale, pw);
    if (!wait_all(bar_mma, w_mma & 1, polls)) { failed = true; break; }
    ++w_mma;
    fence_after();
    float* irec = a.inter ? a.inter + (size_t)item * INTER_REC : nullptr;  // (item = chunk_gc)
    readout_ap<NTH>(cx, tm + TM_A, tm + TM_B, wide, pw, nullptr, K1_PIMG);
    if (irec) {  // the P^T image of the record from the P image: piece x holds P^T(r, k .. k + 3)
      for (int x = tid; x < C * C / 4; x += NTH) {
        const int r = (x >> 7) * 8 + (x & 7), k = ((x & 127) >> 3) * 4;
        uint4 w;
        w.x = *reinterpret_cast<const uint32_t*>(sm + p_off(k, r, K1_PIMG));
        w.y = *reinterpret_cast<const uint32_t*>(sm + p_off(k + 1, r, K1_PIMG));
        w.z = *reinterpret_cast<const uint32_t*>(sm + p_off(k + 2, r, K1_PIMG));
        w.w = *reinterpret_cast<const uint32_t*>(sm + p_off(k + 3, r, K1_PIMG));
        *reinterpret_cast<uint4*>(irec + x * 4) = w;
      }
    }
    invert<NTH>(cx, sBeta);
    {  // T as its operand image (rows i, K = j); with a record also its T, T^T images and Ah
      const float* tr = reinterpret_cast<const float*>(sm + R_TROW);
      for (int x = tid; x < C * 16; x += NTH) {  // 16-byte piece x of the image: x * 16 = kmaj(i, j4, 64)
        const int i = ((x >> 7) << 3) | (x & 7), j4 = ((x >> 3) & 15) * 4;
        const float* pr = tr + i * 65 + j4;
        const uint4 t = make_uint4(tf32_rna(pr[0]), tf32_rna(pr[1]), tf32_rna(pr[2]), tf32_rna(pr[3]));
        // the state pass's image is T diag(beta): U = (T diag(beta)) (V - (K o e^c) M)
        *reinterpret_cast<uint4*>(sm + K1_TIMG + x * 16) =
            make_uint4(tf32_rna(pr[0] * sBeta[j4]), tf32_rna(pr[1] * sBeta[j4 + 1]), tf32_rna(pr[2] * sBeta[j4 + 2]),
                       tf32_rna(pr[3] * sBeta[j4 + 3]));
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
    __syncthreads();  // the raw region is free: the next item's rows may come in
    if (item + (int)gridDim.x < items) {
      if (tid == 0) issue(item + gridDim.x);
      ++n_raw;
    }
    if (tid == 0) {
      unsigned char* rec = a.img + (size_t)item * FWI_BYTES;
      bulk_s2g(rec + FWR_T, sb + K1_TIMG, 16384);
      bulk_s2g(rec + FWR_P, sb + K1_PIMG, 16384);
      bulk_commit();
    }
  }
  if (failed) {  // let every issued copy and product finish before the shared and tensor memory go
    while (w_raw < n_raw) tc::mbar_wait_lim(bar_raw, (w_raw++) & 1, DEFAULT_WAIT_POLLS);
    while (w_mma < n_mma) tc::mbar_wait_lim(bar_mma, (w_mma++) & 1, DEFAULT_WAIT_POLLS);
  }
  if (tid == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  fence_before();
  __syncthreads();
  if (cx.warp == 0) tmem_dealloc(tm, 128);
  if (failed && tid == 0) atomicOr(&g_kda_fwd_chunked_error, 1u);
}

// ============================================================================
// kda_fwd_state_tc_kernel
// ============================================================================
// Warp-specialised, 544 threads (17 warps):
//   issuer warp 0 (lane 0): every tensor-core product and the v, T, P copies
//     (a tcgen05.mma issue can block its thread for about the product's
//     duration, so this warp does nothing else);
//   chain warps 1-8 (warp w: TMEM lanes 32 (w % 4) .. + 31, lane = value
//     column n; column half (w - 1) / 4 of every accumulator): the residual
//     Z^T = V^T - Y^T, the tf32 rounding of U^T, the state's decay (storing
//     the entering state for a training forward), the output rows;
//   builder warps 9-16: the next chunk's decay, [K o e^c ; Q~ o e^c] and
//     (K o e^{c_last-c})^T operands and e^{c_last}; builder thread 0 issues the
//     raw q / k / g copies.
// The output rows of a chunk leave from the chain's registers: the chain reads
// O^T out of TMEM, releases the accumulator (B_O) and then stores.
// The roles meet on mbarriers only: builders and chain threads arrive when an
// operand or a step is done, tensor-core completions arrive through
// tcgen05.commit.  A wait that gives up sets the shared abort word, which
// ends the other roles' waits too.
//
// Per chunk the products run in the order [Y^T | O^T] (m1), the previous
// chunk's O^T += U^T P^T (m4, deferred so that it is off the state's path),
// U^T (m2), M^T += U^T (K o e^{c_last-c}) (m3).
//
// Shared memory (bytes): raw q, k, g / decay, v tiles (TMA); the
// [K o e^c ; Q~ o e^c] operand (rows 0..63 and 64..127, K = key channel,
// K extent 128); (K o e^{c_last - c})^T (rows = key channel, K = step,
// extent 64); the T diag(beta) and P images; then e^{c_last}, the output gate's row sums, the row factors, the
// decay carry, the barriers, the issue counts and the TMEM base.
constexpr uint32_t S2_Q = 0, S2_K = 16384, S2_C = 32768, S2_V = 65536, S2_KQ = 81920, S2_KD = 147456,
                   S2_T = 180224, S2_P = 196608, S2_EL = 212992, S2_RED = S2_EL + 512, S2_NQ = S2_RED + 1024,
                   S2_NK = S2_NQ + 256, S2_CARRY = S2_NK + 256, S2_BAR = S2_CARRY + 512, S2_CNT = S2_BAR + 128,
                   S2_TMEM = S2_CNT + 64, S2_BYTES = S2_TMEM + 16;
static_assert(S2_BYTES + 1024 <= 233472, "one CTA per SM");
constexpr int K2_THREADS = 544, CH0 = 32, CH_THREADS = 256, BU0 = 288, BU_THREADS = 256;
// named barriers: 1 the chain warps, 2 the builder warps, 3 the issuer warp with the chain warps
constexpr int BAR_STATE0 = 3;
// TMEM columns: the state M^T (lane = value column n, column = key channel);
// two [Y^T | O^T] accumulators (chunks alternate; Z^T is written over Y^T);
// U^T
constexpr uint32_t TM_S = 0, TM_D0 = 128, TM_U = 384;
// barriers: async copies and products (counted in S2_CNT for the drain), then the roles' arrivals
enum { B_RAW, B_V, B_T, B_P, B_M1, B_M2, B_M3, B_M4, NB_ASYNC, B_KQ = NB_ASYNC, B_KD, B_Z, B_O, B_UR, NB_ALL };

template <bool PREP>
__global__ void __launch_bounds__(K2_THREADS, 1) kda_fwd_state_tc_kernel(const __grid_constant__ FwdMaps maps,
                                                                         FwdArgs a) {
  using namespace tc;
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  if (sb & 1023u) {  // the 128-byte swizzle of the TMA tiles needs a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(&g_kda_fwd_chunked_error, 2u);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hv = blockIdx.x, sq = blockIdx.y;  // batch row, or sequence of a packed batch
  const int b = row_of(a, sq), c0 = chunk_begin(a, sq), nch = chunk_end(a, sq) - c0;
  const int G = a.HV / a.H, h = hv / G, T = a.T;
  const size_t head = (size_t)sq * a.HV + hv;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S2_BAR);
  int* cnt = reinterpret_cast<int*>(sm + S2_CNT);  // issued phases per async barrier; [15]: abort
  volatile int* abort = cnt + 15;
  uint32_t* sTm = reinterpret_cast<uint32_t*>(sm + S2_TMEM);
  float* sEl = reinterpret_cast<float*>(sm + S2_EL);
  const uint32_t polls = g_kda_wait_polls;

  if (warp == 0) tmem_alloc(sTm, 512);
  if (tid == 0) {
    for (int i = 0; i < NB_ALL; ++i)
      mbar_init(bars + i, i < NB_ASYNC ? 1 : (i == B_KQ || i == B_KD ? BU_THREADS : CH_THREADS));
    for (int i = 0; i < 16; ++i) cnt[i] = 0;
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = *sTm;

  const auto span = [&](int ch) { return chunk_span(a, c0 + ch); };
  const auto rec = [&](int ch) { return a.img + chunk_gc(a, sq, hv, c0 + ch) * (size_t)FWI_BYTES; };

  if (warp == 0) {
    // ======================================================================== issuer warp
    // no product before the chain has written the entering state into TMEM
    named_sync(BAR_STATE0, 32 + CH_THREADS);
    if (lane == 0 && nch > 0) {
      const auto issue_v = [&](int ch) {
        mbar_expect_tx(bars + B_V, TILE_BF16);
        tma_load_4d(sb + S2_V, &maps.v, 0, hv, span(ch).x, b, bars + B_V);
        tma_load_4d(sb + S2_V + 8192, &maps.v, 64, hv, span(ch).x, b, bars + B_V);
        ++cnt[B_V];
      };
      const auto issue_img = [&](int which, uint32_t dst, int ch, uint32_t off) {
        mbar_expect_tx(bars + which, 16384);
        bulk_g2s(dst, rec(ch) + off, 16384, bars + which);
        ++cnt[which];
      };
      const auto commit_to = [&](int which) {
        commit(bars + which);
        ++cnt[which];
      };
      const auto o_part = [&](int ch) {  // O^T += U^T P^T of chunk ch
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(tm + TM_D0 + (ch & 1) * 128 + 64, tm + TM_U + ks * 8, desc(sb + S2_P + ks * 256, 2048),
                 idesc_tf32(128, 64), 1);
        commit_to(B_M4);
      };
      issue_v(0);
      issue_img(B_T, sb + S2_T, 0, FWR_T);
      issue_img(B_P, sb + S2_P, 0, FWR_P);
      for (int ch = 0; ch < nch; ++ch) {
        const uint32_t par = ch & 1, D = TM_D0 + (ch & 1) * 128;
        // [Y^T | O^T] = M^T [K o e^c ; Q~ o e^c]^T once the operand is built, the state updated
        // and the output of two chunks back (same accumulator) read out
        if (!wait_one(bars + B_KQ, par, polls, abort)) break;
        if (ch > 0 && !wait_one(bars + B_M3, par ^ 1, polls, abort)) break;
        if (ch > 1 && !wait_one(bars + B_O, par, polls, abort)) break;
        fence_after();
        for (int ks = 0; ks < 16; ++ks)
          mma_ts(tm + D, tm + TM_S + ks * 8, desc(sb + S2_KQ + ks * 256, 4096), idesc_tf32(128, 128), ks > 0);
        commit_to(B_M1);
        if (ch > 0) {  // (U^T and P of the previous chunk are still resident)
          if (!wait_one(bars + B_P, par ^ 1, polls, abort)) break;
          o_part(ch - 1);
        }
        // U^T = Z^T (T diag(beta))^T
        if (!wait_one(bars + B_Z, par, polls, abort)) break;
        if (!wait_one(bars + B_T, par, polls, abort)) break;
        fence_after();
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(tm + TM_U, tm + D + ks * 8, desc(sb + S2_T + ks * 256, 2048), idesc_tf32(128, 64), ks > 0);
        commit_to(B_M2);
        if (ch + 1 < nch) issue_v(ch + 1);  // this chunk's v is consumed
        if (ch > 0) {  // the previous chunk's P is consumed once its output products are done
          if (!wait_one(bars + B_M4, par ^ 1, polls, abort)) break;
          issue_img(B_P, sb + S2_P, ch, FWR_P);
        }
        if (!wait_one(bars + B_M2, par, polls, abort)) break;
        if (ch + 1 < nch) issue_img(B_T, sb + S2_T, ch + 1, FWR_T);  // this chunk's T is consumed
        // M^T += U^T (K o e^{c_last-c}) once U^T is rounded and the state decayed
        if (!wait_one(bars + B_UR, par, polls, abort)) break;
        if (!wait_one(bars + B_KD, par, polls, abort)) break;
        fence_after();
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(tm + TM_S, tm + TM_U + ks * 8, desc(sb + S2_KD + ks * 256, 2048), idesc_tf32(128, 128), 1);
        commit_to(B_M3);
      }
      if (!*abort && wait_one(bars + B_P, (nch - 1) & 1, polls, abort)) {  // the last chunk's output products
        fence_after();
        o_part(nch - 1);
      }
    }
    __syncwarp();
  } else if (warp <= 8) {
    // ======================================================================== chain warps
    const int n = (warp & 3) * 32 + lane, hc = (warp - 1) >> 2;  // TMEM lane (value column), column half
    const uint32_t lo = (uint32_t)((warp & 3) * 32) << 16;
    // o rows hc * 32 .. + 31 of chunk ch (value column n) from O^T in accumulator d: read
    // out, released to the issuer (B_O), then stored from registers (fp32 into o32 when
    // an output gate follows, else in the output dtype)
    const auto out_rows = [&](int ch, uint32_t d) {
      const int2 s = span(ch);
      float v[32];
      tmem_ld32(tm + lo + d + 64 + hc * 32, v);
      fence_before();
      mbar_arrive(bars + B_O);
      const size_t row0 = (((size_t)b * T + s.x + hc * 32) * a.HV + hv) * VD + n, step = (size_t)a.HV * VD;
      const int rows = min(32, s.y - hc * 32);
      if (a.o32) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < rows) a.o32[row0 + j * step] = v[j];
      } else if (a.o) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.o) + row0;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < rows) dst[j * step] = __float2bfloat16_rn(v[j]);
      }
    };
    {  // entering state, transposed: lane n, columns hc * 64 .. + 63
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hc * 64 + cb * 32;
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(a.S0 ? a.S0[(head * KD + f0 + j) * VD + n] : 0.f);
        tmem_st32(tm + lo + TM_S + f0, r);
      }
      tmem_wait_st();
    }
    fence_before();
    named_sync(BAR_STATE0, 32 + CH_THREADS);  // the state is in TMEM before the issuer starts any product
    bool ok = true;
    for (int ch = 0; ch < nch; ++ch) {
      const uint32_t D = TM_D0 + (ch & 1) * 128, Dp = TM_D0 + ((ch + 1) & 1) * 128;
      const uint32_t par = ch & 1;
      // Z^T = V^T - Y^T (rounded to tf32) over Y^T
      if (!(ok = role_wait(bars + B_V, par, polls, abort, 1, CH_THREADS))) break;
      if (!(ok = role_wait(bars + B_M1, par, polls, abort, 1, CH_THREADS))) break;
      fence_after();
      {
        float y[32];
        uint32_t z[32];
        tmem_ld32(tm + lo + D + hc * 32, y);
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = tf32_rna(ldb(sm + S2_V, hc * 32 + j, n) - y[j]);
        tmem_st32(tm + lo + D + hc * 32, z);
      }
      tmem_wait_st();
      fence_before();
      mbar_arrive(bars + B_Z);
      // M^T <- M^T diag(e^{c_last}), storing the entering state for the backward
      if (!(ok = role_wait(bars + B_KD, par, polls, abort, 1, CH_THREADS))) break;
      {
        float* slot = a.states ? a.states + state_slot(a, sq, hv, c0 + ch) * (KD * VD) : nullptr;
        const float* el = sEl + hc * 64;
#pragma unroll 1
        for (int cb = 0; cb < 2; ++cb) {
          float sv[32];
          uint32_t r[32];
          tmem_ld32(tm + lo + TM_S + hc * 64 + cb * 32, sv);
          if (slot) store_slot32(slot, hc * 2 + cb, n, sv);
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(sv[j] * el[cb * 32 + j]);
          tmem_st32(tm + lo + TM_S + hc * 64 + cb * 32, r);
        }
      }
      // U^T rounded to tf32
      if (!(ok = role_wait(bars + B_M2, par, polls, abort, 1, CH_THREADS))) break;
      fence_after();
      {
        float u[32];
        uint32_t r[32];
        tmem_ld32(tm + lo + TM_U + hc * 32, u);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = tf32_rna(u[j]);
        tmem_st32(tm + lo + TM_U + hc * 32, r);
      }
      tmem_wait_st();
      fence_before();
      mbar_arrive(bars + B_UR);
      // the previous chunk's output rows (its products ended before this chunk's U^T was formed)
      if (ch > 0) {
        if (!(ok = role_wait(bars + B_M4, par ^ 1, polls, abort, 1, CH_THREADS))) break;
        fence_after();
        out_rows(ch - 1, Dp);
      }
    }
    if (ok && nch > 0) {  // the last chunk: its output products, then its rows and the final state
      if ((ok = role_wait(bars + B_M4, (nch - 1) & 1, polls, abort, 1, CH_THREADS))) {
        fence_after();
        out_rows(nch - 1, TM_D0 + ((nch - 1) & 1) * 128);
      }
    }
    if (ok && a.S_T) {
      fence_after();
      for (int cb = 0; cb < 2; ++cb) {
        const int f0 = hc * 64 + cb * 32;
        float sv[32];
        tmem_ld32(tm + lo + TM_S + f0, sv);
#pragma unroll
        for (int j = 0; j < 32; ++j) a.S_T[(head * KD + f0 + j) * VD + n] = sv[j];
      }
    }
  } else {
    // ======================================================================== builder warps
    const int bt = tid - BU0;  // 0 .. 255
    const SyncNamed bsync{2, BU_THREADS};
    float* sNq = reinterpret_cast<float*>(sm + S2_NQ);
    float* sNk = reinterpret_cast<float*>(sm + S2_NK);
    const auto issue_raw = [&](int ch) {
      issue_qkg(maps, sb + S2_Q, sb + S2_K, sb + S2_C, bars + B_RAW, b, span(ch).x, h, hv);
      ++cnt[B_RAW];
    };
    if (nch > 0 && bt == 0) {
      issue_raw(0);
      if (nch > 1) {
        prefetch_qkg(maps, b, span(1).x, h, hv);
        tma_prefetch_4d(&maps.v, 0, hv, span(1).x, b);
        tma_prefetch_4d(&maps.v, 64, hv, span(1).x, b);
      }
    }
    const int rl = bt & 7, fg = bt >> 3, f = 4 * fg;  // rows 8 m + rl, channels f .. f + 3
    for (int ch = 0; ch < nch; ++ch) {
      const int2 sp = span(ch);
      if (!role_wait(bars + B_RAW, ch & 1, polls, abort, 2, BU_THREADS)) break;
      prep_tile<PREP>(sm + S2_Q, sm + S2_K, sm + S2_C, sNq, sNk, bt, sp.y, a.scale, bsync);
      cumsum_tile<false>(sm + S2_C, reinterpret_cast<float*>(sm + S2_CARRY), bt, bsync);
      // [K o e^c ; Q~ o e^c]: its slot is free once the previous chunk's first products are done
      if (ch > 0 && !role_wait(bars + B_M1, (ch - 1) & 1, polls, abort, 2, BU_THREADS)) break;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int i = 8 * m + rl;
        const float4 c4 = ld4f(sm + S2_C, i, f);
        float kf[4], qf[4];
        bf16x4(sm + S2_K + bt_off(i, f), kf);
        bf16x4(sm + S2_Q + bt_off(i, f), qf);
        const float qm = PREP ? sNq[i] : a.scale, km = PREP ? sNk[i] : 1.f;
        const float e[4] = {ex2(c4.x), ex2(c4.y), ex2(c4.z), ex2(c4.w)};
        st_tf32x4(sm, S2_KQ + kmaj(i, f, 128), km * kf[0] * e[0], km * kf[1] * e[1], km * kf[2] * e[2],
                  km * kf[3] * e[3]);
        st_tf32x4(sm, S2_KQ + kmaj(64 + i, f, 128), qm * qf[0] * e[0], qm * qf[1] * e[1], qm * qf[2] * e[2],
                  qm * qf[3] * e[3]);
      }
      fence_async_smem();
      mbar_arrive(bars + B_KQ);
      // K o e^{c_last - c} and e^{c_last}: free once the previous chunk's state products are done
      if (ch > 0 && !role_wait(bars + B_M3, (ch - 1) & 1, polls, abort, 2, BU_THREADS)) break;
      {  // one channel and four consecutive rows per 16-byte piece: lanes hold consecutive channels
        const int fc = bt & 127;
        const float c63 = ldf(sm + S2_C, 63, fc);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int i0 = ((bt >> 7) + 2 * m) * 4;
          float ked[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            const float km = PREP ? sNk[i] : 1.f;
            ked[u] = km * ldb(sm + S2_K, i, fc) * ex2(c63 - ldf(sm + S2_C, i, fc));
          }
          st_tf32x4(sm, S2_KD + kmaj(fc, i0, 64), ked[0], ked[1], ked[2], ked[3]);
        }
        if (bt < KD) sEl[bt] = ex2(c63);
      }
      fence_async_smem();
      mbar_arrive(bars + B_KD);
      bsync();  // every builder is done with this chunk's raw rows
      if (bt == 0 && ch + 1 < nch) {
        issue_raw(ch + 1);
        if (ch + 2 < nch) {
          prefetch_qkg(maps, b, span(ch + 2).x, h, hv);
          tma_prefetch_4d(&maps.v, 0, hv, span(ch + 2).x, b);
          tma_prefetch_4d(&maps.v, 64, hv, span(ch + 2).x, b);
          prefetch_l2(rec(ch + 2), FWI_BYTES);
        }
      }
    }
  }

  __syncthreads();
  if (*abort && tid == 0) {  // let every issued copy and product finish before the shared and tensor memory go
    for (int i = 0; i < NB_ASYNC; ++i)
      if (cnt[i] > 0) tc::mbar_wait_lim(bars + i, (cnt[i] - 1) & 1, DEFAULT_WAIT_POLLS);
  }
  fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
  if (*abort && tid == 0) atomicOr(&g_kda_fwd_chunked_error, 1u);
}

}  // namespace fc

// ---------------------------------------------------------------------------- host side

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 4-D map of [rows, T, heads, 128] (innermost last), box (box0 channels, one
// head, 64 steps, one row), 128-byte swizzle, zero fill past the tensor.
int head_map(CUtensorMap* m, const void* base, bool bf16, int rows, int T, int heads, int box0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return set_error(KDA_ERR_CUDA, "kda_fwd: the driver does not provide cuTensorMapEncodeTiled");
  const cuuint64_t es = bf16 ? 2 : 4;
  const cuuint64_t dims[4] = {128, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)rows};
  const cuuint64_t strides[3] = {128 * es, (cuuint64_t)heads * 128 * es, (cuuint64_t)T * heads * 128 * es};
  const cuuint32_t box[4] = {(cuuint32_t)box0, 1, 64, 1}, estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(KDA_ERR_CUDA, "kda_fwd: cuTensorMapEncodeTiled failed");
  return 0;
}

template <bool PREP>
int launch_t(const FwdArgs& a, cudaStream_t stream) {
  using namespace fc;
  FwdMaps m;
  const int rows = a.ctab ? 1 : a.B;
  int rc = head_map(&m.q, a.q, true, rows, a.T, a.H, 64);
  if (!rc) rc = head_map(&m.k, a.k, true, rows, a.T, a.H, 64);
  if (!rc) rc = head_map(&m.v, a.v, true, rows, a.T, a.HV, 64);
  if (!rc) rc = head_map(&m.g, a.g, false, rows, a.T, a.HV, 32);
  if (rc) return rc;
  cudaError_t e = cudaFuncSetAttribute(kda_fwd_intra_tc_kernel<PREP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)K1_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kda_fwd_state_tc_kernel<PREP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)S2_BYTES);
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: cudaFuncSetAttribute", e);
  const int items = a.ctab ? a.NC * a.HV : (a.T + C - 1) / C * a.HV * a.B;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (items > 0) {  // (packed batches of empty sequences have no chunks)
    kda_fwd_intra_tc_kernel<PREP><<<min(items, 2 * sms), NTH, K1_BYTES, stream>>>(m, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("kda_fwd: chunk-parallel launch", e);
  }
  kda_fwd_state_tc_kernel<PREP><<<dim3(a.HV, a.B), K2_THREADS, S2_BYTES, stream>>>(m, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_fwd: state-pass launch", e);
  return 0;
}
}  // namespace

int make_raw_maps(RawMaps* m, const void* q, const void* k, const void* x, const float* g, const void* v, int rows,
                  int T, int H, int HV) {
  static_assert(sizeof(CUtensorMap) == 128 && alignof(CUtensorMap) <= 64, "tensor map size");
  int rc = head_map(reinterpret_cast<CUtensorMap*>(m->q), q, true, rows, T, H, 64);
  if (!rc) rc = head_map(reinterpret_cast<CUtensorMap*>(m->k), k, true, rows, T, H, 64);
  if (!rc) rc = head_map(reinterpret_cast<CUtensorMap*>(m->x), x, true, rows, T, HV, 64);
  if (!rc) rc = head_map(reinterpret_cast<CUtensorMap*>(m->g), g, false, rows, T, HV, 32);
  if (!rc && v) rc = head_map(reinterpret_cast<CUtensorMap*>(m->v), v, true, rows, T, HV, 64);
  return rc;
}

// The gate of the fused preparation ("kimi_k3_host/kda.rs", bounded_gate):
// g[r][hv][f] = gate(z[r][hv][f] + dt_bias[hv][f]) with e^{A_log[hv]}, eight
// channels (one 16-byte piece of z) per thread.
__global__ void __launch_bounds__(256) kda_prep_gate_kernel(const __nv_bfloat16* __restrict__ z,
                                                             const float* __restrict__ A_log,
                                                             const float* __restrict__ dt_bias, float lb,
                                                             float* __restrict__ g, size_t pieces, int HV) {
  const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= pieces) return;
  const int hv = (int)((x >> 4) % HV), f0 = (int)(x & 15) * 8;  // 16 pieces of 8 channels per (row, hv)
  const uint4 zr = reinterpret_cast<const uint4*>(z)[x];
  const __nv_bfloat16* zb = reinterpret_cast<const __nv_bfloat16*>(&zr);
  const float dec = expf(A_log[hv]);
  float o[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) o[u] = prep_gate_fast(__bfloat162float(zb[u]) + dt_bias[hv * 128 + f0 + u], dec, lb);
  float4* dst = reinterpret_cast<float4*>(g + x * 8);
  dst[0] = make_float4(o[0], o[1], o[2], o[3]);
  dst[1] = make_float4(o[4], o[5], o[6], o[7]);
}

int launch_prep_gate(const void* z, const float* A_log, const float* dt_bias, float lb, float* g, size_t rows, int HV,
                     cudaStream_t stream) {
  const size_t pieces = rows * (size_t)HV * 16;  // K = 128
  if (pieces == 0) return 0;
  kda_prep_gate_kernel<<<(unsigned)((pieces + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(z), A_log, dt_bias, lb, g, pieces, HV);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_fwd_prep: gate launch", e);
  return 0;
}

int launch_fwd_chunked(const FwdArgs& a, cudaStream_t stream) {
  return a.prep.z ? launch_t<true>(a, stream) : launch_t<false>(a, stream);
}

int set_wait_polls(unsigned polls) {
  const unsigned v = polls ? polls : DEFAULT_WAIT_POLLS;
  const cudaError_t e = cudaMemcpyToSymbol(g_kda_wait_polls, &v, sizeof(v));
  if (e != cudaSuccess) return set_cuda_error("kda_set_wait_polls", e);
  return 0;
}

int take_fwd_chunked_error(unsigned* out) {
  unsigned v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_kda_fwd_chunked_error, sizeof(v));
  if (e != cudaSuccess) return set_cuda_error("kda_device_status", e);
  e = cudaMemcpyToSymbol(g_kda_fwd_chunked_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return set_cuda_error("kda_device_status", e);
  *out = v;
  return 0;
}

}  // namespace kda
