// Per-chunk building blocks shared by the tensor-core KDA kernels (K = V =
// 128, chunk C = 64, bf16 q/k/v/dO, fp32 g/beta): loading a chunk, the
// in-chunk cumulative decay, the interaction products Ah and P on the tensor
// cores, and their read-out for the triangular solve.
//
// Chunk algebra ("research_layers.py", delta_recurrence, erase = write = k,
// beta folded into the residual): with c_i = sum_{s<=i} g_s inside the chunk,
//   Ah[i][j] = sum_f k_if k_jf exp(c_if - c_jf)   (j < i)
//   P [i][j] = sum_f q~_if k_jf exp(c_if - c_jf)  (j <= i),  q~ = scale q.
// Both come out of two tf32 products of split-exponent operands:
//   product a: [K o x; Q~ o x] (K o y)^T with x_i = e^{c_i - c_r}, y_j = e^{c_r - c_j}
//              and r the middle row (15 or 47) of the 32-row half holding i and j;
//              it gives the two diagonal 32 x 32 blocks;
//   product b: rows i >= 32 against columns j < 32 with r = 31 (both factors <= 1).
// When the decay from a half's middle row to either end exceeds 80 (only an
// unbounded gate can do that) the same-half entries are formed pair by pair.
//
// Shared-memory map (bytes):
//   [0, 82944)       raw chunk: q, k, a third bf16 row tensor (v or dO), and the
//                    cumulative decay c (log2 units, row stride LDCF floats);
//                    reused after the raw data is consumed for Ah, T, P and W
//   [82944, 230400)  operand region: the interaction operands, then the
//                    kernel's own product operands
//   [230400, ...)    beta, per-channel decay constants, barrier, TMEM base
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_chunk.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace tcc {

constexpr int C = 64, KD = 128, VD = 128, NTH = 256;
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_X = 32768, RAW_C = 49152;
constexpr int LDCF = 132;
constexpr uint32_t R_AH = 0, R_TROW = 16640, R_SW = 33280, R_P = 37888, R_T = 54272, R_WOP = 0;
constexpr uint32_t OP = 82944;
constexpr uint32_t OP_XA = OP, OP_YA = OP + 65536, OP_XB = OP + 98304, OP_YB = OP + 131072;
constexpr uint32_t SMALL = OP + 147456;
constexpr uint32_t S_BETA = SMALL, S_EL = SMALL + 256, S_EMID = S_EL + 512, S_CARRY = S_EMID + 512,
                   S_BAR = S_CARRY + 512, S_TMEM = S_BAR + 8, SMEM_BYTES = S_TMEM + 16;
constexpr float LOG2E = 1.4426950408889634f;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(R_T + 16384 <= OP && R_P + 16384 <= R_T && R_SW + 3072 <= R_P && R_WOP + 36864 <= R_P,
              "raw-region reuse (the padded W overlaps only the dead inverse scratch)");

// A K x V state (or state gradient) slot of the tensor-core path, in its 64 KB
// fp32 slot of the state layout: the values [f][n] as fp16 (32 KB), then one
// power-of-two scale per value column n and group of 32 key channels
// ([4][128] floats at float offset SLOT_SCALES): x = half(x / s) * s.  The
// scale puts the group's largest magnitude in [2^14, 2^15), so every value
// keeps fp16's 11 significant bits (what the tf32 products read anyway:
// 10 stored mantissa bits) whatever the state's range; values below 2^-29 of
// the group's largest lose bits.  Half the bytes of the fp32 slot.
constexpr int SLOT_SCALES = KD * VD / 2;
// one thread's 32 values of column n, channels 32 grp .. 32 grp + 31
__device__ __forceinline__ void store_slot32(float* slot, int grp, int n, const float (&v)[32]) {
  float m = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
  // m < 2^ex (ex from the exponent field; 0 and subnormal m give the clamp)
  const int ex = ((__float_as_int(m) >> 23) & 0xff) - 126;
  const int e = min(126, max(-126, 15 - ex));
  const float up = __int_as_float((127 + e) << 23);
  __half* h = reinterpret_cast<__half*>(slot) + (size_t)(32 * grp) * VD + n;
#pragma unroll
  for (int j = 0; j < 32; ++j) h[(size_t)j * VD] = __float2half_rn(v[j] * up);
  slot[SLOT_SCALES + grp * VD + n] = __int_as_float((127 - e) << 23);
}
__device__ __forceinline__ void load_slot32(const float* slot, int grp, int n, float (&v)[32]) {
  const __half* h = reinterpret_cast<const __half*>(slot) + (size_t)(32 * grp) * VD + n;
  const float s = slot[SLOT_SCALES + grp * VD + n];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __half2float(h[(size_t)j * VD]) * s;
}

// Byte offsets inside a raw tile of 64 rows x 128 channels as the 128-byte
// swizzle of TMA leaves it: bf16 as two 8 KB boxes of 64 channels, fp32 as
// four 8 KB boxes of 32 channels; the 16-byte pieces of row i are permuted
// by i % 8 (each box base 1024-byte aligned).
__device__ __forceinline__ uint32_t bt_off(int i, int f) {
  return (uint32_t)((f >> 6) * 8192 + i * 128 + ((((f & 63) >> 3) ^ (i & 7)) << 4) + (f & 7) * 2);
}
__device__ __forceinline__ uint32_t ft_off(int i, int f) {
  return (uint32_t)((f >> 5) * 8192 + i * 128 + ((((f & 31) >> 2) ^ (i & 7)) << 4) + (f & 3) * 4);
}
__device__ __forceinline__ float ldf(const unsigned char* t, int i, int f) {
  return *reinterpret_cast<const float*>(t + ft_off(i, f));
}
__device__ __forceinline__ float ldb(const unsigned char* t, int i, int f) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(t + bt_off(i, f)));
}

constexpr uint32_t TILE_BF16 = 16384, TILE_F32 = 32768;

// byte offset of bf16 element (row i, channel f) in a raw q / k / x tile:
// the 16-byte pieces of row i are stored XOR-swizzled by i % 8, so that one
// piece of 8 consecutive rows lies in 8 different bank groups
__device__ __forceinline__ uint32_t raw_off(int i, int f) {
  return (uint32_t)(i * 256 + ((f >> 3) ^ (i & 7)) * 16 + (f & 7) * 2);
}

struct Ctx {
  unsigned char* sm;
  uint32_t sb;      // shared address of sm
  uint32_t tm;      // TMEM base
  uint32_t lo;      // this warp's TMEM lane base (<< 16)
  int tid, warp, lane, sub, hcol, Lr;
  __device__ float* c() const { return reinterpret_cast<float*>(sm + RAW_C); }
  __device__ float* beta() const { return reinterpret_cast<float*>(sm + S_BETA); }
};

__device__ __forceinline__ void st_tf32x4(unsigned char* base, uint32_t off, float a, float b, float c, float d) {
  uint4 v = make_uint4(tc::tf32_rna(a), tc::tf32_rna(b), tc::tf32_rna(c), tc::tf32_rna(d));
  *reinterpret_cast<uint4*>(base + off) = v;
}
__device__ __forceinline__ void st_tf32(unsigned char* base, uint32_t off, float a) {
  *reinterpret_cast<uint32_t*>(base + off) = tc::tf32_rna(a);
}
__device__ __forceinline__ void bf16x4(const unsigned char* p, float (&o)[4]) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&r.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&r.y);
  o[0] = __low2float(lo); o[1] = __high2float(lo); o[2] = __low2float(hi); o[3] = __high2float(hi);
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// Asynchronous load of one chunk: q, k rows of query/key head h, x rows of
// value head hv (v or dO), g rows and beta; rows past the sequence end are
// zero.  Issues the copies only; load_raw_wait completes them.  (16-byte
// cp.async per thread: measured faster here than per-row bulk copies issued
// by one warp.)
// (ASYNC_BETA: beta also by cp.async, so that issuing the load never waits)
template <int NT = NTH, bool ASYNC_BETA = false>
__device__ __forceinline__ void load_raw_issue(const Ctx& c, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                               const __nv_bfloat16* x, const float* g, const float* beta,
                                               int b, int T, int t0, int L, int H, int HV, int h, int hv) {
  using namespace tc;
  for (int e = c.tid; e < C * 16; e += NT) {
    const int i = e >> 4, vec = e & 15;
    const bool ok = i < L;
    const size_t t = (size_t)b * T + t0 + (ok ? i : 0);  // row 0 of the chunk is always valid
    const uint32_t d = raw_off(i, vec * 8);
    cp_async16(c.sb + RAW_Q + d, q + (t * H + h) * KD + vec * 8, ok);
    cp_async16(c.sb + RAW_K + d, k + (t * H + h) * KD + vec * 8, ok);
    cp_async16(c.sb + RAW_X + d, x + (t * HV + hv) * VD + vec * 8, ok);
  }
  for (int e = c.tid; e < C * 32; e += NT) {
    const int i = e >> 5, vec = e & 31;
    const bool ok = i < L;
    const size_t t = (size_t)b * T + t0 + (ok ? i : 0);
    cp_async16(c.sb + RAW_C + (i * LDCF + vec * 4) * 4, g + (t * HV + hv) * KD + vec * 4, ok);
  }
  if (c.tid < C) {
    const bool ok = c.tid < L;
    const float* src = beta + ((size_t)b * T + t0 + (ok ? c.tid : 0)) * HV + hv;
    if constexpr (ASYNC_BETA) tc::cp_async4(c.sb + S_BETA + c.tid * 4, src, ok);
    else c.beta()[c.tid] = ok ? *src : 0.f;
  }
}
// The same load for the fused preparation: z (the gate pre-activation, bf16)
// instead of g, as packed rows at the stride of the cumulative-decay rows
// (row i at RAW_C + i * LDCF * 4, so that the per-row norms in the padding
// floats LDCF-4 .. of every row survive), and beta from its logit.
template <int NT = NTH>
__device__ __forceinline__ void load_raw_issue_prep(const Ctx& c, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                                    const __nv_bfloat16* x, const __nv_bfloat16* z,
                                                    const float* beta_logit, int b, int T, int t0, int L, int H,
                                                    int HV, int h, int hv) {
  using namespace tc;
  for (int e = c.tid; e < C * 16; e += NT) {
    const int i = e >> 4, vec = e & 15;
    const bool ok = i < L;
    const size_t t = (size_t)b * T + t0 + (ok ? i : 0);
    const uint32_t d = raw_off(i, vec * 8);
    cp_async16(c.sb + RAW_Q + d, q + (t * H + h) * KD + vec * 8, ok);
    cp_async16(c.sb + RAW_K + d, k + (t * H + h) * KD + vec * 8, ok);
    cp_async16(c.sb + RAW_X + d, x + (t * HV + hv) * VD + vec * 8, ok);
    cp_async16(c.sb + RAW_C + i * LDCF * 4 + vec * 16, z + (t * HV + hv) * KD + vec * 8, ok);
  }
  if (c.tid < C)
    c.beta()[c.tid] = (c.tid < L) ? prep_sigmoid_fast(beta_logit[((size_t)b * T + t0 + c.tid) * HV + hv]) : 0.f;
}

// Per-row factors of the fused preparation ("kimi_k3_host/kda.rs",
// l2norm_rows): scale / sqrt(|q_i|^2 + eps) and 1 / sqrt(|k_i|^2 + eps),
// kept in the padding floats 128 and 129 of row i of the cumulative-decay
// rows.  Run after load_raw_wait; cumsum_span's barriers publish them.
constexpr int NORM_Q = 128, NORM_K = 129;
template <int NT = NTH>
__device__ __forceinline__ void row_norms(const Ctx& c, float scale) {
  constexpr int P = NT / 128, PC = 16 / P;  // threads per row, 16-byte pieces per thread
  const int r = c.tid / P, part = c.tid % P, i = r & 63;
  const unsigned char* base = c.sm + (r < 64 ? RAW_Q : RAW_K);
  float s = 0.f;
#pragma unroll
  for (int pc = 0; pc < PC; ++pc) {
    float x[4];
    const int f = (part * PC + pc) * 8;
    bf16x4(base + raw_off(i, f), x);
    s = fmaf(x[0], x[0], fmaf(x[1], x[1], fmaf(x[2], x[2], fmaf(x[3], x[3], s))));
    bf16x4(base + raw_off(i, f) + 8, x);
    s = fmaf(x[0], x[0], fmaf(x[1], x[1], fmaf(x[2], x[2], fmaf(x[3], x[3], s))));
  }
#pragma unroll
  for (int off = 1; off < P; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (part == 0) c.c()[i * LDCF + (r < 64 ? NORM_Q : NORM_K)] = rsqrtf(s + KDA_L2_EPS_F) * (r < 64 ? scale : 1.f);
}

// Completes load_raw_issue (wait + barrier).  Returns true (the form of a
// bounded wait, for the callers' uniform error path).
__device__ __forceinline__ bool load_raw_wait(const Ctx&) {
  tc::cp_async_wait_all();
  __syncthreads();
  return true;
}

// L2 prefetch of one chunk's q, k, x (v or dO) and g rows, for a chunk that a
// later load_raw will read; one row of one tensor per thread.
// (g_elem: bytes per element of the gate rows, 4 for g or 2 for bf16 z)
__device__ __forceinline__ void prefetch_chunk(const Ctx& c, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                               const __nv_bfloat16* x, const void* g, int b, int T, int t0,
                                               int L, int H, int HV, int h, int hv, int g_elem = 4) {
  const int i = c.tid & 63, which = c.tid >> 6;
  if (i >= L || which > 3) return;
  const size_t t = (size_t)b * T + t0 + i;
  if (which == 0) tc::prefetch_l2(q + (t * H + h) * KD, KD * 2);
  else if (which == 1) tc::prefetch_l2(k + (t * H + h) * KD, KD * 2);
  else if (which == 2) tc::prefetch_l2(x + (t * HV + hv) * VD, VD * 2);
  else tc::prefetch_l2(static_cast<const unsigned char*>(g) + (t * HV + hv) * KD * g_elem, KD * g_elem);
}

// Asynchronous copy of one 64 x 64 operand image of an interaction record
// (16 KB) into shared memory at `dst`; completes with cp_async_wait_all.
template <int NT = NTH>
__device__ __forceinline__ void copy_image(const Ctx& c, uint32_t dst, const float* src) {
#pragma unroll
  for (int e = c.tid; e < 1024; e += NT) tc::cp_async16(c.sb + dst + e * 16, src + e * 4, true);
}

// Sums over the warp's 32 lanes of 32 values at once: lane l returns
// sum over lanes of v[l] (31 shuffles instead of 32 x 5).  v is clobbered.
__device__ __forceinline__ float warp_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < off; ++k) {
      const float send = up ? v[k] : v[k + off];
      const float keep = up ? v[k + off] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

// float index of element (r, k) in a 64 x 64 record image
__device__ __forceinline__ int img(int r, int k) { return (int)(tc::kmaj(r, k, 64) >> 2); }

// Output gate ("kimi_k3_host/kda.rs", full_rank_output_gate) on an O^T tile
// read out of TMEM: warp w holds rows 32 (w / 4) + jj, jj < 32, of the value
// columns 32 (w % 4) + lane.  Scales v[jj] by 1 / sqrt(mean_n o^2 + eps) of
// its row (the sigmoid factor is the caller's); `red` is 256 floats that
// nothing else touches until a later block barrier.  One block barrier
// (256 threads).
// (sync: the barrier of the 256 threads taking part)
template <class Sync>
__device__ __forceinline__ void out_gate_rows(float (&v)[32], float* red, int warp, int lane, float eps, Sync sync) {
  float sq[32];
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) sq[jj] = v[jj] * v[jj];
  const float part = warp_sum32(sq, lane);  // row 32 (warp / 4) + lane, this warp's 32 columns
  red[((warp >> 2) * 32 + lane) * 4 + (warp & 3)] = part;
  sync();
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) {
    const float4 r = *reinterpret_cast<const float4*>(red + ((warp >> 2) * 32 + jj) * 4);
    v[jj] *= rsqrtf((r.x + r.y + r.z + r.w) * (1.f / 128.f) + eps);
  }
}
__device__ __forceinline__ void out_gate_rows(float (&v)[32], float* red, int warp, int lane, float eps) {
  struct All {
    __device__ void operator()() const { __syncthreads(); }
  };
  out_gate_rows(v, red, warp, lane, eps, All());
}

// In-chunk cumulative decay (natural log summed, stored times log2(e)).
// Returns, block-uniformly, whether some half's decay from its middle row to
// either end exceeds 80 (the split exponents would then leave fp32 range).
// (The first 256 threads do the sums, two row halves per channel.)
// With GATE (fused preparation) the rows hold z (bf16, load_raw_issue_prep)
// and g = prep_gate(z + dt_bias) is formed here ("kimi_k3_host/kda.rs",
// bounded_gate); rows at or past L count as g = 0 as in the plain load.
// (GATE: dtb = dt_bias[hv][tid % 128], dec = e^{A_log[hv]}, both loaded by
// the caller ahead of the chunk's load wait, so that no global load sits on
// this critical path)
template <bool GATE = false, int NT = NTH>
__device__ __forceinline__ bool cumsum_span(const Ctx& c, float dtb = 0.f, float dec = 0.f, float lb = 0.f,
                                            int L = C) {
  float* sC = c.c();
  float* sCarry = reinterpret_cast<float*>(c.sm + S_CARRY);
  const int f = c.tid & 127, hh = c.tid >> 7;
  if constexpr (GATE) {  // all threads: z -> g in registers, then over z in place (fp32 rows)
    constexpr int PER = C * KD / NT;
    const __nv_bfloat16* zr = reinterpret_cast<const __nv_bfloat16*>(c.sm + RAW_C);
    float gv[PER];  // element e = tid + m NT has channel e % 128 = f
#pragma unroll
    for (int m = 0; m < PER; ++m) {
      const int i = (c.tid + m * NT) >> 7;
      gv[m] = i < L ? prep_gate_fast(__bfloat162float(zr[i * 2 * LDCF + f]) + dtb, dec, lb) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < PER; ++m) sC[((c.tid + m * NT) >> 7) * LDCF + f] = gv[m];
    __syncthreads();
  }
  float v[32];
  float run = 0.f;
  if (c.tid < 256) {
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      run += sC[(hh * 32 + r) * LDCF + f];
      v[r] = run;
    }
    if (hh == 0) sCarry[f] = run;
  }
  __syncthreads();
  if (c.tid < 256) {
    const float carry = hh ? sCarry[f] : 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) sC[(hh * 32 + r) * LDCF + f] = (v[r] + carry) * LOG2E;
  }
  __syncthreads();
  bool w = false;
  if (c.tid < KD) {
    const float lim = 80.f * LOG2E;
    const int t = c.tid;
    const float c0 = sC[t], c15 = sC[15 * LDCF + t], c31 = sC[31 * LDCF + t];
    const float c32 = sC[32 * LDCF + t], c47 = sC[47 * LDCF + t], c63 = sC[63 * LDCF + t];
    w = fabsf(c0 - c15) > lim || fabsf(c15 - c31) > lim || fabsf(c32 - c47) > lim || fabsf(c47 - c63) > lim;
  }
  return __syncthreads_or(w);
}

// Item mapping of the element-wise operand builders for NT threads (R = NT / 32
// rows per round): thread t owns key channels 4*((t/R)&31) .. +3 and rows
// m*R + t%R, m = 0 .. 64/R - 1 (eight consecutive lanes hold eight rows).
template <int NT = NTH>
__device__ __forceinline__ int item_f(const Ctx& c) { return ((c.tid / (NT / 32)) & 31) * 4; }
template <int NT = NTH>
__device__ __forceinline__ int item_row(const Ctx& c, int m) { return m * (NT / 32) + c.tid % (NT / 32); }

// Interaction operands into the operand region, then the two products on
// the tensor cores (issued by thread 0, completion on `bar`).
// (NORM: q, k rows times their row_norms factors; the q factor includes scale)
template <int NT = NTH, bool NORM = false>
__device__ __forceinline__ void build_op1_and_issue(const Ctx& c, float scale, uint32_t tm_apa,
                                                    uint32_t tm_apb, uint64_t* bar) {
  using namespace tc;
  const float* sC = c.c();
  const int fq = item_f<NT>(c);
  const float4 r15 = ld4(sC + 15 * LDCF + fq), r47 = ld4(sC + 47 * LDCF + fq), r31 = ld4(sC + 31 * LDCF + fq);
  const float c31[4] = {r31.x, r31.y, r31.z, r31.w};
  for (int m = 0; m < 2048 / NT; ++m) {
    const int i = item_row<NT>(c, m);
    const float4 c4 = ld4(sC + i * LDCF + fq);
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
    float kf[4], qf[4];
    bf16x4(c.sm + RAW_K + raw_off(i, fq), kf);
    bf16x4(c.sm + RAW_Q + raw_off(i, fq), qf);
    const float4 rr = (i < 32) ? r15 : r47;
    const float cr[4] = {rr.x, rr.y, rr.z, rr.w};
    const float qmul = NORM ? sC[i * LDCF + NORM_Q] : scale;
    float xa[4], ya[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      qf[u] *= qmul;
      if (NORM) kf[u] *= sC[i * LDCF + NORM_K];
      xa[u] = ex2(cc[u] - cr[u]);
      ya[u] = ex2(cr[u] - cc[u]);
    }
    st_tf32x4(c.sm, OP_XA + kmaj(i, fq, 128), kf[0] * xa[0], kf[1] * xa[1], kf[2] * xa[2], kf[3] * xa[3]);
    st_tf32x4(c.sm, OP_XA + kmaj(64 + i, fq, 128), qf[0] * xa[0], qf[1] * xa[1], qf[2] * xa[2], qf[3] * xa[3]);
    st_tf32x4(c.sm, OP_YA + kmaj(i, fq, 128), kf[0] * ya[0], kf[1] * ya[1], kf[2] * ya[2], kf[3] * ya[3]);
    if (i >= 32) {
      float xb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) xb[u] = ex2(cc[u] - c31[u]);
      st_tf32x4(c.sm, OP_XB + kmaj(i - 32, fq, 128), kf[0] * xb[0], kf[1] * xb[1], kf[2] * xb[2], kf[3] * xb[3]);
      st_tf32x4(c.sm, OP_XB + kmaj(i, fq, 128), qf[0] * xb[0], qf[1] * xb[1], qf[2] * xb[2], qf[3] * xb[3]);
    } else {
      float yb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) yb[u] = ex2(c31[u] - cc[u]);
      st_tf32x4(c.sm, OP_YB + kmaj(i, fq, 128), kf[0] * yb[0], kf[1] * yb[1], kf[2] * yb[2], kf[3] * yb[3]);
    }
  }
  fence_async_smem();
  __syncthreads();
  if (c.tid == 0) {
    fence_after();
    const uint32_t idA = idesc_tf32(128, 64), idB = idesc_tf32(64, 32);
    for (int ks = 0; ks < 16; ++ks)
      mma_ss(tm_apa, desc(c.sb + OP_XA + ks * 256, 4096), desc(c.sb + OP_YA + ks * 256, 4096), idA, ks > 0);
    for (int ks = 0; ks < 16; ++ks)
      mma_ss(tm_apb, desc(c.sb + OP_XB + ks * 256, 4096), desc(c.sb + OP_YB + ks * 256, 4096), idB, ks > 0);
    commit(bar);
  }
}

// Waits for the tensor-core work committed to `bar` (phase parity toggled
// here).  Returns false, block-uniformly, if the bounded wait ran out.
__device__ __forceinline__ bool wait_mma(uint64_t* bar, uint32_t& phase) {
  const bool ok = tc::mbar_wait(bar, phase);
  phase ^= 1;
  const bool bad = __syncthreads_or(!ok);
  tc::fence_after();
  return !bad;
}

// Same-half Ah/P entries pair by pair (only when cumsum_span said so); must
// run while the raw chunk is still in shared memory.
struct Pairwise {
  float v[16];
  int kind, i, j0;
};
template <bool NORM = false>
__device__ __forceinline__ void pairwise_compute(const Ctx& c, float scale, Pairwise& pw) {
  const float* sC = c.c();
  pw.kind = c.tid < 256 ? c.tid >> 7 : -1;  // the first 256 threads
  if (pw.kind < 0) {
    pw.i = pw.j0 = 0;
    return;
  }
  pw.i = (c.tid >> 1) & 63;
  pw.j0 = (pw.i & 32) + (c.tid & 1) * 16;
  const unsigned char* xi = c.sm + (pw.kind ? RAW_Q : RAW_K);
  for (int jj = 0; jj < 16; ++jj) {
    const int j = pw.j0 + jj;
    float acc = 0.f;
    if (pw.kind ? (j <= pw.i) : (j < pw.i)) {
      for (int f = 0; f < KD; ++f) {
        const float xv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(xi + raw_off(pw.i, f)));
        const float kj = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(c.sm + RAW_K + raw_off(j, f)));
        acc = fmaf(xv * kj, tc::ex2(sC[pw.i * LDCF + f] - sC[j * LDCF + f]), acc);
      }
      if (NORM)
        acc *= sC[pw.i * LDCF + (pw.kind ? NORM_Q : NORM_K)] * sC[j * LDCF + NORM_K];
      else if (pw.kind)
        acc *= scale;
    }
    pw.v[jj] = acc;
  }
}

// byte offset of P[i][j] in its operand tile (rows i, K = j)
__device__ __forceinline__ uint32_t p_off(int i, int j, uint32_t base = R_P) { return base + tc::kmaj(i, j, 64); }

// Reads Ah (row-major, stride 65, at R_AH) and P (tf32 operand at R_P) out of
// the two interaction products; the raw region must be free.  With `pt` it
// also stores the P^T image of the interaction record.  Ends with a barrier.
// (p_base: shared-memory byte offset of the P image, R_P by default)
template <int NT = NTH>
__device__ __forceinline__ void readout_ap(const Ctx& c, uint32_t tm_apa, uint32_t tm_apb, bool wide,
                                           const Pairwise& pw, float* pt = nullptr, uint32_t p_base = R_P) {
  using namespace tc;
  constexpr int CW = 64 / (NT / 128), CB = 32 / (NT / 128);  // columns per warp group of [Ah; P], of b
  float* sAh = reinterpret_cast<float*>(c.sm + R_AH);
  {
    float v[CW];
    tmem_ldn<CW>(tm_apa + c.lo + c.hcol * CW, v);
    const bool isA = c.Lr < 64;
    const int i = isA ? c.Lr : c.Lr - 64;
    if (isA) {
#pragma unroll
      for (int jj = 0; jj < CW; ++jj) {
        const int j = c.hcol * CW + jj;
        const bool same = (i >> 5) == (j >> 5);
        if (!same && i >= 32) continue;  // lower-left block comes from product b
        sAh[i * 65 + j] = (same && j < i) ? v[jj] : 0.f;
      }
    } else {  // P rows: four columns per 16-byte store
#pragma unroll
      for (int j4 = 0; j4 < CW; j4 += 4) {
        const int jb = c.hcol * CW + j4;
        if (i >= 32 && jb < 32) continue;  // lower-left block comes from product b
        float w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = jb + u;
          w[u] = ((i >> 5) == (j >> 5) && j <= i) ? v[j4 + u] : 0.f;
          if (pt) pt[img(j, i)] = __uint_as_float(tf32_rna(w[u]));
        }
        st_tf32x4(c.sm, p_off(i, jb, p_base), w[0], w[1], w[2], w[3]);
      }
    }
  }
  {
    float v[CB];
    tmem_ldn<CB>(tm_apb + c.lo + c.hcol * CB, v);
    if (c.lane < 16) {
      const int r = c.sub * 16 + c.lane;  // row of the 64-row product (M = 64 accumulator layout)
      if (r < 32) {
#pragma unroll
        for (int jj = 0; jj < CB; ++jj) sAh[(32 + r) * 65 + c.hcol * CB + jj] = v[jj];
      } else {
#pragma unroll
        for (int j4 = 0; j4 < CB; j4 += 4) {
          const int j = c.hcol * CB + j4;
          st_tf32x4(c.sm, p_off(r, j, p_base), v[j4], v[j4 + 1], v[j4 + 2], v[j4 + 3]);
          if (pt)
#pragma unroll
            for (int u = 0; u < 4; ++u) pt[img(j + u, r)] = __uint_as_float(tf32_rna(v[j4 + u]));
        }
      }
    }
  }
  __syncthreads();
  if (wide) {
    for (int jj = 0; jj < 16; ++jj) {
      const int j = pw.j0 + jj;
      if (pw.kind == 0 && j < pw.i) sAh[pw.i * 65 + j] = pw.v[jj];
      if (pw.kind == 1 && j <= pw.i) {
        st_tf32(c.sm, p_off(pw.i, j, p_base), pw.v[jj]);
        if (pt) pt[img(j, pw.i)] = __uint_as_float(tf32_rna(pw.v[jj]));
      }
    }
    __syncthreads();
  }
}

// T = (I + diag(beta) Ah)^-1 for the 64 x 64 unit lower-triangular system,
// row-major at R_TROW (stride 65).  The four 16 x 16 diagonal blocks are
// solved by forward substitution with a whole column per thread in
// registers; the blocks below follow in three levels of block substitution,
// T_IJ = -T_II sum_{J<=L<I} A_IL T_LJ (level = block distance I - J), one
// warp per block, as tf32 warp MMAs.  (T enters the state products as a tf32
// operand anyway; with single products here the o error stays ~0.5e-3 above
// the bf16 rounding floor, and hi/lo-split products cost 0.06 ms more per
// forward on the fwd+bwd workload.)
// (beta: the chunk's 64 beta values in shared memory, c.beta() by default)
template <int NT = NTH>
__device__ __forceinline__ void invert(const Ctx& c, const float* beta = nullptr) {
  constexpr int LD = 65;
  const float* sAh = reinterpret_cast<const float*>(c.sm + R_AH);
  float* sT = reinterpret_cast<float*>(c.sm + R_TROW);
  float* sW = reinterpret_cast<float*>(c.sm + R_SW);  // one 16 x 16 scratch per warp (3 warps)
  const float* sB = beta ? beta : c.beta();
  const int tid = c.tid;
  for (int x = tid; x < 6 * 256; x += NT) {  // strictly upper blocks
    const int blk = x >> 8, r = (x >> 4) & 15, col = x & 15;
    const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2), J = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
    sT[(16 * I + r) * LD + 16 * J + col] = 0.f;
  }
  if (tid < 64) {
    const int o = (tid >> 4) * 16, col = tid & 15;
    float t[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int m = 0; m < r; ++m) {
        if (m & 1) a1 = fmaf(sAh[(o + r) * LD + o + m], t[m], a1);
        else a0 = fmaf(sAh[(o + r) * LD + o + m], t[m], a0);
      }
      t[r] = (r == col) ? 1.f : (r > col ? -sB[o + r] * (a0 + a1) : 0.f);
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) sT[(o + r) * LD + o + col] = t[r];
  }
  __syncthreads();
  const int warp = c.warp, g = c.lane >> 2, t4 = c.lane & 3;
  for (int d = 1; d < 4; ++d) {
    if (warp < 4 - d) {
      const int J = warp, I = J + d, ri = 16 * I;
      // W = sum_{L=J}^{I-1} diag(beta_I) Ah_IL T_LJ  (16 x 16, K = 16 d)
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const float bg = sB[ri + g], bg8 = sB[ri + g + 8];
      for (int ks = 0; ks < 2 * d; ++ks) {
        const int l = 16 * J + 8 * ks + t4;
        const uint32_t a[4] = {to_tf32(bg * sAh[(ri + g) * LD + l]), to_tf32(bg8 * sAh[(ri + g + 8) * LD + l]),
                               to_tf32(bg * sAh[(ri + g) * LD + l + 4]),
                               to_tf32(bg8 * sAh[(ri + g + 8) * LD + l + 4])};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint32_t bb[2] = {to_tf32(sT[l * LD + 16 * J + nt * 8 + g]),
                                  to_tf32(sT[(l + 4) * LD + 16 * J + nt * 8 + g])};
          mma_16x8x8(acc[nt], a, bb);
        }
      }
      float* w = sW + warp * 256;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) w[(g + ((e & 2) ? 8 : 0)) * 16 + nt * 8 + 2 * t4 + (e & 1)] = acc[nt][e];
      __syncwarp();
      // T_IJ = -T_II W
      float tt[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const int m = 8 * ks + t4;
        const uint32_t a[4] = {to_tf32(sT[(ri + g) * LD + ri + m]), to_tf32(sT[(ri + g + 8) * LD + ri + m]),
                               to_tf32(sT[(ri + g) * LD + ri + m + 4]),
                               to_tf32(sT[(ri + g + 8) * LD + ri + m + 4])};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint32_t bb[2] = {to_tf32(w[m * 16 + nt * 8 + g]), to_tf32(w[(m + 4) * 16 + nt * 8 + g])};
          mma_16x8x8(tt[nt], a, bb);
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sT[(ri + g + ((e & 2) ? 8 : 0)) * LD + 16 * J + nt * 8 + 2 * t4 + (e & 1)] = -tt[nt][e];
    }
    __syncthreads();
  }
}

}  // namespace tcc
}  // namespace kda
