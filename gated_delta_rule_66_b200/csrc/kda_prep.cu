// The preparation around the KDA recurrence ("kimi_k3_host/kda.rs"):
//
//  * kda_decode_token_kernel: one decode token from the raw projections
//    (kda_decode_token): the short-convolution step of the token's q | k | v
//    channels (conv_update: window shift, weighted sum, SiLU), the L2
//    normalisation of q and k (l2norm_rows), the decay gate from its
//    pre-activation (bounded_gate), beta from its logit, the recurrence step
//    on the state in place (kda_recurrent_step) and the optional output gate
//    (full_rank_output_gate), all in one launch.
//  * kda_short_conv_kernel: the same convolution over whole sequences for the
//    prefill (conv_update applied to every step in order), one thread per
//    channel and block of steps with the window in registers; it writes the
//    convolved q, k, v in the input dtype and the final window.
//
// Decode layout as in kda_decode.cu: one CTA per (b, hv), 8 warps; a warp
// owns K/8 state rows, a lane 4 consecutive columns of RPI = 128 / V rows.
#include "kda_chunk.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int CONV_MAX_W = 8;

// One channel's convolution step on a window of W <= CONV_MAX_W inputs held
// in registers (oldest first): shift in x, return SiLU(sum_j w[j] win[j]).
// The loops are unrolled over CONV_MAX_W with predicates, so the window
// never goes to local memory.
__device__ __forceinline__ float conv_step(float (&win)[CONV_MAX_W], const float (&w)[CONV_MAX_W], float x, int W) {
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < CONV_MAX_W; ++j) {
    if (j < W) {
      win[j] = j + 1 < W ? win[j + 1] : x;
      acc = fmaf(w[j], win[j], acc);
    }
  }
  return acc * prep_sigmoid(acc);
}

template <int K, int V, typename TIn>
__global__ void __launch_bounds__(256) kda_decode_token_kernel(DecodeTokenArgs a) {
  constexpr int NW = 8, LPR = V / 4, RPI = 32 / LPR, RPW = K / NW, IT = RPW / RPI;
  static_assert(RPW % RPI == 0, "rows per warp must cover the lanes");
  __shared__ float sK[K], sQ[K], sDec[K], sV[V], sDelta[V], sO[V], sRk[NW][V], sRq[NW][V];
  __shared__ float sNorm[2], sQK, sRms;

  const int hv = blockIdx.x, b = blockIdx.y;
  const int G = a.HV / a.H, h = hv / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c4 = lane % LPR, rsub = lane / LPR;
  float4* S4 = reinterpret_cast<float4*>(a.S + ((size_t)b * a.HV + hv) * K * V);

  float4 s[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int row = warp * RPW + it * RPI + rsub;
    s[it] = __ldcs(S4 + row * LPR + c4);
  }

  // ---- every other global load of the CTA is issued here, next to the state
  // loads, so that their latencies overlap: this thread's (at most two)
  // channels of the convolution (input, window, weights), its gate channel,
  // the beta logit and its output-gate column.
  constexpr int NCH = 2 * K + V, PER = (NCH + 255) / 256;
  const size_t Cn = (size_t)2 * a.H * K + (size_t)a.HV * V;
  const float* win_in = a.conv_in ? a.conv_in + (size_t)b * Cn * a.W : nullptr;  // null: zero window
  float* win_out = a.conv_out + (size_t)b * Cn * a.W;
  float xin[PER], win[PER][CONV_MAX_W], wt[PER][CONV_MAX_W];
  size_t chan[PER];
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    const int e = threadIdx.x + 256 * p;
    size_t ch = 0;
    float x = 0.f;
    if (e < K) {
      ch = (size_t)h * K + e;
      x = to_f(static_cast<const TIn*>(a.xq)[((size_t)b * a.H + h) * K + e]);
    } else if (e < 2 * K) {
      ch = (size_t)a.H * K + (size_t)h * K + (e - K);
      x = to_f(static_cast<const TIn*>(a.xk)[((size_t)b * a.H + h) * K + e - K]);
    } else if (e < NCH) {
      ch = (size_t)2 * a.H * K + (size_t)hv * V + (e - 2 * K);
      x = to_f(static_cast<const TIn*>(a.xv)[((size_t)b * a.HV + hv) * V + e - 2 * K]);
    }
    chan[p] = ch;
    xin[p] = x;
#pragma unroll
    for (int j = 0; j < CONV_MAX_W; ++j) {
      const bool ok = e < NCH && j < a.W;
      win[p][j] = (ok && win_in) ? win_in[ch * a.W + j] : 0.f;
      wt[p][j] = ok ? a.conv_w[ch * a.W + j] : 0.f;
    }
  }
  const int fz = threadIdx.x < K ? threadIdx.x : 0;
  const float zf = to_f(static_cast<const TIn*>(a.prep.z)[((size_t)b * a.HV + hv) * K + fz]);
  const float dtb = a.prep.dt_bias[(size_t)hv * K + fz];
  const float alog = a.prep.A_log[hv];
  const float blog = a.beta[(size_t)b * a.HV + hv];
  const int nog = threadIdx.x < V ? threadIdx.x : 0;
  const float ogv = a.og ? to_f(static_cast<const TIn*>(a.og)[((size_t)b * a.HV + hv) * V + nog]) : 0.f;

  // ---- convolution step of this head's channels: q (K), k (K), v (V)
  const bool own_qk = hv % G == 0;  // one value head of the group writes the shared q/k windows
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    const int e = threadIdx.x + 256 * p;
    if (e >= NCH) continue;
    const float y = conv_step(win[p], wt[p], xin[p], a.W);
    if (e >= 2 * K || own_qk)
#pragma unroll
      for (int j = 0; j < CONV_MAX_W; ++j)
        if (j < a.W) win_out[chan[p] * a.W + j] = win[p][j];
    if (e < K) sQ[e] = y;
    else if (e < 2 * K) sK[e - K] = y;
    else sV[e - 2 * K] = y;
  }
  if (threadIdx.x < K) sDec[threadIdx.x] = expf(prep_gate(zf + dtb, expf(alog), a.prep.gate_lb));
  __syncthreads();
  if (warp < 2) {  // L2 norms of q (warp 0) and k (warp 1)
    const float* x = warp ? sK : sQ;
    float ss = 0.f;
    for (int f = lane; f < K; f += 32) ss = fmaf(x[f], x[f], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) sNorm[warp] = rsqrtf(ss + KDA_L2_EPS_F);
  }
  __syncthreads();
  for (int f = threadIdx.x; f < K; f += 256) {
    sQ[f] *= sNorm[0];
    sK[f] *= sNorm[1];
  }
  __syncthreads();
  if (warp == 0) {
    float x = 0.f;
    for (int f = lane; f < K; f += 32) x = fmaf(sQ[f], sK[f], x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if (lane == 0) sQK = x;
  }

  // ---- the recurrence step (as kda_decode_kernel)
  float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int row = warp * RPW + it * RPI + rsub;
    const float d = sDec[row], kr = sK[row], qr = sQ[row];
    s[it].x *= d; s[it].y *= d; s[it].z *= d; s[it].w *= d;
    pk.x = fmaf(kr, s[it].x, pk.x); pk.y = fmaf(kr, s[it].y, pk.y);
    pk.z = fmaf(kr, s[it].z, pk.z); pk.w = fmaf(kr, s[it].w, pk.w);
    pq.x = fmaf(qr, s[it].x, pq.x); pq.y = fmaf(qr, s[it].y, pq.y);
    pq.z = fmaf(qr, s[it].z, pq.z); pq.w = fmaf(qr, s[it].w, pq.w);
  }
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
    pk.x += __shfl_xor_sync(0xffffffffu, pk.x, off); pk.y += __shfl_xor_sync(0xffffffffu, pk.y, off);
    pk.z += __shfl_xor_sync(0xffffffffu, pk.z, off); pk.w += __shfl_xor_sync(0xffffffffu, pk.w, off);
    pq.x += __shfl_xor_sync(0xffffffffu, pq.x, off); pq.y += __shfl_xor_sync(0xffffffffu, pq.y, off);
    pq.z += __shfl_xor_sync(0xffffffffu, pq.z, off); pq.w += __shfl_xor_sync(0xffffffffu, pq.w, off);
  }
  if (rsub == 0) {
    sRk[warp][4 * c4 + 0] = pk.x; sRk[warp][4 * c4 + 1] = pk.y;
    sRk[warp][4 * c4 + 2] = pk.z; sRk[warp][4 * c4 + 3] = pk.w;
    sRq[warp][4 * c4 + 0] = pq.x; sRq[warp][4 * c4 + 1] = pq.y;
    sRq[warp][4 * c4 + 2] = pq.z; sRq[warp][4 * c4 + 3] = pq.w;
  }
  __syncthreads();
  const float beta = prep_sigmoid(blog);
  for (int n = threadIdx.x; n < V; n += 256) {
    float p = 0.f, qs = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) { p += sRk[w][n]; qs += sRq[w][n]; }
    const float delta = beta * (sV[n] - p);
    sDelta[n] = delta;
    sO[n] = a.scale * fmaf(sQK, delta, qs);
  }
  __syncthreads();
  TIn* o = static_cast<TIn*>(a.o) + ((size_t)b * a.HV + hv) * V;
  if (a.og) {  // output gate: RMS over the row's V values
    if (warp == 0) {
      float ss = 0.f;
      for (int n = lane; n < V; n += 32) ss = fmaf(sO[n], sO[n], ss);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (lane == 0) sRms = rsqrtf(ss / (float)V + a.og_eps);
    }
    __syncthreads();
    if (threadIdx.x < V) o[threadIdx.x] = from_f<TIn>(sO[threadIdx.x] * sRms * prep_sigmoid(ogv));
  } else {
    for (int n = threadIdx.x; n < V; n += 256) o[n] = from_f<TIn>(sO[n]);
  }
  const float4 d4 = make_float4(sDelta[4 * c4], sDelta[4 * c4 + 1], sDelta[4 * c4 + 2], sDelta[4 * c4 + 3]);
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int row = warp * RPW + it * RPI + rsub;
    const float kr = sK[row];
    float4 x = s[it];
    x.x = fmaf(kr, d4.x, x.x); x.y = fmaf(kr, d4.y, x.y);
    x.z = fmaf(kr, d4.z, x.z); x.w = fmaf(kr, d4.w, x.w);
    __stcs(S4 + row * LPR + c4, x);
  }
}

template <int K, int V, typename TIn>
static int launch_decode_token_t(const DecodeTokenArgs& a, cudaStream_t stream) {
  kda_decode_token_kernel<K, V, TIn><<<dim3(a.HV, a.B), 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_decode_token: launch", e);
  return 0;
}

template <int K, typename TIn>
static int launch_decode_token_k(const DecodeTokenArgs& a, int V, cudaStream_t stream) {
  switch (V) {
    case 32: return launch_decode_token_t<K, 32, TIn>(a, stream);
    case 64: return launch_decode_token_t<K, 64, TIn>(a, stream);
    case 128: return launch_decode_token_t<K, 128, TIn>(a, stream);
  }
  return set_error(4, "kda_decode_token: unsupported V");
}

int launch_decode_token(const DecodeTokenArgs& a, int K, int V, int dtype, cudaStream_t stream) {
  const bool bf = dtype == 1;
  switch (K) {
    case 32: return bf ? launch_decode_token_k<32, __nv_bfloat16>(a, V, stream) : launch_decode_token_k<32, float>(a, V, stream);
    case 64: return bf ? launch_decode_token_k<64, __nv_bfloat16>(a, V, stream) : launch_decode_token_k<64, float>(a, V, stream);
    case 128: return bf ? launch_decode_token_k<128, __nv_bfloat16>(a, V, stream) : launch_decode_token_k<128, float>(a, V, stream);
  }
  return set_error(4, "kda_decode_token: unsupported K");
}

// ---------------------------------------------------------------------------
// Prefill convolution.  Thread = (batch b, channel c, block of CONV_TB steps);
// consecutive threads take consecutive channels of one tensor row, so every
// step is one coalesced row read and write per warp.
constexpr int CONV_TB = 32, CONV_NT = 128;

template <typename TIn>
__global__ void __launch_bounds__(CONV_NT) kda_short_conv_kernel(ConvArgs a) {
  const int HK = a.H * a.K, VV = a.HV * a.V, Cn = 2 * HK + VV, W = a.W;
  const int c = blockIdx.x * CONV_NT + threadIdx.x, b = blockIdx.z, t0 = blockIdx.y * CONV_TB;
  if (c >= Cn) return;
  const TIn* x;
  TIn* y;
  int col, stride;
  if (c < HK) {
    x = static_cast<const TIn*>(a.xq); y = static_cast<TIn*>(a.q); col = c; stride = HK;
  } else if (c < 2 * HK) {
    x = static_cast<const TIn*>(a.xk); y = static_cast<TIn*>(a.k); col = c - HK; stride = HK;
  } else {
    x = static_cast<const TIn*>(a.xv); y = static_cast<TIn*>(a.v); col = c - 2 * HK; stride = VV;
  }
  const size_t base = (size_t)b * a.T * stride + col;
  const float* st = a.state_in ? a.state_in + ((size_t)b * Cn + c) * W : nullptr;
  const float* w = a.w + (size_t)c * W;
  float wr[CONV_MAX_W], win[CONV_MAX_W];
  // window before step t0: slot j holds step t0 - W + j (slot 0 drops out first);
  // a step tau < 0 lives in the state's slot tau + W.  (Loops unrolled over
  // CONV_MAX_W with predicates: the window stays in registers.)
#pragma unroll
  for (int j = 0; j < CONV_MAX_W; ++j) {
    wr[j] = j < W ? w[j] : 0.f;
    const int tau = t0 - W + j;
    win[j] = (j < 1 || j >= W) ? 0.f : (tau >= 0 ? to_f(x[base + (size_t)tau * stride]) : (st ? st[tau + W] : 0.f));
  }
  const int t1 = min(t0 + CONV_TB, a.T);
  for (int t = t0; t < t1; ++t) {
    const float xt = to_f(x[base + (size_t)t * stride]);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < CONV_MAX_W; ++j) {
      if (j < W) {
        win[j] = j + 1 < W ? win[j + 1] : xt;
        acc = fmaf(wr[j], win[j], acc);
      }
    }
    y[base + (size_t)t * stride] = from_f<TIn>(acc * prep_sigmoid(acc));
  }
  if (a.state_out && t1 == a.T) {  // the window after the last step
    float* so = a.state_out + ((size_t)b * Cn + c) * W;
    for (int j = 0; j < W; ++j) {
      const int tau = a.T - W + j;
      so[j] = tau >= 0 ? to_f(x[base + (size_t)tau * stride]) : (st ? st[tau + W] : 0.f);
    }
  }
}

int launch_short_conv(const ConvArgs& a, int dtype, cudaStream_t stream) {
  const int Cn = 2 * a.H * a.K + a.HV * a.V;
  const dim3 grid((Cn + CONV_NT - 1) / CONV_NT, (a.T + CONV_TB - 1) / CONV_TB, a.B);
  if (dtype == 1) kda_short_conv_kernel<__nv_bfloat16><<<grid, CONV_NT, 0, stream>>>(a);
  else kda_short_conv_kernel<float><<<grid, CONV_NT, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_short_conv: launch", e);
  return 0;
}

}  // namespace kda
