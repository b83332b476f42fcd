// Single-token KDA decode step on a state updated in place.
//
// "kimi_k3_host/kda.rs", kda_recurrent_step: per head the K x V state is
// decayed row by row by exp(g), the residual v - k^T S_dec is scaled by beta,
// the rank-1 update k (x) delta is added, and the output is scale * q^T S.
// The step is bound by HBM: the fp32 state is read once and written once.
// This kernel streams it with 128-bit loads, and takes both column sums it
// needs in the same pass over the decayed rows, using
//     q^T S_new = q^T S_dec + (q . k) delta,
// so the state never has to be read a second time for the readout.
//
// One CTA per (b, hv), 8 warps.  A warp owns K/8 rows; a lane owns 4
// consecutive columns (one float4) of RPI rows at a time, where RPI = 128 / V.
#include "kda_chunk.cuh"
#include "kda_internal.h"

namespace kda {

template <int K, int V, typename TIn>
__global__ void __launch_bounds__(256) kda_decode_kernel(DecodeArgs a) {
  constexpr int NW = 8, LPR = V / 4, RPI = 32 / LPR, RPW = K / NW, IT = RPW / RPI;
  static_assert(RPW % RPI == 0, "rows per warp must cover the lanes");
  __shared__ float sK[K], sQ[K], sDec[K], sV[V], sDelta[V], sRk[NW][V], sRq[NW][V];
  __shared__ float sQK;

  const int hv = blockIdx.x, b = blockIdx.y;
  const int h = hv / (a.HV / a.H);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c4 = lane % LPR, rsub = lane / LPR;
  float4* S4 = reinterpret_cast<float4*>(a.S + ((size_t)b * a.HV + hv) * K * V);

  float4 s[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int row = warp * RPW + it * RPI + rsub;
    s[it] = __ldcs(S4 + row * LPR + c4);
  }

  const TIn* q = static_cast<const TIn*>(a.q) + ((size_t)b * a.H + h) * K;
  const TIn* k = static_cast<const TIn*>(a.k) + ((size_t)b * a.H + h) * K;
  const TIn* v = static_cast<const TIn*>(a.v) + ((size_t)b * a.HV + hv) * V;
  const float* g = a.g + ((size_t)b * a.HV + hv) * K;
  for (int f = threadIdx.x; f < K; f += 256) {
    sK[f] = to_f(k[f]);
    sQ[f] = to_f(q[f]);
    sDec[f] = expf(g[f]);
  }
  for (int n = threadIdx.x; n < V; n += 256) sV[n] = to_f(v[n]);
  __syncthreads();
  if (warp == 0) {
    float x = 0.f;
    for (int f = lane; f < K; f += 32) x = fmaf(sQ[f], sK[f], x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if (lane == 0) sQK = x;
  }

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
  const float beta = a.beta[(size_t)b * a.HV + hv];
  for (int n = threadIdx.x; n < V; n += 256) {
    float p = 0.f, qs = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) { p += sRk[w][n]; qs += sRq[w][n]; }
    const float delta = beta * (sV[n] - p);
    sDelta[n] = delta;
    static_cast<TIn*>(a.o)[((size_t)b * a.HV + hv) * V + n] = from_f<TIn>(a.scale * fmaf(sQK, delta, qs));
  }
  __syncthreads();
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
static int launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  dim3 grid(a.HV, a.B);
  kda_decode_kernel<K, V, TIn><<<grid, 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_cuda_error("kda_decode_step: launch", e);
  return 0;
}

template <int K, typename TIn>
static int launch_decode_k(const DecodeArgs& a, int V, cudaStream_t stream) {
  switch (V) {
    case 32: return launch_decode_t<K, 32, TIn>(a, stream);
    case 64: return launch_decode_t<K, 64, TIn>(a, stream);
    case 128: return launch_decode_t<K, 128, TIn>(a, stream);
  }
  return set_error(4, "kda_decode_step: unsupported V");
}

int launch_decode(const DecodeArgs& a, int K, int V, int dtype, cudaStream_t stream) {
  const bool bf = dtype == 1;
  switch (K) {
    case 32: return bf ? launch_decode_k<32, __nv_bfloat16>(a, V, stream) : launch_decode_k<32, float>(a, V, stream);
    case 64: return bf ? launch_decode_k<64, __nv_bfloat16>(a, V, stream) : launch_decode_k<64, float>(a, V, stream);
    case 128: return bf ? launch_decode_k<128, __nv_bfloat16>(a, V, stream) : launch_decode_k<128, float>(a, V, stream);
  }
  return set_error(4, "kda_decode_step: unsupported K");
}

}  // namespace kda
