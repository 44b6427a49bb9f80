// Recurrent decode step: one token for each of B x H cached states, in place.
//
// The delta rule at t = 1 ("GPT-2 から Kimi K3 まで", news.ainew.jp, section
// "DeltaNet (Fast weight programmers)", with the cached state; gate as in the
// Gated DeltaNet paragraph of "How a Baseten Engineer Traced 7 Years of
// Attention Mechanism Evolution": decay first, then the precise write):
//     r = k S,  p = q S            (both from the stored state, one pass)
//     u = beta (v - alpha r)
//     o = alpha p + (q . k) u      (= q (alpha S + k^T u), the state after the write)
//     S = alpha S + k^T u
// With a per-dimension decay the rows of S are scaled first (S_i <- alpha_i S_i)
// and the same formulas run with alpha = 1 on the decayed rows.
//
// The step is bound by HBM: each Dk x Dv float32 state is read once and written
// once.  One CTA per head; warp w streams rows w, w + 8, ... with one 16-byte
// (Dv = 128) or 8-byte (Dv = 64) load per lane per row, so every row is one
// fully coalesced request, all of a thread's loads are issued before any is
// used, and the state stays in registers between the reduction and the update.
#include <cuda_bf16.h>

#include "kernels.h"

namespace dn {
namespace {

constexpr int kWarps = 8;

template <typename TI>
__device__ __forceinline__ float ld1(const TI* p, size_t i);
template <>
__device__ __forceinline__ float ld1<float>(const float* p, size_t i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
template <typename TI>
__device__ __forceinline__ void st1(TI* p, size_t i, float x);
template <>
__device__ __forceinline__ void st1<float>(float* p, size_t i, float x) { p[i] = x; }
template <>
__device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

template <int CPL>
struct Vec;
template <>
struct Vec<4> {
  using T = float4;
  __device__ static T load(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
  __device__ static void store(float* p, const float (&x)[4]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
  __device__ static void unpack(const T& v, float (&x)[4]) { x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w; }
};
template <>
struct Vec<2> {
  using T = float2;
  __device__ static T load(const float* p) { return __ldcs(reinterpret_cast<const float2*>(p)); }
  __device__ static void store(float* p, const float (&x)[2]) {
    __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
  }
  __device__ static void unpack(const T& v, float (&x)[2]) { x[0] = v.x; x[1] = v.y; }
};

// Options of the step (template parameters, one instantiation each):
//   PRE   q and k are raw projections and beta holds logits: q, k <- normalize(silu(.))
//         (L2 over Dk, divisor max(norm, 1e-12)), beta <- sigmoid(beta): the DeltaNet
//         layer's feature maps ("GPT-2 から Kimi K3 まで", section "DeltaNet (Fast weight
//         programmers)"), applied here so the maps cost no extra pass over q and k.
//   GATE  0: none; 1: one decay alpha per head; 2: one decay per key dimension,
//         alpha (B,H,Dk), row i of S scaled by alpha[i] (the per-dimension gating of
//         the KDA paragraph of "How a Baseten Engineer Traced 7 Years ...").
template <typename TI, int DK, int DV, int GATE, bool PRE>
__global__ void __launch_bounds__(kWarps * 32, 2) decode_kernel(const DecodeProblem p) {
  constexpr int CPL = DV / 32;     // state columns per lane
  constexpr int RPW = DK / kWarps; // state rows per warp
  using V = Vec<CPL>;
  __shared__ float ks[DK], qs[DK], as[GATE == 2 ? DK : 1];
  __shared__ float red[2][kWarps][DV];
  __shared__ float qk_s;

  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const size_t bh = blockIdx.x;
  float* S = p.S + bh * DK * DV;
  const int c0 = lane * CPL;

  // Issue every state load of this thread first.
  typename V::T raw[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) raw[rr] = V::load(S + (size_t)(rr * kWarps + w) * DV + c0);

  const TI* q = static_cast<const TI*>(p.q) + bh * DK;
  const TI* k = static_cast<const TI*>(p.k) + bh * DK;
  for (int i = threadIdx.x; i < DK; i += kWarps * 32) {
    qs[i] = ld1(q, i);
    ks[i] = ld1(k, i);
    if (GATE == 2) as[i] = p.alpha[bh * DK + i];
  }
  float beta = p.beta[bh];
  if (PRE) beta = 1.f / (1.f + __expf(-beta));
  const float alpha = GATE == 1 ? p.alpha[bh] : 1.f;
  float vj[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) vj[c] = ld1(static_cast<const TI*>(p.v), bh * DV + c0 + c);
  __syncthreads();
  if (PRE && w < 2) {  // warp 0 maps q, warp 1 maps k: silu, then L2 normalise
    float* x = w == 0 ? qs : ks;
    float y[DK / 32], ss = 0.f;
#pragma unroll
    for (int e = 0; e < DK / 32; ++e) {
      const float t = x[lane + 32 * e];
      y[e] = t / (1.f + __expf(-t));
      ss = fmaf(y[e], y[e], ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
    for (int e = 0; e < DK / 32; ++e) x[lane + 32 * e] = y[e] * inv;
  }
  if (PRE) __syncthreads();

  float s[RPW][CPL];
  float rk[CPL], rq[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) rk[c] = rq[c] = 0.f;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    V::unpack(raw[rr], s[rr]);
    const int i = rr * kWarps + w;
    if (GATE == 2) {  // decay first: row i of the state is alpha[i] S_i
      const float a = as[i];
#pragma unroll
      for (int c = 0; c < CPL; ++c) s[rr][c] *= a;
    }
    const float ki = ks[i], qi = qs[i];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      rk[c] = fmaf(ki, s[rr][c], rk[c]);
      rq[c] = fmaf(qi, s[rr][c], rq[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    red[0][w][c0 + c] = rk[c];
    red[1][w][c0 + c] = rq[c];
  }
  if (w == 0) {
    float acc = 0.f;
    for (int i = lane; i < DK; i += 32) acc = fmaf(qs[i], ks[i], acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) qk_s = acc;
  }
  __syncthreads();

  float u[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    float r = 0.f, pq = 0.f;
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) {
      r += red[0][ww][c0 + c];
      pq += red[1][ww][c0 + c];
    }
    u[c] = beta * (vj[c] - alpha * r);
    if (w == 0) st1(static_cast<TI*>(p.o), bh * DV + c0 + c, fmaf(alpha, pq, qk_s * u[c]));
  }
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const float ki = ks[rr * kWarps + w];
    float out[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) out[c] = fmaf(ki, u[c], alpha * s[rr][c]);
    V::store(S + (size_t)(rr * kWarps + w) * DV + c0, out);
  }
}

template <typename TI, int DK, int DV, int GATE>
cudaError_t launch_g(const DecodeProblem& p, cudaStream_t st) {
  const unsigned grid = (unsigned)(p.B * p.H);
  if (p.prestep)
    decode_kernel<TI, DK, DV, GATE, true><<<grid, kWarps * 32, 0, st>>>(p);
  else
    decode_kernel<TI, DK, DV, GATE, false><<<grid, kWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

template <typename TI, int DK, int DV>
cudaError_t launch_t(const DecodeProblem& p, cudaStream_t st) {
  if (!p.alpha) return launch_g<TI, DK, DV, 0>(p, st);
  return p.alpha_per_dim ? launch_g<TI, DK, DV, 2>(p, st) : launch_g<TI, DK, DV, 1>(p, st);
}

template <typename TI>
cudaError_t launch_dt(const DecodeProblem& p, cudaStream_t st) {
  if (p.Dk == 128 && p.Dv == 128) return launch_t<TI, 128, 128>(p, st);
  if (p.Dk == 128 && p.Dv == 64) return launch_t<TI, 128, 64>(p, st);
  if (p.Dk == 64 && p.Dv == 128) return launch_t<TI, 64, 128>(p, st);
  if (p.Dk == 64 && p.Dv == 64) return launch_t<TI, 64, 64>(p, st);
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_decode(const DecodeProblem& p, cudaStream_t st) {
  return p.bf16 ? launch_dt<__nv_bfloat16>(p, st) : launch_dt<float>(p, st);
}

}  // namespace dn
