// Gradient of the chunked delta rule (the training backward), float32 on CUDA
// cores.
//
// The pages present the chunkwise form as what makes linear-time TRAINING
// hardware-efficient ("GPT-2 から Kimi K3 まで", news.ainew.jp, section "DeltaNet
// (Parallelizing linear transformers with delta rule)"); this kernel runs the
// reverse of that form.  Per chunk of C rows entered with state S (g = the
// chunk's cumulative log decay, Gamma_rs = e^(g_r - g_s), gamma = e^g, n = last
// row; ungated g = 0):
//   forward   A = strict_lower(diag(beta) (K K^T * Gamma)),  T = (I + A)^-1
//             X = diag(beta) (V - diag(gamma) K S),  U = T X
//             P = tril(Q K^T) * Gamma,  O = diag(gamma) Q S + P U
//             S+ = gamma_n S + (diag(e^(g_n - g)) K)^T U
//   reverse   dU  = P^T dO + diag(e^(g_n - g)) K dS+
//             dP  = tril(dO U^T)                       dBV = T^T dU
//             dT  = dU X^T,  dA = -strict_lower(T^T dT T^T)
//             dq  = diag(gamma) dO S^T + (dP * Gamma) K
//             dk  = (dP * Gamma)^T Q + diag(e^(g_n - g)) U dS+^T - diag(beta gamma) dBV S^T
//                   + (dMA * Gamma) K + (dMA * Gamma)^T K,    dMA = diag(beta) dA
//             dv  = diag(beta) dBV
//             dbeta = rowsum(dBV * V) - gamma * rowsum(dBV * KS) + rowsum(dA * MA)
//             dS  = (diag(gamma) Q)^T dO + gamma_n dS+ - K^T diag(beta gamma) dBV
//   and the gradient of g (rows and columns of every Gamma-weighted product,
//   gamma_r on the read of S, the S+ carry) summed from the last row gives the
//   gradient of log alpha.
//
// One CTA per (b, h, 64-column slice of Dv), 256 threads, C = 32 (the
// backward's own chunk; the result does not depend on it).  A forward sweep
// stores every chunk's entry state (float32) in the workspace, then the reverse
// sweep walks the chunks from the last.  The forward and the dv, dS0 outputs
// are separable over the columns of v; dq, dk, dbeta and dlog_alpha are sums
// over all columns, so each slice adds its part with one atomicAdd per element
// onto outputs cleared first: with at most two slices (Dv <= 128) the sum is
// the same in either order, so the result is deterministic.
#include <cuda_bf16.h>

#include "kernels.h"

namespace dn {
namespace {

constexpr int kThreads = 256, kWarps = kThreads / 32;
constexpr int C = 32, DVS = 64, VP = DVS + 1, CP = C + 1;

template <typename TI>
__device__ __forceinline__ float ld(const TI* p, size_t i);
template <>
__device__ __forceinline__ float ld<float>(const float* p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

// Register-tiled product for the CTA's 256 threads as a 16 x 16 grid: thread
// (r0, c0) = (tid / 16, tid % 16) accumulates the RX x RY outputs
// (r0 + 16x, c0 + 16y) of sum_{k < nk} A(r, k) B(k, c), A(r, k) = A[r * ars + k * acs],
// B(k, c) = B[k * brs + c * bcs].  RX + RY loads feed RX * RY multiply-adds.
template <int RX, int RY>
__device__ __forceinline__ void mmt(int nk, const float* A, int ars, int acs, const float* B, int brs, int bcs,
                                    float (&acc)[RX][RY]) {
  const int r0 = threadIdx.x >> 4, c0 = threadIdx.x & 15;
#pragma unroll 2
  for (int k = 0; k < nk; ++k) {
    float a[RX], b[RY];
#pragma unroll
    for (int x = 0; x < RX; ++x) a[x] = A[(r0 + 16 * x) * ars + k * acs];
#pragma unroll
    for (int y = 0; y < RY; ++y) b[y] = B[k * brs + (c0 + 16 * y) * bcs];
#pragma unroll
    for (int x = 0; x < RX; ++x)
#pragma unroll
      for (int y = 0; y < RY; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
  }
}
template <int RX, int RY>
__device__ __forceinline__ void zero_acc(float (&acc)[RX][RY]) {
#pragma unroll
  for (int x = 0; x < RX; ++x)
#pragma unroll
    for (int y = 0; y < RY; ++y) acc[x][y] = 0.f;
}

template <int DK>
struct BwdSmem {
  static constexpr int KP = DK + 1;
  static constexpr int kFloats = 2 * C * KP      // Q, K
                                 + 2 * DK * VP   // S, dS
                                 + 9 * C * VP    // V, dO, KS, X, U, dU, dBV, QS, KD
                                 + 3 * C * CP    // T, M1, M2
                                 + 8 * C;        // beta, g, gamma, e_out, dg, dbeta, red, spare
  static constexpr size_t kBytes = sizeof(float) * kFloats;
};

template <typename TI, bool GATED, int DK>
__global__ void __launch_bounds__(kThreads) chunk_bwd_kernel(const BwdProblem p) {
  using L = BwdSmem<DK>;
  constexpr int KP = L::KP;
  extern __shared__ float sm[];
  float* Qs = sm;
  float* Ks = Qs + C * KP;
  float* Ss = Ks + C * KP;
  float* dSs = Ss + DK * VP;
  float* Vs = dSs + DK * VP;
  float* dOs = Vs + C * VP;
  float* KSs = dOs + C * VP;
  float* Xs = KSs + C * VP;
  float* Us = Xs + C * VP;
  float* dUs = Us + C * VP;
  float* dBVs = dUs + C * VP;
  float* QSs = dBVs + C * VP;  // Q S (reverse sweep), e_out U (forward sweep)
  float* KDs = QSs + C * VP;   // K dS+
  float* Ts = KDs + C * VP;
  float* M1 = Ts + C * CP;
  float* M2 = M1 + C * CP;
  float* bs = M2 + C * CP;
  float* gs = bs + C;
  float* gam = gs + C;
  float* eo = gam + C;
  float* dg = eo + C;
  float* db = dg + C;
  float* red = db + C;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tr = tid >> 4, tc = tid & 15;  // this thread's place in the 16 x 16 grid of mmt
  const int bh = blockIdx.x, slice = blockIdx.y, j0 = slice * DVS;
  const int T = p.T, Dv = p.Dv, nch = (T + C - 1) / C;
  const TI* q = static_cast<const TI*>(p.q);
  const TI* k = static_cast<const TI*>(p.k);
  const TI* v = static_cast<const TI*>(p.v);
  const TI* dO = static_cast<const TI*>(p.dO);
  const size_t qk_base = (size_t)bh * T * DK, v_base = (size_t)bh * T * Dv;
  const size_t s_base = (size_t)bh * DK * Dv;
  // entry states of this (b, h, slice): nch x DK x DVS floats
  float* states = p.states + ((size_t)bh * gridDim.y + slice) * (size_t)nch * DK * DVS;

  auto gamma_rs = [&](int r, int s) { return GATED ? __expf(gs[r] - gs[s]) : 1.f; };

  // Stage chunk c: Q, K, V (slice), dO (slice), beta, g (rows past n: zero
  // inputs, beta 0, log alpha 0 so g stays flat), gamma, e^(g_last - g).
  auto stage = [&](int c, bool with_q) {
    const int c0 = c * C, n = min(C, T - c0);
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int r = idx / DK, i = idx % DK;
      const size_t at = qk_base + (size_t)(c0 + r) * DK + i;
      Ks[r * KP + i] = r < n ? ld(k, at) : 0.f;
      if (with_q) Qs[r * KP + i] = r < n ? ld(q, at) : 0.f;
    }
    for (int idx = tid; idx < C * DVS; idx += kThreads) {
      const int r = idx / DVS, j = idx % DVS;
      const size_t at = v_base + (size_t)(c0 + r) * Dv + j0 + j;
      Vs[r * VP + j] = r < n ? ld(v, at) : 0.f;
      if (with_q) dOs[r * VP + j] = r < n ? ld(dO, at) : 0.f;
    }
    if (warp == 0) {  // one lane per row: beta and the inclusive scan of log alpha
      const int r = lane;
      bs[r] = r < n ? p.beta[(size_t)bh * T + c0 + r] : 0.f;
      float la = 0.f;
      if (GATED && r < n) la = fmaxf(__logf(p.alpha[(size_t)bh * T + c0 + r]), -87.f);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, la, off);
        if (lane >= off) la += y;
      }
      gs[r] = la;
      const float glast = __shfl_sync(0xffffffffu, la, 31);
      gam[r] = GATED ? __expf(la) : 1.f;
      eo[r] = GATED ? __expf(glast - la) : 1.f;
    }
  };

  // T = (I + A)^-1 with A = strict_lower(diag(beta) (K K^T * Gamma)): A into
  // M1, then forward substitution, one column per lane of warp 0.
  auto solve_T = [&]() {
    {
      float acc[2][2];
      zero_acc(acc);
      mmt<2, 2>(DK, Ks, KP, 1, Ks, 1, KP, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 2; ++y) {
          const int r = tr + 16 * x, s2 = tc + 16 * y;
          M1[r * CP + s2] = s2 < r ? acc[x][y] * bs[r] * gamma_rs(r, s2) : 0.f;
        }
    }
    __syncthreads();
    if (warp == 0) {  // right-looking: each finished element feeds every later row at once
      const int j = lane;
      float acc[C];
#pragma unroll
      for (int i = 0; i < C; ++i) acc[i] = 0.f;
#pragma unroll
      for (int m = 0; m < C; ++m) {
        const float cm = m == j ? 1.f : (m > j ? -acc[m] : 0.f);
        Ts[m * CP + j] = cm;
#pragma unroll
        for (int i = 0; i < C; ++i)
          if (i > m) acc[i] = fmaf(M1[i * CP + m], cm, acc[i]);
      }
    }
    __syncthreads();
  };

  // KS = K S, X = diag(beta) (V - diag(gamma) K S), U = T X
  auto forward_u = [&]() {
    {
      float acc[2][4];
      zero_acc(acc);
      mmt<2, 4>(DK, Ks, KP, 1, Ss, VP, 1, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int r = tr + 16 * x, j = tc + 16 * y;
          KSs[r * VP + j] = acc[x][y];
          Xs[r * VP + j] = bs[r] * (Vs[r * VP + j] - gam[r] * acc[x][y]);
        }
    }
    __syncthreads();
    {  // T is lower triangular with explicit zeros above the diagonal
      float acc[2][4];
      zero_acc(acc);
      mmt<2, 4>(C, Ts, CP, 1, Xs, VP, 1, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) Us[(tr + 16 * x) * VP + tc + 16 * y] = acc[x][y];
    }
    __syncthreads();
  };

  // ---------------------------------------------------------- forward sweep --
  for (int idx = tid; idx < DK * DVS; idx += kThreads) {
    const int i = idx / DVS, j = idx % DVS;
    Ss[i * VP + j] = p.S0 ? p.S0[s_base + (size_t)i * Dv + j0 + j] : 0.f;
  }
  for (int c = 0; c < nch; ++c) {
    __syncthreads();
    stage(c, false);
    for (int idx = tid; idx < DK * DVS; idx += kThreads)
      states[(size_t)c * DK * DVS + idx] = Ss[(idx / DVS) * VP + idx % DVS];
    __syncthreads();
    solve_T();
    forward_u();
    for (int idx = tid; idx < C * DVS; idx += kThreads) {  // e_out U
      const int r = idx / DVS, j = idx % DVS;
      QSs[r * VP + j] = eo[r] * Us[r * VP + j];
    }
    __syncthreads();
    {
      float acc[DK / 16][4];
      zero_acc(acc);
      mmt<DK / 16, 4>(C, Ks, 1, KP, QSs, VP, 1, acc);
#pragma unroll
      for (int x = 0; x < DK / 16; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int i = tr + 16 * x, j = tc + 16 * y;
          Ss[i * VP + j] = gam[C - 1] * Ss[i * VP + j] + acc[x][y];
        }
    }
  }

  // ---------------------------------------------------------- reverse sweep --
  __syncthreads();
  for (int idx = tid; idx < DK * DVS; idx += kThreads) {
    const int i = idx / DVS, j = idx % DVS;
    dSs[i * VP + j] = p.dS_T ? p.dS_T[s_base + (size_t)i * Dv + j0 + j] : 0.f;
  }
  for (int c = nch - 1; c >= 0; --c) {
    const int c0 = c * C, n = min(C, T - c0);
    __syncthreads();
    stage(c, true);
    for (int idx = tid; idx < DK * DVS; idx += kThreads)
      Ss[(idx / DVS) * VP + idx % DVS] = states[(size_t)c * DK * DVS + idx];
    __syncthreads();
    solve_T();
    forward_u();
    // P = tril(Q K^T) * Gamma into M1
    {
      float acc[2][2];
      zero_acc(acc);
      mmt<2, 2>(DK, Qs, KP, 1, Ks, 1, KP, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 2; ++y) {
          const int r = tr + 16 * x, s2 = tc + 16 * y;
          M1[r * CP + s2] = s2 <= r ? acc[x][y] * gamma_rs(r, s2) : 0.f;
        }
    }
    __syncthreads();
    // KD = K dS+, QS = Q S, then dU = P^T dO + diag(e_out) KD
    {
      float kd[2][4], qs[2][4], pt[2][4];
      zero_acc(kd);
      zero_acc(qs);
      zero_acc(pt);
      mmt<2, 4>(DK, Ks, KP, 1, dSs, VP, 1, kd);
      mmt<2, 4>(DK, Qs, KP, 1, Ss, VP, 1, qs);
      mmt<2, 4>(C, M1, 1, CP, dOs, VP, 1, pt);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int r = tr + 16 * x, j = tc + 16 * y;
          KDs[r * VP + j] = kd[x][y];
          QSs[r * VP + j] = qs[x][y];
          dUs[r * VP + j] = pt[x][y] + eo[r] * kd[x][y];
        }
    }
    __syncthreads();
    // dP = tril(dO U^T) into M2;  dBV = T^T dU
    {
      float acc[2][2];
      zero_acc(acc);
      mmt<2, 2>(DVS, dOs, VP, 1, Us, 1, VP, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 2; ++y) {
          const int r = tr + 16 * x, s2 = tc + 16 * y;
          M2[r * CP + s2] = s2 <= r ? acc[x][y] : 0.f;
        }
    }
    {
      float acc[2][4];
      zero_acc(acc);
      mmt<2, 4>(C, Ts, 1, CP, dUs, VP, 1, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) dBVs[(tr + 16 * x) * VP + tc + 16 * y] = acc[x][y];
    }
    __syncthreads();
    // Per-row sums, one warp per row (lanes over the slice's columns):
    //   dg_r  = gamma_r sum_j dO (Q S) - beta_r gamma_r sum_j dBV KS - c_out_r
    //   db_r  = sum_j dBV V - gamma_r sum_j dBV KS
    //   c_out_r = e_out_r sum_j U (K dS+)        (the S+ carry's decay)
    for (int r = warp; r < C; r += kWarps) {
      float t_qs = 0.f, t_bk = 0.f, t_bv = 0.f, t_co = 0.f;
      for (int j = lane; j < DVS; j += 32) {
        t_qs += dOs[r * VP + j] * QSs[r * VP + j];
        t_bk += dBVs[r * VP + j] * KSs[r * VP + j];
        t_bv += dBVs[r * VP + j] * Vs[r * VP + j];
        t_co += Us[r * VP + j] * KDs[r * VP + j];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        t_qs += __shfl_xor_sync(0xffffffffu, t_qs, off);
        t_bk += __shfl_xor_sync(0xffffffffu, t_bk, off);
        t_bv += __shfl_xor_sync(0xffffffffu, t_bv, off);
        t_co += __shfl_xor_sync(0xffffffffu, t_co, off);
      }
      if (lane == 0) {
        const float co = eo[r] * t_co;
        dg[r] = gam[r] * t_qs - bs[r] * gam[r] * t_bk - co;
        db[r] = t_bv - gam[r] * t_bk;
        red[r] = co;
      }
    }
    // the carry gamma_n S: sum over the slice of dS+ * S (block reduction)
    {
      float acc = 0.f;
      for (int idx = tid; idx < DK * DVS; idx += kThreads)
        acc += dSs[(idx / DVS) * VP + idx % DVS] * Ss[(idx / DVS) * VP + idx % DVS];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      __syncthreads();  // red[] of the row sums is written
      __shared__ float wsum[kWarps];
      if (lane == 0) wsum[warp] = acc;
      __syncthreads();
      if (tid == 0) {
        float tot = 0.f, co = 0.f;
        for (int w = 0; w < kWarps; ++w) tot += wsum[w];
        for (int r = 0; r < C; ++r) co += red[r];
        dg[C - 1] += gam[C - 1] * tot + co;
      }
    }
    __syncthreads();
    // the rows and columns of P's decay: dg += rowsum(dP * P) - colsum(dP * P)
    if (GATED && tid < C) {
      const int r = tid;
      float acc = 0.f;
      for (int s = 0; s < C; ++s) acc += M2[r * CP + s] * M1[r * CP + s] - M2[s * CP + r] * M1[s * CP + r];
      dg[r] += acc;
    }
    __syncthreads();
    if (GATED)  // dP * Gamma in place (dq and dk use only that)
      for (int idx = tid; idx < C * C; idx += kThreads) {
        const int r = idx / C, s2 = idx % C;
        if (s2 <= r) M2[r * CP + s2] *= gamma_rs(r, s2);
      }
    __syncthreads();
    // dq = diag(gamma) dO S^T + (dP * Gamma) K
#pragma unroll 1
    for (int h = 0; h < DK / 64; ++h) {  // columns i of dq in blocks of 64
      float a[2][4], b[2][4];
      zero_acc(a);
      zero_acc(b);
      mmt<2, 4>(DVS, dOs, VP, 1, Ss + 64 * h * VP, 1, VP, a);
      mmt<2, 4>(C, M2, CP, 1, Ks + 64 * h, KP, 1, b);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int r = tr + 16 * x, i = 64 * h + tc + 16 * y;
          if (r < n) atomicAdd(p.dq + qk_base + (size_t)(c0 + r) * DK + i, gam[r] * a[x][y] + b[x][y]);
        }
    }
    __syncthreads();
    // dT = dU X^T (strictly lower part: only it reaches dA), into M1
    {
      float acc[2][2];
      zero_acc(acc);
      mmt<2, 2>(DVS, dUs, VP, 1, Xs, 1, VP, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 2; ++y) {
          const int r = tr + 16 * x, s2 = tc + 16 * y;
          M1[r * CP + s2] = s2 < r ? acc[x][y] : 0.f;
        }
    }
    __syncthreads();
    // Y = dT T^T, row by row in place (row a of Y needs only row a of dT)
    for (int a = warp; a < C; a += kWarps) {
      const float d = M1[a * CP + lane];
      __syncwarp();
      float y = 0.f;
      for (int b = 0; b < C; ++b) y += __shfl_sync(0xffffffffu, d, b) * Ts[lane * CP + b];
      M1[a * CP + lane] = y;
    }
    __syncthreads();
    // dA = -strict_lower(T^T Y), column by column in place (column s of dA
    // needs only column s of Y)
    for (int s = warp; s < C; s += kWarps) {
      const float y = M1[lane * CP + s];
      __syncwarp();
      float acc = 0.f;
      for (int a = 0; a < C; ++a) acc += Ts[a * CP + lane] * __shfl_sync(0xffffffffu, y, a);
      M1[lane * CP + s] = lane > s ? -acc : 0.f;
    }
    __syncthreads();
    // E = dA * MA into Ts (T is no longer needed), MA = K K^T * Gamma
    {
      float acc[2][2];
      zero_acc(acc);
      mmt<2, 2>(DK, Ks, KP, 1, Ks, 1, KP, acc);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 2; ++y) {
          const int r = tr + 16 * x, s2 = tc + 16 * y;
          Ts[r * CP + s2] = s2 < r ? M1[r * CP + s2] * acc[x][y] * gamma_rs(r, s2) : 0.f;
        }
    }
    __syncthreads();
    // dbeta += rowsum(dA * MA);  dg += beta_r rowsum(E) - sum_t beta_t E[t][r];
    // then dMA = diag(beta) dA in place
    if (tid < C) {
      const int r = tid;
      float rs = 0.f, cs = 0.f;
      for (int s = 0; s < C; ++s) {
        rs += Ts[r * CP + s];
        cs += bs[s] * Ts[s * CP + r];
      }
      db[r] += rs;
      if (GATED) dg[r] += bs[r] * rs - cs;
    }
    __syncthreads();
    // (dMA * Gamma) + its transpose into Ts (E is no longer needed), dMA = diag(beta) dA
    for (int idx = tid; idx < C * C; idx += kThreads) {
      const int r = idx / C, s2 = idx % C;
      float m = 0.f;
      if (s2 < r) m = bs[r] * M1[r * CP + s2] * gamma_rs(r, s2);
      if (r < s2) m = bs[s2] * M1[s2 * CP + r] * gamma_rs(s2, r);
      Ts[r * CP + s2] = m;
    }
    __syncthreads();
    // dk = (dP * Gamma)^T Q + diag(e_out) U dS+^T - diag(beta gamma) dBV S^T
    //      + ((dMA * Gamma) + (dMA * Gamma)^T) K
#pragma unroll 1
    for (int h = 0; h < DK / 64; ++h) {  // columns i of dk in blocks of 64
      float pl[2][4], ue[2][4], bg[2][4];
      zero_acc(pl);
      zero_acc(ue);
      zero_acc(bg);
      mmt<2, 4>(C, M2, 1, CP, Qs + 64 * h, KP, 1, pl);
      mmt<2, 4>(C, Ts, CP, 1, Ks + 64 * h, KP, 1, pl);
      mmt<2, 4>(DVS, Us, VP, 1, dSs + 64 * h * VP, 1, VP, ue);
      mmt<2, 4>(DVS, dBVs, VP, 1, Ss + 64 * h * VP, 1, VP, bg);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int s2 = tr + 16 * x, i = 64 * h + tc + 16 * y;
          if (s2 < n)
            atomicAdd(p.dk + qk_base + (size_t)(c0 + s2) * DK + i,
                      pl[x][y] + eo[s2] * ue[x][y] - bs[s2] * gam[s2] * bg[x][y]);
        }
    }
    // dv = diag(beta) dBV (this slice's columns: a plain store)
    for (int idx = tid; idx < C * DVS; idx += kThreads) {
      const int r = idx / DVS, j = idx % DVS;
      if (r < n) p.dv[v_base + (size_t)(c0 + r) * Dv + j0 + j] = bs[r] * dBVs[r * VP + j];
    }
    // dbeta and d(log alpha) = sum of dg over rows >= r within the chunk
    if (warp == 0) {
      const int r = lane;
      float x = GATED ? dg[C - 1 - r] : 0.f;  // reverse inclusive scan
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
      }
      const int row = C - 1 - r;
      if (row < n) {
        atomicAdd(p.dbeta + (size_t)bh * T + c0 + row, db[row]);
        if (GATED && p.dlog_alpha) atomicAdd(p.dlog_alpha + (size_t)bh * T + c0 + row, x);
      }
    }
    __syncthreads();
    // dS = Q^T diag(gamma) dO + gamma_n dS+ - K^T diag(beta gamma) dBV, in place;
    // the row scales go onto dO and dBV first (neither is read again this chunk)
    for (int idx = tid; idx < C * DVS; idx += kThreads) {
      const int r = idx / DVS, j = idx % DVS;
      dOs[r * VP + j] *= gam[r];
      dBVs[r * VP + j] *= -bs[r] * gam[r];
    }
    __syncthreads();
    {
      float acc[DK / 16][4];
      zero_acc(acc);
      mmt<DK / 16, 4>(C, Qs, 1, KP, dOs, VP, 1, acc);
      mmt<DK / 16, 4>(C, Ks, 1, KP, dBVs, VP, 1, acc);
#pragma unroll
      for (int x = 0; x < DK / 16; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int i = tr + 16 * x, j = tc + 16 * y;
          dSs[i * VP + j] = gam[C - 1] * dSs[i * VP + j] + acc[x][y];
        }
    }
  }
  __syncthreads();
  if (p.dS0)
    for (int idx = tid; idx < DK * DVS; idx += kThreads) {
      const int i = idx / DVS, j = idx % DVS;
      p.dS0[s_base + (size_t)i * Dv + j0 + j] = dSs[i * VP + j];
    }
}

template <typename TI, bool GATED, int DK>
cudaError_t launch_one(const BwdProblem& p, cudaStream_t st) {
  using L = BwdSmem<DK>;
  auto kern = chunk_bwd_kernel<TI, GATED, DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)(p.B * p.H), (unsigned)(p.Dv / DVS)), kThreads, L::kBytes, st>>>(p);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t launch_dt(const BwdProblem& p, cudaStream_t st) {
  const bool gated = p.alpha != nullptr;
  if (p.Dk == 128) return gated ? launch_one<TI, true, 128>(p, st) : launch_one<TI, false, 128>(p, st);
  return gated ? launch_one<TI, true, 64>(p, st) : launch_one<TI, false, 64>(p, st);
}

}  // namespace

size_t chunk_bwd_state_bytes(int B, int H, int T, int Dk, int Dv) {
  const size_t nch = ((size_t)T + C - 1) / C;
  return (size_t)B * H * nch * Dk * Dv * sizeof(float);
}

cudaError_t launch_chunk_bwd(const BwdProblem& p, cudaStream_t st) {
  const size_t BH = (size_t)p.B * p.H, T = (size_t)p.T;
  // the slices add their parts of these onto zeros
  cudaError_t e = cudaMemsetAsync(p.dq, 0, BH * T * p.Dk * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(p.dk, 0, BH * T * p.Dk * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(p.dbeta, 0, BH * T * sizeof(float), st);
  if (e == cudaSuccess && p.dlog_alpha) e = cudaMemsetAsync(p.dlog_alpha, 0, BH * T * sizeof(float), st);
  if (e != cudaSuccess) return e;
  return p.bf16 ? launch_dt<__nv_bfloat16>(p, st) : launch_dt<float>(p, st);
}

}  // namespace dn
