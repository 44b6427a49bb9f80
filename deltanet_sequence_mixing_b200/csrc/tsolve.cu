// Chunk-parallel WY pre-pass of the tcgen05 delta-rule forward: for every
// (b, h, chunk of C = 64 or 128 tokens) it forms T = (I + A)^-1 with
//   A = strict_lower(diag(beta) (K K^T * Gamma)),   Gamma_rs = exp(g_r - g_s),
// and writes Tb = T diag(beta) (and, gated, Tbg = Tb diag(exp(g))) as bf16
// C x C tiles into the workspace, plus the chunk's decay prefix g.  These are
// the state-independent parts of the Householder / WY reparameterisation
// ("GPT-2 から Kimi K3 まで", news.ainew.jp, section "DeltaNet (Parallelizing linear
// transformers with delta rule)"); the chunk kernel then applies them with
// tensor-core products, keeping only matrix products on its serial state chain.
//
// One CTA of 2C threads (one warp per 16-row block) per chunk, eight CTAs per
// SM at C = 64 and two at C = 128: the solve is a short chain of dependent
// steps, so it is latency-bound per chunk and the grid's parallelism over
// chunks hides that latency.
//   1. K (rows past T zero) -> shared memory; beta, log-alpha prefix g.
//   2. G = K K^T by tcgen05 (bf16 operands from the swizzled K tile, float32
//      accumulator in TMEM), read back row by row into A, masked and scaled.
//   3. C/16 diagonal 16x16 inverses (two per warp, one per half-warp; one
//      column per lane, right-looking substitution so only one multiply-add
//      per step is on the dependency chain), then the blocks below the
//      diagonal from the 2 x 2 block inverse
//      [[L11, 0], [L21, L22]]^-1 = [[T1, 0], [-T2 L21 T1, T2]] applied
//      recursively (64 x 64 halves of 32 x 32 halves), with tf32 WMMA products
//      spread over all warps: four dependent levels at C = 64, six at C = 128.
//   4. Tb, Tbg -> global (row-major bf16 C x C tiles).
#include <cuda_bf16.h>
#include <mma.h>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

using namespace nvcuda;

template <int C>
struct TsolveShape {
  static constexpr int kThreads = 2 * C;       // one warp per 16-row block
  static constexpr int kWarps = kThreads / 32;  // == C / 16
  static constexpr int kApad = C + 4;           // float row stride of the A / T scratch
  static_assert(kWarps == C / 16, "one warp per 16-row block");
};

// Shared memory: the K tile (128-byte swizzled, KB blocks of C rows x 128 B,
// from TMA) and A, with T built in place of A (every block of A is read for
// the last time in the level before the one that writes that block of T).
// At C = 64, A also shares its region with the K tile (A is written only after
// the Gram has read K), and the region extends 8 KB past the tile: the M = 128
// Gram operand's rows 64-127 read whatever follows a block (those TMEM rows are
// not used).  That keeps the CTA at 26 KB, eight per SM; at C = 128, K and A
// side by side take 103 KB, two per SM.
template <int C, int DK, bool PRE = false>
struct TsolveSmem {
  static constexpr uint32_t kKBytes = (DK / 64) * C * 128;
  static constexpr uint32_t kTBytes = C * TsolveShape<C>::kApad * 4;
  static constexpr uint32_t round1k(uint32_t x) { return (x + 1023) / 1024 * 1024; }
  static constexpr uint32_t AM_OFF = C == 64 ? 0 : round1k(kKBytes);
  static constexpr uint32_t kRegion =
      C == 64 ? round1k(kTBytes > kKBytes + 8192 ? kTBytes : kKBytes + 8192) : AM_OFF + kTBytes;
  // the pre-step maps the chunk's q tile here (TMA, 128-byte swizzle), after the region
  static constexpr uint32_t QT_OFF = round1k(kRegion);
  static constexpr uint32_t VEC_OFF = PRE ? QT_OFF + kKBytes : kRegion;  // beta, g, e^g, e^(m-g), 8 warp totals
  static constexpr uint32_t BAR_OFF = (VEC_OFF + (4 * C + 8) * 4 + 7) / 8 * 8;  // FULL, MMA, TMEM slot
  static constexpr uint32_t BYTES = BAR_OFF + 32;
  static constexpr uint32_t ALLOC = BYTES + 1024;  // 1024-byte alignment of the K tile
  static_assert(C == 128 || kKBytes + 8192 <= BYTES, "M = 128 operand rows past the K tile stay inside");
  static_assert(VEC_OFF % 16 == 0 && AM_OFF % 1024 == 0, "vector loads and the swizzled K tile stay aligned");
};

// tf32 operands by truncation: keep the sign, exponent and top 10 mantissa bits
// (round toward zero, relative error < 2^-10; the factors leave this kernel
// rounded to bf16, 2^-8).  One integer AND per element.
template <typename Frag>
__device__ __forceinline__ void to_tf32(Frag& f) {
#pragma unroll
  for (int t = 0; t < f.num_elements; ++t) f.x[t] = __uint_as_float(__float_as_uint(f.x[t]) & 0xFFFFE000u);
}

template <int C, int DK, bool GATED, bool PRE>
__global__ void __launch_bounds__(2 * C, C == 64 ? 8 : 2)
    tsolve_kernel(const __grid_constant__ CUtensorMap tmK, const float* __restrict__ beta,
                  const __grid_constant__ CUtensorMap tmQ, const float* __restrict__ alpha,
                  __nv_bfloat16* __restrict__ tb_out,
                  __nv_bfloat16* __restrict__ tbg_out, float* __restrict__ g_out,
                  __nv_bfloat16* __restrict__ khat, __nv_bfloat16* __restrict__ qhat, int T, int nchunks,
                  unsigned int* status) {
  using Sh = TsolveShape<C>;
  using SL = TsolveSmem<C, DK, PRE>;
  constexpr int kC = C, kApad = Sh::kApad;
  extern __shared__ uint8_t tsolve_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsolve_smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = warp_uniform(smem_u32(sm));
  float* Am = reinterpret_cast<float*>(sm + SL::AM_OFF);
  float* Tm = Am;  // T is built in place of A
  float* vb = reinterpret_cast<float*>(sm + SL::VEC_OFF);
  float* vg = vb + kC;
  float* veg = vg + kC;
  float* vinv = veg + kC;  // e^(m - g), m the midpoint of the chunk's g range
  float* wsum = vinv + kC;  // per-warp totals of the log-decay scan
  const uint32_t bar_full = sb + SL::BAR_OFF, bar_mma = sb + SL::BAR_OFF + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SL::BAR_OFF + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SL::BAR_OFF + 20);

  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = (int)warp_uniform((uint32_t)tid >> 5);
  // one-dimensional grid over (b, h, chunk), chunks of one head adjacent
  const int chunk = (int)(blockIdx.x % (unsigned)nchunks), bh = (int)(blockIdx.x / (unsigned)nchunks);
  const int c0 = chunk * kC, n = min(kC, T - c0);

  // 1. K tile by TMA (rows past T read as zero), beta and the log-decay prefix g
  //    (rows >= n: beta = 0, alpha = 1) while it lands.
  if (tid == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kC);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = warp_uniform(*tmem_slot);
  const WaitCtl wc{abort_flag, status, kWaitLimitNs};
  if (tid == 0) {
    mbar_expect_tx(bar_full, (uint32_t)SL::kKBytes * (PRE ? 2 : 1));
#pragma unroll
    for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
      for (int rb = 0; rb < kC / 64; ++rb) {
        tma_load_3d(sb + kb * (kC * 128) + rb * 8192, &tmK, bar_full, kb * 64, c0 + rb * 64, bh);
        if (PRE) tma_load_3d(sb + SL::QT_OFF + kb * (kC * 128) + rb * 8192, &tmQ, bar_full, kb * 64, c0 + rb * 64, bh);
      }
  }
  float glog = 0.f;
  if (tid < kC) {
    const size_t tb = (size_t)bh * T + c0;
    float b = tid < n ? beta[tb + tid] : 0.f;
    if (PRE && tid < n) b = 1.f / (1.f + __expf(-b));  // beta holds logits
    vb[tid] = b;
    if (GATED) {  // inclusive scan of max(log alpha, -87) within each warp
      glog = tid < n ? fmaxf(__logf(alpha[tb + tid]), -87.f) : 0.f;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, glog, off);
        if (lane >= off) glog += y;
      }
      if (lane == 31) wsum[warp] = glog;
    }
  }
  bool ok = true;
  if (PRE) {
    // The layer's pre-step on K in shared memory (two threads per row); the
    // mapped rows also go to the workspace, where the chunk kernel reads them.
    ok = __all_sync(0xffffffffu, mbar_wait(bar_full, 0, wc));  // warp-uniform for the shuffles
    const int r = tid >> 1;
    if (ok) {
      const size_t row = ((size_t)bh * T + c0 + r) * DK;
      prestep_row_sw128<DK>(sm, (uint32_t)kC * 128, r, tid & 1, r < n ? khat + row : nullptr);
      // and on the chunk's queries (the chunk kernel reads both from the workspace)
      prestep_row_sw128<DK>(sm + SL::QT_OFF, (uint32_t)kC * 128, r, tid & 1, r < n ? qhat + row : nullptr);
    }
    fence_proxy_async_smem();
    ok = __syncthreads_and(ok);
  }
  // 2. G = K K^T on the tensor cores (M = 128, N = C, into TMEM), issued by one
  //    elected lane of warp 0 once the tile has landed.
  if (warp == 0) {
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar_full, 0, wc));
    if (!ok && lane == 0) {  // never leave with the copy in flight
      int zero = 0;
      const WaitCtl drain{&zero, status, kWaitLimitNs};
      (void)mbar_wait(bar_full, 0, drain);
    }
    if (ok) {
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16(128, kC, false, false);
      const uint64_t d0 = desc_k(sb);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint64_t d = desc_step(d0, (ks >> 2) * (kC * 128) + (ks & 3) * 32);
        mma_bf16_ss_elect(tmem, d, d, id, ks > 0);
      }
    }
    mma_commit_elect(bar_mma);  // arrives even with no MMA in flight
  }
  __syncthreads();
  if (GATED) {  // add the totals of the earlier warps: g = cumsum over the chunk
    if (tid < kC) {
      for (int w = 0; w < warp; ++w) glog += wsum[w];
      vg[tid] = glog;
      veg[tid] = __expf(glog);
      g_out[((size_t)bh * nchunks + chunk) * kC + tid] = glog;
    }
    __syncthreads();
    if (tid < kC) vinv[tid] = __expf(0.5f * (vg[0] + vg[kC - 1]) - vg[tid]);
    __syncthreads();
  }
  //    A = strict_lower(diag(beta) G * Gamma): TMEM row r -> A row r (64 columns
  //    per thread).  Nothing reads A's upper part or T's strictly-upper tiles
  //    unmasked (the diagonal solve writes whole diagonal tiles, the block
  //    solve reads tiles on or below the diagonal, the output masks by column).
  ok = mbar_wait(bar_mma, 0, wc) && ok;
  tc_fence_after();
  if (tid < (kC == 64 ? 64 : 256)) {
    const int r = tid & 127;  // = 32 (warp % 4) + lane: this warp's TMEM lanes
    const int col0 = (kC == 128) ? (tid >> 7) * 64 : 0;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    // Gated: Gamma_rc = e^(g_r - g_c) (c < r) as e^(g_r - m) e^(m - g_c), both
    // factors within e^(+-80) while the chunk's g range is at most 160 (g is
    // non-increasing); a wider range (gates near zero) takes one exponential
    // per element.
    const float gr = GATED ? vg[r] : 0.f;
    const bool fact = !GATED || vg[0] - vg[kC - 1] <= 160.f;
    const float br = GATED && fact ? vb[r] * __expf(gr - 0.5f * (vg[0] + vg[kC - 1])) : vb[r];
    float* arow = Am + r * kApad + col0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t gv[32];
      tmem_ld32(tmem + lane_base + col0 + q * 32, gv);
      tmem_wait_ld();
      if (fact) {
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          float a4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = col0 + q * 32 + e4 + e;
            float a = br * __uint_as_float(gv[e4 + e]);
            if (GATED) a *= vinv[c];
            a4[e] = c < r ? a : 0.f;
          }
          *reinterpret_cast<float4*>(arow + q * 32 + e4) = make_float4(a4[0], a4[1], a4[2], a4[3]);
        }
      } else {
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          float a4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = col0 + q * 32 + e4 + e;
            const float a = br * __uint_as_float(gv[e4 + e]) * __expf(gr - vg[c]);
            a4[e] = c < r ? a : 0.f;
          }
          *reinterpret_cast<float4*>(arow + q * 32 + e4) = make_float4(a4[0], a4[1], a4[2], a4[3]);
        }
      }
    }
  }
  tc_fence_before();
  // At C = 64 warp w extracted rows 32 w .. + 31 of A, exactly the rows of the
  // two diagonal blocks it solves below; at C = 128 other warps wrote half of them.
  if constexpr (kC == 64) __syncwarp();
  else __syncthreads();

  // 3. T = (I + A)^-1.  Diagonal 16x16 blocks D_b: block 2w + (lane / 16) on
  //    warp w, lane j % 16 owning column j % 16 (half the warps issue this phase,
  //    which leaves the SM's issue slots to the other resident CTAs);
  //    right-looking, so only one multiply-add per step is on the dependency chain.
  if (warp < kC / 32) {  // two diagonal blocks per warp, one per half-warp
    const int o = 16 * (2 * warp + (lane >> 4)), j = lane & 15;
    float col[16], acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      col[i] = 0.f;
      acc[i] = 0.f;
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      col[m] = (m == j) ? 1.f : (m > j ? -acc[m] : 0.f);
#pragma unroll
      for (int i = m + 1; i < 16; ++i) acc[i] = fmaf(Am[(o + i) * kApad + o + m], col[m], acc[i]);
    }
    __syncwarp();  // every lane has read its block of A before T may overwrite it
#pragma unroll
    for (int i = 0; i < 16; ++i) Tm[(o + i) * kApad + o + j] = col[i];
  }
  __syncthreads();
  //    The blocks below the diagonal (tf32 tensor-core products of 16 x 16
  //    tiles).  C = 64, by halves, four dependent levels: with L = I + A split
  //    into 32 x 32 blocks, T = [[T1, 0], [-T2 L21 T1, T2]], where T1, T2 are
  //    the inverses of the diagonal halves, each [[D_a, 0], [-D_b A_ba D_a, D_b]]:
  //      1. A10 D0, A32 D2            2. T10 = -D1 (A10 D0), T32 = -D3 (A32 D2)
  //      3. X = L21 T1 (four tiles)   4. T21 = -T2 X (four tiles)
  //    Scratch tiles sit in A's unused upper blocks.  C = 128 applies the same
  //    split once more: both 64 x 64 halves by the four levels, then
  //    T21 = -T2 (L21 T1) in two levels.
  {
    using FragA = wmma::fragment<wmma::matrix_a, 16, 16, 8, wmma::precision::tf32, wmma::row_major>;
    using FragB = wmma::fragment<wmma::matrix_b, 16, 16, 8, wmma::precision::tf32, wmma::row_major>;
    using FragC = wmma::fragment<wmma::accumulator, 16, 16, 8, float>;
    // acc += X Y for 16 x 16 tiles X, Y (row-major, row stride kApad)
    auto mac = [&](FragC& acc, const float* x, const float* y) {
      FragA fa;
      FragB fb;
#pragma unroll
      for (int kk = 0; kk < 16; kk += 8) {
        wmma::load_matrix_sync(fa, x + kk, kApad);
        wmma::load_matrix_sync(fb, y + kk * kApad, kApad);
        to_tf32(fa);
        to_tf32(fb);
        wmma::mma_sync(acc, fa, fb, acc);
      }
    };
    auto put = [&](float* dst, FragC& acc, bool negate) {
      if (negate) {
#pragma unroll
        for (int t = 0; t < acc.num_elements; ++t) acc.x[t] = -acc.x[t];
      }
      wmma::store_matrix_sync(dst, acc, kApad, wmma::mem_row_major);
    };
    auto At = [&](int i, int j) { return Am + (16 * i) * kApad + 16 * j; };  // also the scratch tiles (j > i)
    auto Tt = [&](int i, int j) { return Tm + (16 * i) * kApad + 16 * j; };
    // Levels 1-4 on the 64 x 64 diagonal block starting at 16 x 16 block b0,
    // by the four warps with local index wl (every thread passes the barriers).
    auto half_solve = [&](int b0, int wl) {
      FragC acc;
      if (wl < 2) {  // level 1: A10 D0 -> S01, A32 D2 -> S23
        const int a = b0 + 2 * wl;
        wmma::fill_fragment(acc, 0.f);
        mac(acc, At(a + 1, a), Tt(a, a));
        put(At(a, a + 1), acc, false);
      }
      __syncwarp();  // level 2 reads back only this warp's level-1 tile
      if (wl < 2) {  // level 2: T10 = -D1 S01, T32 = -D3 S23
        const int a = b0 + 2 * wl;
        wmma::fill_fragment(acc, 0.f);
        mac(acc, Tt(a + 1, a + 1), At(a, a + 1));
        put(Tt(a + 1, a), acc, true);
      }
      __syncthreads();
      {  // level 3: X_rc = sum_m A_rm T1_mc for r in {2, 3}, c in {0, 1} -> S_c(r)
        const int r = b0 + 2 + (wl >> 1), cc = b0 + (wl & 1);
        wmma::fill_fragment(acc, 0.f);
        if (cc == b0) {
          mac(acc, At(r, b0), Tt(b0, b0));
          mac(acc, At(r, b0 + 1), Tt(b0 + 1, b0));
        } else {
          mac(acc, At(r, b0 + 1), Tt(b0 + 1, b0 + 1));
        }
        put(At(cc, r), acc, false);
      }
      __syncthreads();
      {  // level 4: T_rc = -sum_m T2_rm X_mc
        const int r = b0 + 2 + (wl >> 1), cc = b0 + (wl & 1);
        wmma::fill_fragment(acc, 0.f);
        if (r == b0 + 2) {
          mac(acc, Tt(b0 + 2, b0 + 2), At(cc, b0 + 2));
        } else {
          mac(acc, Tt(b0 + 3, b0 + 2), At(cc, b0 + 2));
          mac(acc, Tt(b0 + 3, b0 + 3), At(cc, b0 + 3));
        }
        put(Tt(r, cc), acc, true);
      }
    };
    if constexpr (kC == 64) {
      half_solve(0, warp);
    } else {
      // C = 128: the two 64 x 64 halves at once (warps 0-3 and 4-7), then the
      // block below them, T21 = -T2 (L21 T1), in two more levels of 16 tiles
      // (two per warp, paired so that every warp does five products).
      half_solve(4 * (warp >> 2), warp & 3);
      __syncthreads();
      FragC acc;
      {  // level 5: X_rc = sum_{m=c..3} A_rm T1_mc, r in 4..7, c in 0..3 -> S(c, r)
        const int r = 4 + (warp >> 1);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int cc = (warp & 1) ? 1 + t : 3 * t;
          wmma::fill_fragment(acc, 0.f);
          for (int m = cc; m < 4; ++m) mac(acc, At(r, m), Tt(m, cc));
          put(At(cc, r), acc, false);
        }
      }
      __syncthreads();
      {  // level 6: T_rc = -sum_{m=4..r} T2_rm X_mc
        const int cc = warp >> 1;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int r = (warp & 1) ? 5 + t : 4 + 3 * t;
          wmma::fill_fragment(acc, 0.f);
          for (int m = 4; m <= r; ++m) mac(acc, Tt(r, m), At(cc, m));
          put(Tt(r, cc), acc, true);
        }
      }
    }
  }
  __syncthreads();

  // 4. Tb = T diag(beta) and Tbg = Tb diag(e^g) as bf16 rows; each pass writes
  //    16 rows, consecutive threads covering whole rows (contiguous bytes)
  {
    const size_t tile = ((size_t)bh * nchunks + chunk) * kC * kC;
    constexpr int kTpr = kC / 8;  // threads per row
    const int c8 = (tid % kTpr) * 8;
    // this thread's eight columns of beta (and e^g): 16-byte aligned vector loads
    float bcol[8], ecol[8];
    *reinterpret_cast<float4*>(bcol) = *reinterpret_cast<const float4*>(vb + c8);
    *reinterpret_cast<float4*>(bcol + 4) = *reinterpret_cast<const float4*>(vb + c8 + 4);
    if (GATED) {
      *reinterpret_cast<float4*>(ecol) = *reinterpret_cast<const float4*>(veg + c8);
      *reinterpret_cast<float4*>(ecol + 4) = *reinterpret_cast<const float4*>(veg + c8 + 4);
    }
#pragma unroll
    for (int pass = 0; pass < kC / 16; ++pass) {
      const int row = pass * 16 + tid / kTpr;
      const float* trow = Tm + row * kApad + c8;  // 16-byte aligned (kApad * 4 and c8 * 4 are)
      float t8[8], x[8], y[8];
      *reinterpret_cast<float4*>(t8) = *reinterpret_cast<const float4*>(trow);
      *reinterpret_cast<float4*>(t8 + 4) = *reinterpret_cast<const float4*>(trow + 4);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[e] = c8 + e <= row ? t8[e] * bcol[e] : 0.f;
        if (GATED) y[e] = x[e] * ecol[e];
      }
      st_bf16x8(tb_out + tile + row * kC + c8, x);
      if (GATED) st_bf16x8(tbg_out + tile + row * kC + c8, y);
    }
  }
  if (warp == 0) tmem_dealloc(tmem, kC);  // every TMEM read finished before the last barrier
  // The chunk kernel may begin launching once every CTA got here (it still
  // waits for this grid to complete before reading the factors).
  grid_launch_dependents();
}

template <int C, int DK, bool GATED>
cudaError_t launch_t(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st) {
  const int nchunks = (p.T + C - 1) / C;
  const size_t smem = p.prestep ? TsolveSmem<C, DK, true>::ALLOC : TsolveSmem<C, DK, false>::ALLOC;
  CUtensorMap mk, mq;
  if (!make_tmap_3d_bf16(&mk, p.k, DK, p.T, p.B * p.H) || !make_tmap_3d_bf16(&mq, p.q, DK, p.T, p.B * p.H))
    return cudaErrorInvalidValue;
  auto kern = p.prestep ? tsolve_kernel<C, DK, GATED, true> : tsolve_kernel<C, DK, GATED, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((size_t)nchunks * p.B * p.H));  // at most INT_MAX (checked by the caller)
  kern<<<grid, TsolveShape<C>::kThreads, smem, st>>>(mk, p.beta, mq, p.alpha, w.tb, w.tbg, w.g, w.khat, w.qhat,
                                                      p.T, nchunks, p.status);
  return cudaGetLastError();
}

template <int C>
cudaError_t launch_c(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st) {
  const bool gated = p.alpha != nullptr;
  if (p.Dk == 128) return gated ? launch_t<C, 128, true>(p, w, st) : launch_t<C, 128, false>(p, w, st);
  if (p.Dk == 64) return gated ? launch_t<C, 64, true>(p, w, st) : launch_t<C, 64, false>(p, w, st);
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_tsolve(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st) {
  if (p.C == 64) return launch_c<64>(p, w, st);
  if (p.C == 128) return launch_c<128>(p, w, st);
  return cudaErrorNotSupported;
}

size_t wy_workspace_bytes(int B, int H, int T, int C) {
  const size_t nch = ((size_t)T + C - 1) / C;
  const size_t tiles = (size_t)B * H * nch;
  return tiles * (2 * (size_t)C * C * 2 + (size_t)C * 4);  // Tb, Tbg (bf16) and g (f32)
}

size_t wy_khat_bytes(int B, int H, int T, int Dk) {
  const size_t one = ((size_t)B * H * T * Dk * 2 + 255) / 256 * 256;
  return 2 * one;  // k-hat, then q-hat
}

WyWorkspace wy_carve(void* base, int B, int H, int T, int C, int Dk) {
  const size_t nch = ((size_t)T + C - 1) / C;
  const size_t tiles = (size_t)B * H * nch;
  uint8_t* q = static_cast<uint8_t*>(base);
  WyWorkspace w;
  w.tb = reinterpret_cast<__nv_bfloat16*>(q);
  w.tbg = reinterpret_cast<__nv_bfloat16*>(q + tiles * C * C * 2);
  w.g = reinterpret_cast<float*>(q + 2 * tiles * C * C * 2);
  // mapped keys, then queries (pre-step only): after the factors, on 256-byte boundaries
  w.khat = reinterpret_cast<__nv_bfloat16*>(q + (wy_workspace_bytes(B, H, T, C) + 255) / 256 * 256);
  w.qhat = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(w.khat) + wy_khat_bytes(B, H, T, Dk) / 2);
  return w;
}

}  // namespace dn
