// Warp-specialised tcgen05 chunked DeltaNet forward (bf16 operands, float32
// accumulation and state): the bf16 path of deltanet_chunk_fwd.
//
// Method (per chunk of C = 64 rows entered with state S; g_r = sum_{j<=r} log
// alpha_j, Gamma_rs = exp(g_r - g_s) for s <= r, gamma_r = exp(g_r)):
//   G  = [K;Q] K^T                      -> A = strict_lower(diag(beta) KK^T * Gamma),
//                                          P = tril(QK^T) * Gamma
//   T  = (I + A)^-1,  Tb = T diag(beta), Tbg = Tb diag(gamma)
//   W  = Tbg K,  Uh = Tb V              (S-independent)
//   [QS; WS] = [Q; W] S,  U = Uh - WS   (the chunk's deltas)
//   O  = diag(gamma) QS + P U,  S <- gamma_last S + K^T (diag(Gamma_last,.) U)
// the Householder / WY reparameterisation of the delta rule ("GPT-2 から Kimi K3
// まで", news.ainew.jp, section "DeltaNet (Parallelizing linear transformers with
// delta rule)"; gate from the Gated DeltaNet paragraph of "How a Baseten
// Engineer Traced 7 Years of Attention Mechanism Evolution").
//
// One CTA per (b, h, 64-column slice of Dv); 9 warps in three roles so that
// the state-independent work of chunk c+1 overlaps the state chain of chunk c:
//   warps 0-3  chain: [Q;W]S, U, PU and K^T U MMAs, outputs, state update
//   warps 4-7  prep:  Gram MMA, A and P tiles, T = (I + A)^-1, Tb, W and Uh
//   warp  8    producer: TMA loads of q, k, v into a two-stage ring
// Both compute groups cover TMEM lanes 0-127.  Handoffs use mbarriers:
// full/empty (TMA ring), ready (prep -> chain), free (chain -> prep, guarding
// the per-parity buffers P, Uh and the decay vectors).  All waits are bounded.
//
// T-solve: the four 16x16 diagonal blocks of I + A are inverted by forward
// substitution (one column per lane, float32), then merged 16 -> 32 -> 64 with
// tf32 tensor-core products (T_ij = -T_ii A_ij T_jj, T21 = -T22 A21 T11); T is
// rounded to bf16 afterwards, so tf32 merges cost no accuracy that matters.
#include <cuda.h>
#include <cuda_bf16.h>
#include <mma.h>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

using namespace nvcuda;

constexpr int kC = 64;
constexpr int kDVS = 64;
constexpr uint32_t kTile = 8192;  // 64 rows x 128 bytes
constexpr int kWG = 128;
constexpr int kThreads = 2 * kWG + 32;
constexpr int kApad = 68;  // float row stride of the A / T scratch (16-byte and 32-byte friendly)
constexpr int kBarChain = 1, kBarPrep = 2;

// TMEM columns (512 allocated)
constexpr uint32_t TM_G = 0, TM_W = 64, TM_UH = 192, TM_QW = 320, TM_PU = 384, TM_DS = 448;

template <int DK>
struct WsLayout {
  static constexpr int KB = DK / 64;
  static constexpr uint32_t KB_STRIDE = 3 * kTile;  // [K | Q | W] per 64-column block of Dk
  static constexpr uint32_t K_OFF = 0, Q_OFF = kTile, W_OFF = 2 * kTile;
  static constexpr uint32_t V_OFF = KB * KB_STRIDE;
  static constexpr uint32_t STAGE = KB * KB_STRIDE + kTile;
  static constexpr uint32_t P_OFF = 2 * STAGE;  // P0 | P1 | Tb | Tbg | U | UT
  static constexpr uint32_t TB_OFF = P_OFF + 2 * kTile;
  static constexpr uint32_t TBG_OFF = TB_OFF + kTile;
  static constexpr uint32_t U_OFF = TBG_OFF + kTile;
  static constexpr uint32_t UT_OFF = U_OFF + kTile;
  static constexpr uint32_t S_OFF = UT_OFF + kTile;  // bf16 state, DK rows x 128 B
  static constexpr uint32_t AM_OFF = S_OFF + DK * 128;
  static constexpr uint32_t TM_OFF = AM_OFF + 64 * kApad * 4;
  static constexpr uint32_t VEC_OFF = TM_OFF + 64 * kApad * 4;  // [2 parities][beta, g, e^g, pad][64]
  static constexpr uint32_t BAR_OFF = VEC_OFF + 2 * 4 * 64 * 4;
  static constexpr uint32_t BYTES = BAR_OFF + 128;
  static constexpr uint32_t ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// mbarrier slots (byte offsets from BAR_OFF)
constexpr uint32_t B_FULL = 0, B_EMPTY = 16, B_READY = 32, B_FREE = 48, B_PMMA = 64, B_CMMA = 72,
                   B_FINP = 80, B_FINC = 88, B_TMEM = 96, B_ABORT = 100;

template <typename Frag>
__device__ __forceinline__ void to_tf32(Frag& f) {
#pragma unroll
  for (int t = 0; t < f.num_elements; ++t) f.x[t] = wmma::__float_to_tf32(f.x[t]);
}

template <int DK, bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_ws_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const ChunkProblem p) {
  using L = WsLayout<DK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int j0 = blockIdx.y * kDVS;
  const int T = p.T, Dv = p.Dv;
  const int nchunks = (T + kC - 1) / kC;
  const uint32_t bar = sb + L::BAR_OFF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::BAR_OFF + B_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::BAR_OFF + B_ABORT);
  float* Am = reinterpret_cast<float*>(sm + L::AM_OFF);
  float* Tm = reinterpret_cast<float*>(sm + L::TM_OFF);
  float* vec = reinterpret_cast<float*>(sm + L::VEC_OFF);  // vec + b*256 + {0: beta, 64: g, 128: e^g}

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + B_FULL + 8 * i, 1);
      mbar_init(bar + B_EMPTY + 8 * i, 1);
      mbar_init(bar + B_READY + 8 * i, 1);
      mbar_init(bar + B_FREE + 8 * i, 1);
    }
    mbar_init(bar + B_PMMA, 1);
    mbar_init(bar + B_CMMA, 1);
    mbar_init(bar + B_FINP, 1);
    mbar_init(bar + B_FINC, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // T's strictly-upper 16x16 blocks stay zero: the merges read T11 and T22 whole.
  for (int i = tid; i < 64 * 64; i += kThreads) {
    const int r = i >> 6, c = i & 63;
    if ((c >> 4) > (r >> 4)) Tm[r * kApad + c] = 0.f;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, kWaitLimitNs};
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, use = c >> 1;
        if (use > 0 && !mbar_wait(bar + B_EMPTY + 8 * s, (use - 1) & 1, wc)) break;
        const uint32_t st = sb + s * L::STAGE;
        const uint32_t full = bar + B_FULL + 8 * s;
        mbar_expect_tx(full, (2 * L::KB + 1) * kTile);
#pragma unroll
        for (int kb = 0; kb < L::KB; ++kb) {
          tma_load_3d(st + kb * L::KB_STRIDE + L::K_OFF, &tmK, full, kb * 64, c * kC, bh);
          tma_load_3d(st + kb * L::KB_STRIDE + L::Q_OFF, &tmQ, full, kb * 64, c * kC, bh);
        }
        tma_load_3d(st + L::V_OFF, &tmV, full, j0, c * kC, bh);
        issued = c + 1;
      }
      int zero = 0;
      const WaitCtl drain{&zero, p.status, kWaitLimitNs};
      for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c)
        (void)mbar_wait(bar + B_FULL + 8 * (c & 1), (c >> 1) & 1, drain);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- prep --
    const int pt = tid - kWG;
    const int row = pt & 63;
    const int wp = warp & 3;
    uint32_t mph = 0;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1, use = c >> 1;
      const int c0 = c * kC, n = min(kC, T - c0);
      const uint32_t st = sb + b * L::STAGE;
      uint8_t* stp = sm + b * L::STAGE;
      float* vb = vec + b * 256;
      if (c >= 2) {  // the chain is done with this parity's P, Uh and vectors
        ok = named_bar_and(kBarPrep, kWG, mbar_wait(bar + B_FREE + 8 * b, (use - 1) & 1, wc));
        if (!ok) break;
      }
      if (pt < 64) {
        const size_t tb = (size_t)bh * T + c0;
        vb[pt] = pt < n ? p.beta[tb + pt] : 0.f;
        if (GATED) {
          float x = pt < n ? fmaxf(__logf(p.alpha[tb + pt]), -87.f) : 0.f;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
          }
          if (wp == 1) {
            float l0 = lane < n ? fmaxf(__logf(p.alpha[tb + lane]), -87.f) : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            x += l0;
          }
          vb[64 + pt] = x;
          vb[128 + pt] = __expf(x);
        }
      }
      ok = named_bar_and(kBarPrep, kWG, mbar_wait(bar + B_FULL + 8 * b, use & 1, wc));
      if (!ok) break;

      // ---- Gram: G = [K;Q] K^T (lanes 0-63 KK^T, lanes 64-127 QK^T) ----
      if (pt == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t a = st + (ks >> 2) * L::KB_STRIDE + L::K_OFF + (ks & 3) * 32;
          mma_bf16_ss(tmem + TM_G, desc_k(a), desc_k(a), id, ks > 0);
        }
        mma_commit(bar + B_PMMA);
      }
      ok = named_bar_and(kBarPrep, kWG, mbar_wait(bar + B_PMMA, mph & 1, wc));
      ++mph;
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t g[64];
        tmem_ld32(tmem + lane_base + TM_G, *reinterpret_cast<uint32_t(*)[32]>(g));
        tmem_ld32(tmem + lane_base + TM_G + 32, *reinterpret_cast<uint32_t(*)[32]>(g + 32));
        tmem_wait_ld();
        const float gr = GATED ? vb[64 + row] : 0.f;
        if (pt < 64) {  // A row
          const float br = vb[row];
          float* arow = Am + row * kApad;
#pragma unroll
          for (int s4 = 0; s4 < 64; s4 += 4) {
            float a4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int sc = s4 + e;
              float val = br * __uint_as_float(g[sc]);
              if (GATED) val *= __expf(gr - vb[64 + sc]);
              a4[e] = sc < row ? val : 0.f;
            }
            *reinterpret_cast<float4*>(arow + s4) = make_float4(a4[0], a4[1], a4[2], a4[3]);
          }
        } else {  // P row
          uint8_t* ptile = sm + L::P_OFF + b * kTile;
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int sc = c16 * 8 + e;
              float val = __uint_as_float(g[sc]);
              if (GATED) val *= __expf(gr - vb[64 + sc]);
              x[e] = sc <= row ? val : 0.f;
            }
            st_bf16x8(ptile + sw128_off(row, c16), x);
          }
        }
      }
      named_bar_sync(kBarPrep, kWG);

      // ---- T = (I + A)^-1, step 1: 16x16 diagonal blocks (lanes 0-15: one column each) ----
      if (lane < 16) {
        const int o = 16 * wp, j = lane;
        float col[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) col[k] = (k == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 1; i < 16; ++i) {
          const float* ar = Am + (o + i) * kApad + o;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int m4 = 0; m4 < i; m4 += 4) {
            const float4 a = *reinterpret_cast<const float4*>(ar + m4);
            a0 = fmaf(a.x, col[m4], a0);
            a1 = fmaf(a.y, col[m4 + 1], a1);
            a2 = fmaf(a.z, col[m4 + 2], a2);
            a3 = fmaf(a.w, col[m4 + 3], a3);
          }
          if (i > j) col[i] = -((a0 + a1) + (a2 + a3));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[(o + i) * kApad + o + j] = col[i];
      }
      named_bar_sync(kBarPrep, kWG);
      // ---- step 2: T_{r,r-1} = -D_r A_{r,r-1} D_{r-1} for r = 1, 3 (warps 0 and 2) ----
      if ((wp & 1) == 0) {
        const int o = 16 * (wp + 1), q0 = o - 16;
        float* ys = Am + (wp == 0 ? 0 : 16) * kApad + 48;  // scratch: strictly-upper part of A
        wmma::fragment<wmma::matrix_a, 16, 16, 8, wmma::precision::tf32, wmma::row_major> fa;
        wmma::fragment<wmma::matrix_b, 16, 16, 8, wmma::precision::tf32, wmma::row_major> fb;
        wmma::fragment<wmma::accumulator, 16, 16, 8, float> acc;
        wmma::fill_fragment(acc, 0.f);
#pragma unroll
        for (int kk = 0; kk < 16; kk += 8) {
          wmma::load_matrix_sync(fa, Am + o * kApad + q0 + kk, kApad);
          wmma::load_matrix_sync(fb, Tm + (q0 + kk) * kApad + q0, kApad);
          to_tf32(fa);
          to_tf32(fb);
          wmma::mma_sync(acc, fa, fb, acc);
        }
        wmma::store_matrix_sync(ys, acc, kApad, wmma::mem_row_major);
        __syncwarp();
        wmma::fill_fragment(acc, 0.f);
#pragma unroll
        for (int kk = 0; kk < 16; kk += 8) {
          wmma::load_matrix_sync(fa, Tm + o * kApad + o + kk, kApad);
          wmma::load_matrix_sync(fb, ys + kk * kApad, kApad);
          to_tf32(fa);
          to_tf32(fb);
          wmma::mma_sync(acc, fa, fb, acc);
        }
#pragma unroll
        for (int t = 0; t < acc.num_elements; ++t) acc.x[t] = -acc.x[t];
        wmma::store_matrix_sync(Tm + o * kApad + q0, acc, kApad, wmma::mem_row_major);
      }
      named_bar_sync(kBarPrep, kWG);
      // ---- step 3: Y = A21 T11 (one 16x16 tile per warp), then T21 = -T22 Y ----
      {
        const int ti = wp >> 1, tj = wp & 1;
        wmma::fragment<wmma::matrix_a, 16, 16, 8, wmma::precision::tf32, wmma::row_major> fa;
        wmma::fragment<wmma::matrix_b, 16, 16, 8, wmma::precision::tf32, wmma::row_major> fb;
        wmma::fragment<wmma::accumulator, 16, 16, 8, float> acc;
        wmma::fill_fragment(acc, 0.f);
#pragma unroll
        for (int kk = 0; kk < 32; kk += 8) {
          wmma::load_matrix_sync(fa, Am + (32 + 16 * ti) * kApad + kk, kApad);
          wmma::load_matrix_sync(fb, Tm + kk * kApad + 16 * tj, kApad);
          to_tf32(fa);
          to_tf32(fb);
          wmma::mma_sync(acc, fa, fb, acc);
        }
        wmma::store_matrix_sync(Am + (16 * ti) * kApad + 32 + 16 * tj, acc, kApad,
                                wmma::mem_row_major);
        named_bar_sync(kBarPrep, kWG);
        wmma::fill_fragment(acc, 0.f);
#pragma unroll
        for (int kk = 0; kk < 32; kk += 8) {
          wmma::load_matrix_sync(fa, Tm + (32 + 16 * ti) * kApad + 32 + kk, kApad);
          wmma::load_matrix_sync(fb, Am + kk * kApad + 32 + 16 * tj, kApad);
          to_tf32(fa);
          to_tf32(fb);
          wmma::mma_sync(acc, fa, fb, acc);
        }
#pragma unroll
        for (int t = 0; t < acc.num_elements; ++t) acc.x[t] = -acc.x[t];
        wmma::store_matrix_sync(Tm + (32 + 16 * ti) * kApad + 16 * tj, acc, kApad,
                                wmma::mem_row_major);
      }
      named_bar_sync(kBarPrep, kWG);
      // ---- Tb = T diag(beta), Tbg = Tb diag(gamma): row `row`, columns [32h, 32h + 32) ----
      {
        const int h = pt >> 6;
        const float* trow = Tm + row * kApad;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c16 = h * 4 + cc;
          const float4 t0 = *reinterpret_cast<const float4*>(trow + c16 * 8);
          const float4 t1 = *reinterpret_cast<const float4*>(trow + c16 * 8 + 4);
          const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
          float x[8], y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int sc = c16 * 8 + e;
            x[e] = sc <= row ? tv[e] * vb[sc] : 0.f;
            if (GATED) y[e] = x[e] * vb[128 + sc];
          }
          st_bf16x8(sm + L::TB_OFF + sw128_off(row, c16), x);
          if (GATED) st_bf16x8(sm + L::TBG_OFF + sw128_off(row, c16), y);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarPrep, kWG);

      // ---- W = Tbg K (lanes 0-63), Uh = Tb V (lanes 64-127, parity buffer) ----
      if (pt == 0) {
        tc_fence_after();
        const uint32_t aw = sb + (GATED ? L::TBG_OFF : L::TB_OFF);
        const uint32_t au = sb + L::P_OFF + kTile;  // [P1; Tb]: rows 64-127 are Tb
        constexpr uint32_t idw = idesc_bf16(128, DK, false, true);
        constexpr uint32_t idu = idesc_bf16(128, 64, false, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_bf16_ss(tmem + TM_W, desc_k(aw + ks * 32),
                      desc_mn(st + L::K_OFF + ks * 2048, L::KB_STRIDE), idw, ks > 0);
          mma_bf16_ss(tmem + TM_UH + 64 * b, desc_k(au + ks * 32),
                      desc_mn(st + L::V_OFF + ks * 2048, kTile), idu, ks > 0);
        }
        mma_commit(bar + B_PMMA);
      }
      ok = named_bar_and(kBarPrep, kWG, mbar_wait(bar + B_PMMA, mph & 1, wc));
      ++mph;
      if (!ok) break;
      tc_fence_after();
      if (pt < 64) {  // W rows -> bf16, next to Q in the stage
#pragma unroll
        for (int q = 0; q < DK / 32; ++q) {
          uint32_t w[32];
          tmem_ld32(tmem + lane_base + TM_W + q * 32, w);
          tmem_wait_ld();
          uint8_t* wt = stp + (q >> 1) * L::KB_STRIDE + L::W_OFF;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            st_bf16x8(wt + sw128_off(row, (q & 1) * 4 + cc),
                      reinterpret_cast<const float*>(w) + cc * 8);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarPrep, kWG);
      if (pt == 0) mbar_arrive(bar + B_READY + 8 * b);
    }
    if (pt == 0) {  // no MMA of this thread may outlive TMEM
      tc_fence_after();
      mma_commit(bar + B_FINP);
      int zero = 0;
      const WaitCtl fin{&zero, p.status, kWaitLimitNs};
      (void)mbar_wait(bar + B_FINP, 0, fin);
    }
  } else {
    // --------------------------------------------------------------- chain --
    const int ct = tid;
    const int row = ct & 63;
    const size_t s_base = (size_t)bh * DK * Dv;
    float sreg[kDVS];
    if (ct < DK) {
      const float* src = p.S0 ? p.S0 + s_base + (size_t)ct * Dv + j0 : nullptr;
#pragma unroll
      for (int j = 0; j < kDVS; j += 4) {
        const float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        sreg[j] = v.x; sreg[j + 1] = v.y; sreg[j + 2] = v.z; sreg[j + 3] = v.w;
      }
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) st_bf16x8(sm + L::S_OFF + sw128_off(ct, c16), sreg + 8 * c16);
    }
    fence_proxy_async_smem();
    named_bar_sync(kBarChain, kWG);

    uint32_t mph = 0;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1, use = c >> 1;
      const int c0 = c * kC, n = min(kC, T - c0);
      const uint32_t st = sb + b * L::STAGE;
      const float* vb = vec + b * 256;
      ok = named_bar_and(kBarChain, kWG, mbar_wait(bar + B_READY + 8 * b, use & 1, wc));
      if (!ok) break;
      tc_fence_after();

      // ---- [QS; WS] = [Q; W] S ----
      if (ct == 0) {
        constexpr uint32_t id = idesc_bf16(128, 64, false, true);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t a = st + (ks >> 2) * L::KB_STRIDE + L::Q_OFF + (ks & 3) * 32;
          mma_bf16_ss(tmem + TM_QW, desc_k(a), desc_mn(sb + L::S_OFF + ks * 2048, kTile), id, ks > 0);
        }
        mma_commit(bar + B_CMMA);
      }
      ok = named_bar_and(kBarChain, kWG, mbar_wait(bar + B_CMMA, mph & 1, wc));
      ++mph;
      if (!ok) break;
      tc_fence_after();

      // ---- U = Uh - WS (rows on lanes 64-127) ----
      if (ct >= 64) {
        const float wl = GATED ? __expf(vb[64 + n - 1] - vb[64 + row]) : 1.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t ws[32], uh[32];
          tmem_ld32(tmem + lane_base + TM_QW + q * 32, ws);
          tmem_ld32(tmem + lane_base + TM_UH + 64 * b + q * 32, uh);
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float x[8], y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              x[e] = __uint_as_float(uh[cc * 8 + e]) - __uint_as_float(ws[cc * 8 + e]);
              y[e] = x[e] * wl;
            }
            st_bf16x8(sm + L::U_OFF + sw128_off(row, q * 4 + cc), x);
            if (GATED) st_bf16x8(sm + L::UT_OFF + sw128_off(row, q * 4 + cc), y);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarChain, kWG);

      // ---- PU = [P; .] U (lanes 0-63), dS = K^T U~ ----
      if (ct == 0) {
        tc_fence_after();
        const uint32_t ut = sb + (GATED ? L::UT_OFF : L::U_OFF);
        const uint32_t pa = sb + L::P_OFF + b * kTile;
        constexpr uint32_t idp = idesc_bf16(128, 64, false, true);
        constexpr uint32_t ids = idesc_bf16(128, 64, true, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_bf16_ss(tmem + TM_PU, desc_k(pa + ks * 32), desc_mn(sb + L::U_OFF + ks * 2048, kTile),
                      idp, ks > 0);
          mma_bf16_ss(tmem + TM_DS, desc_mn(st + L::K_OFF + ks * 2048, L::KB_STRIDE),
                      desc_mn(ut + ks * 2048, kTile), ids, ks > 0);
        }
        mma_commit(bar + B_CMMA);
        mma_commit(bar + B_EMPTY + 8 * b);
      }
      ok = named_bar_and(kBarChain, kWG, mbar_wait(bar + B_CMMA, mph & 1, wc));
      ++mph;
      if (!ok) break;
      tc_fence_after();

      // ---- outputs (lanes 0-63) and the state update ----
      if (ct < 64) {
        const float gam = GATED ? vb[128 + row] : 1.f;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + ((size_t)bh * T + c0 + row) * Dv + j0;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t qs[32], pu[32];
          tmem_ld32(tmem + lane_base + TM_QW + q * 32, qs);
          tmem_ld32(tmem + lane_base + TM_PU + q * 32, pu);
          tmem_wait_ld();
          if (row < n) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              float x[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                x[e] = fmaf(gam, __uint_as_float(qs[cc * 8 + e]), __uint_as_float(pu[cc * 8 + e]));
              st_bf16x8(orow + q * 32 + cc * 8, x);
            }
          }
        }
      }
      if (ct < DK) {
        const float carry = GATED ? vb[128 + n - 1] : 1.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t ds[32];
          tmem_ld32(tmem + lane_base + TM_DS + q * 32, ds);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) sreg[q * 32 + e] = fmaf(carry, sreg[q * 32 + e], __uint_as_float(ds[e]));
        }
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) st_bf16x8(sm + L::S_OFF + sw128_off(ct, c16), sreg + 8 * c16);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarChain, kWG);
      if (ct == 0) mbar_arrive(bar + B_FREE + 8 * b);
    }
    if (p.S_out && ct < DK) {
      float* dst = p.S_out + s_base + (size_t)ct * Dv + j0;
#pragma unroll
      for (int j = 0; j < kDVS; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
    }
    if (ct == 0) {
      tc_fence_after();
      mma_commit(bar + B_FINC);
      int zero = 0;
      const WaitCtl fin{&zero, p.status, kWaitLimitNs};
      (void)mbar_wait(bar + B_FINC, 0, fin);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DK, bool GATED>
cudaError_t launch_t(const ChunkProblem& p, cudaStream_t st) {
  using L = WsLayout<DK>;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_tmap_3d_bf16(&mq, p.q, DK, p.T, BH) || !make_tmap_3d_bf16(&mk, p.k, DK, p.T, BH) ||
      !make_tmap_3d_bf16(&mv, p.v, p.Dv, p.T, BH))
    return cudaErrorInvalidValue;
  auto kern = chunk_ws_kernel<DK, GATED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)BH, (unsigned)(p.Dv / kDVS));
  kern<<<grid, kThreads, L::ALLOC, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

bool chunk_ws_supported(const ChunkProblem& p) {
  return p.bf16 && p.mode == Mode::Delta && p.T > 0 && p.C == 64 && (p.Dk == 64 || p.Dk == 128) &&
         (p.Dv == 64 || p.Dv == 128);
}

cudaError_t launch_chunk_ws(const ChunkProblem& p, cudaStream_t st) {
  const bool gated = p.alpha != nullptr;
  if (p.Dk == 128) return gated ? launch_t<128, true>(p, st) : launch_t<128, false>(p, st);
  return gated ? launch_t<64, true>(p, st) : launch_t<64, false>(p, st);
}

}  // namespace dn
