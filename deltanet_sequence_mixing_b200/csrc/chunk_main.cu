// tcgen05 chunked DeltaNet forward (bf16 operands, float32 accumulation and
// state): the bf16 path of deltanet_chunk_fwd, run after the chunk-parallel
// WY pre-pass (tsolve.cu) has written Tb = (I + A)^-1 diag(beta), Tbg =
// Tb diag(gamma) and the decay prefix g of every chunk into the workspace.
//
// Per chunk of C = 64 rows entered with state S ("GPT-2 から Kimi K3 まで",
// news.ainew.jp, section "DeltaNet (Parallelizing linear transformers with delta
// rule)"; gate from the Gated DeltaNet paragraph of "How a Baseten Engineer
// Traced 7 Years of Attention Mechanism Evolution"):
//   P  = tril(Q K^T) * Gamma,  W = Tbg K,  Uh = Tb V          (state-independent)
//   [Q S ; W S] = [Q ; W] S                                    (one M = 128 MMA)
//   U  = Uh - W S                                              (the chunk's deltas)
//   O  = diag(gamma) Q S + P U  (Q S rows scaled in TMEM, then P U
//                                accumulated onto the same tile)
//   S <- gamma_last S + K^T (diag(Gamma_last,.) U)             (float32 registers)
//
// One CTA per (b, h, slice of DVS = 64 columns of Dv; 32 when 64-column
// slices would leave most SMs idle and 32-column ones still fit one wave),
// 10 warps:
//   warp 9     MMA issuer (warp-uniform, one elected lane issues): every
//              tcgen05.mma of the CTA, in a fixed order that keeps the state
//              chain fed:
//                [Q;W]S (c), W/Uh (c+1), K^T U (c), PU (c), QK^T (c+1)
//              (gated: W (c+1) before K^T U (c), Uh (c+1) after it)
//              W/Uh (c+1) runs while the U epilogue of chunk c drains (Uh is
//              double-buffered in TMEM); PU (c) and QK^T (c+1) run during the
//              state update.  The single P tile is rewritten only after PU (c)
//              has completed (QK^T (c+1) is committed after it).
//   warp 8     producer: TMA of K, Q, V, Tb (gated: Tbg and the g rows) into
//              a three-stage ring (gated: two), L2 prefetch two chunks ahead
//   warps 6-7  W rows to bf16 next to Q (state-independent, one chunk ahead),
//              then columns 32-63 of the U epilogue
//   warps 4-5  P rows to bf16 (gated: with the decay Gamma)
//   warps 2-3  U = Uh - WS (columns 0-31);   warps 0-3 the state update;
//   warps 0-1  gated: QS rows times gamma in TMEM while the U epilogue runs;
//              drain the output tile O = diag(gamma) QS + PU
// Epilogue warps only wait on mbarriers signalled by tcgen05.commit and
// signal back; the issuer waits on their signals.  Every mbarrier completes
// once per chunk (or per use of a parity), so parity waits are unambiguous.
// Accumulators live in TMEM (512 columns), every operand in the 128-byte-
// swizzled canonical layout, the running state in float32 registers.  All
// waits are bounded; a wait that runs out sets the workspace status word and
// the CTA winds down (copies drained, TMEM freed) without trapping.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

constexpr int kC = 64;
constexpr uint32_t kTile = 8192;  // 64 rows x 128 bytes
constexpr int kWG = 128;
constexpr int kThreads = 2 * kWG + 64;  // chain 0-3, prep 4-7, producer 8, issuer 9
constexpr int kBarChain = 1, kBarChainHi = 2, kBarChainLo = 3, kBarPrepP = 4, kBarPrepW = 5;

// TMEM columns: G (P scores), W, Uh[0], QW[2] (lanes 0-63: O, lanes 64-127: WS),
// dS, Uh[1].  Uh[0] sits right after W (at TM_W + Dk) so that, ungated and for
// even chunks, one N = Dk + 64 product writes both.
constexpr uint32_t TM_G = 0, TM_W = 64, TM_QW = 256, TM_DS = 384, TM_UH1 = 448;

// Shared memory.  A stage holds one chunk's TMA tiles [K | Q | W] per 64
// columns of Dk, V, Tb (gated also Tbg and the g rows); W is written there
// by the W warps, right after Q, so that [Q; W] is one M = 128 operand.
// Ungated runs a three-stage ring (the chunk after next streams in while one
// chunk is on the state chain and the next is being prepared); gated needs
// the Tbg tile, the decay-weighted U and the g rows, and fits two stages.
template <int DK, bool GATED>
struct MainLayout {
  static constexpr int KB = DK / 64;
  static constexpr int NST = GATED ? 2 : 3;           // ring stages
  static constexpr uint32_t KB_STRIDE = 3 * kTile;    // [K | Q | W] per 64 columns of Dk
  static constexpr uint32_t K_OFF = 0, Q_OFF = kTile, W_OFF = 2 * kTile;
  static constexpr uint32_t V_OFF = KB * KB_STRIDE;   // V | Tb | (Tbg | beta, g)
  static constexpr uint32_t TB_OFF = V_OFF + kTile;
  static constexpr uint32_t TBG_OFF = TB_OFF + kTile;
  static constexpr uint32_t VEC_OFF = TBG_OFF + kTile;
  static constexpr uint32_t STAGE = GATED ? VEC_OFF + 1024 : TBG_OFF;
  static constexpr uint32_t P_OFF = NST * STAGE;      // P | U | (UT)
  static constexpr uint32_t U_OFF = P_OFF + kTile;
  static constexpr uint32_t UT_OFF = U_OFF + kTile;
  static constexpr uint32_t S_OFF = U_OFF + (GATED ? 2 : 1) * kTile;  // bf16 state, DK rows x 128 B
  static constexpr uint32_t CV_OFF = S_OFF + DK * 128;  // gated: chain copy of g per parity, [2][64]
  static constexpr uint32_t BAR_OFF = CV_OFF + (GATED ? 2 * 64 * 4 : 0);
  static constexpr uint32_t BYTES = BAR_OFF + 256;
  static constexpr uint32_t ALLOC = BYTES + 1024;
  static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned (128-byte swizzle atoms)");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// mbarrier slots (8 bytes each).  FULL and EMPTY: one per ring stage;
// OFREE, CMMA5 and PREADY: one per chunk parity.
constexpr uint32_t B_FULL = 0, B_EMPTY = 24, B_OFREE = 48, B_CMMA5 = 64, B_PREADY = 80,
                   B_CMMA3 = 96, B_CMMA4 = 104, B_PMMA1 = 112, B_PMMA2 = 120, B_UREADY = 128,
                   B_SREADY = 136, B_WREADY = 144, B_FIN = 152, B_TMEM = 160, B_ABORT = 164, B_QSCALED = 168;

// One half (32 columns, [col0, col0 + 32)) of the U epilogue for the row on
// this thread's TMEM lane: U = Uh - WS to bf16 (gated also U~ = U e^(g_last - g_row)).
template <bool GATED>
__device__ __forceinline__ void u_epilogue_half(uint32_t ws_addr, uint32_t uh_addr, int col0, int row, float wl,
                                                uint8_t* u_tile, uint8_t* ut_tile) {
  uint32_t ws[32], uh[32];
  tmem_ld32(ws_addr + col0, ws);
  tmem_ld32(uh_addr + col0, uh);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float x[8], y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[e] = __uint_as_float(uh[q * 8 + e]) - __uint_as_float(ws[q * 8 + e]);
      y[e] = x[e] * wl;
    }
    const int c16 = col0 / 8 + q;
    st_bf16x8(u_tile + sw128_off(row, c16), x);
    if (GATED) st_bf16x8(ut_tile + sw128_off(row, c16), y);
  }
}

// HOM: the homogeneous chain of the sequence split (v = 0, S0 = I); a
// template switch, so that the plain kernels carry none of its code.
template <int DK, bool GATED, int DVS, bool HOM>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmTb,
                      const __grid_constant__ CUtensorMap tmTbg, const ChunkProblem p,
                      const float* __restrict__ gw) {
  using L = MainLayout<DK, GATED>;
  constexpr int NST = L::NST;
  constexpr uint32_t TM_UH0 = TM_W + DK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = warp_uniform(smem_u32(sm));
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = (int)warp_uniform((uint32_t)tid >> 5);  // role branches stay warp-uniform
  // 1-D grid with the D_v slices of a head adjacent: they are scheduled
  // together, so the second slice's K, Q (and pre-pass) tiles come from L2
  // even when the grid takes more than one wave.
  const int nsl = p.Dv / DVS;
  const int bh = blockIdx.x / nsl, slice = blockIdx.x % nsl;
  const int j0 = slice * DVS;
  // V comes as the 64-column box holding the slice; a 32-column slice starts
  // 64 bytes into the box's 128-byte rows when it is the box's second half
  const int jv = j0 & ~63;
  const uint32_t vcol = (uint32_t)(j0 & 63) * 2;
  const int T = p.T, Dv = p.Dv;
  const int nchunks = (T + kC - 1) / kC;
  const uint32_t bar = sb + L::BAR_OFF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::BAR_OFF + B_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::BAR_OFF + B_ABORT);
  float* cvec = reinterpret_cast<float*>(sm + L::CV_OFF);

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(bar + B_FULL + 8 * i, 2);  // TMA bytes + the producer's arrival (after the g rows)
      mbar_init(bar + B_EMPTY + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + B_OFREE + 8 * i, 1);
      mbar_init(bar + B_CMMA5 + 8 * i, 1);
      mbar_init(bar + B_PREADY + 8 * i, 1);
    }
    mbar_init(bar + B_CMMA3, 1);
    mbar_init(bar + B_CMMA4, 1);
    mbar_init(bar + B_PMMA1, 1);
    mbar_init(bar + B_PMMA2, 1);
    mbar_init(bar + B_UREADY, DVS / 32);  // the column halves of the U epilogue
    mbar_init(bar + B_SREADY, 1);
    mbar_init(bar + B_WREADY, 1);
    mbar_init(bar + B_QSCALED, 1);  // gated: the QS rows of TM_QW scaled by gamma
    mbar_init(bar + B_FIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (HOM) {  // the homogeneous chain: V is zero (no copy ever lands on these tiles)
    for (int s = 0; s < NST; ++s)
      for (int i = tid; i < (int)(kTile / 16); i += kThreads)
        *reinterpret_cast<uint4*>(sm + s * L::STAGE + L::V_OFF + i * 16) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = warp_uniform(*tmem_slot);
  const WaitCtl wc{abort_flag, p.status, kWaitLimitNs};
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tile_bytes = (2 * L::KB + (GATED ? 3 : 2) - (HOM ? 1 : 0)) * kTile;

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmTb);
      if (GATED) prefetch_tmap(&tmTbg);
    }
    // Tb, Tbg and g come from the pre-pass launched just before this kernel
    grid_dependency_wait();
    int issued = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int s = c % NST, use = c / NST;
      const int c0 = c * kC, n = min(kC, T - c0);
      bool ok = true;
      if (lane == 0 && use > 0) ok = mbar_wait(bar + B_EMPTY + 8 * s, (use - 1) & 1, wc);
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
      const uint32_t st = sb + s * L::STAGE;
      const uint32_t full = bar + B_FULL + 8 * s;
      if (lane == 0) {
        mbar_expect_tx(full, tile_bytes);
#pragma unroll
        for (int kb = 0; kb < L::KB; ++kb) {
          tma_load_3d(st + kb * L::KB_STRIDE + L::K_OFF, &tmK, full, kb * 64, c0, bh);
          tma_load_3d(st + kb * L::KB_STRIDE + L::Q_OFF, &tmQ, full, kb * 64, c0, bh);
        }
        if (!HOM) tma_load_3d(st + L::V_OFF, &tmV, full, jv, c0, bh);
        tma_load_3d(st + L::TB_OFF, &tmTb, full, 0, c0, bh);
        if (GATED) tma_load_3d(st + L::TBG_OFF, &tmTbg, full, 0, c0, bh);
      }
      if (GATED) {  // g rows of the chunk (rows >= n: g flat); beta is folded into Tb
        float* vs = reinterpret_cast<float*>(sm + s * L::STAGE + L::VEC_OFF);
#pragma unroll
        for (int h = 0; h < 2; ++h) vs[64 + lane + 32 * h] = gw[((size_t)bh * nchunks + c) * kC + lane + 32 * h];
      }
      (void)n;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(full);
        if (c + 2 < nchunks) {  // warm L2 for the chunk after next
          const int cn = c0 + 2 * kC;
#pragma unroll
          for (int kb = 0; kb < L::KB; ++kb) {
            prefetch_l2_3d(&tmK, kb * 64, cn, bh);
            prefetch_l2_3d(&tmQ, kb * 64, cn, bh);
          }
          if (!HOM) prefetch_l2_3d(&tmV, jv, cn, bh);
          prefetch_l2_3d(&tmTb, 0, cn, bh);
          if (GATED) {
            prefetch_l2_3d(&tmTbg, 0, cn, bh);
            const float* gn = gw + ((size_t)bh * nchunks + c + 2) * kC;  // its g rows: two 128-byte lines
            prefetch_l2(gn);
            prefetch_l2(gn + 32);
          }
        }
      }
      issued = c + 1;
    }
    if (lane == 0) {  // never leave with copies in flight
      int zero = 0;
      const WaitCtl drain{&zero, p.status, kWaitLimitNs};
      for (int c = issued > NST ? issued - NST : 0; c < issued; ++c)
        (void)mbar_wait(bar + B_FULL + 8 * (c % NST), (c / NST) & 1, drain);
    }
  } else if (warp == 9) {
    // -------------------------------------------------------------- issuer --
    // The whole warp runs the issuer (warp-uniform control flow and operands);
    // each MMA and commit is issued by one elected lane.  Wait results are
    // combined over the warp so every lane takes the same path.
    auto stage = [&](int c) { return sb + (c % NST) * L::STAGE; };
    // P scores = Q K^T of chunk c (lanes 0-63 of TM_G)
    auto issue_qkt = [&](int c) {
      const uint32_t st = stage(c);
      constexpr uint32_t id = idesc_bf16(128, 64, false, false);
      const uint64_t dq = desc_k(st + L::Q_OFF), dk = desc_k(st + L::K_OFF);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t off = (ks >> 2) * L::KB_STRIDE + (ks & 3) * 32;
        mma_bf16_ss_elect(tmem + TM_G, desc_step(dq, off), desc_step(dk, off), id, ks > 0);
      }
    };
    // W = Tbg K (lanes 64-127 of TM_W), Uh = Tb V (lanes 64-127 of Uh[c & 1]).
    // Ungated both share the A operand Tb, and K's 64-column blocks and V sit
    // KB_STRIDE apart, so for even chunks [W | Uh[0]] = Tb [K | V] is one
    // N = Dk + 64 product.
    auto issue_wu = [&](int c) {
      const uint32_t st = stage(c);
      if (!GATED && DVS == 64 && (c & 1) == 0) {
        constexpr uint32_t id = idesc_bf16(128, DK + 64, false, true);
        const uint64_t da = desc_k(st + L::V_OFF), db = desc_mn(st + L::K_OFF, L::KB_STRIDE);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss_elect(tmem + TM_W, desc_step(da, ks * 32),  // rows 64-127: Tb
                            desc_step(db, ks * 2048), id, ks > 0);
      } else {
        constexpr uint32_t idw = idesc_bf16(128, DK, false, true);
        constexpr uint32_t idu = idesc_bf16(128, DVS, false, true);
        // rows 64-127 of the A operand: Tbg (gated) or Tb
        const uint32_t wa = st + (GATED ? L::TB_OFF : L::V_OFF);
        const uint32_t uh = (c & 1) ? TM_UH1 : TM_UH0;
        const uint64_t dw = desc_k(wa), dk = desc_mn(st + L::K_OFF, L::KB_STRIDE);
        const uint64_t dt = desc_k(st + L::V_OFF), dv = desc_mn(st + L::V_OFF + vcol, kTile);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_bf16_ss_elect(tmem + TM_W, desc_step(dw, ks * 32), desc_step(dk, ks * 2048), idw, ks > 0);
          mma_bf16_ss_elect(tmem + uh, desc_step(dt, ks * 32),  // rows 64-127: Tb
                            desc_step(dv, ks * 2048), idu, ks > 0);
        }
      }
    };
    // Gated: W (c) and Uh (c) issued apart (they share no operand), so that
    // only W (c+1) sits in the pipe ahead of K^T U (c)
    auto issue_w_only = [&](int c) {
      const uint32_t st = stage(c);
      constexpr uint32_t idw = idesc_bf16(128, DK, false, true);
      const uint64_t dw = desc_k(st + L::TB_OFF), dk = desc_mn(st + L::K_OFF, L::KB_STRIDE);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_W, desc_step(dw, ks * 32), desc_step(dk, ks * 2048), idw, ks > 0);
    };
    auto issue_uh_only = [&](int c) {
      const uint32_t st = stage(c);
      constexpr uint32_t idu = idesc_bf16(128, DVS, false, true);
      const uint64_t dt = desc_k(st + L::V_OFF), dv = desc_mn(st + L::V_OFF + vcol, kTile);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + ((c & 1) ? TM_UH1 : TM_UH0), desc_step(dt, ks * 32), desc_step(dv, ks * 2048), idu,
                          ks > 0);
    };
    // [Q S ; W S] (lanes 0-63 ; 64-127 of TM_QW[c & 1])
    auto issue_qw = [&](int c) {
      const uint32_t st = stage(c);
      constexpr uint32_t id = idesc_bf16(128, DVS, false, true);
      const uint64_t dq = desc_k(st + L::Q_OFF), ds = desc_mn(sb + L::S_OFF, kTile);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks)
        mma_bf16_ss_elect(tmem + TM_QW + 64 * (c & 1), desc_step(dq, (ks >> 2) * L::KB_STRIDE + (ks & 3) * 32),
                          desc_step(ds, ks * 2048), id, ks > 0);
    };
    // dS = K^T U~
    auto issue_ds = [&](int c) {
      const uint32_t st = stage(c);
      const uint32_t ut = sb + (GATED ? L::UT_OFF : L::U_OFF);
      constexpr uint32_t id = idesc_bf16(128, DVS, true, true);
      const uint64_t dk = desc_mn(st + L::K_OFF, L::KB_STRIDE), du = desc_mn(ut, kTile);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_DS, desc_step(dk, ks * 2048), desc_step(du, ks * 2048), id, ks > 0);
    };
    // O = diag(gamma) QS + P U (accumulated onto lanes 0-63 of TM_QW[c & 1])
    auto issue_pu = [&](int c) {
      constexpr uint32_t id = idesc_bf16(128, DVS, false, true);
      const uint64_t dp = desc_k(sb + L::P_OFF), du = desc_mn(sb + L::U_OFF, kTile);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_QW + 64 * (c & 1), desc_step(dp, ks * 32), desc_step(du, ks * 2048), id, 1);
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FULL, 0, wc));
    if (ok) {
      tc_fence_after();
      issue_wu(0);
      mma_commit_elect(bar + B_PMMA2);
      issue_qkt(0);
      mma_commit_elect(bar + B_PMMA1);
    }
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      const bool nxt = c + 1 < nchunks;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar + B_WREADY, c & 1, wc) && mbar_wait(bar + B_SREADY, c & 1, wc) &&
                          (c < 2 || mbar_wait(bar + B_OFREE + 8 * b, ((c >> 1) - 1) & 1, wc)));
      if (!ok) break;
      tc_fence_after();
      issue_qw(c);
      mma_commit_elect(bar + B_CMMA3);
      if (nxt) {  // W (c) is already in shared memory and Uh[(c+1) & 1] was consumed by chunk c-1
        ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FULL + 8 * ((c + 1) % NST), ((c + 1) / NST) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        if (GATED) issue_w_only(c + 1);
        else issue_wu(c + 1);
        mma_commit_elect(bar + B_PMMA2);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar + B_UREADY, c & 1, wc));
      if (!ok) break;
      tc_fence_after();
      issue_ds(c);
      mma_commit_elect(bar + B_CMMA4);
      // gated: Uh (c+1) after K^T U (c); the U epilogue of chunk c+1 reads it after
      // [Q;W]S (c+1), which the in-order pipe completes later still
      if (GATED && c + 1 < nchunks) issue_uh_only(c + 1);
      // K^T U (c) is the last MMA that reads stage c.  Ungated the stage is
      // free now (its W / Q epilogues came before W_READY); gated the P rows
      // of chunk c still read its g rows, so it goes once they are done.
      if (!GATED) mma_commit_elect(bar + B_EMPTY + 8 * (c % NST));
      ok = __all_sync(0xffffffffu, mbar_wait(bar + B_PREADY + 8 * b, (c >> 1) & 1, wc) &&
                                       (!GATED || mbar_wait(bar + B_QSCALED, c & 1, wc)));
      if (!ok) break;
      tc_fence_after();
      if (GATED) mma_commit_elect(bar + B_EMPTY + 8 * (c % NST));
      issue_pu(c);
      mma_commit_elect(bar + B_CMMA5 + 8 * b);
      if (nxt) {  // after PU (c): the single P tile is free once PMMA1 fires
        issue_qkt(c + 1);
        mma_commit_elect(bar + B_PMMA1);
      }
    }
    tc_fence_after();  // no MMA may outlive TMEM
    mma_commit_elect(bar + B_FIN);
    int zero = 0;
    const WaitCtl fin{&zero, p.status, kWaitLimitNs};
    (void)mbar_wait(bar + B_FIN, 0, fin);
  } else if (warp >= 6) {
    // ------------------------------------------------------- W rows (6-7) --
    const int row = (tid - 192) & 63;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      uint8_t* stp = sm + (c % NST) * L::STAGE;
      // (gated: the FULL wait orders the producer's g rows before the copy below)
      ok = named_bar_and(kBarPrepW, 64,
                         (!GATED || mbar_wait(bar + B_FULL + 8 * (c % NST), (c / NST) & 1, wc)) &&
                             mbar_wait(bar + B_PMMA2, c & 1, wc));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < DK / 32; ++q) {
        uint32_t w[32];
        tmem_ld32(tmem + lane_base + TM_W + q * 32, w);
        tmem_wait_ld();
        uint8_t* wt = stp + (q >> 1) * L::KB_STRIDE + L::W_OFF;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_bf16x8(wt + sw128_off(row, (q & 1) * 4 + cc), reinterpret_cast<const float*>(w) + cc * 8);
      }
      if (GATED) {  // the chain's copy of g (the stage is released before the chain is done)
        const float* vs = reinterpret_cast<const float*>(stp + L::VEC_OFF);
        cvec[(c & 1) * 64 + row] = vs[64 + row];
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarPrepW, 64);
      if (tid == 192) mbar_arrive(bar + B_WREADY);

      // ---- columns 32-63 of the U epilogue of chunk c (rows on lanes 64-127) ----
      if (DVS == 32) continue;  // a 32-column slice: the chain warps take all of it
      ok = named_bar_and(kBarPrepW, 64, mbar_wait(bar + B_CMMA3, c & 1, wc));
      if (!ok) break;
      tc_fence_after();
      {
        const int n = min(kC, T - c * kC);
        const float* vb = cvec + (c & 1) * 64;
        const float wl = GATED ? __expf(vb[n - 1] - vb[row]) : 1.f;
        u_epilogue_half<GATED>(tmem + lane_base + TM_QW + 64 * (c & 1),
                               tmem + lane_base + ((c & 1) ? TM_UH1 : TM_UH0), 32, row, wl, sm + L::U_OFF,
                               sm + L::UT_OFF);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarPrepW, 64);
      if (tid == 192) mbar_arrive(bar + B_UREADY);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------- P rows (4-5) --
    const int row = tid - 128;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      uint8_t* stp = sm + (c % NST) * L::STAGE;
      float* vs = reinterpret_cast<float*>(stp + L::VEC_OFF);  // gated only: g at [64, 128)
      ok = named_bar_and(kBarPrepP, 64, mbar_wait(bar + B_FULL + 8 * (c % NST), (c / NST) & 1, wc));
      if (!ok) break;
      // Gated: Gamma_rs = e^(g_r - g_s) (s <= r) as a_r b_s, a_r = e^(g_r - m),
      // b_s = e^(m - g_s) with m the midpoint of the chunk's g range (g is
      // non-increasing, rows past T flat).  Both factors stay within e^(+-80)
      // while the range is at most 160; a wider range (gates near zero) takes
      // one exponential per element.  b_s goes next to the g rows of the stage.
      float gr = 0.f, ar = 1.f;
      bool fact = true;
      if (GATED) {
        const float mid = 0.5f * (vs[64] + vs[127]);
        fact = vs[64] - vs[127] <= 160.f;
        gr = vs[64 + row];
        ar = __expf(gr - mid);
        vs[128 + row] = __expf(mid - gr);
      }
      ok = named_bar_and(kBarPrepP, 64, mbar_wait(bar + B_PMMA1, c & 1, wc));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t g[64];
        tmem_ld32(tmem + lane_base + TM_G, *reinterpret_cast<uint32_t(*)[32]>(g));
        tmem_ld32(tmem + lane_base + TM_G + 32, *reinterpret_cast<uint32_t(*)[32]>(g + 32));
        tmem_wait_ld();
        uint8_t* ptile = sm + L::P_OFF;
        // every value of the row in registers (the shared-memory reads of the
        // decay factors all come before the first store of the P tile)
        float* pv = reinterpret_cast<float*>(g);
        if (!GATED || fact) {
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {
            float bc[8];
            if (GATED) {
              *reinterpret_cast<float4*>(bc) = *reinterpret_cast<const float4*>(vs + 128 + c16 * 8);
              *reinterpret_cast<float4*>(bc + 4) = *reinterpret_cast<const float4*>(vs + 132 + c16 * 8);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int sc = c16 * 8 + e;
              float val = pv[sc];
              if (GATED) val *= ar * bc[e];
              pv[sc] = sc <= row ? val : 0.f;
            }
          }
        } else {
#pragma unroll
          for (int sc = 0; sc < 64; ++sc) pv[sc] = sc <= row ? pv[sc] * __expf(gr - vs[64 + sc]) : 0.f;
        }
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) st_bf16x8(ptile + sw128_off(row, c16), pv + c16 * 8);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarPrepP, 64);
      if (row == 0) mbar_arrive(bar + B_PREADY + 8 * b);
    }
  } else {
    // --------------------------------------------------------------- chain --
    const int ct = tid;
    const int row = ct & 63;
    const size_t s_base = (size_t)bh * DK * Dv;
    float sreg[DVS];
    if (ct < DK) {
      const float* src = p.S0 ? p.S0 + s_base + (size_t)ct * Dv + j0 : nullptr;
#pragma unroll
      for (int j = 0; j < DVS; j += 4) {
        const float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        sreg[j] = v.x; sreg[j + 1] = v.y; sreg[j + 2] = v.z; sreg[j + 3] = v.w;
      }
      if (HOM) {  // the identity (Dv == Dk): row ct has its 1 in column ct
#pragma unroll
        for (int j = 0; j < DVS; ++j) sreg[j] = (ct == j0 + j) ? 1.f : 0.f;
      }
#pragma unroll
      for (int c16 = 0; c16 < DVS / 8; ++c16) st_bf16x8(sm + L::S_OFF + sw128_off(ct, c16), sreg + 8 * c16);
    }
    fence_proxy_async_smem();
    named_bar_sync(kBarChain, kWG);
    if (ct == 0) mbar_arrive(bar + B_SREADY);  // the initial state tile is in place

    bool ok = true, ok_hi = true, ok_lo = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      const int c0 = c * kC, n = min(kC, T - c0);
      const uint32_t qw = tmem + TM_QW + 64 * b;
      const float* vb = cvec + b * 64;
      if (ct >= 64) {
        // ---- U = Uh - WS (rows on lanes 64-127) ----
        ok_hi = named_bar_and(kBarChainHi, 64, mbar_wait(bar + B_CMMA3, c & 1, wc));
        if (ok_hi) {
          tc_fence_after();
          const float wl = GATED ? __expf(vb[n - 1] - vb[row]) : 1.f;
          // columns 0-31 here, 32-63 in the W warps (same TMEM lanes)
          u_epilogue_half<GATED>(qw + lane_base, tmem + lane_base + ((c & 1) ? TM_UH1 : TM_UH0), 0, row, wl,
                                 sm + L::U_OFF, sm + L::UT_OFF);
          fence_proxy_async_smem();
          tc_fence_before();
          named_bar_sync(kBarChainHi, 64);
          if (ct == 64) mbar_arrive(bar + B_UREADY);
        }
      }
      if (GATED && ct < 64) {
        // ---- QS rows (lanes 0-63) times gamma, in TMEM, before P U lands on them ----
        ok_lo = named_bar_and(kBarChainLo, 64, ok_lo && mbar_wait(bar + B_CMMA3, c & 1, wc));
        if (ok_lo) {
          tc_fence_after();
          const float gam = __expf(vb[row]);
#pragma unroll
          for (int q = 0; q < DVS / 32; ++q) {
            uint32_t v[32];
            tmem_ld32(qw + lane_base + q * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * gam);
            tmem_st32(qw + lane_base + q * 32, v);
          }
          tmem_wait_st();
          tc_fence_before();
          named_bar_sync(kBarChainLo, 64);
          if (ct == 0) mbar_arrive(bar + B_QSCALED);
        }
      }
      ok = named_bar_and(kBarChain, kWG, ok_hi && ok_lo && mbar_wait(bar + B_CMMA4, c & 1, wc));
      if (!ok) break;
      tc_fence_after();

      // ---- state update (lanes 0..DK-1) ----
      if (ct < DK) {
        const float carry = GATED ? __expf(vb[n - 1]) : 1.f;
        uint32_t ds[DVS];
#pragma unroll
        for (int q = 0; q < DVS / 32; ++q)
          tmem_ld32(tmem + lane_base + TM_DS + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(ds + 32 * q));
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < DVS; ++e) sreg[e] = fmaf(carry, sreg[e], __uint_as_float(ds[e]));
#pragma unroll
        for (int c16 = 0; c16 < DVS / 8; ++c16) st_bf16x8(sm + L::S_OFF + sw128_off(ct, c16), sreg + 8 * c16);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarChain, kWG);
      if (ct == 0) mbar_arrive(bar + B_SREADY);

      // ---- outputs O = gamma QS + PU (lanes 0-63), drained by warps 0-1 ----
      if (ct < 64) {
        ok_lo = named_bar_and(kBarChainLo, 64, mbar_wait(bar + B_CMMA5 + 8 * b, (c >> 1) & 1, wc));
        if (ok_lo) {
          tc_fence_after();
          __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + ((size_t)bh * T + c0 + row) * Dv + j0;
#pragma unroll
          for (int q = 0; q < DVS / 32; ++q) {
            uint32_t ov[32];
            tmem_ld32(qw + lane_base + q * 32, ov);
            tmem_wait_ld();
            if (row < n) {
#pragma unroll
              for (int cc = 0; cc < 4; ++cc)
                st_bf16x8(orow + q * 32 + cc * 8, reinterpret_cast<const float*>(ov) + cc * 8);
            }
          }
          tc_fence_before();
          named_bar_sync(kBarChainLo, 64);
          if (ct == 0) mbar_arrive(bar + B_OFREE + 8 * b);
        }
      }
    }
    if (p.S_out && ct < DK) {
      float* dst = p.S_out + s_base + (size_t)ct * Dv + j0;
#pragma unroll
      for (int j = 0; j < DVS; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DK, bool GATED, int DVS, bool HOM>
cudaError_t launch_t(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st, bool after_prepass) {
  using L = MainLayout<DK, GATED>;
  const int BH = p.B * p.H;
  const int nchunks = (p.T + kC - 1) / kC;
  cudaError_t e = cudaSuccess;
  CUtensorMap mq, mk, mv, mtb, mtbg;
  // with the layer's pre-step, q and k come mapped from the pre-pass (workspace)
  const void* qsrc = p.prestep ? static_cast<const void*>(w.qhat) : p.q;
  const void* ksrc = p.prestep ? static_cast<const void*>(w.khat) : p.k;
  if (!make_tmap_3d_bf16(&mq, qsrc, DK, p.T, BH) || !make_tmap_3d_bf16(&mk, ksrc, DK, p.T, BH) ||
      !make_tmap_3d_bf16(&mv, p.v, p.Dv, p.T, BH) ||
      !make_tmap_3d_bf16(&mtb, w.tb, kC, nchunks * kC, BH) ||
      !make_tmap_3d_bf16(&mtbg, GATED ? w.tbg : w.tb, kC, nchunks * kC, BH))
    return cudaErrorInvalidValue;
  auto kern = chunk_main_kernel<DK, GATED, DVS, HOM>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(BH * (p.Dv / DVS)));
  // Programmatic dependent launch: CTAs may start (TMEM, barriers, state
  // load) while the pre-pass drains; the producer waits for its results.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_prepass ? 1 : 0;  // otherwise griddepcontrol.wait returns at once
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mtb, mtbg, p, w.g);
}

}  // namespace

bool chunk_main_supported(const ChunkProblem& p) {
  return p.bf16 && p.mode == Mode::Delta && p.T > 0 && p.C == 64 && (p.Dk == 64 || p.Dk == 128) &&
         (p.Dv == 64 || p.Dv == 128);
}

// The SM count of the current device (queried once per device).
static int sm_count() {
  static int counts[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    counts[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
  }
  return counts[dev];
}

template <int DK, bool GATED>
cudaError_t launch_dvs(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st, int dvs, bool after) {
  // Each CTA runs the whole chunk chain of its (b, h, slice); the chain's
  // length per chunk hardly depends on the slice width.  When 64-column
  // slices leave most SMs idle (long sequences over few heads), 32-column
  // slices give twice the CTAs, as long as they still fit one wave.
  if (p.hom) return dvs == 64 ? launch_t<DK, GATED, 64, true>(p, w, st, after) : cudaErrorInvalidValue;
  if (dvs == 0) dvs = (long long)p.B * p.H * (p.Dv / 32) <= sm_count() ? 32 : 64;
  if (dvs == 32) return launch_t<DK, GATED, 32, false>(p, w, st, after);
  return launch_t<DK, GATED, 64, false>(p, w, st, after);
}

cudaError_t launch_chunk_main_only(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st, int dvs,
                                   bool after_prepass) {
  const bool gated = p.alpha != nullptr;
  if (p.Dk == 128)
    return gated ? launch_dvs<128, true>(p, w, st, dvs, after_prepass)
                 : launch_dvs<128, false>(p, w, st, dvs, after_prepass);
  return gated ? launch_dvs<64, true>(p, w, st, dvs, after_prepass)
               : launch_dvs<64, false>(p, w, st, dvs, after_prepass);
}

cudaError_t launch_chunk_main(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st) {
  cudaError_t e = launch_tsolve(p, w, st);
  if (e != cudaSuccess) return e;
  return launch_chunk_main_only(p, w, st, 0, true);
}

}  // namespace dn
