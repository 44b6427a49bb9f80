// tcgen05 chunked DeltaNet forward with chunks of C = 128 tokens (bf16
// operands, float32 accumulation and state): the bf16 C = 128 path of
// deltanet_chunk_fwd, run after the WY pre-pass (tsolve.cu) has written
// Tb = (I + A)^-1 diag(beta), Tbg = Tb diag(gamma) and g for every chunk.
//
// The chunk form is the one of the C = 64 kernel ("GPT-2 から Kimi K3 まで",
// news.ainew.jp, section "DeltaNet (Parallelizing linear transformers with delta
// rule)"; gate from the Gated DeltaNet paragraph of "How a Baseten Engineer
// Traced 7 Years of Attention Mechanism Evolution"), with the state applied
// once per 128 tokens.  A chunk fills an M = 128 tile by itself, so no
// operand stacking is needed; per chunk of n <= 128 rows entered with state S:
//   phase A   P = Q K^T (N = 128),  W = Tbg K,  Uh = Tb V
//   epilogue  P <- tril(P) * Gamma, W -> bf16 (gated: Q <- diag(gamma) Q)
//   phase B   QS = Q S,  WS = W S
//   epilogue  U = Uh - WS (gated also U~ = diag(Gamma_last,.) U)
//   phase C   O = QS + P U (same TMEM tile),  dS = K^T U~
//   epilogue  O -> global,  S <- gamma_last S + dS
//
// At C = 128 and Dk = 128 one chunk's operands (K, Q, V, Tb, Tbg, W, P, U,
// U~, S: up to 224 KB) fill shared memory, so the phases run one after the
// other; the next chunk's tiles are loaded (TMA, L2 prefetched one chunk
// ahead) as soon as the last MMA of a chunk has read them, overlapping the
// output / state epilogue.
//
// One CTA per (b, h, 64-column slice of Dv), 9 warps: warps 0-7 run the
// epilogues, warps w and w + 4 on the same TMEM lanes 32 (w % 4) .. + 31 (one
// chunk row per lane), each taking one half of every epilogue's columns (and
// of the state's); warp 8 loads (one lane) and issues the MMAs (warp-uniform,
// one elected lane).  Waits are bounded; a
// wait that runs out sets the status word and the CTA winds down without
// trapping.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

constexpr int kC = 128;
constexpr int kDVS = 64;
constexpr uint32_t kBlk = 16384;  // 128 rows x 128 bytes: one 64-column block of a 128-row tile
constexpr int kThreads = 288;  // epilogues 0-7, loads and MMA issue 8
constexpr int kEpi = 256;
constexpr int kBarEpi = 1;

template <int DK, bool GATED>
struct Layout128 {
  static constexpr int KB = DK / 64;
  static constexpr uint32_t K_OFF = 0;                    // K   [KB][128 x 64]
  static constexpr uint32_t Q_OFF = K_OFF + KB * kBlk;    // Q   [KB][128 x 64]
  static constexpr uint32_t V_OFF = Q_OFF + KB * kBlk;    // V   128 x 64
  static constexpr uint32_t TB_OFF = V_OFF + kBlk;        // Tb  [2][128 x 64]
  static constexpr uint32_t TBG_OFF = TB_OFF + 2 * kBlk;  // Tbg [2][128 x 64] (gated; then P)
  static constexpr uint32_t W_OFF = TBG_OFF + (GATED ? 2 * kBlk : 0);  // W [KB][128 x 64]
  static constexpr uint32_t P_OFF = GATED ? TBG_OFF : W_OFF + KB * kBlk;  // P [2][128 x 64]
  static constexpr uint32_t U_OFF = GATED ? W_OFF + KB * kBlk : P_OFF + 2 * kBlk;  // U 128 x 64
  static constexpr uint32_t UT_OFF = U_OFF + kBlk;        // U~ (gated)
  static constexpr uint32_t S_OFF = U_OFF + (GATED ? 2 : 1) * kBlk;  // bf16 state, DK rows x 128 B
  static constexpr uint32_t VEC_OFF = S_OFF + DK * 128;   // g rows per parity: [2][128] (gated)
  static constexpr uint32_t BAR_OFF = VEC_OFF + (GATED ? 2 * kC * 4 : 0);
  static constexpr uint32_t BYTES = BAR_OFF + 128;
  static constexpr uint32_t ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// TMEM columns: P (128), W (Dk), Uh (64), QS / O (64), WS (64), dS (64)
template <int DK>
struct Tmem128 {
  static constexpr uint32_t P = 0, W = 128, UH = 128 + DK, QS = UH + 64, WS = QS + 64, DS = WS + 64;
  static_assert(DS + 64 <= 512, "TMEM columns");
};

// mbarriers: FULL (TMA + g rows), MMA_A/B/C (commits), EPI_A/B (epilogue ->
// issuer), SREADY (state tile and O tile consumed), FIN
constexpr uint32_t B_FULL = 0, B_MMAA = 8, B_MMAB = 16, B_MMAC = 24, B_EPIA = 32, B_EPIB = 40,
                   B_SREADY = 48, B_FIN = 56, B_TMEM = 64, B_ABORT = 68;

template <int DK, bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    chunk128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmTb,
                    const __grid_constant__ CUtensorMap tmTbg, const ChunkProblem p,
                    const float* __restrict__ gw) {
  using L = Layout128<DK, GATED>;
  using TM = Tmem128<DK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = warp_uniform(smem_u32(sm));
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = (int)warp_uniform((uint32_t)tid >> 5);
  const int bh = blockIdx.x;
  const int j0 = blockIdx.y * kDVS;
  const int T = p.T, Dv = p.Dv;
  const int nchunks = (T + kC - 1) / kC;
  const uint32_t bar = sb + L::BAR_OFF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::BAR_OFF + B_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::BAR_OFF + B_ABORT);
  float* gvec = reinterpret_cast<float*>(sm + L::VEC_OFF);

  if (tid == 0) {
    mbar_init(bar + B_FULL, 2);  // TMA bytes + the g rows
    mbar_init(bar + B_MMAA, 1);
    mbar_init(bar + B_MMAB, 1);
    mbar_init(bar + B_MMAC, 1);
    mbar_init(bar + B_EPIA, 1);
    mbar_init(bar + B_EPIB, 1);
    mbar_init(bar + B_SREADY, 1);
    mbar_init(bar + B_FIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
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
  const uint32_t tile_bytes = (2 * L::KB * 2 + 2 + 4 + (GATED ? 4 : 0)) * 8192u;

  if (warp == 8) {
    // --------------------------------------------------- loads and MMA issue --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmTb);
      if (GATED) prefetch_tmap(&tmTbg);
    }
    // Tb, Tbg and g come from the pre-pass launched just before this kernel
    grid_dependency_wait();
    auto load_chunk = [&](int c) {
      const int c0 = c * kC;
      const uint32_t full = bar + B_FULL;
      if (lane == 0) {
        mbar_expect_tx(full, tile_bytes);
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
#pragma unroll
          for (int kb = 0; kb < L::KB; ++kb) {
            tma_load_3d(sb + L::K_OFF + kb * kBlk + rb * 8192, &tmK, full, kb * 64, c0 + rb * 64, bh);
            tma_load_3d(sb + L::Q_OFF + kb * kBlk + rb * 8192, &tmQ, full, kb * 64, c0 + rb * 64, bh);
          }
          tma_load_3d(sb + L::V_OFF + rb * 8192, &tmV, full, j0, c0 + rb * 64, bh);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(sb + L::TB_OFF + kb * kBlk + rb * 8192, &tmTb, full, kb * 64, c0 + rb * 64, bh);
            if (GATED)
              tma_load_3d(sb + L::TBG_OFF + kb * kBlk + rb * 8192, &tmTbg, full, kb * 64, c0 + rb * 64, bh);
          }
        }
        if (c + 1 < nchunks) {  // warm L2 for the next chunk
          const int cn = c0 + kC;
#pragma unroll
          for (int rb = 0; rb < 2; ++rb) {
#pragma unroll
            for (int kb = 0; kb < L::KB; ++kb) {
              prefetch_l2_3d(&tmK, kb * 64, cn + rb * 64, bh);
              prefetch_l2_3d(&tmQ, kb * 64, cn + rb * 64, bh);
            }
            prefetch_l2_3d(&tmV, j0, cn + rb * 64, bh);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
              prefetch_l2_3d(&tmTb, kb * 64, cn + rb * 64, bh);
              if (GATED) prefetch_l2_3d(&tmTbg, kb * 64, cn + rb * 64, bh);
            }
          }
        }
      }
      if (GATED) {  // g rows of the chunk (rows past T: g flat)
        float* gv = gvec + (c & 1) * kC;
        for (int r = lane; r < kC; r += 32) gv[r] = gw[((size_t)bh * nchunks + c) * kC + r];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(full);
    };
    bool ok = true, pending = true;
    int pend_parity = 0;
    load_chunk(0);
    for (int c = 0; c < nchunks && ok; ++c) {
      const uint32_t par = c & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FULL, par, wc));
      if (!ok) break;
      pending = false;
      tc_fence_after();
      // ---- phase A: P = Q K^T, W = Tb(g) K, Uh = Tb V ----
      {
        constexpr uint32_t idp = idesc_bf16(128, 128, false, false);
        const uint64_t dq = desc_k(sb + L::Q_OFF), dk = desc_k(sb + L::K_OFF);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
          mma_bf16_ss_elect(tmem + TM::P, desc_step(dq, off), desc_step(dk, off), idp, ks > 0);
        }
        constexpr uint32_t idw = idesc_bf16(128, DK, false, true);
        constexpr uint32_t idu = idesc_bf16(128, 64, false, true);
        const uint64_t dw = desc_k(sb + (GATED ? L::TBG_OFF : L::TB_OFF)), dt = desc_k(sb + L::TB_OFF);
        const uint64_t dkm = desc_mn(sb + L::K_OFF, kBlk), dv = desc_mn(sb + L::V_OFF, kBlk);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
          mma_bf16_ss_elect(tmem + TM::W, desc_step(dw, off), desc_step(dkm, ks * 2048), idw, ks > 0);
          mma_bf16_ss_elect(tmem + TM::UH, desc_step(dt, off), desc_step(dv, ks * 2048), idu, ks > 0);
        }
        mma_commit_elect(bar + B_MMAA);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar + B_EPIA, par, wc) && mbar_wait(bar + B_SREADY, par, wc));
      if (!ok) break;
      tc_fence_after();
      // ---- phase B: QS = Q S, WS = W S ----
      {
        constexpr uint32_t id = idesc_bf16(128, 64, false, true);
        const uint64_t ds = desc_mn(sb + L::S_OFF, kBlk), dq = desc_k(sb + L::Q_OFF), dw = desc_k(sb + L::W_OFF);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
          const uint64_t bs = desc_step(ds, ks * 2048);
          mma_bf16_ss_elect(tmem + TM::QS, desc_step(dq, off), bs, id, ks > 0);
          mma_bf16_ss_elect(tmem + TM::WS, desc_step(dw, off), bs, id, ks > 0);
        }
        mma_commit_elect(bar + B_MMAB);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar + B_EPIB, par, wc));
      if (!ok) break;
      tc_fence_after();
      // ---- phase C: O = QS + P U, dS = K^T U~ ----
      {
        constexpr uint32_t ido = idesc_bf16(128, 64, false, true);
        constexpr uint32_t idd = idesc_bf16(128, 64, true, true);
        const uint64_t dp = desc_k(sb + L::P_OFF), du = desc_mn(sb + L::U_OFF, kBlk);
        const uint64_t dkm = desc_mn(sb + L::K_OFF, kBlk), dut = desc_mn(sb + (GATED ? L::UT_OFF : L::U_OFF), kBlk);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
          mma_bf16_ss_elect(tmem + TM::QS, desc_step(dp, off), desc_step(du, ks * 2048), ido, 1);
          mma_bf16_ss_elect(tmem + TM::DS, desc_step(dkm, ks * 2048), desc_step(dut, ks * 2048), idd, ks > 0);
        }
        mma_commit_elect(bar + B_MMAC);
      }
      if (c + 1 < nchunks) {  // every operand tile of chunk c has been read: stream in the next chunk
        ok = __all_sync(0xffffffffu, mbar_wait(bar + B_MMAC, par, wc));
        if (!ok) break;
        load_chunk(c + 1);
        pending = true;
        pend_parity = (c + 1) & 1;
      }
    }
    if (pending) {  // never leave with copies in flight
      int zero = 0;
      const WaitCtl drain{&zero, p.status, kWaitLimitNs};
      (void)mbar_wait(bar + B_FULL, pend_parity, drain);
    }
    tc_fence_after();  // no MMA may outlive TMEM
    mma_commit_elect(bar + B_FIN);
    int zero = 0;
    const WaitCtl fin{&zero, p.status, kWaitLimitNs};
    (void)mbar_wait(bar + B_FIN, 0, fin);
  } else {
    // -------------------------------------------------------------- epilogues --
    const int r = tid & 127;  // chunk row = TMEM lane
    const int hf = tid >> 7;  // which half of the columns this thread takes
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const size_t s_base = (size_t)bh * DK * Dv;
    float sreg[kDVS / 2];  // columns j0 + 32 hf .. + 31 of state row r
    if (r < DK) {
      const float* src = p.S0 ? p.S0 + s_base + (size_t)r * Dv + j0 + 32 * hf : nullptr;
#pragma unroll
      for (int j = 0; j < kDVS / 2; j += 4) {
        const float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        sreg[j] = v.x; sreg[j + 1] = v.y; sreg[j + 2] = v.z; sreg[j + 3] = v.w;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) st_bf16x8(sm + L::S_OFF + sw128_off(r, 4 * hf + c), sreg + 8 * c);
    }
    fence_proxy_async_smem();
    named_bar_sync(kBarEpi, kEpi);
    if (tid == 0) mbar_arrive(bar + B_SREADY);  // the initial state tile is in place

    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const uint32_t par = c & 1;
      const int c0 = c * kC, n = min(kC, T - c0);
      const float* gv = gvec + par * kC;
      // ---- P rows (masked, decayed), W rows; gated: Q <- diag(gamma) Q ----
      ok = named_bar_and(kBarEpi, kEpi, mbar_wait(bar + B_MMAA, par, wc));
      if (!ok) break;
      tc_fence_after();
      {
        const float gr = GATED ? gv[r] : 0.f;
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {  // P columns 64 hf .. + 63, 32 at a time
          const int q = 2 * hf + qq;
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + TM::P + q * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int s = q * 32 + cc * 8 + e;
              float val = __uint_as_float(v[cc * 8 + e]);
              if (GATED) val *= __expf(gr - gv[s]);
              x[e] = s <= r ? val : 0.f;
            }
            st_bf16x8(sm + L::P_OFF + (q >> 1) * kBlk + sw128_off(r, (q & 1) * 4 + cc), x);
          }
        }
        constexpr int WQ = DK / 64;  // 32-column groups of W per half
#pragma unroll
        for (int qq = 0; qq < WQ; ++qq) {
          const int q = hf * WQ + qq;
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + TM::W + q * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            st_bf16x8(sm + L::W_OFF + (q >> 1) * kBlk + sw128_off(r, (q & 1) * 4 + cc),
                      reinterpret_cast<const float*>(v) + cc * 8);
        }
        if (GATED) {
          // (this thread's half of each 64-column block loaded whole before its
          // stores, which the compiler cannot tell apart from the loads)
          const float gam = __expf(gr);
#pragma unroll
          for (int kb = 0; kb < DK / 64; ++kb) {
            uint4 u[4];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
              u[c4] = *reinterpret_cast<const uint4*>(sm + L::Q_OFF + kb * kBlk + sw128_off(r, 4 * hf + c4));
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              float x[8];
              unpack_bf16x8(u[c4], x);
#pragma unroll
              for (int e = 0; e < 8; ++e) x[e] *= gam;
              st_bf16x8(sm + L::Q_OFF + kb * kBlk + sw128_off(r, 4 * hf + c4), x);
            }
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kEpi);
      if (tid == 0) mbar_arrive(bar + B_EPIA);

      // ---- U = Uh - WS (gated also U~ = U e^(g_last - g_r)), columns 32 hf .. + 31 ----
      ok = named_bar_and(kBarEpi, kEpi, mbar_wait(bar + B_MMAB, par, wc));
      if (!ok) break;
      tc_fence_after();
      {
        const float wl = GATED ? __expf(gv[n - 1] - gv[r]) : 1.f;
        uint32_t ws[32], uh[32];
        tmem_ld32(tmem + lane_base + TM::WS + hf * 32, ws);
        tmem_ld32(tmem + lane_base + TM::UH + hf * 32, uh);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float x[8], y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[e] = __uint_as_float(uh[cc * 8 + e]) - __uint_as_float(ws[cc * 8 + e]);
            y[e] = x[e] * wl;
          }
          st_bf16x8(sm + L::U_OFF + sw128_off(r, hf * 4 + cc), x);
          if (GATED) st_bf16x8(sm + L::UT_OFF + sw128_off(r, hf * 4 + cc), y);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kEpi);
      if (tid == 0) mbar_arrive(bar + B_EPIB);

      // ---- O rows -> global; S <- gamma_last S + dS (columns 32 hf .. + 31) ----
      ok = named_bar_and(kBarEpi, kEpi, mbar_wait(bar + B_MMAC, par, wc));
      if (!ok) break;
      tc_fence_after();
      {
        __nv_bfloat16* orow =
            static_cast<__nv_bfloat16*>(p.o) + ((size_t)bh * T + c0 + r) * Dv + j0 + 32 * hf;
        {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + TM::QS + hf * 32, ov);
          tmem_wait_ld();
          if (r < n) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) st_bf16x8(orow + cc * 8, reinterpret_cast<const float*>(ov) + cc * 8);
          }
        }
        if (r < DK) {
          const float carry = GATED ? __expf(gv[n - 1]) : 1.f;
          uint32_t ds[32];
          tmem_ld32(tmem + lane_base + TM::DS + hf * 32, ds);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) sreg[e] = fmaf(carry, sreg[e], __uint_as_float(ds[e]));
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) st_bf16x8(sm + L::S_OFF + sw128_off(r, 4 * hf + c4), sreg + 8 * c4);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kEpi);
      if (tid == 0) mbar_arrive(bar + B_SREADY);
    }
    if (p.S_out && r < DK) {
      float* dst = p.S_out + s_base + (size_t)r * Dv + j0 + 32 * hf;
#pragma unroll
      for (int j = 0; j < kDVS / 2; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DK, bool GATED>
cudaError_t launch_t(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st) {
  using L = Layout128<DK, GATED>;
  const int BH = p.B * p.H;
  const int nchunks = (p.T + kC - 1) / kC;
  cudaError_t e = launch_tsolve(p, w, st);
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk, mv, mtb, mtbg;
  if (!make_tmap_3d_bf16(&mq, p.q, DK, p.T, BH) || !make_tmap_3d_bf16(&mk, p.k, DK, p.T, BH) ||
      !make_tmap_3d_bf16(&mv, p.v, p.Dv, p.T, BH) ||
      !make_tmap_3d_bf16(&mtb, w.tb, kC, nchunks * kC, BH) ||
      !make_tmap_3d_bf16(&mtbg, GATED ? w.tbg : w.tb, kC, nchunks * kC, BH))
    return cudaErrorInvalidValue;
  auto kern = chunk128_kernel<DK, GATED>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: CTAs may start while the pre-pass drains;
  // the loading warp waits for its results.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)BH, (unsigned)(p.Dv / kDVS));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mtb, mtbg, p, w.g);
}

}  // namespace

bool chunk128_supported(const ChunkProblem& p) {
  return p.bf16 && p.mode == Mode::Delta && p.T > 0 && p.C == 128 && (p.Dk == 64 || p.Dk == 128) &&
         (p.Dv == 64 || p.Dv == 128);
}

cudaError_t launch_chunk128(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st) {
  const bool gated = p.alpha != nullptr;
  if (p.Dk == 128) return gated ? launch_t<128, true>(p, w, st) : launch_t<128, false>(p, w, st);
  return gated ? launch_t<64, true>(p, w, st) : launch_t<64, false>(p, w, st);
}

}  // namespace dn
