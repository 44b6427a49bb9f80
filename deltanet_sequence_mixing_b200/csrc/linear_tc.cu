// tcgen05 chunked ELU+1 linear attention (bf16 operands, float32 accumulation,
// state and normaliser): the bf16 path of linear_attn_fwd.
//
// Additive chunk loop of "GPT-2 から Kimi K3 まで" (news.ainew.jp), section
// "DeltaNet (Parallelizing linear transformers with delta rule)", on the ELU+1
// feature maps of section "Linear attention" (and of the linear-attention
// snippet of "How a Baseten Engineer Traced 7 Years of Attention Mechanism
// Evolution"), with the normaliser z carried like S.  Per chunk c of 64 rows
// (Q' = ELU(Q) + 1, K' = ELU(K) + 1, rows past T zero), entered with S, z:
//   P = tril(Q' K'^T)                                (M = 128 MMA [K'; Q'] K'^T)
//   O = (Q' S + P V) / (Q' z + P 1)                  (Q'S + PV in one TMEM tile)
//   S <- S + K'^T V,  z <- z + K'^T 1
// Only S (and z) carry from chunk to chunk, and S's update K'^T V does not
// depend on S, so everything but the state accumulate is pipelined ahead of it.
//
// One CTA per (b, h, 64-column slice of Dv), 10 warps:
//   warp 8     producer: TMA of K, Q, V into a three-stage ring
//   warp 9     MMA issuer (warp-uniform, one elected lane): Gram (c+1) and
//              K'^T V (c+1) while chunk c waits for its state tile, then
//              O (c) = Q'S + PV
//   warps 4-7  prep: feature maps in place, K' column sums, Q' z per row,
//              P rows to bf16 with their row sums (warps 6-7, TMEM lanes
//              64-127)
//   warps 0-3  state: S += K'^T V in float32 registers, the bf16 state tile
//              for the next chunk (double-buffered); warps 0-1 also drain
//              O / (Q' z + P 1) to global memory
// Accumulators live in TMEM (G[2], dS[2], O[2]: 384 of 512 columns).  Every
// mbarrier completes once per chunk or per use of a parity, so parity waits
// are unambiguous.  All waits are bounded; a wait that runs out sets the
// status word and the CTA winds down (copies drained, MMAs retired, TMEM
// freed) without trapping.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

constexpr int kC = 64;
constexpr int kDVS = 64;
constexpr int NST = 3;
constexpr uint32_t kTile = 8192;  // 64 rows x 128 bytes
constexpr int kWG = 128;
constexpr int kThreads = 2 * kWG + 64;  // state 0-3, prep 4-7, producer 8, issuer 9
constexpr int kBarState = 1, kBarLo = 2, kBarPrep = 3, kBarPrepHi = 4;

// TMEM columns: Gram[2] (lanes 64-127: Q'K'^T), dS[2] (K'^T V), O[2] (lanes 0-63)
constexpr uint32_t TM_G = 0, TM_DS = 128, TM_O = 256;

template <int DK>
struct LinLayout {
  static constexpr int KB = DK / 64;
  static constexpr uint32_t KB_STRIDE = 2 * kTile;  // [K | Q] per 64 columns of Dk
  static constexpr uint32_t K_OFF = 0, Q_OFF = kTile;
  static constexpr uint32_t V_OFF = KB * KB_STRIDE;
  static constexpr uint32_t STAGE = V_OFF + kTile;
  static constexpr uint32_t P_OFF = NST * STAGE;           // P[2]
  static constexpr uint32_t S_OFF = P_OFF + 2 * kTile;     // bf16 state tiles [2], DK rows x 128 B
  static constexpr uint32_t Z_OFF = S_OFF + 2 * DK * 128;  // z (DK), Q'z [2][64], row sums [2][64]
  static constexpr uint32_t RED_OFF = Z_OFF + (DK + 4 * 64) * 4;  // K' column partial sums [16][DK]
  static constexpr uint32_t BAR_OFF = RED_OFF + 16 * DK * 4;
  static constexpr uint32_t BYTES = BAR_OFF + 256;
  static constexpr uint32_t ALLOC = BYTES + 1024;
  static_assert(STAGE % 1024 == 0 && P_OFF % 1024 == 0, "128-byte swizzle atoms stay aligned");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// mbarrier slots (8 bytes each).  FULL / EMPTY per stage; the rest per chunk
// parity except FMAP (once per chunk, never two phases ahead of its waiter).
constexpr uint32_t B_FULL = 0, B_EMPTY = 24, B_GDONE = 48, B_DSDONE = 64, B_PREADY = 80,
                   B_DSFREE = 96, B_SREADY = 112, B_ODONE = 128, B_OFREE = 144, B_FMAP = 160,
                   B_FIN = 168, B_TMEM = 176, B_ABORT = 180;

// ELU(x) + 1: x + 1 for x > 0, and e^x (= (e^x - 1) + 1) otherwise.
__device__ __forceinline__ float elu1(float x) { return x > 0.f ? x + 1.f : __expf(x); }

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const ChunkProblem p) {
  using L = LinLayout<DK>;
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
  float* zs = reinterpret_cast<float*>(sm + L::Z_OFF);  // z entering the chunk the prep is on
  float* dq = zs + DK;                                   // Q' z per row, [2][64]
  float* rs = dq + 128;                                  // row sums of P, [2][64]
  float* red = reinterpret_cast<float*>(sm + L::RED_OFF);

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(bar + B_FULL + 8 * i, 1);
      mbar_init(bar + B_EMPTY + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + B_GDONE + 8 * i, 1);
      mbar_init(bar + B_DSDONE + 8 * i, 1);
      mbar_init(bar + B_PREADY + 8 * i, 1);
      mbar_init(bar + B_DSFREE + 8 * i, 1);
      mbar_init(bar + B_SREADY + 8 * i, 1);
      mbar_init(bar + B_ODONE + 8 * i, 1);
      mbar_init(bar + B_OFREE + 8 * i, 1);
    }
    mbar_init(bar + B_FMAP, 1);
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
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  auto stage = [&](int c) { return sb + (c % NST) * L::STAGE; };

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % NST, use = c / NST;
        if (use > 0 && !mbar_wait(bar + B_EMPTY + 8 * s, (use - 1) & 1, wc)) break;
        const uint32_t st = stage(c);
        const uint32_t full = bar + B_FULL + 8 * s;
        mbar_expect_tx(full, (2 * L::KB + 1) * kTile);
#pragma unroll
        for (int kb = 0; kb < L::KB; ++kb) {
          tma_load_3d(st + kb * L::KB_STRIDE + L::K_OFF, &tmK, full, kb * 64, c * kC, bh);
          tma_load_3d(st + kb * L::KB_STRIDE + L::Q_OFF, &tmQ, full, kb * 64, c * kC, bh);
        }
        tma_load_3d(st + L::V_OFF, &tmV, full, j0, c * kC, bh);
        if (c + 2 < nchunks) {  // warm L2 for the chunk after next
#pragma unroll
          for (int kb = 0; kb < L::KB; ++kb) {
            prefetch_l2_3d(&tmK, kb * 64, (c + 2) * kC, bh);
            prefetch_l2_3d(&tmQ, kb * 64, (c + 2) * kC, bh);
          }
          prefetch_l2_3d(&tmV, j0, (c + 2) * kC, bh);
        }
        issued = c + 1;
      }
      int zero = 0;  // never leave with copies in flight
      const WaitCtl drain{&zero, p.status, kWaitLimitNs};
      for (int c = issued > NST ? issued - NST : 0; c < issued; ++c)
        (void)mbar_wait(bar + B_FULL + 8 * (c % NST), (c / NST) & 1, drain);
    }
  } else if (warp == 9) {
    // -------------------------------------------------------------- issuer --
    // Gram (c) = [K'; Q'] K'^T into G[c & 1] and dS (c) = K'^T V into dS[c & 1]
    auto issue_gram_ds = [&](int c) {
      const uint32_t st = stage(c);
      const int b = c & 1;
      constexpr uint32_t idg = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t a = st + (ks >> 2) * L::KB_STRIDE + L::K_OFF + (ks & 3) * 32;
        mma_bf16_ss_elect(tmem + TM_G + 64 * b, desc_k(a), desc_k(a), idg, ks > 0);
      }
      mma_commit_elect(bar + B_GDONE + 8 * b);
      constexpr uint32_t idd = idesc_bf16(128, 64, true, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_DS + 64 * b, desc_mn(st + L::K_OFF + ks * 2048, L::KB_STRIDE),
                          desc_mn(st + L::V_OFF + ks * 2048, kTile), idd, ks > 0);
      mma_commit_elect(bar + B_DSDONE + 8 * b);
    };
    // O (c) = Q' S + P V into O[c & 1] (lanes 0-63)
    auto issue_o = [&](int c) {
      const uint32_t st = stage(c);
      const int b = c & 1;
      constexpr uint32_t ido = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t a = st + (ks >> 2) * L::KB_STRIDE + L::Q_OFF + (ks & 3) * 32;
        mma_bf16_ss_elect(tmem + TM_O + 64 * b, desc_k(a),
                          desc_mn(sb + L::S_OFF + b * (DK * 128) + ks * 2048, kTile), ido, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_O + 64 * b, desc_k(sb + L::P_OFF + b * kTile + ks * 32),
                          desc_mn(st + L::V_OFF + ks * 2048, kTile), ido, 1);
      mma_commit_elect(bar + B_ODONE + 8 * b);
      mma_commit_elect(bar + B_EMPTY + 8 * (c % NST));  // stage c: Gram, dS and O have read it
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FMAP, 0, wc));
    if (ok) {
      tc_fence_after();
      issue_gram_ds(0);
    }
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      if (c + 1 < nchunks) {  // the next chunk's Gram and K'^T V run while chunk c waits for its state
        // G[(c+1) & 1] was read by the P rows of chunk c-1 (PREADY waited below in
        // iteration c-1); dS[(c+1) & 1] must have been added to S (DSFREE of chunk c-1)
        ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FMAP, (c + 1) & 1, wc) &&
                                         (c < 1 || mbar_wait(bar + B_DSFREE + 8 * (b ^ 1), ((c - 1) >> 1) & 1, wc)));
        if (!ok) break;
        tc_fence_after();
        issue_gram_ds(c + 1);
      }
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar + B_PREADY + 8 * b, (c >> 1) & 1, wc) &&
                          mbar_wait(bar + B_SREADY + 8 * b, (c >> 1) & 1, wc) &&
                          (c < 2 || mbar_wait(bar + B_OFREE + 8 * b, ((c >> 1) - 1) & 1, wc)));
      if (!ok) break;
      tc_fence_after();
      issue_o(c);
    }
    tc_fence_after();  // no MMA may outlive TMEM
    mma_commit_elect(bar + B_FIN);
    int zero = 0;
    const WaitCtl fin{&zero, p.status, kWaitLimitNs};
    (void)mbar_wait(bar + B_FIN, 0, fin);
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- prep --
    const int pt = tid - kWG;
    const int row = pt & 63;
    if (pt < DK) zs[pt] = p.z0 ? p.z0[(size_t)bh * DK + pt] : 0.f;
    bool ok = true, okp = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      const int n = min(kC, T - c * kC);
      uint8_t* stp = sm + (c % NST) * L::STAGE;
      ok = named_bar_and(kBarPrep, kWG, okp && mbar_wait(bar + B_FULL + 8 * (c % NST), (c / NST) & 1, wc));
      if (!ok) break;
      // ---- feature maps in place: K, Q -> ELU + 1 (rows >= n -> 0) ----
      constexpr int kPieces = L::KB * 2 * (int)(kTile / 16);  // 16-byte pieces of the K and Q tiles
      for (int i = pt; i < kPieces; i += kWG) {
        const int t16 = i / (int)(kTile / 16), off = (i % (int)(kTile / 16)) * 16;
        uint8_t* ptr = stp + (t16 >> 1) * L::KB_STRIDE + (t16 & 1) * kTile + off;
        uint4 u = *reinterpret_cast<uint4*>(ptr);
        if ((off >> 7) >= n) {
          u = make_uint4(0, 0, 0, 0);
        } else {
          uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
            w[e] = pack2_bf16(elu1(f.x), elu1(f.y));
          }
        }
        *reinterpret_cast<uint4*>(ptr) = u;
      }
      fence_proxy_async_smem();
      named_bar_sync(kBarPrep, kWG);
      if (pt == 0) mbar_arrive(bar + B_FMAP);
      {  // partial column sums of K': thread -> (8 columns, row group)
        constexpr int kCC = DK / 8, kRG = kWG / kCC, kRows = kC / kRG;
        const int cc = pt % kCC, rg = pt / kCC;
        const uint8_t* kt = stp + (cc >> 3) * L::KB_STRIDE + L::K_OFF;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          const uint4 u = *reinterpret_cast<const uint4*>(kt + sw128_off(rg * kRows + i, cc & 7));
          const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            acc[2 * e] += f.x;
            acc[2 * e + 1] += f.y;
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[rg * DK + cc * 8 + e] = acc[e];
      }
      // ---- Q' z per row, z entering chunk c (dq[b] was read by the output of chunk c-2) ----
      bool okq = true;
      if (pt < 64) {
        okq = c < 2 || mbar_wait(bar + B_OFREE + 8 * b, ((c >> 1) - 1) & 1, wc);
        float acc = 0.f;
#pragma unroll
        for (int c16 = 0; c16 < DK / 8; ++c16) {
          const uint4 u = *reinterpret_cast<const uint4*>(stp + (c16 >> 3) * L::KB_STRIDE + L::Q_OFF +
                                                          sw128_off(row, c16 & 7));
          const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            acc = fmaf(f.x, zs[c16 * 8 + 2 * e], acc);
            acc = fmaf(f.y, zs[c16 * 8 + 2 * e + 1], acc);
          }
        }
        dq[b * 64 + row] = acc;
      }
      ok = named_bar_and(kBarPrep, kWG, okq);  // every read of the old z is done
      if (!ok) break;
      if (pt < DK) {
        constexpr int kRG = kWG / (DK / 8);
        float a = 0.f;
#pragma unroll
        for (int rg = 0; rg < kRG; ++rg) a += red[rg * DK + pt];
        zs[pt] += a;
      }
      // ---- P rows (TMEM lanes 64-127) to bf16, with their sums ----
      if (pt >= 64) {
        okp = named_bar_and(kBarPrepHi, 64, mbar_wait(bar + B_GDONE + 8 * b, (c >> 1) & 1, wc));
        if (okp) {
          tc_fence_after();
          uint32_t g[64];
          tmem_ld32(tmem + lane_base + TM_G + 64 * b, *reinterpret_cast<uint32_t(*)[32]>(g));
          tmem_ld32(tmem + lane_base + TM_G + 64 * b + 32, *reinterpret_cast<uint32_t(*)[32]>(g + 32));
          tmem_wait_ld();
          float sum = 0.f;
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int sc = c16 * 8 + e;
              x[e] = sc <= row ? __uint_as_float(g[sc]) : 0.f;
              sum += x[e];
            }
            st_bf16x8(sm + L::P_OFF + b * kTile + sw128_off(row, c16), x);
          }
          rs[b * 64 + row] = sum;
          fence_proxy_async_smem();
          tc_fence_before();
          named_bar_sync(kBarPrepHi, 64);
          if (pt == 64) mbar_arrive(bar + B_PREADY + 8 * b);
        }
      }
    }
    if (p.z_out && blockIdx.y == 0 && pt < DK) p.z_out[(size_t)bh * DK + pt] = zs[pt];
  } else {
    // --------------------------------------------------------------- state --
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
    named_bar_sync(kBarState, kWG);
    if (ct == 0) mbar_arrive(bar + B_SREADY);  // the state entering chunk 0, in tile 0

    bool ok = true, ok_lo = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      const int n = min(kC, T - c * kC);
      // ---- S += K'^T V (c) ----
      ok = named_bar_and(kBarState, kWG, ok_lo && mbar_wait(bar + B_DSDONE + 8 * b, (c >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      if (ct < DK) {
        uint32_t ds[64];
        tmem_ld32(tmem + lane_base + TM_DS + 64 * b, *reinterpret_cast<uint32_t(*)[32]>(ds));
        tmem_ld32(tmem + lane_base + TM_DS + 64 * b + 32, *reinterpret_cast<uint32_t(*)[32]>(ds + 32));
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; ++e) sreg[e] += __uint_as_float(ds[e]);
      }
      tc_fence_before();
      named_bar_sync(kBarState, kWG);
      if (ct == 0) mbar_arrive(bar + B_DSFREE + 8 * b);
      // ---- the state entering chunk c+1, as bf16, into tile (c+1) & 1 (last read by O (c-1)) ----
      if (c + 1 < nchunks) {
        ok = named_bar_and(kBarState, kWG,
                           c < 1 || mbar_wait(bar + B_ODONE + 8 * (b ^ 1), ((c - 1) >> 1) & 1, wc));
        if (!ok) break;
        if (ct < DK) {
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16)
            st_bf16x8(sm + L::S_OFF + (b ^ 1) * (DK * 128) + sw128_off(ct, c16), sreg + 8 * c16);
        }
        fence_proxy_async_smem();
        named_bar_sync(kBarState, kWG);
        if (ct == 0) mbar_arrive(bar + B_SREADY + 8 * (b ^ 1));
      }
      // ---- O (c) / (Q' z + P 1) -> global (warps 0-1, TMEM lanes 0-63) ----
      if (ct < 64) {
        ok_lo = named_bar_and(kBarLo, 64, mbar_wait(bar + B_ODONE + 8 * b, (c >> 1) & 1, wc));
        if (ok_lo) {
          tc_fence_after();
          const float inv = 1.f / (dq[b * 64 + row] + rs[b * 64 + row]);
          __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + ((size_t)bh * T + c * kC + row) * Dv + j0;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t ov[32];
            tmem_ld32(tmem + lane_base + TM_O + 64 * b + q * 32, ov);
            tmem_wait_ld();
            if (row < n) {
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(ov[cc * 8 + e]) * inv;
                st_bf16x8(orow + q * 32 + cc * 8, x);
              }
            }
          }
          tc_fence_before();
          named_bar_sync(kBarLo, 64);
          if (ct == 0) mbar_arrive(bar + B_OFREE + 8 * b);
        }
      }
    }
    if (p.S_out && ct < DK) {
      float* dst = p.S_out + s_base + (size_t)ct * Dv + j0;
#pragma unroll
      for (int j = 0; j < kDVS; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DK>
cudaError_t launch_t(const ChunkProblem& p, cudaStream_t st) {
  using L = LinLayout<DK>;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_tmap_3d_bf16(&mq, p.q, DK, p.T, BH) || !make_tmap_3d_bf16(&mk, p.k, DK, p.T, BH) ||
      !make_tmap_3d_bf16(&mv, p.v, p.Dv, p.T, BH))
    return cudaErrorInvalidValue;
  auto kern = linear_tc_kernel<DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)BH, (unsigned)(p.Dv / kDVS));
  kern<<<grid, kThreads, L::ALLOC, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

bool linear_tc_supported(const ChunkProblem& p) {
  return p.bf16 && p.mode == Mode::Linear && p.T > 0 && p.C == 64 && (p.Dk == 64 || p.Dk == 128) &&
         (p.Dv == 64 || p.Dv == 128);
}

cudaError_t launch_linear_tc(const ChunkProblem& p, cudaStream_t st) {
  return p.Dk == 128 ? launch_t<128>(p, st) : launch_t<64>(p, st);
}

}  // namespace dn
