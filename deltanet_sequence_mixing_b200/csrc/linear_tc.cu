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
// The normaliser rides along in the products: V is augmented with a column of
// ones and S with z as an extra column ([V | 1], [S | z], N = 80), so K'^T [V|1]
// gives both state increments, Q'[S|z] + P[V|1] both numerator and
// denominator.  Only S and z carry from chunk to chunk, and their increment
// does not depend on them, so everything but the accumulate is pipelined ahead.
//
// One CTA per (b, h, 64-column slice of Dv), 14 warps:
//   warp 12    producer: TMA of K, Q, V into a three-stage ring
//   warp 13    MMA issuer (warp-uniform, one elected lane): Gram (c+1) and
//              K'^T [V|1] (c+1) while chunk c waits for its state tile, then
//              O (c) = Q'[S|z] + P[V|1]
//   warps 4-11 prep: feature maps in place (rows past T zeroed)
//   warps 0-3  state: [S|z] += K'^T [V|1] in float32 registers, the bf16
//              state tile for the next chunk (double-buffered); warps 2-3 turn
//              the Gram rows (TMEM lanes 64-127) into P; warps 0-1 drain
//              O / (Q'z + P 1) to global memory
// Accumulators live in TMEM (G[2], dS[2], O[2]: 448 of 512 columns).  Every
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
constexpr int kPrep = 256;                  // prep threads (warps 4-11)
constexpr int kThreads = kWG + kPrep + 64;  // state 0-3, prep 4-11, producer 12, issuer 13
constexpr int kBarState = 1, kBarLo = 2, kBarHi = 3, kBarPrep = 4;
constexpr int kNA = 80;  // augmented width: 64 columns of V (or S) + the ones (or z) column, padded to 16

// TMEM columns: Gram[2] (lanes 64-127: Q'K'^T), dS[2] (K'^T [V|1]), O[2] (lanes 0-63)
constexpr uint32_t TM_G = 0, TM_DS = 128, TM_O = 320, kAugStride = 96;

template <int DK>
struct LinLayout {
  static constexpr int KB = DK / 64;
  static constexpr uint32_t KB_STRIDE = 2 * kTile;  // [K | Q] per 64 columns of Dk
  static constexpr uint32_t K_OFF = 0, Q_OFF = kTile;
  static constexpr uint32_t V_OFF = KB * KB_STRIDE;
  static constexpr uint32_t STAGE = V_OFF + kTile;
  static constexpr uint32_t ONES_OFF = NST * STAGE;       // 64 x 64 bf16: column 0 ones, rest zero
  static constexpr uint32_t P_OFF = ONES_OFF + kTile;      // P[2]
  // bf16 [S | z] tiles [2]: block 0 = S (DK rows x 128 B), block 1 = z in column 0
  static constexpr uint32_t SBLK = DK * 128;
  static constexpr uint32_t S_OFF = P_OFF + 2 * kTile;
  static constexpr uint32_t BAR_OFF = S_OFF + 4 * SBLK;
  static constexpr uint32_t BYTES = BAR_OFF + 256;
  static constexpr uint32_t ALLOC = BYTES + 1024;
  static_assert(STAGE % 1024 == 0 && P_OFF % 1024 == 0, "128-byte swizzle atoms stay aligned");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// One 32-bit column of this thread's TMEM lane (z or the denominator Q'z + P 1).
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  return r;
}

// mbarrier slots (8 bytes each).  FULL, EMPTY and FMAP per stage; the rest per
// chunk parity.
constexpr uint32_t B_FULL = 0, B_EMPTY = 24, B_FMAP = 48, B_GDONE = 72, B_DSDONE = 88, B_PREADY = 104,
                   B_DSFREE = 120, B_SREADY = 136, B_ODONE = 152, B_OFREE = 168, B_FIN = 184,
                   B_TMEM = 192, B_ABORT = 196;

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

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(bar + B_FULL + 8 * i, 1);
      mbar_init(bar + B_EMPTY + 8 * i, 1);
      mbar_init(bar + B_FMAP + 8 * i, 1);
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
    mbar_init(bar + B_FIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // constant column of ones next to V; the z blocks of the state tiles start at zero
  for (int i = tid; i < (int)(kTile / 16); i += kThreads) {
    const int r = i >> 3, c16 = i & 7;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (c16 == 0) u.x = 0x3F80u;  // bf16 1.0 in the first element of the row's first chunk
    *reinterpret_cast<uint4*>(sm + L::ONES_OFF + sw128_off(r, c16)) = u;
  }
  for (int i = tid; i < (int)(2 * L::SBLK / 16); i += kThreads)
    *reinterpret_cast<uint4*>(sm + L::S_OFF + (i / (L::SBLK / 16)) * 2 * L::SBLK + L::SBLK +
                              (i % (L::SBLK / 16)) * 16) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
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

  if (warp == 12) {
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
  } else if (warp == 13) {
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
      constexpr uint32_t idd = idesc_bf16(128, kNA, true, true);
      const uint32_t ones_lbo = sb + L::ONES_OFF - (st + L::V_OFF);  // [V | 1]: the ones block follows V
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_DS + kAugStride * b, desc_mn(st + L::K_OFF + ks * 2048, L::KB_STRIDE),
                          desc_mn(st + L::V_OFF + ks * 2048, ones_lbo), idd, ks > 0);
      mma_commit_elect(bar + B_DSDONE + 8 * b);
    };
    // O (c) = Q' [S|z] + P [V|1] into O[c & 1] (lanes 0-63)
    auto issue_o = [&](int c) {
      const uint32_t st = stage(c);
      const int b = c & 1;
      constexpr uint32_t ido = idesc_bf16(128, kNA, false, true);
      const uint32_t ones_lbo = sb + L::ONES_OFF - (st + L::V_OFF);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t a = st + (ks >> 2) * L::KB_STRIDE + L::Q_OFF + (ks & 3) * 32;
        mma_bf16_ss_elect(tmem + TM_O + kAugStride * b, desc_k(a),
                          desc_mn(sb + L::S_OFF + b * 2 * L::SBLK + ks * 2048, L::SBLK), ido, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_O + kAugStride * b, desc_k(sb + L::P_OFF + b * kTile + ks * 32),
                          desc_mn(st + L::V_OFF + ks * 2048, ones_lbo), ido, 1);
      mma_commit_elect(bar + B_ODONE + 8 * b);
      mma_commit_elect(bar + B_EMPTY + 8 * (c % NST));  // stage c: Gram, dS and O have read it
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FMAP, 0, wc));  // stage 0, first use
    if (ok) {
      tc_fence_after();
      issue_gram_ds(0);
    }
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      if (c + 1 < nchunks) {  // the next chunk's Gram and K'^T V run while chunk c waits for its state
        // G[(c+1) & 1] was read by the P rows of chunk c-1 (PREADY waited below in
        // iteration c-1); dS[(c+1) & 1] must have been added to S (DSFREE of chunk c-1)
        ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FMAP + 8 * ((c + 1) % NST), ((c + 1) / NST) & 1, wc) &&
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
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int n = min(kC, T - c * kC);
      uint8_t* stp = sm + (c % NST) * L::STAGE;
      ok = named_bar_and(kBarPrep, kPrep, mbar_wait(bar + B_FULL + 8 * (c % NST), (c / NST) & 1, wc));
      if (!ok) break;
      // ---- feature maps in place: K, Q -> ELU + 1 (rows >= n -> 0) ----
      // Four 16-byte pieces per thread per round, in stages (all loads, all
      // exponentials, then the packs and stores) so the exponentials of 32
      // elements are in flight together.
      constexpr int kPieces = L::KB * 2 * (int)(kTile / 16);  // 16-byte pieces of the K and Q tiles
      constexpr int kNpf = 4;
      static_assert(kPieces % (kNpf * kPrep) == 0, "whole rounds of pieces per thread");
      for (int i0 = pt; i0 < kPieces; i0 += kNpf * kPrep) {
        uint4 u[kNpf];
        uint8_t* ptr[kNpf];
        bool live[kNpf];
#pragma unroll
        for (int j = 0; j < kNpf; ++j) {
          const int i = i0 + j * kPrep;
          const int t16 = i / (int)(kTile / 16), off = (i % (int)(kTile / 16)) * 16;
          ptr[j] = stp + (t16 >> 1) * L::KB_STRIDE + (t16 & 1) * kTile + off;
          live[j] = (off >> 7) < n;
          u[j] = live[j] ? *reinterpret_cast<const uint4*>(ptr[j]) : make_uint4(0, 0, 0, 0);
        }
        float f[kNpf * 8], ex[kNpf * 8];
#pragma unroll
        for (int j = 0; j < kNpf; ++j) {
          const uint32_t* w = reinterpret_cast<const uint32_t*>(&u[j]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {  // bf16 pair -> two floats (low element first)
            f[j * 8 + 2 * e] = __uint_as_float(w[e] << 16);
            f[j * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
          }
        }
#pragma unroll
        for (int k = 0; k < kNpf * 8; ++k) ex[k] = __expf(fminf(f[k], 0.f));
#pragma unroll
        for (int j = 0; j < kNpf; ++j) {
          uint4 r;
          uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
          for (int e = 0; e < 4; ++e)  // ELU(x) + 1 = max(x, 0) + e^min(x, 0)
            w[e] = pack2_bf16(fmaxf(f[j * 8 + 2 * e], 0.f) + ex[j * 8 + 2 * e],
                              fmaxf(f[j * 8 + 2 * e + 1], 0.f) + ex[j * 8 + 2 * e + 1]);
          if (!live[j]) r = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(ptr[j]) = r;
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(kBarPrep, kPrep);
      if (pt == 0) mbar_arrive(bar + B_FMAP + 8 * (c % NST));
    }
  } else {
    // --------------------------------------------------------------- state --
    const int ct = tid;
    const int row = ct & 63;
    const size_t s_base = (size_t)bh * DK * Dv;
    float sreg[kDVS], zreg = 0.f;
    // one row of [S | z] as bf16 into tile t (z in column 0 of the second block)
    auto put_state = [&](int t) {
      uint8_t* tile = sm + L::S_OFF + t * 2 * L::SBLK;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) st_bf16x8(tile + sw128_off(ct, c16), sreg + 8 * c16);
      const float zrow[8] = {zreg, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      st_bf16x8(tile + L::SBLK + sw128_off(ct, 0), zrow);
    };
    if (ct < DK) {
      const float* src = p.S0 ? p.S0 + s_base + (size_t)ct * Dv + j0 : nullptr;
#pragma unroll
      for (int j = 0; j < kDVS; j += 4) {
        const float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        sreg[j] = v.x; sreg[j + 1] = v.y; sreg[j + 2] = v.z; sreg[j + 3] = v.w;
      }
      zreg = p.z0 ? p.z0[(size_t)bh * DK + ct] : 0.f;
      put_state(0);
    }
    fence_proxy_async_smem();
    named_bar_sync(kBarState, kWG);
    if (ct == 0) mbar_arrive(bar + B_SREADY);  // the state entering chunk 0, in tile 0

    bool ok = true, ok_lo = true, ok_hi = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      const int n = min(kC, T - c * kC);
      // ---- P = tril(Q'K'^T) rows (TMEM lanes 64-127) to bf16 (warps 2-3) ----
      if (ct >= 64) {
        ok_hi = named_bar_and(kBarHi, 64, mbar_wait(bar + B_GDONE + 8 * b, (c >> 1) & 1, wc));
        if (ok_hi) {
          tc_fence_after();
          uint32_t g[64];
          tmem_ld32(tmem + lane_base + TM_G + 64 * b, *reinterpret_cast<uint32_t(*)[32]>(g));
          tmem_ld32(tmem + lane_base + TM_G + 64 * b + 32, *reinterpret_cast<uint32_t(*)[32]>(g + 32));
          tmem_wait_ld();
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int sc = c16 * 8 + e;
              x[e] = sc <= row ? __uint_as_float(g[sc]) : 0.f;
            }
            st_bf16x8(sm + L::P_OFF + b * kTile + sw128_off(row, c16), x);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          named_bar_sync(kBarHi, 64);
          if (ct == 64) mbar_arrive(bar + B_PREADY + 8 * b);
        }
      }
      // ---- [S | z] += K'^T [V | 1] (c) ----
      ok = named_bar_and(kBarState, kWG,
                         ok_hi && ok_lo && mbar_wait(bar + B_DSDONE + 8 * b, (c >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      if (ct < DK) {
        const uint32_t d0 = tmem + lane_base + TM_DS + kAugStride * b;
        uint32_t ds[64];
        tmem_ld32(d0, *reinterpret_cast<uint32_t(*)[32]>(ds));
        tmem_ld32(d0 + 32, *reinterpret_cast<uint32_t(*)[32]>(ds + 32));
        const uint32_t dz = tmem_ld1(d0 + 64);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; ++e) sreg[e] += __uint_as_float(ds[e]);
        zreg += __uint_as_float(dz);
      }
      tc_fence_before();
      named_bar_sync(kBarState, kWG);
      if (ct == 0) mbar_arrive(bar + B_DSFREE + 8 * b);
      // ---- the state entering chunk c+1, as bf16, into tile (c+1) & 1 (last read by O (c-1)) ----
      if (c + 1 < nchunks) {
        ok = named_bar_and(kBarState, kWG,
                           c < 1 || mbar_wait(bar + B_ODONE + 8 * (b ^ 1), ((c - 1) >> 1) & 1, wc));
        if (!ok) break;
        if (ct < DK) put_state(b ^ 1);
        fence_proxy_async_smem();
        named_bar_sync(kBarState, kWG);
        if (ct == 0) mbar_arrive(bar + B_SREADY + 8 * (b ^ 1));
      }
      // ---- O (c) / (Q'z + P 1) -> global (warps 0-1, TMEM lanes 0-63) ----
      if (ct < 64) {
        ok_lo = named_bar_and(kBarLo, 64, mbar_wait(bar + B_ODONE + 8 * b, (c >> 1) & 1, wc));
        if (ok_lo) {
          tc_fence_after();
          const uint32_t o0 = tmem + lane_base + TM_O + kAugStride * b;
          uint32_t ov[64];
          tmem_ld32(o0, *reinterpret_cast<uint32_t(*)[32]>(ov));
          tmem_ld32(o0 + 32, *reinterpret_cast<uint32_t(*)[32]>(ov + 32));
          const uint32_t od = tmem_ld1(o0 + 64);
          tmem_wait_ld();
          if (row < n) {
            const float inv = 1.f / __uint_as_float(od);
            __nv_bfloat16* orow =
                static_cast<__nv_bfloat16*>(p.o) + ((size_t)bh * T + c * kC + row) * Dv + j0;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              float x[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(ov[cc * 8 + e]) * inv;
              st_bf16x8(orow + cc * 8, x);
            }
          }
          tc_fence_before();
          named_bar_sync(kBarLo, 64);
          if (ct == 0) mbar_arrive(bar + B_OFREE + 8 * b);
        }
      }
    }
    if (ct < DK) {
      if (p.S_out) {
        float* dst = p.S_out + s_base + (size_t)ct * Dv + j0;
#pragma unroll
        for (int j = 0; j < kDVS; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
      }
      if (p.z_out && blockIdx.y == 0) p.z_out[(size_t)bh * DK + ct] = zreg;
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
