// tcgen05 chunked ELU+1 linear attention (bf16 operands, float32 accumulation,
// state and normaliser): the bf16 path of linear_attn_fwd.
//
// Additive chunk loop of "GPT-2 から Kimi K3 まで" (news.ainew.jp), section
// "DeltaNet (Parallelizing linear transformers with delta rule)", on the ELU+1
// feature maps of section "Linear attention" (and of the linear-attention
// snippet of "How a Baseten Engineer Traced 7 Years of Attention Mechanism
// Evolution"), with the normaliser z carried like S.  Per chunk c of 64 rows
// (Q' = ELU(Q) + 1, K' = ELU(K) + 1, rows past T zero), entered with S, z:
//   P = tril(Q' K'^T)
//   O = (Q' S + P V) / (Q' z + P 1)                  (Q'S + PV in one TMEM tile)
//   S <- S + K'^T V,  z <- z + K'^T 1
// The normaliser rides along in the products: V is augmented with a column of
// ones and S with z as an extra column ([V | 1], [S | z], N = 80), so K'^T [V|1]
// gives both state increments, Q'[S|z] + P[V|1] both numerator and
// denominator.  Only S and z carry from chunk to chunk, and their increment
// does not depend on them, so everything but the accumulate is pipelined ahead.
//
// One CTA per (b, h, 64-column slice of Dv), 18 warps, each role on warps of
// its own so that the per-chunk steps of different roles overlap:
//   warp 16     producer: TMA of K, Q, V into a three-stage ring
//   warp 17     MMA issuer (warp-uniform, one elected lane), per chunk c:
//               Gram (c+1), O (c) = Q'[S|z] + P[V|1] once chunk c's state and
//               P tiles are ready, then dS (c+1) = K'^T [V|1] (c+1)
//   warps 4-11  prep: feature maps in place (rows past T zeroed)
//   warps 0-3   state: [S|z] += K'^T [V|1] in float32 registers, then the
//               bf16 state tile for the next chunk (double-buffered)
//   warps 12-15 P and O: per chunk c, the Gram rows to the bf16 P tile (c),
//               then O (c-1) / (Q'z + P 1) to a bf16 staging tile, stored to
//               global memory by TMA (double-buffered)
// The 64-row products (Q'K'^T, Q'[S|z] + P[V|1]) are M = 64 MMAs: their left
// operands are the 64-row Q' and P tiles alone, and their accumulators hold
// row r on TMEM lane 32 (r / 16) + r % 16, so each of warps 12-15 owns 16
// rows.  Accumulators live in TMEM (G[2], dS[2], O[2]: 448 of 512 columns).
// Every
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
constexpr int kThreads = kWG + kPrep + 192;  // state 0-3, prep 4-11, P and O 12-15, producer 16, issuer 17
constexpr int kWarpProducer = 16, kWarpIssuer = 17;
constexpr int kBarState = 1, kBarPO = 2, kBarPrep = 4;
constexpr int kNA = 80;  // augmented width: 64 columns of V (or S) + the ones (or z) column, padded to 16

// TMEM columns: Gram[2] (Q'K'^T), dS[2] (K'^T [V|1]), O[2]
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
  static constexpr uint32_t OST_OFF = S_OFF + 4 * SBLK;  // O staging tiles [2] for the TMA store
  static constexpr uint32_t BAR_OFF = OST_OFF + 2 * kTile;
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

// ELU(x) + 1 = max(x, 0) + 2^(min(x, 0) log2(e)) on a pair of bf16 values, in
// bf16 arithmetic: the result is a bf16 MMA operand, and a pair costs six
// instructions (one of them the exponential for both halves) instead of a
// float32 round trip per element.  log2(e) is split into two bf16 constants
// (1.4453125 - 0.00262451171875, within 5e-6 of it) so the exponent argument
// is the exactly rounded product; the argument's own bf16 rounding leaves the
// mapped values within 1.4 % (relative, largest for the most negative inputs)
// of the exact map, against 0.4 % for rounding the exact map to bf16.
__device__ __forceinline__ uint32_t elu1_bf16x2(uint32_t x) {
  constexpr uint32_t kZero = 0u, kOne = 0x3F803F80u, kL1 = 0x3FB93FB9u, kL2 = 0xBB2CBB2Cu;
  uint32_t m, u, t, e, pos, r;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(x), "r"(kZero));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(u) : "r"(m), "r"(kL2), "r"(kZero));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(t) : "r"(m), "r"(kL1), "r"(u));
  asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(e) : "r"(t));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(pos) : "r"(x), "r"(kZero));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(pos), "r"(kOne), "r"(e));
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
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const ChunkProblem p) {
  using L = LinLayout<DK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = warp_uniform(smem_u32(sm));
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = (int)warp_uniform((uint32_t)tid >> 5);
  // 1-D grid with the D_v slices of a head adjacent: they are scheduled
  // together, so the second slice's K, Q (and pre-pass) tiles come from L2
  // even when the grid takes more than one wave.
  const int nsl = p.Dv / kDVS;
  const int bh = blockIdx.x / nsl, slice = blockIdx.x % nsl;
  const int j0 = slice * kDVS;
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

  if (warp == kWarpProducer) {
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
  } else if (warp == kWarpIssuer) {
    // -------------------------------------------------------------- issuer --
    // Descriptors are formed once per product and stepped (desc_step): the
    // single issuing warp shares its scheduler with busy warps.
    // Gram (c) = Q' K'^T into G[c & 1] (M = 64)
    auto issue_gram = [&](int c) {
      const uint32_t st = stage(c);
      const int b = c & 1;
      constexpr uint32_t idg = idesc_bf16(64, 64, false, false);
      const uint64_t dq = desc_k(st + L::Q_OFF), dk = desc_k(st + L::K_OFF);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t off = (ks >> 2) * L::KB_STRIDE + (ks & 3) * 32;
        mma_bf16_ss_elect(tmem + TM_G + 64 * b, desc_step(dq, off), desc_step(dk, off), idg, ks > 0);
      }
      mma_commit_elect(bar + B_GDONE + 8 * b);
    };
    // dS (c) = K'^T [V|1] into dS[c & 1]
    auto issue_ds = [&](int c) {
      const uint32_t st = stage(c);
      const int b = c & 1;
      constexpr uint32_t idd = idesc_bf16(128, kNA, true, true);
      const uint32_t ones_lbo = sb + L::ONES_OFF - (st + L::V_OFF);  // [V | 1]: the ones block follows V
      const uint64_t da = desc_mn(st + L::K_OFF, L::KB_STRIDE), dv = desc_mn(st + L::V_OFF, ones_lbo);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_DS + kAugStride * b, desc_step(da, ks * 2048), desc_step(dv, ks * 2048), idd,
                          ks > 0);
      mma_commit_elect(bar + B_DSDONE + 8 * b);
    };
    // O (c) = Q' [S|z] + P [V|1] into O[c & 1] (M = 64)
    auto issue_o = [&](int c) {
      const uint32_t st = stage(c);
      const int b = c & 1;
      constexpr uint32_t ido = idesc_bf16(64, kNA, false, true);
      const uint32_t ones_lbo = sb + L::ONES_OFF - (st + L::V_OFF);
      const uint64_t dq = desc_k(st + L::Q_OFF), ds = desc_mn(sb + L::S_OFF + b * 2 * L::SBLK, L::SBLK);
      const uint64_t dp = desc_k(sb + L::P_OFF + b * kTile), dv = desc_mn(st + L::V_OFF, ones_lbo);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks)
        mma_bf16_ss_elect(tmem + TM_O + kAugStride * b, desc_step(dq, (ks >> 2) * L::KB_STRIDE + (ks & 3) * 32),
                          desc_step(ds, ks * 2048), ido, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_elect(tmem + TM_O + kAugStride * b, desc_step(dp, ks * 32), desc_step(dv, ks * 2048), ido, 1);
      mma_commit_elect(bar + B_ODONE + 8 * b);
      mma_commit_elect(bar + B_EMPTY + 8 * (c % NST));  // stage c: Gram, dS and O have read it
    };
    // Per iteration c: Gram (c+1), then O (c) once chunk c's state and P tiles
    // are ready, then dS (c+1).  The tensor pipe runs MMAs in issue order, so
    // Gram (c+1) (all that P (c+1) needs) runs before O (c) and P (c+1)
    // overlaps O (c); O (c), the last reader of stage c, runs before dS (c+1),
    // so the ring turns over as soon as the state allows.
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FMAP, 0, wc));  // stage 0, first use
    if (ok) {
      tc_fence_after();
      issue_gram(0);
      issue_ds(0);
    }
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      const bool next = c + 1 < nchunks;
      // G[(c+1) & 1] was read by the P rows of chunk c-1 (PREADY waited in iteration c-1)
      if (next) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar + B_FMAP + 8 * ((c + 1) % NST), ((c + 1) / NST) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        issue_gram(c + 1);
      }
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar + B_PREADY + 8 * b, (c >> 1) & 1, wc) &&
                          mbar_wait(bar + B_SREADY + 8 * b, (c >> 1) & 1, wc) &&
                          (c < 2 || mbar_wait(bar + B_OFREE + 8 * b, ((c >> 1) - 1) & 1, wc)));
      if (!ok) break;
      tc_fence_after();
      issue_o(c);
      if (next) {  // dS[(c+1) & 1] must have been added to S (DSFREE of chunk c-1)
        ok = __all_sync(0xffffffffu, c < 1 || mbar_wait(bar + B_DSFREE + 8 * (b ^ 1), ((c - 1) >> 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        issue_ds(c + 1);
      }
    }
    tc_fence_after();  // no MMA may outlive TMEM
    mma_commit_elect(bar + B_FIN);
    int zero = 0;
    const WaitCtl fin{&zero, p.status, kWaitLimitNs};
    (void)mbar_wait(bar + B_FIN, 0, fin);
  } else if (warp >= 4 && warp < 12) {
    // ---------------------------------------------------------------- prep --
    const int pt = tid - kWG;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int n = min(kC, T - c * kC);
      uint8_t* stp = sm + (c % NST) * L::STAGE;
      ok = named_bar_and(kBarPrep, kPrep, mbar_wait(bar + B_FULL + 8 * (c % NST), (c / NST) & 1, wc));
      if (!ok) break;
      // ---- feature maps in place: K, Q -> ELU + 1 (rows >= n -> 0) ----
      // Four 16-byte pieces per thread per round, loaded together so that
      // their exponentials are in flight together.
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
          u[j] = *reinterpret_cast<const uint4*>(ptr[j]);
        }
#pragma unroll
        for (int j = 0; j < kNpf; ++j) {
          uint4 r = make_uint4(elu1_bf16x2(u[j].x), elu1_bf16x2(u[j].y), elu1_bf16x2(u[j].z),
                               elu1_bf16x2(u[j].w));
          if (!live[j]) r = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(ptr[j]) = r;
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(kBarPrep, kPrep);
      if (pt == 0) mbar_arrive(bar + B_FMAP + 8 * (c % NST));
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------- P and O --
    // Row r of the M = 64 accumulators is lane r % 16 of warp 12 + r / 16.
    // Per chunk c: P (c) = tril(Q'K'^T) into the bf16 tile P[c & 1] (the O
    // product that read it two chunks ago was drained by these warps in the
    // previous iteration), then O (c-1) / (Q'z + P 1) into the staging tile
    // [(c-1) & 1] and one TMA store of the 64 x 64 tile (rows past T clipped).
    const int row = 16 * (warp & 3) + lane;
    const bool live = lane < 16;
    const bool leader = warp == 12 && lane == 0;
    auto make_p = [&](int c) -> bool {
      const int b = c & 1;
      if (!named_bar_and(kBarPO, 128, mbar_wait(bar + B_GDONE + 8 * b, (c >> 1) & 1, wc))) return false;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // 32 columns at a time
        uint32_t g[32];
        tmem_ld32(tmem + lane_base + TM_G + 64 * b + 32 * h, g);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int sc = 32 * h + c16 * 8 + e;
              x[e] = sc <= row ? __uint_as_float(g[c16 * 8 + e]) : 0.f;
            }
            st_bf16x8(sm + L::P_OFF + b * kTile + sw128_off(row, 4 * h + c16), x);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarPO, 128);
      if (leader) mbar_arrive(bar + B_PREADY + 8 * b);
      return true;
    };
    auto drain_o = [&](int c) -> bool {
      const int b = c & 1;
      if (leader) bulk_wait_group_read<1>();  // the store of chunk c-2 has read staging tile b
      if (!named_bar_and(kBarPO, 128, mbar_wait(bar + B_ODONE + 8 * b, (c >> 1) & 1, wc))) return false;
      tc_fence_after();
      const uint32_t o0 = tmem + lane_base + TM_O + kAugStride * b;
      const float inv = 1.f / __uint_as_float(tmem_ld1(o0 + 64));
      uint8_t* stg = sm + L::OST_OFF + b * kTile;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t ov[32];
        tmem_ld32(o0 + 32 * h, ov);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(ov[c16 * 8 + e]) * inv;
            st_bf16x8(stg + sw128_off(row, 4 * h + c16), x);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarPO, 128);
      if (leader) {
        mbar_arrive(bar + B_OFREE + 8 * b);
        tma_store_3d(&tmO, smem_u32(stg), j0, c * kC, bh);
        bulk_commit_group();
      }
      return true;
    };
    bool ok = true;
    for (int c = 0; c <= nchunks && ok; ++c) {
      if (c < nchunks) ok = make_p(c);
      if (ok && c >= 1) ok = drain_o(c - 1);
    }
    if (leader) bulk_wait_group_all();
  } else {
    // --------------------------------------------------------------- state --
    const int ct = tid;
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

    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int b = c & 1;
      // ---- [S | z] += K'^T [V | 1] (c) ----
      ok = named_bar_and(kBarState, kWG, mbar_wait(bar + B_DSDONE + 8 * b, (c >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      if (ct < DK) {
        const uint32_t d0 = tmem + lane_base + TM_DS + kAugStride * b;
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // 16 columns at a time (the state already holds 64 registers)
          uint32_t ds[16];
          tmem_ld16(d0 + 16 * h, ds);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) sreg[16 * h + e] += __uint_as_float(ds[e]);
        }
        zreg += __uint_as_float(tmem_ld1(d0 + 64));
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
    }
    if (ct < DK) {
      if (p.S_out) {
        float* dst = p.S_out + s_base + (size_t)ct * Dv + j0;
#pragma unroll
        for (int j = 0; j < kDVS; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
      }
      if (p.z_out && slice == 0) p.z_out[(size_t)bh * DK + ct] = zreg;
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
  CUtensorMap mq, mk, mv, mo;
  const int BH = p.B * p.H;
  if (!make_tmap_3d_bf16(&mq, p.q, DK, p.T, BH) || !make_tmap_3d_bf16(&mk, p.k, DK, p.T, BH) ||
      !make_tmap_3d_bf16(&mv, p.v, p.Dv, p.T, BH) || !make_tmap_3d_bf16(&mo, p.o, p.Dv, p.T, BH))
    return cudaErrorInvalidValue;
  auto kern = linear_tc_kernel<DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(BH * (p.Dv / kDVS)));
  kern<<<grid, kThreads, L::ALLOC, st>>>(mq, mk, mv, mo, p);
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
