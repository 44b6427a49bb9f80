// tcgen05 chunked ELU+1 linear attention (bf16 operands, float32 accumulation,
// state and normaliser): the bf16 path of linear_attn_fwd.
//
// Additive chunk loop of "GPT-2 から Kimi K3 まで" (news.ainew.jp), section
// "DeltaNet (Parallelizing linear transformers with delta rule)", on the ELU+1
// feature maps of section "Linear attention" (and of the linear-attention
// snippet of "How a Baseten Engineer Traced 7 Years of Attention Mechanism
// Evolution"), with the normaliser z carried like S.
//
// Hardware mapping (sm_100a): one CTA per (b, h, 64-column slice of Dv).
// Warps 0-3 own TMEM lanes 0-127 and do the epilogues; warp 4 streams q, k, v
// chunks with TMA (128-byte swizzle, 3-D maps so a ragged tail reads zeros)
// into a two-stage ring; thread 0 issues the tcgen05 MMAs.  All operands live in
// shared memory in the 128-byte-swizzled canonical layout, accumulators in
// TMEM, the running state in float32 registers (one state row per thread).
// Every wait is bounded; a wait that runs out sets the workspace status word
// and the CTA winds down cleanly (outstanding copies drained, TMEM freed).
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

constexpr int kC = 64;              // chunk rows
constexpr int kDVS = 64;            // state columns per CTA
constexpr uint32_t kTile = 8192;    // 64 rows x 128 bytes
constexpr int kCompute = 128;       // warps 0-3
constexpr int kThreads = kCompute + 32;
constexpr int kApad = 68;           // float row stride of the A / T scratch

// TMEM column map (512 columns allocated).
constexpr uint32_t TM_G = 0, TM_W = 64, TM_UH = 192, TM_QW = 256, TM_PU = 320, TM_DS = 384;

template <int DK>
struct TcLayout {
  static constexpr int KB = DK / 64;                       // 64-column blocks of Dk
  static constexpr uint32_t KB_STRIDE = 3 * kTile;         // [K | Q | W] per block
  static constexpr uint32_t K_OFF = 0, Q_OFF = kTile, W_OFF = 2 * kTile;
  static constexpr uint32_t V_OFF = KB * KB_STRIDE;
  static constexpr uint32_t STAGE = KB * KB_STRIDE + kTile;
  static constexpr uint32_t PT_OFF = 2 * STAGE;            // [P | Tb | Tbg]
  static constexpr uint32_t S_OFF = PT_OFF + 3 * kTile;    // bf16 state, DK rows x 128 B
  static constexpr uint32_t U_OFF = S_OFF + DK * 128;
  static constexpr uint32_t UT_OFF = U_OFF + kTile;        // decay-weighted U (gated)
  static constexpr uint32_t AM_OFF = UT_OFF + kTile;       // fp32 A (64 x kApad)
  static constexpr uint32_t TM_OFF = AM_OFF + 64 * kApad * 4;
  static constexpr uint32_t VEC_OFF = TM_OFF + 64 * kApad * 4;  // beta[64], g[64]
  static constexpr uint32_t BAR_OFF = VEC_OFF + 2 * 64 * 4;
  static constexpr uint32_t BYTES = BAR_OFF + 64;
  static constexpr uint32_t ALLOC = BYTES + 1024;          // 1024-byte alignment slack
  static_assert(BYTES + 1024 <= 232448, "shared memory budget");
};

__device__ __forceinline__ bool bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred pi, po; setp.ne.u32 pi, %1, 0; bar.red.and.pred po, 1, 128, pi;"
      " selp.u32 %0, 1, 0, po; }"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_compute() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Write 8 consecutive floats as one 16-byte bf16 chunk.
__device__ __forceinline__ void st_chunk(uint8_t* dst, const float* x) {
  uint4 u;
  u.x = pack_bf16(x[0], x[1]);
  u.y = pack_bf16(x[2], x[3]);
  u.z = pack_bf16(x[4], x[5]);
  u.w = pack_bf16(x[6], x[7]);
  *reinterpret_cast<uint4*>(dst) = u;
}

__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return sw128_desc(addr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) {
  return sw128_desc(addr, lbo, 1024);
}

// ------------------------------------------------- ELU+1 linear attention --
//
// Additive chunk loop of "GPT-2 から Kimi K3 まで" (news.ainew.jp), section "DeltaNet
// (Parallelizing linear transformers with delta rule)", on the ELU+1 feature
// maps of section "Linear attention", with the normaliser z carried like S:
//   Q' = ELU(Q)+1, K' = ELU(K)+1 (applied in shared memory after the TMA load;
//   rows past T are zeroed so they add nothing)
//   P  = tril(Q' K'^T)                              (M = 128 MMA [K';Q'] K'^T)
//   O  = (Q' S + P V) / (Q' z + P 1)                (Q'S + PV in one TMEM tile)
//   S += K'^T V,  z += K'^T 1
// Warps 0-3 compute, warp 4 streams tiles.
template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const ChunkProblem p) {
  using L = TcLayout<DK>;
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

  const uint32_t bar_full0 = sb + L::BAR_OFF, bar_empty0 = sb + L::BAR_OFF + 16;
  const uint32_t bar_mma = sb + L::BAR_OFF + 32, bar_fin = sb + L::BAR_OFF + 40;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::BAR_OFF + 48);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::BAR_OFF + 52);
  // fp32 scratch (reuses the A / T area of the delta layout)
  float* zs = reinterpret_cast<float*>(sm + L::AM_OFF);  // z, DK
  float* zc = zs + 128;                                  // chunk column sums of K', DK
  float* dq = zc + 128;                                  // Q' z per row, 64
  float* rs = dq + 64;                                   // row sums of P, 64
  // partial column sums of K' per row group: [128 / (DK / 8)][DK]
  float* red = reinterpret_cast<float*>(sm + L::AM_OFF + 4096);

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_full0 + 8 * s, 1);
      mbar_init(bar_empty0 + 8 * s, 1);
    }
    mbar_init(bar_mma, 1);
    mbar_init(bar_fin, 1);
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

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, use = c >> 1;
        if (use > 0 && !mbar_wait(bar_empty0 + 8 * s, (use - 1) & 1, wc)) break;
        const uint32_t st = sb + s * L::STAGE;
        const uint32_t full = bar_full0 + 8 * s;
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
        (void)mbar_wait(bar_full0 + 8 * (c & 1), (c >> 1) & 1, drain);
    }
  } else {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const size_t s_base = (size_t)bh * DK * Dv;
    const int row = tid & 63;
    float sreg[kDVS];
    if (tid < DK) {
      const float* src = p.S0 ? p.S0 + s_base + (size_t)tid * Dv + j0 : nullptr;
#pragma unroll
      for (int j = 0; j < kDVS; j += 4) {
        float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        sreg[j] = v.x; sreg[j + 1] = v.y; sreg[j + 2] = v.z; sreg[j + 3] = v.w;
      }
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) st_chunk(sm + L::S_OFF + sw128_off(tid, c16), sreg + 8 * c16);
      zs[tid] = p.z0 ? p.z0[(size_t)bh * DK + tid] : 0.f;
    }
    fence_proxy_async_smem();
    bar_compute();

    uint32_t mma_count = 0;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int s = c & 1, use = c >> 1;
      const int c0 = c * kC, n = min(kC, T - c0);
      const uint32_t st = sb + s * L::STAGE;
      uint8_t* stp = sm + s * L::STAGE;
      ok = bar_and(mbar_wait(bar_full0 + 8 * s, use & 1, wc));
      if (!ok) break;

      // ---- feature map in place: K, Q tiles -> ELU + 1 (rows >= n -> 0) ----
      constexpr int kChunks = L::KB * 2 * (int)(kTile / 16);
      for (int i = tid; i < kChunks; i += kCompute) {
        const int t16 = i / (int)(kTile / 16), off = (i % (int)(kTile / 16)) * 16;
        uint8_t* ptr = stp + (t16 >> 1) * L::KB_STRIDE + (t16 & 1) * kTile + off;
        const int r = off >> 7;
        uint4 u = *reinterpret_cast<uint4*>(ptr);
        if (r >= n) {
          u = make_uint4(0, 0, 0, 0);
        } else {
          uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w[e]);
            float2 f = __bfloat1622float2(h);
            f.x = f.x > 0.f ? f.x + 1.f : __expf(f.x);
            f.y = f.y > 0.f ? f.y + 1.f : __expf(f.y);
            w[e] = pack_bf16(f.x, f.y);
          }
        }
        *reinterpret_cast<uint4*>(ptr) = u;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      bar_compute();

      if (warp == 0) {  // warp-uniform issue, one elected lane
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t a = st + (ks >> 2) * L::KB_STRIDE + L::K_OFF + (ks & 3) * 32;
          mma_bf16_ss_elect(tmem + TM_G, kdesc(a), kdesc(a), id, ks > 0);
        }
        mma_commit_elect(bar_mma);
      }
      // meanwhile: Q' z per row (threads 0-63) and K' column sums (threads < DK)
      if (tid < 64) {
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
        dq[row] = acc;
      }
      {  // partial column sums of K' (rows past n are zero): thread -> (8 columns, row group)
        constexpr int kCC = DK / 8, kRG = kCompute / kCC, kRows = kC / kRG;
        const int cc = tid % kCC, rg = tid / kCC;
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
      ok = bar_and(mbar_wait(bar_mma, mma_count & 1, wc));
      ++mma_count;
      if (!ok) break;
      tc_fence_after();

      // ---- P = tril(Q'K'^T) (lanes 64-127) and its row sums ----
      {
        uint32_t g[64];
        tmem_ld32(tmem + lane_base + TM_G, *reinterpret_cast<uint32_t(*)[32]>(g));
        tmem_ld32(tmem + lane_base + TM_G + 32, *reinterpret_cast<uint32_t(*)[32]>(g + 32));
        tmem_wait_ld();
        if (tid >= 64) {
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
            st_chunk(sm + L::PT_OFF + sw128_off(row, c16), x);
          }
          rs[row] = sum;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      bar_compute();

      // ---- O = Q'S + P V (lanes 0-63), dS = K'^T V ----
      if (warp == 0) {  // warp-uniform issue, one elected lane
        tc_fence_after();
        constexpr uint32_t ido = idesc_bf16(128, 64, false, true);
        constexpr uint32_t ids = idesc_bf16(128, 64, true, true);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t a = st + (ks >> 2) * L::KB_STRIDE + L::Q_OFF + (ks & 3) * 32;
          mma_bf16_ss_elect(tmem + TM_QW, kdesc(a), mndesc(sb + L::S_OFF + ks * 2048, kTile), ido, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_bf16_ss_elect(tmem + TM_QW, kdesc(sb + L::PT_OFF + ks * 32),
                            mndesc(st + L::V_OFF + ks * 2048, kTile), ido, 1);
          mma_bf16_ss_elect(tmem + TM_DS, mndesc(st + L::K_OFF + ks * 2048, L::KB_STRIDE),
                            mndesc(st + L::V_OFF + ks * 2048, kTile), ids, ks > 0);
        }
        mma_commit_elect(bar_mma);
        mma_commit_elect(bar_empty0 + 8 * s);
      }
      ok = bar_and(mbar_wait(bar_mma, mma_count & 1, wc));
      ++mma_count;
      if (!ok) break;
      tc_fence_after();

      if (tid < 64) {
        const float inv = 1.f / (dq[row] + rs[row]);
        __nv_bfloat16* orow =
            static_cast<__nv_bfloat16*>(p.o) + ((size_t)bh * T + c0 + row) * Dv + j0;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + TM_QW + q * 32, ov);
          tmem_wait_ld();
          if (row < n) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              float x[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(ov[cc * 8 + e]) * inv;
              st_chunk(reinterpret_cast<uint8_t*>(orow + q * 32 + cc * 8), x);
            }
          }
        }
      }
      if (tid < DK) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t ds[32];
          tmem_ld32(tmem + lane_base + TM_DS + q * 32, ds);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) sreg[q * 32 + e] += __uint_as_float(ds[e]);
        }
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) st_chunk(sm + L::S_OFF + sw128_off(tid, c16), sreg + 8 * c16);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      bar_compute();  // every read of the old z is done
      if (tid < DK) {
        constexpr int kRG = kCompute / (DK / 8);
        float a = 0.f;
#pragma unroll
        for (int rg = 0; rg < kRG; ++rg) a += red[rg * DK + tid];
        zs[tid] += a;
      }
    }

    if (tid < DK) {
      if (p.S_out) {
        float* dst = p.S_out + s_base + (size_t)tid * Dv + j0;
#pragma unroll
        for (int j = 0; j < kDVS; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
      }
      if (p.z_out && blockIdx.y == 0) p.z_out[(size_t)bh * DK + tid] = zs[tid];
    }
    if (warp == 0) {
      tc_fence_after();
      mma_commit_elect(bar_fin);
      int zero = 0;
      const WaitCtl fin{&zero, p.status, kWaitLimitNs};
      (void)mbar_wait(bar_fin, 0, fin);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host ---

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D map over a (BH, T, D) bf16 tensor with a 64 x 64 box, 128-byte swizzle;
// rows past T read as zeros.
bool make_map(CUtensorMap* m, const void* base, int D, int T, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK>
cudaError_t launch_t(const ChunkProblem& p, cudaStream_t st) {
  using L = TcLayout<DK>;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_map(&mq, p.q, DK, p.T, BH) || !make_map(&mk, p.k, DK, p.T, BH) ||
      !make_map(&mv, p.v, p.Dv, p.T, BH))
    return cudaErrorInvalidValue;
  auto kern = linear_tc_kernel<DK>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
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
