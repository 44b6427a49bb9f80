// The two small kernels of the sequence split.  The chunk transition of the
// delta rule is affine in the state ("GPT-2 から Kimi K3 まで", news.ainew.jp,
// section "DeltaNet (Parallelizing linear transformers with delta rule)": a
// product of generalised Householder factors plus a write), so a sequence cut
// into G segments can run the segments side by side and join them afterwards:
//
//   pass 1 (the chunk kernel on the sequence reshaped to (B*H*G, T/G)):
//     segment 0 from S0, segments g >= 1 from zero: outputs O'_g, end states Send[g];
//     beside it the homogeneous chain of every segment (v = 0, S0 = I): the
//     product A[g] of its transitions and the rows R_g = (diag(gamma) Q - P W) S^hom;
//   combine: Sin[1] = Send[0], Sin[g+1] = A[g] Sin[g] + Send[g], S_out = A[G-1] Sin[G-1] + Send[G-1];
//   correct: O_g = O'_g + R_g Sin[g] for g >= 1 (the outputs are linear in the entry state).
#include <cuda_bf16.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

// 16-byte asynchronous copy global -> shared; src_bytes = 0 fills zeros and reads nothing.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}


// tf32 tensor-core product D += A B on one 16 x 8 tile (mma.sync m16n8k8,
// float32 accumulation).  Lane l holds A at rows l/4 (a0, a2) and l/4 + 8
// (a1, a3), columns l % 4 (a0, a1) and l % 4 + 4 (a2, a3); B at rows l % 4
// (b0) and l % 4 + 4 (b1), column l/4; D as for the bf16 product below.
__device__ __forceinline__ void mma_1688_tf32(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// x = hi + lo with hi, lo tf32 (round to nearest): the three products
// hi*hi + hi*lo + lo*hi carry x*y to about float32 accuracy (the split
// product of Markidis et al., "NVIDIA Tensor Core Programmability,
// Performance & Precision", 2018).
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
  const float r = x - __uint_as_float(hi);
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(r));
}

// One CTA per (b, h, NC-column slice of Dv; NC = 8 or 16), DK / 8 warps: the G - 1
// sequential steps S <- A[g] S + Send[g], each product on the tensor cores as
// three tf32 products of the split operands, accumulated in float32.  Warp w
// takes rows 16 (w % (DK/16)) .. + 15 of the slice and one half of the k
// range; the second half's partial sums meet the first's in shared memory.
// The state is kept already split (tf32 hi and lo words), A[g + 1] streams
// into shared memory while step g computes, and each step's Send values are
// loaded before its product and added after it.
template <int DK, int NC>
__global__ void __launch_bounds__(4 * DK) seg_combine_kernel(const float* __restrict__ Send,
                                                              const float* __restrict__ A, float* __restrict__ Sin,
                                                              float* __restrict__ S_out, int G, int Dv) {
  constexpr int NT = 4 * DK;   // threads
  constexpr int RW = DK / 16;  // row groups (warps per k half)
  constexpr int AP = DK + 4;   // padded row of A: fragment reads hit 32 banks
  constexpr int NTL = NC / 8;  // 8-column tiles of the slice
  constexpr int CS = NC == 16 ? 24 : 8;  // (padded) row of the state slice: fragment reads hit 32 banks
  constexpr int KH = DK / 16;  // 8-wide k tiles per half
  extern __shared__ __align__(16) float seg_smem[];
  float* As = seg_smem;                                             // 2 x DK x AP
  uint32_t* ch = reinterpret_cast<uint32_t*>(As + 2 * DK * AP);     // DK x CS, state (tf32 hi)
  uint32_t* cl = ch + DK * CS;                                      // DK x CS, state (tf32 lo)
  float* red = reinterpret_cast<float*>(cl + DK * CS);              // RW x (NTL x 128), second-half sums
  const int nsl = Dv / NC;
  const int bh = blockIdx.x / nsl, j0 = (blockIdx.x % nsl) * NC;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rw = warp % RW, kh = warp / RW, r0 = 16 * rw;
  const int lr = lane / 4, lc = lane % 4;
  const size_t sblk = (size_t)DK * Dv, ablk = (size_t)DK * DK;
  auto load_a = [&](int g, int buf) {
    const float* src = A + ((size_t)bh * G + g) * ablk;
    for (int i = tid; i < DK * DK / 4; i += NT) {
      const int r = (4 * i) / DK, c = (4 * i) % DK;
      cp_async16(As + buf * DK * AP + r * AP + c, src + 4 * i, 16);
    }
    cp_async_commit();
  };
  // this lane's values of the slice: rows r0 + lr + 8 h, columns 8 nt + 2 lc + {0, 1}
  auto elem = [&](int nt, int h) { return (size_t)(r0 + lr + 8 * h) * Dv + j0 + 8 * nt + 2 * lc; };
  auto put_state = [&](int nt, int h, float x0, float x1) {
    const int c = (r0 + lr + 8 * h) * CS + 8 * nt + 2 * lc;
    uint32_t h0, l0, h1, l1;
    split_tf32(x0, h0, l0);
    split_tf32(x1, h1, l1);
    *reinterpret_cast<uint2*>(ch + c) = make_uint2(h0, h1);
    *reinterpret_cast<uint2*>(cl + c) = make_uint2(l0, l1);
  };
  load_a(1, 0);
  // Sin[1] = Send[0]
  if (kh == 0) {
#pragma unroll
    for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 x = *reinterpret_cast<const float2*>(Send + (size_t)bh * G * sblk + elem(nt, h));
        put_state(nt, h, x.x, x.y);
        *reinterpret_cast<float2*>(Sin + ((size_t)bh * G + 1) * sblk + elem(nt, h)) = x;
      }
  }
  for (int g = 1; g < G; ++g) {
    const int buf = (g - 1) & 1;
    float2 sg[NTL][2];
    if (kh == 0) {
#pragma unroll
      for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          sg[nt][h] = *reinterpret_cast<const float2*>(Send + ((size_t)bh * G + g) * sblk + elem(nt, h));
    }
    if (g + 1 < G) {
      load_a(g + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // A[g] and the state are complete; red is free
    // independent accumulators (k-tile parity x column tile, the hi*hi
    // product apart from the two correction terms) keep eight mma chains in flight
    float big[2][NTL][4] = {}, sml[2][NTL][4] = {};
    const float* Ab = As + buf * DK * AP + (r0 + lr) * AP + lc;
#pragma unroll
    for (int j = 0; j < KH; ++j) {
      const int kt = kh * KH + j;
      uint32_t ah[4], al[4];
      split_tf32(Ab[8 * kt], ah[0], al[0]);
      split_tf32(Ab[8 * AP + 8 * kt], ah[1], al[1]);
      split_tf32(Ab[8 * kt + 4], ah[2], al[2]);
      split_tf32(Ab[8 * AP + 8 * kt + 4], ah[3], al[3]);
#pragma unroll
      for (int nt = 0; nt < NTL; ++nt) {
        const int b0 = (8 * kt + lc) * CS + 8 * nt + lr, b1 = b0 + 4 * CS;
        const uint32_t bhi[2] = {ch[b0], ch[b1]}, blo[2] = {cl[b0], cl[b1]};
        mma_1688_tf32(sml[j & 1][nt], al, bhi);
        mma_1688_tf32(sml[j & 1][nt], ah, blo);
        mma_1688_tf32(big[j & 1][nt], ah, bhi);
      }
    }
    float acc[NTL][4];
#pragma unroll
    for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        acc[nt][e] = (big[0][nt][e] + big[1][nt][e]) + (sml[0][nt][e] + sml[1][nt][e]);
    if (kh == 1) {
#pragma unroll
      for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[rw * NTL * 128 + (4 * nt + e) * 32 + lane] = acc[nt][e];
    }
    __syncthreads();  // every warp has read the state and As[buf]; red holds the second halves
    if (kh == 0) {
      // the next segment's entry state, or the final state (S_out may be NULL)
      float* dst =
          g + 1 < G ? Sin + ((size_t)bh * G + g + 1) * sblk : (S_out ? S_out + (size_t)bh * sblk : nullptr);
#pragma unroll
      for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float x0 = acc[nt][2 * h] + red[rw * NTL * 128 + (4 * nt + 2 * h) * 32 + lane] + sg[nt][h].x;
          const float x1 =
              acc[nt][2 * h + 1] + red[rw * NTL * 128 + (4 * nt + 2 * h + 1) * 32 + lane] + sg[nt][h].y;
          put_state(nt, h, x0, x1);
          if (dst) *reinterpret_cast<float2*>(dst + elem(nt, h)) = make_float2(x0, x1);
        }
    }
  }
}

// bf16 tensor-core product D += A B on one 16 x 8 tile (mma.sync m16n8k16,
// float32 accumulation).  Lane l holds A rows l/4 and l/4 + 8, B column l/4,
// and D at rows l/4 (d0, d1) and l/4 + 8 (d2, d3), columns 2 (l % 4) + {0, 1}.
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// The four 8 x 8 bf16 matrices of a 16 x 16 A tile from shared memory.
__device__ __forceinline__ void ldmatrix_x4(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// One CTA per (b, h, segment g >= 1, run of `rpc` 64-row blocks), DV / 32
// warps: O[rows] += R[rows] Sin[g].  Warp w owns output columns 32 w .. + 31
// and keeps that slice of Sin[g], rounded to bf16, in registers as the
// product's B operand for the whole run; the 64-row R blocks stream through
// shared memory (cp.async, two buffers) and every warp reads them as A.  The
// block's output values are loaded before the products (in flight while they
// run) and written back from the accumulators.
template <int DK, int DV>
__global__ void __launch_bounds__(DV) seg_correct_kernel(__nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ R,
                                                         const float* __restrict__ Sin, int G, int Tg, int rpc) {
  constexpr int NT = DV;                // threads: DV / 32 warps
  constexpr int RP = DK + 8;            // padded bf16 row of an R block (conflict-free ldmatrix)
  constexpr int RV = 64 * DK / 8 / NT;  // 16-byte pieces of an R block per thread
  constexpr int KT = DK / 16;           // k tiles
  extern __shared__ __align__(128) unsigned char seg_smem_c[];
  __nv_bfloat16* Rs = reinterpret_cast<__nv_bfloat16*>(seg_smem_c);  // 2 x 64 x RP
  const int nrb = (Tg + 63) / 64, per = (nrb + rpc - 1) / rpc;
  int blk = blockIdx.x;
  const int q = blk % per;
  blk /= per;
  const int g = 1 + blk % (G - 1), bh = blk / (G - 1);
  const int rb0 = q * rpc, rb1 = min(nrb, rb0 + rpc);
  const size_t seg0 = ((size_t)bh * G + g) * Tg;  // first global row of the segment
  const int tid = threadIdx.x, lane = tid & 31, col0 = (tid >> 5) * 32;
  auto load_r = [&](int rb, int buf) {
#pragma unroll
    for (int u = 0; u < RV; ++u) {
      const int i = tid + u * NT, r = i / (DK / 8), c8 = (i % (DK / 8)) * 8;
      const int t = rb * 64 + r;
      const bool in = t < Tg;  // rows past the segment read as zero
      cp_async16(Rs + (buf * 64 + r) * RP + c8, R + (seg0 + (in ? t : 0)) * DK + c8, in ? 16 : 0);
    }
    cp_async_commit();
  };
  if (rb0 < rb1) load_r(rb0, 0);
  // B fragments: Sin[g][k][n] for n = col0 + 8 nt + lane / 4, k = 16 kt + 2 (lane % 4) + {0, 1, 8, 9}
  uint32_t bf[KT][4][2];
  {
    const float* Sg = Sin + ((size_t)bh * G + g) * DK * DV + col0 + lane / 4;
    const int kl = 2 * (lane % 4);
#pragma unroll
    for (int kt = 0; kt < KT; ++kt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const float* p = Sg + (size_t)(16 * kt + kl) * DV + 8 * nt;
        bf[kt][nt][0] = pack2_bf16(p[0], p[DV]);
        bf[kt][nt][1] = pack2_bf16(p[8 * DV], p[9 * DV]);
      }
  }
  const int lr = lane / 4, lc = 2 * (lane % 4);  // accumulator row / column of this lane
  for (int rb = rb0; rb < rb1; ++rb) {
    const int buf = (rb - rb0) & 1;
    // this block's output values, in the accumulator layout (in flight over the products)
    uint32_t ov[4][4][2];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = rb * 64 + 16 * mt + lr + 8 * h;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(o + (seg0 + t) * DV + col0 + lc);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) ov[mt][nt][h] = t < Tg ? src[4 * nt] : 0u;
      }
    if (rb + 1 < rb1) {
      load_r(rb + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // this R block is in place
    float acc[4][4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
    const __nv_bfloat16* Rb = Rs + (buf * 64 + (lane % 16)) * RP + (lane / 16) * 8;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt)
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t af[4];
        ldmatrix_x4(af, Rb + 16 * mt * RP + 16 * kt);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_16816(acc[mt][nt], af, bf[kt][nt]);
      }
    __syncthreads();  // every warp is done with Rs[buf]; the next prefetch may refill it
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = rb * 64 + 16 * mt + lr + 8 * h;
        if (t >= Tg) continue;
        uint32_t* dst = reinterpret_cast<uint32_t*>(o + (seg0 + t) * DV + col0 + lc);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const uint32_t w = ov[mt][nt][h];
          const float x0 = __uint_as_float(w << 16) + acc[mt][nt][2 * h];
          const float x1 = __uint_as_float(w & 0xFFFF0000u) + acc[mt][nt][2 * h + 1];
          dst[4 * nt] = pack2_bf16(x0, x1);
        }
      }
  }
}

template <int DK, int NC>
cudaError_t combine_t(const float* Send, const float* A, float* Sin, float* S_out, int BH, int G, int Dv,
                      cudaStream_t st) {
  constexpr int CS = NC == 16 ? 24 : 8;
  const size_t smem = (size_t)(2 * DK * (DK + 4) + 2 * DK * CS + (DK / 16) * (NC / 8) * 128) * sizeof(float);
  auto kern = seg_combine_kernel<DK, NC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(BH * (Dv / NC)), 4 * DK, smem, st>>>(Send, A, Sin, S_out, G, Dv);
  return cudaGetLastError();
}

int sm_count_dev() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n;
}

template <int DK, int DV>
cudaError_t correct_t(void* o, const void* R, const float* Sin, int BH, int G, int Tg, cudaStream_t st) {
  const size_t smem = (size_t)2 * 64 * (DK + 8) * 2;
  auto kern = seg_correct_kernel<DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, DV, smem);
  if (e != cudaSuccess) return e;
  // one wave: each (b, h, segment) gets slots / (B H (G - 1)) CTAs (at least
  // one), each a run of consecutive 64-row blocks
  const long long segs = (long long)BH * (G - 1);
  const int nrb = (Tg + 63) / 64;
  const long long slots = (long long)std::max(occ, 1) * sm_count_dev();
  const long long per_seg = std::max(1LL, std::min<long long>(nrb, slots / segs));
  const int rpc = (int)((nrb + per_seg - 1) / per_seg);
  const long long blocks = segs * ((nrb + rpc - 1) / rpc);
  if (blocks > INT_MAX) return cudaErrorInvalidValue;
  kern<<<(unsigned)blocks, DV, smem, st>>>(static_cast<__nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(R),
                                           Sin, G, Tg, rpc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_seg_combine(const float* Send, const float* A, float* Sin, float* S_out, int BH, int G,
                               int Dk, int Dv, cudaStream_t st) {
  if (G < 2 || Dv % 16 != 0) return cudaErrorInvalidValue;
  // The steps are sequential, so every CTA of one call should be resident at
  // once: 8-column slices (twice the CTAs, half the work per step) while they fit one wave.
  const bool narrow = (long long)BH * (Dv / 8) <= sm_count_dev();
  if (Dk == 128)
    return narrow ? combine_t<128, 8>(Send, A, Sin, S_out, BH, G, Dv, st)
                  : combine_t<128, 16>(Send, A, Sin, S_out, BH, G, Dv, st);
  if (Dk == 64)
    return narrow ? combine_t<64, 8>(Send, A, Sin, S_out, BH, G, Dv, st)
                  : combine_t<64, 16>(Send, A, Sin, S_out, BH, G, Dv, st);
  return cudaErrorNotSupported;
}

cudaError_t launch_seg_correct(void* o, const void* R, const float* Sin, int BH, int G, int Tg, int Dk, int Dv,
                               cudaStream_t st) {
  if (G < 2 || Tg < 1) return cudaErrorInvalidValue;
  if (Dk == 128 && Dv == 128) return correct_t<128, 128>(o, R, Sin, BH, G, Tg, st);
  if (Dk == 128 && Dv == 64) return correct_t<128, 64>(o, R, Sin, BH, G, Tg, st);
  if (Dk == 64 && Dv == 128) return correct_t<64, 128>(o, R, Sin, BH, G, Tg, st);
  if (Dk == 64 && Dv == 64) return correct_t<64, 64>(o, R, Sin, BH, G, Tg, st);
  return cudaErrorNotSupported;
}

}  // namespace dn
