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
#include <mma.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

using namespace nvcuda;

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

constexpr int kCombCols = 16;  // Dv columns per combine CTA

// One CTA per (b, h, 16-column slice of Dv), 2 DK threads (thread: one row of
// the slice, 8 columns): the G - 1 sequential steps S <- A[g] S + Send[g] in
// float32.  A[g + 1] streams into shared memory while step g computes.
template <int DK>
__global__ void __launch_bounds__(2 * DK) seg_combine_kernel(const float* __restrict__ Send,
                                                              const float* __restrict__ A, float* __restrict__ Sin,
                                                              float* __restrict__ S_out, int G, int Dv) {
  constexpr int NT = 2 * DK;  // threads
  constexpr int AP = DK + 4;  // padded row of A (16-byte aligned, two wavefronts per warp read)
  extern __shared__ __align__(16) float seg_smem[];
  float* As = seg_smem;           // 2 x DK x AP
  float* cur = As + 2 * DK * AP;  // DK x 16, the state entering the next segment
  const int nsl = Dv / kCombCols;
  const int bh = blockIdx.x / nsl, j0 = (blockIdx.x % nsl) * kCombCols;
  const int tid = threadIdx.x, row = tid >> 1, cg = (tid & 1) * 8;
  const size_t sblk = (size_t)DK * Dv, ablk = (size_t)DK * DK;
  auto load_a = [&](int g, int buf) {
    const float* src = A + ((size_t)bh * G + g) * ablk;
    for (int i = tid; i < DK * DK / 4; i += NT) {
      const int r = (4 * i) / DK, c = (4 * i) % DK;
      cp_async16(As + buf * DK * AP + r * AP + c, src + 4 * i, 16);
    }
    cp_async_commit();
  };
  load_a(1, 0);
  // Sin[1] = Send[0]
  {
    const size_t at = (size_t)row * Dv + j0 + cg;
    const float4 x0 = *reinterpret_cast<const float4*>(Send + (size_t)bh * G * sblk + at);
    const float4 x1 = *reinterpret_cast<const float4*>(Send + (size_t)bh * G * sblk + at + 4);
    *reinterpret_cast<float4*>(cur + row * kCombCols + cg) = x0;
    *reinterpret_cast<float4*>(cur + row * kCombCols + cg + 4) = x1;
    float* d = Sin + ((size_t)bh * G + 1) * sblk + at;
    *reinterpret_cast<float4*>(d) = x0;
    *reinterpret_cast<float4*>(d + 4) = x1;
  }
  for (int g = 1; g < G; ++g) {
    const int buf = (g - 1) & 1;
    if (g + 1 < G) {
      load_a(g + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // A[g] and cur are complete
    const size_t at = (size_t)row * Dv + j0 + cg;
    const float* Sg = Send + ((size_t)bh * G + g) * sblk + at;
    const float4 s0 = *reinterpret_cast<const float4*>(Sg);
    const float4 s1 = *reinterpret_cast<const float4*>(Sg + 4);
    float acc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    const float* Ar = As + buf * DK * AP + row * AP;
#pragma unroll 4
    for (int k4 = 0; k4 < DK; k4 += 4) {
      const float4 a4 = *reinterpret_cast<const float4*>(Ar + k4);
      const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const float4 b0 = *reinterpret_cast<const float4*>(cur + (k4 + kk) * kCombCols + cg);
        const float4 b1 = *reinterpret_cast<const float4*>(cur + (k4 + kk) * kCombCols + cg + 4);
        acc[0] = fmaf(a[kk], b0.x, acc[0]); acc[1] = fmaf(a[kk], b0.y, acc[1]);
        acc[2] = fmaf(a[kk], b0.z, acc[2]); acc[3] = fmaf(a[kk], b0.w, acc[3]);
        acc[4] = fmaf(a[kk], b1.x, acc[4]); acc[5] = fmaf(a[kk], b1.y, acc[5]);
        acc[6] = fmaf(a[kk], b1.z, acc[6]); acc[7] = fmaf(a[kk], b1.w, acc[7]);
      }
    }
    __syncthreads();  // every thread has read cur and As[buf]
    const float4 r0 = make_float4(acc[0], acc[1], acc[2], acc[3]);
    const float4 r1 = make_float4(acc[4], acc[5], acc[6], acc[7]);
    *reinterpret_cast<float4*>(cur + row * kCombCols + cg) = r0;
    *reinterpret_cast<float4*>(cur + row * kCombCols + cg + 4) = r1;
    // the next segment's entry state, or the final state (S_out may be NULL)
    float* dst = g + 1 < G ? Sin + ((size_t)bh * G + g + 1) * sblk : (S_out ? S_out + (size_t)bh * sblk : nullptr);
    if (dst) {
      *reinterpret_cast<float4*>(dst + at) = r0;
      *reinterpret_cast<float4*>(dst + at + 4) = r1;
    }
  }
}

// One CTA per (b, h, segment g >= 1, run of `rpc` 64-row blocks): O[rows] +=
// R[rows] Sin[g] over the full Dv, bf16 tensor-core products (WMMA, float32
// accumulation) with Sin[g] rounded to bf16 once per CTA.  The next R block
// streams in (cp.async, two buffers) and the block's output rows are loaded
// into registers while the products run; then one read-modify-write of the
// bf16 output rows.
template <int DK, int DV>
__global__ void __launch_bounds__(256, 2) seg_correct_kernel(__nv_bfloat16* __restrict__ o,
                                                             const __nv_bfloat16* __restrict__ R,
                                                             const float* __restrict__ Sin, int G, int Tg, int rpc) {
  constexpr int RP = DK + 8;            // padded bf16 row of an R block
  constexpr int SP = DV + 8;            // padded bf16 row of Sin[g]
  constexpr int CP = DV + 4;            // padded float row of the product
  constexpr int NTW = DV / 32;          // 16-column tiles per warp (two warps per 16 rows)
  constexpr int RV = 64 * DK / 8 / 256; // 16-byte pieces of an R block per thread
  constexpr int OV = 64 * DV / 8 / 256; // 16-byte pieces of an output block per thread
  extern __shared__ __align__(128) unsigned char seg_smem_c[];
  __nv_bfloat16* Ss = reinterpret_cast<__nv_bfloat16*>(seg_smem_c);  // DK x SP
  __nv_bfloat16* Rs = Ss + DK * SP;                                    // 2 x 64 x RP
  float* Cs = reinterpret_cast<float*>(Rs + 2 * 64 * RP);              // 64 x CP
  const int nrb = (Tg + 63) / 64, per = (nrb + rpc - 1) / rpc;
  int blk = blockIdx.x;
  const int q = blk % per;
  blk /= per;
  const int g = 1 + blk % (G - 1), bh = blk / (G - 1);
  const int rb0 = q * rpc, rb1 = min(nrb, rb0 + rpc);
  const size_t seg0 = ((size_t)bh * G + g) * Tg;  // first global row of the segment
  const int tid = threadIdx.x, warp = tid >> 5;
  auto load_r = [&](int rb, int buf) {
#pragma unroll
    for (int u = 0; u < RV; ++u) {
      const int i = tid + u * 256, r = i / (DK / 8), c8 = (i % (DK / 8)) * 8;
      const int t = rb * 64 + r;
      const bool in = t < Tg;  // rows past the segment read as zero
      cp_async16(Rs + (buf * 64 + r) * RP + c8, R + (seg0 + (in ? t : 0)) * DK + c8, in ? 16 : 0);
    }
    cp_async_commit();
  };
  if (rb0 < rb1) load_r(rb0, 0);
  const float* Sg = Sin + ((size_t)bh * G + g) * DK * DV;
  for (int i = tid; i < DK * DV / 4; i += 256) {
    const float4 x = reinterpret_cast<const float4*>(Sg)[i];
    const int r = (4 * i) / DV, c = (4 * i) % DV;
    uint2 u;
    u.x = pack2_bf16(x.x, x.y);
    u.y = pack2_bf16(x.z, x.w);
    *reinterpret_cast<uint2*>(Ss + r * SP + c) = u;
  }
  using FragA = wmma::fragment<wmma::matrix_a, 16, 16, 16, __nv_bfloat16, wmma::row_major>;
  using FragB = wmma::fragment<wmma::matrix_b, 16, 16, 16, __nv_bfloat16, wmma::row_major>;
  using FragC = wmma::fragment<wmma::accumulator, 16, 16, 16, float>;
  const int wr = 16 * (warp & 3), wc = (DV / 2) * (warp >> 2);
  for (int rb = rb0; rb < rb1; ++rb) {
    const int buf = (rb - rb0) & 1;
    uint4 ov[OV];
#pragma unroll
    for (int u = 0; u < OV; ++u) {
      const int i = tid + u * 256, r = i / (DV / 8), c8 = (i % (DV / 8)) * 8;
      const int t = rb * 64 + r;
      ov[u] = t < Tg ? *reinterpret_cast<const uint4*>(o + (seg0 + t) * DV + c8) : make_uint4(0, 0, 0, 0);
    }
    if (rb + 1 < rb1) {
      load_r(rb + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // this R block (and Sin[g]) are in place; Cs is free
    FragC acc[NTW];
#pragma unroll
    for (int n = 0; n < NTW; ++n) wmma::fill_fragment(acc[n], 0.f);
#pragma unroll
    for (int kk = 0; kk < DK; kk += 16) {
      FragA fa;
      wmma::load_matrix_sync(fa, Rs + (buf * 64 + wr) * RP + kk, RP);
#pragma unroll
      for (int n = 0; n < NTW; ++n) {
        FragB fb;
        wmma::load_matrix_sync(fb, Ss + kk * SP + wc + 16 * n, SP);
        wmma::mma_sync(acc[n], fa, fb, acc[n]);
      }
    }
#pragma unroll
    for (int n = 0; n < NTW; ++n) wmma::store_matrix_sync(Cs + wr * CP + wc + 16 * n, acc[n], CP, wmma::mem_row_major);
    __syncthreads();  // the product is complete; Rs[buf] may be refilled
#pragma unroll
    for (int u = 0; u < OV; ++u) {
      const int i = tid + u * 256, r = i / (DV / 8), c8 = (i % (DV / 8)) * 8;
      const int t = rb * 64 + r;
      if (t >= Tg) continue;
      float x[8];
      unpack_bf16x8(ov[u], x);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] += Cs[r * CP + c8 + e];
      st_bf16x8(o + (seg0 + t) * DV + c8, x);
    }
  }
}

template <int DK>
cudaError_t combine_t(const float* Send, const float* A, float* Sin, float* S_out, int BH, int G, int Dv,
                      cudaStream_t st) {
  const size_t smem = (size_t)(2 * DK * (DK + 4) + DK * kCombCols) * sizeof(float);
  auto kern = seg_combine_kernel<DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(BH * (Dv / kCombCols)), 2 * DK, smem, st>>>(Send, A, Sin, S_out, G, Dv);
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
  const size_t smem = (size_t)DK * (DV + 8) * 2 + (size_t)2 * 64 * (DK + 8) * 2 + (size_t)64 * (DV + 4) * 4;
  auto kern = seg_correct_kernel<DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // one wave of two CTAs per SM: each (b, h, segment) gets slots / (B H (G - 1))
  // CTAs (at least one), each a run of consecutive 64-row blocks
  const long long segs = (long long)BH * (G - 1);
  const int nrb = (Tg + 63) / 64;
  const long long per_seg = std::max(1LL, std::min<long long>(nrb, 2LL * sm_count_dev() / segs));
  const int rpc = (int)((nrb + per_seg - 1) / per_seg);
  const long long blocks = segs * ((nrb + rpc - 1) / rpc);
  if (blocks > INT_MAX) return cudaErrorInvalidValue;
  kern<<<(unsigned)blocks, 256, smem, st>>>(static_cast<__nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(R),
                                            Sin, G, Tg, rpc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_seg_combine(const float* Send, const float* A, float* Sin, float* S_out, int BH, int G,
                               int Dk, int Dv, cudaStream_t st) {
  if (G < 2 || Dv % kCombCols != 0) return cudaErrorInvalidValue;
  if (Dk == 128) return combine_t<128>(Send, A, Sin, S_out, BH, G, Dv, st);
  if (Dk == 64) return combine_t<64>(Send, A, Sin, S_out, BH, G, Dv, st);
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
