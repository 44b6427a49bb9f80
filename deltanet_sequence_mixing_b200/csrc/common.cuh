// Inline-PTX building blocks for the sm_100a kernels: mbarriers with bounded
// waits, TMA tile loads, tcgen05 (TMEM alloc, MMA, commit, load) and the
// shared-memory matrix descriptors of the 128-byte-swizzled operand layout.
// Written from the public PTX ISA description of these instructions.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kernels.h"

namespace dn {

// Default limit of every device-side wait: two seconds of global time.  A
// healthy kernel never comes near it; a wait that runs out records a timeout
// and the kernel winds down instead of spinning forever.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------ programmatic dependent launch --
// Block until the grids this one depends on (launched before it on the stream
// with programmatic serialisation) have completed and their writes are visible.
// A no-op for a normal launch.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the dependent grid begin launching (its CTAs still wait for this grid's
// completion before reading its results).
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-CTA wait control: a shared abort flag (set by the first thread that gives
// up, so the others stop waiting quickly), the global status word, and the
// time limit.
struct WaitCtl {
  volatile int* abort_flag;  // shared memory
  unsigned int* status;      // global, may be null
  unsigned long long limit_ns;
};

__device__ __forceinline__ void record_timeout(const WaitCtl& w) {
  *w.abort_flag = 1;
  if (w.status) atomicOr(w.status, kStatusTimeoutBit);
}

// Longest time one suspended poll may keep the thread asleep (the hardware
// wakes it as soon as the phase completes).
constexpr uint32_t kSuspendHintNs = 200000u;

// One poll that may suspend the thread until the phase completes or the hint
// runs out, so a waiting warp leaves its scheduler's issue slots to the warps
// that are working.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false if the
// limit ran out (the timeout is recorded) or another thread already gave up.
// kSuspend: poll with suspension (the default) or spin on plain polls.
template <bool kSuspend = true>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtl& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (kSuspend ? mbar_try_wait_suspend(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if (kSuspend || (it & 15u) == 0) {
      if (*w.abort_flag) return false;
      if (global_ns() - t0 > w.limit_ns) {
        record_timeout(w);
        return false;
      }
    }
  }
}

// -------------------------------------------------------------------- TMA --
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// Warm L2 with the cache line holding a global address.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}
// 3-D tiled load (no multicast) completing on `bar` with a byte count.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// 3-D tiled store of a shared-memory tile (rows past the tensor's extent are
// not written), tracked by the issuing thread's bulk-async group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed bulk groups still read their source.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every bulk group of this thread has completed (writes performed).
__device__ __forceinline__ void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Warm L2 with a 3-D tile (no shared-memory destination).
__device__ __forceinline__ void prefetch_l2_3d(const CUtensorMap* m, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05 --
// TMEM allocation: `ncols` columns (power of two >= 32), address written to smem.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] x B[smem], bf16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same MMA issued by one elected lane of a warp whose 32 lanes all execute
// the call with identical (warp-uniform) operands.  Keeping the issuing code
// warp-uniform lets the descriptors stay in uniform registers; issuing from a
// single divergent lane costs extra instructions per MMA.
__device__ __forceinline__ void mma_bf16_ss_elect(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred e, p; .reg .b32 x; elect.sync x|e, 0xffffffff; setp.ne.b32 p, %4, 0;"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] x B[smem] (the A operand in tensor memory: row m of A on
// TMEM lane m, 32-bit column c holding elements 2c (low half) and 2c + 1 (high
// half); one K = 16 step spans 8 columns), issued by one elected lane.  Only B
// is read from shared memory, which halves (N = 128) or thirds (N = 64) the
// shared-memory traffic of the product.
__device__ __forceinline__ void mma_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred e, p; .reg .b32 x; elect.sync x|e, 0xffffffff; setp.ne.b32 p, %4, 0;"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Commit from one elected lane of a warp-uniform issuer (see mma_bf16_ss_elect).
__device__ __forceinline__ void mma_commit_elect(uint32_t bar) {
  asm volatile(
      "{ .reg .pred e; .reg .b32 x; elect.sync x|e, 0xffffffff;"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0]; }" ::"r"(bar)
      : "memory");
}
// A value every lane of the warp holds, made visibly warp-uniform (lane 0's).
__device__ __forceinline__ uint32_t warp_uniform(uint32_t v) { return __shfl_sync(0xffffffffu, v, 0); }
// Arrive on `bar` once every previously issued MMA of this thread has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Warp-collective load of 32 lanes x 32 consecutive 32-bit columns: thread i of
// the warp receives lane (base lane + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Store 32 consecutive 32-bit columns of this thread's TMEM lane (the
// inverse of tmem_ld32); complete with tmem_wait_st before signalling.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Shared-memory matrix descriptor for the 128-byte-swizzle canonical layout
// (atoms of 8 rows x 128 bytes, 1024 bytes, 1024-byte aligned).
//   K-major operand : rows are M (or N), 128-byte rows hold 64 bf16 along K;
//                     sbo = byte distance between 8-row groups; lbo unused (1).
//   MN-major operand: rows are K, 128-byte rows hold 64 bf16 along M (or N);
//                     lbo = byte distance between 64-element M (N) blocks,
//                     sbo = byte distance between 8-row K groups.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // swizzle mode: 128-byte
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, f32 accumulator.
// a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                      // D format f32
         | (1u << 7)                    // A format bf16
         | (1u << 10)                   // B format bf16
         | ((a_mn ? 1u : 0u) << 15)     // A major
         | ((b_mn ? 1u : 0u) << 16)     // B major
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// Byte offset of the 16-byte chunk `c16` (0..7) of row `r` inside a
// 128-byte-swizzled tile whose 8-row groups are 1024 bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int c16) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c16 ^ (r & 7)) << 4));
}

// K-major and MN-major descriptors of 128-byte-swizzled bf16 tiles (8-row
// groups 1024 bytes apart).
__device__ __forceinline__ uint64_t desc_k(uint32_t addr) { return sw128_desc(addr, 16, 1024); }
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr, uint32_t lbo) {
  return sw128_desc(addr, lbo, 1024);
}

// The descriptor of the same layout `bytes` further on: the start address is
// the low 14-bit field (address / 16), and shared memory ends below 2^18 bytes,
// so the sum never carries into the next field.  Forming a product's
// descriptors once and stepping them keeps the issuing warp's instruction
// count per MMA low.
__device__ __forceinline__ uint64_t desc_step(uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); }

// Named barrier over `count` threads; the AND form returns true only if every
// participating thread passed true (a uniform decision for the whole group).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ bool named_bar_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred pi, po; setp.ne.u32 pi, %1, 0; bar.red.and.pred po, %2, %3, pi;"
      " selp.u32 %0, 1, 0, po; }"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}
// Store 8 floats as one 16-byte chunk of bf16 (shared or global address).
__device__ __forceinline__ void st_bf16x8(void* dst, const float* x) {
  uint4 u;
  u.x = pack2_bf16(x[0], x[1]);
  u.y = pack2_bf16(x[2], x[3]);
  u.z = pack2_bf16(x[4], x[5]);
  u.w = pack2_bf16(x[6], x[7]);
  *reinterpret_cast<uint4*>(dst) = u;
}

// ------------------------------------------------- the layer's pre-step --
// silu(x) = x sigmoid(x) = x (1 + tanh(x / 2)) / 2, with the hardware tanh
// approximation (one MUFU operation; relative error about 2^-11, below the
// bf16 rounding the mapped values then take on the tensor-core paths).
__device__ __forceinline__ float silu_f(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return 0.5f * x * (1.f + t);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* x) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// The DeltaNet layer's map x <- silu(x) / max(||silu(x)||_2, 1e-12) on one row
// of a K-major, 128-byte-swizzled bf16 tile in shared memory (DK columns in
// 64-column blocks `blk_stride` bytes apart), in place.  Two adjacent lanes
// share a row: lane parity `part` takes the 16-byte chunks [part * DK/16,
// (part + 1) * DK/16) and the two partial sums of squares are combined with
// one shuffle, so every kernel that maps the same row gets bit-identical bf16
// values (the sum is always (first half) + (second half)).  All 32 lanes of
// the warp must call it.  If `dst` is not null, the mapped chunks are also
// stored there (the row's first element at dst[0], row-major bf16).
template <int DK>
__device__ __forceinline__ void prestep_row_sw128(uint8_t* tile, uint32_t blk_stride, int row, int part,
                                                  __nv_bfloat16* dst = nullptr) {
  constexpr int NCH = DK / 16;  // 16-byte chunks per thread
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NCH; ++j) {
    const int cg = part * NCH + j, blk = cg >> 3, c16 = cg & 7;
    float x[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(tile + blk * blk_stride + sw128_off(row, c16)), x);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float y = silu_f(x[e]);
      ss = fmaf(y, y, ss);
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, ss, 1);
  const float tot = part == 0 ? ss + other : other + ss;
  const float inv = 1.f / fmaxf(sqrtf(tot), 1e-12f);
  // Rewrite in groups of four chunks, each group loaded whole before its
  // stores (a store may alias a later load as far as the compiler knows, so a
  // load issued after it waits for it).
#pragma unroll
  for (int j0 = 0; j0 < NCH; j0 += 4) {
    uint4 raw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cg = part * NCH + j0 + j;
      raw[j] = *reinterpret_cast<const uint4*>(tile + (cg >> 3) * blk_stride + sw128_off(row, cg & 7));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cg = part * NCH + j0 + j;
      float x[8];
      unpack_bf16x8(raw[j], x);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = silu_f(x[e]) * inv;
      uint4 m;
      m.x = pack2_bf16(x[0], x[1]);
      m.y = pack2_bf16(x[2], x[3]);
      m.z = pack2_bf16(x[4], x[5]);
      m.w = pack2_bf16(x[6], x[7]);
      *reinterpret_cast<uint4*>(tile + (cg >> 3) * blk_stride + sw128_off(row, cg & 7)) = m;
      if (dst) *reinterpret_cast<uint4*>(dst + cg * 8) = m;
    }
  }
}

}  // namespace dn
