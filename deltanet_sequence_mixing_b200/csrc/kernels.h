// Internal launcher declarations shared by the ABI layer and the kernel files.
// Not part of the public interface (that is include/deltanet.h).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dn {

// Bits of the device status word kept in the first bytes of the workspace.
// Kernels only ever set bits; the host clears the word.
constexpr unsigned int kStatusTimeoutBit = 1u;  // a bounded wait ran out

enum class Mode : int { Delta = 0, Linear = 1 };

// Problem description passed from the ABI layer to the launchers.  All pointers
// are device pointers that the ABI layer has validated.
struct ChunkProblem {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;   // Delta only
  const float* alpha;  // Delta only, nullable
  const float* S0;     // nullable
  const float* z0;     // Linear only, nullable
  void* o;
  float* S_out;        // nullable
  float* z_out;        // Linear only, nullable
  int B, H, T, Dk, Dv, C;
  int bf16;            // 1: q/k/v/o are bfloat16, 0: float32
  Mode mode;
  int prestep;         // Delta only: q, k raw and beta logits (silu + L2 normalise, sigmoid inside)
  int alpha_per_dim;   // Delta only: alpha is (B,H,T,Dk), one decay per key dimension
  unsigned int* status;  // device status word (workspace)
  // Delta, tcgen05 C = 64 only: the homogeneous chain (v taken as zero, S0 as the
  // identity, Dv == Dk): o receives the rows of R = (diag(gamma) Q - P W) S and
  // S_out the product of the chunk transitions.  v must still point at a
  // (B,H,T,Dv) bf16 tensor (it is mapped, never read).
  int hom;
};

// CUDA-core (float32 arithmetic) chunked kernel: both modes, both input types.
// Returns cudaErrorNotSupported for shapes it does not instantiate.
cudaError_t launch_chunk_simt(const ChunkProblem& p, cudaStream_t st);
bool chunk_simt_supported(int Dk, int Dv, int C);

// tcgen05 (bf16 operands, float32 accumulate) chunked ELU+1 linear attention.
cudaError_t launch_linear_tc(const ChunkProblem& p, cudaStream_t st);
bool linear_tc_supported(const ChunkProblem& p);

// Decode step (in-place state update).
struct DecodeProblem {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;
  const float* alpha;  // nullable
  float* S;
  void* o;
  int B, H, Dk, Dv;
  int bf16;
  int prestep;        // q, k raw and beta logits: silu + L2 normalise, sigmoid inside
  int alpha_per_dim;  // alpha is (B,H,Dk): one decay per key dimension
};
cudaError_t launch_decode(const DecodeProblem& p, cudaStream_t st);

// 3-D TMA map over a (BH, T, D) bf16 tensor: 64 x 64 boxes, 128-byte swizzle,
// rows past T read as zeros.
bool make_tmap_3d_bf16(CUtensorMap* m, const void* base, int D, int T, int BH);

// Per-chunk WY factors written by the pre-pass and read by the chunk kernels
// (C = 64 or 128 token chunks).
struct WyWorkspace {
  __nv_bfloat16* tb;   // [B*H][chunks][C][C]  T diag(beta)
  __nv_bfloat16* tbg;  // [B*H][chunks][C][C]  T diag(beta) diag(exp(g))   (gated)
  float* g;            // [B*H][chunks][C]     cumulative log decay        (gated)
  __nv_bfloat16* khat; // [B*H][T][Dk]          keys after the layer's pre-step (pre-step only)
  __nv_bfloat16* qhat; // [B*H][T][Dk]          queries after the layer's pre-step (pre-step only)
};
size_t wy_workspace_bytes(int B, int H, int T, int C);
// Bytes of the mapped keys and queries the pre-step adds after the factors
// (each region starts on a 256-byte boundary).
size_t wy_khat_bytes(int B, int H, int T, int Dk);
// Dk: head size of q and k, for the pre-step regions (any value when unused)
WyWorkspace wy_carve(void* base, int B, int H, int T, int C, int Dk);
cudaError_t launch_tsolve(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st);

// tcgen05 chunked delta rule after the pre-pass (bf16, C = 64).
bool chunk_main_supported(const ChunkProblem& p);
cudaError_t launch_chunk_main(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st);
// The chunk kernel alone, its factors already in `w`: `dvs` = 64 or 32 (the Dv
// slice width; 0 picks as launch_chunk_main does), `after_prepass` = launched
// as a programmatic dependent of a pre-pass just enqueued on `st`.
cudaError_t launch_chunk_main_only(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st, int dvs,
                                   bool after_prepass);

// The sequence split (segments run side by side, then combined; abi.cu):
//   combine: per (b, h), Sin[1] = Send[0], Sin[g+1] = A[g] Sin[g] + Send[g],
//            S_out = A[G-1] Sin[G-1] + Send[G-1]  (float32; G >= 2)
//   correct: o rows of segment g >= 1 += R rows of segment g  Sin[g]  (bf16 o, R)
cudaError_t launch_seg_combine(const float* Send, const float* A, float* Sin, float* S_out, int BH, int G,
                               int Dk, int Dv, cudaStream_t st);
cudaError_t launch_seg_correct(void* o, const void* R, const float* Sin, int BH, int G, int Tg, int Dk,
                               int Dv, cudaStream_t st);

// tcgen05 chunked delta rule after the pre-pass (bf16, C = 128).
bool chunk128_supported(const ChunkProblem& p);
cudaError_t launch_chunk128(const ChunkProblem& p, const WyWorkspace& w, cudaStream_t st);

// Gradient of the chunked delta rule (float32 arithmetic on CUDA cores).
struct BwdProblem {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;
  const float* alpha;   // nullable (ungated)
  const float* S0;      // nullable
  const void* dO;       // (B,H,T,Dv), element type of q
  const float* dS_T;    // nullable
  float* dq;            // (B,H,T,Dk)
  float* dk;
  float* dv;            // (B,H,T,Dv)
  float* dbeta;         // (B,H,T)
  float* dlog_alpha;    // (B,H,T), nullable
  float* dS0;           // (B,H,Dk,Dv), nullable
  float* states;        // workspace: entry state of every 32-token chunk
  int B, H, T, Dk, Dv;
  int bf16;
};
size_t chunk_bwd_state_bytes(int B, int H, int T, int Dk, int Dv);
cudaError_t launch_chunk_bwd(const BwdProblem& p, cudaStream_t st);

// Bounded-wait self test.
cudaError_t launch_wait_selftest(unsigned int* status, long long wait_ns, cudaStream_t st);

}  // namespace dn
