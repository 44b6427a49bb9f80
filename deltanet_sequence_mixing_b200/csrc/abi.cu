// C ABI of the library (declared in include/deltanet.h): host-side argument
// validation, workspace layout and kernel dispatch.  Every check runs before
// the first CUDA call, so a rejected call launches nothing.
#include <stdint.h>
#include <string.h>

#include <climits>

#include "deltanet.h"
#include "kernels.h"

namespace {

constexpr size_t kStatusBytes = 256;  // status word + padding (keeps 256-byte alignment)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};
Range range_of(const void* p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return Range{a, a + bytes};
}
bool overlap(const Range& a, const Range& b) {
  if (a.lo == a.hi || b.lo == b.hi || a.lo == 0 || b.lo == 0) return false;
  return a.lo < b.hi && b.lo < a.hi;
}

bool valid_dim(int d) { return d == 64 || d == 128; }

int map_cuda(cudaError_t e) {
  if (e == cudaSuccess) return DN_OK;
  if (e == cudaErrorNotSupported) return DN_ERR_UNSUPPORTED;
  return DN_ERR_CUDA;
}

// Shared validation of the chunked calls.  Returns DN_OK or an error.
int validate_chunked(const dn::ChunkProblem& p, size_t ws_bytes, const void* ws) {
  if (p.B < 0 || p.H < 0 || p.T < 0) return DN_ERR_INVALID_ARG;
  if (p.bf16 != 0 && p.bf16 != 1) return DN_ERR_INVALID_ARG;
  if (!valid_dim(p.Dk) || !valid_dim(p.Dv)) return DN_ERR_UNSUPPORTED;
  if (p.C != 64 && p.C != 128) return DN_ERR_UNSUPPORTED;
  if ((long long)p.B * p.H > INT_MAX) return DN_ERR_UNSUPPORTED;
  // With T == 0 no token buffer is ever dereferenced (empty tensors may carry a
  // null data pointer); otherwise every token buffer is required.
  if (p.T > 0) {
    if (!p.q || !p.k || !p.v || !p.o) return DN_ERR_INVALID_ARG;
    if (p.mode == dn::Mode::Delta && !p.beta) return DN_ERR_INVALID_ARG;
  }
  if (!ws) return DN_ERR_WORKSPACE;
  if (ws_bytes < deltanet_workspace_bytes(p.B, p.H, p.T, p.Dk, p.Dv, p.C,
                                          p.bf16 ? DN_BF16 : DN_F32))
    return DN_ERR_WORKSPACE;
  if (!aligned16(p.q) || !aligned16(p.k) || !aligned16(p.v) || !aligned16(p.o))
    return DN_ERR_ALIGNMENT;
  if ((p.S0 && !aligned16(p.S0)) || (p.S_out && !aligned16(p.S_out)) ||
      (p.z0 && !aligned16(p.z0)) || (p.z_out && !aligned16(p.z_out)) || !aligned16(ws))
    return DN_ERR_ALIGNMENT;

  const size_t es = p.bf16 ? 2 : 4;
  const size_t BH = (size_t)p.B * p.H, T = (size_t)p.T;
  const Range q = range_of(p.q, BH * T * p.Dk * es), k = range_of(p.k, BH * T * p.Dk * es);
  const Range v = range_of(p.v, BH * T * p.Dv * es), o = range_of(p.o, BH * T * p.Dv * es);
  const Range beta = range_of(p.beta, p.beta ? BH * T * 4 : 0);
  const Range alpha = range_of(p.alpha, p.alpha ? BH * T * 4 : 0);
  const Range S0 = range_of(p.S0, p.S0 ? BH * p.Dk * p.Dv * 4 : 0);
  const Range So = range_of(p.S_out, p.S_out ? BH * p.Dk * p.Dv * 4 : 0);
  const Range z0 = range_of(p.z0, p.z0 ? BH * p.Dk * 4 : 0);
  const Range zo = range_of(p.z_out, p.z_out ? BH * p.Dk * 4 : 0);
  const Range w = range_of(ws, ws_bytes);
  const Range inputs[] = {q, k, v, beta, alpha, S0, z0};
  // o overlaps nothing; S_out / z_out overlap nothing except exactly S0 / z0.
  for (const Range& r : inputs) {
    if (overlap(o, r)) return DN_ERR_INVALID_ARG;
    if (overlap(So, r) && !(r.lo == S0.lo && So.lo == S0.lo && So.hi == S0.hi))
      return DN_ERR_INVALID_ARG;
    if (overlap(zo, r) && !(r.lo == z0.lo && zo.lo == z0.lo && zo.hi == z0.hi))
      return DN_ERR_INVALID_ARG;
    if (overlap(w, r)) return DN_ERR_INVALID_ARG;
  }
  if (overlap(o, So) || overlap(o, zo) || overlap(So, zo) || overlap(w, o) || overlap(w, So) ||
      overlap(w, zo))
    return DN_ERR_INVALID_ARG;
  return DN_OK;
}

int run_chunked(dn::ChunkProblem& p, void* ws, void* stream) {
  if ((size_t)p.B * p.H == 0) return DN_OK;  // nothing to compute
  p.status = static_cast<unsigned int*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dn::chunk_main_supported(p) || dn::chunk128_supported(p)) {
    const dn::WyWorkspace w =
        dn::wy_carve(static_cast<uint8_t*>(ws) + kStatusBytes, p.B, p.H, p.T, p.C);
    return map_cuda(p.C == 64 ? dn::launch_chunk_main(p, w, st) : dn::launch_chunk128(p, w, st));
  }
  if (dn::linear_tc_supported(p)) return map_cuda(dn::launch_linear_tc(p, st));
  if (dn::chunk_simt_supported(p.Dk, p.Dv, p.C)) return map_cuda(dn::launch_chunk_simt(p, st));
  return DN_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

size_t deltanet_workspace_bytes(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt) {
  if (B < 0 || H < 0 || T < 0 || !valid_dim(Dk) || !valid_dim(Dv)) return 0;
  if ((C != 64 && C != 128) || (dt != DN_F32 && dt != DN_BF16)) return 0;
  // bf16: room for the per-chunk WY factors of the pre-pass
  if (dt == DN_BF16 && T > 0) return kStatusBytes + dn::wy_workspace_bytes(B, H, T, C);
  return kStatusBytes;
}

int deltanet_workspace_init(void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (!workspace || ws_bytes < kStatusBytes) return DN_ERR_WORKSPACE;
  return map_cuda(
      cudaMemsetAsync(workspace, 0, kStatusBytes, static_cast<cudaStream_t>(cuda_stream)));
}

int deltanet_chunk_fwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* alpha, const float* S0, void* o, float* S_out, int B, int H,
                       int T, int Dk, int Dv, int C, dn_dtype dt, void* workspace,
                       size_t ws_bytes, void* cuda_stream) {
  if (dt != DN_F32 && dt != DN_BF16) return DN_ERR_UNSUPPORTED;
  dn::ChunkProblem p{};
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.alpha = alpha; p.S0 = S0;
  p.o = o; p.S_out = S_out;
  p.B = B; p.H = H; p.T = T; p.Dk = Dk; p.Dv = Dv; p.C = C;
  p.bf16 = dt == DN_BF16;
  p.mode = dn::Mode::Delta;
  const int rc = validate_chunked(p, ws_bytes, workspace);
  if (rc != DN_OK) return rc;
  return run_chunked(p, workspace, cuda_stream);
}

int linear_attn_fwd(const void* q, const void* k, const void* v, const float* S0,
                    const float* z0, void* o, float* S_out, float* z_out, int B, int H, int T,
                    int Dk, int Dv, int C, dn_dtype dt, void* workspace, size_t ws_bytes,
                    void* cuda_stream) {
  if (dt != DN_F32 && dt != DN_BF16) return DN_ERR_UNSUPPORTED;
  dn::ChunkProblem p{};
  p.q = q; p.k = k; p.v = v; p.S0 = S0; p.z0 = z0;
  p.o = o; p.S_out = S_out; p.z_out = z_out;
  p.B = B; p.H = H; p.T = T; p.Dk = Dk; p.Dv = Dv; p.C = C;
  p.bf16 = dt == DN_BF16;
  p.mode = dn::Mode::Linear;
  const int rc = validate_chunked(p, ws_bytes, workspace);
  if (rc != DN_OK) return rc;
  return run_chunked(p, workspace, cuda_stream);
}

int deltanet_decode_step(const void* q, const void* k, const void* v, const float* beta,
                         const float* alpha, float* S, void* o, int B, int H, int Dk, int Dv,
                         dn_dtype dt, void* cuda_stream) {
  if (dt != DN_F32 && dt != DN_BF16) return DN_ERR_UNSUPPORTED;
  if (B < 0 || H < 0) return DN_ERR_INVALID_ARG;
  if (!valid_dim(Dk) || !valid_dim(Dv)) return DN_ERR_UNSUPPORTED;
  if ((long long)B * H > INT_MAX) return DN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !beta || !S || !o) return DN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(S))
    return DN_ERR_ALIGNMENT;
  const size_t es = dt == DN_BF16 ? 2 : 4, BH = (size_t)B * H;
  const Range rs = range_of(S, BH * Dk * Dv * 4), ro = range_of(o, BH * Dv * es);
  const Range ins[] = {range_of(q, BH * Dk * es), range_of(k, BH * Dk * es),
                       range_of(v, BH * Dv * es), range_of(beta, BH * 4),
                       range_of(alpha, alpha ? BH * 4 : 0)};
  for (const Range& r : ins)
    if (overlap(rs, r) || overlap(ro, r)) return DN_ERR_INVALID_ARG;
  if (overlap(rs, ro)) return DN_ERR_INVALID_ARG;
  if (BH == 0) return DN_OK;
  dn::DecodeProblem p{q, k, v, beta, alpha, S, o, B, H, Dk, Dv, dt == DN_BF16};
  return map_cuda(dn::launch_decode(p, static_cast<cudaStream_t>(cuda_stream)));
}

int deltanet_get_device_status(const void* workspace, void* cuda_stream) {
  if (!workspace) return DN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  unsigned int word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return DN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DN_ERR_CUDA;
  if (word == 0) return DN_OK;
  if (word & dn::kStatusTimeoutBit) return DN_ERR_DEVICE_TIMEOUT;
  return DN_ERR_CUDA;
}

int deltanet_selftest_wait_timeout(void* workspace, size_t ws_bytes, long long wait_ns,
                                   void* cuda_stream) {
  if (!workspace || ws_bytes < kStatusBytes) return DN_ERR_WORKSPACE;
  if (wait_ns <= 0 || wait_ns > 2000000000LL) return DN_ERR_INVALID_ARG;
  return map_cuda(dn::launch_wait_selftest(static_cast<unsigned int*>(workspace), wait_ns,
                                           static_cast<cudaStream_t>(cuda_stream)));
}

const char* deltanet_status_string(int status) {
  switch (status) {
    case DN_OK: return "ok";
    case DN_ERR_INVALID_ARG: return "invalid argument";
    case DN_ERR_UNSUPPORTED: return "unsupported shape, chunk size or dtype";
    case DN_ERR_ALIGNMENT: return "buffer not 16-byte aligned";
    case DN_ERR_CUDA: return "CUDA error";
    case DN_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
    case DN_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int deltanet_version(void) { return 100; }

}  // extern "C"
