// C ABI of the library (declared in include/deltanet.h): host-side argument
// validation, workspace layout and kernel dispatch.  Every check runs before
// the first CUDA call, so a rejected call launches nothing.
#include <stdint.h>
#include <string.h>

#include <climits>
#include <mutex>

#include "deltanet.h"
#include "kernels.h"

namespace {

constexpr size_t kStatusBytes = 256;  // status word + padding (keeps 256-byte alignment)
constexpr unsigned int kKnownOptions = DN_OPT_PRESTEP | DN_OPT_GATE_PER_DIM | DN_OPT_SEQ_SPLIT;

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

// Shape and presence checks shared by the chunked calls.
int validate_problem(const dn::ChunkProblem& p) {
  if (p.B < 0 || p.H < 0 || p.T < 0) return DN_ERR_INVALID_ARG;
  if (p.bf16 != 0 && p.bf16 != 1) return DN_ERR_INVALID_ARG;
  if (!valid_dim(p.Dk) || !valid_dim(p.Dv)) return DN_ERR_UNSUPPORTED;
  if (p.C != 64 && p.C != 128) return DN_ERR_UNSUPPORTED;
  // C = 128 is built for the bf16 delta rule only, without the options
  if (p.C == 128 && (!p.bf16 || p.mode != dn::Mode::Delta || p.prestep || p.alpha_per_dim))
    return DN_ERR_UNSUPPORTED;
  if (p.alpha_per_dim && !p.alpha && p.T > 0) return DN_ERR_INVALID_ARG;
  if ((long long)p.B * p.H > INT_MAX) return DN_ERR_UNSUPPORTED;
  // the chunk kernels run one CTA per (b, h, 64-column slice of Dv) on a
  // one-dimensional grid, the pre-pass one CTA per (b, h, chunk)
  if ((long long)p.B * p.H * ((p.Dv + 63) / 64) > INT_MAX) return DN_ERR_UNSUPPORTED;
  if ((long long)p.B * p.H * ((p.T + (long long)p.C - 1) / p.C) > INT_MAX) return DN_ERR_UNSUPPORTED;
  // With T == 0 no token buffer is ever dereferenced (empty tensors may carry a
  // null data pointer); otherwise every token buffer is required.
  if (p.T > 0) {
    if (!p.q || !p.k || !p.v || !p.o) return DN_ERR_INVALID_ARG;
    if (p.mode == dn::Mode::Delta && !p.beta) return DN_ERR_INVALID_ARG;
  }
  return DN_OK;
}

// Overlap rules of the chunked calls: o overlaps nothing, S_out / z_out only
// exactly S0 / z0, and the workspace none of the caller's buffers.
int validate_overlaps(const dn::ChunkProblem& p, const void* ws, size_t ws_bytes) {
  const size_t es = p.bf16 ? 2 : 4;
  const size_t BH = (size_t)p.B * p.H, T = (size_t)p.T;
  const Range q = range_of(p.q, BH * T * p.Dk * es), k = range_of(p.k, BH * T * p.Dk * es);
  const Range v = range_of(p.v, BH * T * p.Dv * es), o = range_of(p.o, BH * T * p.Dv * es);
  const Range beta = range_of(p.beta, p.beta ? BH * T * 4 : 0);
  const Range alpha = range_of(p.alpha, p.alpha ? BH * T * 4 * (p.alpha_per_dim ? p.Dk : 1) : 0);
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

// Full validation of a chunked call on device buffers.  Returns DN_OK or an error.
int validate_chunked(const dn::ChunkProblem& p, size_t ws_bytes, const void* ws,
                     unsigned int options = 0) {
  int rc = validate_problem(p);
  if (rc != DN_OK) return rc;
  if (!ws) return DN_ERR_WORKSPACE;
  if (ws_bytes < deltanet_workspace_bytes_ex(p.B, p.H, p.T, p.Dk, p.Dv, p.C,
                                             p.bf16 ? DN_BF16 : DN_F32, options))
    return DN_ERR_WORKSPACE;
  if (!aligned16(p.q) || !aligned16(p.k) || !aligned16(p.v) || !aligned16(p.o))
    return DN_ERR_ALIGNMENT;
  if ((p.S0 && !aligned16(p.S0)) || (p.S_out && !aligned16(p.S_out)) ||
      (p.z0 && !aligned16(p.z0)) || (p.z_out && !aligned16(p.z_out)) || !aligned16(ws))
    return DN_ERR_ALIGNMENT;
  return validate_overlaps(p, ws, ws_bytes);
}

// Launch the kernels of a validated chunked problem; `status` is the device
// status word, `wy` the start of the pre-pass factor region.
// Problems the tcgen05 chunk kernels take: the plain and scalar-gated delta rule
// on bf16 inputs, with the layer's pre-step at C = 64; the per-dimension gate
// (and float32 inputs) run on the CUDA-core kernel (C = 64).
bool tensor_core_path(const dn::ChunkProblem& p) {
  if (p.alpha_per_dim) return false;
  return dn::chunk_main_supported(p) || (!p.prestep && dn::chunk128_supported(p));
}

int run_chunked_at(dn::ChunkProblem& p, unsigned int* status, void* wy, cudaStream_t st) {
  if ((size_t)p.B * p.H == 0) return DN_OK;  // nothing to compute
  p.status = status;
  if (p.T == 0) {  // no tokens: the final state (and normaliser) is the initial one
    const size_t BH = (size_t)p.B * p.H;
    auto carry = [&](float* dst, const float* src, size_t bytes) {
      if (!dst || dst == src) return cudaSuccess;
      return src ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st)
                 : cudaMemsetAsync(dst, 0, bytes, st);
    };
    cudaError_t e = carry(p.S_out, p.S0, BH * p.Dk * p.Dv * sizeof(float));
    if (e == cudaSuccess && p.mode == dn::Mode::Linear) e = carry(p.z_out, p.z0, BH * p.Dk * sizeof(float));
    return map_cuda(e);
  }
  if (tensor_core_path(p)) {
    const dn::WyWorkspace w = dn::wy_carve(wy, p.B, p.H, p.T, p.C, p.Dk);
    return map_cuda(p.C == 64 ? dn::launch_chunk_main(p, w, st) : dn::launch_chunk128(p, w, st));
  }
  if (dn::linear_tc_supported(p)) return map_cuda(dn::launch_linear_tc(p, st));
  if (dn::chunk_simt_supported(p.Dk, p.Dv, p.C)) return map_cuda(dn::launch_chunk_simt(p, st));
  return DN_ERR_UNSUPPORTED;
}

int run_chunked(dn::ChunkProblem& p, void* ws, void* stream) {
  return run_chunked_at(p, static_cast<unsigned int*>(ws), static_cast<uint8_t*>(ws) + kStatusBytes,
                        static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------ host buffers --
// The host-buffer call streams the heads through the device in kHostGroups
// groups, two staging slots in the workspace, on three library streams.
constexpr int kHostGroups = 4;

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

int host_group_heads(long long BH) { return (int)((BH + kHostGroups - 1) / kHostGroups); }

struct HostSlot {  // byte offsets inside one staging slot
  size_t q, k, v, o, beta, alpha, S0, S_out, wy, bytes;
};

HostSlot host_slot(int Hg, int T, int Dk, int Dv, int C, bool bf16) {
  const size_t es = bf16 ? 2 : 4, tok = (size_t)Hg * T, st = (size_t)Hg * Dk * Dv * 4;
  HostSlot L{};
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t at = off;
    off += round256(n);
    return at;
  };
  L.q = take(tok * Dk * es);
  L.k = take(tok * Dk * es);
  L.v = take(tok * Dv * es);
  L.o = take(tok * Dv * es);
  L.beta = take(tok * 4);
  L.alpha = take(tok * 4);
  L.S0 = take(st);
  L.S_out = take(st);
  L.wy = take(bf16 && T > 0 ? dn::wy_workspace_bytes(1, Hg, T, C) : 0);
  L.bytes = off;
  return L;
}

// Streams and events of the host-buffer call, created once per device.
struct HostQueues {
  bool ready = false;
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t loaded[2] = {}, computed[2] = {}, drained[2] = {};
};
constexpr int kMaxDevices = 64;
HostQueues g_host_queues[kMaxDevices];
std::mutex g_host_mutex;  // held while a call creates or enqueues on them

cudaError_t host_queues(int dev, HostQueues** out) {
  HostQueues& h = g_host_queues[dev];
  if (!h.ready) {
    cudaError_t e = cudaSuccess;
    for (cudaStream_t* s : {&h.h2d, &h.comp, &h.d2h})
      if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
    cudaEvent_t* evs[] = {&h.start, &h.end, &h.loaded[0], &h.loaded[1], &h.computed[0],
                          &h.computed[1], &h.drained[0], &h.drained[1]};
    for (cudaEvent_t* ev : evs)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    h.ready = true;
  }
  *out = &h;
  return cudaSuccess;
}

// ----------------------------------------------------------- sequence split --
// DN_OPT_SEQ_SPLIT: the sequence reshaped to (B*H*G, T/G) runs through the
// pre-pass once; the forward from the segments' entry states (S0 for segment
// 0, zero for the rest) and the homogeneous chain of every segment then run
// side by side on two streams, and two small kernels join the segments.
constexpr int kMinSegChunks = 8;       // 64-token chunks per segment, at least
constexpr int kMaxSegments = 16;
// The segment count minimises an estimate of the critical path in units of one
// chunk of the chain (about 1.35 us on the B200): the chunks of one segment,
// plus the sequential join (one step per segment boundary, about 2.7 us, two
// chunks), plus the fixed cost of the split (the homogeneous chain's start,
// the join's launches and the output correction, about eight chunks).
constexpr int kJoinStepChunks = 2;
constexpr int kSplitFixedChunks = 8;

int sm_count_now() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

int seq_segments_for(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt, unsigned int options, int sms) {
  // the split runs the tcgen05 path: bf16, C = 64, optionally with the layer's pre-step
  if ((options & ~DN_OPT_PRESTEP) != DN_OPT_SEQ_SPLIT || dt != DN_BF16 || C != 64 || T <= 0) return 1;
  if (!valid_dim(Dk) || !valid_dim(Dv) || B < 1 || H < 1 || sms < 1) return 1;
  int best = 1;
  long long best_cost = (T + 63) / 64;  // the plain call
  for (int G = 2; G <= kMaxSegments; ++G) {
    const int chunks = (T / G + 63) / 64;
    if (T % G != 0 || chunks < kMinSegChunks) continue;
    // both chunk kernels of pass 1 at once, one wave: 64-column slices of Dv and of Dk
    if ((long long)B * H * G * (Dv / 64 + Dk / 64) > sms) continue;
    const long long cost = chunks + (long long)kJoinStepChunks * (G - 1) + kSplitFixedChunks;
    if (cost < best_cost) {
      best = G;
      best_cost = cost;
    }
  }
  return best;
}

int seq_segments(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt, unsigned int options) {
  return seq_segments_for(B, H, T, Dk, Dv, C, dt, options, sm_count_now());
}

struct SplitLayout {  // byte offsets inside the workspace
  size_t wy, R, S0seg, Send, A, Sin, bytes;
};

SplitLayout split_layout(int B, int H, int T, int Dk, int Dv, int G, bool prestep) {
  const size_t BH = (size_t)B * H, BHG = BH * G;
  SplitLayout L{};
  size_t off = kStatusBytes;
  auto take = [&](size_t n) {
    const size_t at = off;
    off += (n + 255) / 256 * 256;
    return at;
  };
  // the pre-pass factors (and, with the pre-step, the mapped k and q after them)
  const size_t wy = dn::wy_workspace_bytes(1, (int)BHG, T / G, 64);
  L.wy = take(prestep ? (wy + 255) / 256 * 256 + dn::wy_khat_bytes(1, (int)BHG, T / G, Dk) : wy);
  L.R = take(BH * T * Dk * 2);
  L.S0seg = take(BHG * Dk * Dv * 4);
  L.Send = take(BHG * Dk * Dv * 4);
  L.A = take(BHG * Dk * Dk * 4);
  L.Sin = take(BHG * Dk * Dv * 4);
  L.bytes = off;
  return L;
}

// The second stream and its events, created once per device.
struct SplitQueues {
  bool ready = false;
  cudaStream_t side = nullptr;
  cudaEvent_t prepass = nullptr, hom = nullptr;
};
SplitQueues g_split_queues[64];
std::mutex g_split_mutex;  // held while a call creates or enqueues on them

int run_split(dn::ChunkProblem& p, int G, void* ws, cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_split_mutex);
  SplitQueues& q = g_split_queues[dev];
  cudaError_t e = cudaSuccess;
  if (!q.ready) {
    e = cudaStreamCreateWithFlags(&q.side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q.prepass, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q.hom, cudaEventDisableTiming);
    if (e != cudaSuccess) return map_cuda(e);
    q.ready = true;
  }
  const SplitLayout L = split_layout(p.B, p.H, p.T, p.Dk, p.Dv, G, p.prestep);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int BH = p.B * p.H, Tg = p.T / G;
  const size_t blk = (size_t)p.Dk * p.Dv * sizeof(float);
  float* S0seg = reinterpret_cast<float*>(base + L.S0seg);
  float* Send = reinterpret_cast<float*>(base + L.Send);
  float* A = reinterpret_cast<float*>(base + L.A);
  float* Sin = reinterpret_cast<float*>(base + L.Sin);
  void* R = base + L.R;
  // entry states of pass 1: S0 for segment 0 of every head, zero for the others
  e = cudaMemsetAsync(S0seg, 0, (size_t)BH * G * blk, st);
  if (e == cudaSuccess && p.S0)
    e = cudaMemcpy2DAsync(S0seg, G * blk, p.S0, blk, blk, BH, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return map_cuda(e);
  // the sequence as (B*H*G, T/G): a view of the same contiguous tensors
  dn::ChunkProblem p1 = p;
  p1.B = BH * G;
  p1.H = 1;
  p1.T = Tg;
  p1.S0 = S0seg;
  p1.S_out = Send;
  p1.status = static_cast<unsigned int*>(ws);
  const dn::WyWorkspace w = dn::wy_carve(base + L.wy, p1.B, 1, Tg, 64, p.Dk);
  e = dn::launch_tsolve(p1, w, st);
  if (e == cudaSuccess) e = cudaEventRecord(q.prepass, st);
  // the homogeneous chains on the side stream, once the factors are in place
  dn::ChunkProblem p2 = p1;
  p2.hom = 1;
  p2.v = p1.k;  // mapped, never read
  p2.Dv = p.Dk;
  p2.o = R;
  p2.S0 = nullptr;
  p2.S_out = A;
  if (e == cudaSuccess) e = cudaStreamWaitEvent(q.side, q.prepass, 0);
  if (e == cudaSuccess) e = dn::launch_chunk_main_only(p2, w, q.side, 64, false);
  if (e == cudaSuccess) e = cudaEventRecord(q.hom, q.side);
  // the forward beside it
  if (e == cudaSuccess) e = dn::launch_chunk_main_only(p1, w, st, 64, false);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, q.hom, 0);
  // join: the entry state of every segment and S_out, then the outputs
  if (e == cudaSuccess) e = dn::launch_seg_combine(Send, A, Sin, p.S_out, BH, G, p.Dk, p.Dv, st);
  if (e == cudaSuccess) e = dn::launch_seg_correct(p.o, R, Sin, BH, G, Tg, p.Dk, p.Dv, st);
  return map_cuda(e);
}

}  // namespace

extern "C" {

int deltanet_seq_segments(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt, unsigned int options) {
  return seq_segments(B, H, T, Dk, Dv, C, dt, options);
}

int deltanet_seq_segments_sm(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt, unsigned int options,
                             int sm_count) {
  return seq_segments_for(B, H, T, Dk, Dv, C, dt, options, sm_count);
}

size_t deltanet_workspace_bytes_ex(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                                   unsigned int options) {
  if (options & ~kKnownOptions) return 0;
  if (options & DN_OPT_SEQ_SPLIT) {
    const size_t plain = deltanet_workspace_bytes_ex(B, H, T, Dk, Dv, C, dt, options & ~DN_OPT_SEQ_SPLIT);
    const int G = seq_segments(B, H, T, Dk, Dv, C, dt, options);
    if (plain == 0 || G == 1) return plain;
    const size_t split = split_layout(B, H, T, Dk, Dv, G, (options & DN_OPT_PRESTEP) != 0).bytes;
    return split > plain ? split : plain;
  }
  if (options == 0) return deltanet_workspace_bytes(B, H, T, Dk, Dv, C, dt);
  if (C != 64 || deltanet_workspace_bytes(B, H, T, Dk, Dv, C, dt) == 0) return 0;
  // the pre-step alone runs on the tcgen05 path for bf16 (the per-chunk factors
  // of the pre-pass); the per-dimension gate runs on the CUDA-core kernel
  // (status word only)
  if (options == DN_OPT_PRESTEP) {
    if (dt != DN_BF16 || T == 0) return kStatusBytes;  // the CUDA-core kernel
    const size_t wy = dn::wy_workspace_bytes(B, H, T, C);
    return kStatusBytes + (wy + 255) / 256 * 256 + dn::wy_khat_bytes(B, H, T, Dk);  // + mapped k and q
  }
  return kStatusBytes;
}

size_t deltanet_workspace_bytes(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt) {
  if (B < 0 || H < 0 || T < 0 || !valid_dim(Dk) || !valid_dim(Dv)) return 0;
  if ((C != 64 && C != 128) || (dt != DN_F32 && dt != DN_BF16)) return 0;
  if (C == 128 && dt != DN_BF16) return 0;  // C = 128 is built for bf16 only
  if ((long long)B * H * (((long long)T + C - 1) / C) > INT_MAX) return 0;
  // bf16: room for the per-chunk WY factors of the pre-pass
  if (dt == DN_BF16 && T > 0) return kStatusBytes + dn::wy_workspace_bytes(B, H, T, C);
  return kStatusBytes;
}

int deltanet_workspace_init(void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (!workspace || ws_bytes < kStatusBytes) return DN_ERR_WORKSPACE;
  return map_cuda(
      cudaMemsetAsync(workspace, 0, kStatusBytes, static_cast<cudaStream_t>(cuda_stream)));
}

int deltanet_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* beta,
                          const float* alpha, const float* S0, void* o, float* S_out, int B, int H,
                          int T, int Dk, int Dv, int C, dn_dtype dt, unsigned int options,
                          void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (dt != DN_F32 && dt != DN_BF16) return DN_ERR_UNSUPPORTED;
  if (options & ~kKnownOptions) return DN_ERR_INVALID_ARG;
  dn::ChunkProblem p{};
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.alpha = alpha; p.S0 = S0;
  p.o = o; p.S_out = S_out;
  p.B = B; p.H = H; p.T = T; p.Dk = Dk; p.Dv = Dv; p.C = C;
  p.bf16 = dt == DN_BF16;
  p.mode = dn::Mode::Delta;
  p.prestep = (options & DN_OPT_PRESTEP) != 0;
  p.alpha_per_dim = (options & DN_OPT_GATE_PER_DIM) != 0;
  const int rc = validate_chunked(p, ws_bytes, workspace, options);
  if (rc != DN_OK) return rc;
  const int G = seq_segments(B, H, T, Dk, Dv, C, dt, options);
  if (G > 1) return run_split(p, G, workspace, static_cast<cudaStream_t>(cuda_stream));
  return run_chunked(p, workspace, cuda_stream);
}

int deltanet_chunk_fwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* alpha, const float* S0, void* o, float* S_out, int B, int H,
                       int T, int Dk, int Dv, int C, dn_dtype dt, void* workspace,
                       size_t ws_bytes, void* cuda_stream) {
  return deltanet_chunk_fwd_ex(q, k, v, beta, alpha, S0, o, S_out, B, H, T, Dk, Dv, C, dt, 0u,
                               workspace, ws_bytes, cuda_stream);
}

size_t deltanet_host_workspace_bytes(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt) {
  if (deltanet_workspace_bytes(B, H, T, Dk, Dv, C, dt) == 0) return 0;
  const long long BH = (long long)B * H;
  if (BH > INT_MAX) return 0;
  return kStatusBytes + 2 * host_slot(host_group_heads(BH), T, Dk, Dv, C, dt == DN_BF16).bytes;
}

int deltanet_chunk_fwd_host(const void* q, const void* k, const void* v, const float* beta,
                            const float* alpha, const float* S0, void* o, float* S_out, int B,
                            int H, int T, int Dk, int Dv, int C, dn_dtype dt, void* workspace,
                            size_t ws_bytes, void* cuda_stream) {
  if (dt != DN_F32 && dt != DN_BF16) return DN_ERR_UNSUPPORTED;
  dn::ChunkProblem p{};
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.alpha = alpha; p.S0 = S0;
  p.o = o; p.S_out = S_out;
  p.B = B; p.H = H; p.T = T; p.Dk = Dk; p.Dv = Dv; p.C = C;
  p.bf16 = dt == DN_BF16;
  p.mode = dn::Mode::Delta;
  int rc = validate_problem(p);
  if (rc != DN_OK) return rc;
  if (!workspace) return DN_ERR_WORKSPACE;
  if (ws_bytes < deltanet_host_workspace_bytes(B, H, T, Dk, Dv, C, dt)) return DN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DN_ERR_ALIGNMENT;
  rc = validate_overlaps(p, workspace, ws_bytes);
  if (rc != DN_OK) return rc;
  const long long BH = (long long)B * H;
  if (BH == 0) return DN_OK;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return DN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_host_mutex);
  HostQueues* hq = nullptr;
  if (host_queues(dev, &hq) != cudaSuccess) return DN_ERR_CUDA;

  const int Hg = host_group_heads(BH);
  const HostSlot L = host_slot(Hg, T, Dk, Dv, C, p.bf16 != 0);
  const size_t es = p.bf16 ? 2 : 4;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  unsigned int* status = reinterpret_cast<unsigned int*>(ws);
  cudaStream_t cs = static_cast<cudaStream_t>(cuda_stream);
  auto ok = [&](cudaError_t r) { return (e = (e == cudaSuccess ? r : e)) == cudaSuccess; };
  auto h2d = [&](void* dst, const void* src, size_t n) {
    return n == 0 || ok(cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, hq->h2d));
  };
  auto d2h = [&](void* dst, const void* src, size_t n) {
    return n == 0 || ok(cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, hq->d2h));
  };
  // everything already queued on the caller's stream comes first
  ok(cudaEventRecord(hq->start, cs));
  for (cudaStream_t s : {hq->h2d, hq->comp, hq->d2h}) ok(cudaStreamWaitEvent(s, hq->start, 0));
  int launch_rc = DN_OK;
  for (long long h0 = 0, g = 0; h0 < BH && e == cudaSuccess && launch_rc == DN_OK; h0 += Hg, ++g) {
    const int hn = (int)(BH - h0 < Hg ? BH - h0 : Hg), sl = (int)(g & 1);
    uint8_t* slot = ws + kStatusBytes + sl * L.bytes;
    const size_t tok = (size_t)hn * T, t0 = (size_t)h0 * T;
    const size_t st = (size_t)hn * Dk * Dv * 4, s0 = (size_t)h0 * Dk * Dv * 4;
    // 1. inputs of group g into slot g % 2, once group g - 2 has left it
    ok(cudaStreamWaitEvent(hq->h2d, hq->drained[sl], 0));
    if (T > 0) {  // with T == 0 the token buffers may be null
      h2d(slot + L.q, static_cast<const uint8_t*>(q) + t0 * Dk * es, tok * Dk * es);
      h2d(slot + L.k, static_cast<const uint8_t*>(k) + t0 * Dk * es, tok * Dk * es);
      h2d(slot + L.v, static_cast<const uint8_t*>(v) + t0 * Dv * es, tok * Dv * es);
      if (beta) h2d(slot + L.beta, beta + t0, tok * 4);
      if (alpha) h2d(slot + L.alpha, alpha + t0, tok * 4);
    }
    if (S0) h2d(slot + L.S0, reinterpret_cast<const uint8_t*>(S0) + s0, st);
    ok(cudaEventRecord(hq->loaded[sl], hq->h2d));
    // 2. the group's chunked forward on the compute stream
    ok(cudaStreamWaitEvent(hq->comp, hq->loaded[sl], 0));
    if (e != cudaSuccess) break;
    dn::ChunkProblem pg = p;
    pg.q = slot + L.q; pg.k = slot + L.k; pg.v = slot + L.v; pg.o = slot + L.o;
    pg.beta = beta ? reinterpret_cast<const float*>(slot + L.beta) : nullptr;
    pg.alpha = alpha ? reinterpret_cast<const float*>(slot + L.alpha) : nullptr;
    pg.S0 = S0 ? reinterpret_cast<const float*>(slot + L.S0) : nullptr;
    pg.S_out = S_out ? reinterpret_cast<float*>(slot + L.S_out) : nullptr;
    pg.B = 1;
    pg.H = hn;
    launch_rc = run_chunked_at(pg, status, slot + L.wy, hq->comp);
    ok(cudaEventRecord(hq->computed[sl], hq->comp));
    // 3. outputs of group g back to the host
    ok(cudaStreamWaitEvent(hq->d2h, hq->computed[sl], 0));
    if (T > 0) d2h(static_cast<uint8_t*>(o) + t0 * Dv * es, slot + L.o, tok * Dv * es);
    if (S_out) d2h(reinterpret_cast<uint8_t*>(S_out) + s0, slot + L.S_out, st);
    ok(cudaEventRecord(hq->drained[sl], hq->d2h));
  }
  // the caller's stream continues once the last group is back on the host
  // (also after a failed launch, so that nothing queued here outlives the call
  // on the caller's stream)
  ok(cudaEventRecord(hq->end, hq->d2h));
  ok(cudaStreamWaitEvent(cs, hq->end, 0));
  return launch_rc != DN_OK ? launch_rc : map_cuda(e);
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
  return deltanet_decode_step_ex(q, k, v, beta, alpha, S, o, B, H, Dk, Dv, dt, 0u, cuda_stream);
}

int deltanet_decode_step_ex(const void* q, const void* k, const void* v, const float* beta,
                            const float* alpha, float* S, void* o, int B, int H, int Dk, int Dv,
                            dn_dtype dt, unsigned int options, void* cuda_stream) {
  if (dt != DN_F32 && dt != DN_BF16) return DN_ERR_UNSUPPORTED;
  if (options & ~kKnownOptions) return DN_ERR_INVALID_ARG;
  const bool per_dim = (options & DN_OPT_GATE_PER_DIM) != 0;
  if (per_dim && !alpha) return DN_ERR_INVALID_ARG;
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
                       range_of(alpha, alpha ? BH * 4 * (per_dim ? Dk : 1) : 0)};
  for (const Range& r : ins)
    if (overlap(rs, r) || overlap(ro, r)) return DN_ERR_INVALID_ARG;
  if (overlap(rs, ro)) return DN_ERR_INVALID_ARG;
  if (BH == 0) return DN_OK;
  dn::DecodeProblem p{q, k, v, beta, alpha, S, o, B, H, Dk, Dv, dt == DN_BF16,
                      (options & DN_OPT_PRESTEP) != 0, per_dim};
  return map_cuda(dn::launch_decode(p, static_cast<cudaStream_t>(cuda_stream)));
}

size_t deltanet_chunk_bwd_workspace_bytes(int B, int H, int T, int Dk, int Dv, dn_dtype dt) {
  if (B < 0 || H < 0 || T < 0 || !valid_dim(Dk) || !valid_dim(Dv)) return 0;
  if (dt != DN_F32 && dt != DN_BF16) return 0;
  if ((long long)B * H > INT_MAX) return 0;
  return kStatusBytes + dn::chunk_bwd_state_bytes(B, H, T, Dk, Dv);
}

int deltanet_chunk_bwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* alpha, const float* S0, const void* dO, const float* dS_T,
                       float* dq, float* dk, float* dv, float* dbeta, float* dlog_alpha, float* dS0,
                       int B, int H, int T, int Dk, int Dv, dn_dtype dt, void* workspace,
                       size_t ws_bytes, void* cuda_stream) {
  if (dt != DN_F32 && dt != DN_BF16) return DN_ERR_UNSUPPORTED;
  if (B < 0 || H < 0 || T < 0) return DN_ERR_INVALID_ARG;
  if (!valid_dim(Dk) || !valid_dim(Dv)) return DN_ERR_UNSUPPORTED;
  if ((long long)B * H > INT_MAX) return DN_ERR_UNSUPPORTED;
  if (T > 0 && (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta))
    return DN_ERR_INVALID_ARG;
  if (dlog_alpha && !alpha) return DN_ERR_INVALID_ARG;
  if (!workspace) return DN_ERR_WORKSPACE;
  if (ws_bytes < deltanet_chunk_bwd_workspace_bytes(B, H, T, Dk, Dv, dt)) return DN_ERR_WORKSPACE;
  const void* f32s[] = {beta, alpha, S0, dS_T, dq, dk, dv, dbeta, dlog_alpha, dS0, workspace};
  for (const void* x : f32s)
    if (x && (reinterpret_cast<uintptr_t>(x) & 3u)) return DN_ERR_ALIGNMENT;
  if (!aligned16(workspace)) return DN_ERR_ALIGNMENT;
  const size_t es = dt == DN_BF16 ? 2 : 4, BH = (size_t)B * H, TT = (size_t)T;
  const Range ins[] = {range_of(q, BH * TT * Dk * es), range_of(k, BH * TT * Dk * es),
                       range_of(v, BH * TT * Dv * es), range_of(beta, BH * TT * 4),
                       range_of(alpha, alpha ? BH * TT * 4 : 0), range_of(S0, S0 ? BH * Dk * Dv * 4 : 0),
                       range_of(dO, BH * TT * Dv * es), range_of(dS_T, dS_T ? BH * Dk * Dv * 4 : 0)};
  const Range outs[] = {range_of(dq, BH * TT * Dk * 4), range_of(dk, BH * TT * Dk * 4),
                        range_of(dv, BH * TT * Dv * 4), range_of(dbeta, BH * TT * 4),
                        range_of(dlog_alpha, dlog_alpha ? BH * TT * 4 : 0),
                        range_of(dS0, dS0 ? BH * Dk * Dv * 4 : 0), range_of(workspace, ws_bytes)};
  for (size_t a = 0; a < sizeof outs / sizeof outs[0]; ++a) {
    for (const Range& r : ins)
      if (overlap(outs[a], r)) return DN_ERR_INVALID_ARG;
    for (size_t b = a + 1; b < sizeof outs / sizeof outs[0]; ++b)
      if (overlap(outs[a], outs[b])) return DN_ERR_INVALID_ARG;
  }
  if (BH == 0) return DN_OK;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (T == 0) {  // no tokens: dL/dS0 is dL/dS_T
    if (!dS0) return DN_OK;
    const size_t nb = BH * Dk * Dv * 4;
    return map_cuda(dS_T ? cudaMemcpyAsync(dS0, dS_T, nb, cudaMemcpyDeviceToDevice, st)
                         : cudaMemsetAsync(dS0, 0, nb, st));
  }
  dn::BwdProblem p{};
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.alpha = alpha; p.S0 = S0; p.dO = dO; p.dS_T = dS_T;
  p.dq = dq; p.dk = dk; p.dv = dv; p.dbeta = dbeta; p.dlog_alpha = dlog_alpha; p.dS0 = dS0;
  p.states = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kStatusBytes);
  p.B = B; p.H = H; p.T = T; p.Dk = Dk; p.Dv = Dv;
  p.bf16 = dt == DN_BF16;
  return map_cuda(dn::launch_chunk_bwd(p, st));
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
