// C-ABI entry points of libw4a16: host-side argument checks, the N-based
// dispatcher between the CUDA-core GEMV and the tcgen05 GEMM (for the plain
// product and its fused QKV form), the quantiser, packing and residual
// add + normalisation launches, and status mapping.  "PerfXLLM on Snapdragon 8 Gen2", section 3.3: prefill (tokens > 1)
// is a GEMM and decode (tokens = 1) a GEMV; few tokens make the GEMM
// memory-bound and many make it compute-bound, and each regime gets its own
// tiling.  Here each regime gets its own kernel.
#include "w4a16_internal.cuh"

namespace w4a16 {
// Largest N the dispatcher sends to the CUDA-core GEMV kernel; above it the
// tensor-core kernel runs.  Chosen from the measured N sweep on the fused QKV
// shape (M = 12288, K = 4096).
int gemv_max_n();
}

namespace {

using namespace w4a16;

constexpr int kMaxM = 1 << 24;
constexpr int kMaxK = 1 << 16;
constexpr int kMaxN = 1 << 20;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Whether the byte ranges [a, a + na) and [b, b + nb) share a byte (a null
// pointer or an empty range shares none).
bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || !na || !nb) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Byte sizes of the packed buffers of an M x K weight (group 128).
struct PackedBytes {
  size_t wq, scales, zeros;
};

PackedBytes packed_bytes(int M, int K) {
  const size_t mp = (size_t)ceil_div(M, kRowBlock) * kRowBlock;
  const size_t kg = (size_t)K / kGroup;
  return {mp * (size_t)K / 2, mp * kg * 2, mp * kg / 2};
}

// Whether the output range [y, y + ny) overlaps the packed weight.
bool overlaps_weight(const void* y, size_t ny, const void* wq, const void* sp, const void* zp,
                     const PackedBytes& pb) {
  return overlap(y, ny, wq, pb.wq) || overlap(y, ny, sp, pb.scales) || overlap(y, ny, zp, pb.zeros);
}

w4a16_status check_shape(int M, int K, int group) {
  if (M <= 0 || K <= 0) return W4A16_ERR_INVALID_ARG;
  if (group != kGroup || K % kGroup != 0) return W4A16_ERR_UNSUPPORTED;
  if (M > kMaxM || K > kMaxK) return W4A16_ERR_UNSUPPORTED;
  return W4A16_OK;
}

w4a16_status map_cuda(cudaError_t e) {
  if (e == cudaSuccess) return W4A16_OK;
  if (e == cudaErrorNotSupported) return W4A16_ERR_UNSUPPORTED;
  return W4A16_ERR_CUDA;
}

// Largest M at which two decode launches beat the tile kernel: up to 64 row
// blocks the tile kernel has too few tiles to fill the SMs (32 at M = 4096).
// Measured at N = 16: the 4096 x 4096 projection takes 12 us as two decode
// launches against 24 us on the tile kernel; the 12288 x 4096 one 22 us
// against 17 us.
constexpr int kTwoLaunchMaxM = 8192;

// The decode kernel up to one launch of tokens, or two launches on weights of
// at most kTwoLaunchMaxM rows; the tile kernel above.  with_ws: a workspace is
// available (it would open the split decode kernel, which is never the faster
// one: forced only).
int select_path_impl(int M, int K, int N, bool with_ws) {
  if (M <= 0 || K <= 0 || N <= 0 || K % kGroup) return -1;
  (void)with_ws;
  if (N <= gemv_max_n()) return W4A16_PATH_GEMV;
  if (N <= 2 * gemv_max_n() && M <= kTwoLaunchMaxM) return W4A16_PATH_GEMV;
  return W4A16_PATH_TC;
}

size_t workspace_for(int path, int M, int K, int N) {
  return path == W4A16_PATH_GEMV_TC ? gemv_tc_workspace_bytes(M, K, N) : 0;
}

// Checks shared by the plain and the workspace entry points, then the launch
// on the chosen path.  ws may be null (ws_bytes 0).
w4a16_status gemm_impl(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                       const uint16_t* X, uint16_t* Y, int M, int K, int N, int group, int path, void* ws,
                       size_t ws_bytes, unsigned flags, void* stream) {
  if (!wq_packed || !scales_packed || !zeros_packed || !X || !Y) return W4A16_ERR_INVALID_ARG;
  if (N <= 0 || path < W4A16_PATH_AUTO || path > W4A16_PATH_GEMV_TC) return W4A16_ERR_INVALID_ARG;
  if (flags & ~W4A16_FLAG_EARLY_WEIGHTS) return W4A16_ERR_INVALID_ARG;
  if (!ws && ws_bytes) return W4A16_ERR_INVALID_ARG;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (N > kMaxN) return W4A16_ERR_UNSUPPORTED;
  if (!aligned16(wq_packed) || !aligned16(scales_packed) || !aligned16(zeros_packed) ||
      !aligned16(X) || !aligned16(Y) || (ws && !aligned16(ws)))
    return W4A16_ERR_MISALIGNED;
  if (path == W4A16_PATH_AUTO) path = select_path_impl(M, K, N, ws != nullptr);
  if (path == W4A16_PATH_GEMV_TC && N > kGemvTcMaxTokens) return W4A16_ERR_UNSUPPORTED;
  const size_t need = workspace_for(path, M, K, N);
  if (need > ws_bytes) return W4A16_ERR_INVALID_ARG;
  {
    const PackedBytes pb = packed_bytes(M, K);
    const size_t ny = (size_t)N * M * 2, nx = (size_t)N * K * 2;
    if (overlap(Y, ny, X, nx) || overlaps_weight(Y, ny, wq_packed, scales_packed, zeros_packed, pb))
      return W4A16_ERR_INVALID_ARG;
    if (ws && (overlap(ws, ws_bytes, X, nx) || overlap(ws, ws_bytes, Y, ny) ||
               overlaps_weight(ws, ws_bytes, wq_packed, scales_packed, zeros_packed, pb)))
      return W4A16_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* wq = static_cast<const uint8_t*>(wq_packed);
  const uint16_t* sp = static_cast<const uint16_t*>(scales_packed);
  const uint8_t* zp = static_cast<const uint8_t*>(zeros_packed);
  cudaError_t e;
  if (path == W4A16_PATH_GEMV_TC)
    e = launch_gemv_tc(wq, sp, zp, X, Y, M, K, N, ws, (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0, s);
  else if (path == W4A16_PATH_TC)
    e = launch_gemm_tc(wq, sp, zp, X, Y, M, K, N, s);
  else
    e = launch_gemv(wq, sp, zp, X, Y, M, K, N, s, nullptr, (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0);
  return map_cuda(e);
}

w4a16_status gemm_qkv_impl(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                           const uint16_t* X, const uint16_t* bias, int Mq, int Mk, int Mv, int K, int N,
                           int group, uint16_t* Yq, uint16_t* Yk, uint16_t* Yv, void* ws, size_t ws_bytes,
                           unsigned flags, void* stream) {
  if (!wq_packed || !scales_packed || !zeros_packed || !X || !Yq || !Yk || !Yv) return W4A16_ERR_INVALID_ARG;
  if (Mq <= 0 || Mk <= 0 || Mv <= 0 || N <= 0) return W4A16_ERR_INVALID_ARG;
  if (flags & ~W4A16_FLAG_EARLY_WEIGHTS) return W4A16_ERR_INVALID_ARG;
  if (!ws && ws_bytes) return W4A16_ERR_INVALID_ARG;
  if ((long long)Mq + Mk + Mv > kMaxM) return W4A16_ERR_UNSUPPORTED;
  const int M = Mq + Mk + Mv;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (N > kMaxN) return W4A16_ERR_UNSUPPORTED;
  if (!aligned16(wq_packed) || !aligned16(scales_packed) || !aligned16(zeros_packed) || !aligned16(X) ||
      !aligned16(Yq) || !aligned16(Yk) || !aligned16(Yv) || (reinterpret_cast<uintptr_t>(bias) & 1u) ||
      (ws && !aligned16(ws)))
    return W4A16_ERR_MISALIGNED;
  const int path = select_path_impl(M, K, N, ws != nullptr);
  const size_t need = workspace_for(path, M, K, N);
  if (need > ws_bytes) return W4A16_ERR_INVALID_ARG;
  {
    const PackedBytes pb = packed_bytes(M, K);
    const void* outs[4] = {Yq, Yk, Yv, ws};
    const size_t out_n[4] = {(size_t)N * Mq * 2, (size_t)N * Mk * 2, (size_t)N * Mv * 2, ws ? ws_bytes : 0};
    for (int i = 0; i < 4; ++i) {
      if (overlap(outs[i], out_n[i], X, (size_t)N * K * 2) || overlap(outs[i], out_n[i], bias, (size_t)M * 2) ||
          overlaps_weight(outs[i], out_n[i], wq_packed, scales_packed, zeros_packed, pb))
        return W4A16_ERR_INVALID_ARG;
      for (int j = i + 1; j < 4; ++j)
        if (overlap(outs[i], out_n[i], outs[j], out_n[j])) return W4A16_ERR_INVALID_ARG;
    }
  }
  OutMap om = {};
  om.kind = kEpiQkv;
  om.y0 = Yq;
  om.y1 = Yk;
  om.y2 = Yv;
  om.end0 = Mq;
  om.end1 = Mq + Mk;
  om.bias = bias;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* wq = static_cast<const uint8_t*>(wq_packed);
  const uint16_t* sp = static_cast<const uint16_t*>(scales_packed);
  const uint8_t* zp = static_cast<const uint8_t*>(zeros_packed);
  cudaError_t e;
  if (path == W4A16_PATH_GEMV_TC)
    e = launch_gemv_tc(wq, sp, zp, X, nullptr, M, K, N, ws, (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0, s, &om);
  else if (path == W4A16_PATH_TC)
    e = launch_gemm_tc(wq, sp, zp, X, nullptr, M, K, N, s, &om);
  else
    e = launch_gemv(wq, sp, zp, X, nullptr, M, K, N, s, &om, (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0);
  return map_cuda(e);
}

}  // namespace

extern "C" {

const char* w4a16_status_string(int status) {
  switch (status) {
    case W4A16_OK: return "ok";
    case W4A16_ERR_INVALID_ARG: return "invalid argument";
    case W4A16_ERR_UNSUPPORTED: return "unsupported size or group";
    case W4A16_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case W4A16_ERR_CUDA: return "CUDA error";
    case W4A16_ERR_TIMEOUT: return "device wait timed out";
    case W4A16_ERR_BOUNDS: return "in-kernel index check failed (debug build)";
    default: return "unknown status";
  }
}

w4a16_status w4a16_packed_sizes(int M, int K, int group, size_t* wq_bytes,
                                size_t* scales_bytes, size_t* zeros_bytes) {
  if (!wq_bytes || !scales_bytes || !zeros_bytes) return W4A16_ERR_INVALID_ARG;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  const PackedBytes pb = packed_bytes(M, K);
  *wq_bytes = pb.wq;
  *scales_bytes = pb.scales;
  *zeros_bytes = pb.zeros;
  return W4A16_OK;
}

w4a16_status w4a16_quantize(const uint16_t* W, int M, int K, int group, uint8_t* q, uint16_t* scales,
                            uint8_t* zeros, void* stream) {
  if (!W || !q || !scales || !zeros) return W4A16_ERR_INVALID_ARG;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (!aligned16(W) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 1u))
    return W4A16_ERR_MISALIGNED;
  const size_t mk = (size_t)M * K, mg = (size_t)M * (K / kGroup);
  if (overlap(q, mk, W, mk * 2) || overlap(scales, mg * 2, W, mk * 2) || overlap(zeros, mg, W, mk * 2) ||
      overlap(q, mk, scales, mg * 2) || overlap(q, mk, zeros, mg) || overlap(scales, mg * 2, zeros, mg))
    return W4A16_ERR_INVALID_ARG;
  return map_cuda(launch_quantize(W, M, K, q, scales, zeros, static_cast<cudaStream_t>(stream)));
}

w4a16_status w4a16_add_rmsnorm(const uint16_t* h, const uint16_t* d, const uint16_t* gamma, float eps,
                               int N, int K, uint16_t* r_out, uint16_t* X, void* stream) {
  if (!h || !gamma || !X) return W4A16_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || !(eps >= 0.0f) || !(eps <= 3.4028234663852886e38f)) return W4A16_ERR_INVALID_ARG;
  if (K % 8 != 0 || K > kMaxNormK || N > kMaxN) return W4A16_ERR_UNSUPPORTED;
  if (!aligned16(h) || (d && !aligned16(d)) || !aligned16(gamma) || (r_out && !aligned16(r_out)) ||
      !aligned16(X))
    return W4A16_ERR_MISALIGNED;
  const size_t bytes = (size_t)N * K * 2;
  // r_out may be h or d itself; X shares no byte with the other rows' data.
  const size_t gbytes = (size_t)K * 2;
  if (overlap(X, bytes, h, bytes) || overlap(X, bytes, d, bytes) || overlap(X, bytes, r_out, bytes) ||
      overlap(X, bytes, gamma, gbytes))
    return W4A16_ERR_INVALID_ARG;
  if (r_out && ((r_out != h && overlap(r_out, bytes, h, bytes)) ||
                (r_out != d && overlap(r_out, bytes, d, bytes)) || overlap(r_out, bytes, gamma, gbytes)))
    return W4A16_ERR_INVALID_ARG;
  return map_cuda(launch_add_rmsnorm(h, d, gamma, eps, N, K, r_out, X, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

w4a16_status pack_impl(const uint8_t* q, const uint16_t* scales, const uint8_t* zeros, int M, int K, int group,
                       void* wq_packed, void* scales_packed, void* zeros_packed, void* stream, int mi) {
  if (!q || !scales || !zeros || !wq_packed || !scales_packed || !zeros_packed)
    return W4A16_ERR_INVALID_ARG;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (!aligned16(wq_packed) || !aligned16(scales_packed) || !aligned16(zeros_packed) ||
      (reinterpret_cast<uintptr_t>(scales) & 1u))
    return W4A16_ERR_MISALIGNED;
  {
    const PackedBytes pb = packed_bytes(M, K);
    const size_t mk = (size_t)M * K, mg = (size_t)M * (K / kGroup);
    const void* outs[3] = {wq_packed, scales_packed, zeros_packed};
    const size_t out_n[3] = {pb.wq, pb.scales, pb.zeros};
    for (int i = 0; i < 3; ++i) {
      if (overlap(outs[i], out_n[i], q, mk) || overlap(outs[i], out_n[i], scales, mg * 2) ||
          overlap(outs[i], out_n[i], zeros, mg))
        return W4A16_ERR_INVALID_ARG;
      for (int j = i + 1; j < 3; ++j)
        if (overlap(outs[i], out_n[i], outs[j], out_n[j])) return W4A16_ERR_INVALID_ARG;
    }
  }
  return map_cuda(launch_pack(q, scales, zeros, M, K, static_cast<uint8_t*>(wq_packed),
                              static_cast<uint16_t*>(scales_packed), static_cast<uint8_t*>(zeros_packed),
                              static_cast<cudaStream_t>(stream), mi));
}

w4a16_status gemm_gate_up_impl(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                               const uint16_t* X, uint16_t* H, int Mi, int K, int N, int group, int path,
                               void* ws, size_t ws_bytes, unsigned flags, void* stream) {
  if (!wq_packed || !scales_packed || !zeros_packed || !X || !H) return W4A16_ERR_INVALID_ARG;
  if (Mi <= 0 || N <= 0 || path < W4A16_PATH_AUTO || path > W4A16_PATH_GEMV_TC) return W4A16_ERR_INVALID_ARG;
  if (flags & ~W4A16_FLAG_EARLY_WEIGHTS) return W4A16_ERR_INVALID_ARG;
  if (!ws && ws_bytes) return W4A16_ERR_INVALID_ARG;
  if (Mi > kMaxM / 2) return W4A16_ERR_UNSUPPORTED;
  const int M = 2 * Mi;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (N > kMaxN) return W4A16_ERR_UNSUPPORTED;
  if (!aligned16(wq_packed) || !aligned16(scales_packed) || !aligned16(zeros_packed) || !aligned16(X) ||
      !aligned16(H) || (ws && !aligned16(ws)))
    return W4A16_ERR_MISALIGNED;
  if (path == W4A16_PATH_AUTO) path = select_path_impl(M, K, N, ws != nullptr);
  if (path == W4A16_PATH_GEMV_TC && N > kGemvTcMaxTokens) return W4A16_ERR_UNSUPPORTED;
  const size_t need = workspace_for(path, M, K, N);
  if (need > ws_bytes) return W4A16_ERR_INVALID_ARG;
  {
    const PackedBytes pb = packed_bytes(M, K);
    const size_t nh = (size_t)N * Mi * 2, nx = (size_t)N * K * 2;
    if (overlap(H, nh, X, nx) || overlaps_weight(H, nh, wq_packed, scales_packed, zeros_packed, pb))
      return W4A16_ERR_INVALID_ARG;
    if (ws && (overlap(ws, ws_bytes, X, nx) || overlap(ws, ws_bytes, H, nh) ||
               overlaps_weight(ws, ws_bytes, wq_packed, scales_packed, zeros_packed, pb)))
      return W4A16_ERR_INVALID_ARG;
  }
  OutMap om = {};
  om.kind = kEpiGateUp;
  om.h = H;
  om.mi = Mi;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* wq = static_cast<const uint8_t*>(wq_packed);
  const uint16_t* sp = static_cast<const uint16_t*>(scales_packed);
  const uint8_t* zp = static_cast<const uint8_t*>(zeros_packed);
  cudaError_t e;
  if (path == W4A16_PATH_GEMV_TC)
    e = launch_gemv_tc(wq, sp, zp, X, nullptr, M, K, N, ws, (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0, s, &om);
  else if (path == W4A16_PATH_TC)
    e = launch_gemm_tc(wq, sp, zp, X, nullptr, M, K, N, s, &om);
  else
    e = launch_gemv(wq, sp, zp, X, nullptr, M, K, N, s, &om, (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0);
  return map_cuda(e);
}

}  // namespace

extern "C" {

w4a16_status w4a16_pack(const uint8_t* q, const uint16_t* scales, const uint8_t* zeros,
                        int M, int K, int group, void* wq_packed, void* scales_packed,
                        void* zeros_packed, void* stream) {
  return pack_impl(q, scales, zeros, M, K, group, wq_packed, scales_packed, zeros_packed, stream, 0);
}

w4a16_status w4a16_pack_gate_up(const uint8_t* q, const uint16_t* scales, const uint8_t* zeros,
                                int Mi, int K, int group, void* wq_packed, void* scales_packed,
                                void* zeros_packed, void* stream) {
  if (Mi <= 0) return W4A16_ERR_INVALID_ARG;
  if (Mi > kMaxM / 2) return W4A16_ERR_UNSUPPORTED;
  return pack_impl(q, scales, zeros, 2 * Mi, K, group, wq_packed, scales_packed, zeros_packed, stream, Mi);
}

w4a16_status w4a16_gemm_gate_up(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                                const uint16_t* X, uint16_t* H, int Mi, int K, int N, int group, void* stream) {
  return gemm_gate_up_impl(wq_packed, scales_packed, zeros_packed, X, H, Mi, K, N, group, W4A16_PATH_AUTO,
                           nullptr, 0, 0u, stream);
}

w4a16_status w4a16_gemm_gate_up_ws(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                                   const uint16_t* X, uint16_t* H, int Mi, int K, int N, int group, int path,
                                   void* workspace, size_t workspace_bytes, unsigned flags, void* stream) {
  return gemm_gate_up_impl(wq_packed, scales_packed, zeros_packed, X, H, Mi, K, N, group, path, workspace,
                           workspace_bytes, flags, stream);
}

w4a16_status w4a16_gemm_noalloc(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                                const uint16_t* X, uint16_t* Y, int M, int K, int N, int group, unsigned flags,
                                void* stream) {
  if (!wq_packed || !scales_packed || !zeros_packed || !X || !Y || N <= 0) return W4A16_ERR_INVALID_ARG;
  if (flags & ~W4A16_FLAG_EARLY_WEIGHTS) return W4A16_ERR_INVALID_ARG;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (N > kGemvTcMaxTokens || gemv_tc_workspace_bytes(M, K, N) > kNoallocScratchBytes)
    return W4A16_ERR_UNSUPPORTED;
  if (!aligned16(wq_packed) || !aligned16(scales_packed) || !aligned16(zeros_packed) || !aligned16(X) ||
      !aligned16(Y))
    return W4A16_ERR_MISALIGNED;
  {
    const PackedBytes pb = packed_bytes(M, K);
    const size_t ny = (size_t)N * M * 2, nx = (size_t)N * K * 2;
    if (overlap(Y, ny, X, nx) || overlaps_weight(Y, ny, wq_packed, scales_packed, zeros_packed, pb))
      return W4A16_ERR_INVALID_ARG;
  }
  return map_cuda(launch_gemv_tc_noalloc(static_cast<const uint8_t*>(wq_packed),
                                         static_cast<const uint16_t*>(scales_packed),
                                         static_cast<const uint8_t*>(zeros_packed), X, Y, M, K, N,
                                         (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0,
                                         static_cast<cudaStream_t>(stream)));
}

int w4a16_select_path(int M, int K, int N) { return select_path_impl(M, K, N, false); }

int w4a16_select_path_ws(int M, int K, int N) { return select_path_impl(M, K, N, true); }

w4a16_status w4a16_gemm_ex(const void* wq_packed, const void* scales_packed,
                           const void* zeros_packed, const uint16_t* X, uint16_t* Y,
                           int M, int K, int N, int group, int path, void* stream) {
  return gemm_impl(wq_packed, scales_packed, zeros_packed, X, Y, M, K, N, group, path, nullptr, 0, 0u, stream);
}

w4a16_status w4a16_gemm_ws(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                           const uint16_t* X, uint16_t* Y, int M, int K, int N, int group, int path,
                           void* workspace, size_t workspace_bytes, unsigned flags, void* stream) {
  return gemm_impl(wq_packed, scales_packed, zeros_packed, X, Y, M, K, N, group, path, workspace,
                   workspace_bytes, flags, stream);
}

w4a16_status w4a16_gemm_workspace_size(int M, int K, int N, int group, size_t* bytes) {
  if (!bytes || N <= 0) return W4A16_ERR_INVALID_ARG;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (N > kMaxN) return W4A16_ERR_UNSUPPORTED;
  // Enough for the automatic choice and for a forced W4A16_PATH_GEMV_TC.
  *bytes = N <= kGemvTcMaxTokens ? workspace_for(W4A16_PATH_GEMV_TC, M, K, N) : 0;
  return W4A16_OK;
}

w4a16_status w4a16_gemm_qkv(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                            const uint16_t* X, const uint16_t* bias, int Mq, int Mk, int Mv, int K, int N,
                            int group, uint16_t* Yq, uint16_t* Yk, uint16_t* Yv, void* stream) {
  return gemm_qkv_impl(wq_packed, scales_packed, zeros_packed, X, bias, Mq, Mk, Mv, K, N, group, Yq, Yk, Yv,
                       nullptr, 0, 0u, stream);
}

w4a16_status w4a16_add_rmsnorm_gemm_qkv(const uint16_t* h, const uint16_t* d, const uint16_t* gamma, float eps,
                                        uint16_t* r_out, const void* wq_packed, const void* scales_packed,
                                        const void* zeros_packed, const uint16_t* bias, int Mq, int Mk, int Mv,
                                        int K, int N, int group, uint16_t* Yq, uint16_t* Yk, uint16_t* Yv,
                                        unsigned flags, void* stream) {
  if (!h || !gamma || !wq_packed || !scales_packed || !zeros_packed || !Yq || !Yk || !Yv)
    return W4A16_ERR_INVALID_ARG;
  if (Mq <= 0 || Mk <= 0 || Mv <= 0 || N <= 0 || !(eps >= 0.0f) || !(eps <= 3.4028234663852886e38f))
    return W4A16_ERR_INVALID_ARG;
  if (flags & ~W4A16_FLAG_EARLY_WEIGHTS) return W4A16_ERR_INVALID_ARG;
  if ((long long)Mq + Mk + Mv > kMaxM) return W4A16_ERR_UNSUPPORTED;
  const int M = Mq + Mk + Mv;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (N > kGemvMaxTokens) return W4A16_ERR_UNSUPPORTED;
  if (!aligned16(h) || (d && !aligned16(d)) || !aligned16(gamma) || (r_out && !aligned16(r_out)) ||
      !aligned16(wq_packed) || !aligned16(scales_packed) || !aligned16(zeros_packed) || !aligned16(Yq) ||
      !aligned16(Yk) || !aligned16(Yv) || (reinterpret_cast<uintptr_t>(bias) & 1u))
    return W4A16_ERR_MISALIGNED;
  {
    // Outputs (Yq, Yk, Yv, r_out) share no byte with an input or with each
    // other; r_out may not be h or d here (every CTA reads whole rows of h
    // and d while the first row block's CTAs write r).
    const PackedBytes pb = packed_bytes(M, K);
    const size_t nk = (size_t)N * K * 2;
    const void* outs[4] = {Yq, Yk, Yv, r_out};
    const size_t out_n[4] = {(size_t)N * Mq * 2, (size_t)N * Mk * 2, (size_t)N * Mv * 2, r_out ? nk : 0};
    for (int i = 0; i < 4; ++i) {
      if (overlap(outs[i], out_n[i], h, nk) || overlap(outs[i], out_n[i], d, nk) ||
          overlap(outs[i], out_n[i], gamma, (size_t)K * 2) || overlap(outs[i], out_n[i], bias, (size_t)M * 2) ||
          overlaps_weight(outs[i], out_n[i], wq_packed, scales_packed, zeros_packed, pb))
        return W4A16_ERR_INVALID_ARG;
      for (int j = i + 1; j < 4; ++j)
        if (overlap(outs[i], out_n[i], outs[j], out_n[j])) return W4A16_ERR_INVALID_ARG;
    }
  }
  OutMap om = {};
  om.kind = kEpiQkv;
  om.y0 = Yq;
  om.y1 = Yk;
  om.y2 = Yv;
  om.end0 = Mq;
  om.end1 = Mq + Mk;
  om.bias = bias;
  const NormIn nin = {h, d, gamma, eps, r_out};
  return map_cuda(launch_gemv(static_cast<const uint8_t*>(wq_packed), static_cast<const uint16_t*>(scales_packed),
                              static_cast<const uint8_t*>(zeros_packed), nullptr, nullptr, M, K, N,
                              static_cast<cudaStream_t>(stream), &om, (flags & W4A16_FLAG_EARLY_WEIGHTS) != 0,
                              &nin));
}

w4a16_status w4a16_gemm_qkv_ws(const void* wq_packed, const void* scales_packed, const void* zeros_packed,
                               const uint16_t* X, const uint16_t* bias, int Mq, int Mk, int Mv, int K, int N,
                               int group, uint16_t* Yq, uint16_t* Yk, uint16_t* Yv, void* workspace,
                               size_t workspace_bytes, unsigned flags, void* stream) {
  return gemm_qkv_impl(wq_packed, scales_packed, zeros_packed, X, bias, Mq, Mk, Mv, K, N, group, Yq, Yk, Yv,
                       workspace, workspace_bytes, flags, stream);
}

w4a16_status w4a16_gemm(const void* wq_packed, const void* scales_packed,
                        const void* zeros_packed, const uint16_t* X, uint16_t* Y,
                        int M, int K, int N, int group, void* stream) {
  return w4a16_gemm_ex(wq_packed, scales_packed, zeros_packed, X, Y, M, K, N, group,
                       W4A16_PATH_AUTO, stream);
}

w4a16_status w4a16_dequant_debug(const void* wq_packed, const void* scales_packed,
                                 const void* zeros_packed, uint16_t* W_out,
                                 int M, int K, int group, void* stream) {
  if (!wq_packed || !scales_packed || !zeros_packed || !W_out) return W4A16_ERR_INVALID_ARG;
  w4a16_status st = check_shape(M, K, group);
  if (st != W4A16_OK) return st;
  if (!aligned16(wq_packed) || !aligned16(scales_packed) || !aligned16(zeros_packed) ||
      !aligned16(W_out))
    return W4A16_ERR_MISALIGNED;
  if (overlaps_weight(W_out, (size_t)M * K * 2, wq_packed, scales_packed, zeros_packed, packed_bytes(M, K)))
    return W4A16_ERR_INVALID_ARG;
  return map_cuda(launch_dequant(static_cast<const uint8_t*>(wq_packed),
                                 static_cast<const uint16_t*>(scales_packed),
                                 static_cast<const uint8_t*>(zeros_packed), W_out, M, K,
                                 static_cast<cudaStream_t>(stream)));
}

w4a16_status w4a16_device_status(void* stream, int* status) {
  if (!status) return W4A16_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  int a = 0, b = 0, c = 0;
  if (e == cudaSuccess) e = read_and_clear_tc_status(&a);
  if (e == cudaSuccess) e = read_and_clear_gemv_status(&b);
  if (e == cudaSuccess) e = read_and_clear_gvtc_status(&c);
  if (e != cudaSuccess) return map_cuda(e);
  // The decode kernel's word: 1 = a cluster wait gave up, 2 = (debug build)
  // an index check failed; the other families record timeouts only.
  if (a || c || b == 1)
    *status = W4A16_ERR_TIMEOUT;
  else
    *status = b ? W4A16_ERR_BOUNDS : W4A16_OK;
  return W4A16_OK;
}

w4a16_status w4a16_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 0 || limit_cycles > (1LL << 32)) return W4A16_ERR_INVALID_ARG;
  return map_cuda(launch_wait_timeout_selftest(limit_cycles, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
