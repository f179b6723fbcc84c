// tq_api.cu -- the C ABI declared in include/tq.h: argument validation, then
// one launch per call on the caller's stream.  No allocation, no host sync
// (except tq_query_device_status, which exists to synchronise).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_block(int b) { return b >= 1 && b <= 256 && (b & (b - 1)) == 0; }

int check_device() {
  static int cached = -1;
  if (cached < 0) {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return TQ_ERR_NO_DEVICE;
    }
    cached = (major == 10) ? TQ_OK : TQ_ERR_NO_DEVICE;
  }
  return cached;
}

int check_k(int K, int had_block) {
  if (K < 128 || K > 32768 || K % 128 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if (!pow2_block(had_block) || K % had_block != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  return TQ_OK;
}

int check_r(int r) {
  if (r < 0) return TQ_ERR_INVALID_VALUE;
  if (r % 16 != 0 || r > 512) return TQ_ERR_UNSUPPORTED_SHAPE;
  return TQ_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

}  // namespace

namespace tq {

// Argument checks of the packed-code GEMM's operands (everything except the
// workspace and the device), in the order every GEMM entry applies them.
int gemm_operand_status(const uint8_t* Xq, const float* s_x, const uint8_t* Wq, const float* s_w,
                        const float* XL1, const uint16_t* L2t, int M, int N, int K, int r,
                        const uint16_t* Y, const int32_t* acc) {
  if (!Xq || !Wq || M <= 0 || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (!Y && !acc) return TQ_ERR_INVALID_VALUE;
  if (Y && (!s_x || !s_w)) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, 1)) return s;
  if (int s = check_r(r)) return s;
  if (N < 8 || N % 8 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0) != (XL1 != nullptr) || (r > 0) != (L2t != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(Xq) || !aligned16(Wq) || (s_x && !aligned16(s_x)) ||
      (s_w && !aligned16(s_w)) || (XL1 && !aligned16(XL1)) || (L2t && !aligned16(L2t)) ||
      (Y && !aligned16(Y)) || (acc && !aligned16(acc)))
    return TQ_ERR_MISALIGNED;
  return TQ_OK;
}

int device_status() { return check_device(); }

}  // namespace tq

extern "C" {

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_VALUE: return "TQ_ERR_INVALID_VALUE";
    case TQ_ERR_UNSUPPORTED_SHAPE: return "TQ_ERR_UNSUPPORTED_SHAPE";
    case TQ_ERR_MISALIGNED: return "TQ_ERR_MISALIGNED";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT";
    case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE";
    case TQ_ERR_NO_DEVICE: return "TQ_ERR_NO_DEVICE";
    default: return "TQ_ERR_UNKNOWN";
  }
}

int tq_version(void) { return 100; }

int tq_pack_weight(const float* Rt, int N, int K, int had_block, uint8_t* Wq, float* s_w,
                   void* stream) {
  if (!Rt || !Wq || !s_w || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (!aligned16(Rt) || !aligned16(Wq) || !aligned16(s_w)) return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_pack_weight(Rt, N, K, had_block, Wq, s_w,
                                          static_cast<cudaStream_t>(stream)));
}

int tq_quantize_act(const uint16_t* X, int M, int K, int had_block, const uint16_t* L1t, int r,
                    uint8_t* Xq, float* s_x, float* XL1, void* stream) {
  if (!X || !Xq || !s_x || M <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if ((r > 0) != (L1t != nullptr) || (r > 0) != (XL1 != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(s_x) || (r > 0 && !aligned16(L1t)) ||
      (r > 0 && !aligned16(XL1)))
    return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_quantize_act(X, M, K, had_block, L1t, r, Xq, s_x, XL1,
                                           static_cast<cudaStream_t>(stream)));
}

size_t tq_gemm_workspace_bytes(int M, int N, int K, int r) {
  if (M <= 0 || N <= 0 || K <= 0) return 256;
  return tq::gemm_workspace_bytes(M, N, K, r);
}

static int gemm_common(const uint8_t* Xq, const float* s_x, const uint8_t* Wq, const float* s_w,
                       const float* XL1, const uint16_t* L2t, int M, int N, int K, int r,
                       uint16_t* Y, int32_t* acc, void* ws, size_t ws_bytes, void* stream) {
  if (int s = tq::gemm_operand_status(Xq, s_x, Wq, s_w, XL1, L2t, M, N, K, r, Y, acc)) return s;
  if (ws && !aligned16(ws)) return TQ_ERR_MISALIGNED;
  if (!ws || ws_bytes < tq::gemm_workspace_bytes(M, N, K, r)) return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  tq::GemmArgs a{};
  a.Xq = Xq;
  a.s_x = s_x;
  a.Wq = Wq;
  a.s_w = s_w;
  a.XL1 = XL1;
  a.L2t = L2t;
  a.M = M;
  a.N = N;
  a.K = K;
  a.r = r;
  a.Y = Y;
  a.acc_out = acc;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return from_cuda(tq::launch_gemm(a, static_cast<cudaStream_t>(stream)));
}

int tq_w4a4_lr_gemm(const uint8_t* Xq, const float* s_x, const uint8_t* Wq, const float* s_w,
                    const float* XL1, const uint16_t* L2t, int M, int N, int K, int r,
                    uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream) {
  if (!Y) return TQ_ERR_INVALID_VALUE;
  return gemm_common(Xq, s_x, Wq, s_w, XL1, L2t, M, N, K, r, Y, nullptr, workspace,
                     workspace_bytes, stream);
}

int tq_debug_w4a4_gemm_acc(const uint8_t* Xq, const uint8_t* Wq, int M, int N, int K,
                           int32_t* acc, void* workspace, size_t workspace_bytes, void* stream) {
  if (!acc) return TQ_ERR_INVALID_VALUE;
  return gemm_common(Xq, nullptr, Wq, nullptr, nullptr, nullptr, M, N, K, 0, nullptr, acc,
                     workspace, workspace_bytes, stream);
}

int tq_quantize_act_i8(const uint16_t* X, int M, int K, int had_block, const uint16_t* L1t, int r,
                       int8_t* Xq8, float* s_x, uint16_t* XL1b, void* stream) {
  if (!X || !Xq8 || !s_x || M <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if (had_block > 128) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0) != (L1t != nullptr) || (r > 0) != (XL1b != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(X) || !aligned16(Xq8) || !aligned16(s_x) || (r > 0 && !aligned16(L1t)) ||
      (r > 0 && !aligned16(XL1b)))
    return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_act_tc(X, M, K, had_block, L1t, r, nullptr, Xq8, s_x, nullptr, XL1b,
                                     static_cast<cudaStream_t>(stream)));
}

// The a8 GEMM's stream-K scratch at byte `off` of a workspace, if it fits.
static void* a8_sk(void* ws, size_t ws_bytes, size_t off) {
  return ws && ws_bytes >= off + tq::gemm_a8_sk_bytes() ? static_cast<uint8_t*>(ws) + off
                                                          : nullptr;
}

size_t tq_gemm_a8_workspace_bytes(int M, int N, int K, int r) {
  (void)M; (void)N; (void)K; (void)r;
  return 256 + tq::gemm_a8_sk_bytes();
}

int tq_w4a4_lr_gemm_a8(const int8_t* Xq8, const float* s_x, const uint8_t* Wq, const float* s_w,
                       const uint16_t* XL1b, const uint16_t* L2t, int M, int N, int K, int r,
                       uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (!Xq8 || !s_x || !Wq || !s_w || !Y || M <= 0 || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, 1)) return s;
  if (int s = check_r(r)) return s;
  if (N < 8 || N % 8 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0) != (XL1b != nullptr) || (r > 0) != (L2t != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(Xq8) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y) ||
      (XL1b && !aligned16(XL1b)) || (L2t && !aligned16(L2t)) || (ws && !aligned16(ws)))
    return TQ_ERR_MISALIGNED;
  if (!ws || ws_bytes < tq::gemm_workspace_bytes(M, N, K, r)) return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  tq::GemmA8Args a{};
  a.Xq8 = Xq8;
  a.s_x = s_x;
  a.Wq = Wq;
  a.s_w = s_w;
  a.XL1b = XL1b;
  a.L2t = L2t;
  a.M = M;
  a.N = N;
  a.K = K;
  a.r = r;
  a.Y = Y;
  a.ws = ws;
  a.sk = a8_sk(ws, ws_bytes, 256);
  return from_cuda(tq::launch_gemm_a8(a, static_cast<cudaStream_t>(stream)));
}

// Layer workspace, 256-aligned parts after the 256-byte status word: either
// [Xq M*K/2][s_x 4M][XL1 4Mr] (packed codes) or [Xq8 M*K][s_x 4M][XL1b 2Mr]
// [stream-K scratch] (codes one per byte, M > 128).
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static bool layer_uses_a8(int M, int r, int had_block) {
  (void)r;
  return tq::tuning().layer_a8 && M > 128 && had_block <= 128;
}

int tq_layer_path(int M, int N, int K, int r, int had_block) {
  if (M <= 0 || N <= 0) return -TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return -s;
  if (int s = check_r(r)) return -s;
  if (N < 8 || N % 8 != 0) return -TQ_ERR_UNSUPPORTED_SHAPE;
  if (tq::layer_decode2_supported(M, N, K, r, had_block)) return TQ_PATH_FUSED;
  if (layer_uses_a8(M, r, had_block)) return TQ_PATH_CODES_I8;
  return TQ_PATH_CODES_PACKED;
}

size_t tq_layer_workspace_bytes(int M, int N, int K, int r) {
  if (M <= 0 || N <= 0 || K <= 0 || r < 0) return 256;
  const size_t packed =
      align256((size_t)M * K / 2) + align256((size_t)M * 4) + align256((size_t)M * r * 4);
  const size_t bytes8 = align256((size_t)M * K) + align256((size_t)M * 4) +
                        align256((size_t)M * r * 2) + tq::gemm_a8_sk_bytes();
  return 256 + (M > 128 ? std::max(packed, bytes8) : packed);
}

static int layer_impl(const uint16_t* X, const uint32_t* signs, int n_rht, const uint16_t* L1t,
                      const uint8_t* Wq, const float* s_w, const uint16_t* L2t, int M, int N,
                      int K, int r, int had_block, uint16_t* Y, void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (!X || !Wq || !s_w || !Y || M <= 0 || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if (N < 8 || N % 8 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0) != (L1t != nullptr) || (r > 0) != (L2t != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y) ||
      (L1t && !aligned16(L1t)) || (L2t && !aligned16(L2t)) ||
      (workspace && !aligned16(workspace)))
    return TQ_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < tq_layer_workspace_bytes(M, N, K, r))
    return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tq::layer_decode2_supported(M, N, K, r, had_block)) {
    tq::LayerArgs a{};
    a.signs = signs;
    a.n_rht = n_rht;
    a.X = X;
    a.L1t = L1t;
    a.Wq = Wq;
    a.s_w = s_w;
    a.L2t = L2t;
    a.M = M;
    a.N = N;
    a.K = K;
    a.r = r;
    a.had_block = had_block;
    a.Y = Y;
    a.ws = workspace;
    return from_cuda(tq::launch_layer_decode2(a, st));
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (layer_uses_a8(M, r, had_block)) {
    int8_t* Xq8 = reinterpret_cast<int8_t*>(ws + 256);
    float* s_x8 = reinterpret_cast<float*>(ws + 256 + align256((size_t)M * K));
    uint16_t* XL1b =
        reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(s_x8) + align256((size_t)M * 4));
    // the tensor-core activation kernel applies one sign mask (in shared
    // memory, before its rotation MMA); composed transforms take the
    // butterfly kernel (same int8 outputs)
    if (cudaError_t e = (signs && n_rht > 1)
                            ? tq::launch_quantize_act_bf_i8(X, M, K, had_block, L1t, r, Xq8, s_x8,
                                                            r > 0 ? XL1b : nullptr, st, signs,
                                                            n_rht)
                            : tq::launch_act_tc(X, M, K, had_block, L1t, r, nullptr, Xq8, s_x8,
                                                nullptr, r > 0 ? XL1b : nullptr, st, nullptr,
                                                signs))
      return from_cuda(e);
    tq::GemmA8Args a{};
    a.Xq8 = Xq8;
    a.s_x = s_x8;
    a.Wq = Wq;
    a.s_w = s_w;
    a.XL1b = r > 0 ? XL1b : nullptr;
    a.L2t = L2t;
    a.M = M;
    a.N = N;
    a.K = K;
    a.r = r;
    a.Y = Y;
    a.ws = workspace;
    a.sk = a8_sk(workspace, workspace_bytes,
                 256 + align256((size_t)M * K) + align256((size_t)M * 4) +
                     align256((size_t)M * r * 2));
    return from_cuda(tq::launch_gemm_a8(a, st));
  }
  uint8_t* Xq = ws + 256;
  float* s_x = reinterpret_cast<float*>(Xq + align256((size_t)M * K / 2));
  float* XL1 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(s_x) + align256((size_t)M * 4));
  if (cudaError_t e = tq::launch_quantize_act(X, M, K, had_block, L1t, r, Xq, s_x,
                                              r > 0 ? XL1 : nullptr, st, signs, n_rht))
    return from_cuda(e);
  tq::GemmArgs g{};
  g.Xq = Xq;
  g.s_x = s_x;
  g.Wq = Wq;
  g.s_w = s_w;
  g.XL1 = r > 0 ? XL1 : nullptr;
  g.L2t = L2t;
  g.M = M;
  g.N = N;
  g.K = K;
  g.r = r;
  g.Y = Y;
  g.acc_out = nullptr;
  g.ws = workspace;
  g.ws_bytes = 256;
  return from_cuda(tq::launch_gemm(g, st));
}

int tq_w4a4_lr_layer(const uint16_t* X, const uint16_t* L1t, const uint8_t* Wq, const float* s_w,
                     const uint16_t* L2t, int M, int N, int K, int r, int had_block, uint16_t* Y,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return layer_impl(X, nullptr, 1, L1t, Wq, s_w, L2t, M, N, K, r, had_block, Y, workspace,
                    workspace_bytes, stream);
}

// ------------------------------------------------ randomized Hadamard
// n_rht composed randomized Hadamard transforms: masks [n_rht][K / 32]
static bool rht_count_ok(int n_rht) { return n_rht >= 1 && n_rht <= 3; }

int tq_pack_weight_rhtn(const float* Rt, int N, int K, int had_block, const uint32_t* signs,
                        int n_rht, uint8_t* Wq, float* s_w, void* stream) {
  if (!Rt || !Wq || !s_w || !signs || N <= 0 || !rht_count_ok(n_rht)) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (!aligned16(Rt) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(signs))
    return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_pack_weight(Rt, N, K, had_block, Wq, s_w,
                                          static_cast<cudaStream_t>(stream), signs, n_rht));
}

int tq_pack_weight_rht(const float* Rt, int N, int K, int had_block, const uint32_t* signs,
                       uint8_t* Wq, float* s_w, void* stream) {
  return tq_pack_weight_rhtn(Rt, N, K, had_block, signs, 1, Wq, s_w, stream);
}

int tq_quantize_act_rhtn(const uint16_t* X, int M, int K, int had_block, const uint32_t* signs,
                         int n_rht, const uint16_t* L1t, int r, uint8_t* Xq, float* s_x,
                         float* XL1, void* stream) {
  if (!X || !Xq || !s_x || !signs || M <= 0 || !rht_count_ok(n_rht)) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if ((r > 0) != (L1t != nullptr) || (r > 0) != (XL1 != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(s_x) || !aligned16(signs) ||
      (r > 0 && !aligned16(L1t)) || (r > 0 && !aligned16(XL1)))
    return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_quantize_act(X, M, K, had_block, L1t, r, Xq, s_x, XL1,
                                           static_cast<cudaStream_t>(stream), signs, n_rht));
}

int tq_quantize_act_rht(const uint16_t* X, int M, int K, int had_block, const uint32_t* signs,
                        const uint16_t* L1t, int r, uint8_t* Xq, float* s_x, float* XL1,
                        void* stream) {
  return tq_quantize_act_rhtn(X, M, K, had_block, signs, 1, L1t, r, Xq, s_x, XL1, stream);
}

int tq_w4a4_lr_layer_rhtn(const uint16_t* X, const uint32_t* signs, int n_rht,
                          const uint16_t* L1t, const uint8_t* Wq, const float* s_w,
                          const uint16_t* L2t, int M, int N, int K, int r, int had_block,
                          uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream) {
  if (!signs || !rht_count_ok(n_rht)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(signs)) return TQ_ERR_MISALIGNED;
  return layer_impl(X, signs, n_rht, L1t, Wq, s_w, L2t, M, N, K, r, had_block, Y, workspace,
                    workspace_bytes, stream);
}

int tq_w4a4_lr_layer_rht(const uint16_t* X, const uint32_t* signs, const uint16_t* L1t,
                         const uint8_t* Wq, const float* s_w, const uint16_t* L2t, int M, int N,
                         int K, int r, int had_block, uint16_t* Y, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return tq_w4a4_lr_layer_rhtn(X, signs, 1, L1t, Wq, s_w, L2t, M, N, K, r, had_block, Y,
                               workspace, workspace_bytes, stream);
}

int tq_debug_w4a4_lr_layer_decode(const uint16_t* X, const uint16_t* L1t, const uint8_t* Wq,
                                   const float* s_w, const uint16_t* L2t, int M, int N, int K,
                                   int r, int had_block, uint16_t* Y, int8_t* codes, float* s_x,
                                   int32_t* acc, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (!X || !Wq || !s_w || !Y || M <= 0 || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if (N < 8 || N % 8 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0) != (L1t != nullptr) || (r > 0) != (L2t != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!tq::layer_decode2_supported(M, N, K, r, had_block)) return TQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y) ||
      (L1t && !aligned16(L1t)) || (L2t && !aligned16(L2t)) || (codes && !aligned16(codes)) ||
      (s_x && !aligned16(s_x)) || (acc && !aligned16(acc)) ||
      (workspace && !aligned16(workspace)))
    return TQ_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < 256) return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  tq::LayerArgs a{};
  a.X = X;
  a.L1t = L1t;
  a.Wq = Wq;
  a.s_w = s_w;
  a.L2t = L2t;
  a.M = M;
  a.N = N;
  a.K = K;
  a.r = r;
  a.had_block = had_block;
  a.Y = Y;
  a.ws = workspace;
  return from_cuda(
      tq::launch_layer_decode2(a, static_cast<cudaStream_t>(stream), codes, s_x, acc));
}

int tq_query_device_status(void* workspace, void* stream) {
  if (!workspace) return TQ_ERR_INVALID_VALUE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TQ_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyAsync(workspace, &zero, 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return TQ_ERR_CUDA;
    return TQ_ERR_TIMEOUT;
  }
  return TQ_OK;
}

// ------------------------------------------------------------- gate / up
// Workspace of tq_w4a4_lr_gate_up: [status 256][Xq8 M*K][s_x 4M][XL1b 2M r2]
// [stream-K scratch], 256-aligned parts.
size_t tq_gate_up_workspace_bytes(int M, int N, int K, int r2) {
  (void)N;
  if (M <= 0 || K <= 0 || r2 < 0) return 256;
  return 256 + align256((size_t)M * K) + align256((size_t)M * 4) +
         align256((size_t)M * r2 * 2) + tq::gemm_a8_sk_bytes();
}

int tq_pack_gate_up(const uint8_t* Wq_g, const float* s_w_g, const uint16_t* L1t_g,
                    const uint16_t* L2t_g, const uint8_t* Wq_u, const float* s_w_u,
                    const uint16_t* L1t_u, const uint16_t* L2t_u, int N, int K, int r, uint8_t* Wq2,
                    float* s_w2, uint16_t* L1t2, uint16_t* L2t2, void* stream) {
  if (!Wq_g || !s_w_g || !Wq_u || !s_w_u || !Wq2 || !s_w2 || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, 1)) return s;
  if (int s = check_r(r)) return s;
  if (2 * r > 512) return TQ_ERR_UNSUPPORTED_SHAPE;
  const bool lr = r > 0;
  if (lr != (L1t_g && L2t_g && L1t_u && L2t_u && L1t2 && L2t2) ||
      (!lr && (L1t_g || L2t_g || L1t_u || L2t_u || L1t2 || L2t2)))
    return TQ_ERR_INVALID_VALUE;
  if (!aligned16(Wq_g) || !aligned16(Wq_u) || !aligned16(Wq2) ||
      (lr && (!aligned16(L2t_g) || !aligned16(L2t_u) || !aligned16(L2t2) || !aligned16(L1t2))))
    return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_pack_gate_up(Wq_g, s_w_g, L1t_g, L2t_g, Wq_u, s_w_u, L1t_u, L2t_u, N,
                                           K, r, Wq2, s_w2, L1t2, L2t2,
                                           static_cast<cudaStream_t>(stream)));
}

int tq_w4a4_lr_gate_up(const uint16_t* X, const uint16_t* L1t2, const uint8_t* Wq2,
                       const float* s_w2, const uint16_t* L2t2, int M, int N, int K, int r2,
                       int had_block, uint16_t* Y, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!X || !Wq2 || !s_w2 || !Y || M <= 0 || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r2)) return s;
  if (had_block > 128 || N % 8 != 0 || r2 % 32 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r2 > 0) != (L1t2 != nullptr) || (r2 > 0) != (L2t2 != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(X) || !aligned16(Wq2) || !aligned16(s_w2) || !aligned16(Y) ||
      (L1t2 && !aligned16(L1t2)) || (L2t2 && !aligned16(L2t2)) ||
      (workspace && !aligned16(workspace)))
    return TQ_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < tq_gate_up_workspace_bytes(M, N, K, r2))
    return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* Xq8 = reinterpret_cast<int8_t*>(ws + 256);
  float* s_x = reinterpret_cast<float*>(ws + 256 + align256((size_t)M * K));
  uint16_t* XL1b = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(s_x) + align256((size_t)M * 4));
  if (cudaError_t e = tq::launch_act_tc(X, M, K, had_block, L1t2, r2, nullptr, Xq8, s_x, nullptr,
                                        r2 > 0 ? XL1b : nullptr, st))
    return from_cuda(e);
  tq::GemmA8Args a{};
  a.Xq8 = Xq8;
  a.s_x = s_x;
  a.Wq = Wq2;
  a.s_w = s_w2;
  a.XL1b = r2 > 0 ? XL1b : nullptr;
  a.L2t = L2t2;
  a.M = M;
  a.N = 2 * N;
  a.K = K;
  a.r = r2;
  a.Y = Y;
  a.ws = workspace;
  a.sk = a8_sk(workspace, workspace_bytes,
               256 + align256((size_t)M * K) + align256((size_t)M * 4) +
                   align256((size_t)M * r2 * 2));
  a.swiglu = 1;
  return from_cuda(tq::launch_gemm_a8(a, st));
}

// ------------------------------------------------------- shared input
// Layers reading the same X (Q, K and V; any n <= 8) as one layer: their
// rows concatenated, L1^T stacked along the rank, L2^T block-diagonal.  Only
// copies (no arithmetic): the concatenated layer's Y [M][sum N] holds each
// projection's Y as a column slice, from one activation pass and one GEMM.
int tq_pack_shared_input(int n, const uint8_t* const* Wq, const float* const* s_w,
                         const uint16_t* const* L1t, const uint16_t* const* L2t, const int* N,
                         const int* r, int K, uint8_t* Wq_cat, float* s_w_cat, uint16_t* L1t_cat,
                         uint16_t* L2t_cat, void* stream) {
  if (n < 1 || n > 8 || !Wq || !s_w || !N || !r || !Wq_cat || !s_w_cat) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, 1)) return s;
  long long n_cat = 0, r_cat = 0;
  for (int i = 0; i < n; ++i) {
    if (!Wq[i] || !s_w[i]) return TQ_ERR_INVALID_VALUE;
    if (N[i] < 8 || N[i] % 8 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
    if (int s = check_r(r[i])) return s;
    if (r[i] > 0 && (!L1t || !L2t || !L1t[i] || !L2t[i])) return TQ_ERR_INVALID_VALUE;
    if (!aligned16(Wq[i]) || !aligned16(s_w[i]) ||
        (r[i] > 0 && (!aligned16(L1t[i]) || !aligned16(L2t[i]))))
      return TQ_ERR_MISALIGNED;
    n_cat += N[i];
    r_cat += r[i];
  }
  if (r_cat > 512 || n_cat > (1ll << 30)) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r_cat > 0) != (L1t_cat != nullptr) || (r_cat > 0) != (L2t_cat != nullptr))
    return TQ_ERR_INVALID_VALUE;
  if (!aligned16(Wq_cat) || !aligned16(s_w_cat) || (L1t_cat && !aligned16(L1t_cat)) ||
      (L2t_cat && !aligned16(L2t_cat)))
    return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = (size_t)K / 2;
  if (r_cat > 0 &&
      cudaMemsetAsync(L2t_cat, 0, (size_t)n_cat * (size_t)r_cat * 2, st) != cudaSuccess)
    return TQ_ERR_CUDA;
  size_t off_n = 0, off_r = 0;
  for (int i = 0; i < n; ++i) {
    if (cudaMemcpyAsync(Wq_cat + off_n * row_bytes, Wq[i], (size_t)N[i] * row_bytes,
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(s_w_cat + off_n, s_w[i], (size_t)N[i] * 4, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess)
      return TQ_ERR_CUDA;
    if (r[i] > 0) {
      if (cudaMemcpyAsync(L1t_cat + off_r * (size_t)K, L1t[i], (size_t)r[i] * K * 2,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
          cudaMemcpy2DAsync(L2t_cat + off_n * (size_t)r_cat + off_r, (size_t)r_cat * 2, L2t[i],
                            (size_t)r[i] * 2, (size_t)r[i] * 2, (size_t)N[i],
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return TQ_ERR_CUDA;
    }
    off_n += (size_t)N[i];
    off_r += (size_t)r[i];
  }
  return TQ_OK;
}

// ------------------------------------------------ asymmetric activations
int tq_weight_code_sums(const uint8_t* Wq, int N, int K, int32_t* wsum, void* stream) {
  if (!Wq || !wsum || N <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, 1)) return s;
  if (!aligned16(Wq)) return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_weight_code_sums(Wq, N, K, wsum, static_cast<cudaStream_t>(stream)));
}

int tq_quantize_act_asym_i8(const uint16_t* X, int M, int K, int had_block, const uint16_t* L1t,
                            int r, int8_t* Xq8, float* s_x, float* z_x, uint16_t* XL1b,
                            void* stream) {
  if (!X || !Xq8 || !s_x || !z_x || M <= 0) return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if (had_block > 128) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0) != (L1t != nullptr) || (r > 0) != (XL1b != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(X) || !aligned16(Xq8) || !aligned16(s_x) || !aligned16(z_x) ||
      (r > 0 && !aligned16(L1t)) || (r > 0 && !aligned16(XL1b)))
    return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_act_tc(X, M, K, had_block, L1t, r, nullptr, Xq8, s_x, nullptr, XL1b,
                                     static_cast<cudaStream_t>(stream), z_x));
}

int tq_w4a4_lr_gemm_a8_asym(const int8_t* Xq8, const float* s_x, const float* z_x,
                            const uint8_t* Wq, const float* s_w, const int32_t* wsum,
                            const uint16_t* XL1b, const uint16_t* L2t, int M, int N, int K, int r,
                            uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (!Xq8 || !s_x || !z_x || !Wq || !s_w || !wsum || !Y || M <= 0 || N <= 0)
    return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, 1)) return s;
  if (int s = check_r(r)) return s;
  if (N < 8 || N % 8 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if ((r > 0) != (XL1b != nullptr) || (r > 0) != (L2t != nullptr)) return TQ_ERR_INVALID_VALUE;
  if (!aligned16(Xq8) || !aligned16(s_x) || !aligned16(z_x) || !aligned16(Wq) ||
      !aligned16(s_w) || !aligned16(wsum) || !aligned16(Y) || (XL1b && !aligned16(XL1b)) ||
      (L2t && !aligned16(L2t)) || (ws && !aligned16(ws)))
    return TQ_ERR_MISALIGNED;
  if (!ws || ws_bytes < tq::gemm_workspace_bytes(M, N, K, r)) return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  tq::GemmA8Args a{};
  a.Xq8 = Xq8;
  a.s_x = s_x;
  a.Wq = Wq;
  a.s_w = s_w;
  a.XL1b = XL1b;
  a.L2t = L2t;
  a.M = M;
  a.N = N;
  a.K = K;
  a.r = r;
  a.Y = Y;
  a.ws = ws;
  a.sk = a8_sk(ws, ws_bytes, 256);
  a.z_x = z_x;
  a.wsum = wsum;
  return from_cuda(tq::launch_gemm_a8(a, static_cast<cudaStream_t>(stream)));
}

// ----------------------------------------------- INT4 low-rank branch
int tq_pack_lowrank_q4(const uint16_t* L1t, const uint16_t* L2t, int N, int K, int r,
                       int had_block, int8_t* qL1, float* s_L1, uint16_t* qL2, float* s_L2,
                       void* stream) {
  if (!L1t || !L2t || !qL1 || !s_L1 || !qL2 || !s_L2 || N <= 0 || r <= 0)
    return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if (!aligned16(L1t) || !aligned16(qL1)) return TQ_ERR_MISALIGNED;
  if (int s = check_device()) return s;
  return from_cuda(tq::launch_pack_lowrank_q4(L1t, L2t, N, K, r, had_block, qL1, s_L1, qL2, s_L2,
                                              static_cast<cudaStream_t>(stream)));
}

// Workspace of tq_quantize_act_qlr_i8: [status 256][X L1 INT32 sums 4Mr,
// used for ranks above 256].
size_t tq_quantize_act_qlr_workspace_bytes(int M, int K, int r) {
  (void)K;
  if (M <= 0 || r <= 0) return 256;
  return 256 + align256((size_t)M * r * 4);
}

int tq_quantize_act_qlr_i8(const uint16_t* X, int M, int K, int had_block, const int8_t* qL1,
                           const float* s_L1, int r, int8_t* Xq8, float* s_x, uint16_t* XL1q,
                           float* s_xl1, void* workspace, size_t workspace_bytes, void* stream) {
  if (!X || !qL1 || !s_L1 || !Xq8 || !s_x || !XL1q || !s_xl1 || M <= 0 || r <= 0)
    return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, had_block)) return s;
  if (int s = check_r(r)) return s;
  if (had_block > 128) return TQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(qL1) || !aligned16(Xq8) || !aligned16(s_x) ||
      !aligned16(XL1q) || (workspace && !aligned16(workspace)))
    return TQ_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < tq_quantize_act_qlr_workspace_bytes(M, K, r))
    return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* acc = reinterpret_cast<int32_t*>(ws + 256);
  // the rotated activation codes, one per byte
  if (cudaError_t e = tq::launch_act_tc(X, M, K, had_block, nullptr, 0, nullptr, Xq8, s_x, nullptr,
                                        nullptr, st))
    return from_cuda(e);
  // X L1 in INT32 from those codes and the INT4 L1 (H^T L1 per column),
  // dequantized with s_x s_L1 and requantized per token to INT4
  return from_cuda(tq::launch_xl1_codes(Xq8, qL1, s_x, s_L1, M, K, r, XL1q, s_xl1, acc,
                                        reinterpret_cast<uint32_t*>(ws), st));
}

int tq_w4a4_lr_gemm_a8_qlr(const int8_t* Xq8, const float* s_x, const uint8_t* Wq,
                           const float* s_w, const uint16_t* XL1q, const float* s_xl1,
                           const uint16_t* qL2, const float* s_L2, int M, int N, int K, int r,
                           uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (!Xq8 || !s_x || !Wq || !s_w || !XL1q || !s_xl1 || !qL2 || !s_L2 || !Y || M <= 0 ||
      N <= 0 || r <= 0)
    return TQ_ERR_INVALID_VALUE;
  if (int s = check_k(K, 1)) return s;
  if (int s = check_r(r)) return s;
  if (N < 8 || N % 8 != 0) return TQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(Xq8) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_w) ||
      !aligned16(XL1q) || !aligned16(s_xl1) || !aligned16(qL2) || !aligned16(s_L2) ||
      !aligned16(Y) || (ws && !aligned16(ws)))
    return TQ_ERR_MISALIGNED;
  if (!ws || ws_bytes < tq::gemm_workspace_bytes(M, N, K, r)) return TQ_ERR_WORKSPACE;
  if (int s = check_device()) return s;
  tq::GemmA8Args a{};
  a.Xq8 = Xq8;
  a.s_x = s_x;
  a.Wq = Wq;
  a.s_w = s_w;
  a.XL1b = XL1q;
  a.L2t = qL2;
  a.M = M;
  a.N = N;
  a.K = K;
  a.r = r;
  a.Y = Y;
  a.ws = ws;
  a.sk = a8_sk(ws, ws_bytes, 256);
  a.s_xl1 = s_xl1;
  a.s_l2 = s_L2;
  return from_cuda(tq::launch_gemm_a8(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

