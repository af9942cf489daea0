// ql_api.cu -- the C ABI of libqlinear.so: argument checks, dispatch, status.
//
// Every entry point validates its arguments on the host and returns an error
// before launching anything; none of them allocates, frees or synchronises
// (except qlinear_get_device_status, whose job is to synchronise).
#include <cstdio>
#include <cstring>
#include <mutex>

#include "ql_common.cuh"
#include "ql_internal.h"

// One status word per device (a __device__ variable exists once per device
// context); kernels get its address as an argument.
__device__ ql::DevStatus g_ql_status;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int major = 0;
  int minor = 0;
  ql::DevStatus* status = nullptr;
};

DeviceInfo g_devices[kMaxDevices];
std::mutex g_devices_mu;
thread_local char g_last_cuda_error[256] = "";

ql_status cuda_fail(cudaError_t e, const char* where) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s (%s)", where,
                cudaGetErrorName(e), cudaGetErrorString(e));
  return e == cudaErrorNotSupported ? QL_ERR_UNSUPPORTED_SHAPE : QL_ERR_CUDA;
}

// Properties of the current device, queried once per device.
ql_status current_device(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return QL_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_devices_mu);
  DeviceInfo& d = g_devices[dev];
  if (!d.ready) {
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_ql_status)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress");
    d.status = static_cast<ql::DevStatus*>(p);
    d.ready = true;
  }
  if (d.major != 10 || d.minor != 0) return QL_ERR_DEVICE;  // built for sm_100a only
  *out = d;
  return QL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_scheme(ql_scheme s) {
  return s == QL_W8A8_INT8_ROW || s == QL_FP8_E4M3_ROW || s == QL_FP8_E4M3_BLOCK128;
}

constexpr int64_t kIndexLimit = int64_t(1) << 31;

// Shape rules shared by every entry point.
ql_status check_k(ql_scheme s, int64_t K) {
  if (K <= 0) return QL_ERR_INVALID_ARG;
  if (K % 16) return QL_ERR_UNSUPPORTED_SHAPE;
  if (s == QL_FP8_E4M3_BLOCK128 && K % 128) return QL_ERR_UNSUPPORTED_SHAPE;
  if (s == QL_W8A8_INT8_ROW && K > 133144) return QL_ERR_UNSUPPORTED_SHAPE;  // K * 127^2 < 2^31
  if (s != QL_W8A8_INT8_ROW && K >= 131072) return QL_ERR_UNSUPPORTED_SHAPE;
  return QL_OK;
}

ql_status check_n(ql_scheme s, int64_t N, int64_t K) {
  if (N <= 0) return QL_ERR_INVALID_ARG;
  if (s == QL_FP8_E4M3_BLOCK128 && N % 128) return QL_ERR_UNSUPPORTED_SHAPE;
  if (N * K >= kIndexLimit) return QL_ERR_UNSUPPORTED_SHAPE;
  return QL_OK;
}

ql_status check_m(int64_t M, int64_t N, int64_t K) {
  if (M < 0) return QL_ERR_INVALID_ARG;
  if (M * K >= kIndexLimit || M * N >= kIndexLimit) return QL_ERR_UNSUPPORTED_SHAPE;
  return QL_OK;
}

#define QL_TRY(expr)                   \
  do {                                 \
    ql_status _s = (expr);             \
    if (_s != QL_OK) return _s;        \
  } while (0)

ql_status need(const void* p) {
  if (!p) return QL_ERR_INVALID_ARG;
  return aligned16(p) ? QL_OK : QL_ERR_MISALIGNED;
}

ql_status check_debug(const ql_debug* dbg) {
  if (!dbg) return QL_OK;
  const void* ps[4] = {dbg->qx, dbg->sx, dbg->acc_i32, dbg->acc_f32};
  for (const void* p : ps)
    if (p && !aligned16(p)) return QL_ERR_MISALIGNED;
  return QL_OK;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

extern "C" {

ql_status qlinear_quantize_weight(ql_scheme scheme, const uint16_t* w, int64_t N, int64_t K,
                                  void* wq, float* sw, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  QL_TRY(need(w));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  cudaError_t e = ql::launch_quantize_weight(scheme, w, N, K, static_cast<uint8_t*>(wq), sw,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_quantize_weight");
}

ql_status qlinear_quantize_act(ql_scheme scheme, const uint16_t* x, int64_t M, int64_t K,
                               void* qx, float* sx, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_m(M, 1, K));
  if (M == 0) return QL_OK;
  QL_TRY(need(x));
  QL_TRY(need(qx));
  QL_TRY(need(sx));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  cudaError_t e = ql::launch_quantize_act(scheme, x, M, K, static_cast<uint8_t*>(qx), sx,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_quantize_act");
}

ql_status qlinear_gemv(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                       int64_t N, int64_t K, uint16_t* y, const ql_debug* dbg, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  if (K > ql::gemv_max_k()) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(need(x));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  QL_TRY(check_debug(dbg));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  cudaError_t e = ql::launch_gemv(scheme, x, wq, sw, 1, N, K, y, dbg, d.sms, d.status,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemv");
}

ql_status qlinear_gemv_grouped(ql_scheme scheme, const ql_gemv_problem* problems, int count,
                               int64_t K, void* stream) {
  if (!valid_scheme(scheme) || !problems) return QL_ERR_INVALID_ARG;
  if (count < 1 || count > QL_GEMV_MAX_GROUP) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  if (K > ql::gemv_max_k()) return QL_ERR_UNSUPPORTED_SHAPE;
  for (int j = 0; j < count; ++j) {
    const ql_gemv_problem& pr = problems[j];
    QL_TRY(check_n(scheme, pr.N, K));
    if (pr.x) {
      QL_TRY(need(pr.x));
    } else {
      QL_TRY(need(pr.qx));
      QL_TRY(need(pr.sx));
    }
    QL_TRY(need(pr.wq));
    QL_TRY(need(pr.sw));
    QL_TRY(need(pr.y));
  }
  DeviceInfo d;
  QL_TRY(current_device(&d));
  cudaError_t e = ql::launch_gemv_grouped(scheme, problems, count, 1, K, d.sms, d.status,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemv_grouped");
}

ql_status qlinear_gemv_prequant(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                                const float* sw, int64_t N, int64_t K, uint16_t* y, void* stream) {
  if (!qx || !sx) return QL_ERR_INVALID_ARG;
  const ql_gemv_problem one{nullptr, qx, sx, wq, sw, y, N};
  return qlinear_gemv_grouped(scheme, &one, 1, K, stream);
}

ql_status qlinear_debug_gemv_stalled(ql_scheme scheme, const uint16_t* x, const void* wq,
                                    const float* sw, int64_t N, int64_t K, uint16_t* y,
                                    void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  if (K > ql::gemv_max_k()) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(need(x));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  cudaError_t e = ql::launch_gemv(scheme, x, wq, sw, 1, N, K, y, nullptr, d.sms, d.status,
                                  static_cast<cudaStream_t>(stream), true);
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_debug_gemv_stalled");
}

ql_status qlinear_gemv_weight_only(ql_scheme scheme, const uint16_t* x, const void* wq,
                                   const float* sw, int64_t N, int64_t K, uint16_t* y,
                                   void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  if (K > ql::gemv_weight_only_max_k()) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(need(x));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  cudaError_t e = ql::launch_gemv_weight_only(scheme, x, wq, sw, 1, N, K, y, d.sms, d.status,
                                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemv_weight_only");
}

ql_status qlinear_forward_weight_only(ql_scheme scheme, const uint16_t* x, const void* wq,
                                      const float* sw, int64_t M, int64_t N, int64_t K,
                                      uint16_t* y, void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  QL_TRY(check_m(M, N, K));
  if (M == 0) return QL_OK;
  if (M > 32) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(need(x));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  const size_t need_ws = ql::gemm_small_wo_workspace_bytes(scheme, M, N, K);
  if (need_ws && (!workspace || ws_bytes < need_ws)) return QL_ERR_WORKSPACE;
  if (need_ws && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return QL_ERR_MISALIGNED;
  cudaError_t e = ql::launch_gemm_small_wo(scheme, x, wq, sw, M, N, K, y, workspace, ws_bytes, d.sms,
                                           d.status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_forward_weight_only");
}

size_t qlinear_weight_only_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K) {
  if (!valid_scheme(scheme) || M <= 0 || M > 32 || N <= 0 || K <= 0) return 0;
  return ql::gemm_small_wo_workspace_bytes(scheme, M, N, K);
}

ql_status qlinear_gemm_small(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                             int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace,
                             size_t ws_bytes, const ql_debug* dbg, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  QL_TRY(check_m(M, N, K));
  if (M == 0) return QL_OK;
  if (M > 32) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(need(x));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  QL_TRY(check_debug(dbg));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  const size_t need_ws = ql::gemm_small_workspace_bytes(scheme, M, N, K, d.sms);
  if (need_ws && (!workspace || ws_bytes < need_ws)) return QL_ERR_WORKSPACE;
  if (need_ws && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return QL_ERR_MISALIGNED;
  cudaError_t e = ql::launch_gemm_small(scheme, x, wq, sw, M, N, K, y, workspace, ws_bytes, dbg,
                                        d.sms, d.status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemm_small");
}

ql_status qlinear_gemm_small_grouped(ql_scheme scheme, const uint16_t* x, const void* qx, const float* sx,
                                     const ql_gemm_problem* problems, int count, int64_t M, int64_t K,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  if (!problems || count < 1 || count > QL_GEMM_MAX_GROUP) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  int64_t Ns[QL_GEMM_MAX_GROUP];
  for (int j = 0; j < count; ++j) {
    QL_TRY(check_n(scheme, problems[j].N, K));
    QL_TRY(check_m(M, problems[j].N, K));
    Ns[j] = problems[j].N;
  }
  if (M == 0) return QL_OK;
  if (M > 32) return QL_ERR_UNSUPPORTED_SHAPE;
  if (x) {
    QL_TRY(need(x));
  } else {
    QL_TRY(need(qx));
    QL_TRY(need(sx));
  }
  for (int j = 0; j < count; ++j) {
    QL_TRY(need(problems[j].wq));
    QL_TRY(need(problems[j].sw));
    QL_TRY(need(problems[j].y));
    if (problems[j].qy || problems[j].sy) return QL_ERR_INVALID_ARG;  // no output codes on this path
  }
  DeviceInfo d;
  QL_TRY(current_device(&d));
  const size_t need_ws = ql::gemm_small_group_workspace_bytes(scheme, M, Ns, count, K);
  if (!workspace || ws_bytes < need_ws) return QL_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return QL_ERR_MISALIGNED;
  cudaError_t e = ql::launch_gemm_small_group(scheme, x, problems, count, M, K, workspace, ws_bytes, nullptr, d.sms,
                                              d.status, static_cast<cudaStream_t>(stream),
                                              x ? nullptr : static_cast<const uint8_t*>(qx), x ? nullptr : sx);
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemm_small_grouped");
}

size_t qlinear_gemm_small_grouped_workspace_bytes(ql_scheme scheme, const int64_t* Ns, int count, int64_t M,
                                                  int64_t K) {
  if (!valid_scheme(scheme) || !Ns || count < 1 || count > QL_GEMM_MAX_GROUP || M <= 0 || M > 32 || K <= 0)
    return 0;
  for (int j = 0; j < count; ++j)
    if (Ns[j] <= 0) return 0;
  return ql::gemm_small_group_workspace_bytes(scheme, M, Ns, count, K);
}

ql_status qlinear_gemm_small_prequant(ql_scheme scheme, const void* qx, const float* sx,
                                      const void* wq, const float* sw, int64_t M, int64_t N,
                                      int64_t K, uint16_t* y, void* workspace, size_t ws_bytes,
                                      void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  QL_TRY(check_m(M, N, K));
  if (M == 0) return QL_OK;
  if (M > 32) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(need(qx));
  QL_TRY(need(sx));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  const size_t need_ws = ql::gemm_small_workspace_bytes(scheme, M, N, K, d.sms);
  if (!workspace || ws_bytes < need_ws) return QL_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return QL_ERR_MISALIGNED;
  cudaError_t e = ql::launch_gemm_small(scheme, nullptr, wq, sw, M, N, K, y, workspace, ws_bytes,
                                        nullptr, d.sms, d.status, static_cast<cudaStream_t>(stream),
                                        static_cast<const uint8_t*>(qx), sx);
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemm_small_prequant");
}

ql_status qlinear_gemm(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                       const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                       void* workspace, size_t ws_bytes, const ql_debug* dbg, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  QL_TRY(check_m(M, N, K));
  if (M == 0) return QL_OK;
  QL_TRY(need(qx));
  QL_TRY(need(sx));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  QL_TRY(check_debug(dbg));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  // The workspace is optional here: with it, block-scheme shapes that fill
  // less than one wave of tiles split K over more CTAs; without it, whole tiles.
  const size_t need_ws = ql::gemm_workspace_bytes(scheme, M, N, K, d.sms);
  const bool use_ws = need_ws && workspace && ws_bytes >= need_ws;
  if (use_ws && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return QL_ERR_MISALIGNED;
  cudaError_t e = ql::launch_gemm(scheme, qx, sx, wq, sw, M, N, K, y, use_ws ? workspace : nullptr,
                                  use_ws ? ws_bytes : 0, dbg, d.sms, d.status,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemm");
}

ql_status qlinear_gemm_quant_out(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                                 const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                 void* qy, float* sy, void* workspace, size_t ws_bytes,
                                 void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  if (scheme != QL_FP8_E4M3_BLOCK128) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  QL_TRY(check_m(M, N, K));
  if (M == 0) return QL_OK;
  QL_TRY(need(qx));
  QL_TRY(need(sx));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(qy));
  QL_TRY(need(sy));
  if (y) QL_TRY(need(y));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  const size_t need_ws = ql::gemm_workspace_bytes(scheme, M, N, K, d.sms);
  const bool use_ws = need_ws && workspace && ws_bytes >= need_ws;
  if (use_ws && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return QL_ERR_MISALIGNED;
  cudaError_t e = ql::launch_gemm(scheme, qx, sx, wq, sw, M, N, K, y, use_ws ? workspace : nullptr,
                                  use_ws ? ws_bytes : 0, nullptr, d.sms, d.status,
                                  static_cast<cudaStream_t>(stream), static_cast<uint8_t*>(qy), sy);
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemm_quant_out");
}

ql_status qlinear_gemm_grouped(ql_scheme scheme, const void* qx, const float* sx,
                               const ql_gemm_problem* problems, int count, int64_t M, int64_t K,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  if (!problems || count < 1 || count > QL_GEMM_MAX_GROUP) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  int64_t Ns[QL_GEMM_MAX_GROUP];
  for (int j = 0; j < count; ++j) {
    QL_TRY(check_n(scheme, problems[j].N, K));
    QL_TRY(check_m(M, problems[j].N, K));
    Ns[j] = problems[j].N;
  }
  if (M == 0) return QL_OK;
  QL_TRY(need(qx));
  QL_TRY(need(sx));
  const bool quant_out = problems[0].qy != nullptr;
  for (int j = 0; j < count; ++j) {
    QL_TRY(need(problems[j].wq));
    QL_TRY(need(problems[j].sw));
    if ((problems[j].qy != nullptr) != quant_out || (problems[j].sy != nullptr) != quant_out)
      return QL_ERR_INVALID_ARG;
    if (!quant_out || problems[j].y) QL_TRY(need(problems[j].y));
    if (quant_out) {
      QL_TRY(need(problems[j].qy));
      QL_TRY(need(problems[j].sy));
    }
  }
  if (quant_out && scheme != QL_FP8_E4M3_BLOCK128) return QL_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo d;
  QL_TRY(current_device(&d));
  const size_t need_ws = ql::gemm_group_workspace_bytes(scheme, M, Ns, count, K, d.sms);
  const bool use_ws = need_ws && workspace && ws_bytes >= need_ws;
  if (use_ws && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return QL_ERR_MISALIGNED;
  cudaError_t e = ql::launch_gemm_group(scheme, qx, sx, problems, count, M, K, use_ws ? workspace : nullptr,
                                        use_ws ? ws_bytes : 0, nullptr, d.sms, d.status,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemm_grouped");
}

size_t qlinear_gemm_grouped_workspace_bytes(ql_scheme scheme, const int64_t* Ns, int count, int64_t M,
                                            int64_t K) {
  DeviceInfo d;
  if (!valid_scheme(scheme) || !Ns || count < 1 || count > QL_GEMM_MAX_GROUP || M <= 0 || K <= 0 ||
      current_device(&d) != QL_OK)
    return 0;
  for (int j = 0; j < count; ++j)
    if (Ns[j] <= 0) return 0;
  return ql::gemm_group_workspace_bytes(scheme, M, Ns, count, K, d.sms);
}

size_t qlinear_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K) {
  DeviceInfo d;
  if (!valid_scheme(scheme) || M <= 0 || N <= 0 || K <= 0 || current_device(&d) != QL_OK) return 0;
  if (M <= 32) return ql::gemm_small_workspace_bytes(scheme, M, N, K, d.sms);
  return ql::gemm_workspace_bytes(scheme, M, N, K, d.sms);
}

static size_t forward_act_bytes(ql_scheme scheme, int64_t M, int64_t K) {
  const size_t q = round_up((size_t)(M * K), 256);
  const size_t s = round_up((size_t)M * (scheme == QL_FP8_E4M3_BLOCK128 ? K / 128 : 1) * 4, 256);
  return q + s;
}

size_t qlinear_forward_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K) {
  DeviceInfo d;
  if (!valid_scheme(scheme) || M <= 0 || N <= 0 || K <= 0 || current_device(&d) != QL_OK) return 0;
  if (M == 1 && K <= ql::gemv_max_k()) return 0;
  if (M <= 32) return ql::gemm_small_workspace_bytes(scheme, M, N, K, d.sms);
  return forward_act_bytes(scheme, M, K) + ql::gemm_workspace_bytes(scheme, M, N, K, d.sms);
}

ql_status qlinear_forward(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                          int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace,
                          size_t ws_bytes, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_m(M, N, K));
  if (M == 0) return QL_OK;
  if (M == 1 && K > 0 && K <= ql::gemv_max_k())
    return qlinear_gemv(scheme, x, wq, sw, N, K, y, nullptr, stream);
  if (M <= 32)
    return qlinear_gemm_small(scheme, x, wq, sw, M, N, K, y, workspace, ws_bytes, nullptr, stream);
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  const size_t act = forward_act_bytes(scheme, M, K);
  if (!workspace || ws_bytes < act) return QL_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return QL_ERR_MISALIGNED;
  uint8_t* qx = static_cast<uint8_t*>(workspace);
  float* sx = reinterpret_cast<float*>(qx + round_up((size_t)(M * K), 256));
  QL_TRY(qlinear_quantize_act(scheme, x, M, K, qx, sx, stream));
  uint8_t* rest = static_cast<uint8_t*>(workspace) + act;
  return qlinear_gemm(scheme, qx, sx, wq, sw, M, N, K, y, ws_bytes > act ? rest : nullptr,
                      ws_bytes - act, nullptr, stream);
}

ql_status qlinear_get_device_status(void* stream, uint32_t* detail) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  ql::DevStatus h{0, 0}, zero{0, 0};
  if ((e = cudaMemcpyFromSymbol(&h, g_ql_status, sizeof(h))) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpyFromSymbol");
  if (h.code && (e = cudaMemcpyToSymbol(g_ql_status, &zero, sizeof(zero))) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpyToSymbol");
  if (detail) *detail = h.detail;
  return static_cast<ql_status>(h.code);
}

const char* qlinear_status_string(ql_status status) {
  switch (status) {
    case QL_OK: return "ok";
    case QL_ERR_INVALID_ARG: return "invalid argument (null pointer, unknown scheme or negative size)";
    case QL_ERR_UNSUPPORTED_SHAPE: return "shape not supported by this scheme or entry point";
    case QL_ERR_MISALIGNED: return "device pointer not 16-byte aligned (workspace: 256-byte)";
    case QL_ERR_CUDA: return "CUDA call failed (see qlinear_last_cuda_error)";
    case QL_ERR_TIMEOUT: return "a kernel's bounded wait gave up";
    case QL_ERR_DEVICE: return "no usable sm_100 device is current";
    case QL_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* qlinear_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free small-M entry point.
//
// Scratch for qlinear_gemm_small_noalloc: a fixed array in device global
// memory that every GPU loading the library holds until the process exits.
// Host code must not hand `g_noalloc_scratch` itself to a kernel (on the host
// it is only a stand-in symbol); it uses the device address looked up below.
// ---------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
void* g_noalloc_ptr[kMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, looked up once
// per device with that device current.
ql_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return QL_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return QL_OK;
}
}  // namespace

extern "C" ql_status qlinear_gemm_small_noalloc(ql_scheme scheme, const uint16_t* x, const void* wq,
                                                const float* sw, int64_t M, int64_t N, int64_t K,
                                                uint16_t* y, void* stream) {
  if (!valid_scheme(scheme)) return QL_ERR_INVALID_ARG;
  QL_TRY(check_k(scheme, K));
  QL_TRY(check_n(scheme, N, K));
  QL_TRY(check_m(M, N, K));
  if (M == 0) return QL_OK;
  if (M > 32) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(need(x));
  QL_TRY(need(wq));
  QL_TRY(need(sw));
  QL_TRY(need(y));
  DeviceInfo d;
  QL_TRY(current_device(&d));
  const size_t need_ws = ql::gemm_small_workspace_bytes(scheme, M, N, K, d.sms);
  if (need_ws > kNoAllocScratchBytes) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "qlinear_gemm_small_noalloc: this shape needs %zu bytes of scratch, the static "
                  "scratch holds %zu",
                  need_ws, kNoAllocScratchBytes);
    return QL_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  QL_TRY(noalloc_scratch(&scratch));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The arrival counters and the atomic-sum slots must start at zero; the
  // scratch keeps whatever the previous call left, so clear them (no
  // allocation).  Nothing to clear when the shape runs on the GEMV kernel.
  const size_t zeroed = ql::gemm_small_zeroed_bytes(scheme, M, N, K, d.sms);
  cudaError_t e = cudaSuccess;
  if (zeroed && (e = cudaMemsetAsync(scratch, 0, zeroed, st)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync(scratch sums and counters)");
  e = ql::launch_gemm_small(scheme, x, wq, sw, M, N, K, y, scratch, kNoAllocScratchBytes, nullptr,
                            d.sms, d.status, st);
  return e == cudaSuccess ? QL_OK : cuda_fail(e, "qlinear_gemm_small_noalloc");
}
