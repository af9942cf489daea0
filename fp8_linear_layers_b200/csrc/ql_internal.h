// ql_internal.h -- host-side launchers shared between the qlinear translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "../../include/qlinear.h"

namespace ql {

struct DevStatus;

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), and
// again only if a larger size is asked for, so launches skip the attribute call.
template <auto kKernel>
inline cudaError_t ensure_smem(int bytes) {
  static int done[64] = {0};  // one table per kernel instantiation
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && __atomic_load_n(&done[dev], __ATOMIC_ACQUIRE) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kKernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) {
    int cur = __atomic_load_n(&done[dev], __ATOMIC_ACQUIRE);
    while (cur < bytes && !__atomic_compare_exchange_n(&done[dev], &cur, bytes, false,
                                                        __ATOMIC_ACQ_REL, __ATOMIC_ACQUIRE)) {
    }
  }
  return e;
}

// 2-D TMA map over a row-major byte matrix, 128-byte swizzle, zero fill.
cudaError_t make_tmap_u8_sw128(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                               uint64_t stride, uint32_t box_inner, uint32_t box_rows);

cudaError_t launch_quantize_act(ql_scheme scheme, const uint16_t* x, int64_t M, int64_t K,
                                uint8_t* qx, float* sx, cudaStream_t st);
cudaError_t launch_quantize_weight(ql_scheme scheme, const uint16_t* w, int64_t N, int64_t K,
                                   uint8_t* wq, float* sw, cudaStream_t st);

int gemv_max_k();
int gemv_max_k_tokens(int64_t M);  // largest K the GEMV takes for M tokens (0: none)
// M = 1 to 4 tokens (extra tokens ride on the MMA's B columns at no extra weight traffic).
// stall: test hook, the producer issues no copies (every consumer wait runs out).
cudaError_t launch_gemv(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, const ql_debug* dbg,
                        int num_sms, DevStatus* status, cudaStream_t st, bool stall = false);
// Up to QL_GEMV_MAX_GROUP products of the same K and token count (1..4) in one
// launch; K <= gemv_max_k_tokens(M).
cudaError_t launch_gemv_grouped(ql_scheme scheme, const ql_gemv_problem* probs, int count, int64_t M,
                                int64_t K, int num_sms, DevStatus* status, cudaStream_t st);
// 5 <= M <= 8 tokens, K <= gemv_max_k_tokens(4), up to QL_GEMV_MAX_GROUP / 2
// products on the same bf16 tokens x [M, K]: one GEMV launch in which each
// product runs as two (tokens 0-3 and 4 .. M-1) over the same weights.
// gemv_token_halves_pay: the shapes where that beats the split-K kernel (the
// products' weights small enough for the launch's fixed cost to dominate).
bool gemv_token_halves_pay(int64_t M, int64_t K, const int64_t* Ns, int count);
cudaError_t launch_gemv_token_halves(ql_scheme scheme, const uint16_t* x, const ql_gemm_problem* probs,
                                     int count, int64_t M, int64_t K, int num_sms, DevStatus* status,
                                     cudaStream_t st);
// 1 <= M <= 4 weight-only product: x stays bf16 (staged as exactly scaled f16),
// W codes dequantized to f16 in registers, f32 sums; K <= gemv_weight_only_max_k().
// Returns cudaErrorNotSupported for shapes whose staged tokens and two ring
// stages do not fit the shared memory.
int gemv_weight_only_max_k();
// largest K the weight-only GEMV takes for M (1..4) tokens (0: none)
int gemv_weight_only_max_k_tokens(int64_t M);
// 1 <= M <= 32 weight-only product: the GEMV kernel up to four tokens (within
// its K limits), else tcgen05 kind::f16 with the weights converted to bf16.
size_t gemm_small_wo_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K);
size_t gemm_small_wo_zeroed_bytes(int64_t M, int64_t N);
cudaError_t launch_gemm_small_wo(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                                 int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace,
                                 size_t ws_bytes, int num_sms, DevStatus* status, cudaStream_t st);
cudaError_t launch_gemv_weight_only(ql_scheme scheme, const uint16_t* x, const void* wq,
                                    const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                    int num_sms, DevStatus* status, cudaStream_t st);

// Large-M tcgen05 GEMM on pre-quantized activations.
size_t gemm_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K, int num_sms);
// a group of 1..QL_GEMM_MAX_GROUP products on one q_x (their N in Ns)
size_t gemm_group_workspace_bytes(ql_scheme scheme, int64_t M, const int64_t* Ns, int count, int64_t K,
                                  int num_sms);
cudaError_t launch_gemm_group(ql_scheme scheme, const void* qx, const float* sx, const ql_gemm_problem* probs,
                              int count, int64_t M, int64_t K, void* workspace, size_t ws_bytes,
                              const ql_debug* dbg, int num_sms, DevStatus* status, cudaStream_t st);
// qy / sy (block scheme only): also write y's E4M3 codes [M,N] and per-128
// scales [M,N/128]; y may then be null.
cudaError_t launch_gemm(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                        const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                        void* workspace, size_t ws_bytes, const ql_debug* dbg, int num_sms,
                        DevStatus* status, cudaStream_t st, uint8_t* qy = nullptr,
                        float* sy = nullptr);

// Small-M (1..32) tensor-core GEMM, K split across the SMs.
size_t gemm_small_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K, int num_sms);
// Bytes at the start of that workspace that must be zero when a call starts
// (split-tile arrival counters, then the atomic-sum slot of every tile); a
// completed call leaves them zero.  0 when the shape runs on the GEMV kernel,
// which does not use the workspace.
size_t gemm_small_zeroed_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K, int num_sms);
// A group of 1..QL_GEMM_MAX_GROUP products on the same tokens (their N in
// Ns): one quantization of the tokens and one launch (up to four tokens within
// the GEMV's K limits, or five to eight on at most 8 MiB of weights with no
// debug captures: one grouped GEMV launch, no workspace used).
size_t gemm_small_group_workspace_bytes(ql_scheme scheme, int64_t M, const int64_t* Ns, int count, int64_t K);
cudaError_t launch_gemm_small_group(ql_scheme scheme, const uint16_t* x, const ql_gemm_problem* probs, int count,
                                    int64_t M, int64_t K, void* workspace, size_t ws_bytes, const ql_debug* dbg,
                                    int num_sms, DevStatus* status, cudaStream_t st,
                                    const uint8_t* pre_qx = nullptr, const float* pre_sx = nullptr);
// pre_qx / pre_sx: the input already quantized (x unused; no quantization
// launch and no GEMV route).
cudaError_t launch_gemm_small(ql_scheme scheme, const uint16_t* x, const void* wq,
                              const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                              void* workspace, size_t ws_bytes, const ql_debug* dbg, int num_sms,
                              DevStatus* status, cudaStream_t st, const uint8_t* pre_qx = nullptr,
                              const float* pre_sx = nullptr);

}  // namespace ql
