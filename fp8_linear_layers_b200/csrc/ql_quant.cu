// ql_quant.cu -- activation and weight quantization kernels.
//
// Activations ("Llama 3.1 8B Instruct W8A8", intro and "Loading": int8 per
// token; "Meta-Llama-3.1-8B-Instruct-FP8-dynamic" recipe: per-token dynamic
// symmetric FP8; "Qwen3 8B FP8", "Loading": E4M3 in groups of 128 along K) and
// weights (the same pages' weight formats: a scale for each output row, or for
// each 128x128 block).
//
// Every kernel here is HBM-bound: it reads bf16 once and writes one byte per
// element.  Absmax reductions are warp shuffles (plus one shared-memory step
// for a whole row); the scale is one IEEE f32 division and each code takes the
// correctly rounded quotient (quant_chunk8).
#include <type_traits>

#include "ql_common.cuh"
#include "ql_internal.h"
#include "ql_tc.cuh"

namespace ql {

// Row-wise quantization of [rows, K] bf16: one CTA per row, one scale per row.
//   kInt8       int8 codes clamp(rne(x/s)) with s = a/127, else E4M3 with s = a/448
//   kBf16Scale  the scale is rounded to bf16 before use (W8A8 weight scales)
// Each thread keeps up to kCache 16-byte chunks of the row in registers so the
// row is read from HBM once; longer rows re-read the remainder from L2.
//   kTrigger    activations: the kernel is itself launched with programmatic
//               dependent launch (its CTAs may start while the previous kernel
//               drains; x is read only after the grid dependency wait) and lets
//               its own dependents start early (they stream their weights
//               before waiting; weight writers never trigger)
template <bool kInt8, bool kBf16Scale, bool kTrigger, int kThreads, int kCache>
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(const uint16_t* __restrict__ x,
                                                              int64_t K, uint8_t* __restrict__ q,
                                                              float* __restrict__ s_out) {
  if (kTrigger) {
    if (threadIdx.x == 0) tc::launch_dependents();
    tc::grid_dependency_wait();  // x may be produced by the previous kernel
  }
  const int64_t row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * K);
  const int64_t nchunk = K / 8;  // 8 bf16 per 16-byte chunk
  const int t = threadIdx.x;

  uint4 cache[kCache];
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < kCache; ++i) {
    int64_t c = t + (int64_t)i * kThreads;
    if (c < nchunk) {
      cache[i] = __ldg(xr + c);
      a = fmaxf(a, absmax_chunk8(cache[i]));
    }
  }
  for (int64_t c = t + (int64_t)kCache * kThreads; c < nchunk; c += kThreads)
    a = fmaxf(a, absmax_chunk8(__ldg(xr + c)));

  __shared__ float red[kThreads / 32];
  a = warp_max(a);
  if ((t & 31) == 0) red[t >> 5] = a;
  __syncthreads();
  if (t < 32) {
    float v = (t < kThreads / 32) ? red[t] : 0.0f;
    v = warp_max(v);
    if (t == 0) red[0] = v;
  }
  __syncthreads();
  a = red[0];
  float s = a / (kInt8 ? 127.0f : 448.0f);
  if (kBf16Scale) s = __uint_as_float((uint32_t)f32_to_bf16_rn(s) << 16);
  if (t == 0) s_out[row] = s;
  const Divisor dv = make_divisor(s);

  uint2* qr = reinterpret_cast<uint2*>(q + row * K);
  auto emit_all = [&](auto fast) {
    constexpr bool kFast = decltype(fast)::value;
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
      int64_t c = t + (int64_t)i * kThreads;
      if (c < nchunk) qr[c] = quant_chunk8<kInt8, kFast>(cache[i], dv);
    }
    for (int64_t c = t + (int64_t)kCache * kThreads; c < nchunk; c += kThreads)
      qr[c] = quant_chunk8<kInt8, kFast>(__ldg(xr + c), dv);
  };
  if (dv.fast)
    emit_all(std::true_type{});
  else
    emit_all(std::false_type{});
}

// Per-(token, 128-group) E4M3 quantization: 16 lanes per group, each lane one
// 16-byte chunk (8 bf16); the group absmax is a 16-lane shuffle reduction.
__global__ void __launch_bounds__(256) quant_groups_kernel(const uint16_t* __restrict__ x,
                                                           int64_t ngroups,
                                                           uint8_t* __restrict__ q,
                                                           float* __restrict__ s_out) {
  if (threadIdx.x == 0) tc::launch_dependents();  // activations: dependents may start early
  tc::grid_dependency_wait();                      // x may be produced by the previous kernel
  const int64_t g = (int64_t)blockIdx.x * 16 + (threadIdx.x >> 4);
  const int lane16 = threadIdx.x & 15;
  const bool live = g < ngroups;
  uint4 v = make_uint4(0, 0, 0, 0);
  // group g covers elements [128 g, 128 g + 128) of the flattened [M, K]
  // (K is a multiple of 128, so groups never straddle tokens)
  if (live) v = __ldg(reinterpret_cast<const uint4*>(x + g * 128) + lane16);
  float a = absmax_chunk8(v);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (!live) return;
  const float s = a / 448.0f;
  const Divisor dv = make_divisor(s);
  reinterpret_cast<uint2*>(q + g * 128)[lane16] = quant_chunk8<false>(v, dv);
  if (lane16 == 0) s_out[g] = s;
}

// 128x128 weight blocks: one CTA per block, 256 threads x 8 chunks of 8 bf16.
__global__ void __launch_bounds__(256) quant_wblock_kernel(const uint16_t* __restrict__ w,
                                                           int64_t K, uint8_t* __restrict__ q,
                                                           float* __restrict__ s_out) {
  const int64_t KB = K / 128;
  const int64_t nb = blockIdx.x / KB, kb = blockIdx.x % KB;
  const int t = threadIdx.x;
  uint4 v[8];
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = t + i * 256;  // 2048 chunks: 128 rows x 16 chunks
    const int64_t r = nb * 128 + (c >> 4);
    v[i] = __ldg(reinterpret_cast<const uint4*>(w + r * K + kb * 128) + (c & 15));
    a = fmaxf(a, absmax_chunk8(v[i]));
  }
  __shared__ float red[8];
  a = warp_max(a);
  if ((t & 31) == 0) red[t >> 5] = a;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
  const float s = m / 448.0f;
  if (t == 0) s_out[nb * KB + kb] = s;
  const Divisor dv = make_divisor(s);
  auto emit_all = [&](auto fast) {
    constexpr bool kFast = decltype(fast)::value;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = t + i * 256;
      const int64_t r = nb * 128 + (c >> 4);
      reinterpret_cast<uint2*>(q + r * K + kb * 128)[c & 15] = quant_chunk8<false, kFast>(v[i], dv);
    }
  };
  if (dv.fast)
    emit_all(std::true_type{});
  else
    emit_all(std::false_type{});
}

// Launch with programmatic dependent launch allowed (activation quantizers).
template <typename... Args>
static cudaError_t launch_pdl(void (*kernel)(Args...), unsigned grid, unsigned block, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <bool kInt8, bool kBf16Scale, bool kTrigger>
static cudaError_t launch_rows(const uint16_t* x, int64_t rows, int64_t K, uint8_t* q, float* s,
                               cudaStream_t st) {
  if (K <= 8 * 8 * 256) {
    auto* k = quant_rows_kernel<kInt8, kBf16Scale, kTrigger, 256, 8>;
    if (kTrigger) return launch_pdl(k, (unsigned)rows, 256u, st, x, K, q, s);
    k<<<(unsigned)rows, 256, 0, st>>>(x, K, q, s);
  } else {
    auto* k = quant_rows_kernel<kInt8, kBf16Scale, kTrigger, 512, 8>;
    if (kTrigger) return launch_pdl(k, (unsigned)rows, 512u, st, x, K, q, s);
    k<<<(unsigned)rows, 512, 0, st>>>(x, K, q, s);
  }
  return cudaGetLastError();
}

// An empty kernel launched normally after the weight quantizer: a following
// kernel launched with programmatic dependent launch may start as soon as
// this one exits, and this one starts only once the weights are complete and
// visible, so weights are never streamed before they are written.
__global__ void stream_order_kernel() {}

cudaError_t launch_quantize_act(ql_scheme scheme, const uint16_t* x, int64_t M, int64_t K,
                                uint8_t* qx, float* sx, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  switch (scheme) {
    case QL_W8A8_INT8_ROW: return launch_rows<true, false, true>(x, M, K, qx, sx, st);
    case QL_FP8_E4M3_ROW: return launch_rows<false, false, true>(x, M, K, qx, sx, st);
    default: {
      const int64_t ngroups = M * (K / 128);
      return launch_pdl(quant_groups_kernel, (unsigned)((ngroups + 15) / 16), 256u, st, x, ngroups, qx, sx);
    }
  }
}

cudaError_t launch_quantize_weight(ql_scheme scheme, const uint16_t* w, int64_t N, int64_t K,
                                   uint8_t* wq, float* sw, cudaStream_t st) {
  cudaError_t e;
  switch (scheme) {
    case QL_W8A8_INT8_ROW: e = launch_rows<true, true, false>(w, N, K, wq, sw, st); break;
    case QL_FP8_E4M3_ROW: e = launch_rows<false, false, false>(w, N, K, wq, sw, st); break;
    default:
      quant_wblock_kernel<<<(unsigned)((N / 128) * (K / 128)), 256, 0, st>>>(w, K, wq, sw);
      e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  stream_order_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

}  // namespace ql
