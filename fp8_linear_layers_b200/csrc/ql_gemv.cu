// ql_gemv.cu -- M = 1 decode product y = (s_x s_w) . (Q(x) . W_q^T), one kernel.
//
// "Llama 3.1 8B Instruct W8A8", "Loading": a single token runs "one row in a
// kernel that reads each byte once"; "Qwen3 8B FP8", "Loading": the same for
// the FP8 block scheme.  The kernel is bound by the weight stream: N*K bytes
// from HBM, everything else is L2/shared-memory traffic.
//
// Design (B200, one persistent CTA per SM):
//  * CTA b owns the contiguous output rows [b N / G, (b+1) N / G).  Those rows
//    are one contiguous byte range of W_q, which a producer warp streams into
//    a shared-memory ring (as many stages as fit, each holding whole rows)
//    with bulk copies on the TMA engine, completion tracked by mbarriers.
//  * The kernel is launched with programmatic dependent launch: it lets the
//    next kernel on the stream start as soon as SMs free up, and streams its
//    own weights before the previous kernel has finished; x (which a previous
//    kernel may produce) is read, and y written, only after the grid
//    dependency wait.  Weights must therefore not be written by work still in
//    flight on the stream.
//  * 16 consumer warps quantize x (fused per-token or per-128-group absmax,
//    IEEE-divided scale, rounded codes) into shared memory and keep their
//    fixed slice of the codes in registers.
//  * Each consumer thread owns fixed 16-byte k-chunks of a row group; per
//    chunk it runs 4 dp4a (int8, exact int32) or unpacks 16 E4M3 weights to
//    f32 and does 16 FMAs (E4M3 x E4M3 products are exact in f32).
//  * No CTA-wide barrier per stage: each warp reduces its partial sums with
//    shuffles into a per-stage slot and counts itself in; the last warp to
//    finish a stage adds the slots in a fixed order, writes y and releases the
//    ring stage.  Warps drift freely between stages.
//  * Every wait is bounded; a warp that gives up raises a CTA abort flag that
//    every other wait checks, so all roles leave without further barriers.
#include "ql_common.cuh"
#include "ql_internal.h"
#include "ql_tc.cuh"

namespace ql {

constexpr int kGemvConsumers = 512;  // 16 warps
constexpr int kGemvWarps = kGemvConsumers / 32;
constexpr int kGemvThreads = kGemvConsumers + 32;
constexpr int kGemvMaxStages = 8;
constexpr int kGemvStageTarget = 32768;
constexpr int kGemvSmemBudget = 200 * 1024;
constexpr int kGemvMaxK = 32768;
constexpr int kGemvMaxAcc = 4;
constexpr uint32_t kBarConsumers = 1;  // named barrier id used by the consumer warps

struct GemvParams {
  const uint16_t* x;
  const uint8_t* wq;
  const float* sw;
  uint16_t* y;
  int64_t N, K;
  int rows_per_stage;  // R_s: whole rows per ring stage
  int tg;              // threads per row group (power of two, 32..512)
  int stage_bytes;     // R_s * K rounded up to 128
  int stages;          // ring depth
  ql_debug dbg;
  DevStatus* status;
};

struct GemvSmemLayout {
  int ring, qx, sx, part, bars, flags, total;
};

__host__ __device__ inline GemvSmemLayout gemv_layout(int64_t K, int stage_bytes, int stages) {
  GemvSmemLayout L;
  int off = 0;
  L.ring = off;
  off += stages * stage_bytes;
  L.qx = off;
  off += (int)((K + 127) / 128) * 128;
  L.sx = off;
  off += (int)((K / 128 + 1 + 31) / 32) * 128;
  L.part = off;  // [stages][16 warps][kGemvMaxAcc] partial sums
  off += kGemvMaxStages * kGemvWarps * kGemvMaxAcc * 4;
  L.bars = off;  // full[stages], empty[stages]
  off += 2 * kGemvMaxStages * 8;
  L.flags = off;  // abort flag, per-stage arrival counters, block reduction scratch
  off += 16 + kGemvMaxStages * 4 + kGemvWarps * 4;
  L.total = (off + 127) / 128 * 128;
  return L;
}

QL_DEVINL uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// 16 E4M3 codes (one 16-byte chunk) -> 16 f32 values.
QL_DEVINL void e4m3x16_to_f32(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = e4m3x2_to_f16x2((uint16_t)(w[j] & 0xFFFFu));
    const uint32_t hi = e4m3x2_to_f16x2((uint16_t)(w[j] >> 16));
    f[4 * j + 0] = f16_lo_to_f32(lo);
    f[4 * j + 1] = f16_hi_to_f32(lo);
    f[4 * j + 2] = f16_lo_to_f32(hi);
    f[4 * j + 3] = f16_hi_to_f32(hi);
  }
}

// Sum of the 16 products of one chunk: exact products, f32 sums in two chains.
QL_DEVINL float e4m3_chunk_dot(const uint4& wv, const float* xf) {
  const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
  float p0 = 0.0f, p1 = 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = e4m3x2_to_f16x2((uint16_t)(w[j] & 0xFFFFu));
    const uint32_t hi = e4m3x2_to_f16x2((uint16_t)(w[j] >> 16));
    p0 = fmaf(f16_lo_to_f32(lo), xf[4 * j + 0], p0);
    p1 = fmaf(f16_hi_to_f32(lo), xf[4 * j + 1], p1);
    p0 = fmaf(f16_lo_to_f32(hi), xf[4 * j + 2], p0);
    p1 = fmaf(f16_hi_to_f32(hi), xf[4 * j + 3], p1);
  }
  return p0 + p1;
}

template <bool kInt8>
QL_DEVINL uint32_t quant4(float f0, float f1, float f2, float f3, float s) {
  if (kInt8)
    return (uint32_t)(int8_code(f0, s) & 0xFF) | ((uint32_t)(int8_code(f1, s) & 0xFF) << 8) |
           ((uint32_t)(int8_code(f2, s) & 0xFF) << 16) | ((uint32_t)(int8_code(f3, s) & 0xFF) << 24);
  return f32x2_to_e4m3x2(e4m3_quotient(f0, s), e4m3_quotient(f1, s)) |
         (f32x2_to_e4m3x2(e4m3_quotient(f2, s), e4m3_quotient(f3, s)) << 16);
}

template <ql_scheme kScheme, int kXC>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
  constexpr bool kInt8 = kScheme == QL_W8A8_INT8_ROW;
  constexpr bool kBlock = kScheme == QL_FP8_E4M3_BLOCK128;
  using Acc = typename std::conditional<kInt8, int, float>::type;

  extern __shared__ __align__(1024) uint8_t smem[];
  const int nst = p.stages;
  const GemvSmemLayout L = gemv_layout(p.K, p.stage_bytes, nst);
  uint8_t* ring = smem + L.ring;
  uint8_t* qx_s = smem + L.qx;
  float* sx_s = reinterpret_cast<float*>(smem + L.sx);
  Acc* part = reinterpret_cast<Acc*>(smem + L.part);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kGemvMaxStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flags);
  int* arrivals = reinterpret_cast<int*>(smem + L.flags + 16);
  float* blockred = reinterpret_cast<float*>(smem + L.flags + 16 + kGemvMaxStages * 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t N = p.N, K = p.K;
  const int G = gridDim.x;
  const int64_t row_begin = ((int64_t)blockIdx.x * N) / G;
  const int64_t row_end = ((int64_t)(blockIdx.x + 1) * N) / G;
  const int Rs = p.rows_per_stage;
  const int nstages = (int)((row_end - row_begin + Rs - 1) / Rs);

  if (tid == 0) {
    tc::launch_dependents();  // the next kernel may start as SMs free up
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);  // released by the warp that finishes the stage last
      arrivals[s] = 0;
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kGemvWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      int issued = 0;
      for (int i = 0; i < nstages; ++i) {
        const int slot = i % nst;
        if (i >= nst && !mbar_wait_bounded(&empty[slot], ((i / nst) - 1) & 1, abort_flag)) {
          if (!*abort_flag) record_timeout(p.status, KID_GEMV, 1);
          *abort_flag = 1;
          break;
        }
        const int64_t r0 = row_begin + (int64_t)i * Rs;
        const int64_t nr = min((int64_t)Rs, row_end - r0);
        const uint32_t bytes = (uint32_t)(nr * K);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(ring + slot * p.stage_bytes, p.wq + r0 * K, bytes, &full[slot], policy);
        issued = i + 1;
      }
      // Drain: no copy may still be writing this CTA's shared memory when it
      // exits.  Only this thread arms the full barriers, so after its last
      // arm the parity test below cannot alias a later phase.
      for (int i = max(0, issued - nst); i < issued; ++i)
        mbar_wait_bounded(&full[i % nst], (i / nst) & 1, nullptr);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  tc::grid_dependency_wait();  // x may be produced by the previous kernel
  // 1. Fused activation quantization of x [1, K] into shared memory.
  {
    const int64_t nchunk8 = K / 8;  // 16-byte chunks of 8 bf16
    constexpr int kXCache = kGemvMaxK / 8 / kGemvConsumers;  // 8
    uint4 xc[kXCache];
    float a_tok = 0.0f;
#pragma unroll
    for (int i = 0; i < kXCache; ++i) {
      const int64_t c = tid + (int64_t)i * kGemvConsumers;
      xc[i] = make_uint4(0, 0, 0, 0);
      if (c < nchunk8) xc[i] = __ldg(reinterpret_cast<const uint4*>(p.x) + c);
      const uint32_t w[4] = {xc[i].x, xc[i].y, xc[i].z, xc[i].w};
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
      if (kBlock) {
        // 16 consecutive chunks (lanes) form one 128-wide group
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const float s = a / 448.0f;
        if (c < nchunk8) {
          if ((lane & 15) == 0) sx_s[c >> 4] = s;
          reinterpret_cast<uint2*>(qx_s)[c] =
              make_uint2(quant4<false>(bf16_lo(w[0]), bf16_hi(w[0]), bf16_lo(w[1]), bf16_hi(w[1]), s),
                         quant4<false>(bf16_lo(w[2]), bf16_hi(w[2]), bf16_lo(w[3]), bf16_hi(w[3]), s));
        }
      } else {
        a_tok = fmaxf(a_tok, a);
      }
    }
    if (!kBlock) {
      a_tok = warp_max(a_tok);
      if (lane == 0) blockred[warp] = a_tok;
      named_bar_sync(kBarConsumers, kGemvConsumers);
      float a = blockred[0];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, blockred[w]);
      const float s = a / (kInt8 ? 127.0f : 448.0f);
      if (tid == 0) sx_s[0] = s;
#pragma unroll
      for (int i = 0; i < kXCache; ++i) {
        const int64_t c = tid + (int64_t)i * kGemvConsumers;
        if (c < nchunk8) {
          const uint32_t w[4] = {xc[i].x, xc[i].y, xc[i].z, xc[i].w};
          reinterpret_cast<uint2*>(qx_s)[c] =
              make_uint2(quant4<kInt8>(bf16_lo(w[0]), bf16_hi(w[0]), bf16_lo(w[1]), bf16_hi(w[1]), s),
                         quant4<kInt8>(bf16_lo(w[2]), bf16_hi(w[2]), bf16_lo(w[3]), bf16_hi(w[3]), s));
        }
      }
    }
    named_bar_sync(kBarConsumers, kGemvConsumers);
  }
  if (blockIdx.x == 0 && (p.dbg.qx || p.dbg.sx)) {
    for (int64_t c = tid; c < K / 16; c += kGemvConsumers)
      if (p.dbg.qx) reinterpret_cast<uint4*>(p.dbg.qx)[c] = reinterpret_cast<const uint4*>(qx_s)[c];
    const int ns = kBlock ? (int)(K / 128) : 1;
    for (int i = tid; i < ns; i += kGemvConsumers)
      if (p.dbg.sx) p.dbg.sx[i] = sx_s[i];
  }

  // 2. This thread's fixed k-chunks of a row: kk = u + j * TG (16 bytes each).
  const int TG = p.tg;
  const int RP = kGemvConsumers / TG;  // row groups working side by side
  const int wpg = TG / 32;             // warps per row group
  const int grp = tid / TG, u = tid % TG;
  const int64_t CR = K / 16;
  uint4 xq[kXC];
  float xf[kInt8 ? 1 : kXC * 16];
  float xs[kBlock ? kXC : 1];
  bool have[kXC];
#pragma unroll
  for (int j = 0; j < kXC; ++j) {
    const int64_t kk = u + (int64_t)j * TG;
    have[j] = kk < CR;
    xq[j] = have[j] ? reinterpret_cast<const uint4*>(qx_s)[kk] : make_uint4(0, 0, 0, 0);
    if (!kInt8) e4m3x16_to_f32(xq[j], &xf[16 * j]);
    if (kBlock) xs[j] = have[j] ? sx_s[kk >> 3] : 0.0f;
  }
  const float sx_tok = kBlock ? 0.0f : sx_s[0];
  const int64_t KB = K / 128;

  // 3. Stream the ring.
  const uint32_t ring_a = smem_u32(ring);
  for (int i = 0; i < nstages; ++i) {
    const int slot = i % nst;
    const int64_t r0 = row_begin + (int64_t)i * Rs;
    const int nr = (int)min((int64_t)Rs, row_end - r0);
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (i / nst) & 1, abort_flag))) {
      if (lane == 0 && !*abort_flag) record_timeout(p.status, KID_GEMV, 2);
      *abort_flag = 1;
      break;
    }
    Acc acc[kGemvMaxAcc];
#pragma unroll
    for (int a = 0; a < kGemvMaxAcc; ++a) acc[a] = 0;
    const uint32_t stage_a = ring_a + slot * p.stage_bytes;
#pragma unroll
    for (int a = 0; a < kGemvMaxAcc; ++a) {
      const int r = grp + a * RP;
      if (r < nr) {
        const uint32_t row_a = stage_a + (uint32_t)(r * K);
        float sw_blk[kBlock ? kXC : 1];
        if (kBlock) {
          const float* swr = p.sw + ((r0 + r) >> 7) * KB;
#pragma unroll
          for (int j = 0; j < kXC; ++j) sw_blk[j] = have[j] ? __ldg(swr + ((u + j * TG) >> 3)) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < kXC; ++j) {
          if (have[j]) {
            const uint4 wv = lds128(row_a + (uint32_t)((u + j * TG) * 16));
            if constexpr (kInt8) {
              int s = acc[a];
              s = __dp4a((int)wv.x, (int)xq[j].x, s);
              s = __dp4a((int)wv.y, (int)xq[j].y, s);
              s = __dp4a((int)wv.z, (int)xq[j].z, s);
              s = __dp4a((int)wv.w, (int)xq[j].w, s);
              acc[a] = s;
            } else if constexpr (kBlock) {
              acc[a] = fmaf(e4m3_chunk_dot(wv, &xf[16 * j]), xs[j] * sw_blk[j], acc[a]);
            } else {
              acc[a] += e4m3_chunk_dot(wv, &xf[16 * j]);
            }
          }
        }
      }
    }
    // Reduce over the warp into this stage's partial slot, then count in.
    Acc* ps = part + slot * kGemvWarps * kGemvMaxAcc;
#pragma unroll
    for (int a = 0; a < kGemvMaxAcc; ++a) {
      Acc v = acc[a];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) ps[warp * kGemvMaxAcc + a] = v;
    }
    __syncwarp();
    int before = 0;
    if (lane == 0) {
      __threadfence_block();
      before = atomicAdd(&arrivals[slot], 1);
    }
    before = __shfl_sync(0xffffffffu, before, 0);
    if (before == kGemvWarps - 1) {
      // last warp of this stage: every warp has read the stage and written its slot
      __threadfence_block();
      if (lane < nr) {
        const int r = lane, g = r % RP, a = r / RP;
        Acc v = ps[(g * wpg) * kGemvMaxAcc + a];
        for (int w = 1; w < wpg; ++w) v += ps[(g * wpg + w) * kGemvMaxAcc + a];
        const int64_t n = r0 + r;
        float yv;
        if constexpr (kInt8) {
          if (p.dbg.acc_i32) p.dbg.acc_i32[n] = v;
          yv = __fmul_rn(__fmul_rn(__int2float_rn(v), sx_tok), __ldg(p.sw + n));
        } else if constexpr (kBlock) {
          yv = v;
        } else {
          if (p.dbg.acc_f32) p.dbg.acc_f32[n] = v;
          yv = __fmul_rn(__fmul_rn(v, sx_tok), __ldg(p.sw + n));
        }
        p.y[n] = f32_to_bf16_rn(yv);
      }
      __syncwarp();
      if (lane == 0) {
        arrivals[slot] = 0;
        mbar_arrive(&empty[slot]);
      }
    }
  }
}

static int pow2_floor(int64_t v) {
  int r = 1;
  while ((int64_t)r * 2 <= v) r *= 2;
  return r;
}

int gemv_max_k() { return kGemvMaxK; }

template <ql_scheme S, int XC>
static cudaError_t launch_gemv_x(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem<gemv_kernel<S, XC>>((int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<S, XC>, p);
}

template <ql_scheme S>
static cudaError_t launch_gemv_t(const GemvParams& p, int xc, int grid, size_t smem, cudaStream_t st) {
  switch (xc) {
    case 1: return launch_gemv_x<S, 1>(p, grid, smem, st);
    case 2: return launch_gemv_x<S, 2>(p, grid, smem, st);
    case 4: return launch_gemv_x<S, 4>(p, grid, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemv(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                        int64_t N, int64_t K, uint16_t* y, const ql_debug* dbg, int num_sms,
                        DevStatus* status, cudaStream_t st) {
  GemvParams p;
  p.x = x;
  p.wq = static_cast<const uint8_t*>(wq);
  p.sw = sw;
  p.y = y;
  p.N = N;
  p.K = K;
  p.rows_per_stage = (int)std::max<int64_t>(1, std::min<int64_t>(32, kGemvStageTarget / K));
  const int64_t CR = K / 16;
  p.tg = (int)std::max<int64_t>(32, std::min<int64_t>(kGemvConsumers, pow2_floor(CR)));
  p.stage_bytes = (int)(((int64_t)p.rows_per_stage * K + 127) / 128 * 128);
  const int fixed = gemv_layout(K, p.stage_bytes, 0).total;
  p.stages = (int)std::min<int64_t>(kGemvMaxStages, (kGemvSmemBudget - fixed) / p.stage_bytes);
  if (p.stages < 2) return cudaErrorInvalidConfiguration;
  p.dbg = dbg ? *dbg : ql_debug{nullptr, nullptr, nullptr, nullptr};
  p.status = status;
  const int64_t xc_needed = (CR + p.tg - 1) / p.tg;
  const int xc = xc_needed <= 1 ? 1 : (xc_needed <= 2 ? 2 : 4);
  const int RP = kGemvConsumers / p.tg;
  if ((p.rows_per_stage + RP - 1) / RP > kGemvMaxAcc) return cudaErrorInvalidConfiguration;
  const int64_t stage_rows_total = (N + p.rows_per_stage - 1) / p.rows_per_stage;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms, stage_rows_total));
  const size_t smem = gemv_layout(K, p.stage_bytes, p.stages).total;
  switch (scheme) {
    case QL_W8A8_INT8_ROW: return launch_gemv_t<QL_W8A8_INT8_ROW>(p, xc, grid, smem, st);
    case QL_FP8_E4M3_ROW: return launch_gemv_t<QL_FP8_E4M3_ROW>(p, xc, grid, smem, st);
    default: return launch_gemv_t<QL_FP8_E4M3_BLOCK128>(p, xc, grid, smem, st);
  }
}

}  // namespace ql
