// ql_gemm_small_wo.cu -- weight-only ("equivalent") product for 1 <= M <= 32
// tokens on the tensor cores (tcgen05 kind::f16, bf16 x bf16 -> f32).
//
// "Llama 3.1 8B Instruct W8A8" and "Qwen3 8B FP8", "Against bf16": a loader
// option never rounds the input; the W8A8 post's "Context": W8A16 quantizes
// only the weights and keeps computing in bf16.  So
//   y[m,n] = bf16( sum_k x[m,k] * (q_w[n,k] * s_w) ),
// s_w = s_w[n] (row schemes) or s_w[n/128, k/128] (block scheme).
//
// The layout follows the quantized small-M kernel (swap-AB: a 128-row weight
// tile is the MMA's A side, the tokens its N side; the weight stream split
// evenly over the SMs; split tiles summed by the last contributor), with two
// changes:
//  * the tensor cores multiply bf16: the producer's TMA brings the weight
//    codes (128 rows x 128 K bytes) and the tokens' bf16 x (two 128-byte
//    swizzle atoms of 64 elements) into a ring; eight converter warps turn
//    the codes into bf16 (exact: int8 codes and E4M3 values have at most 8
//    significant bits and bf16's exponent range) in a second ring laid out
//    as the MMA's 128-byte-swizzled K-major A operand;
//  * the epilogue applies only the weight scale (x is not quantized).
// The products of two bf16 values are exact in f32; the sums are f32.
//
// Warps: 0 TMA producer, 1 TMEM owner + MMA issuer, 2..9 converters,
// 10..13 epilogue.  Every mbarrier wait is bounded.
#include "ql_tc.cuh"
#include "ql_internal.h"

namespace ql {

constexpr int kWoFirstConv = 2;
constexpr int kWoConvWarps = 8;
constexpr int kWoFirstEpi = kWoFirstConv + kWoConvWarps;
constexpr int kWoEpiWarps = 4;
constexpr int kWoThreads = (kWoFirstEpi + kWoEpiWarps) * 32;
constexpr int kWoTmemCols = 128;
constexpr int kWoBufs = 4;  // TMEM accumulators of 32 columns
constexpr int kWoBufCols = 32;
constexpr int kWoSlots = 2;  // parked partials per split tile (more contributors: atomics)
constexpr int kWoEarlyStages = 2;  // weight stages issued before the grid dependency wait
constexpr uint32_t kWoEpiBar = 1;

template <int NTOK>
struct WoCfg {
  static constexpr int kStageW = 128 * 128;   // codes: 128 weight rows x 128 K
  static constexpr int kStageX = NTOK * 256;  // x: NTOK rows x 128 bf16 (two 128-byte atoms)
  static constexpr int kStage = kStageW + kStageX;
  static constexpr int kStages = 4;
  static constexpr int kConv = 128 * 256;     // bf16 weights: two atoms of 128 rows x 64 elements
  static constexpr int kConvStages = 3;
  static constexpr int kSmem = kStages * kStage + kConvStages * kConv + 1024 + 512;
  static_assert(kStage % 1024 == 0, "stage alignment");
};

struct WoParams {
  const float* sw;
  uint16_t* y;
  int M, N, K;
  int ntn;             // 128-row tiles of W_q
  int nkb;             // 128-wide K blocks
  int units;           // ntn * nkb
  float* accum;        // [kWoSlots][ntn][NTOK][128]: parked partials, or atomic sums in slot 0
  unsigned* counters;  // [ntn], zero between calls
  DevStatus* status;
};

QL_DEVINL bool wo_epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(kWoEpiBar), "r"(kWoEpiWarps * 32)
      : "memory");
  return r != 0;
}

QL_DEVINL int wo_unit_begin(int c, int U, int G) { return (int)(((int64_t)c * U) / G); }
QL_DEVINL int wo_unit_owner(int u, int U, int G) { return (int)((((int64_t)u + 1) * G - 1) / U); }

QL_DEVINL uint32_t f32x2_to_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 16 int8 codes -> 8 bf16 pairs, exact.  With its sign bit flipped, code c
// reads as the byte c + 128; under the f32 exponent of 2^23 (unit spacing) it
// is the f32 value 2^23 + 128 + c, and subtracting 2^23 + 128 leaves c.
QL_DEVINL void s8x16_to_bf16(const uint4& v, uint32_t (&h)[8]) {
  const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u, v.w ^ 0x80808080u};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float f[4];
#pragma unroll
    for (int b = 0; b < 4; ++b)
      f[b] = __fsub_rn(__uint_as_float(__byte_perm(w[q], 0x4B000000u, 0x7650u + b)), 8388736.0f);
    h[2 * q] = f32x2_to_bf16x2(f[0], f[1]);
    h[2 * q + 1] = f32x2_to_bf16x2(f[2], f[3]);
  }
}

// 16 E4M3 codes -> 8 bf16 pairs, exact (E4M3 -> f16 -> f32 -> bf16, no rounding).
QL_DEVINL void e4m3x16_to_bf16(const uint4& v, uint32_t (&h)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const uint32_t f2 = e4m3x2_to_f16x2((uint16_t)(w[q] >> (16 * b)));
      h[2 * q + b] = f32x2_to_bf16x2(f16_lo_to_f32(f2), f16_hi_to_f32(f2));
    }
  }
}

template <ql_scheme S, int NTOK>
__global__ void __launch_bounds__(kWoThreads, 1)
    gemm_small_wo_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                         const WoParams p) {
  using Cfg = WoCfg<NTOK>;
  constexpr bool kInt8 = S == QL_W8A8_INT8_ROW;
  constexpr bool kBlock = S == QL_FP8_E4M3_BLOCK128;
  constexpr uint32_t kIdesc = tc::idesc_bf16(128, NTOK);
  constexpr int kStages = Cfg::kStages;
  constexpr int kConvStages = Cfg::kConvStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* conv = ring + kStages * Cfg::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(conv + kConvStages * Cfg::kConv);
  uint64_t* empty = full + kStages;
  uint64_t* cfull = empty + kStages;
  uint64_t* cempty = cfull + kConvStages;
  uint64_t* tfull = cempty + kConvStages;
  uint64_t* tempty = tfull + kWoBufs;
  uint64_t* mma_done = tempty + kWoBufs;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int u0 = wo_unit_begin(c, p.units, G), u1 = wo_unit_begin(c + 1, p.units, G);
  const int nkb = p.nkb;
  const int n_units = u1 - u0;

  if (threadIdx.x == 0) {
    tc::launch_dependents();
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kWoConvWarps);  // the MMAs (x) and every converter warp (codes)
    }
    for (int s = 0; s < kConvStages; ++s) {
      mbar_init(&cfull[s], kWoConvWarps);
      mbar_init(&cempty[s], 1);
    }
    for (int b = 0; b < kWoBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kWoEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tc::prefetch_tmap(&tmW);
    tc::prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, kWoTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      const int pre = n_units < kWoEarlyStages ? n_units : kWoEarlyStages;
      for (int j = 0; j < pre; ++j) {
        const int u = u0 + j;
        mbar_arrive_expect_tx(&full[j], Cfg::kStage);
        tc::tma_load_2d(ring + j * Cfg::kStage, &tmW, (u % nkb) * 128, (u / nkb) * 128, &full[j], pol_w);
      }
      tc::grid_dependency_wait();  // x may be written by the preceding kernel
      auto load_x = [&](uint8_t* st, int u, uint64_t* bar) {
        const int xb = (u % nkb) * 256;  // bytes of bf16 x: 128 elements per K block
        tc::tma_load_2d(st + Cfg::kStageW, &tmX, xb, 0, bar, pol_x);
        tc::tma_load_2d(st + Cfg::kStageW + NTOK * 128, &tmX, xb + 128, 0, bar, pol_x);
      };
      for (int j = 0; j < pre; ++j) load_x(ring + j * Cfg::kStage, u0 + j, &full[j]);
      int issued = pre;
      for (int j = pre; j < n_units; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait_bounded(&empty[s], ((j / kStages) - 1) & 1, abort_flag)) {
          if (!*abort_flag) record_timeout(p.status, KID_GEMM_SMALL, 4);
          *abort_flag = 1;
          break;
        }
        const int u = u0 + j;
        uint8_t* st = ring + s * Cfg::kStage;
        mbar_arrive_expect_tx(&full[s], Cfg::kStage);
        tc::tma_load_2d(st, &tmW, (u % nkb) * 128, (u / nkb) * 128, &full[s], pol_w);
        load_x(st, u, &full[s]);
        issued = j + 1;
      }
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t jt = 0;
      bool ok = true;
      int j = 0;
      for (int u = u0; u < u1 && ok;) {
        const int t = u / nkb;
        const int seg_end = min(u1, (t + 1) * nkb);
        uint32_t d = 0;
        for (int v = u; v < seg_end; ++v, ++j) {
          const bool first_of_seg = v == u;
          if (kBlock || first_of_seg) {
            const uint32_t buf = jt % kWoBufs;
            if (jt >= (uint32_t)kWoBufs &&
                !mbar_wait_bounded(&tempty[buf], ((jt / kWoBufs) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc::fence_after();
            d = tmem + buf * kWoBufCols;
          }
          const int s = j % kStages, cs = j % kConvStages;
          if (!mbar_wait_bounded(&full[s], (j / kStages) & 1, abort_flag) ||
              !mbar_wait_bounded(&cfull[cs], (j / kConvStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after();
          const uint32_t a_addr = smem_u32(conv + cs * Cfg::kConv);
          const uint32_t b_addr = smem_u32(ring + s * Cfg::kStage + Cfg::kStageW);
#pragma unroll
          for (int at = 0; at < 2; ++at) {
            const uint64_t adesc = tc::sw128_desc(a_addr + at * 16384);
            const uint64_t bdesc = tc::sw128_desc(b_addr + at * NTOK * 128);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc::mma_bf16(d, adesc + 2 * k, bdesc + 2 * k, kIdesc,
                           kBlock ? (at != 0 || k != 0) : (!first_of_seg || at != 0 || k != 0));
          }
          tc::commit(&empty[s]);
          tc::commit(&cempty[cs]);
          if (kBlock) {
            tc::commit(&tfull[jt % kWoBufs]);
            ++jt;
          }
        }
        if (!ok) break;
        if (!kBlock) {
          tc::commit(&tfull[jt % kWoBufs]);
          ++jt;
        }
        u = seg_end;
      }
      if (!ok) {
        if (!*abort_flag) record_timeout(p.status, KID_GEMM_SMALL, 5);
        *abort_flag = 1;
      }
      tc::commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr);
    }
  } else if (warp < kWoFirstEpi) {
    // ------------------------------------------------------------ converters
    // Thread (atom a, row r) turns the 64 codes of row r in K half a of the
    // stage into bf16: code chunk jj (16 bytes, 128-byte swizzle as TMA wrote
    // it) becomes the 32 bytes at chunks 2q, 2q + 1 of atom a's row r, in the
    // swizzled layout the MMA descriptor reads (chunk k of row r at k ^ (r % 8)).
    const int ct = threadIdx.x - kWoFirstConv * 32;  // 0..255
    const int r = ct & 127, a = ct >> 7;
    const uint32_t rsw = (uint32_t)(r & 7);
    for (int j = 0; j < n_units; ++j) {
      const int s = j % kStages, cs = j % kConvStages;
      bool ok = mbar_wait_bounded(&full[s], (j / kStages) & 1, abort_flag);
      if (ok && j >= kConvStages)
        ok = mbar_wait_bounded(&cempty[cs], ((j / kConvStages) - 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0 && !*abort_flag) record_timeout(p.status, KID_GEMM_SMALL, 6);
        *abort_flag = 1;
        break;
      }
      const uint8_t* src = ring + s * Cfg::kStage + r * 128;
      uint8_t* dst = conv + cs * Cfg::kConv + a * 16384 + r * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t jj = (uint32_t)(4 * a + q);
        const uint4 v = *reinterpret_cast<const uint4*>(src + ((jj ^ rsw) << 4));
        uint32_t h[8];
        if constexpr (kInt8)
          s8x16_to_bf16(v, h);
        else
          e4m3x16_to_bf16(v, h);
        *reinterpret_cast<uint4*>(dst + (((uint32_t)(2 * q) ^ rsw) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(dst + (((uint32_t)(2 * q + 1) ^ rsw) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
      }
      fence_proxy_async_smem();  // the tensor cores read these bytes through the async proxy
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&cfull[cs]);
        mbar_arrive(&empty[s]);  // this warp's codes are read
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - kWoFirstEpi * 32;  // 0..127: slot index of this thread
    const int q = warp & 3;                         // TMEM lane quarter this warp may access
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int KB = (p.K + 127) / 128;
    uint32_t jt = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok;) {
      const int t = u / nkb;
      const int seg_end = min(u1, (t + 1) * nkb);
      const bool whole = (u == t * nkb) && (seg_end == (t + 1) * nkb);
      const int n = t * 128 + q * 32 + lane;
      float acc[NTOK];
#pragma unroll
      for (int m = 0; m < NTOK; ++m) acc[m] = 0.0f;
      if constexpr (!kBlock) {
        const uint32_t buf = jt % kWoBufs;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[buf], (jt / kWoBufs) & 1, abort_flag));
        if (ok) {
          tc::fence_after();
          uint32_t rr[32];
          tc::ld32(tmem + lane_addr + buf * kWoBufCols, rr);
          tc::ld_wait();
#pragma unroll
          for (int m = 0; m < NTOK; ++m) acc[m] = __uint_as_float(rr[m]);
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          ++jt;
        }
      } else {
        // one weight block row per tile: promote each 128-deep partial with its scale
        const float* swt = p.sw + (int64_t)t * KB;
        float sw_next = __ldg(swt + (u - t * nkb));
        for (int v = u; v < seg_end; ++v) {
          const int kb = v - t * nkb;
          const float swv = sw_next;
          if (v + 1 < seg_end) sw_next = __ldg(swt + kb + 1);
          const uint32_t buf = jt % kWoBufs;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[buf], (jt / kWoBufs) & 1, abort_flag));
          if (!ok) break;
          tc::fence_after();
          uint32_t rr[32];
          tc::ld32(tmem + lane_addr + buf * kWoBufCols, rr);
          tc::ld_wait();
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          ++jt;
#pragma unroll
          for (int m = 0; m < NTOK; ++m) acc[m] = fmaf(__uint_as_float(rr[m]), swv, acc[m]);
        }
      }
      if (wo_epi_any(!ok)) {
        ok = false;
        break;
      }
      bool do_epilogue = whole;
      if (!whole) {
        // split tile: two contributors park their partials and the second
        // to arrive adds them in a fixed order; more contributors add into
        // slot 0 with L2 atomics and the last reads and clears it
        const int c_first = wo_unit_owner(t * nkb, p.units, G);
        const int c_last = wo_unit_owner((t + 1) * nkb - 1, p.units, G);
        const int ncon = c_last - c_first + 1;
        const bool few = ncon <= kWoSlots;
        float* tacc = p.accum + (int64_t)t * NTOK * 128;
        const int64_t slot_stride = (int64_t)p.ntn * NTOK * 128;
        if (few) {
          float* slot = tacc + (c - c_first) * slot_stride;
#pragma unroll
          for (int m = 0; m < NTOK; ++m)
            if (m < p.M) slot[m * 128 + et] = acc[m];
        } else {
#pragma unroll
          for (int m = 0; m < NTOK; ++m)
            if (m < p.M) atomicAdd(tacc + m * 128 + et, acc[m]);
        }
        __threadfence();
        named_bar_sync(kWoEpiBar, kWoEpiWarps * 32);
        if (et == 0) {
          const unsigned old = atomicAdd(p.counters + t, 1u);
          *last_flag = (old == (unsigned)(c_last - c_first));
        }
        named_bar_sync(kWoEpiBar, kWoEpiWarps * 32);
        do_epilogue = *last_flag != 0;
        if (do_epilogue) {
          __threadfence();
          if (few) {
#pragma unroll
            for (int m = 0; m < NTOK; ++m)
              acc[m] = m < p.M ? __ldcg(tacc + m * 128 + et) + __ldcg(tacc + slot_stride + m * 128 + et) : 0.0f;
          } else {
#pragma unroll
            for (int m = 0; m < NTOK; ++m) acc[m] = m < p.M ? __ldcg(tacc + m * 128 + et) : 0.0f;
#pragma unroll
            for (int m = 0; m < NTOK; ++m)
              if (m < p.M) tacc[m * 128 + et] = 0.0f;
          }
          if (et == 0) p.counters[t] = 0u;
        }
      }
      if (do_epilogue && n < p.N) {
        const float swn = kBlock ? 1.0f : __ldg(p.sw + n);
#pragma unroll
        for (int m = 0; m < NTOK; ++m)
          if (m < p.M) p.y[(int64_t)m * p.N + n] = f32_to_bf16_rn(kBlock ? acc[m] : __fmul_rn(acc[m], swn));
      }
      u = seg_end;
    }
    if (!ok) {
      if (lane == 0 && !*abort_flag) record_timeout(p.status, KID_GEMM_SMALL, 7);
      *abort_flag = 1;
    }
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kWoTmemCols);
  }
}

// ---------------------------------------------------------------- host side

namespace {
struct WoLayout {
  size_t accum, zeroed, total;
};
// arrival counters, then partial-sum slot 0 of every tile (must be zero when
// a call starts), then slot 1 (written before it is read)
WoLayout wo_layout(int64_t M, int64_t N) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  const int ntok = M <= 16 ? 16 : 32;
  const size_t slot_bytes = (size_t)((N + 127) / 128) * ntok * 128 * 4;
  WoLayout L;
  L.accum = up((size_t)((N + 127) / 128) * 4);
  L.zeroed = L.accum + slot_bytes;
  L.total = L.accum + up(kWoSlots * slot_bytes);
  return L;
}
}  // namespace

size_t gemm_small_wo_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K) {
  (void)scheme;
  if (M >= 1 && M <= 4 && K <= gemv_weight_only_max_k_tokens(M)) return 0;  // the GEMV kernel
  return wo_layout(M, N).total;
}

template <ql_scheme S, int NTOK>
static cudaError_t launch_wo_t(const WoParams& p, const CUtensorMap& tw, const CUtensorMap& tx, int grid,
                               cudaStream_t st) {
  using Cfg = WoCfg<NTOK>;
  cudaError_t e = ensure_smem<gemm_small_wo_kernel<S, NTOK>>(Cfg::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kWoThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_small_wo_kernel<S, NTOK>, tw, tx, p);
}

cudaError_t launch_gemm_small_wo(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                                 int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace,
                                 size_t ws_bytes, int num_sms, DevStatus* status, cudaStream_t st) {
  // Up to four tokens within the GEMV's shared-memory limits: the GEMV kernel
  // carries them on its MMA's spare columns (no workspace).
  if (M <= 4 && K <= gemv_weight_only_max_k_tokens(M))
    return launch_gemv_weight_only(scheme, x, wq, sw, M, N, K, y, num_sms, status, st);
  const WoLayout L = wo_layout(M, N);
  if (ws_bytes < L.total) return cudaErrorInvalidValue;
  WoParams p;
  p.sw = sw;
  p.y = y;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.ntn = (int)((N + 127) / 128);
  p.nkb = (int)((K + 127) / 128);
  p.units = p.ntn * p.nkb;
  p.accum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + L.accum);
  p.counters = static_cast<unsigned*>(workspace);
  p.status = status;
  const int ntok = M <= 16 ? 16 : 32;
  CUtensorMap tw, tx;
  cudaError_t e = make_tmap_u8_sw128(&tw, wq, (uint64_t)K, (uint64_t)N, (uint64_t)K, 128, 128);
  if (e != cudaSuccess) return e;
  // x bf16 [M, K] read as bytes [M, 2K]: one box = 64 elements of NTOK rows
  e = make_tmap_u8_sw128(&tx, x, (uint64_t)(2 * K), (uint64_t)M, (uint64_t)(2 * K), 128, (uint32_t)ntok);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<int64_t>(p.units, num_sms);
  switch (scheme) {
    case QL_W8A8_INT8_ROW:
      return ntok == 16 ? launch_wo_t<QL_W8A8_INT8_ROW, 16>(p, tw, tx, grid, st)
                        : launch_wo_t<QL_W8A8_INT8_ROW, 32>(p, tw, tx, grid, st);
    case QL_FP8_E4M3_ROW:
      return ntok == 16 ? launch_wo_t<QL_FP8_E4M3_ROW, 16>(p, tw, tx, grid, st)
                        : launch_wo_t<QL_FP8_E4M3_ROW, 32>(p, tw, tx, grid, st);
    default:
      return ntok == 16 ? launch_wo_t<QL_FP8_E4M3_BLOCK128, 16>(p, tw, tx, grid, st)
                        : launch_wo_t<QL_FP8_E4M3_BLOCK128, 32>(p, tw, tx, grid, st);
  }
}

size_t gemm_small_wo_zeroed_bytes(int64_t M, int64_t N) { return wo_layout(M, N).zeroed; }

}  // namespace ql
