// ql_gemm_small.cu -- 1 <= M <= 32 tokens on the tensor cores (tcgen05).
//
// "Llama 3.1 8B Instruct W8A8", "Loading": batches of at most 32 tokens run on
// the tensor cores;
// "Qwen3 8B FP8", "Loading": the same for the FP8 block scheme.  With at most
// 32 tokens the product is still bound by the weight stream (<= 64 ops per
// weight byte), so the design spreads W_q evenly over every SM:
//
//  * swap-AB: the MMA's 128-row A side is a 128-row tile of W_q, the tokens
//    are its N side (16 or 32 columns); one MMA is 128 x NTOK x 32.
//  * the W_q stream is cut into units of (128 weight rows x 128 bytes of K);
//    CTA c owns the contiguous units [c U / G, (c+1) U / G), so every SM
//    streams the same number of bytes.  A run of units inside one 128-row
//    tile accumulates in TMEM; a tile that was split between CTAs is summed
//    by the CTA that finishes last (an atomic arrival counter, no waiting),
//    in a fixed contributor order, from per-CTA partial slots.
//  * activation quantization runs first as its own short kernel writing q_x
//    and s_x into the workspace; this kernel is launched with programmatic
//    dependent launch, starts its weight loads at once and waits for the
//    quantized tokens only before loading them; it releases the next kernel
//    on the stream as soon as its own CTAs have started.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2..5
// epilogue (one TMEM lane = one weight row per thread).  Every mbarrier wait is
// bounded.
#include <climits>
#include <cstring>

#include "ql_tc.cuh"
#include "ql_internal.h"

namespace ql {

constexpr int kSmallEpiWarps = 4;
constexpr int kSmallThreads = 64 + kSmallEpiWarps * 32;
constexpr int kSmallTmemCols = 128;
constexpr int kSmallBufs = 4;  // TMEM accumulators of 32 columns
constexpr int kSmallBufCols = 32;
constexpr int kSmallSlots = 2;  // parked partials per split tile (more contributors: atomics)
constexpr int kSmallEarlyStages = 2;  // weight stages issued before the tokens
constexpr uint32_t kSmallEpiBar = 1;

template <int NTOK>
struct SmallCfg {
  static constexpr int kStageA = 128 * 128;
  static constexpr int kStageB = NTOK * 128;
  static constexpr int kStage = kStageA + kStageB;
  static constexpr int kStages = (200 * 1024 / kStage) > 12 ? 12 : (200 * 1024 / kStage);
  static constexpr int kRing = kStages * kStage;
  static constexpr int kSmem = kRing + 1024 + 512;
  static_assert(kStage % 1024 == 0, "stage alignment");
};

// A launch runs 1 to kSmallMaxGroup products that read the same tokens (a
// layer's q, k, v; gate, up): product j owns 128-row tiles [t0[j], t0[j+1]).
constexpr int kSmallMaxGroup = QL_GEMM_MAX_GROUP;

struct SmallParams {
  const float* sx;  // workspace: [M] or [M, K/128]
  const float* sw[kSmallMaxGroup];
  uint16_t* y[kSmallMaxGroup];
  int N[kSmallMaxGroup];
  int t0[kSmallMaxGroup + 1];  // INT_MAX past the last product
  int nprob;
  int M, K;
  int ntn;          // 128-row tiles of W_q, all products
  int nkb;          // 128-byte K blocks
  int units;        // ntn * nkb
  void* accum;         // [kSmallSlots][ntn][NTOK][128] int32 or f32: parked partials, or atomic
                       // sums in slot 0 (slot 0 zero between calls; slot 1 written before read)
  unsigned* counters;  // [ntn], zero between calls
  int32_t* acc_i32;
  float* acc_f32;
  DevStatus* status;
};

// The products' W_q tensor maps (kernel parameters, read by TMA from the
// parameter space).
struct SmallMapsW {
  CUtensorMap m[kSmallMaxGroup];
};

// Tile t's product and its tile index inside it, by constant-index selects.
struct SmallProd {
  const float* sw;
  uint16_t* y;
  int N, tl, j;
};
static_assert(kSmallMaxGroup == 4, "small_prod selects among four products");
QL_DEVINL SmallProd small_prod(const SmallParams& p, int t) {
  const int j = (t >= p.t0[1]) + (t >= p.t0[2]) + (t >= p.t0[3]);
  SmallProd v;
  v.j = j;
  v.sw = j == 0 ? p.sw[0] : j == 1 ? p.sw[1] : j == 2 ? p.sw[2] : p.sw[3];
  v.y = j == 0 ? p.y[0] : j == 1 ? p.y[1] : j == 2 ? p.y[2] : p.y[3];
  v.N = j == 0 ? p.N[0] : j == 1 ? p.N[1] : j == 2 ? p.N[2] : p.N[3];
  v.tl = t - (j == 0 ? 0 : j == 1 ? p.t0[1] : j == 2 ? p.t0[2] : p.t0[3]);
  return v;
}
QL_DEVINL const CUtensorMap* small_map(const SmallMapsW& w, int j) {
  return j == 0 ? &w.m[0] : j == 1 ? &w.m[1] : j == 2 ? &w.m[2] : &w.m[3];
}

// OR vote over the epilogue warps that doubles as their barrier.
QL_DEVINL bool epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(kSmallEpiBar), "r"(kSmallEpiWarps * 32)
      : "memory");
  return r != 0;
}

// First unit of CTA c, and the CTA that owns unit u, under the even split.
QL_DEVINL int unit_begin(int c, int U, int G) { return (int)(((int64_t)c * U) / G); }
QL_DEVINL int unit_owner(int u, int U, int G) { return (int)((((int64_t)u + 1) * G - 1) / U); }

template <ql_scheme S, int NTOK>
__global__ void __launch_bounds__(kSmallThreads, 1)
    gemm_small_kernel(const __grid_constant__ SmallMapsW tmW, const __grid_constant__ CUtensorMap tmX,
                      const SmallParams p) {
  using Cfg = SmallCfg<NTOK>;
  constexpr bool kInt8 = S == QL_W8A8_INT8_ROW;
  constexpr bool kBlock = S == QL_FP8_E4M3_BLOCK128;
  constexpr uint32_t kIdesc = tc::idesc(kInt8, 128, NTOK);
  constexpr int kStages = Cfg::kStages;
  using Acc = typename std::conditional<kInt8, int, float>::type;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + Cfg::kRing);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + kSmallBufs;
  uint64_t* mma_done = tempty + kSmallBufs;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int u0 = unit_begin(c, p.units, G), u1 = unit_begin(c + 1, p.units, G);
  const int nkb = p.nkb;

  if (threadIdx.x == 0) {
    tc::launch_dependents();  // the next kernel's CTAs may start as SMs free up
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kSmallBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kSmallEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    for (int j = 0; j < p.nprob; ++j) tc::prefetch_tmap(small_map(tmW, j));
    tc::prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, kSmallTmemCols);
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
      const int n = u1 - u0;
      // weights first: they do not depend on the quantization kernel.  Only a
      // couple of stages go out before the quantized tokens are requested: a
      // full ring fill from every SM would queue those (L2-resident) loads
      // behind ~30 MB of weight reads.
      const int pre = n < kSmallEarlyStages ? n : kSmallEarlyStages;
      for (int j = 0; j < pre; ++j) {
        const int u = u0 + j;
        const SmallProd pv = small_prod(p, u / nkb);
        mbar_arrive_expect_tx(&full[j], Cfg::kStage);
        tc::tma_load_2d(ring + j * Cfg::kStage, small_map(tmW, pv.j), (u % nkb) * 128, pv.tl * 128, &full[j], pol_w);
      }
      tc::grid_dependency_wait();  // q_x is written by the preceding kernel
      for (int j = 0; j < pre; ++j) {
        const int u = u0 + j;
        tc::tma_load_2d(ring + j * Cfg::kStage + Cfg::kStageA, &tmX, (u % nkb) * 128, 0, &full[j], pol_x);
      }
      int issued = pre;
      for (int j = pre; j < n; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait_bounded(&empty[s], ((j / kStages) - 1) & 1, abort_flag)) {
          if (!*abort_flag) record_timeout(p.status, KID_GEMM_SMALL, 1);
          *abort_flag = 1;
          break;
        }
        const int u = u0 + j;
        uint8_t* st = ring + s * Cfg::kStage;
        mbar_arrive_expect_tx(&full[s], Cfg::kStage);
        const SmallProd pv = small_prod(p, u / nkb);
        tc::tma_load_2d(st, small_map(tmW, pv.j), (u % nkb) * 128, pv.tl * 128, &full[s], pol_w);
        tc::tma_load_2d(st + Cfg::kStageA, &tmX, (u % nkb) * 128, 0, &full[s], pol_x);
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
      int j = 0;  // unit index inside this CTA's range
      for (int u = u0; u < u1 && ok;) {
        const int t = u / nkb;
        const int seg_end = min(u1, (t + 1) * nkb);
        uint32_t d = 0;
        for (int v = u; v < seg_end; ++v, ++j) {
          const bool first_of_seg = v == u;
          if (kBlock || first_of_seg) {
            const uint32_t buf = jt % kSmallBufs;
            if (jt >= (uint32_t)kSmallBufs &&
                !mbar_wait_bounded(&tempty[buf], ((jt / kSmallBufs) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc::fence_after();
            d = tmem + buf * kSmallBufCols;
          }
          const int s = j % kStages;
          if (!mbar_wait_bounded(&full[s], (j / kStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after();
          const uint32_t a_addr = smem_u32(ring + s * Cfg::kStage);
          const uint64_t adesc = tc::sw128_desc(a_addr);
          const uint64_t bdesc = tc::sw128_desc(a_addr + Cfg::kStageA);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma<kInt8>(d, adesc + 2 * k, bdesc + 2 * k, kIdesc,
                           kBlock ? (k != 0) : (!first_of_seg || k != 0));
          tc::commit(&empty[s]);
          if (kBlock) {
            tc::commit(&tfull[jt % kSmallBufs]);
            ++jt;
          }
        }
        if (!ok) break;
        if (!kBlock) {
          tc::commit(&tfull[jt % kSmallBufs]);
          ++jt;
        }
        u = seg_end;
      }
      if (!ok) {
        if (!*abort_flag) record_timeout(p.status, KID_GEMM_SMALL, 2);
        *abort_flag = 1;
      }
      tc::commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;  // 0..127 = TMEM lane = weight row in the tile
    const int q = warp & 3;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int KB = p.K / 128;
    tc::grid_dependency_wait();  // s_x comes from the quantization kernel
    uint32_t jt = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok;) {
      const int t = u / nkb;
      const int seg_end = min(u1, (t + 1) * nkb);
      const bool whole = (u == t * nkb) && (seg_end == (t + 1) * nkb);
      const SmallProd pv = small_prod(p, t);
      const int n = pv.tl * 128 + q * 32 + lane;  // this thread's output row in its product
      Acc acc[NTOK];
#pragma unroll
      for (int m = 0; m < NTOK; ++m) acc[m] = 0;
      if constexpr (!kBlock) {
        const uint32_t buf = jt % kSmallBufs;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[buf], (jt / kSmallBufs) & 1, abort_flag));
      }
      if (!kBlock && ok) {
        const uint32_t buf = jt % kSmallBufs;
        tc::fence_after();
        uint32_t r[32];
        tc::ld32(tmem + lane_addr + buf * kSmallBufCols, r);
        tc::ld_wait();
#pragma unroll
        for (int m = 0; m < NTOK; ++m) acc[m] = kInt8 ? (Acc)(int)r[m] : (Acc)__uint_as_float(r[m]);
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        ++jt;
      } else if (kBlock) {
        const float* swt = pv.sw + (int64_t)pv.tl * KB;
        // the next K block's scales are loaded while this block's MMAs run
        float sx_next[NTOK];
        float sw_next = __ldg(swt + (u - t * nkb));
#pragma unroll
        for (int m = 0; m < NTOK; ++m)
          sx_next[m] = m < p.M ? __ldg(p.sx + (int64_t)m * KB + (u - t * nkb)) : 0.0f;
        for (int v = u; v < seg_end; ++v) {
          const int kb = v - t * nkb;
          float sxv[NTOK];
#pragma unroll
          for (int m = 0; m < NTOK; ++m) sxv[m] = sx_next[m];
          const float swv = sw_next;
          if (v + 1 < seg_end) {
            sw_next = __ldg(swt + kb + 1);
#pragma unroll
            for (int m = 0; m < NTOK; ++m) sx_next[m] = m < p.M ? __ldg(p.sx + (int64_t)m * KB + kb + 1) : 0.0f;
          }
          const uint32_t buf = jt % kSmallBufs;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[buf], (jt / kSmallBufs) & 1, abort_flag));
          if (!ok) break;
          tc::fence_after();
          uint32_t r[32];
          tc::ld32(tmem + lane_addr + buf * kSmallBufCols, r);
          tc::ld_wait();
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          ++jt;
#pragma unroll
          for (int m = 0; m < NTOK; ++m) acc[m] = fmaf(__uint_as_float(r[m]), sxv[m] * swv, acc[m]);
        }
      }
      // every epilogue warp leaves together if any of them gave up a wait
      if (epi_any(!ok)) {
        ok = false;
        break;
      }

      bool do_epilogue = whole;
      if (!whole) {
        // A tile split between two CTAs: each parks its partial in its own
        // slot and the second to arrive adds the two in a fixed order.  A tile
        // with more contributors (small N: up to ~20) adds into one slot with
        // L2 atomics (int32 exact for int8; f32 for E4M3, whose order of
        // addition then varies from call to call), and the last to arrive
        // reads the sums and zeroes them for the next call -- summing parked
        // partials there took one L2 round trip per contributor.
        const int c_first = unit_owner(t * nkb, p.units, G);
        const int c_last = unit_owner((t + 1) * nkb - 1, p.units, G);
        const int ncon = c_last - c_first + 1;
        const bool few = ncon <= kSmallSlots;
        // slot k of tile t; slot 0 is also the atomic-sum slot
        Acc* tacc = reinterpret_cast<Acc*>(p.accum) + (int64_t)t * NTOK * 128;
        const int64_t slot_stride = (int64_t)p.ntn * NTOK * 128;
        if (few) {
          Acc* slot = tacc + (c - c_first) * slot_stride;
#pragma unroll
          for (int m = 0; m < NTOK; ++m)
            if (m < p.M) slot[m * 128 + et] = acc[m];
        } else {
#pragma unroll
          for (int m = 0; m < NTOK; ++m)
            if (m < p.M) atomicAdd(tacc + m * 128 + et, acc[m]);
        }
        __threadfence();
        named_bar_sync(kSmallEpiBar, kSmallEpiWarps * 32);
        if (et == 0) {
          const unsigned old = atomicAdd(p.counters + t, 1u);
          *last_flag = (old == (unsigned)(c_last - c_first));
        }
        named_bar_sync(kSmallEpiBar, kSmallEpiWarps * 32);
        do_epilogue = *last_flag != 0;
        if (do_epilogue) {
          __threadfence();
          if (few) {
#pragma unroll
            for (int m = 0; m < NTOK; ++m) {
              Acc v = 0;
              if (m < p.M) {
                // fixed order: the first contributor's part, then the second's
                v = __ldcg(tacc + m * 128 + et) + __ldcg(tacc + slot_stride + m * 128 + et);
              }
              acc[m] = v;
            }
          } else {
#pragma unroll
            for (int m = 0; m < NTOK; ++m) acc[m] = m < p.M ? __ldcg(tacc + m * 128 + et) : (Acc)0;
#pragma unroll
            for (int m = 0; m < NTOK; ++m)
              if (m < p.M) tacc[m * 128 + et] = (Acc)0;  // zero again for the next call
          }
          if (et == 0) p.counters[t] = 0u;  // every contributor has arrived: reset for the next call
        }
      }
      if (do_epilogue && n < pv.N) {
        const float swn = kBlock ? 1.0f : __ldg(pv.sw + n);
#pragma unroll
        for (int m = 0; m < NTOK; ++m) {
          if (m < p.M) {
            float yv;
            if constexpr (kInt8) {
              if (p.acc_i32) p.acc_i32[(int64_t)m * pv.N + n] = acc[m];
              yv = __fmul_rn(__fmul_rn(__int2float_rn(acc[m]), __ldg(p.sx + m)), swn);
            } else if constexpr (kBlock) {
              yv = acc[m];
            } else {
              if (p.acc_f32) p.acc_f32[(int64_t)m * pv.N + n] = acc[m];
              yv = __fmul_rn(__fmul_rn(acc[m], __ldg(p.sx + m)), swn);
            }
            pv.y[(int64_t)m * pv.N + n] = f32_to_bf16_rn(yv);
          }
        }
      }
      u = seg_end;
    }
    if (!ok) {
      if (lane == 0 && !*abort_flag) record_timeout(p.status, KID_GEMM_SMALL, 3);
      *abort_flag = 1;
    }
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kSmallTmemCols);
  }
}

// ---------------------------------------------------------------- host side

namespace {
struct SmallLayout {
  size_t qx, sx, accum, counters, zeroed, total;
};

// ntiles: the 128-row W_q tiles of every product of the launch
SmallLayout small_layout(ql_scheme s, int64_t M, int64_t ntiles, int64_t K) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  const int ntok = M <= 16 ? 16 : 32;
  // The region that must be zero when a call starts comes first: the arrival
  // counters, then partial-sum slot 0 of every tile (the atomic-sum slot);
  // slot 1 (parked partials, always written before they are read) follows.
  const size_t slot_bytes = (size_t)ntiles * ntok * 128 * 4;
  SmallLayout L;
  L.counters = 0;
  L.accum = up((size_t)ntiles * 4);
  L.zeroed = L.accum + slot_bytes;
  L.qx = L.accum + up(kSmallSlots * slot_bytes);
  L.sx = L.qx + up((size_t)(M * K));
  L.total = L.sx + up((size_t)M * (s == QL_FP8_E4M3_BLOCK128 ? K / 128 : 1) * 4);
  return L;
}

int64_t small_tiles(const int64_t* Ns, int count) {
  int64_t t = 0;
  for (int j = 0; j < count; ++j) t += (Ns[j] + 127) / 128;
  return t;
}
}  // namespace

size_t gemm_small_group_workspace_bytes(ql_scheme scheme, int64_t M, const int64_t* Ns, int count, int64_t K) {
  return small_layout(scheme, M, small_tiles(Ns, count), K).total;
}

size_t gemm_small_workspace_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K, int num_sms) {
  (void)num_sms;
  return gemm_small_group_workspace_bytes(scheme, M, &N, 1, K);
}

size_t gemm_small_zeroed_bytes(ql_scheme scheme, int64_t M, int64_t N, int64_t K, int num_sms) {
  (void)num_sms;
  // the GEMV routes (up to four tokens; five to eight on small weights) do
  // not touch the workspace
  if (K <= gemv_max_k_tokens(M) || gemv_token_halves_pay(M, K, &N, 1)) return 0;
  return small_layout(scheme, M, (N + 127) / 128, K).zeroed;
}

template <ql_scheme S, int NTOK>
static cudaError_t launch_small_t(const SmallParams& p, const SmallMapsW& tw, const CUtensorMap& tx,
                                  int grid, cudaStream_t st) {
  using Cfg = SmallCfg<NTOK>;
  cudaError_t e = ensure_smem<gemm_small_kernel<S, NTOK>>(Cfg::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSmallThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_small_kernel<S, NTOK>, tw, tx, p);
}

cudaError_t launch_gemm_small_group(ql_scheme scheme, const uint16_t* x, const ql_gemm_problem* probs, int count,
                                    int64_t M, int64_t K, void* workspace, size_t ws_bytes, const ql_debug* dbg,
                                    int num_sms, DevStatus* status, cudaStream_t st, const uint8_t* pre_qx,
                                    const float* pre_sx) {
  if (count < 1 || count > kSmallMaxGroup || (dbg && count != 1)) return cudaErrorInvalidValue;
  int64_t Ns[kSmallMaxGroup];
  for (int j = 0; j < count; ++j) Ns[j] = probs[j].N;
  const int64_t ntiles = small_tiles(Ns, count);
  const SmallLayout L = small_layout(scheme, M, ntiles, K);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const uint8_t* qx = pre_qx;
  const float* sx = pre_sx;
  cudaError_t e = cudaSuccess;
  if (!pre_qx) {
    // Up to four tokens: the GEMV kernel carries them on its MMA's B columns
    // with the activation quantization fused, at the weight traffic of one
    // token and without the split-K reduction (the workspace is not used).
    if (K <= gemv_max_k_tokens(M)) {
      if (count == 1) return launch_gemv(scheme, x, probs[0].wq, probs[0].sw, M, probs[0].N, K, probs[0].y, dbg,
                                         num_sms, status, st);
      ql_gemv_problem g[kSmallMaxGroup];
      for (int j = 0; j < count; ++j) g[j] = ql_gemv_problem{x, nullptr, nullptr, probs[j].wq, probs[j].sw,
                                                              probs[j].y, probs[j].N};
      return launch_gemv_grouped(scheme, g, count, M, K, num_sms, status, st);
    }
    // Five to eight tokens on small weights: the same kernel, each product
    // as two of four tokens or fewer on the same weights.
    if (!dbg && gemv_token_halves_pay(M, K, Ns, count))
      return launch_gemv_token_halves(scheme, x, probs, count, M, K, num_sms, status, st);
    if (ws_bytes < L.total) return cudaErrorInvalidValue;
    uint8_t* wqx = ws + L.qx;
    float* wsx = reinterpret_cast<float*>(ws + L.sx);
    if ((e = launch_quantize_act(scheme, x, M, K, wqx, wsx, st)) != cudaSuccess) return e;
    qx = wqx;
    sx = wsx;
  } else if (ws_bytes < L.total) {
    return cudaErrorInvalidValue;
  }

  SmallParams p;
  p.sx = sx;
  p.nprob = count;
  p.M = (int)M;
  p.K = (int)K;
  SmallMapsW tw;
  memset(&tw, 0, sizeof(tw));
  int t = 0;
  for (int j = 0; j < kSmallMaxGroup; ++j) {
    if (j < count) {
      p.sw[j] = probs[j].sw;
      p.y[j] = probs[j].y;
      p.N[j] = (int)probs[j].N;
      p.t0[j] = t;
      t += (int)((probs[j].N + 127) / 128);
      if ((e = make_tmap_u8_sw128(&tw.m[j], probs[j].wq, (uint64_t)K, (uint64_t)probs[j].N, (uint64_t)K, 128,
                                  128)) != cudaSuccess)
        return e;
    } else {
      p.sw[j] = nullptr;
      p.y[j] = nullptr;
      p.N[j] = 0;
      p.t0[j] = INT_MAX;
    }
  }
  p.t0[kSmallMaxGroup] = INT_MAX;
  p.ntn = t;
  p.nkb = (int)((K + 127) / 128);
  p.units = p.ntn * p.nkb;
  p.accum = ws + L.accum;
  p.counters = reinterpret_cast<unsigned*>(ws + L.counters);
  p.acc_i32 = dbg ? dbg->acc_i32 : nullptr;
  p.acc_f32 = dbg ? dbg->acc_f32 : nullptr;
  p.status = status;
  const int ntok = M <= 16 ? 16 : 32;
  CUtensorMap tx;
  if ((e = make_tmap_u8_sw128(&tx, qx, (uint64_t)K, (uint64_t)M, (uint64_t)K, 128, (uint32_t)ntok)) !=
      cudaSuccess)
    return e;
  const int grid = (int)std::min<int64_t>(p.units, num_sms);
  switch (scheme) {
    case QL_W8A8_INT8_ROW:
      e = ntok == 16 ? launch_small_t<QL_W8A8_INT8_ROW, 16>(p, tw, tx, grid, st)
                     : launch_small_t<QL_W8A8_INT8_ROW, 32>(p, tw, tx, grid, st);
      break;
    case QL_FP8_E4M3_ROW:
      e = ntok == 16 ? launch_small_t<QL_FP8_E4M3_ROW, 16>(p, tw, tx, grid, st)
                     : launch_small_t<QL_FP8_E4M3_ROW, 32>(p, tw, tx, grid, st);
      break;
    default:
      e = ntok == 16 ? launch_small_t<QL_FP8_E4M3_BLOCK128, 16>(p, tw, tx, grid, st)
                     : launch_small_t<QL_FP8_E4M3_BLOCK128, 32>(p, tw, tx, grid, st);
  }
  if (e != cudaSuccess) return e;
  if (dbg && !pre_qx && (dbg->qx || dbg->sx)) {
    // debug capture of the quantized tokens (stream-ordered device copies)
    if (dbg->qx && (e = cudaMemcpyAsync(dbg->qx, qx, (size_t)(M * K), cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
      return e;
    const size_t sx_bytes = (size_t)M * (scheme == QL_FP8_E4M3_BLOCK128 ? K / 128 : 1) * 4;
    if (dbg->sx && (e = cudaMemcpyAsync(dbg->sx, sx, sx_bytes, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm_small(ql_scheme scheme, const uint16_t* x, const void* wq,
                              const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                              void* workspace, size_t ws_bytes, const ql_debug* dbg, int num_sms,
                              DevStatus* status, cudaStream_t st, const uint8_t* pre_qx,
                              const float* pre_sx) {
  const ql_gemm_problem one{wq, sw, y, nullptr, nullptr, N};
  return launch_gemm_small_group(scheme, x, &one, 1, M, K, workspace, ws_bytes, dbg, num_sms, status, st, pre_qx,
                                 pre_sx);
}

}  // namespace ql
