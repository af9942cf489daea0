// ql_gemm.cu -- large-M product on pre-quantized activations, tcgen05 + TMA.
//
// "Llama 3.1 8B Instruct W8A8", "Loading": larger batches quantize the
// activations to int8 per token and accumulate the int8 products in int32.
// "Qwen3 8B FP8", "Loading": larger batches quantize them to E4M3 in groups of
// 128 along K and apply the block scales.  Here:
//   acc[m,n] = sum_k q_x[m,k] q_w[n,k]       tcgen05.mma kind::i8  -> s32 TMEM
//                                            tcgen05.mma kind::f8f6f4 (E4M3) -> f32 TMEM
//   y[m,n]   = bf16(((f32)acc * s_x[m]) * s_w[n])                (row schemes)
//   y[m,n]   = bf16(sum_kb P_kb[m,n] * s_x[m,kb] * s_w[n/128,kb])  (block scheme:
//              each 128-deep partial P_kb gets its own TMEM buffer and is
//              promoted into f32 registers by the epilogue warps)
//
// Persistent CTAs (one per SM), 128 x BN output tiles, warp roles:
//   warp 0      TMA producer: A = q_x [128 x 128 B] and B = W_q [BN x 128 B]
//               tiles into a 4..6-stage shared-memory ring (128-byte swizzle)
//   warp 1      TMEM allocation and the single MMA-issuing thread: 4 MMAs of
//               K = 32 per stage, tcgen05.commit releases the stage
//   warps 2..9  epilogue: tcgen05.ld from TMEM, scales, bf16, global stores;
//               two TMEM accumulators (or per-K-block buffers) let the
//               epilogue of one tile overlap the MMAs of the next
// Launched with programmatic dependent launch: the W tiles of the first two
// stages are requested before the grid dependency wait (they do not depend on
// the preceding kernel), q_x, s_x and y only after it.
// Every mbarrier wait is bounded; on a timeout the kernel records it, drains
// its own copies and MMAs, frees TMEM and returns.
#include <climits>
#include <cstring>

#include "ql_tc.cuh"
#include "ql_internal.h"

namespace ql {

// 32 lanes x 16 consecutive 32-bit TMEM columns (the narrower load keeps
// the 256-column block epilogue's 128 running sums in registers).
namespace tc {
QL_DEVINL void ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
}  // namespace tc

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;  // bytes of K per stage: one 128-byte swizzle row
constexpr int kGemmEpiWarps = 8;
constexpr int kGemmThreads = 64 + kGemmEpiWarps * 32;
constexpr int kTmemCols = 512;
constexpr int kGemmSmemBudget = 200 * 1024;
constexpr int kGemmEarlyStages = 2;  // W tiles requested before the grid dependency wait

// A launch runs 1 to kGemmMaxGroup products that read the same q_x (e.g. a
// layer's q, k and v projections): product j owns tiles [t0[j], t0[j+1]).
constexpr int kGemmMaxGroup = QL_GEMM_MAX_GROUP;

struct GemmParams {
  const float* sx;
  const float* sw[kGemmMaxGroup];
  uint16_t* y[kGemmMaxGroup];
  int N[kGemmMaxGroup];
  int t0[kGemmMaxGroup + 1];  // first tile of each product; INT_MAX past the last
  int nprob;
  int M, K;
  int mt, ntiles, nkb;  // tiles along M, tiles in all, K blocks of 128
  int split;        // K parts per tile (1 = whole tiles; 2, or up to 8 for 128-wide block tiles)
  float* parts;     // split > 1: partial sums, [part][tile][warp][column / 4][lane][4]
  uint32_t* counters;  // split > 1: [tiles] arrivals per tile, zero between calls
  int32_t* acc_i32;
  float* acc_f32;
  uint8_t* qy[kGemmMaxGroup];  // block scheme: E4M3 codes of each y [M,N] for the product that reads it next
  float* sy[kGemmMaxGroup];    // and their scales [M, N/128] (kQ launches)
  DevStatus* status;
};

// The W_q tensor maps of the products (kernel parameters: read by TMA from
// the parameter space).
struct GemmMapsB {
  CUtensorMap m[kGemmMaxGroup];
};

// The product of tile t and t's index inside it, by constant-index selects
// (a dynamic index would copy the parameter arrays to local memory).
struct ProdView {
  const float* sw;
  uint16_t* y;
  int N, tl, j;
};
QL_DEVINL uint8_t* qy_of(const GemmParams& p, int j) {
  return j == 0 ? p.qy[0] : j == 1 ? p.qy[1] : j == 2 ? p.qy[2] : p.qy[3];
}
QL_DEVINL float* sy_of(const GemmParams& p, int j) {
  return j == 0 ? p.sy[0] : j == 1 ? p.sy[1] : j == 2 ? p.sy[2] : p.sy[3];
}
QL_DEVINL ProdView prod_of(const GemmParams& p, int t) {
  const int j = (t >= p.t0[1]) + (t >= p.t0[2]) + (t >= p.t0[3]);
  ProdView v;
  v.j = j;
  v.sw = j == 0 ? p.sw[0] : j == 1 ? p.sw[1] : j == 2 ? p.sw[2] : p.sw[3];
  v.y = j == 0 ? p.y[0] : j == 1 ? p.y[1] : j == 2 ? p.y[2] : p.y[3];
  v.N = j == 0 ? p.N[0] : j == 1 ? p.N[1] : j == 2 ? p.N[2] : p.N[3];
  v.tl = t - (j == 0 ? 0 : j == 1 ? p.t0[1] : j == 2 ? p.t0[2] : p.t0[3]);
  return v;
}
QL_DEVINL const CUtensorMap* map_of(const GemmMapsB& b, int j) {
  return j == 0 ? &b.m[0] : j == 1 ? &b.m[1] : j == 2 ? &b.m[2] : &b.m[3];
}

static_assert(kGemmMaxGroup == 4, "prod_of and map_of select among four products");
constexpr uint32_t kGemmEpiBar = 1;  // named barrier of the epilogue warps

// OR vote over the epilogue warps that doubles as their barrier.
QL_DEVINL bool gemm_epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(kGemmEpiBar), "r"(kGemmEpiWarps * 32)
      : "memory");
  return r != 0;
}



// The epilogue passes its bf16 rows through a 32 x 32 shared-memory box per
// warp so that its global stores are row-contiguous.  kBlock: the block
// scheme's ring budget (its per-K-block promotion holds TMEM buffers longer).
template <int BN, bool kBlock>
struct GemmCfg {
  static constexpr int kStageA = kGemmBM * kGemmBK;
  static constexpr int kStageB = BN * kGemmBK;
  static constexpr int kStage = kStageA + kStageB;
  static constexpr int kBudget = kBlock ? 192 * 1024 : kGemmSmemBudget;
  static constexpr int kStages = (kBudget / kStage) > 8 ? 8 : (kBudget / kStage);
  static constexpr int kRing = kStages * kStage;
  static constexpr int kBox = 32 * 32 * 2;                             // 32 x 32 bf16
  static constexpr int kStaging = kGemmEpiWarps * kBox;  // one box per warp
  static constexpr int kBufCols = BN <= 128 ? 128 : 256;  // TMEM columns per accumulator
  static constexpr int kBufs = kTmemCols / kBufCols;
  static constexpr int kHalf = BN / 2;                    // columns per epilogue warp
  static constexpr int kRed = kGemmEpiWarps * 32 * 4;  // per-lane group maxima (output quantization)
  static constexpr int kSmem = kRing + kStaging + kRed + 1024 + 256;
  static_assert(BN % 32 == 0 && BN <= 256, "tile N");
  static_assert(kStage % 1024 == 0, "stages must stay 1024-byte aligned");
};

QL_DEVINL uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// Store W (16 or 32) consecutive bf16 outputs of row m starting at column n.
template <int W>
QL_DEVINL void store_row(uint16_t* __restrict__ y, int64_t m, int n, int N, const float* v) {
  uint16_t* dst = y + m * (int64_t)N + n;
  if (n + W <= N && (N & 7) == 0) {
#pragma unroll
    for (int q = 0; q < W / 8; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = (uint32_t)f32_to_bf16_rn(v[8 * q + 2 * j]) |
               ((uint32_t)f32_to_bf16_rn(v[8 * q + 2 * j + 1]) << 16);
      reinterpret_cast<uint4*>(dst)[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < W; ++j)
      if (n + j < N) dst[j] = f32_to_bf16_rn(v[j]);
  }
}

// Each lane holds one row of 32 bf16 values (w: 16 packed pairs); stored as
// is, every warp store would touch 32 rows.  The warp writes its 32 x 32 box
// to shared memory (row r's 16-byte chunk k at slot k ^ ((r / 2) % 4): one
// bank pass per 8 rows) and reads it back as 8 rows x 4 chunks, so that each
// global store instruction writes 8 contiguous 64-byte row pieces.  Rows
// past M are not written; the caller keeps the 32 columns inside N, N % 8 == 0.
QL_DEVINL void store_box32(uint8_t* box, int lane, const uint32_t (&w)[16], uint16_t* __restrict__ y,
                           int mrow, int ncol, int M, int N) {
  __syncwarp();  // the box's previous reads are done
#pragma unroll
  for (int k = 0; k < 4; ++k)
    *reinterpret_cast<uint4*>(box + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)) =
        make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  __syncwarp();
  const int k = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = 8 * i + (lane >> 2);
    const uint4 v = *reinterpret_cast<const uint4*>(box + rr * 64 + ((k ^ ((rr >> 1) & 3)) << 4));
    if (mrow + rr < M) *reinterpret_cast<uint4*>(y + (int64_t)(mrow + rr) * N + ncol + k * 8) = v;
  }
}

// kQ (block scheme only): the epilogue also writes y's E4M3 codes and scales.
template <ql_scheme S, int BN, bool kQ = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ GemmMapsB tmB,
                const GemmParams p) {
  constexpr bool kInt8 = S == QL_W8A8_INT8_ROW;
  constexpr bool kBlock = S == QL_FP8_E4M3_BLOCK128;
  using Cfg = GemmCfg<BN, kBlock>;
  constexpr uint32_t kIdesc = tc::idesc(kInt8, kGemmBM, BN);
  constexpr int kStages = Cfg::kStages;
  constexpr int kBufs = Cfg::kBufs;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = align1024(smem_raw);
  uint8_t* staging = ring + Cfg::kRing;  // 1024-byte aligned (stages are)
  float* red = reinterpret_cast<float*>(staging + Cfg::kStaging);
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + Cfg::kStaging + Cfg::kRed);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + kBufs;
  uint64_t* mma_done = tempty + kBufs;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* last_flag = abort_flag + 1;  // split tiles: this CTA adds the last part

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.ntiles;
  // this CTA's work items b, b + G, ... as (tile, K blocks [lo, hi)): item i
  // is K range i % split of tile i / split; fn returns false to stop
  const int nitems = ntiles * p.split;
  auto for_each_item = [&](auto&& fn) {
    for (int i = blockIdx.x; i < nitems; i += gridDim.x) {
      const int t = i / p.split, r = i - t * p.split;
      if (!fn(t, (int)(((int64_t)r * p.nkb) / p.split), (int)(((int64_t)(r + 1) * p.nkb) / p.split))) return;
    }
  };

  if (threadIdx.x == 0) {
    tc::launch_dependents();  // the next kernel's CTAs may start as SMs free up
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kGemmEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tc::prefetch_tmap(&tmA);
    for (int j = 0; j < p.nprob; ++j) tc::prefetch_tmap(map_of(tmB, j));
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_a = l2_policy_evict_last();   // q_x: re-read by every N tile
      const uint64_t pol_b = l2_policy_evict_first();  // W_q: read by the few M tiles at once
      // The kernel is launched with programmatic dependent launch.  The W
      // tiles of the first stages do not depend on the preceding kernel (the
      // quantization that writes q_x and s_x): they are requested before the
      // grid dependency wait, the q_x tiles that complete those stages after
      // it.  Only two stages go out early: more would queue the preceding
      // kernel's own loads behind this kernel's weight reads.
      uint32_t pre = 0;
      for_each_item([&](int t, int lo, int hi) -> bool {
        const ProdView pv = prod_of(p, t);
        const int n0 = (pv.tl / p.mt) * BN;
        const CUtensorMap* mb = map_of(tmB, pv.j);
        for (int kb = lo; kb < hi && pre < (uint32_t)kGemmEarlyStages; ++kb, ++pre) {
          mbar_arrive_expect_tx(&full[pre], Cfg::kStage);
          tc::tma_load_2d(ring + pre * Cfg::kStage + Cfg::kStageA, mb, kb * kGemmBK, n0, &full[pre], pol_b);
        }
        return pre < (uint32_t)kGemmEarlyStages;
      });
      tc::grid_dependency_wait();
      uint32_t it = 0;
      bool ok = true;
      for_each_item([&](int t, int lo, int hi) -> bool {
        const ProdView pv = prod_of(p, t);
        const int m0 = (pv.tl % p.mt) * kGemmBM, n0 = (pv.tl / p.mt) * BN;
        const CUtensorMap* mb = map_of(tmB, pv.j);
        for (int kb = lo; kb < hi; ++kb, ++it) {
          const int s = it % kStages;
          if (it < pre) {  // its W tile is on the way: the q_x tile completes the stage
            tc::tma_load_2d(ring + s * Cfg::kStage, &tmA, kb * kGemmBK, m0, &full[s], pol_a);
            continue;
          }
          if (it >= (uint32_t)kStages &&
              !mbar_wait_bounded(&empty[s], ((it / kStages) - 1) & 1, abort_flag)) {
            ok = false;
            return false;
          }
          uint8_t* st = ring + s * Cfg::kStage;
          mbar_arrive_expect_tx(&full[s], Cfg::kStage);
          tc::tma_load_2d(st, &tmA, kb * kGemmBK, m0, &full[s], pol_a);
          tc::tma_load_2d(st + Cfg::kStageA, mb, kb * kGemmBK, n0, &full[s], pol_b);
        }
        return true;
      });
      if (!ok) {
        if (!*abort_flag) record_timeout(p.status, KID_GEMM, 1);
        *abort_flag = 1;
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (uint32_t j = it > (uint32_t)kStages ? it - kStages : 0; j < it; ++j)
        mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, jt = 0;
      bool ok = true;
      for_each_item([&](int, int lo, int hi) -> bool {
        uint32_t d = 0;
        if (!kBlock) {
          const uint32_t buf = jt % kBufs;
          if (jt >= (uint32_t)kBufs &&
              !mbar_wait_bounded(&tempty[buf], ((jt / kBufs) - 1) & 1, abort_flag)) {
            ok = false;
            return false;
          }
          tc::fence_after();
          d = tmem + buf * Cfg::kBufCols;
        }
        for (int kb = lo; kb < hi; ++kb, ++it) {
          if (kBlock) {
            const uint32_t buf = jt % kBufs;
            if (jt >= (uint32_t)kBufs &&
                !mbar_wait_bounded(&tempty[buf], ((jt / kBufs) - 1) & 1, abort_flag)) {
              ok = false;
              return false;
            }
            tc::fence_after();
            d = tmem + buf * Cfg::kBufCols;
          }
          const int s = it % kStages;
          if (!mbar_wait_bounded(&full[s], (it / kStages) & 1, abort_flag)) {
            ok = false;
            return false;
          }
          tc::fence_after();
          const uint32_t a_addr = smem_u32(ring + s * Cfg::kStage);
          const uint64_t adesc = tc::sw128_desc(a_addr);
          const uint64_t bdesc = tc::sw128_desc(a_addr + Cfg::kStageA);
#pragma unroll
          for (int k = 0; k < kGemmBK / 32; ++k)
            tc::mma<kInt8>(d, adesc + 2 * k, bdesc + 2 * k, kIdesc,
                           kBlock ? (k != 0) : (kb != lo || k != 0));
          tc::commit(&empty[s]);  // the stage is free once these MMAs have read it
          if (kBlock) {
            tc::commit(&tfull[jt % kBufs]);
            ++jt;
          }
        }
        if (!kBlock) {
          tc::commit(&tfull[jt % kBufs]);
          ++jt;
        }
        return true;
      });
      if (!ok) {
        if (!*abort_flag) record_timeout(p.status, KID_GEMM, 2);
        *abort_flag = 1;
      }
      tc::commit(mma_done);  // every MMA of this CTA has finished when this completes
      mbar_wait_bounded(mma_done, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int h = ew >> 2;    // which half of the tile's columns
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int KB = p.K / 128;
    tc::grid_dependency_wait();  // s_x (and y's previous readers) belong to the preceding kernels
    uint32_t jt = 0;
    bool ok = true;
    for_each_item([&](int t, int lo, int hi) -> bool {
      const ProdView pv = prod_of(p, t);
      const int N = pv.N;
      uint16_t* const Y = pv.y;
      const float* const SW = pv.sw;
      const int m0 = (pv.tl % p.mt) * kGemmBM, n0 = (pv.tl / p.mt) * BN;
      const int m = m0 + q * 32 + lane;
      const bool live_m = m < p.M;
      const int c0 = h * Cfg::kHalf;  // first column of this warp inside the tile
      if constexpr (!kBlock) {
        // The scales do not depend on the MMAs: their L2 latency overlaps the
        // wait for the accumulator.  Lane j holds s_w of column 32 c + j of
        // this warp's chunk c; the chunk's lanes share them by shuffles.
        constexpr int kChunks = (Cfg::kHalf + 31) / 32;
        const float sxm = live_m ? __ldg(p.sx + m) : 0.0f;
        float swl[kChunks];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int n = n0 + c0 + c * 32 + lane;
          swl[c] = c * 32 + lane < Cfg::kHalf && n < N ? __ldg(SW + n) : 0.0f;
        }
        const bool whole = p.split == 1;
        const uint32_t buf = jt % kBufs;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[buf], (jt / kBufs) & 1, abort_flag));
        // a split tile meets the other epilogue warps at barriers below: all vote first
        if (!whole) {
          if (gemm_epi_any(!ok)) return false;
        } else if (!ok) {
          return false;
        }
        tc::fence_after();
        // scales, debug copies and bf16 stores of W raw accumulators r (s32 or
        // f32 bits) of this thread's row from column col on (W = 32, or a
        // 16-column tail for 160- and 224-wide tiles)
        auto finish = [&](int col, float swc, const uint32_t* r, auto wtag) {
          constexpr int W = decltype(wtag)::value;
          const int n = n0 + col;
          float v[W];
#pragma unroll
          for (int j = 0; j < W; ++j) {
            const float a = kInt8 ? __int2float_rn((int)r[j]) : __uint_as_float(r[j]);
            v[j] = __fmul_rn(__fmul_rn(a, sxm), __shfl_sync(0xffffffffu, swc, j));
          }
          if (live_m && n < N) {
            if (p.acc_i32 || p.acc_f32) {
#pragma unroll
              for (int j = 0; j < W; ++j) {
                if (n + j < N) {
                  if (kInt8 && p.acc_i32) p.acc_i32[(int64_t)m * N + n + j] = (int)r[j];
                  if (!kInt8 && p.acc_f32) p.acc_f32[(int64_t)m * N + n + j] = __uint_as_float(r[j]);
                }
              }
            }
          }
          // whole 32-column chunks inside N leave through the box (uniform per warp)
          if (W == 32 && n + 32 <= N && (N & 7) == 0) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              w[j] = (uint32_t)f32_to_bf16_rn(v[2 * j]) | ((uint32_t)f32_to_bf16_rn(v[2 * j + 1]) << 16);
            store_box32(staging + ew * Cfg::kBox, lane, w, Y, m0 + q * 32, n, p.M, N);
          } else if (live_m && n < N) {
            store_row<W>(Y, m, n, N, v);
          }
        };
        // K split: this item's part of the tile's K blocks (lo = floor(part nkb / split)),
        // parked raw in its slab laid out the way the warps hold it (lane-minor:
        // each warp store writes 512 contiguous bytes)
        const int part = whole ? 0 : (int)(((int64_t)lo * p.split + p.nkb - 1) / p.nkb);
        auto slab = [&](int hf) {
          return reinterpret_cast<uint4*>(p.parts) +
                 ((int64_t)(hf * ntiles + t) * kGemmEpiWarps + ew) * (Cfg::kHalf / 4) * 32 + lane;
        };
        auto chunk = [&](int col, float swc, auto wtag) {
          constexpr int W = decltype(wtag)::value;
          uint32_t r[W];
          if constexpr (W == 32)
            tc::ld32(tmem + lane_base + buf * Cfg::kBufCols + col, r);
          else
            tc::ld16(tmem + lane_base + buf * Cfg::kBufCols + col, r);
          tc::ld_wait();
          if (whole) {
            finish(col, swc, r, wtag);
          } else {
            uint4* mine = slab(part);
#pragma unroll
            for (int i = 0; i < W / 4; ++i)
              __stcg(mine + ((col - c0) / 4 + i) * 32, make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]));
          }
        };
#pragma unroll
        for (int c = 0; c < Cfg::kHalf / 32; ++c) chunk(c0 + c * 32, swl[c], std::integral_constant<int, 32>{});
        if constexpr (Cfg::kHalf % 32 != 0)
          chunk(c0 + Cfg::kHalf / 32 * 32, swl[kChunks - 1], std::integral_constant<int, 16>{});
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        ++jt;
        if (!whole) {
          __threadfence();
          named_bar_sync(kGemmEpiBar, kGemmEpiWarps * 32);
          if (ew == 0 && lane == 0) {
            const unsigned old = atomicAdd(p.counters + t, 1u);
            *last_flag = old == (unsigned)(p.split - 1);
          }
          named_bar_sync(kGemmEpiBar, kGemmEpiWarps * 32);
          if (!*last_flag) return true;
          __threadfence();
          // the last part to arrive adds every part's raw sums in part order
          // (s32 adds are exact; f32 adds in a fixed order give the same bits
          // whichever part arrived last) and finishes the tile
          auto merged = [&](int col, float swc, auto wtag) {
            constexpr int W = decltype(wtag)::value;
            const int v0 = (col - c0) / 4;
            uint32_t r[W];
            {
              const uint4* b0 = slab(0);
#pragma unroll
              for (int i = 0; i < W / 4; ++i) {
                const uint4 x = __ldcg(b0 + (v0 + i) * 32);
                r[4 * i] = x.x, r[4 * i + 1] = x.y, r[4 * i + 2] = x.z, r[4 * i + 3] = x.w;
              }
            }
            for (int hf = 1; hf < p.split; ++hf) {
              const uint4* o = slab(hf);
#pragma unroll
              for (int i = 0; i < W / 4; ++i) {
                const uint4 x = __ldcg(o + (v0 + i) * 32);
                const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  r[4 * i + k] = kInt8 ? r[4 * i + k] + xv[k]
                                       : __float_as_uint(__fadd_rn(__uint_as_float(r[4 * i + k]), __uint_as_float(xv[k])));
              }
            }
            finish(col, swc, r, wtag);
          };
#pragma unroll
          for (int c = 0; c < Cfg::kHalf / 32; ++c) merged(c0 + c * 32, swl[c], std::integral_constant<int, 32>{});
          if constexpr (Cfg::kHalf % 32 != 0)
            merged(c0 + Cfg::kHalf / 32 * 32, swl[kChunks - 1], std::integral_constant<int, 16>{});
          if (ew == 0 && lane == 0) p.counters[t] = 0u;  // every part has arrived
        }
      } else {
        // block scheme: promote each 128-deep partial into f32 registers
        static_assert(BN == 128 || BN == 256, "block tiles are 128 or 256 wide");
        const int ncol = n0 + c0;
        const bool live_n = ncol < N;
        const int nbw = ncol >> 7;  // this warp's columns lie in one 128-row weight block
        // running sums as pairs: one packed f32x2 FMA (two IEEE fmas) per pair
        float2 acc[Cfg::kHalf / 2];
#pragma unroll
        for (int j = 0; j < Cfg::kHalf / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
        // scales of K block kb+1 are loaded while the MMAs of block kb run
        const bool live = live_m && live_n;
        float sx_next = live ? __ldg(p.sx + (int64_t)m * KB + lo) : 0.0f;
        float sw_next = live ? __ldg(SW + (int64_t)nbw * KB + lo) : 0.0f;
        for (int kb = lo; kb < hi; ++kb) {
          const float scale = sx_next * sw_next;
          if (live && kb + 1 < hi) {
            sx_next = __ldg(p.sx + (int64_t)m * KB + kb + 1);
            sw_next = __ldg(SW + (int64_t)nbw * KB + kb + 1);
          }
          const uint32_t buf = jt % kBufs;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[buf], (jt / kBufs) & 1, abort_flag));
          if (!ok) break;
          tc::fence_after();
          // 64 columns: 32-column loads; 128 columns: 16-column loads (registers)
          constexpr int kW = Cfg::kHalf == 64 ? 32 : 16;
          constexpr int kChunks = Cfg::kHalf / kW;
          const uint32_t tbase = tmem + lane_base + buf * Cfg::kBufCols + c0;
          auto ldw = [&](int c, uint32_t (&r)[kW]) {
            if constexpr (kW == 32)
              tc::ld32(tbase + c * kW, r);
            else
              tc::ld16(tbase + c * kW, r);
          };
          // software pipeline: chunk c + 1 is loaded while chunk c is promoted
          uint32_t rb[2][kW];
          ldw(0, rb[0]);
          tc::ld_wait();
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            if (c + 1 < kChunks) ldw(c + 1, rb[(c + 1) & 1]);
#pragma unroll
            for (int j = 0; j < kW / 2; ++j)
              acc[(c * kW) / 2 + j] = __ffma2_rn(make_float2(__uint_as_float(rb[c & 1][2 * j]), __uint_as_float(rb[c & 1][2 * j + 1])),
                                                 make_float2(scale, scale), acc[(c * kW) / 2 + j]);
            if (c + 1 < kChunks) tc::ld_wait();
          }
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          ++jt;
        }
        if (p.split == 1) {
          // the output quantization of 128-wide tiles meets the partner warp
          // at a barrier: every warp votes first, so that all leave together
          if (kQ && Cfg::kHalf < 128) {
            if (gemm_epi_any(!ok)) return false;
          } else if (!ok) {
            return false;
          }
        } else {
          // Split tile: every epilogue warp reaches the votes and barriers
          // below, so they leave together if any of them gave up a wait.
          if (gemm_epi_any(!ok)) return false;
          // Each K half parks its sums in its own slab, laid out the way the
          // warps hold them (lane-minor, so each warp store writes 512
          // contiguous bytes; stored as [M, N] rows, every store touched 32
          // rows), and the CTA that arrives second reads the other half's and
          // adds the two (f32 addition commutes: the same bits in either order
          // of arrival) and writes y.  (Adding the halves with L2 reductions
          // measured slower than the work saved.)
          // this item's part of the tile's K blocks: lo = floor(part nkb / split)
          const int half = (int)(((int64_t)lo * p.split + p.nkb - 1) / p.nkb);
          constexpr int kV = Cfg::kHalf / 4;     // float4 per thread
          auto slot = [&](int hf) {
            return reinterpret_cast<float4*>(p.parts) +
                   ((int64_t)(hf * ntiles + t) * kGemmEpiWarps + ew) * kV * 32 + lane;
          };
          {
            float4* mine = slot(half);
#pragma unroll
            for (int j = 0; j < kV; ++j)
              __stcg(mine + j * 32, make_float4(acc[2 * j].x, acc[2 * j].y, acc[2 * j + 1].x, acc[2 * j + 1].y));
          }
          __threadfence();
          named_bar_sync(kGemmEpiBar, kGemmEpiWarps * 32);
          if (ew == 0 && lane == 0) {
            const unsigned old = atomicAdd(p.counters + t, 1u);
            *last_flag = old == (unsigned)(p.split - 1);
          }
          named_bar_sync(kGemmEpiBar, kGemmEpiWarps * 32);
          if (!*last_flag) return true;
          __threadfence();
          if (p.split == 2) {
            const float4* other = slot(1 - half);
            // eight 16-byte loads in flight at a time (the 128 running sums
            // leave no registers for more)
#pragma unroll
            for (int j0 = 0; j0 < kV; j0 += 8) {
              float4 v[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) v[j] = __ldcg(other + (j0 + j) * 32);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                acc[2 * (j0 + j)] = make_float2(acc[2 * (j0 + j)].x + v[j].x, acc[2 * (j0 + j)].y + v[j].y);
                acc[2 * (j0 + j) + 1] =
                    make_float2(acc[2 * (j0 + j) + 1].x + v[j].z, acc[2 * (j0 + j) + 1].y + v[j].w);
              }
              asm volatile("" ::: "memory");
            }
          } else if constexpr (BN == 128) {
            // more parts (128-wide tiles only): summed in part order 0, 1, ..., split - 1 whichever
            // arrives last (this CTA's own part from its registers), so the
            // bits do not depend on the order of arrival
#pragma unroll
            for (int j0 = 0; j0 < kV; j0 += 4) {
              float4 tot[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) tot[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              for (int hf = 0; hf < p.split; ++hf) {
                float4 v[4];
                if (hf == half) {
#pragma unroll
                  for (int j = 0; j < 4; ++j)
                    v[j] = make_float4(acc[2 * (j0 + j)].x, acc[2 * (j0 + j)].y, acc[2 * (j0 + j) + 1].x,
                                       acc[2 * (j0 + j) + 1].y);
                } else {
                  const float4* o = slot(hf);
#pragma unroll
                  for (int j = 0; j < 4; ++j) v[j] = __ldcg(o + (j0 + j) * 32);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  tot[j] = make_float4(tot[j].x + v[j].x, tot[j].y + v[j].y, tot[j].z + v[j].z, tot[j].w + v[j].w);
              }
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                acc[2 * (j0 + j)] = make_float2(tot[j].x, tot[j].y);
                acc[2 * (j0 + j) + 1] = make_float2(tot[j].z, tot[j].w);
              }
              asm volatile("" ::: "memory");
            }
          }
          if (ew == 0 && lane == 0) p.counters[t] = 0u;  // every part has arrived
        }
        const int mrow = m0 + q * 32;
        if constexpr (kQ) {
          // The output's own quantization for the product that reads it next
          // (E4M3, one scale per token per 128 outputs: the group of 128
          // columns is this thread's row here, split over the warps of the
          // two column halves on 128-wide tiles).  The codes are those of the
          // bf16 y: s = absmax / 448 (one IEEE division), code = E4M3(y / s).
          // Rounding to bf16 is monotonic in |v|, so the largest |bf16(v)| of
          // the group is bf16(max |v|).
          float a = 0.0f;
#pragma unroll
          for (int j = 0; j < Cfg::kHalf / 2; ++j) a = fmaxf(a, fmaxf(fabsf(acc[j].x), fabsf(acc[j].y)));
          a = bf16_lo(f32_to_bf16_rn(a));
          if constexpr (Cfg::kHalf < 128) {
            red[ew * 32 + lane] = a;
            named_bar_sync(kGemmEpiBar, kGemmEpiWarps * 32);
            a = fmaxf(a, red[(ew ^ 4) * 32 + lane]);
            named_bar_sync(kGemmEpiBar, kGemmEpiWarps * 32);  // red is free again
          }
          auto pack = [&](int j) {
            return (uint32_t)f32_to_bf16_rn(acc[j].x) | ((uint32_t)f32_to_bf16_rn(acc[j].y) << 16);
          };
          if (Y && live_n && mrow < p.M) {
#pragma unroll
            for (int c = 0; c < Cfg::kHalf / 32; ++c) {
              uint32_t w[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) w[j] = pack(c * 16 + j);
              store_box32(staging + ew * Cfg::kBox, lane, w, Y, mrow, ncol + c * 32, p.M, N);
            }
          }
          const float sc = a / 448.0f;
          const Divisor dv = make_divisor(sc);
          if (live_n && live_m) {
            uint8_t* qrow = qy_of(p, pv.j) + (int64_t)m * N + ncol;
#pragma unroll
            for (int c = 0; c < Cfg::kHalf / 16; ++c) {
              const uint2 q0 = quant_chunk8<false>(make_uint4(pack(8 * c), pack(8 * c + 1), pack(8 * c + 2), pack(8 * c + 3)), dv);
              const uint2 q1 = quant_chunk8<false>(make_uint4(pack(8 * c + 4), pack(8 * c + 5), pack(8 * c + 6), pack(8 * c + 7)), dv);
              *reinterpret_cast<uint4*>(qrow + c * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
            }
            if ((ncol & 127) == 0) sy_of(p, pv.j)[(int64_t)m * (N / 128) + (ncol >> 7)] = sc;
          }
        } else if (live_n && mrow < p.M) {
#pragma unroll
          for (int c = 0; c < Cfg::kHalf / 32; ++c) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              w[j] = (uint32_t)f32_to_bf16_rn(acc[c * 16 + j].x) | ((uint32_t)f32_to_bf16_rn(acc[c * 16 + j].y) << 16);
            store_box32(staging + ew * Cfg::kBox, lane, w, Y, mrow, ncol + c * 32, p.M, N);
          }
        }
      }
      return true;
    });
    if (!ok) {
      if (lane == 0 && !*abort_flag) record_timeout(p.status, KID_GEMM, 3);
      *abort_flag = 1;
    }
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

// Tile width for a launch: fill the SMs' waves best (the products of a group
// share the width; their tiles add up).
static int64_t group_tiles(int64_t mt, const int64_t* Ns, int count, int bn) {
  int64_t t = 0;
  for (int j = 0; j < count; ++j) t += mt * ((Ns[j] + bn - 1) / bn);
  return t;
}

static int pick_bn(ql_scheme s, int64_t M, const int64_t* Ns, int count, int sms) {
  const int cands_row[5] = {256, 224, 192, 160, 128};
  const int cands_blk[2] = {256, 128};
  const int* c = s == QL_FP8_E4M3_BLOCK128 ? cands_blk : cands_row;
  const int nc = s == QL_FP8_E4M3_BLOCK128 ? 2 : 5;
  const int64_t mt = (M + kGemmBM - 1) / kGemmBM;
  int64_t ncols = 0;
  for (int j = 0; j < count; ++j) ncols += Ns[j];
  int best = c[0];
  double best_eff = -1.0;
  for (int i = 0; i < nc; ++i) {
    const int64_t tiles = group_tiles(mt, Ns, count, c[i]);
    const int64_t waves = (tiles + sms - 1) / sms;
    double eff = (double)(mt * ncols) / (double)(waves * sms * (int64_t)c[i]);
    // measured: 128-wide tiles run the MMAs at ~85% of the wider tiles' rate
    // (row schemes) and ~60% for the block scheme, whose per-K-block
    // promotion costs the same per tile at either width
    if (c[i] == 128) eff *= s == QL_FP8_E4M3_BLOCK128 ? 0.6 : 0.85;
    if (c[i] == 160) eff *= 0.92;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = c[i];
    }
  }
  return best;
}

// At most half a wave of 256-wide tiles and a long K (M = 512 with N = 4096,
// K >= 8192: down_proj): each tile's K blocks are split in two halves run by
// two CTAs, which meet in the workspace (the block scheme's f32 running sums;
// the row schemes' raw s32 or f32 accumulators, added before the scales).
// Measured per K block, 256-wide tiles run at ~1.5x the 128-wide rate (block
// scheme: promote at ~1.6x), so a split 256-wide tile beats a whole 128-wide
// one once K is long enough to repay parking and re-reading the halves
// (Qwen3-8B down_proj at M = 512: 47 -> 36 us; at K = 4096 the split
// measured 2% slower than whole 128-wide tiles).  Otherwise whole tiles,
// except the block scheme's small-N rule below.
struct GemmPlan {
  int bn, split;
};

static GemmPlan plan_gemm(ql_scheme s, int64_t M, const int64_t* Ns, int count, int64_t K, int sms) {
  GemmPlan pl{pick_bn(s, M, Ns, count, sms), 1};
  const int64_t mt = (M + kGemmBM - 1) / kGemmBM;
  const int64_t tiles = group_tiles(mt, Ns, count, 256);
  const int64_t nkb = (K + kGemmBK - 1) / kGemmBK;
  if (2 * tiles <= sms && nkb >= 64) return GemmPlan{256, 2};
  if (s != QL_FP8_E4M3_BLOCK128) return pl;
  // Tiles of the chosen width that fill at most a quarter of the SMs (small
  // N, e.g. k/v at M = 512: 32 tiles of 128): split each tile's K blocks over
  // 2, 4 or 8 CTAs, as many as fit one wave, keeping >= 8 K blocks a part.
  const int64_t t_bn = group_tiles(mt, Ns, count, pl.bn);
  int split = 1;
  while (pl.bn == 128 && split < 8 && 4 * t_bn * split <= 2 * sms && t_bn * split * 2 <= sms &&
         nkb / (split * 2) >= 8)
    split *= 2;
  if (split > 1) pl.split = split;
  return pl;
}

static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// One slab of one 128 x 256 f32 tile per part per tile.
static size_t split_parts_bytes(int64_t tiles, int split) {
  return (size_t)split * tiles * kGemmBM * 256 * 4;
}

size_t gemm_group_workspace_bytes(ql_scheme s, int64_t M, const int64_t* Ns, int count, int64_t K, int sms) {
  const GemmPlan pl = plan_gemm(s, M, Ns, count, K, sms);
  if (pl.split == 1) return 0;
  const int64_t tiles = group_tiles((M + kGemmBM - 1) / kGemmBM, Ns, count, pl.bn);
  return align256(split_parts_bytes(tiles, pl.split)) + align256((size_t)tiles * 4);
}

size_t gemm_workspace_bytes(ql_scheme s, int64_t M, int64_t N, int64_t K, int sms) {
  return gemm_group_workspace_bytes(s, M, &N, 1, K, sms);
}

template <ql_scheme S, int BN, bool kQ = false>
static cudaError_t launch_gemm_t(const GemmParams& p, const CUtensorMap& a, const GemmMapsB& b,
                                 int sms, cudaStream_t st) {
  using Cfg = GemmCfg<BN, S == QL_FP8_E4M3_BLOCK128>;
  cudaError_t e = ensure_smem<gemm_kernel<S, BN, kQ>>(Cfg::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<int64_t>((int64_t)p.ntiles * p.split, sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_kernel<S, BN, kQ>, a, b, p);
}

cudaError_t launch_gemm_group(ql_scheme scheme, const void* qx, const float* sx, const ql_gemm_problem* probs,
                              int count, int64_t M, int64_t K, void* workspace, size_t ws_bytes,
                              const ql_debug* dbg, int num_sms, DevStatus* status, cudaStream_t st) {
  if (count < 1 || count > kGemmMaxGroup) return cudaErrorInvalidValue;
  // output quantization: every product of the launch or none, block scheme only
  const bool quant_out = probs[0].qy != nullptr;
  for (int j = 0; j < count; ++j) {
    if ((probs[j].qy != nullptr) != quant_out || (probs[j].sy != nullptr) != quant_out) return cudaErrorInvalidValue;
    if (!quant_out && probs[j].y == nullptr) return cudaErrorInvalidValue;
  }
  if (quant_out && scheme != QL_FP8_E4M3_BLOCK128) return cudaErrorInvalidValue;
  if (dbg && count != 1) return cudaErrorInvalidValue;
  int64_t Ns[kGemmMaxGroup];
  for (int j = 0; j < count; ++j) Ns[j] = probs[j].N;
  // the K split needs its workspace; without one, whole tiles
  GemmPlan pl = plan_gemm(scheme, M, Ns, count, K, num_sms);
  const size_t need = gemm_group_workspace_bytes(scheme, M, Ns, count, K, num_sms);
  if (pl.split > 1 && (workspace == nullptr || ws_bytes < need))
    pl = GemmPlan{pick_bn(scheme, M, Ns, count, num_sms), 1};
  const int BN = pl.bn;
  GemmParams p;
  p.sx = sx;
  p.nprob = count;
  p.M = (int)M;
  p.K = (int)K;
  p.mt = (int)((M + kGemmBM - 1) / kGemmBM);
  p.nkb = (int)((K + kGemmBK - 1) / kGemmBK);
  GemmMapsB tb;
  memset(&tb, 0, sizeof(tb));
  int t = 0;
  for (int j = 0; j < kGemmMaxGroup; ++j) {
    if (j < count) {
      p.sw[j] = probs[j].sw;
      p.y[j] = probs[j].y;
      p.qy[j] = static_cast<uint8_t*>(probs[j].qy);
      p.sy[j] = probs[j].sy;
      p.N[j] = (int)probs[j].N;
      p.t0[j] = t;
      t += p.mt * (int)((probs[j].N + BN - 1) / BN);
      cudaError_t e = make_tmap_u8_sw128(&tb.m[j], probs[j].wq, (uint64_t)K, (uint64_t)probs[j].N, (uint64_t)K,
                                         kGemmBK, (uint32_t)BN);
      if (e != cudaSuccess) return e;
    } else {
      p.sw[j] = nullptr;
      p.y[j] = nullptr;
      p.qy[j] = nullptr;
      p.sy[j] = nullptr;
      p.N[j] = 0;
      p.t0[j] = INT_MAX;
    }
  }
  p.t0[kGemmMaxGroup] = INT_MAX;
  p.ntiles = t;
  p.split = pl.split;
  p.parts = pl.split > 1 ? static_cast<float*>(workspace) : nullptr;
  p.counters = pl.split > 1 ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) +
                                                          align256(split_parts_bytes((int64_t)p.ntiles, pl.split)))
                            : nullptr;
  p.acc_i32 = dbg ? dbg->acc_i32 : nullptr;
  p.acc_f32 = dbg ? dbg->acc_f32 : nullptr;
  p.status = status;
  CUtensorMap ta;
  cudaError_t e = make_tmap_u8_sw128(&ta, qx, (uint64_t)K, (uint64_t)M, (uint64_t)K, kGemmBK, kGemmBM);
  if (e != cudaSuccess) return e;
  switch (scheme) {
    case QL_W8A8_INT8_ROW:
      if (BN == 256) return launch_gemm_t<QL_W8A8_INT8_ROW, 256>(p, ta, tb, num_sms, st);
      if (BN == 224) return launch_gemm_t<QL_W8A8_INT8_ROW, 224>(p, ta, tb, num_sms, st);
      if (BN == 192) return launch_gemm_t<QL_W8A8_INT8_ROW, 192>(p, ta, tb, num_sms, st);
      if (BN == 160) return launch_gemm_t<QL_W8A8_INT8_ROW, 160>(p, ta, tb, num_sms, st);
      return launch_gemm_t<QL_W8A8_INT8_ROW, 128>(p, ta, tb, num_sms, st);
    case QL_FP8_E4M3_ROW:
      if (BN == 256) return launch_gemm_t<QL_FP8_E4M3_ROW, 256>(p, ta, tb, num_sms, st);
      if (BN == 224) return launch_gemm_t<QL_FP8_E4M3_ROW, 224>(p, ta, tb, num_sms, st);
      if (BN == 192) return launch_gemm_t<QL_FP8_E4M3_ROW, 192>(p, ta, tb, num_sms, st);
      if (BN == 160) return launch_gemm_t<QL_FP8_E4M3_ROW, 160>(p, ta, tb, num_sms, st);
      return launch_gemm_t<QL_FP8_E4M3_ROW, 128>(p, ta, tb, num_sms, st);
    default:
      if (quant_out) {
        if (BN == 256) return launch_gemm_t<QL_FP8_E4M3_BLOCK128, 256, true>(p, ta, tb, num_sms, st);
        return launch_gemm_t<QL_FP8_E4M3_BLOCK128, 128, true>(p, ta, tb, num_sms, st);
      }
      if (BN == 256) return launch_gemm_t<QL_FP8_E4M3_BLOCK128, 256>(p, ta, tb, num_sms, st);
      return launch_gemm_t<QL_FP8_E4M3_BLOCK128, 128>(p, ta, tb, num_sms, st);
  }
}

cudaError_t launch_gemm(ql_scheme scheme, const void* qx, const float* sx, const void* wq,
                        const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace,
                        size_t ws_bytes, const ql_debug* dbg, int num_sms, DevStatus* status,
                        cudaStream_t st, uint8_t* qy, float* sy) {
  if ((qy != nullptr) != (sy != nullptr)) return cudaErrorInvalidValue;
  const ql_gemm_problem one{wq, sw, y, qy, sy, N};
  return launch_gemm_group(scheme, qx, sx, &one, 1, M, K, workspace, ws_bytes, dbg, num_sms, status, st);
}

}  // namespace ql
