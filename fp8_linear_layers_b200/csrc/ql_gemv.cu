// ql_gemv.cu -- M = 1 decode product y = (s_x s_w) . (Q(x) . W_q^T), one kernel.
//
// "Llama 3.1 8B Instruct W8A8", "Loading": a single token runs in a kernel
// that touches every weight byte once; "Qwen3 8B FP8", "Loading": the same for
// the FP8 block scheme.  The kernel is bound by the weight stream: N*K bytes
// from HBM, everything else is L2/shared-memory traffic.
//
// Design (B200):
//  * One CTA per SM; CTA b owns the contiguous output rows [b N / G,
//    (b+1) N / G), one contiguous byte range of W_q.  A producer warp streams
//    it into a shared-memory ring of whole-row stages (~32 KB bulk copies on
//    the TMA engine, the size at which one SM's copy engine runs at full HBM
//    rate), completion tracked by mbarriers.
//  * The kernel is launched with programmatic dependent launch: as each CTA
//    of this kernel exits, a CTA of the next kernel on the stream takes the
//    SM and starts streaming its own weights while the rest of this kernel
//    drains.  x (which a previous kernel may produce) is read, and y written,
//    only after the grid dependency wait; weights and weight scales are read
//    before it, so they must not be written by work still in flight on the
//    stream.  (Letting two GEMV CTAs share an SM was measured slower: the
//    block scheduler then stacks two CTAs of one kernel on some SMs.)
//  * 8 consumer warps first quantize x (fused per-token or per-128-group
//    absmax, IEEE-divided scale, correctly rounded quotients, codes) into
//    shared memory.  Until they are done the producer has only two stages in
//    flight (measured: a full ring fill from every SM at kernel start delays
//    the quantization's own x reads and instruction fetches by microseconds).
//  * The products run on the tensor cores with mma.sync: the weights are the
//    16-row A operand (16 units of the stage: rows x K segments) and x the
//    8-column B operand, so that units j and j + 8 meet x segment j and every
//    MMA keeps 16 products (512 weight bytes per s8 m16n8k32, exact; E4M3
//    converts exactly to f16 for m16n8k16 with f32 accumulation, 256 bytes
//    per instruction -- an E4M3 k32 MMA costs the same issue time for the same
//    bytes).  The k order inside each 64-byte window is permuted identically
//    for x and W so that every lane loads 16 contiguous bytes; a dot product
//    does not depend on the order.  Each warp owns a fixed range of 64-byte
//    k windows of every unit.
//  * No CTA-wide barrier per stage: each warp parks its 8 row partials in a
//    per-stage slot and counts itself in; the last warp adds the slots in a
//    fixed order, applies the scales, writes y and releases the stage.
//  * Every wait is bounded; a warp that gives up raises a CTA abort flag that
//    every other wait checks, so all roles leave without further barriers.
//  * Weight-only variant (kWO, the pages' "equivalent" numerics that never
//    round the input): the same weight stream and MMA mapping with x staged
//    as f16 (scaled by an exact power of two) instead of codes, and int8
//    weights converted exactly to f16 for the f16 MMAs; sums in f32.
#include <type_traits>

#include "ql_common.cuh"
#include "ql_internal.h"
#include "ql_tc.cuh"

namespace ql {

constexpr int kGemvWarps = 8;                  // consumer warps (a multiple of 4)
constexpr int kGemvConsumers = kGemvWarps * 32;
constexpr int kGemvThreads = kGemvConsumers + 32;
constexpr int kGemvMaxStages = 6;
constexpr int kEarlyStages = 2;                 // stages copied before x is quantized
constexpr int kGemvStageTarget = 32768;
constexpr int kGemvSmemBudget = 224 * 1024;     // one CTA per SM
constexpr int64_t kGemvStashMaxK = 16384;       // one token's bf16 x parked in shared memory up to this K
constexpr int kGemvMaxK = 32768;
constexpr int64_t kGemvMaxK2 = 16384;           // two tokens: units of at most 64 windows
constexpr int64_t kGemvMaxK4 = 8192;            // three or four tokens: stages of 8 rows
constexpr int64_t kGemvMaxKWO = 16384;          // weight-only: 2K bytes of staged x beside the ring
// Five to eight tokens run on this kernel as two products of up to four
// tokens over the same weights when the launch's weights take at most this
// many bytes.  The halves' SMs each take the weight bytes in, so a launch
// streams them twice over the SMs' ports (L2 hits arrive no faster than HBM
// reads under a full stream).  Measured on B200, M = 8 int8, per launch: a
// 4 MiB product 8.2 us against 10.3 us on the split-K kernel, 16 MiB equal
// (12.3 us), 24 MiB 15.9 against 14.4 us, 112 MiB 45 against 28.7 us.
constexpr int64_t kGemvHalvesMaxWeightBytes = 8ll << 20;
constexpr int kGemvUnits = 16;                  // units per stage (the MMA's 16 A rows)
constexpr int kGemvSwCache = 2048;              // row scales kept in shared memory
constexpr uint32_t kBarConsumers = 1;           // named barrier of the consumer warps
constexpr int kGemvMaxGroup = QL_GEMV_MAX_GROUP;  // products of one grouped launch

// One product of a launch.  A grouped launch runs up to kGemvMaxGroup
// products of the same K side by side, each on its own set of CTAs.
struct GemvProblem {
  const uint16_t* x;   // bf16 input, or (when sx is set) its codes as the producer of x wrote them
  const float* sx;     // pre-quantized input: its scales ([1] or [K/128]); null: quantize x here
  const uint8_t* wq;
  const float* sw;
  uint16_t* y;
  int64_t N;
  int M;  // tokens of this product (at most the launch's M)
};

struct GemvParams {
  GemvProblem prob[kGemvMaxGroup];
  int cta0[kGemvMaxGroup + 1];  // CTAs [cta0[j], cta0[j+1]) run product j
  int nprob;
  int64_t K;
  int M;               // tokens: 1 to 4 (extra tokens ride on the MMA's B columns); the largest product's
  int rows_per_stage;  // 2 kRs whole rows per ring stage (kRs = 1, 2 or 4: the kernel's template)
  int stage_bytes;     // R_s * K rounded up to 128
  int stages;          // ring depth
  int64_t seg_len;     // bytes per unit segment: ceil(K R_s / 8) rounded up to 128
  ql_debug dbg;
  DevStatus* status;
  int stall;  // test hook: the producer issues no copies, so every consumer wait runs out
};

struct GemvSmemLayout {
  int ring, qx, stash, sx, swc, part, bars, flags, total;
};

// Shared-memory carve-up; `sw_floats` is the number of weight scales cached,
// `xelem` the bytes per staged x element (1: codes; 2: f16 for weight-only).
__host__ __device__ inline GemvSmemLayout gemv_layout(int64_t K, int stage_bytes, int stages,
                                                      int sw_floats, int M = 1, int xelem = 1) {
  GemvSmemLayout L;
  int off = 0;
  L.ring = off;
  off += stages * stage_bytes;
  L.qx = off;  // M rows of K codes (or f16 values), each padded to whole 128-element blocks
  off += M * (int)((K + 127) / 128) * 128 * xelem;
  L.stash = off;  // one token's bf16 x, read once from global memory and quantized from here
  off += (M == 1 && K <= kGemvStashMaxK) ? (int)((K * 2 + 127) / 128 * 128) : 0;
  L.sx = off;
  off += (int)((M * (K / 128 + 1) + 31) / 32) * 128;
  L.swc = off;
  off += (sw_floats + 31) / 32 * 128;
  L.part = off;  // [stages][8 warps][8 rows] partial sums
  off += kGemvMaxStages * kGemvWarps * kGemvUnits * M * 4;
  L.bars = off;  // full[stages], empty[stages], x ready
  off += 2 * kGemvMaxStages * 8 + 8;
  L.flags = off;  // abort flag, per-stage arrival counters, block reduction scratch
  off += 16 + kGemvMaxStages * 4 + kGemvWarps * 4 * M;
  L.total = (off + 127) / 128 * 128;
  return L;
}

// Plain 16-byte shared-memory load: ordered after the barrier waits (which
// clobber memory), free to be scheduled ahead of the tensor-core instructions.
QL_DEVINL uint4 ld_s128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// D[16x8] += A[16x32] * B[32x8], s8 x s8 -> s32 (exact).
QL_DEVINL void mma_s8(uint32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                      uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x16] * B[16x8], f16 x f16 -> f32.  E4M3 codes convert to f16
// exactly and the products of two are exact in f32, so this computes what an
// E4M3 MMA does with f32 accumulation, with half the tensor instructions per
// weight byte (measured: one f16 k16 MMA costs what one E4M3 k32 MMA does).
QL_DEVINL void mma_f16(uint32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                       uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Eight f16x2 registers from 16 E4M3 codes (byte order kept).
QL_DEVINL void e4m3x16_to_f16(const uint4& v, uint32_t (&h)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    h[2 * q] = e4m3x2_to_f16x2((uint16_t)(w[q] & 0xFFFFu));
    h[2 * q + 1] = e4m3x2_to_f16x2((uint16_t)(w[q] >> 16));
  }
}

// a - b on f16x2 (exact for the integers below 2048 used here).
QL_DEVINL uint32_t sub_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Eight f16x2 registers from 16 int8 codes (byte order kept), exact.  With
// its sign bit flipped, code c reads as the unsigned byte c + 128; placed
// under the f16 exponent of 1024 (unit spacing there) it is the f16 value
// 1024 + c + 128, and subtracting 1152 leaves c.
QL_DEVINL void s8x16_to_f16(const uint4& v, uint32_t (&h)[8]) {
  const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u,
                         v.w ^ 0x80808080u};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    h[2 * q] = sub_f16x2(__byte_perm(w[q], 0x64646464u, 0x4140), 0x64806480u);
    h[2 * q + 1] = sub_f16x2(__byte_perm(w[q], 0x64646464u, 0x4342), 0x64806480u);
  }
}

// Two f32 -> f16x2 (lo in bits [15:0]), round to nearest even.
QL_DEVINL uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// kWO: weight-only product (x is not quantized; see the weight-only prologue).
template <ql_scheme kScheme, int kRs, int kMaxSteps, int kM, bool kWO = false>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
  // kM tokens x kQ = 8 / kRs segment classes must fit the 8 B columns
  static_assert(kM == 1 || (kM * (8 / kRs) <= 8 && kRs >= 2), "tokens do not fit the B columns");
  constexpr bool kInt8 = kScheme == QL_W8A8_INT8_ROW;
  constexpr bool kBlock = kScheme == QL_FP8_E4M3_BLOCK128;
  constexpr bool kIntAcc = kInt8 && !kWO;  // exact int32 sums on s8 MMAs

  extern __shared__ __align__(1024) uint8_t smem[];
  // The product this CTA runs and its place among that product's CTAs
  // (constant-index parameter reads and selects: no local copy of the table).
  int pj = 0;
#pragma unroll
  for (int j = 1; j < kGemvMaxGroup; ++j)
    if (j < p.nprob && (int)blockIdx.x >= p.cta0[j]) pj = j;
  const uint16_t* px = p.prob[0].x;
  const float* psx = p.prob[0].sx;
  const uint8_t* pwq = p.prob[0].wq;
  const float* psw = p.prob[0].sw;
  uint16_t* py = p.prob[0].y;
  int64_t N = p.prob[0].N;
  int Mt = p.prob[0].M;  // this product's tokens (padding tokens past them are zero)
  int cta_lo = p.cta0[0], cta_hi = p.cta0[1];
#pragma unroll
  for (int j = 1; j < kGemvMaxGroup; ++j)
    if (j == pj) {
      px = p.prob[j].x;
      psx = p.prob[j].sx;
      pwq = p.prob[j].wq;
      psw = p.prob[j].sw;
      py = p.prob[j].y;
      N = p.prob[j].N;
      Mt = p.prob[j].M;
      cta_lo = p.cta0[j];
      cta_hi = p.cta0[j + 1];
    }
  const int64_t K = p.K;
  const int G = cta_hi - cta_lo;               // this product's CTAs
  const int bid = (int)blockIdx.x - cta_lo;    // this CTA among them
  const int64_t row_begin = ((int64_t)bid * N) / G;
  const int64_t row_end = ((int64_t)(bid + 1) * N) / G;
  const int64_t KB = K / 128;
  // weight scales this CTA needs: its rows (row schemes) or its 128-row blocks
  const int64_t sw_first = kBlock ? (row_begin >> 7) * KB : row_begin;
  const int64_t sw_count = kBlock ? (((row_end - 1) >> 7) - (row_begin >> 7) + 1) * KB : row_end - row_begin;
  const int sw_cached = (int)min(sw_count, (int64_t)kGemvSwCache);
  const int nst = p.stages;
  const GemvSmemLayout L = gemv_layout(K, p.stage_bytes, nst, kGemvSwCache, kM, kWO ? 2 : 1);
  const int64_t xstride = (K + 127) / 128 * 128;  // bytes between the tokens' codes
  uint8_t* ring = smem + L.ring;
  uint8_t* qx_s = smem + L.qx;
  float* sx_s = reinterpret_cast<float*>(smem + L.sx);
  float* sw_s = reinterpret_cast<float*>(smem + L.swc);
  float* part = reinterpret_cast<float*>(smem + L.part);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kGemvMaxStages;
  uint64_t* xready = full + 2 * kGemvMaxStages;  // consumers have quantized x
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flags);
  int* arrivals = reinterpret_cast<int*>(smem + L.flags + 16);
  float* blockred = reinterpret_cast<float*>(smem + L.flags + 16 + kGemvMaxStages * 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int kStageRows = 2 * kRs;  // rows per full stage
  const int nstages = (int)((row_end - row_begin + kStageRows - 1) / kStageRows);
  // A ragged row count puts its partial stage first, so that it streams with
  // the first full stages instead of adding one stage of latency at the end.
  const int lead = (int)((row_end - row_begin) % kStageRows);
  auto stage_r0 = [&](int i) -> int64_t {
    return lead == 0 ? row_begin + (int64_t)i * kStageRows
                     : (i == 0 ? row_begin : row_begin + lead + (int64_t)(i - 1) * kStageRows);
  };
  auto stage_rows = [&](int i) -> int { return (lead != 0 && i == 0) ? lead : kStageRows; };

  if (tid == 0) {
    tc::launch_dependents();  // the next kernel's CTAs may start as SMs free up
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);  // released by the warp that finishes the stage last
      arrivals[s] = 0;
    }
    *abort_flag = 0;
    mbar_init(xready, 1);
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kGemvWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !p.stall) {
      const uint64_t policy = l2_policy_evict_first();
      int issued = 0;
      for (int i = 0; i < nstages; ++i) {
        const int slot = i % nst;
        // Only kEarlyStages copies go out before x is quantized: a full ring
        // fill from every SM at once queues the consumers' x reads and
        // instruction fetches behind ~25 MB of weight requests.
        if (i == kEarlyStages && !mbar_wait_bounded(xready, 0, abort_flag)) {
          if (!*abort_flag) record_timeout(p.status, KID_GEMV, 3);
          *abort_flag = 1;
          break;
        }
        if (i >= nst && !mbar_wait_bounded(&empty[slot], ((i / nst) - 1) & 1, abort_flag)) {
          if (!*abort_flag) record_timeout(p.status, KID_GEMV, 1);
          *abort_flag = 1;
          break;
        }
        const int64_t r0 = stage_r0(i);
        const int64_t nr = stage_rows(i);
        const uint32_t bytes = (uint32_t)(nr * K);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(ring + slot * p.stage_bytes, pwq + r0 * K, bytes, &full[slot], policy);
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
  // 0. The CTA's weight scales into shared memory (immutable inputs: no wait).
  for (int i = tid; i < sw_cached; i += kGemvConsumers) sw_s[i] = __ldg(psw + sw_first + i);

  tc::grid_dependency_wait();  // x may be produced by the previous kernel
  bool xready_done = false;  // xready arrives once, as soon as x is loaded where the path allows
  // 1. Fused activation quantization of x [kM, K] into shared memory: one pass
  //    for the absmax (the first kXLoads chunks per thread loaded together),
  //    one for the codes (x is L2-resident by then).
  if constexpr (kWO && kM == 1) {
    // Weight-only: x is not quantized.  The MMAs run on f16, so x is staged
    // as x * 2^e in f16, e the power of two that puts the token's absmax in
    // [2^14, 2^15): a bf16 significand (8 bits) fits f16's 11, so every element
    // within a factor 2^31 of the absmax is carried exactly (smaller ones round
    // to f16's subnormal spacing).  The products with the f16 weight values
    // are exact in f32; the epilogue multiplies the sums by 2^-e (exact).
    const int64_t nchunk8 = K / 8;  // 16-byte chunks of 8 bf16
    constexpr int kXLoads = 8;
    const uint4* xg = reinterpret_cast<const uint4*>(px);
    uint4* stash = K <= kGemvStashMaxK ? reinterpret_cast<uint4*>(smem + L.stash) : nullptr;
    float a_tok = 0.0f;
#pragma unroll
    for (int i = 0; i < kXLoads; ++i) {
      const int64_t c = tid + (int64_t)i * kGemvConsumers;
      const uint4 v = c < nchunk8 ? __ldg(xg + c) : make_uint4(0, 0, 0, 0);
      if (stash && c < nchunk8) stash[c] = v;
      a_tok = fmaxf(a_tok, absmax_chunk8(v));
    }
    for (int64_t c = tid + (int64_t)kXLoads * kGemvConsumers; c < nchunk8; c += kGemvConsumers) {
      const uint4 v = __ldg(xg + c);
      if (stash) stash[c] = v;
      a_tok = fmaxf(a_tok, absmax_chunk8(v));
    }
    a_tok = warp_max(a_tok);
    if (lane == 0) blockred[warp] = a_tok;
    named_bar_sync(kBarConsumers, kGemvConsumers);
    if (tid == 0) mbar_arrive(xready);  // x is loaded: the producer may fill the ring
    xready_done = true;
    float a = blockred[0];
#pragma unroll
    for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, blockred[w]);
    // e = 14 - exponent(a), kept within [-113, 126] so that 2^e and 2^-e are
    // normal f32 (a zero or subnormal absmax takes e = 126)
    int e2 = 126;
    const int ea = (int)((__float_as_uint(a) >> 23) & 0xFFu);
    if (ea != 0) e2 = min(126, 14 - (ea - 127));
    const float up = __uint_as_float((uint32_t)(127 + e2) << 23);
    const float down = __uint_as_float((uint32_t)(127 - e2) << 23);
    for (int i = tid; i < (kBlock ? (int)KB : 1); i += kGemvConsumers) sx_s[i] = down;
    uint4* xs4 = reinterpret_cast<uint4*>(qx_s);
#pragma unroll 1
    for (int64_t c = tid; c < nchunk8; c += kGemvConsumers) {
      const uint4 v = stash ? stash[c] : __ldg(xg + c);
      xs4[c] = make_uint4(f32x2_to_f16x2(bf16_lo(v.x) * up, bf16_hi(v.x) * up),
                          f32x2_to_f16x2(bf16_lo(v.y) * up, bf16_hi(v.y) * up),
                          f32x2_to_f16x2(bf16_lo(v.z) * up, bf16_hi(v.z) * up),
                          f32x2_to_f16x2(bf16_lo(v.w) * up, bf16_hi(v.w) * up));
    }
    // zero the padding of the last 64-element window so it adds nothing
    for (int64_t b = 2 * K + tid * 16; b < 2 * ((K + 63) / 64 * 64); b += kGemvConsumers * 16)
      *reinterpret_cast<uint4*>(qx_s + b) = make_uint4(0, 0, 0, 0);
    named_bar_sync(kBarConsumers, kGemvConsumers);
  } else if constexpr (kWO) {
    // Weight-only, kM tokens side by side: one absmax pass and one staging
    // pass for all of them, each token with its own power of two.  Padding
    // tokens (past Mt) read nothing and stage zeros.
    const int nchunk8 = (int)(K / 8);
    const uint4* xg = reinterpret_cast<const uint4*>(px);  // token tok at tok * nchunk8
    const int64_t xs2 = 2 * xstride;                        // bytes between staged tokens
    float amax[kM];
#pragma unroll
    for (int tok = 0; tok < kM; ++tok) amax[tok] = 0.0f;
    for (int c = tid; c < nchunk8; c += kGemvConsumers) {
#pragma unroll
      for (int tok = 0; tok < kM; ++tok) {
        const uint4 v = tok < Mt ? __ldg(xg + tok * nchunk8 + c) : make_uint4(0, 0, 0, 0);
        amax[tok] = fmaxf(amax[tok], absmax_chunk8(v));
      }
    }
#pragma unroll
    for (int tok = 0; tok < kM; ++tok) {
      const float a = warp_max(amax[tok]);
      if (lane == 0) blockred[tok * kGemvWarps + warp] = a;
    }
    named_bar_sync(kBarConsumers, kGemvConsumers);
    float up[kM];
    const int sx_per_tok = kBlock ? (int)KB : 1;  // block scheme: one scale per group
#pragma unroll
    for (int tok = 0; tok < kM; ++tok) {
      float a = blockred[tok * kGemvWarps];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, blockred[tok * kGemvWarps + w]);
      int e2 = 126;
      const int ea = (int)((__float_as_uint(a) >> 23) & 0xFFu);
      if (ea != 0) e2 = min(126, 14 - (ea - 127));
      up[tok] = __uint_as_float((uint32_t)(127 + e2) << 23);
      const float down = __uint_as_float((uint32_t)(127 - e2) << 23);
      for (int i = tid; i < sx_per_tok; i += kGemvConsumers) sx_s[tok * sx_per_tok + i] = down;
    }
#pragma unroll 1
    for (int c = tid; c < nchunk8; c += kGemvConsumers) {
#pragma unroll
      for (int tok = 0; tok < kM; ++tok) {
        const uint4 v = tok < Mt ? __ldg(xg + tok * nchunk8 + c) : make_uint4(0, 0, 0, 0);
        const float u = up[tok];
        reinterpret_cast<uint4*>(qx_s + tok * xs2)[c] =
            make_uint4(f32x2_to_f16x2(bf16_lo(v.x) * u, bf16_hi(v.x) * u),
                       f32x2_to_f16x2(bf16_lo(v.y) * u, bf16_hi(v.y) * u),
                       f32x2_to_f16x2(bf16_lo(v.z) * u, bf16_hi(v.z) * u),
                       f32x2_to_f16x2(bf16_lo(v.w) * u, bf16_hi(v.w) * u));
      }
    }
    // zero the padding of each token's last 64-element window
    for (int tok = 0; tok < kM; ++tok)
      for (int64_t b = 2 * K + tid * 16; b < 2 * ((K + 63) / 64 * 64); b += kGemvConsumers * 16)
        *reinterpret_cast<uint4*>(qx_s + tok * xs2 + b) = make_uint4(0, 0, 0, 0);
    named_bar_sync(kBarConsumers, kGemvConsumers);
  } else if constexpr (kM == 1) {
    const int64_t nchunk8 = K / 8;  // 16-byte chunks of 8 bf16
    constexpr int kXLoads = 8;
    const uint4* xg = reinterpret_cast<const uint4*>(px);
    uint8_t* qx_t = qx_s;
    float* sx_t = sx_s;
    if (psx) {
      // Pre-quantized input (the producer of x wrote its codes and scales):
      // the codes go to shared memory as they are.
      const uint4* qg = reinterpret_cast<const uint4*>(px);
      for (int64_t c = tid; c < K / 16; c += kGemvConsumers) reinterpret_cast<uint4*>(qx_t)[c] = __ldg(qg + c);
      for (int i = tid; i < (kBlock ? (int)KB : 1); i += kGemvConsumers) sx_t[i] = __ldg(psx + i);
    } else if (kBlock) {
      // 16 consecutive chunks (lanes) form one 128-wide group: no CTA barrier
      for (int64_t base = 0; base < nchunk8; base += kGemvConsumers) {
        const int64_t c = base + tid;
        const uint4 v = c < nchunk8 ? __ldg(xg + c) : make_uint4(0, 0, 0, 0);
        float a = absmax_chunk8(v);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const float s = a / 448.0f;
        if (c < nchunk8) {
          if ((lane & 15) == 0) sx_t[c >> 4] = s;
          reinterpret_cast<uint2*>(qx_t)[c] = quant_chunk8<false>(v, make_divisor(s));
        }
      }
    } else {
      // When x fits, the absmax pass parks its chunks in shared memory and
      // the code pass reads them there instead of a second trip to L2; the
      // producer resumes the weight stream as soon as x is loaded (xready),
      // while the codes are computed.
      uint4* stash = K <= kGemvStashMaxK ? reinterpret_cast<uint4*>(smem + L.stash) : nullptr;
      float a_tok = 0.0f;
#pragma unroll
      for (int i = 0; i < kXLoads; ++i) {
        const int64_t c = tid + (int64_t)i * kGemvConsumers;
        const uint4 v = c < nchunk8 ? __ldg(xg + c) : make_uint4(0, 0, 0, 0);
        if (stash && c < nchunk8) stash[c] = v;
        a_tok = fmaxf(a_tok, absmax_chunk8(v));
      }
      for (int64_t c = tid + (int64_t)kXLoads * kGemvConsumers; c < nchunk8; c += kGemvConsumers) {
        const uint4 v = __ldg(xg + c);
        if (stash) stash[c] = v;
        a_tok = fmaxf(a_tok, absmax_chunk8(v));
      }
      a_tok = warp_max(a_tok);
      if (lane == 0) blockred[warp] = a_tok;
      named_bar_sync(kBarConsumers, kGemvConsumers);
      if (tid == 0) mbar_arrive(xready);  // x is loaded: the producer may fill the ring
      xready_done = true;
      float a = blockred[0];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, blockred[w]);
      const float s = a / (kInt8 ? 127.0f : 448.0f);
      if (tid == 0) sx_t[0] = s;
      const Divisor dv = make_divisor(s);
      // one uniform branch: the eight values of every chunk run side by side
      auto emit_all = [&](auto fast) {
        constexpr bool kFast = decltype(fast)::value;
        // a rolled loop re-reading x (parked in shared memory, else
        // L2-resident): the straight-line form measured slower inside a step,
        // where its instructions are fetched while the weight stream congests L2
        uint2* q2 = reinterpret_cast<uint2*>(qx_t);
#pragma unroll 1
        for (int64_t c = tid; c < nchunk8; c += 2 * kGemvConsumers) {
          const int64_t c2 = c + kGemvConsumers;
          const uint4 v0 = stash ? stash[c] : __ldg(xg + c);
          const uint4 v1 = c2 < nchunk8 ? (stash ? stash[c2] : __ldg(xg + c2)) : make_uint4(0, 0, 0, 0);
          q2[c] = quant_chunk8<kInt8, kFast>(v0, dv);
          if (c2 < nchunk8) q2[c2] = quant_chunk8<kInt8, kFast>(v1, dv);
        }
      };
      if (dv.fast)
        emit_all(std::true_type{});
      else
        emit_all(std::false_type{});
    }
    // zero the padding of the last 64-byte window so it adds nothing
    for (int64_t b = K + tid * 16; b < (K + 63) / 64 * 64; b += kGemvConsumers * 16)
      *reinterpret_cast<uint4*>(qx_t + b) = make_uint4(0, 0, 0, 0);
    named_bar_sync(kBarConsumers, kGemvConsumers);
  } else {
    // kM tokens side by side: one absmax pass and one code pass for all of
    // them, every token's loads in flight together.  Padding tokens (past
    // Mt) read nothing and get zero codes and scales.
    const int nchunk8 = (int)(K / 8);  // 16-byte chunks of 8 bf16 per token
    const uint4* xg = reinterpret_cast<const uint4*>(px);  // token tok at tok * nchunk8
    if constexpr (kBlock) {
      // flat chunk f = tok * nchunk8 + c; 16 consecutive chunks (lanes) form
      // one 128-wide group of one token (K % 128 == 0)
      constexpr int kB = 4;
      const int total = kM * nchunk8;
      for (int base = 0; base < total; base += kB * kGemvConsumers) {
        uint4 v[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) {
          const int f = base + b * kGemvConsumers + tid;
          v[b] = f < total && f / nchunk8 < Mt ? __ldg(xg + f) : make_uint4(0, 0, 0, 0);
        }
        float sc[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) {
          float a = absmax_chunk8(v[b]);
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
          sc[b] = a / 448.0f;
        }
        // one copy of the code conversion (a rolled loop picking its chunk by
        // selects)
#pragma unroll 1
        for (int b = 0; b < kB; ++b) {
          uint4 vb = v[0];
          float sb = sc[0];
#pragma unroll
          for (int j = 1; j < kB; ++j)
            if (b == j) {
              vb = v[j];
              sb = sc[j];
            }
          const int f = base + b * kGemvConsumers + tid;
          if (f < total) {
            const int tok = f / nchunk8, c = f - tok * nchunk8;
            if ((lane & 15) == 0) sx_s[tok * KB + (c >> 4)] = sb;
            reinterpret_cast<uint2*>(qx_s + tok * xstride)[c] = quant_chunk8<false>(vb, make_divisor(sb));
          }
        }
      }
    } else {
      float amax[kM];
#pragma unroll
      for (int tok = 0; tok < kM; ++tok) amax[tok] = 0.0f;
      for (int c = tid; c < nchunk8; c += 2 * kGemvConsumers) {
        const int c2 = c + kGemvConsumers;
        uint4 v[2 * kM];
#pragma unroll
        for (int tok = 0; tok < kM; ++tok) {
          v[2 * tok] = tok < Mt ? __ldg(xg + tok * nchunk8 + c) : make_uint4(0, 0, 0, 0);
          v[2 * tok + 1] = tok < Mt && c2 < nchunk8 ? __ldg(xg + tok * nchunk8 + c2) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int tok = 0; tok < kM; ++tok)
          amax[tok] = fmaxf(amax[tok], fmaxf(absmax_chunk8(v[2 * tok]), absmax_chunk8(v[2 * tok + 1])));
      }
#pragma unroll
      for (int tok = 0; tok < kM; ++tok) {
        const float a = warp_max(amax[tok]);
        if (lane == 0) blockred[tok * kGemvWarps + warp] = a;
      }
      named_bar_sync(kBarConsumers, kGemvConsumers);
      Divisor dv[kM];
      bool all_fast = true;
#pragma unroll
      for (int tok = 0; tok < kM; ++tok) {
        float a = blockred[tok * kGemvWarps];
#pragma unroll
        for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, blockred[tok * kGemvWarps + w]);
        const float sc = a / (kInt8 ? 127.0f : 448.0f);
        if (tid == 0) sx_s[tok] = sc;
        dv[tok] = make_divisor(sc);
        if (tok < Mt) all_fast = all_fast && dv[tok].fast;
      }
      // one uniform branch for all tokens: the IEEE path gives the same codes
      auto emit_all = [&](auto fast) {
        constexpr bool kFast = decltype(fast)::value;
#pragma unroll 1
        for (int c = tid; c < nchunk8; c += kGemvConsumers) {
          uint4 v[kM];
#pragma unroll
          for (int tok = 0; tok < kM; ++tok)
            v[tok] = tok < Mt ? __ldg(xg + tok * nchunk8 + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int tok = 0; tok < kM; ++tok)
            reinterpret_cast<uint2*>(qx_s + tok * xstride)[c] =
                tok < Mt ? quant_chunk8<kInt8, kFast>(v[tok], dv[tok]) : make_uint2(0, 0);
        }
      };
      if (all_fast)
        emit_all(std::true_type{});
      else
        emit_all(std::false_type{});
    }
    // zero the padding of each token's last 64-byte window so it adds nothing
    for (int tok = 0; tok < kM; ++tok)
      for (int64_t b = K + tid * 16; b < (K + 63) / 64 * 64; b += kGemvConsumers * 16)
        *reinterpret_cast<uint4*>(qx_s + tok * xstride + b) = make_uint4(0, 0, 0, 0);
    named_bar_sync(kBarConsumers, kGemvConsumers);
  }
  if (tid == 0 && !xready_done) mbar_arrive(xready);  // the producer may fill the whole ring now
  if (!kWO && blockIdx.x == 0 && (p.dbg.qx || p.dbg.sx)) {  // product 0's first CTA
    // [token, K] codes and [token, groups] scales; rows of K bytes (K % 16 == 0)
    const int ns = kBlock ? (int)KB : 1;
    for (int64_t c = tid; c < (kM == 1 ? 1 : Mt) * (K / 16); c += kGemvConsumers) {
      const int64_t tok = kM == 1 ? 0 : c / (K / 16), cc = kM == 1 ? c : c % (K / 16);
      if (p.dbg.qx)
        reinterpret_cast<uint4*>(p.dbg.qx)[c] = reinterpret_cast<const uint4*>(qx_s + tok * xstride)[cc];
    }
    for (int i = tid; i < (kM == 1 ? 1 : Mt) * ns; i += kGemvConsumers)
      if (p.dbg.sx) p.dbg.sx[i] = sx_s[i];
  }

  // 2. Work split.  A stage holds 2 kRs whole rows (kRs = 1, 2 or 4) cut into
  //    16 units of the MMA's 16 A rows: unit u = (row (u / 8) kRs + (u % 8) / kQ,
  //    segment u % kQ), kQ = 8 / kRs, segment q covering bytes [q seg,
  //    (q+1) seg) of its row.  The weights are the A operand and the 8 B columns
  //    carry x: column j holds the x bytes of segment j % kQ at the window the
  //    units j and j + 8 read, so D[j][j] and D[j+8][j] are those units'
  //    partials (held by one lane) and the other products are discarded.  A
  //    step feeds one 64-byte window of every unit; odd units take the two
  //    windows of each pair in swapped order, so that the lanes of one
  //    shared-memory phase (units 2p and 2p+1) read opposite halves of the
  //    banks.  Each warp owns the same steps of every stage, so its x
  //    fragments stay in registers for the whole kernel.  The block scheme
  //    splits whole window pairs (128-byte groups) so that each group's
  //    partial is scaled alone.  E4M3 runs as f16 MMAs (exact conversion).
  constexpr int kQ = 8 / kRs;
  // kMaxSteps: steps per warp, >= ceil(windows per unit / warps) (host-chosen)
  const int64_t seg = p.seg_len;     // a multiple of 128
  const int segW = (int)(seg / 64);  // windows per unit (even)
  int st0, st1;                      // this warp's steps [st0, st1)
  if (kBlock) {
    st0 = 2 * ((warp * (segW / 2)) / kGemvWarps);
    st1 = 2 * (((warp + 1) * (segW / 2)) / kGemvWarps);
  } else {
    st0 = (warp * segW) / kGemvWarps;
    st1 = ((warp + 1) * segW) / kGemvWarps;
  }
  const int nsteps = st1 - st0;           // <= kMaxSteps
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const int ur = g / kQ, uq = g % kQ;     // units g and g + 8: rows ur and kRs + ur, segment uq
  const int flip = g & 1;                 // odd units swap the windows of each pair
  const int e = g & 1;                    // D[g][g], D[g+8][g] are elements e, 2 + e
  // The lane's B column g carries token xtok.  One token: every column holds
  // x of segment class g % kQ, and the lane keeps D[g][g], D[g+8][g] when it
  // holds column g (t = g / 2).  kM tokens: column kQ tok + c holds token tok,
  // class c (columns past kM kQ repeat the last token and are discarded), and
  // the products of units g, g + 8 with token tok sit in column kQ tok + uq,
  // held by lane t = (kQ tok + uq) / 2 as element uq % 2 = e (kQ is even).
  const int c0 = 2 * t + e;  // the column whose products this lane may keep
  const int xtok = kM == 1 ? 0 : min(g / kQ, kM - 1);
  const bool diag = kM == 1 ? t == (g >> 1) : (c0 % kQ == uq && c0 / kQ < kM);
  const int ktok = kM == 1 ? 0 : min(c0 / kQ, kM - 1);  // token of the kept products
  const int64_t ulen = min(seg, K - (int64_t)uq * seg);  // unit bytes inside K
  uint4 xr[kMaxSteps];
  uint32_t vmask = 0;  // steps whose 16 bytes of this lane lie inside the unit
  if constexpr (!kWO) {
#pragma unroll
    for (int s = 0; s < kMaxSteps; ++s) {
      const int64_t off = (int64_t)((st0 + s) ^ flip) * 64 + t * 16;
      const bool v = s < nsteps && off < ulen;
      xr[s] = v ? ld_s128(qx_s + xtok * xstride + (int64_t)uq * seg + off) : make_uint4(0, 0, 0, 0);
      vmask |= (uint32_t)v << s;
    }
  }
  uint32_t xh[kIntAcc ? 1 : kMaxSteps][8];  // f16 MMA schemes: x fragments as f16
  if constexpr (kWO) {
    // the lane's 16 staged f16 values at the same K positions (32 bytes)
#pragma unroll
    for (int s = 0; s < kMaxSteps; ++s) {
      const int64_t off = (int64_t)((st0 + s) ^ flip) * 64 + t * 16;
      const bool v = s < nsteps && off < ulen;
      const uint8_t* src = qx_s + 2 * (xtok * xstride + (int64_t)uq * seg + off);
      const uint4 lo = v ? ld_s128(src) : make_uint4(0, 0, 0, 0);
      const uint4 hi = v ? ld_s128(src + 16) : make_uint4(0, 0, 0, 0);
      xh[s][0] = lo.x, xh[s][1] = lo.y, xh[s][2] = lo.z, xh[s][3] = lo.w;
      xh[s][4] = hi.x, xh[s][5] = hi.y, xh[s][6] = hi.z, xh[s][7] = hi.w;
      vmask |= (uint32_t)v << s;
    }
  } else if constexpr (!kInt8) {
#pragma unroll
    for (int s = 0; s < kMaxSteps; ++s) e4m3x16_to_f16(xr[s], xh[s]);
  }
  const float sx_tok = (kBlock || kM > 1) ? 0.0f : sx_s[0];  // one token, row schemes
  float sxr[kMaxSteps / 2];  // block scheme: x scale of each pair's 128-wide group
  int64_t grp0 = 0;
  if constexpr (kBlock) {
    grp0 = ((int64_t)uq * seg + (int64_t)st0 * 64) / 128;
#pragma unroll
    for (int m = 0; m < kMaxSteps / 2; ++m) sxr[m] = sx_s[ktok * KB + min(grp0 + m, KB - 1)];
  }
  const uint32_t w_lane = (uint32_t)(ur * K + (int64_t)uq * seg + t * 16);
  const uint32_t w_half = (uint32_t)(kRs * K);  // units g + 8: kRs rows further

  // One step: the 16-byte fragments of units g and g + 8, 2 s8 MMAs or 4 f16 MMAs.
  auto step = [&](uint32_t (&dd)[2][4], int s, const uint8_t* wb, uint32_t vm0, uint32_t vm1) {
    const int off = ((st0 + s) ^ flip) * 64;
    const uint4 w0 = (vm0 >> s) & 1u ? ld_s128(wb + off) : make_uint4(0, 0, 0, 0);
    const uint4 w1 = (vm1 >> s) & 1u ? ld_s128(wb + w_half + off) : make_uint4(0, 0, 0, 0);
    if constexpr (kIntAcc) {
      mma_s8(dd[0], w0.x, w1.x, w0.y, w1.y, xr[s].x, xr[s].y);
      mma_s8(dd[1], w0.z, w1.z, w0.w, w1.w, xr[s].z, xr[s].w);
    } else {
      uint32_t h0[8], h1[8];
      if constexpr (kInt8) {  // weight-only int8: codes to f16 (exact)
        s8x16_to_f16(w0, h0);
        s8x16_to_f16(w1, h1);
      } else {
        e4m3x16_to_f16(w0, h0);
        e4m3x16_to_f16(w1, h1);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        mma_f16(dd[q & 1], h0[2 * q], h1[2 * q], h0[2 * q + 1], h1[2 * q + 1], xh[s][2 * q], xh[s][2 * q + 1]);
    }
  };

  // 3. Stream the ring.
  for (int i = 0; i < nstages; ++i) {
    const int slot = i % nst;
    const int64_t r0 = stage_r0(i);
    const int nr = stage_rows(i);
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (i / nst) & 1, abort_flag))) {
      if (lane == 0 && !*abort_flag) record_timeout(p.status, KID_GEMV, 2);
      *abort_flag = 1;
      break;
    }
    const uint8_t* wb = ring + slot * p.stage_bytes + w_lane;
    const uint32_t vm0 = ur < nr ? vmask : 0u;        // a unit past the stage's rows has no data
    const uint32_t vm1 = kRs + ur < nr ? vmask : 0u;
    float kept0, kept1;                               // units g and g + 8 (diagonal lanes)
    if constexpr (!kBlock) {
      // Always kMaxSteps steps: a step past this warp's range has zero x and W
      // fragments and adds nothing (a uniform branch per step measured 2x
      // slower than the spare MMAs).  Two accumulator pairs alternate by step.
      uint32_t d[2][2][4] = {};
#pragma unroll
      for (int s = 0; s < kMaxSteps; ++s) step(d[s & 1], s, wb, vm0, vm1);
      uint32_t k0[4], k1[4];  // elements e and 2 + e of each accumulator (selects, no local memory)
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        k0[a] = e ? d[a >> 1][a & 1][1] : d[a >> 1][a & 1][0];
        k1[a] = e ? d[a >> 1][a & 1][3] : d[a >> 1][a & 1][2];
      }
      if constexpr (kIntAcc) {  // carried bit-for-bit through the float slot, summed as int32
        kept0 = __int_as_float((int)(k0[0] + k0[1] + k0[2] + k0[3]));
        kept1 = __int_as_float((int)(k1[0] + k1[1] + k1[2] + k1[3]));
      } else {
        kept0 = (__uint_as_float(k0[0]) + __uint_as_float(k0[1])) +
                (__uint_as_float(k0[2]) + __uint_as_float(k0[3]));
        kept1 = (__uint_as_float(k1[0]) + __uint_as_float(k1[1])) +
                (__uint_as_float(k1[2]) + __uint_as_float(k1[3]));
      }
    } else {
      // per 128-wide group (a window pair): its own partials, scaled by
      // s_x[group] * s_w[row block, group] for each of the two units
      const int64_t blk0 = (min(r0 + ur, row_end - 1) >> 7) * KB - sw_first;
      const int64_t blk1 = (min(r0 + kRs + ur, row_end - 1) >> 7) * KB - sw_first;
      float res0 = 0.0f, res1 = 0.0f;
#pragma unroll
      for (int m = 0; m < kMaxSteps / 2; ++m) {
        // pairs past this warp's range have zero fragments and add nothing
        uint32_t d[2][4] = {};
        step(d, 2 * m, wb, vm0, vm1);
        step(d, 2 * m + 1, wb, vm0, vm1);
        const float p0 = __uint_as_float(e ? d[0][1] : d[0][0]) + __uint_as_float(e ? d[1][1] : d[1][0]);
        const float p1 = __uint_as_float(e ? d[0][3] : d[0][2]) + __uint_as_float(e ? d[1][3] : d[1][2]);
        const int64_t grp = min(grp0 + m, KB - 1);
        const float sw0 = blk0 + grp < sw_cached ? sw_s[blk0 + grp] : __ldg(psw + sw_first + blk0 + grp);
        const float sw1 = blk1 + grp < sw_cached ? sw_s[blk1 + grp] : __ldg(psw + sw_first + blk1 + grp);
        res0 = fmaf(p0, sxr[m] * sw0, res0);
        res1 = fmaf(p1, sxr[m] * sw1, res1);
      }
      kept0 = res0;
      kept1 = res1;
    }
    // Park the unit partials, then count in.
    float* ps = part + slot * kM * kGemvWarps * kGemvUnits;  // [token][warp][unit]
    if (diag) {
      ps[(ktok * kGemvWarps + warp) * kGemvUnits + g] = kept0;
      ps[(ktok * kGemvWarps + warp) * kGemvUnits + 8 + g] = kept1;
    }
    __syncwarp();
    int before = 0;
    if (lane == 0) {
      __threadfence_block();
      before = atomicAdd(&arrivals[slot], 1);
    }
    before = __shfl_sync(0xffffffffu, before, 0);
    if (before == kGemvWarps - 1) {
      // last warp of this stage: every warp has read the stage and parked its
      // partials.
      __threadfence_block();
      // One token: lane (wg, u) adds warps wg, wg + 2, ... of unit u and the
      // two warp groups are then added.  kM tokens: lane (wg, u) adds all
      // warps of unit u for tokens wg, wg + 2, ...  Then across the kQ units
      // of each row; every order is fixed.
      const int u = lane & 15, wg = lane >> 4;
      const int r = (u >> 3) * kRs + (u & 7) / kQ;
#pragma unroll
      for (int tt = 0; tt < (kM + 1) / 2; ++tt) {
        const int otok = kM == 1 ? 0 : wg + 2 * tt;  // output token of this lane
        int vi = 0;
        float vf = 0.0f;
#pragma unroll
        for (int w = (kM == 1 ? wg : 0); w < kGemvWarps; w += (kM == 1 ? 2 : 1)) {
          const float pv = ps[(otok * kGemvWarps + w) * kGemvUnits + u];
          if constexpr (kIntAcc)
            vi += __float_as_int(pv);
          else
            vf += pv;
        }
        if constexpr (kIntAcc) {
          if (kM == 1) vi += __shfl_xor_sync(0xffffffffu, vi, 16);
#pragma unroll
          for (int o = 1; o < kQ; o <<= 1) vi += __shfl_xor_sync(0xffffffffu, vi, o);
        } else {
          if (kM == 1) vf += __shfl_xor_sync(0xffffffffu, vf, 16);
#pragma unroll
          for (int o = 1; o < kQ; o <<= 1) vf += __shfl_xor_sync(0xffffffffu, vf, o);
        }
        if ((kM == 1 ? wg == 0 : otok < Mt) && u % kQ == 0 && r < nr) {
          const int64_t n = r0 + r;
          const int64_t o = otok * N + n;  // y and debug index [token, row]
          float yv;
          if constexpr (kBlock) {
            yv = vf;
          } else {
            const int64_t si = n - row_begin;
            const float swn = si < sw_cached ? sw_s[si] : __ldg(psw + n);
            const float sxt = kM == 1 ? sx_tok : sx_s[otok];
            if constexpr (kIntAcc) {
              if (p.dbg.acc_i32) p.dbg.acc_i32[o] = vi;
              yv = __fmul_rn(__fmul_rn(__int2float_rn(vi), sxt), swn);
            } else {
              if (p.dbg.acc_f32) p.dbg.acc_f32[o] = vf;
              yv = __fmul_rn(__fmul_rn(vf, sxt), swn);
            }
          }
          py[o] = f32_to_bf16_rn(yv);
        }
      }
      __syncwarp();
      if (lane == 0) {
        arrivals[slot] = 0;
        mbar_arrive(&empty[slot]);
      }
    }
  }
}

int gemv_max_k() { return kGemvMaxK; }

bool gemv_token_halves_pay(int64_t M, int64_t K, const int64_t* Ns, int count) {
  if (M < 5 || M > 8 || K > kGemvMaxK4 || count < 1 || 2 * count > kGemvMaxGroup) return false;
  int64_t bytes = 0;
  for (int j = 0; j < count; ++j) bytes += Ns[j] * K;
  return bytes <= kGemvHalvesMaxWeightBytes;
}
int gemv_weight_only_max_k() { return (int)kGemvMaxKWO; }

template <ql_scheme S, int kRs, int kSteps, int kM, bool kWO = false>
static cudaError_t launch_gemv_r(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem<gemv_kernel<S, kRs, kSteps, kM, kWO>>((int)smem);
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
  return cudaLaunchKernelEx(&cfg, gemv_kernel<S, kRs, kSteps, kM, kWO>, p);
}

// Steps per warp: 4 when a unit has at most 32 windows of 64 bytes, else 8.
template <ql_scheme S>
static cudaError_t launch_gemv_t(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  const bool long_units = p.seg_len > 32 * 64;
  if (p.M > 2)
    return long_units ? launch_gemv_r<S, 4, 8, 4>(p, grid, smem, st) : launch_gemv_r<S, 4, 4, 4>(p, grid, smem, st);
  if (p.M == 2) {
    if (p.rows_per_stage == 8)
      return long_units ? launch_gemv_r<S, 4, 8, 2>(p, grid, smem, st) : launch_gemv_r<S, 4, 4, 2>(p, grid, smem, st);
    return long_units ? launch_gemv_r<S, 2, 8, 2>(p, grid, smem, st) : launch_gemv_r<S, 2, 4, 2>(p, grid, smem, st);
  }
  switch (p.rows_per_stage / 2) {
    case 1:
      return long_units ? launch_gemv_r<S, 1, 8, 1>(p, grid, smem, st) : launch_gemv_r<S, 1, 4, 1>(p, grid, smem, st);
    case 2: return launch_gemv_r<S, 2, 4, 1>(p, grid, smem, st);
    case 4: return launch_gemv_r<S, 4, 4, 1>(p, grid, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

// Weight-only: the stage shapes of the quantized GEMV for the same token count.
template <ql_scheme S>
static cudaError_t launch_gemv_wo_t(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  const bool long_units = p.seg_len > 32 * 64;
  if (p.M > 2)
    return long_units ? launch_gemv_r<S, 4, 8, 4, true>(p, grid, smem, st)
                      : launch_gemv_r<S, 4, 4, 4, true>(p, grid, smem, st);
  if (p.M == 2) {
    if (p.rows_per_stage == 8)
      return long_units ? launch_gemv_r<S, 4, 8, 2, true>(p, grid, smem, st)
                        : launch_gemv_r<S, 4, 4, 2, true>(p, grid, smem, st);
    return long_units ? launch_gemv_r<S, 2, 8, 2, true>(p, grid, smem, st)
                      : launch_gemv_r<S, 2, 4, 2, true>(p, grid, smem, st);
  }
  if (long_units) return cudaErrorNotSupported;  // one token: K <= 16384 keeps units short
  switch (p.rows_per_stage / 2) {
    case 1: return launch_gemv_r<S, 1, 4, 1, true>(p, grid, smem, st);
    case 2: return launch_gemv_r<S, 2, 4, 1, true>(p, grid, smem, st);
    case 4: return launch_gemv_r<S, 4, 4, 1, true>(p, grid, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

int gemv_max_k_tokens(int64_t M) {
  return M == 1 ? (int)kGemvMaxK : M == 2 ? (int)kGemvMaxK2 : M <= 4 ? (int)kGemvMaxK4 : 0;
}

// Stage shape, ring depth and CTA split for `count` products of M tokens and
// K inputs (xelem: bytes per staged x element).  The SMs are shared out so
// that the largest number of weight rows any CTA streams is as small as it
// can be (one CTA at a time to the product whose CTAs carry the most rows;
// no product gets more CTAs than it has ring stages).  Returns
// cudaErrorInvalidValue / InvalidConfiguration for shapes the kernel does not
// take.
static cudaError_t gemv_setup(GemvParams& p, int64_t M, const ql_gemv_problem* probs, int count,
                              int64_t K, int xelem, int num_sms, int* grid, size_t* smem,
                              const int* Ms = nullptr) {
  if (count < 1 || count > kGemvMaxGroup) return cudaErrorInvalidValue;
  p.nprob = count;
  p.K = K;
  p.M = (int)M;
  // kRs: the largest power of two <= 4 whose stage of 2 kRs rows fits the
  // ~32 KB copy size (kRs = 1 above 16 KB rows: stages of two rows); the 16
  // MMA rows are then 2 kRs rows x 8 / kRs segments.  M tokens need M x 8 / kRs
  // B columns: kRs >= 2 for two tokens, kRs = 4 for three or four.
  int rs = 1;
  while (rs < 4 && (int64_t)(4 * rs) * K <= kGemvStageTarget) rs *= 2;
  if (M == 2) rs = std::max(rs, 2);
  if (M > 2) rs = 4;
  const int km = M <= 2 ? (int)M : 4;  // the kernel's token count (three tokens pad to four)
  p.rows_per_stage = 2 * rs;
  p.stage_bytes = (int)(((int64_t)p.rows_per_stage * K + 127) / 128 * 128);
  const int fixed = gemv_layout(K, p.stage_bytes, 0, kGemvSwCache, km, xelem).total;
  p.stages = (int)std::min<int64_t>(kGemvMaxStages, (kGemvSmemBudget - fixed) / p.stage_bytes);
  if (p.stages < 2) return cudaErrorInvalidConfiguration;
  const int q = 8 / rs;
  p.seg_len = ((K + q - 1) / q + 127) / 128 * 128;
  // the kernel keeps at most 64 windows of 64 bytes per unit
  if (p.seg_len > 64 * 64) return cudaErrorInvalidValue;
  int g[kGemvMaxGroup];
  int64_t cap[kGemvMaxGroup];
  int used = 0;
  for (int j = 0; j < count; ++j) {
    p.prob[j] = GemvProblem{probs[j].x ? probs[j].x : static_cast<const uint16_t*>(probs[j].qx),
                            probs[j].x ? nullptr : probs[j].sx,
                            static_cast<const uint8_t*>(probs[j].wq), probs[j].sw, probs[j].y,
                            probs[j].N, Ms ? Ms[j] : (int)M};
    cap[j] = (probs[j].N + p.rows_per_stage - 1) / p.rows_per_stage;
    g[j] = 1;
    ++used;
  }
  for (; used < num_sms; ++used) {
    int best = -1;
    for (int j = 0; j < count; ++j)
      if (g[j] < cap[j] && (best < 0 || probs[j].N * g[best] > probs[best].N * g[j])) best = j;
    if (best < 0) break;  // every product has one CTA per ring stage
    ++g[best];
  }
  p.cta0[0] = 0;
  for (int j = 0; j < kGemvMaxGroup; ++j) p.cta0[j + 1] = p.cta0[j] + (j < count ? g[j] : 0);
  for (int j = count; j < kGemvMaxGroup; ++j) p.prob[j] = p.prob[0];
  *grid = p.cta0[count];
  *smem = gemv_layout(K, p.stage_bytes, p.stages, kGemvSwCache, km, xelem).total;
  return cudaSuccess;
}

template <bool kWO>
static cudaError_t launch_gemv_scheme(ql_scheme scheme, const GemvParams& p, int grid, size_t smem,
                                      cudaStream_t st) {
  switch (scheme) {
    case QL_W8A8_INT8_ROW:
      return kWO ? launch_gemv_wo_t<QL_W8A8_INT8_ROW>(p, grid, smem, st)
                 : launch_gemv_t<QL_W8A8_INT8_ROW>(p, grid, smem, st);
    case QL_FP8_E4M3_ROW:
      return kWO ? launch_gemv_wo_t<QL_FP8_E4M3_ROW>(p, grid, smem, st)
                 : launch_gemv_t<QL_FP8_E4M3_ROW>(p, grid, smem, st);
    default:
      return kWO ? launch_gemv_wo_t<QL_FP8_E4M3_BLOCK128>(p, grid, smem, st)
                 : launch_gemv_t<QL_FP8_E4M3_BLOCK128>(p, grid, smem, st);
  }
}

cudaError_t launch_gemv(ql_scheme scheme, const uint16_t* x, const void* wq, const float* sw,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, const ql_debug* dbg,
                        int num_sms, DevStatus* status, cudaStream_t st, bool stall) {
  if (M < 1 || M > 4 || K > gemv_max_k_tokens(M)) return cudaErrorInvalidValue;
  const ql_gemv_problem one{x, nullptr, nullptr, wq, sw, y, N};
  GemvParams p;
  int grid = 0;
  size_t smem = 0;
  cudaError_t e = gemv_setup(p, M, &one, 1, K, 1, num_sms, &grid, &smem);
  if (e != cudaSuccess) return e;
  p.dbg = dbg ? *dbg : ql_debug{nullptr, nullptr, nullptr, nullptr};
  p.status = status;
  p.stall = stall ? 1 : 0;
  return launch_gemv_scheme<false>(scheme, p, grid, smem, st);
}

cudaError_t launch_gemv_grouped(ql_scheme scheme, const ql_gemv_problem* probs, int count, int64_t M,
                                int64_t K, int num_sms, DevStatus* status, cudaStream_t st) {
  if (M < 1 || M > 4 || K > gemv_max_k_tokens(M)) return cudaErrorInvalidValue;
  GemvParams p;
  int grid = 0;
  size_t smem = 0;
  cudaError_t e = gemv_setup(p, M, probs, count, K, 1, num_sms, &grid, &smem);
  if (e != cudaSuccess) return e;
  p.dbg = ql_debug{nullptr, nullptr, nullptr, nullptr};
  p.status = status;
  p.stall = 0;
  return launch_gemv_scheme<false>(scheme, p, grid, smem, st);
}

cudaError_t launch_gemv_token_halves(ql_scheme scheme, const uint16_t* x, const ql_gemm_problem* probs,
                                     int count, int64_t M, int64_t K, int num_sms, DevStatus* status,
                                     cudaStream_t st) {
  if (M < 5 || M > 8 || K > kGemvMaxK4 || count < 1 || 2 * count > kGemvMaxGroup) return cudaErrorInvalidValue;
  // Each product becomes two products of the same weights: tokens 0-3 and
  // tokens 4 .. M-1.  The two get the same number of CTAs, so CTA b of each
  // streams the same weight rows at about the same time and the second read
  // of a row is mostly served by L2 (the SMs still take in the weight bytes
  // twice: worth it only while the launch's fixed cost dominates).
  ql_gemv_problem g[kGemvMaxGroup];
  int Ms[kGemvMaxGroup];
  for (int j = 0; j < count; ++j) {
    const ql_gemm_problem& q = probs[j];
    g[2 * j] = ql_gemv_problem{x, nullptr, nullptr, q.wq, q.sw, q.y, q.N};
    g[2 * j + 1] = ql_gemv_problem{x + 4 * K, nullptr, nullptr, q.wq, q.sw, q.y + 4 * q.N, q.N};
    Ms[2 * j] = 4;
    Ms[2 * j + 1] = (int)M - 4;
  }
  GemvParams p;
  int grid = 0;
  size_t smem = 0;
  cudaError_t e = gemv_setup(p, 4, g, 2 * count, K, 1, num_sms, &grid, &smem, Ms);
  if (e != cudaSuccess) return e;
  p.dbg = ql_debug{nullptr, nullptr, nullptr, nullptr};
  p.status = status;
  p.stall = 0;
  return launch_gemv_scheme<false>(scheme, p, grid, smem, st);
}

int gemv_weight_only_max_k_tokens(int64_t M) {
  // the largest K (a multiple of 16) whose staged f16 tokens and two ring
  // stages fit the shared memory, found once per token count
  static int cache[5] = {-1, -1, -1, -1, -1};
  if (M < 1 || M > 4) return 0;
  if (cache[M] < 0) {
    int best = 0;
    for (int64_t K = 16; K <= kGemvMaxKWO; K += 16) {
      GemvParams p;
      int grid = 0;
      size_t smem = 0;
      const ql_gemv_problem one{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 128};
      if (gemv_setup(p, M, &one, 1, K, 2, 148, &grid, &smem) == cudaSuccess &&
          (M > 1 || p.seg_len <= 32 * 64))
        best = (int)K;
    }
    cache[M] = best;
  }
  return cache[M];
}

cudaError_t launch_gemv_weight_only(ql_scheme scheme, const uint16_t* x, const void* wq,
                                    const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                    int num_sms, DevStatus* status, cudaStream_t st) {
  if (M < 1 || M > 4 || K > kGemvMaxKWO) return cudaErrorNotSupported;
  const ql_gemv_problem one{x, nullptr, nullptr, wq, sw, y, N};
  GemvParams p;
  int grid = 0;
  size_t smem = 0;
  // the staged f16 tokens and two ring stages must fit the shared memory
  if (gemv_setup(p, M, &one, 1, K, 2, num_sms, &grid, &smem) != cudaSuccess) return cudaErrorNotSupported;
  p.dbg = ql_debug{nullptr, nullptr, nullptr, nullptr};
  p.status = status;
  p.stall = 0;
  return launch_gemv_scheme<true>(scheme, p, grid, smem, st);
}

}  // namespace ql
