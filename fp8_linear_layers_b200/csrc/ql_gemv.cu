// ql_gemv.cu -- M = 1 decode product y = (s_x s_w) . (Q(x) . W_q^T), one kernel.
//
// "Llama 3.1 8B Instruct W8A8", "Loading": a single token runs "one row in a
// kernel that reads each byte once"; "Qwen3 8B FP8", "Loading": the same for
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
//  * The products run on the tensor cores with mma.sync m16n8k32 (s8 x s8 ->
//    s32, exact; or E4M3 x E4M3 -> f32): the stage's rows are the MMA's 8
//    columns, the token is row 0 of its 16 rows.  The k order inside each
//    64-byte window is permuted identically for x and W so that every lane
//    loads 16 contiguous bytes; a dot product does not depend on the order.
//    Each warp owns a fixed range of 64-byte k windows of every row.
//  * No CTA-wide barrier per stage: each warp parks its 8 row partials in a
//    per-stage slot and counts itself in; the last warp adds the slots in a
//    fixed order, applies the scales, writes y and releases the stage.
//  * Every wait is bounded; a warp that gives up raises a CTA abort flag that
//    every other wait checks, so all roles leave without further barriers.
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
constexpr int kGemvSmemBudget = 200 * 1024;     // one CTA per SM
constexpr int kGemvMaxK = 32768;
constexpr int kGemvRows = 8;                    // rows per stage at most (the MMA's N)
constexpr int kGemvSwCache = 2048;              // row scales kept in shared memory
constexpr uint32_t kBarConsumers = 1;           // named barrier of the consumer warps

struct GemvParams {
  const uint16_t* x;
  const uint8_t* wq;
  const float* sw;
  uint16_t* y;
  int64_t N, K;
  int rows_per_stage;  // R_s: whole rows per ring stage (1, 2, 4 or 8; the kernel's kRs)
  int stage_bytes;     // R_s * K rounded up to 128
  int stages;          // ring depth
  int64_t seg_len;     // bytes per unit segment: ceil(K R_s / 8) rounded up to 128
  ql_debug dbg;
  DevStatus* status;
};

struct GemvSmemLayout {
  int ring, qx, sx, swc, part, bars, flags, total;
};

// Shared-memory carve-up; `sw_floats` is the number of weight scales cached.
__host__ __device__ inline GemvSmemLayout gemv_layout(int64_t K, int stage_bytes, int stages,
                                                      int sw_floats) {
  GemvSmemLayout L;
  int off = 0;
  L.ring = off;
  off += stages * stage_bytes;
  L.qx = off;  // K codes, padded to whole 64-byte windows
  off += (int)((K + 127) / 128) * 128;
  L.sx = off;
  off += (int)((K / 128 + 1 + 31) / 32) * 128;
  L.swc = off;
  off += (sw_floats + 31) / 32 * 128;
  L.part = off;  // [stages][8 warps][8 rows] partial sums
  off += kGemvMaxStages * kGemvWarps * kGemvRows * 4;
  L.bars = off;  // full[stages], empty[stages], x ready
  off += 2 * kGemvMaxStages * 8 + 8;
  L.flags = off;  // abort flag, per-stage arrival counters, block reduction scratch
  off += 16 + kGemvMaxStages * 4 + kGemvWarps * 4;
  L.total = (off + 127) / 128 * 128;
  return L;
}

// Plain 16-byte shared-memory load: ordered after the barrier waits (which
// clobber memory), free to be scheduled ahead of the tensor-core instructions.
QL_DEVINL uint4 ld_s128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// D[16x8] += A[16x32] * B[32x8]; A rows 1..15 are zero here (one token).
template <bool kInt8>
QL_DEVINL void mma_16832(uint32_t (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  if constexpr (kInt8) {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  } else {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  }
}

template <ql_scheme kScheme, int kRs>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
  constexpr bool kInt8 = kScheme == QL_W8A8_INT8_ROW;
  constexpr bool kBlock = kScheme == QL_FP8_E4M3_BLOCK128;

  extern __shared__ __align__(1024) uint8_t smem[];
  const int64_t N = p.N, K = p.K;
  const int G = gridDim.x;
  const int64_t row_begin = ((int64_t)blockIdx.x * N) / G;
  const int64_t row_end = ((int64_t)(blockIdx.x + 1) * N) / G;
  const int64_t KB = K / 128;
  // weight scales this CTA needs: its rows (row schemes) or its 128-row blocks
  const int64_t sw_first = kBlock ? (row_begin >> 7) * KB : row_begin;
  const int64_t sw_count = kBlock ? (((row_end - 1) >> 7) - (row_begin >> 7) + 1) * KB : row_end - row_begin;
  const int sw_cached = (int)min(sw_count, (int64_t)kGemvSwCache);
  const int nst = p.stages;
  const GemvSmemLayout L = gemv_layout(K, p.stage_bytes, nst, kGemvSwCache);
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
  const int nstages = (int)((row_end - row_begin + kRs - 1) / kRs);
  // A ragged row count puts its partial stage first, so that it streams with
  // the first full stages instead of adding one stage of latency at the end.
  const int lead = (int)((row_end - row_begin) % kRs);
  auto stage_r0 = [&](int i) -> int64_t {
    return lead == 0 ? row_begin + (int64_t)i * kRs
                     : (i == 0 ? row_begin : row_begin + lead + (int64_t)(i - 1) * kRs);
  };
  auto stage_rows = [&](int i) -> int { return (lead != 0 && i == 0) ? lead : kRs; };

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
    if (lane == 0) {
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
  // 0. The CTA's weight scales into shared memory (immutable inputs: no wait).
  for (int i = tid; i < sw_cached; i += kGemvConsumers) sw_s[i] = __ldg(p.sw + sw_first + i);

  tc::grid_dependency_wait();  // x may be produced by the previous kernel
  // 1. Fused activation quantization of x [1, K] into shared memory: one pass
  //    for the absmax (the first kXLoads chunks per thread loaded together),
  //    one for the codes (x is L2-resident by then).
  {
    const int64_t nchunk8 = K / 8;  // 16-byte chunks of 8 bf16
    constexpr int kXLoads = 8;
    const uint4* xg = reinterpret_cast<const uint4*>(p.x);
    if (kBlock) {
      // 16 consecutive chunks (lanes) form one 128-wide group: no CTA barrier
      for (int64_t base = 0; base < nchunk8; base += kGemvConsumers) {
        const int64_t c = base + tid;
        const uint4 v = c < nchunk8 ? __ldg(xg + c) : make_uint4(0, 0, 0, 0);
        float a = absmax_chunk8(v);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const float s = a / 448.0f;
        if (c < nchunk8) {
          if ((lane & 15) == 0) sx_s[c >> 4] = s;
          reinterpret_cast<uint2*>(qx_s)[c] = quant_chunk8<false>(v, make_divisor(s));
        }
      }
    } else {
      float a_tok = 0.0f;
#pragma unroll
      for (int i = 0; i < kXLoads; ++i) {
        const int64_t c = tid + (int64_t)i * kGemvConsumers;
        a_tok = fmaxf(a_tok, absmax_chunk8(c < nchunk8 ? __ldg(xg + c) : make_uint4(0, 0, 0, 0)));
      }
      for (int64_t c = tid + (int64_t)kXLoads * kGemvConsumers; c < nchunk8; c += kGemvConsumers)
        a_tok = fmaxf(a_tok, absmax_chunk8(__ldg(xg + c)));
      a_tok = warp_max(a_tok);
      if (lane == 0) blockred[warp] = a_tok;
      named_bar_sync(kBarConsumers, kGemvConsumers);
      float a = blockred[0];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, blockred[w]);
      const float s = a / (kInt8 ? 127.0f : 448.0f);
      if (tid == 0) sx_s[0] = s;
      const Divisor dv = make_divisor(s);
      // one uniform branch: the eight values of every chunk run side by side
      auto emit_all = [&](auto fast) {
        constexpr bool kFast = decltype(fast)::value;
        // a rolled loop re-reading x (L2-resident): the straight-line form
        // measured slower inside a step, where its instructions are fetched
        // while the weight stream congests L2
        uint2* q2 = reinterpret_cast<uint2*>(qx_s);
#pragma unroll 1
        for (int64_t c = tid; c < nchunk8; c += 2 * kGemvConsumers) {
          const int64_t c2 = c + kGemvConsumers;
          const uint4 v0 = __ldg(xg + c);
          const uint4 v1 = c2 < nchunk8 ? __ldg(xg + c2) : make_uint4(0, 0, 0, 0);
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
      *reinterpret_cast<uint4*>(qx_s + b) = make_uint4(0, 0, 0, 0);
    named_bar_sync(kBarConsumers, kGemvConsumers);
  }
  if (tid == 0) mbar_arrive(xready);  // the producer may fill the whole ring now
  if (blockIdx.x == 0 && (p.dbg.qx || p.dbg.sx)) {
    for (int64_t c = tid; c < K / 16; c += kGemvConsumers)
      if (p.dbg.qx) reinterpret_cast<uint4*>(p.dbg.qx)[c] = reinterpret_cast<const uint4*>(qx_s)[c];
    const int ns = kBlock ? (int)KB : 1;
    for (int i = tid; i < ns; i += kGemvConsumers)
      if (p.dbg.sx) p.dbg.sx[i] = sx_s[i];
  }

  // 2. Work split.  A stage holds kRs (1, 2, 4 or 8) whole rows and the
  //    MMA's 8 columns are the stage's 8 units: unit j = (row j / kQ, segment
  //    j % kQ), kQ = 8 / kRs, segment q covering bytes [q seg, (q+1) seg) of
  //    its row.  Row j of A carries the x bytes that unit j meets, so D[j][j]
  //    is unit j's partial, held by one lane, and the other products are
  //    discarded.  A step feeds one 64-byte window of every unit; odd units
  //    take the two windows of each pair in swapped order, so that the lanes
  //    of one shared-memory phase (units 2p and 2p+1) read opposite halves of
  //    the banks.  Each warp owns the same steps of every stage, so its x
  //    fragments stay in registers for the whole kernel.  The block scheme
  //    splits whole window pairs (128-byte groups) so that each group's
  //    partial is scaled alone.
  constexpr int kQ = 8 / kRs;
  constexpr int kMaxSteps = 64 / kGemvWarps;  // steps per warp (a unit has <= 64 windows)
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
  const int nsteps = st1 - st0;           // <= kMaxSteps (segW <= 64)
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const int ur = g / kQ, uq = g % kQ;     // this lane's unit: row ur, segment uq
  const int flip = g & 1;                 // odd units swap the windows of each pair
  const int e = g & 1;                    // D[g][g] is element e of this lane's pair
  const bool diag = t == (g >> 1);        // this lane holds D[g][g]
  const int64_t ulen = min(seg, K - (int64_t)uq * seg);  // unit bytes inside K
  uint4 xr[kMaxSteps];
  uint32_t vmask = 0;  // steps whose 16 bytes of this lane lie inside the unit
#pragma unroll
  for (int s = 0; s < kMaxSteps; ++s) {
    const int64_t off = (int64_t)((st0 + s) ^ flip) * 64 + t * 16;
    const bool v = s < nsteps && off < ulen;
    xr[s] = v ? ld_s128(qx_s + (int64_t)uq * seg + off) : make_uint4(0, 0, 0, 0);
    vmask |= (uint32_t)v << s;
  }
  const float sx_tok = kBlock ? 0.0f : sx_s[0];
  float sxr[kMaxSteps / 2];  // block scheme: x scale of each pair's 128-wide group
  int64_t grp0 = 0;
  if constexpr (kBlock) {
    grp0 = ((int64_t)uq * seg + (int64_t)st0 * 64) / 128;
#pragma unroll
    for (int m = 0; m < kMaxSteps / 2; ++m) sxr[m] = sx_s[min(grp0 + m, KB - 1)];
  }
  const uint32_t w_lane = (uint32_t)(ur * K + (int64_t)uq * seg + t * 16);

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
    const uint32_t vm = ur < nr ? vmask : 0u;  // a unit past the stage's rows has no data
    float kept;                                // this lane's unit partial (diagonal lanes)
    if constexpr (!kBlock) {
      // four accumulators: consecutive MMAs do not wait on each other
      // Always kMaxSteps steps: a step past this warp's range has zero x and
      // W fragments and adds nothing (a uniform branch per step measured 2x
      // slower than the spare MMAs).
      uint32_t d[4][4] = {};
#pragma unroll
      for (int s = 0; s < kMaxSteps; ++s) {
        const uint4 wv = (vm >> s) & 1u ? ld_s128(wb + ((st0 + s) ^ flip) * 64) : make_uint4(0, 0, 0, 0);
        mma_16832<kInt8>(d[2 * (s & 1)], xr[s].x, xr[s].y, wv.x, wv.y);
        mma_16832<kInt8>(d[2 * (s & 1) + 1], xr[s].z, xr[s].w, wv.z, wv.w);
      }
      uint32_t de[4];  // element e of each accumulator (selects: no local memory)
#pragma unroll
      for (int a = 0; a < 4; ++a) de[a] = e ? d[a][1] : d[a][0];
      if constexpr (kInt8)  // carried bit-for-bit through the float slot, summed as int32
        kept = __int_as_float((int)(de[0] + de[1] + de[2] + de[3]));
      else
        kept = (__uint_as_float(de[0]) + __uint_as_float(de[1])) +
               (__uint_as_float(de[2]) + __uint_as_float(de[3]));
    } else {
      // per 128-wide group (a window pair): its own partial, scaled by
      // s_x[group] * s_w[row block, group]
      const int64_t ublk = (min(r0 + ur, row_end - 1) >> 7) * KB - sw_first;
      float res = 0.0f;
#pragma unroll
      for (int m = 0; m < kMaxSteps / 2; ++m) {
        {  // pairs past this warp's range have zero fragments and add nothing
          uint32_t d[4][4] = {};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int s = 2 * m + h;
            const uint4 wv = (vm >> s) & 1u ? ld_s128(wb + ((st0 + s) ^ flip) * 64) : make_uint4(0, 0, 0, 0);
            mma_16832<false>(d[2 * h], xr[s].x, xr[s].y, wv.x, wv.y);
            mma_16832<false>(d[2 * h + 1], xr[s].z, xr[s].w, wv.z, wv.w);
          }
          uint32_t de[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) de[a] = e ? d[a][1] : d[a][0];
          const float pg = (__uint_as_float(de[0]) + __uint_as_float(de[1])) +
                           (__uint_as_float(de[2]) + __uint_as_float(de[3]));
          const int64_t si = ublk + min(grp0 + m, KB - 1);
          const float swv = si < sw_cached ? sw_s[si] : __ldg(p.sw + sw_first + si);
          res = fmaf(pg, sxr[m] * swv, res);
        }
      }
      kept = res;
    }
    // Park the unit partial, then count in.
    float* ps = part + slot * kGemvWarps * kGemvRows;
    if (diag) ps[warp * kGemvRows + g] = kept;
    __syncwarp();
    int before = 0;
    if (lane == 0) {
      __threadfence_block();
      before = atomicAdd(&arrivals[slot], 1);
    }
    before = __shfl_sync(0xffffffffu, before, 0);
    if (before == kGemvWarps - 1) {
      // last warp of this stage: every warp has read the stage and parked its
      // partials.  Lane (wg, u) adds warps wg, wg + 4, ... of unit u; the
      // lanes then add across warp groups and across the kQ units of each
      // row, in a fixed order.
      __threadfence_block();
      const int u = lane & 7, wg = lane >> 3;
      int vi = 0;
      float vf = 0.0f;
#pragma unroll
      for (int w = wg; w < kGemvWarps; w += 4) {
        if constexpr (kInt8)
          vi += __float_as_int(ps[w * kGemvRows + u]);
        else
          vf += ps[w * kGemvRows + u];
      }
      if constexpr (kInt8) {
        vi += __shfl_xor_sync(0xffffffffu, vi, 8);
        vi += __shfl_xor_sync(0xffffffffu, vi, 16);
#pragma unroll
        for (int o = 1; o < kQ; o <<= 1) vi += __shfl_xor_sync(0xffffffffu, vi, o);
      } else {
        vf += __shfl_xor_sync(0xffffffffu, vf, 8);
        vf += __shfl_xor_sync(0xffffffffu, vf, 16);
#pragma unroll
        for (int o = 1; o < kQ; o <<= 1) vf += __shfl_xor_sync(0xffffffffu, vf, o);
      }
      const int r = u / kQ;
      if (wg == 0 && u % kQ == 0 && r < nr) {
        const int64_t n = r0 + r;
        float yv;
        if constexpr (kBlock) {
          yv = vf;
        } else {
          const int64_t si = n - row_begin;
          const float swn = si < sw_cached ? sw_s[si] : __ldg(p.sw + n);
          if constexpr (kInt8) {
            if (p.dbg.acc_i32) p.dbg.acc_i32[n] = vi;
            yv = __fmul_rn(__fmul_rn(__int2float_rn(vi), sx_tok), swn);
          } else {
            if (p.dbg.acc_f32) p.dbg.acc_f32[n] = vf;
            yv = __fmul_rn(__fmul_rn(vf, sx_tok), swn);
          }
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

int gemv_max_k() { return kGemvMaxK; }

template <ql_scheme S, int kRs>
static cudaError_t launch_gemv_r(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem<gemv_kernel<S, kRs>>((int)smem);
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
  return cudaLaunchKernelEx(&cfg, gemv_kernel<S, kRs>, p);
}

template <ql_scheme S>
static cudaError_t launch_gemv_t(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  switch (p.rows_per_stage) {
    case 1: return launch_gemv_r<S, 1>(p, grid, smem, st);
    case 2: return launch_gemv_r<S, 2>(p, grid, smem, st);
    case 4: return launch_gemv_r<S, 4>(p, grid, smem, st);
    case 8: return launch_gemv_r<S, 8>(p, grid, smem, st);
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
  // rows per stage: the largest power of two <= 8 whose stage fits the
  // ~32 KB copy size; the 8 MMA columns are then R_s rows x 8/R_s segments
  int rs = 1;
  while (rs < kGemvRows && (int64_t)(2 * rs) * K <= kGemvStageTarget) rs *= 2;
  p.rows_per_stage = rs;
  p.stage_bytes = (int)(((int64_t)rs * K + 127) / 128 * 128);
  const int fixed = gemv_layout(K, p.stage_bytes, 0, kGemvSwCache).total;
  p.stages = (int)std::min<int64_t>(kGemvMaxStages, (kGemvSmemBudget - fixed) / p.stage_bytes);
  if (p.stages < 2) return cudaErrorInvalidConfiguration;
  const int q = kGemvRows / rs;
  p.seg_len = ((K + q - 1) / q + 127) / 128 * 128;
  // the kernel keeps at most 8 steps of 64-byte windows per warp: seg <= 4096
  if (p.seg_len > 64 * 64) return cudaErrorInvalidValue;
  p.dbg = dbg ? *dbg : ql_debug{nullptr, nullptr, nullptr, nullptr};
  p.status = status;
  const int64_t stage_rows_total = (N + p.rows_per_stage - 1) / p.rows_per_stage;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms, stage_rows_total));
  const size_t smem = gemv_layout(K, p.stage_bytes, p.stages, kGemvSwCache).total;
  switch (scheme) {
    case QL_W8A8_INT8_ROW: return launch_gemv_t<QL_W8A8_INT8_ROW>(p, grid, smem, st);
    case QL_FP8_E4M3_ROW: return launch_gemv_t<QL_FP8_E4M3_ROW>(p, grid, smem, st);
    default: return launch_gemv_t<QL_FP8_E4M3_BLOCK128>(p, grid, smem, st);
  }
}

}  // namespace ql
