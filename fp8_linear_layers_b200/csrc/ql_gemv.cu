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
//    shared memory.
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

constexpr int kGemvWarps = 8;                  // consumer warps
constexpr int kGemvConsumers = kGemvWarps * 32;
constexpr int kGemvThreads = kGemvConsumers + 32;
constexpr int kGemvMaxStages = 6;
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
  int rows_per_stage;  // R_s: whole rows per ring stage (<= 8)
  int stage_bytes;     // R_s * K rounded up to 128
  int stages;          // ring depth
  int q_segs;          // K segments per row carried by separate MMA columns (8 / rows)
  int64_t seg_len;     // bytes per segment (multiple of 64, or of 128 for blocks)
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

// D[16x8] += A[16x32] * B[32x8]; A rows 1..15 are zero here (one token).
template <bool kInt8>
QL_DEVINL void mma_16832(uint32_t (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  if constexpr (kInt8) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  }
}

template <ql_scheme kScheme, int Q>
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
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flags);
  int* arrivals = reinterpret_cast<int*>(smem + L.flags + 16);
  float* blockred = reinterpret_cast<float*>(smem + L.flags + 16 + kGemvMaxStages * 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int Rs = p.rows_per_stage;
  const int nstages = (int)((row_end - row_begin + Rs - 1) / Rs);

  if (tid == 0) {
    tc::launch_dependents();  // the next kernel's CTAs may start as SMs free up
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
  // 0. The CTA's weight scales into shared memory (immutable inputs: no wait).
  for (int i = tid; i < sw_cached; i += kGemvConsumers) sw_s[i] = __ldg(p.sw + sw_first + i);

  tc::grid_dependency_wait();  // x may be produced by the previous kernel
  // 1. Fused activation quantization of x [1, K] into shared memory.  Up to
  //    kXCache 16-byte chunks per thread stay in registers between the absmax
  //    and the rounding; longer rows re-read the rest (x sits in L2).
  {
    const int64_t nchunk8 = K / 8;  // 16-byte chunks of 8 bf16
    constexpr int kXCache = 8;
    const uint4* xg = reinterpret_cast<const uint4*>(p.x);
    uint4 xc[kXCache];
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
      for (int i = 0; i < kXCache; ++i) {
        const int64_t c = tid + (int64_t)i * kGemvConsumers;
        xc[i] = c < nchunk8 ? __ldg(xg + c) : make_uint4(0, 0, 0, 0);
        a_tok = fmaxf(a_tok, absmax_chunk8(xc[i]));
      }
      for (int64_t c = tid + (int64_t)kXCache * kGemvConsumers; c < nchunk8; c += kGemvConsumers)
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
        uint2* q2 = reinterpret_cast<uint2*>(qx_s);
#pragma unroll
        for (int i = 0; i < kXCache; ++i) {
          const int64_t c = tid + (int64_t)i * kGemvConsumers;
          if (c < nchunk8) q2[c] = quant_chunk8<kInt8, kFast>(xc[i], dv);
        }
        for (int64_t c = tid + (int64_t)kXCache * kGemvConsumers; c < nchunk8; c += kGemvConsumers)
          q2[c] = quant_chunk8<kInt8, kFast>(__ldg(xg + c), dv);
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
  if (blockIdx.x == 0 && (p.dbg.qx || p.dbg.sx)) {
    for (int64_t c = tid; c < K / 16; c += kGemvConsumers)
      if (p.dbg.qx) reinterpret_cast<uint4*>(p.dbg.qx)[c] = reinterpret_cast<const uint4*>(qx_s)[c];
    const int ns = kBlock ? (int)KB : 1;
    for (int i = tid; i < ns; i += kGemvConsumers)
      if (p.dbg.sx) p.dbg.sx[i] = sx_s[i];
  }

  // 2. Work split.  A stage holds Rs (<= 8) whole rows and the MMA has 8
  //    columns.  With Q = 8 / Rs' (Rs' = Rs rounded up to 1, 2, 4 or 8),
  //    row r's K range is cut into Q segments of seg_len bytes: column
  //    j = r * Q + q of B carries segment q of row r, row q of A carries
  //    segment q of x, so D[q][j] with q == j % Q is row r's partial over
  //    segment q (the other products are discarded).  Every column carries
  //    real bytes whatever Rs is.  Each warp owns the same local 64-byte
  //    windows [lw0, lw1) of every segment; the block scheme splits whole
  //    128-byte groups so that each group's partial is scaled alone.
  const int64_t seg = p.seg_len;  // Q (segments per row) is a template parameter
  const int64_t NWs = seg / 64;
  int64_t lw0, lw1;
  if (kBlock) {
    const int64_t GS = seg / 128;  // groups per segment
    lw0 = 2 * ((warp * GS) / kGemvWarps);
    lw1 = 2 * (((warp + 1) * GS) / kGemvWarps);
  } else {
    lw0 = (warp * NWs) / kGemvWarps;
    lw1 = ((warp + 1) * NWs) / kGemvWarps;
  }
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const int rB = g / Q, qB = g % Q;       // this lane's B column: row rB, segment qB
  const bool useful0 = g == (2 * t) % Q;      // D[g][2t] is a kept product
  const bool useful1 = g == (2 * t + 1) % Q;  // D[g][2t+1] is a kept product
  const float sx_tok = kBlock ? 0.0f : sx_s[0];
  const uint32_t qx_a = smem_u32(qx_s);
  const uint32_t ring_a = smem_u32(ring);
  // per-lane 32-bit bases and limits of the two fragments (bytes past the
  // lane's first window that still lie inside K; <= 0 means no data)
  const int x_lim = (g < Q) ? (int)(K - (int64_t)g * seg - t * 16) : 0;
  const int w_lim = (int)(K - (int64_t)qB * seg - t * 16);
  const uint32_t x_base = qx_a + (uint32_t)((int64_t)g * seg + t * 16);
  const uint32_t w_off = (uint32_t)(rB * K + (int64_t)qB * seg + t * 16);

  // 3. Stream the ring.
  for (int i = 0; i < nstages; ++i) {
    const int slot = i % nst;
    const int64_t r0 = row_begin + (int64_t)i * Rs;
    const int nr = (int)min((int64_t)Rs, row_end - r0);
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (i / nst) & 1, abort_flag))) {
      if (lane == 0 && !*abort_flag) record_timeout(p.status, KID_GEMV, 2);
      *abort_flag = 1;
      break;
    }
    const int wl = rB < nr ? w_lim : 0;  // zero unless this B column is a real row of the stage
    const uint32_t w_base = ring_a + slot * p.stage_bytes + w_off;
    float res0 = 0.0f, res1 = 0.0f;  // kept products D[g][2t], D[g][2t+1]
    if constexpr (!kBlock) {
      // four independent accumulators: consecutive MMAs do not wait on each other
      uint32_t d[4][4] = {};
      int64_t lw = lw0;
      for (; lw + 1 < lw1; lw += 2) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int off = (int)(lw + h) * 64;
          const uint4 xv = off < x_lim ? lds128(x_base + off) : make_uint4(0, 0, 0, 0);
          const uint4 wv = off < wl ? lds128(w_base + off) : make_uint4(0, 0, 0, 0);
          mma_16832<kInt8>(d[2 * h], xv.x, xv.y, wv.x, wv.y);
          mma_16832<kInt8>(d[2 * h + 1], xv.z, xv.w, wv.z, wv.w);
        }
      }
      if (lw < lw1) {
        const int off = (int)lw * 64;
        const uint4 xv = off < x_lim ? lds128(x_base + off) : make_uint4(0, 0, 0, 0);
        const uint4 wv = off < wl ? lds128(w_base + off) : make_uint4(0, 0, 0, 0);
        mma_16832<kInt8>(d[0], xv.x, xv.y, wv.x, wv.y);
        mma_16832<kInt8>(d[1], xv.z, xv.w, wv.z, wv.w);
      }
      if constexpr (kInt8) {
        // carried bit-for-bit through the float slot, summed as int32
        res0 = __int_as_float((int)(d[0][0] + d[1][0] + d[2][0] + d[3][0]));
        res1 = __int_as_float((int)(d[0][1] + d[1][1] + d[2][1] + d[3][1]));
      } else {
        res0 = (__uint_as_float(d[0][0]) + __uint_as_float(d[1][0])) +
               (__uint_as_float(d[2][0]) + __uint_as_float(d[3][0]));
        res1 = (__uint_as_float(d[0][1]) + __uint_as_float(d[1][1])) +
               (__uint_as_float(d[2][1]) + __uint_as_float(d[3][1]));
      }
    } else {
      // per 128-wide group: its own partial, scaled by s_x[group] * s_w[block, group]
      const int64_t GS = seg / 128;
      const int64_t rowA = r0 + (2 * t) / Q, rowB = r0 + (2 * t + 1) / Q;
      const int64_t bA = (min(rowA, row_end - 1) >> 7) * KB - sw_first;
      const int64_t bB = (min(rowB, row_end - 1) >> 7) * KB - sw_first;
      for (int64_t lw = lw0; lw < lw1; lw += 2) {
        uint32_t d[4][4] = {};  // independent chains inside the 128-wide group
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int off = (int)(lw + h) * 64;
          const uint4 xv = off < x_lim ? lds128(x_base + off) : make_uint4(0, 0, 0, 0);
          const uint4 wv = off < wl ? lds128(w_base + off) : make_uint4(0, 0, 0, 0);
          mma_16832<false>(d[2 * h], xv.x, xv.y, wv.x, wv.y);
          mma_16832<false>(d[2 * h + 1], xv.z, xv.w, wv.z, wv.w);
        }
        // the kept products of this lane belong to segment g: global group g*GS + lw/2
        const int64_t grp = min((int64_t)g * GS + (lw >> 1), KB - 1);
        const float sxg = sx_s[grp];
        const float swA = bA + grp < sw_cached ? sw_s[bA + grp] : __ldg(p.sw + sw_first + bA + grp);
        const float swB = bB + grp < sw_cached ? sw_s[bB + grp] : __ldg(p.sw + sw_first + bB + grp);
        const float pA = (__uint_as_float(d[0][0]) + __uint_as_float(d[1][0])) +
                         (__uint_as_float(d[2][0]) + __uint_as_float(d[3][0]));
        const float pB = (__uint_as_float(d[0][1]) + __uint_as_float(d[1][1])) +
                         (__uint_as_float(d[2][1]) + __uint_as_float(d[3][1]));
        res0 = fmaf(pA, sxg * swA, res0);
        res1 = fmaf(pB, sxg * swB, res1);
      }
    }
    // Park the kept partials (column j = r * Q + q), then count in.
    float* ps = part + slot * kGemvWarps * kGemvRows;
    if (useful0) ps[warp * kGemvRows + 2 * t] = res0;
    if (useful1) ps[warp * kGemvRows + 2 * t + 1] = res1;
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
        const int64_t n = r0 + lane;
        const int c0 = lane * Q;  // this row's columns c0 .. c0 + Q - 1
        float yv;
        if constexpr (kInt8) {
          int v = 0;
          for (int w = 0; w < kGemvWarps; ++w)
            for (int q = 0; q < Q; ++q) v += __float_as_int(ps[w * kGemvRows + c0 + q]);
          if (p.dbg.acc_i32) p.dbg.acc_i32[n] = v;
          const int64_t si = n - row_begin;
          const float swn = si < sw_cached ? sw_s[si] : __ldg(p.sw + n);
          yv = __fmul_rn(__fmul_rn(__int2float_rn(v), sx_tok), swn);
        } else {
          float v = 0.0f;
          for (int w = 0; w < kGemvWarps; ++w)
            for (int q = 0; q < Q; ++q) v += ps[w * kGemvRows + c0 + q];
          if constexpr (kBlock) {
            yv = v;
          } else {
            if (p.dbg.acc_f32) p.dbg.acc_f32[n] = v;
            const int64_t si = n - row_begin;
            const float swn = si < sw_cached ? sw_s[si] : __ldg(p.sw + n);
            yv = __fmul_rn(__fmul_rn(v, sx_tok), swn);
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

template <ql_scheme S, int Q>
static cudaError_t launch_gemv_q(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem<gemv_kernel<S, Q>>((int)smem);
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
  return cudaLaunchKernelEx(&cfg, gemv_kernel<S, Q>, p);
}

template <ql_scheme S>
static cudaError_t launch_gemv_t(const GemvParams& p, int grid, size_t smem, cudaStream_t st) {
  switch (p.q_segs) {
    case 1: return launch_gemv_q<S, 1>(p, grid, smem, st);
    case 2: return launch_gemv_q<S, 2>(p, grid, smem, st);
    case 4: return launch_gemv_q<S, 4>(p, grid, smem, st);
    case 8: return launch_gemv_q<S, 8>(p, grid, smem, st);
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
  p.rows_per_stage = (int)std::max<int64_t>(1, std::min<int64_t>(kGemvRows, kGemvStageTarget / K));
  p.stage_bytes = (int)(((int64_t)p.rows_per_stage * K + 127) / 128 * 128);
  const int fixed = gemv_layout(K, p.stage_bytes, 0, kGemvSwCache).total;
  p.stages = (int)std::min<int64_t>(kGemvMaxStages, (kGemvSmemBudget - fixed) / p.stage_bytes);
  if (p.stages < 2) return cudaErrorInvalidConfiguration;
  const int rq = p.rows_per_stage <= 1 ? 1 : p.rows_per_stage <= 2 ? 2 : p.rows_per_stage <= 4 ? 4 : 8;
  p.q_segs = kGemvRows / rq;
  const int64_t unit = scheme == QL_FP8_E4M3_BLOCK128 ? 128 : 64;
  p.seg_len = ((K + p.q_segs - 1) / p.q_segs + unit - 1) / unit * unit;
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
