// ql_common.cuh -- device helpers shared by the qlinear kernels (sm_100a).
//
// Hand-written inline PTX for the pieces the kernels need: mbarriers with
// bounded waits, bulk and tensor (TMA) copies, E4M3 / bf16 conversions and the
// device status word.  Nothing here allocates memory.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlinear.h"

#define QL_DEVINL __device__ __forceinline__

namespace ql {

// ---------------------------------------------------------------------------
// Status word: kernels that give up a bounded wait record where, and return.
// ---------------------------------------------------------------------------
struct DevStatus {
  unsigned int code;    // 0 = ok, else a ql_status
  unsigned int detail;  // kernel id << 8 | wait site
};

enum KernelId : unsigned int {
  KID_GEMV = 1,
  KID_GEMM = 2,
  KID_GEMM_SMALL = 3,
};

// Wall-clock bound of one wait: a kernel that waits longer than this on a
// barrier records QL_ERR_TIMEOUT instead of waiting for ever.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

QL_DEVINL unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

QL_DEVINL void record_timeout(DevStatus* st, unsigned int kid, unsigned int site) {
  if (st && atomicCAS(&st->code, 0u, (unsigned int)QL_ERR_TIMEOUT) == 0u)
    atomicExch(&st->detail, (kid << 8) | site);
}

// ---------------------------------------------------------------------------
// Shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
QL_DEVINL uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

QL_DEVINL void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Make mbarrier initialisation visible to the async (TMA / tensor core) proxy.
QL_DEVINL void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

QL_DEVINL void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

QL_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

QL_DEVINL void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

QL_DEVINL bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Returns
// false if it has not completed within kWaitLimitNs, or if *abort becomes
// non-zero (another role of the CTA gave up first).
QL_DEVINL bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  unsigned long long t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    if ((i & 255u) == 0u) {
      if (abort && *abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
  }
}

// ---------------------------------------------------------------------------
// Bulk copies (TMA engine)
// ---------------------------------------------------------------------------
QL_DEVINL uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

QL_DEVINL uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Contiguous global -> shared copy completing on `bar` (16-byte aligned
// addresses, size a multiple of 16).
QL_DEVINL void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar,
                        uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---------------------------------------------------------------------------
// Named barriers (a subset of the CTA's warps)
// ---------------------------------------------------------------------------
QL_DEVINL void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Number formats
// ---------------------------------------------------------------------------
QL_DEVINL float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
QL_DEVINL float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// f32 -> bf16 bits, round to nearest even (hardware cvt).
QL_DEVINL uint16_t f32_to_bf16_rn(float f) {
  uint16_t h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}

// Two f32 -> two E4M3 codes, round to nearest even, saturating to +-448.
// Returns the codes in bits [7:0] (lo) and [15:8] (hi).
QL_DEVINL uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 codes (bits [7:0], [15:8]) -> f16x2 (exact: every E4M3 value is an f16).
QL_DEVINL uint32_t e4m3x2_to_f16x2(uint16_t c) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(c));
  return r;
}

QL_DEVINL float f16_lo_to_f32(uint32_t h2) {
  float f;
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; cvt.f32.f16 %0, l; }" : "=f"(f) : "r"(h2));
  return f;
}
QL_DEVINL float f16_hi_to_f32(uint32_t h2) {
  float f;
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; cvt.f32.f16 %0, h; }" : "=f"(f) : "r"(h2));
  return f;
}

// Quantization of one 16-byte chunk (8 bf16 values) with one scale s:
// int8 code clamp(rne(x/s), -127, 127) or E4M3 code of x/s, x/s the
// correctly rounded f32 quotient (the value one IEEE division gives); a zero
// scale (all-zero token, group or row) gives codes 0.
//
// For 2^-100 <= s <= 2^100 ("fast" scales) the quotient takes the correctly
// rounded reciprocal r of s and two correction steps of Markstein's method
// (P. W. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Develop. 34(1), 1990): q = x r, then
// q <- q + (x - s q) r twice, the residual exact through an FMA.  The code is
// branch-free, so the eight values of a chunk run side by side.  Other scales
// take the IEEE division.  The GPU tests compare the codes bit for bit with
// codes from IEEE division on every bf16 x at scales on both sides of the
// range.
struct Divisor {
  float s, r;
  bool fast;
};
QL_DEVINL Divisor make_divisor(float s) {
  Divisor d;
  d.s = s;
  d.fast = s >= 0x1p-100f && s <= 0x1p100f;
  d.r = d.fast ? __frcp_rn(s) : 0.0f;
  return d;
}

// x / s for a fast scale; the sign of a zero result is not fixed here.
QL_DEVINL float quotient_fast(float x, const Divisor& d) {
  float q = __fmul_rn(x, d.r);
  float e = __fmaf_rn(-q, d.s, x);
  q = __fmaf_rn(e, d.r, q);
  e = __fmaf_rn(-q, d.s, x);
  return __fmaf_rn(e, d.r, q);
}

// int8 code in bits [7:0] (the other bits are not part of the result).
// Fast scales: clamp first (the same code for every x), then adding 1.5 * 2^23
// rounds to the nearest integer, ties to even, and leaves that integer in the
// low bits of the sum (|t| <= 127, far inside 2^22).
QL_DEVINL uint32_t int8_bits_fast(float x, const Divisor& d) {
  const float t = fminf(fmaxf(quotient_fast(x, d), -127.0f), 127.0f);
  return __float_as_uint(__fadd_rn(t, 0x1.8p23f));
}
QL_DEVINL uint32_t int8_bits_ieee(float x, const Divisor& d) {
  const int q = __float2int_rn(d.s > 0.0f ? x / d.s : 0.0f);
  return (uint32_t)max(-127, min(127, q));
}
// The correctly rounded quotient of a finite x by s > 0 has the sign of x,
// which also decides the E4M3 code of a zero (0x00 / 0x80).
QL_DEVINL float e4m3_quotient_fast(float x, const Divisor& d) {
  return copysignf(quotient_fast(x, d), x);
}
QL_DEVINL float e4m3_quotient_ieee(float x, const Divisor& d) {
  return d.s > 0.0f ? x / d.s : 0.0f;
}

// Bytes [7:0] of a, b, c, d -> one word, a in the lowest byte.
QL_DEVINL uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

template <bool kInt8, bool kFast>
QL_DEVINL uint2 quant_chunk8(const uint4& v, const Divisor& d) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = bf16_lo(w[j]);
    f[2 * j + 1] = bf16_hi(w[j]);
  }
  uint32_t o[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float* g = f + 4 * h;
    if constexpr (kInt8) {
      if constexpr (kFast)
        o[h] = pack_low_bytes(int8_bits_fast(g[0], d), int8_bits_fast(g[1], d),
                              int8_bits_fast(g[2], d), int8_bits_fast(g[3], d));
      else
        o[h] = pack_low_bytes(int8_bits_ieee(g[0], d), int8_bits_ieee(g[1], d),
                              int8_bits_ieee(g[2], d), int8_bits_ieee(g[3], d));
    } else {
      if constexpr (kFast)
        o[h] = __byte_perm(f32x2_to_e4m3x2(e4m3_quotient_fast(g[0], d), e4m3_quotient_fast(g[1], d)),
                           f32x2_to_e4m3x2(e4m3_quotient_fast(g[2], d), e4m3_quotient_fast(g[3], d)),
                           0x5410);
      else
        o[h] = __byte_perm(f32x2_to_e4m3x2(e4m3_quotient_ieee(g[0], d), e4m3_quotient_ieee(g[1], d)),
                           f32x2_to_e4m3x2(e4m3_quotient_ieee(g[2], d), e4m3_quotient_ieee(g[3], d)),
                           0x5410);
    }
  }
  return make_uint2(o[0], o[1]);
}

// Either path, chosen per chunk (uniform where the scale is).
template <bool kInt8>
QL_DEVINL uint2 quant_chunk8(const uint4& v, const Divisor& d) {
  return d.fast ? quant_chunk8<kInt8, true>(v, d) : quant_chunk8<kInt8, false>(v, d);
}

// Largest |x| of one chunk of 8 bf16.
QL_DEVINL float absmax_chunk8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  return a;
}

QL_DEVINL float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace ql
