// The order, buckets and min-p threshold of the support program, shared by the
// per-row resolver and the vocabulary-parallel merge ("Consolidate
// sampling-transform scoring on one shared chunked core", xorl PR 74, "What
// this PR does", item 1: tokens ordered by (s desc, id asc), min-p against the
// unfiltered row max).
//
//   key32(s)     a monotone 32-bit key of the fp32 logit (-0 and +0 equal)
//   ckey(s, id)  (key32(s) << 32) | (2^32 - 1 - id): distinct per token, and
//                "earlier in the order" is "larger key"
//   bin0(s, m)   floor((m - s) * 128) clamped to [0, 4095]: monotone in s, so
//                every bucket is a contiguous run of the order
//   min_p_threshold_key(m, mu)  the smallest fp32 t (as a key) with
//                exp(t - m) >= mu in float64
#pragma once

#include <cfloat>
#include <cstdint>
#include <cmath>

namespace sts {
namespace {

constexpr int NB = 4096;            // histogram buckets per level
constexpr float BIN_SCALE = 128.f;  // level-0 buckets per logit unit

__device__ __forceinline__ uint32_t key32(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;  // -0 and +0 are the same logit
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key32_value(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ unsigned long long ckey(float s, int id) {
  return ((unsigned long long)key32(s) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)id);
}

__device__ __forceinline__ float ckey_value(unsigned long long K) { return key32_value((uint32_t)(K >> 32)); }

__device__ __forceinline__ int ckey_id(unsigned long long K) {
  return (int)(0xFFFFFFFFu - (uint32_t)(K & 0xFFFFFFFFull));
}

// Level-0 bucket of s: floor((m - s) * 128) clamped to [0, NB - 1]. The floor
// takes no conversion instruction: adding 2^23 rounding toward -inf leaves
// floor(f) in the low mantissa bits (f < 2^23, one unit per ulp).
__device__ __forceinline__ int bin0(float s, float m) {
  // fma(s, -128, 128 m) rounds 128 (m - s) once, which equals 128 fl(m - s):
  // scaling by a power of two commutes with rounding
  const float f = fminf(fmaxf(fmaf(s, -BIN_SCALE, m * BIN_SCALE), 0.0f), (float)(NB - 1));
  return __float_as_int(__fadd_rd(f, 8388608.0f)) - 0x4B000000;
}

// Smallest fp32 t (as a key) with exp(t - m) >= mu, mu in (0, 1]: start at
// the fp32 value nearest m + ln(mu), walk a few keys to the boundary, and
// finish by bisection over fp32 bit patterns if the walk did not close it.
__device__ __noinline__ uint32_t min_p_threshold_key(float m, float mu) {
  const double md = (double)m, mud = (double)mu;
  auto keep = [&](uint32_t k) { return exp((double)key32_value(k) - md) >= mud; };
  uint32_t lo = key32(-FLT_MAX), hi = key32(m);  // keep(lo) false, keep(hi) true
  if (exp((double)(-FLT_MAX) - md) >= mud) return lo;
  const double t0 = md + log(mud);
  uint32_t k0 = key32(t0 > -FLT_MAX ? (float)t0 : -FLT_MAX);
  if (k0 <= lo) k0 = lo + 1;
  if (k0 > hi) k0 = hi;
  if (keep(k0)) {
    hi = k0;
    for (int i = 0; i < 8 && hi - lo > 1; ++i) {
      if (keep(hi - 1)) {
        --hi;
      } else {
        lo = hi - 1;
        break;
      }
    }
  } else {
    lo = k0;
    for (int i = 0; i < 8 && hi - lo > 1; ++i) {
      if (!keep(lo + 1)) {
        ++lo;
      } else {
        hi = lo + 1;
        break;
      }
    }
  }
  while (hi - lo > 1u) {
    const uint32_t mid = lo + (hi - lo) / 2u;
    if (keep(mid))
      hi = mid;
    else
      lo = mid;
  }
  return hi;
}

}  // namespace
}  // namespace sts
