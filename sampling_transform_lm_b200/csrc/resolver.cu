// Row validation and the exact per-row support resolver.
//
// The resolver runs the pinned sampling-transform program ("Consolidate
// sampling-transform scoring on one shared chunked core; implement
// top-k/top-p/min-p replay for generic ce_modes", xorl PR 74, "What this PR
// does", item 1) on one row of fp32 scaled logits s[0..V) held in global
// memory (L2-resident while the CTA works on it):
//
//   order      (s desc, token id asc): every token gets a distinct 64-bit
//              composite key K = (monotone key of s) << 32 | (2^32-1 - id),
//              so "earlier in the order" is "larger K" and ties in s are
//              broken by the lower id.
//   top-k      the k-th element of the order (radix select on K, refined
//              through histograms until the boundary bucket fits in shared
//              memory, then sorted)
//   top-p      the first element whose inclusive running mass reaches
//              p * Z_k (Z_k = mass of the top-k prefix; masses are
//              exp(s - m) in float64, m the unfiltered row max)
//   min-p      the smallest fp32 threshold t with exp(t - m) >= min_p,
//              found by bisection over fp32 bit patterns; all s >= t kept
//   support    the shortest of the three prefixes; its size, mass Z_S, and
//              last element (cut) give LSE_S = m + log Z_S
//
// Level-0 buckets are uniform in (m - s): bucket = floor((m - s) * 128),
// clamped to 4095 -- monotone in s, so every bucket is a contiguous run of
// the order. A bucket too large for the 4096-entry candidate buffer is split
// again on its composite keys (12 bits per level) until it fits; the keys
// are distinct, so this ends after at most six levels.
#include <cfloat>
#include <cmath>

#include "sts_device.cuh"

namespace sts {

namespace {

constexpr int RT = 512;               // threads per resolver CTA
constexpr int NWARP = RT / 32;
constexpr int NB = 4096;              // histogram buckets per level
constexpr int CAP = 4096;             // candidate buffer (composite keys)
constexpr float BIN_SCALE = 128.f;    // level-0 buckets per logit unit
constexpr int MAX_LEVELS = 8;

struct RSmem {
  double mass[NB];
  unsigned long long cand[CAP];
  double cq[CAP];
  int cnt[NB];
  double red_d[NWARP];
  unsigned long long red_u[NWARP];
  long long red_l[NWARP];
  float red_f[NWARP];
  // broadcast slots
  double bd[4];
  long long bl[4];
  unsigned long long bu[4];
  int bi[4];
  int ncand;
};

// ---------------------------------------------------------------- keys

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

__device__ __forceinline__ int bin0(float s, float m) {
  const float f = fminf((m - s) * BIN_SCALE, (float)(NB - 1));
  const int b = (int)f;
  return b < 0 ? 0 : b;
}

__device__ __forceinline__ double qmass(float s, double m) { return exp((double)s - m); }

// ---------------------------------------------------------------- block reductions
// Fixed shuffle-down trees: results are identical on every run.

__device__ float block_max_f(float v, RSmem& sm) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_down_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sm.red_f[w] = v;
  __syncthreads();
  if (w == 0) {
    v = l < NWARP ? sm.red_f[l] : -INFINITY;
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_down_sync(0xffffffffu, v, o));
    if (l == 0) sm.red_f[0] = v;
  }
  __syncthreads();
  const float r = sm.red_f[0];
  __syncthreads();
  return r;
}

__device__ double block_sum_d(double v, RSmem& sm) {
  for (int o = 16; o; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sm.red_d[w] = v;
  __syncthreads();
  if (w == 0) {
    v = l < NWARP ? sm.red_d[l] : 0.0;
    for (int o = 16; o; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if (l == 0) sm.red_d[0] = v;
  }
  __syncthreads();
  const double r = sm.red_d[0];
  __syncthreads();
  return r;
}

__device__ long long block_sum_l(long long v, RSmem& sm) {
  for (int o = 16; o; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sm.red_l[w] = v;
  __syncthreads();
  if (w == 0) {
    v = l < NWARP ? sm.red_l[l] : 0;
    for (int o = 16; o; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if (l == 0) sm.red_l[0] = v;
  }
  __syncthreads();
  const long long r = sm.red_l[0];
  __syncthreads();
  return r;
}

template <bool kMax>
__device__ unsigned long long block_ext_u(unsigned long long v, RSmem& sm) {
  for (int o = 16; o; o >>= 1) {
    const unsigned long long x = __shfl_down_sync(0xffffffffu, v, o);
    v = kMax ? (x > v ? x : v) : (x < v ? x : v);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sm.red_u[w] = v;
  __syncthreads();
  if (w == 0) {
    v = l < NWARP ? sm.red_u[l] : (kMax ? 0ull : ~0ull);
    for (int o = 16; o; o >>= 1) {
      const unsigned long long x = __shfl_down_sync(0xffffffffu, v, o);
      v = kMax ? (x > v ? x : v) : (x < v ? x : v);
    }
    if (l == 0) sm.red_u[0] = v;
  }
  __syncthreads();
  const unsigned long long r = sm.red_u[0];
  __syncthreads();
  return r;
}

// Exclusive scan over threads in thread order (deterministic).
template <typename T>
__device__ T block_exscan(T v, T* warp_tot, T& total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  T x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, x, o);
    if (l >= o) x += y;
  }
  if (l == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    T t = l < NWARP ? warp_tot[l] : T(0);
    for (int o = 1; o < 32; o <<= 1) {
      const T y = __shfl_up_sync(0xffffffffu, t, o);
      if (l >= o) t += y;
    }
    if (l < NWARP) warp_tot[l] = t;  // inclusive warp prefix
  }
  __syncthreads();
  const T before_warp = w > 0 ? warp_tot[w - 1] : T(0);
  total = warp_tot[NWARP - 1];
  __syncthreads();
  return before_warp + x - v;
}

// ---------------------------------------------------------------- selection

enum Crit : int { kCount = 0, kMassGE = 1, kMassGT = 2 };

struct Cut {
  unsigned long long K;  // composite key of the last element of the prefix
  long long cnt;         // prefix length
  double mass;           // prefix mass sum exp(s - m)
};

__device__ __forceinline__ bool crit_ok(int crit, long long c, double mss, long long need, double target) {
  return crit == kCount ? (c >= need) : (crit == kMassGE ? (mss >= target) : (mss > target));
}

// Over the NB buckets in sm.cnt / sm.mass (bucket 0 = earliest in the order),
// pick the first bucket where (above + inclusive prefix) meets the criterion,
// or the last non-empty bucket if none does. Returns it with the count and
// mass of everything before it (above included).
__device__ void pick_bucket(RSmem& sm, int crit, long long need, double target, long long above_cnt,
                            double above_mass, int& b_out, long long& cnt_excl, double& mass_excl) {
  constexpr int PER = NB / RT;
  const int base = threadIdx.x * PER;
  long long lc = 0;
  double lm = 0.0;
  int last_nz = -1;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    lc += sm.cnt[base + i];
    lm += sm.mass[base + i];
    if (sm.cnt[base + i] > 0) last_nz = base + i;
  }
  long long tc;
  double tm;
  const long long pc = block_exscan<long long>(lc, sm.red_l, tc);
  const double pm = block_exscan<double>(lm, sm.red_d, tm);
  // first satisfying bucket owned by this thread
  int mine = NB;
  {
    long long c = above_cnt + pc;
    double mss = above_mass + pm;
    for (int i = 0; i < PER; ++i) {
      c += sm.cnt[base + i];
      mss += sm.mass[base + i];
      if (sm.cnt[base + i] > 0 && crit_ok(crit, c, mss, need, target)) {
        mine = base + i;
        break;
      }
    }
  }
  int b = (int)(~block_ext_u<true>(~(unsigned long long)(unsigned)mine, sm));  // min
  if (b >= NB) b = (int)block_ext_u<true>((unsigned long long)(unsigned)(last_nz + 1), sm) - 1;
  if (b < 0) b = 0;
  if (threadIdx.x == b / PER) {
    long long c = above_cnt + pc;
    double mss = above_mass + pm;
    for (int i = base; i < b; ++i) {
      c += sm.cnt[i];
      mss += sm.mass[i];
    }
    sm.bl[0] = c;
    sm.bd[0] = mss;
  }
  __syncthreads();
  b_out = b;
  cnt_excl = sm.bl[0];
  mass_excl = sm.bd[0];
  __syncthreads();
}

// Level-0 histogram of the row (counts and float64 masses per bucket).
__device__ void build_hist0(RSmem& sm, const float* __restrict__ x, int V, float m) {
  for (int i = threadIdx.x; i < NB; i += RT) {
    sm.cnt[i] = 0;
    sm.mass[i] = 0.0;
  }
  __syncthreads();
  const double md = (double)m;
  for (int i = threadIdx.x; i < V; i += RT) {
    const float s = x[i];
    const int b = bin0(s, m);
    atomicAdd(&sm.cnt[b], 1);
    atomicAdd(&sm.mass[b], qmass(s, md));
  }
  __syncthreads();
}

// Find the element of the (s desc, id asc) order where the criterion is first
// met. Returns false (and sets *overflow) only if the refinement bound is hit.
__device__ bool locate(RSmem& sm, const float* __restrict__ x, int V, float m, bool& hist_valid,
                       int crit, long long need, double target, Cut& out) {
  const double md = (double)m;
  if (!hist_valid) {
    build_hist0(sm, x, V, m);
    hist_valid = true;
  }
  int b;
  long long above_cnt;
  double above_mass;
  pick_bucket(sm, crit, need, target, 0, 0.0, b, above_cnt, above_mass);
  long long set_cnt = sm.cnt[b];
  unsigned long long Klo = 0ull, Khi = ~0ull;
  bool refined = false;
  __syncthreads();

  for (int level = 0; set_cnt > CAP; ++level) {
    if (level >= MAX_LEVELS) return false;
    // exact key range of the current set
    unsigned long long kmin = ~0ull, kmax = 0ull;
    for (int i = threadIdx.x; i < V; i += RT) {
      const float s = x[i];
      if (bin0(s, m) != b) continue;
      const unsigned long long K = ckey(s, i);
      if (refined && (K < Klo || K > Khi)) continue;
      kmin = K < kmin ? K : kmin;
      kmax = K > kmax ? K : kmax;
    }
    Klo = block_ext_u<false>(kmin, sm);
    Khi = block_ext_u<true>(kmax, sm);
    refined = true;
    const unsigned long long span = Khi - Klo;
    const int bits = span ? 64 - __clzll((long long)span) : 0;
    const int shift = bits > 12 ? bits - 12 : 0;
    for (int i = threadIdx.x; i < NB; i += RT) {
      sm.cnt[i] = 0;
      sm.mass[i] = 0.0;
    }
    hist_valid = false;
    __syncthreads();
    for (int i = threadIdx.x; i < V; i += RT) {
      const float s = x[i];
      if (bin0(s, m) != b) continue;
      const unsigned long long K = ckey(s, i);
      if (K < Klo || K > Khi) continue;
      const int sb = (int)((Khi - K) >> shift);
      atomicAdd(&sm.cnt[sb], 1);
      atomicAdd(&sm.mass[sb], qmass(s, md));
    }
    __syncthreads();
    int c;
    long long ce;
    double me;
    pick_bucket(sm, crit, need, target, above_cnt, above_mass, c, ce, me);
    set_cnt = sm.cnt[c];
    above_cnt = ce;
    above_mass = me;
    const unsigned long long hi_off = (unsigned long long)c << shift;
    const unsigned long long lo_off = hi_off + ((1ull << shift) - 1ull);
    const unsigned long long new_hi = Khi - hi_off;
    const unsigned long long new_lo = (lo_off >= Khi - Klo) ? Klo : Khi - lo_off;
    Khi = new_hi;
    Klo = new_lo;
    __syncthreads();
  }

  // gather the boundary set
  if (threadIdx.x == 0) sm.ncand = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < V; i += RT) {
    const float s = x[i];
    if (bin0(s, m) != b) continue;
    const unsigned long long K = ckey(s, i);
    if (refined && (K < Klo || K > Khi)) continue;
    const int slot = atomicAdd(&sm.ncand, 1);
    if (slot < CAP) sm.cand[slot] = K;
  }
  __syncthreads();
  const int n = min(sm.ncand, CAP);
  int n2 = 2;
  while (n2 < n) n2 <<= 1;
  for (int i = n + (int)threadIdx.x; i < n2; i += RT) sm.cand[i] = 0ull;  // sorts last
  __syncthreads();
  // bitonic sort, descending
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += RT) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = sm.cand[i], c = sm.cand[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (a < c) : (a > c)) {
            sm.cand[i] = c;
            sm.cand[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // inclusive scan of masses in sorted order (8 per thread, thread order)
  constexpr int PER = CAP / RT;
  const int base = threadIdx.x * PER;
  double loc[PER];
  double run = 0.0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = base + i;
    const double qv = j < n ? qmass(ckey_value(sm.cand[j]), md) : 0.0;
    run += qv;
    loc[i] = run;
  }
  double tot;
  const double off = block_exscan<double>(run, sm.red_d, tot);
#pragma unroll
  for (int i = 0; i < PER; ++i) sm.cq[base + i] = off + loc[i];
  __syncthreads();

  int jstar;
  if (crit == kCount) {
    jstar = (int)(need - above_cnt - 1);
  } else {
    int mine = CAP;
    for (int i = 0; i < PER; ++i) {
      const int j = base + i;
      if (j < n && crit_ok(crit, 0, above_mass + sm.cq[j], 0, target)) {
        mine = j;
        break;
      }
    }
    jstar = (int)(~block_ext_u<true>(~(unsigned long long)(unsigned)mine, sm));
    if (jstar >= n) jstar = n - 1;
  }
  if (jstar < 0) jstar = 0;
  if (jstar > n - 1) jstar = n - 1;
  out.K = sm.cand[jstar];
  out.cnt = above_cnt + jstar + 1;
  out.mass = above_mass + sm.cq[jstar];
  __syncthreads();
  return true;
}

__device__ __forceinline__ void take_earlier(Cut& best, const Cut& c) {
  if (c.K > best.K) best = c;
}

// Smallest fp32 t (as a key) with exp(t - m) >= mu, mu in (0, 1].
__device__ uint32_t min_p_threshold_key(float m, float mu) {
  uint32_t lo = key32(-FLT_MAX), hi = key32(m);  // P(lo) false, P(hi) true
  const double md = (double)m, mud = (double)mu;
  if (exp((double)(-FLT_MAX) - md) >= mud) return lo;
  while (hi - lo > 1u) {
    const uint32_t mid = lo + (hi - lo) / 2u;
    if (exp((double)key32_value(mid) - md) >= mud)
      hi = mid;
    else
      lo = mid;
  }
  return hi;
}

__global__ void __launch_bounds__(RT) resolve_kernel(const ResolveArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RSmem& sm = *reinterpret_cast<RSmem*>(smem_raw);
  const int V = a.V;

  for (int r = blockIdx.x; r < a.rows; r += gridDim.x) {
    const float* __restrict__ x = a.S + (size_t)r * (size_t)a.ld;
    const bool invalid = a.row_flags && (a.row_flags[r] & STS_ROW_INVALID);
    if (invalid) {
      if (threadIdx.x == 0) {
        const float nan = __int_as_float(0x7fc00000);
        if (a.logprob) a.logprob[r] = nan;
        if (a.row_max) a.row_max[r] = nan;
        if (a.lse_support) a.lse_support[r] = nan;
        if (a.cut_logit) a.cut_logit[r] = nan;
        if (a.cut_id) a.cut_id[r] = -1;
        if (a.support_size) a.support_size[r] = 0;
        if (a.flags_out) a.flags_out[r] = STS_ROW_INVALID;
        if (a.sampled) a.sampled[r] = -1;
      }
      if (a.mask)
        for (int i = threadIdx.x; i < V; i += RT) a.mask[(size_t)r * V + i] = 0;
      continue;
    }

    // unfiltered row max
    float lm = -INFINITY;
    for (int i = threadIdx.x; i < V; i += RT) lm = fmaxf(lm, x[i]);
    const float m = block_max_f(lm, sm);
    const double md = (double)m;

    // level-0 histogram, total mass and the last element of the order
    build_hist0(sm, x, V, m);
    bool hist_valid = true;
    double zl = 0.0;
    unsigned long long kmin = ~0ull;
    for (int i = threadIdx.x; i < V; i += RT) {
      const float s = x[i];
      zl += qmass(s, md);
      const unsigned long long K = ckey(s, i);
      kmin = K < kmin ? K : kmin;
    }
    const double Z = block_sum_d(zl, sm);
    Cut best{block_ext_u<false>(kmin, sm), (long long)V, Z};

    const int k = a.top_k[r];
    const float p = a.top_p[r];
    const float mu = a.min_p[r];
    const bool k_on = k >= 1 && k < V;
    const bool p_on = p < 1.0f;
    const bool mu_on = mu > 0.0f;
    bool ok = true;

    double Zk = Z;
    if (k_on) {
      Cut ck;
      ok = ok && locate(sm, x, V, m, hist_valid, kCount, (long long)k, 0.0, ck);
      Zk = ck.mass;
      take_earlier(best, ck);
    }
    if (ok && p_on) {
      Cut cp;
      ok = ok && locate(sm, x, V, m, hist_valid, kMassGE, 0, (double)p * Zk, cp);
      take_earlier(best, cp);
    }
    if (ok && mu_on) {
      if (threadIdx.x == 0) sm.bi[0] = (int)min_p_threshold_key(m, mu);
      __syncthreads();
      const uint32_t kt = (uint32_t)sm.bi[0];
      __syncthreads();
      long long c = 0;
      double ms = 0.0;
      unsigned long long kl = ~0ull;
      for (int i = threadIdx.x; i < V; i += RT) {
        const float s = x[i];
        if (key32(s) >= kt) {
          ++c;
          ms += qmass(s, md);
          const unsigned long long K = ckey(s, i);
          kl = K < kl ? K : kl;
        }
      }
      Cut cm{block_ext_u<false>(kl, sm), block_sum_l(c, sm), 0.0};
      cm.mass = block_sum_d(ms, sm);
      take_earlier(best, cm);
    }

    if (!ok) {
      if (threadIdx.x == 0) {
        atomicCAS(&a.hdr->err, 0, (int)STS_ERR_OVERFLOW);
        const float nan = __int_as_float(0x7fc00000);
        if (a.logprob) a.logprob[r] = nan;
        if (a.sampled) a.sampled[r] = -1;
        if (a.support_size) a.support_size[r] = 0;
        if (a.flags_out) a.flags_out[r] = STS_ROW_INVALID;
      }
      continue;
    }

    const double lse = md + log(best.mass);
    const float cut_v = ckey_value(best.K);
    const int cut_i = ckey_id(best.K);

    if (a.mode == kModeSample) {
      Cut cs;
      const double tgt = a.u[r] * best.mass;
      const bool ok2 = locate(sm, x, V, m, hist_valid, kMassGT, 0, tgt, cs);
      if (!ok2 || cs.K < best.K) cs = best;
      if (threadIdx.x == 0) a.sampled[r] = ckey_id(cs.K);
    }
    if (threadIdx.x == 0) {
      if (a.support_size) a.support_size[r] = (int32_t)best.cnt;
      if (a.cut_logit) a.cut_logit[r] = cut_v;
      if (a.cut_id) a.cut_id[r] = cut_i;
      if (a.row_max) a.row_max[r] = m;
      if (a.lse_support) a.lse_support[r] = (float)lse;
      int fl = (!k_on && !p_on && !mu_on) ? STS_ROW_IDENTITY : 0;
      if (a.mode == kModeForward) {
        const long long y = a.target[r];
        const float sy = x[y];
        const bool in = ckey(sy, (int)y) >= best.K;
        if (in) fl |= STS_ROW_TARGET_IN_SUPPORT;
        a.logprob[r] = in ? (float)fmin((double)sy - lse, 0.0) : -INFINITY;
      }
      if (a.flags_out) a.flags_out[r] = fl;
    }
    if (a.mask) {
      for (int i = threadIdx.x; i < V; i += RT)
        a.mask[(size_t)r * V + i] = ckey(x[i], i) >= best.K ? 1 : 0;
    }
    __syncthreads();
  }
}

__global__ void validate_kernel(const int64_t* target, const float* temperature, const float* top_p,
                                const float* min_p, int64_t T, int64_t V, int32_t* flags,
                                WsHeader* hdr, int check_target) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= T) return;
  int code = 0;
  if (temperature) {
    const float t = temperature[r];
    if (!(t > 0.f) || !isfinite(t)) code = STS_ERR_TEMPERATURE;
  }
  if (!code) {
    const float p = top_p[r];
    if (!(p > 0.f && p <= 1.f)) code = STS_ERR_TOP_P;
  }
  if (!code) {
    const float mu = min_p[r];
    if (!(mu >= 0.f && mu <= 1.f)) code = STS_ERR_MIN_P;
  }
  if (!code && check_target) {
    const int64_t y = target[r];
    if (y < 0 || y >= V) code = STS_ERR_TARGET;
  }
  flags[r] = code ? STS_ROW_INVALID : 0;
  if (code)
    atomicMin(&hdr->bad_row_code, ((unsigned long long)r << 32) | (unsigned long long)code);
}

}  // namespace

void launch_validate(const int64_t* target, const float* temperature, const float* top_p,
                     const float* min_p, int64_t T, int64_t V, int32_t* flags, WsHeader* hdr,
                     bool check_target, cudaStream_t stream) {
  const int threads = 256;
  const int blocks = (int)((T + threads - 1) / threads);
  validate_kernel<<<blocks, threads, 0, stream>>>(target, temperature, top_p, min_p, T, V, flags,
                                                  hdr, check_target ? 1 : 0);
}

size_t resolve_smem_bytes() { return sizeof(RSmem); }

cudaError_t launch_resolve(const ResolveArgs& a, int num_sms, cudaStream_t stream) {
  const size_t smem = sizeof(RSmem);
  cudaError_t e = cudaFuncSetAttribute(resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = a.rows < num_sms ? a.rows : num_sms;
  if (grid <= 0) return cudaSuccess;
  resolve_kernel<<<grid, RT, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace sts
