// Vocabulary-parallel tensor parallelism: the rank-order gather of the
// vocabulary shards' scaled logits into full rows ("Consolidate
// sampling-transform scoring on one shared chunked core", xorl PR 74, "What
// this PR does", item 2: ordinary vocabulary-parallel body TP is handled
// inside the core; chunk-local logits are gathered in rank order, hidden
// gradients summed across vocabulary ranks, weight-shard gradients local).
//
// Two forms. The gather: after an all-gather, rank k's shard of every row
// sits in one contiguous block src[k] = [T][Vl]; the support program needs
// each row whole, so the blocks are interleaved: dst[r][k Vl + j] =
// src[k][r][j] (one read and one write of the T x (world Vl) fp32 logits).
//
// The statistics merge, which moves per-row statistics instead of logits
// (every stage is the same deterministic computation on every rank, and the
// caller combines the stages' outputs across ranks with collectives):
//   1. each rank's row maxima, combined by max: the unfiltered row max m;
//   2. each rank's 4096-bucket count histogram of floor((m - s) 128),
//      combined by sum;
//   3. from the merged counts every rank plans the same row: the bucket of the
//      k-th element (top-k), a bracket of buckets that certainly holds the
//      top-p crossing (each bucket's mass lies between its count times the
//      masses of its two edges, so the running mass before every bucket and
//      the target p Z_k have rigorous bounds), and the min-p threshold key;
//      one pass over the shard then forms float64 sums (the total mass, the
//      mass before the top-k bucket and before the bracket, the mass and count
//      of the min-p-kept tokens), the smallest kept key and the smallest key
//      overall, and gathers the composite keys of the top-k bucket and the
//      bracket (global token ids); sums are combined by sum, keys by min, the
//      gathered keys by an all-gather;
//      When the certain bracket holds more keys than one sort (flat rows),
//      a run of its buckets around the crossing estimated from mid-bucket
//      masses, up to TP_WINDOW keys, is gathered instead;
//   4. every rank sorts the merged keys of each row, scans their float64
//      masses from the mass before the gathered buckets and places the cuts
//      exactly; a row whose crossing turns out to lie outside the gathered
//      buckets, or whose keys exceed one sort or a rank's share, takes the
//      gather form.
#include "sts_internal.h"
#include "support_keys.cuh"

namespace sts {
namespace {

__global__ void gather_shards4_kernel(const float4* __restrict__ src, int64_t world, int64_t T,
                                      int64_t vl4, float4* __restrict__ dst, int64_t ld4) {
  const int64_t total = world * T * vl4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = i % vl4;
    const int64_t kr = i / vl4;
    const int64_t r = kr % T, k = kr / T;
    dst[r * ld4 + k * vl4 + j] = src[i];
  }
}

__global__ void gather_shards_kernel(const float* __restrict__ src, int64_t world, int64_t T,
                                     int64_t vl, float* __restrict__ dst, int64_t ld) {
  const int64_t total = world * T * vl;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = i % vl;
    const int64_t kr = i / vl;
    const int64_t r = kr % T, k = kr / T;
    dst[r * ld + k * vl + j] = src[i];
  }
}


// ---------------------------------------------------------------- statistics merge
constexpr int TP_RT = 512;            // threads per row CTA
constexpr int TP_NW = TP_RT / 32;
constexpr int TP_SORT = 8192;         // merged keys of a row sorted at once
constexpr int TP_WINDOW = 2048;       // keys gathered around an estimated top-p crossing
constexpr int TP_BPT = NB / TP_RT;    // buckets per thread in the plan scans

// Per-row plan (int32 fields) and per-row float64 sums / keys of stage 3.
enum : int {
  kPlanBk = 0,      // bucket of the k-th element, -1 when top-k is off
  kPlanCk = 1,      // elements before bucket bk
  kPlanBlo = 2,     // top-p bracket [blo, bhi]; blo = NB, bhi = -1 when top-p is off
  kPlanBhi = 3,
  kPlanCntLo = 4,   // elements before bucket blo
  kPlanKt = 5,      // min-p threshold key (uint32 bits), 0 when min-p is off
  kPlanRules = 6,   // bit 0 top-k, bit 1 top-p, bit 2 min-p
  kPlanFields = 8
};
// kSumZ is the total mass when top-k is off (unused, and partial, otherwise)
enum : int { kSumZ = 0, kSumBk = 1, kSumLo = 2, kSumKept = 3, kSumKeptCnt = 4, kSumFields = 5 };
enum : int { kKeyKept = 0, kKeyAll = 1, kKeyFields = 2 };

// Composite keys travel as int64 with the top bit flipped, so that a signed
// minimum (the collectives' int64 min) is the unsigned minimum.
__device__ __forceinline__ long long key_to_i64(unsigned long long K) {
  return (long long)(K ^ 0x8000000000000000ull);
}
__device__ __forceinline__ unsigned long long key_from_i64(long long v) {
  return (unsigned long long)v ^ 0x8000000000000000ull;
}

struct TpRed {
  double d[TP_NW * kSumFields];
  unsigned long long u[TP_NW * kKeyFields];
  float f[TP_NW];
  long long l[TP_NW];
};

// Deterministic block sums (fixed shuffle tree, then warp 0 over the warps).
template <int N>
__device__ void tp_sum_d(double (&v)[N], double* red) {
#pragma unroll
  for (int i = 0; i < N; ++i)
    for (int o = 16; o; o >>= 1) v[i] += __shfl_down_sync(0xffffffffu, v[i], o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0)
#pragma unroll
    for (int i = 0; i < N; ++i) red[w * N + i] = v[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) {
    double x = l < TP_NW ? red[l * N + i] : 0.0;
    for (int o = 16; o; o >>= 1) x += __shfl_down_sync(0xffffffffu, x, o);
    v[i] = __shfl_sync(0xffffffffu, x, 0);
  }
}

template <int N>
__device__ void tp_min_u(unsigned long long (&v)[N], unsigned long long* red) {
#pragma unroll
  for (int i = 0; i < N; ++i)
    for (int o = 16; o; o >>= 1) {
      const unsigned long long x = __shfl_down_sync(0xffffffffu, v[i], o);
      v[i] = x < v[i] ? x : v[i];
    }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0)
#pragma unroll
    for (int i = 0; i < N; ++i) red[w * N + i] = v[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) {
    unsigned long long x = l < TP_NW ? red[l * N + i] : ~0ull;
    for (int o = 16; o; o >>= 1) {
      const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
      x = y < x ? y : x;
    }
    v[i] = __shfl_sync(0xffffffffu, x, 0);
  }
}

__device__ float tp_max_f(float v, float* red) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_down_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float x = l < TP_NW ? red[l] : -INFINITY;
  for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_down_sync(0xffffffffu, x, o));
  return __shfl_sync(0xffffffffu, x, 0);
}

// Exclusive scan over the block of one value per thread (thread order);
// returns the thread's exclusive prefix, *total the sum.
template <typename T>
__device__ T tp_exscan(T v, T* red, T& total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  T x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, x, o);
    if (l >= o) x += y;
  }
  __syncthreads();
  if (l == 31) red[w] = x;
  __syncthreads();
  T before = 0, tot = 0;
  for (int i = 0; i < TP_NW; ++i) {
    if (i < w) before += red[i];
    tot += red[i];
  }
  total = tot;
  return before + x - v;
}

__global__ void __launch_bounds__(TP_RT) tp_row_max_kernel(const float* __restrict__ S, int64_t ld,
                                                          int Vl, int T, float* __restrict__ out) {
  __shared__ float red[TP_NW];
  for (int r = blockIdx.x; r < T; r += gridDim.x) {
    const float* x = S + (size_t)r * (size_t)ld;
    float v = -INFINITY;
    for (int j = threadIdx.x; j < Vl; j += TP_RT) v = fmaxf(v, x[j]);
    v = tp_max_f(v, red);
    if (threadIdx.x == 0) out[r] = v;
  }
}

__global__ void __launch_bounds__(TP_RT) tp_count_kernel(const float* __restrict__ S, int64_t ld,
                                                        int Vl, int T, const float* __restrict__ m,
                                                        int32_t* __restrict__ counts) {
  __shared__ int cnt[NB];
  for (int r = blockIdx.x; r < T; r += gridDim.x) {
    for (int b = threadIdx.x; b < NB; b += TP_RT) cnt[b] = 0;
    __syncthreads();
    const float* x = S + (size_t)r * (size_t)ld;
    const float mr = m[r];
    for (int j = threadIdx.x; j < Vl; j += TP_RT) atomicAdd(&cnt[bin0(x[j], mr)], 1);
    __syncthreads();
    for (int b = threadIdx.x; b < NB; b += TP_RT) counts[(size_t)r * NB + b] = cnt[b];
    __syncthreads();
  }
}

struct TpExactArgs {
  const float* S;
  int64_t ld;
  int Vl, T;
  int64_t off, V;
  const int64_t* target;
  const int32_t* top_k;
  const float* top_p;
  const float* min_p;
  const float* m;
  const int32_t* counts;   // merged [T][NB]
  int32_t* plan;           // [T][kPlanFields]
  double* sums;            // [T][kSumFields]
  long long* keys;         // [T][kKeyFields]
  float* ylogit;           // [T][2]: the target's logit (when in this shard), 1
  unsigned long long* cand;  // [T][cap]
  int32_t* ncand;          // [T]: keys this shard gathered (may exceed cap)
  int cap;
};

// Rigorous bounds of a bucket's per-element mass exp(s - m): the bucket is
// [b, b + 1) in 128 (m - s) up to the fp32 rounding of that product, which
// the 1e-6 relative widening covers; the clamped last bucket is (0, e^-b].
__device__ __forceinline__ double unit_lo(int b) {
  return b >= NB - 1 ? 0.0 : exp(-(double)(b + 1) / 128.0) * (1.0 - 1e-6);
}
__device__ __forceinline__ double unit_hi(int b) { return exp(-(double)b / 128.0) * (1.0 + 1e-6); }

// exp(s - m) in float64 for an element of bucket b (b = bin0(s, m)): the
// bucket's factor exp(-b/128) from a per-CTA table times exp(r), r = (s - m)
// + b/128 in [-1/128, 0], from its Taylor polynomial to degree 6 (truncation
// below 4e-19, under half an ulp); the clamped last bucket takes the library
// exp.
constexpr size_t TP_EXACT_SMEM = NB * sizeof(double);

__device__ __forceinline__ double tp_mass(const double* tab, float s, double md, int b) {
  const double x = (double)s - md;
  if (b >= NB - 1) return exp(x);
  const double r = fma((double)b, 1.0 / 128.0, x);
  double q = 1.0 / 720.0;
  q = fma(q, r, 1.0 / 120.0);
  q = fma(q, r, 1.0 / 24.0);
  q = fma(q, r, 1.0 / 6.0);
  q = fma(q, r, 0.5);
  q = fma(q, r, 1.0);
  q = fma(q, r, 1.0);
  return tab[b] * q;
}

__global__ void __launch_bounds__(TP_RT) tp_exact_kernel(const TpExactArgs a) {
  extern __shared__ __align__(16) double tp_tab[];  // exp(-b / 128), b < NB
  __shared__ TpRed red;
  __shared__ long long redl[TP_NW];
  __shared__ double redd[TP_NW];
  __shared__ int sp[8];
  __shared__ int ngath;
  __shared__ int cnt_s[NB];
  const int tid = threadIdx.x;
  for (int b = tid; b < NB; b += TP_RT) tp_tab[b] = exp(-(double)b / 128.0);
  __syncthreads();
  for (int r = blockIdx.x; r < a.T; r += gridDim.x) {
    const float mr = a.m[r];
    const double md = (double)mr;
    const int k = a.top_k[r];
    const float p = a.top_p[r], mu = a.min_p[r];
    const bool k_on = k >= 1 && (int64_t)k < a.V;
    const bool p_on = p < 1.0f && p > 0.0f;
    const bool mu_on = mu > 0.0f && mu <= 1.0f;
    // ---- the plan, from the merged counts (thread t: buckets [t BPT, (t + 1) BPT))
    int c[TP_BPT];
    long long mine = 0;
#pragma unroll
    for (int i = 0; i < TP_BPT; ++i) {
      c[i] = a.counts[(size_t)r * NB + tid * TP_BPT + i];
      mine += c[i];
    }
    long long tot;
    const long long before = tp_exscan<long long>(mine, redl, tot);
    if (tid == 0) {
      sp[0] = -1;  // bk
      sp[1] = 0;   // ck
      sp[2] = NB;  // blo
      sp[3] = -1;  // bhi
      sp[4] = 0;   // cnt before blo
    }
    __syncthreads();
    if (k_on) {
      long long cum = before;
#pragma unroll
      for (int i = 0; i < TP_BPT; ++i) {
        if (cum < k && k <= cum + c[i]) {
          sp[0] = tid * TP_BPT + i;
          sp[1] = (int)cum;
        }
        cum += c[i];
      }
    }
    __syncthreads();
    const int bk = sp[0], ck = sp[1];
    if (p_on) {
      // bounds of the running mass before each bucket and of Z_k (buckets up
      // to bk; of bk only its first k - ck elements)
      double lo_i[TP_BPT], hi_i[TP_BPT];
      double slo = 0.0, shi = 0.0;
#pragma unroll
      for (int i = 0; i < TP_BPT; ++i) {
        const int b = tid * TP_BPT + i;
        double n = (double)c[i];
        if (k_on && b > bk) n = 0.0;
        if (k_on && b == bk) n = (double)(k - ck);
        lo_i[i] = n * unit_lo(b);
        hi_i[i] = n * unit_hi(b);
        slo += lo_i[i];
        shi += hi_i[i];
      }
      double zlo, zhi;
      const double blo_before = tp_exscan<double>(slo, redd, zlo);
      const double bhi_before = tp_exscan<double>(shi, redd, zhi);
      const double tlo = (double)p * zlo, thi = (double)p * zhi;
      int first = NB, last = -1;
      double clo = blo_before, chi = bhi_before;
#pragma unroll
      for (int i = 0; i < TP_BPT; ++i) {
        const int b = tid * TP_BPT + i;
        // the crossing lies in b only if the mass before b can be below the
        // target and the mass through b can reach it
        const bool can = (clo < thi) && (chi + hi_i[i] >= tlo) && !(k_on && b > bk);
        if (can) {
          first = min(first, b);
          last = max(last, b);
        }
        clo += lo_i[i];
        chi += hi_i[i];
      }
      // block min / max of the candidate buckets
      unsigned long long mm[2] = {(unsigned long long)first, (unsigned long long)(NB - 1 - last)};
      tp_min_u<2>(mm, red.u);
      const int rlo = (int)mm[0], rhi = NB - 1 - (int)mm[1];
      // the crossing's bucket from mid-bucket mass estimates (used when the
      // certain bracket holds more keys than one sort)
      double est_i[TP_BPT], sest = 0.0;
#pragma unroll
      for (int i = 0; i < TP_BPT; ++i) {
        const int b = tid * TP_BPT + i;
        double n = (double)c[i];
        if (k_on && b > bk) n = 0.0;
        if (k_on && b == bk) n = (double)(k - ck);
        est_i[i] = n * exp(-((double)b + 0.5) / 128.0);
        sest += est_i[i];
      }
      double zest;
      double cest = tp_exscan<double>(sest, redd, zest);
      const double test = (double)p * zest;
      unsigned long long hit[1] = {~0ull};
#pragma unroll
      for (int i = 0; i < TP_BPT; ++i) {
        if (cest + est_i[i] >= test) hit[0] = min(hit[0], (unsigned long long)(tid * TP_BPT + i));
        cest += est_i[i];
      }
      tp_min_u<1>(hit, red.u);
#pragma unroll
      for (int i = 0; i < TP_BPT; ++i) cnt_s[tid * TP_BPT + i] = c[i];
      __syncthreads();
      if (tid == 0) {
        // keys the sort can take for the bracket (the top-k bucket is gathered
        // too when it lies after the bracket)
        const long long extra = (k_on && bk > rhi) ? cnt_s[bk] : 0;
        const long long budget = (long long)TP_SORT - extra;
        long long n = 0;
        for (int b = rlo; b <= rhi; ++b) n += cnt_s[b];
        int lo = rlo, hi = rhi;
        if (n > budget && rlo <= rhi) {
          // the certain bracket does not fit: a run of buckets around the
          // estimated crossing, grown to TP_WINDOW keys (the mid-bucket
          // estimate is off by a bucket or two on flat rows; the finish checks
          // that the run holds the crossing, else the row takes the gather form)
          const long long want = budget < TP_WINDOW ? budget : TP_WINDOW;
          int c0 = (int)min(max((long long)hit[0], (long long)rlo), (long long)rhi);
          lo = hi = c0;
          n = cnt_s[c0];
          for (bool grew = true; grew;) {
            grew = false;
            if (hi < rhi && n + cnt_s[hi + 1] <= want) {
              n += cnt_s[++hi];
              grew = true;
            }
            if (lo > rlo && n + cnt_s[lo - 1] <= want) {
              n += cnt_s[--lo];
              grew = true;
            }
          }
        }
        sp[2] = lo;
        sp[3] = hi;
      }
      __syncthreads();
      const int blo = sp[2];
      long long cb = 0;
      long long cum = before;
#pragma unroll
      for (int i = 0; i < TP_BPT; ++i) {
        if (tid * TP_BPT + i == blo) cb = cum;
        cum += c[i];
      }
      unsigned long long cbm[1] = {tid * TP_BPT <= blo && blo < (tid + 1) * TP_BPT
                                       ? (unsigned long long)cb : ~0ull};
      tp_min_u<1>(cbm, red.u);
      if (tid == 0) sp[4] = blo < NB ? (int)cbm[0] : 0;
      __syncthreads();
    }
    const int blo = sp[2], bhi = sp[3];
    uint32_t kt = 0;
    if (mu_on) {
      if (tid == 0) sp[5] = (int)min_p_threshold_key(mr, mu);
      __syncthreads();
      kt = (uint32_t)sp[5];
    }
    if (tid == 0) {
      int32_t* pl = a.plan + (size_t)r * kPlanFields;
      pl[kPlanBk] = bk;
      pl[kPlanCk] = ck;
      pl[kPlanBlo] = blo;
      pl[kPlanBhi] = bhi;
      pl[kPlanCntLo] = sp[4];
      pl[kPlanKt] = (int32_t)kt;
      pl[kPlanRules] = (k_on ? 1 : 0) | (p_on ? 2 : 0) | (mu_on ? 4 : 0);
      pl[7] = 0;
      ngath = 0;
    }
    __syncthreads();
    // ---- one pass over the shard
    const float* x = a.S + (size_t)r * (size_t)a.ld;
    double z = 0.0, mbk = 0.0, mlo = 0.0, mk = 0.0, ckept = 0.0;
    unsigned long long kkept = ~0ull, kall = ~0ull;
    unsigned long long* cand = a.cand + (size_t)r * (size_t)a.cap;
    // the total mass is only used when top-k is off (the top-p target and
    // identity rows); otherwise only the logits before the top-k bucket, the
    // bracket and the min-p-kept ones are weighed
    const bool zneed = !k_on;
    for (int j = tid; j < a.Vl; j += TP_RT) {
      const float s = x[j];
      const int b = bin0(s, mr);
      const unsigned long long K = ckey(s, (int)(a.off + j));
      const bool kept = mu_on & (key32(s) >= kt);
      if (zneed | (b < bk) | (b < blo) | kept) {
        const double q = tp_mass(tp_tab, s, md, b);
        z += q;
        if (b < bk) mbk += q;
        if (b < blo) mlo += q;
        if (kept) mk += q;
      }
      if (kept) {
        ckept += 1.0;
        kkept = K < kkept ? K : kkept;
      }
      kall = K < kall ? K : kall;
      if (((b >= blo) & (b <= bhi)) | (b == bk)) {
        const int slot = atomicAdd(&ngath, 1);
        if (slot < a.cap) cand[slot] = K;
      }
    }
    double sums[kSumFields] = {z, mbk, mlo, mk, ckept};
    tp_sum_d<kSumFields>(sums, red.d);
    unsigned long long keys[kKeyFields] = {kkept, kall};
    tp_min_u<kKeyFields>(keys, red.u);
    if (tid == 0) {
      for (int i = 0; i < kSumFields; ++i) a.sums[(size_t)r * kSumFields + i] = sums[i];
      a.keys[(size_t)r * kKeyFields + kKeyKept] = key_to_i64(keys[0]);
      a.keys[(size_t)r * kKeyFields + kKeyAll] = key_to_i64(keys[1]);
      a.ncand[r] = ngath;
      const int64_t y = a.target[r];
      const bool mine_y = y >= a.off && y < a.off + a.Vl;
      a.ylogit[(size_t)r * 2] = mine_y ? x[y - a.off] : 0.0f;
      a.ylogit[(size_t)r * 2 + 1] = mine_y ? 1.0f : 0.0f;
    }
    __syncthreads();
  }
}

struct TpFinishArgs {
  int T;
  int64_t V;
  int world, cap;
  const int64_t* target;
  const int32_t* top_k;
  const float* top_p;
  const int32_t* row_flags;        // validation (STS_ROW_INVALID)
  const float* m;
  const int32_t* plan;
  const double* sums;              // merged
  const long long* keys;           // merged
  const float* ylogit;             // merged
  const unsigned long long* cand;  // [world][T][cap]
  const int32_t* ncand;            // [world][T]
  float* logprob;
  float* row_max;
  float* lse_support;
  float* cut_logit;
  int32_t* cut_id;
  int32_t* support_size;
  int32_t* flags_out;
  int32_t* need_gather;            // [T]: 1 where the bracket overflowed the sort
};

constexpr size_t TP_FINISH_SMEM =
    TP_SORT * (sizeof(unsigned long long) + sizeof(double)) + NB * sizeof(double);

__global__ void __launch_bounds__(TP_RT) tp_finish_kernel(const TpFinishArgs a) {
  extern __shared__ __align__(16) uint8_t tp_smem[];
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(tp_smem);
  double* scan = reinterpret_cast<double*>(tp_smem + TP_SORT * sizeof(unsigned long long));
  double* tab = scan + TP_SORT;  // exp(-b / 128): the masses of the exact pass's stage
  for (int b = threadIdx.x; b < NB; b += TP_RT) tab[b] = exp(-(double)b / 128.0);
  __syncthreads();
  __shared__ TpRed red;
  __shared__ double redd[TP_NW];
  __shared__ int ntot_s;
  const int tid = threadIdx.x;
  for (int r = blockIdx.x; r < a.T; r += gridDim.x) {
    const float nan = __int_as_float(0x7fc00000);
    const bool invalid = (a.row_flags[r] & STS_ROW_INVALID) != 0;
    if (tid == 0) {
      int tot = 0;
      bool over = false;
      for (int w = 0; w < a.world; ++w) {
        const int n = a.ncand[(size_t)w * a.T + r];
        over |= n > a.cap;
        tot += n;
      }
      ntot_s = (over || tot > TP_SORT) ? -1 : tot;
    }
    __syncthreads();
    const int ntot = ntot_s;
    if (invalid || ntot < 0) {
      if (tid == 0) {
        a.need_gather[r] = invalid ? 0 : 1;
        if (invalid) {
          a.logprob[r] = nan;
          a.row_max[r] = nan;
          a.lse_support[r] = nan;
          a.cut_logit[r] = nan;
          a.cut_id[r] = -1;
          a.support_size[r] = 0;
          a.flags_out[r] = STS_ROW_INVALID;
        }
      }
      __syncthreads();
      continue;
    }
    // the merged keys, in rank order, padded with 0 (below every key)
    int n2 = 64;
    while (n2 < ntot) n2 <<= 1;
    for (int i = tid; i < n2; i += TP_RT) keys[i] = 0ull;
    __syncthreads();
    {
      int base = 0;
      for (int w = 0; w < a.world; ++w) {
        const int n = a.ncand[(size_t)w * a.T + r];
        const unsigned long long* src = a.cand + ((size_t)w * a.T + r) * (size_t)a.cap;
        for (int i = tid; i < n; i += TP_RT) keys[base + i] = src[i];
        base += n;
      }
    }
    __syncthreads();
    // bitonic sort, descending (earlier in the order first)
    for (int kk = 2; kk <= n2; kk <<= 1)
      for (int j = kk >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < n2; i += TP_RT) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const unsigned long long u = keys[i], v = keys[ixj];
            const bool desc = (i & kk) == 0;
            if (desc ? (u < v) : (u > v)) {
              keys[i] = v;
              keys[ixj] = u;
            }
          }
        }
        __syncthreads();
      }
    const float mr = a.m[r];
    const double md = (double)mr;
    // inclusive scan of the sorted keys' masses (thread t: a contiguous run)
    const int per = (n2 + TP_RT - 1) / TP_RT;
    {
      double run = 0.0;
      const int i0 = tid * per;
      auto qm = [&](int i) {
        const float v = ckey_value(keys[i]);
        return tp_mass(tab, v, md, bin0(v, mr));
      };
      for (int i = i0; i < i0 + per && i < ntot; ++i) run += qm(i);
      double total;
      double acc = tp_exscan<double>(run, redd, total);
      for (int i = i0; i < i0 + per && i < ntot; ++i) {
        acc += qm(i);
        scan[i] = acc;
      }
    }
    __syncthreads();
    const int32_t* pl = a.plan + (size_t)r * kPlanFields;
    const int rules = pl[kPlanRules], bk = pl[kPlanBk], ck = pl[kPlanCk], bhi = pl[kPlanBhi];
    const int cnt_lo = pl[kPlanCntLo];
    const double* sm = a.sums + (size_t)r * kSumFields;
    const double z = sm[kSumZ], mbk = sm[kSumBk], mlo = sm[kSumLo], mkept = sm[kSumKept];
    const long long ckept = (long long)sm[kSumKeptCnt];
    const unsigned long long kkept = key_from_i64(a.keys[(size_t)r * kKeyFields + kKeyKept]);
    const unsigned long long kall = key_from_i64(a.keys[(size_t)r * kKeyFields + kKeyAll]);
    const int k = a.top_k[r];
    const float p = a.top_p[r];
    // top-k: the k-th element is the (k - ck)-th of bucket bk, whose keys are
    // contiguous in the sorted run
    unsigned long long Kk = 0ull;
    double zk = z;
    bool bad = false;
    if (rules & 1) {
      unsigned long long first[1] = {~0ull};
      for (int i = tid; i < ntot; i += TP_RT)
        if (bin0(ckey_value(keys[i]), mr) == bk) first[0] = min(first[0], (unsigned long long)i);
      tp_min_u<1>(first, red.u);
      const long long i0 = (long long)first[0];
      const long long ik = i0 + (k - ck) - 1;
      if (first[0] == ~0ull || ik >= ntot) {
        bad = true;
      } else {
        Kk = keys[ik];
        const double before_bk = i0 > 0 ? scan[i0 - 1] : 0.0;
        zk = mbk + (scan[ik] - before_bk);
      }
    }
    // top-p: the first sorted key of the bracket whose inclusive running mass
    // (from the mass before the bracket) reaches p Z_k
    unsigned long long Kp = 0ull;
    long long sp_ = 0;
    double mp_ = 0.0;
    if ((rules & 2) && !bad) {
      const double target = (double)p * zk;
      if (mlo >= target) bad = true;  // the crossing lies before the gathered window
    }
    if ((rules & 2) && !bad) {
      const double target = (double)p * zk;
      unsigned long long hit[1] = {~0ull};
      for (int i = tid; i < ntot; i += TP_RT)
        if (bin0(ckey_value(keys[i]), mr) <= bhi && mlo + scan[i] >= target)
          hit[0] = min(hit[0], (unsigned long long)i);
      tp_min_u<1>(hit, red.u);
      if (hit[0] == ~0ull) {
        bad = true;
      } else {
        const long long j = (long long)hit[0];
        Kp = keys[j];
        sp_ = cnt_lo + j + 1;
        mp_ = mlo + scan[j];
      }
    }
    if (tid == 0) {
      if (bad) {
        a.need_gather[r] = 1;
      } else {
        // the support is the shortest prefix: the cut with the largest key
        unsigned long long K = 0ull;
        long long size = 0;
        double mass = 0.0;
        bool any = false;
        if (rules & 1) {
          K = Kk;
          size = k;
          mass = zk;
          any = true;
        }
        if ((rules & 2) && (!any || Kp > K)) {
          K = Kp;
          size = sp_;
          mass = mp_;
          any = true;
        }
        if ((rules & 4) && (!any || kkept > K)) {
          K = kkept;
          size = ckept;
          mass = mkept;
          any = true;
        }
        if (!any) {  // identity
          K = kall;
          size = a.V;
          mass = z;
        }
        const double lse = md + log(mass);
        const float sy = a.ylogit[(size_t)r * 2];
        const int64_t y = a.target[r];
        const bool in = ckey(sy, (int)y) >= K;
        a.need_gather[r] = 0;
        a.logprob[r] = in ? (float)fmin((double)sy - lse, 0.0) : -INFINITY;
        a.row_max[r] = mr;
        a.lse_support[r] = (float)lse;
        a.cut_logit[r] = ckey_value(K);
        a.cut_id[r] = ckey_id(K);
        a.support_size[r] = (int32_t)size;
        a.flags_out[r] = (any ? 0 : STS_ROW_IDENTITY) | (in ? STS_ROW_TARGET_IN_SUPPORT : 0);
      }
    }
    __syncthreads();
  }
}

}  // namespace
}  // namespace sts

using namespace sts;

extern "C" sts_status sts_gather_vocab_shards(const float* src, int64_t world, int64_t T,
                                              int64_t vocab_per_rank, float* dst, int64_t ld,
                                              sts_stream_t stream) {
  if (!src || !dst) return STS_ERR_NULL;
  if (world < 1 || T < 1 || vocab_per_rank < 1 || ld < world * vocab_per_rank) return STS_ERR_SHAPE;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return STS_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool vec = (vocab_per_rank % 4 == 0) && (ld % 4 == 0) &&
                   ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) == 0;
  const int threads = 256;
  const int blocks = sms * 8;  // a grid-stride copy, eight CTAs per SM
  if (vec)
    gather_shards4_kernel<<<blocks, threads, 0, st>>>(reinterpret_cast<const float4*>(src), world, T,
                                                      vocab_per_rank / 4,
                                                      reinterpret_cast<float4*>(dst), ld / 4);
  else
    gather_shards_kernel<<<blocks, threads, 0, st>>>(src, world, T, vocab_per_rank, dst, ld);
  return cudaGetLastError() == cudaSuccess ? STS_OK : STS_ERR_CUDA;
}


namespace {

int tp_grid(int64_t T) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t g = T < (int64_t)sms * 2 ? T : (int64_t)sms * 2;  // two row CTAs per SM
  return (int)(g > 0 ? g : 1);
}

bool rows_ok(const sts_rows* rows, int64_t T) {
  return rows && rows->len == T && rows->target && rows->temperature && rows->top_k &&
         rows->top_p && rows->min_p;
}

}  // namespace

extern "C" sts_status sts_tp_constants(int64_t* buckets, int64_t* plan_fields, int64_t* sum_fields,
                                       int64_t* key_fields, int64_t* sort_cap) {
  if (!buckets || !plan_fields || !sum_fields || !key_fields || !sort_cap) return STS_ERR_NULL;
  *buckets = NB;
  *plan_fields = kPlanFields;
  *sum_fields = kSumFields;
  *key_fields = kKeyFields;
  *sort_cap = TP_SORT;
  return STS_OK;
}

extern "C" sts_status sts_tp_row_max(const float* S, int64_t T, int64_t Vl, int64_t ld, float* row_max,
                                     sts_stream_t stream) {
  if (!S || !row_max) return STS_ERR_NULL;
  if (T < 1 || Vl < 1 || ld < Vl || Vl > INT32_MAX || T > INT32_MAX) return STS_ERR_SHAPE;
  tp_row_max_kernel<<<tp_grid(T), TP_RT, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      S, ld, (int)Vl, (int)T, row_max);
  return cudaGetLastError() == cudaSuccess ? STS_OK : STS_ERR_CUDA;
}

extern "C" sts_status sts_tp_count(const float* S, int64_t T, int64_t Vl, int64_t ld, const float* m,
                                   int32_t* counts, sts_stream_t stream) {
  if (!S || !m || !counts) return STS_ERR_NULL;
  if (T < 1 || Vl < 1 || ld < Vl || Vl > INT32_MAX || T > INT32_MAX) return STS_ERR_SHAPE;
  tp_count_kernel<<<tp_grid(T), TP_RT, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      S, ld, (int)Vl, (int)T, m, counts);
  return cudaGetLastError() == cudaSuccess ? STS_OK : STS_ERR_CUDA;
}

extern "C" sts_status sts_tp_exact(const float* S, int64_t T, int64_t Vl, int64_t ld,
                                   int64_t vocab_offset, int64_t V, const sts_rows* rows,
                                   const float* m, const int32_t* counts, int32_t* plan,
                                   double* sums, int64_t* keys, float* ylogit, uint64_t* cand,
                                   int32_t* ncand, int64_t cap, sts_stream_t stream) {
  if (!S || !m || !counts || !plan || !sums || !keys || !ylogit || !cand || !ncand)
    return STS_ERR_NULL;
  if (!rows_ok(rows, T)) return rows ? STS_ERR_SHAPE : STS_ERR_NULL;
  if (T < 1 || Vl < 1 || ld < Vl || T > INT32_MAX || cap < 1 || cap > INT32_MAX ||
      vocab_offset < 0 || V < vocab_offset + Vl || V > INT32_MAX)
    return STS_ERR_SHAPE;
  TpExactArgs a{};
  a.S = S;
  a.ld = ld;
  a.Vl = (int)Vl;
  a.T = (int)T;
  a.off = vocab_offset;
  a.V = V;
  a.target = rows->target;
  a.top_k = rows->top_k;
  a.top_p = rows->top_p;
  a.min_p = rows->min_p;
  a.m = m;
  a.counts = counts;
  a.plan = plan;
  a.sums = sums;
  a.keys = reinterpret_cast<long long*>(keys);
  a.ylogit = ylogit;
  a.cand = reinterpret_cast<unsigned long long*>(cand);
  a.ncand = ncand;
  a.cap = (int)cap;
  if (cudaFuncSetAttribute(tp_exact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)TP_EXACT_SMEM) != cudaSuccess)
    return STS_ERR_CUDA;
  tp_exact_kernel<<<tp_grid(T), TP_RT, TP_EXACT_SMEM, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? STS_OK : STS_ERR_CUDA;
}

extern "C" sts_status sts_tp_finish(int64_t T, int64_t V, int64_t world, const sts_rows* rows,
                                    const float* m, const int32_t* plan, const double* sums,
                                    const int64_t* keys, const float* ylogit, const uint64_t* cand,
                                    const int32_t* ncand, int64_t cap, float* logprob,
                                    const sts_saved* saved, int32_t* need_gather, void* ws,
                                    size_t ws_bytes, sts_stream_t stream) {
  if (!m || !plan || !sums || !keys || !ylogit || !cand || !ncand || !logprob || !need_gather)
    return STS_ERR_NULL;
  if (!saved || !saved->row_max || !saved->lse_support || !saved->cut_logit || !saved->cut_id ||
      !saved->support_size || !saved->flags)
    return STS_ERR_NULL;
  if (!rows_ok(rows, T)) return rows ? STS_ERR_SHAPE : STS_ERR_NULL;
  if (T < 1 || V < 1 || V > INT32_MAX || world < 1 || cap < 1 || cap > INT32_MAX || T > INT32_MAX)
    return STS_ERR_SHAPE;
  if (!ws || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return STS_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  if (cudaMemsetAsync(&hdr->bad_row_code, 0xFF, sizeof(hdr->bad_row_code), st) != cudaSuccess ||
      cudaMemsetAsync(&hdr->err, 0, 8 + sizeof(hdr->path_rows), st) != cudaSuccess)
    return STS_ERR_CUDA;
  launch_validate(rows->target, rows->temperature, rows->top_p, rows->min_p, T, V, saved->flags, hdr,
                  true, st);
  if (cudaFuncSetAttribute(tp_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)TP_FINISH_SMEM) != cudaSuccess)
    return STS_ERR_CUDA;
  TpFinishArgs a{};
  a.T = (int)T;
  a.V = V;
  a.world = (int)world;
  a.cap = (int)cap;
  a.target = rows->target;
  a.top_k = rows->top_k;
  a.top_p = rows->top_p;
  a.row_flags = saved->flags;
  a.m = m;
  a.plan = plan;
  a.sums = sums;
  a.keys = reinterpret_cast<const long long*>(keys);
  a.ylogit = ylogit;
  a.cand = reinterpret_cast<const unsigned long long*>(cand);
  a.ncand = ncand;
  a.logprob = logprob;
  a.row_max = saved->row_max;
  a.lse_support = saved->lse_support;
  a.cut_logit = saved->cut_logit;
  a.cut_id = saved->cut_id;
  a.support_size = saved->support_size;
  a.flags_out = saved->flags;
  a.need_gather = need_gather;
  tp_finish_kernel<<<tp_grid(T), TP_RT, TP_FINISH_SMEM, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? STS_OK : STS_ERR_CUDA;
}
