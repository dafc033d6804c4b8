// Row validation and the exact per-row support resolver.
//
// The resolver runs the pinned sampling-transform program ("Consolidate
// sampling-transform scoring on one shared chunked core; implement
// top-k/top-p/min-p replay for generic ce_modes", xorl PR 74, "What this PR
// does", item 1) on one row of fp32 scaled logits s[0..V) held in global
// memory:
//
//   order      (s desc, token id asc): every token gets a distinct 64-bit
//              composite key K = (monotone key of s) << 32 | (2^32-1 - id),
//              so "earlier in the order" is "larger K" and ties in s are
//              broken by the lower id.
//   top-k      the k-th element of the order
//   top-p      the first element whose inclusive running mass reaches
//              p * Z_k (Z_k = mass of the top-k prefix; masses are
//              exp(s - m) in float64, m the unfiltered row max)
//   min-p      the smallest fp32 threshold t with exp(t - m) >= min_p,
//              found by bisection over fp32 bit patterns; every s >= t kept
//   support    the shortest of the three prefixes; its size, mass Z_S and
//              last element (the cut) give LSE_S = m + log Z_S
//
// Work per row (one 512-thread CTA per SM, persistent over rows; a row's
// metadata and the projection epilogue's per-tile maxima, which give the
// unfiltered max m, are loaded one row ahead). Rows with a 16-byte aligned
// start stream through a shared-memory ring filled by bulk copies (one thread
// keeps two 32 KB chunks in flight), so no pass holds its loads in registers.
//
//   buckets      floor((m - s) * 128), clamped to 4095: monotone in s, so
//                every bucket is a contiguous run of the order.
//   planned path (first) a count histogram of one chunk in eight plans the
//                range to gather: for top-k the buckets up to the k-th
//                element, for min-p the buckets around its threshold (when
//                top-p is on too, only where the sample puts the crossing
//                clearly after the min-p prefix). One pass gathers that range
//                and, for min-p, weighs and counts everything before it, and
//                the row is decided from the gathered elements. Without the
//                entropy output (and outside the sampler) a min-p-decided row
//                is weighed in fp32 instead (kept iff s >= t; the support's
//                mass only enters LSE_S and, with top-p on, a certificate
//                checked against the fp32 error bound), as are identity rows.
//   fast path    (rows whose plan does not hold, and top-p rows) a count pass
//                adds the rest of the row to the sample's histogram; the top-p
//                crossing's bucket is estimated from the counts with
//                mid-bucket weights (with a neighbour where the estimate lies
//                within six sigma of an edge; one retry with a 3-bucket window
//                if the exact masses then place the crossing outside), the
//                min-p threshold's bucket and the non-empty bucket before it
//                planned. The exact pass (from L2: the count pass marks the
//                row's lines evict-last) forms float64 masses of every element,
//                summed in registers (the total, the mass before the window, the
//                mass before the min-p bucket), and gathers the planned buckets'
//                elements into per-thread slots of a candidate buffer. A pass
//                that only gathers (top-k) tests values against the planned
//                buckets widened by one, without forming bucket indices.
//   large top-k  (the prefix up to the k-th element's bucket exceeds the sort)
//                one exact pass gathers that bucket alone; its sorted elements
//                give the k-th element and Z_k.
//   finish       exact masses of the window buckets place the crossing in one
//                bucket; its elements are sorted by composite key (a bitonic
//                network held mostly in registers and warp shuffles) and
//                scanned, which places each cut exactly.
//   entropy      (when asked) each region's sum of exp(s - m) (s - m) next to
//                its mass, in the same pass, gives the entropy of the
//                renormalised support: ln Z_S - sum_S q (s - m) / Z_S.
//
// When the plan cannot be proven to hold a cut (a crossing outside the
// window, too many candidates) the row falls back to the exact search: a float64 mass histogram, then the candidate buckets gathered from
// the row, refining a bucket too large for the 4096-entry sort on its
// composite keys (12 bits per level) until it fits; the keys are distinct, so
// this ends after at most six levels.
//
// Masses use a table-driven float64 exponential (P. T. P. Tang, "Table-driven
// implementation of the exponential function in IEEE floating-point
// arithmetic", ACM TOMS 15(2), 1989): exp(x) = exp(-b/128) * exp(x + b/128)
// with b the element's bucket, the table entries computed once per CTA with
// the CUDA library exp, and the reduced factor (|r| <= 1/128) from its
// degree-6 Taylor polynomial, whose truncation error (< 4e-19) is below half
// an ulp. Elements in the clamped far-tail bucket use the library exp.
#include <cfloat>
#include <climits>
#include <type_traits>
#include <cmath>

#include "sts_device.cuh"
#include "support_keys.cuh"

namespace sts {

namespace {

constexpr int RT = 512;             // threads per resolver CTA
constexpr int NWARP = RT / 32;
constexpr int CAP = 8192;           // candidate buffer (composite keys)
constexpr int SCAP = 4096;          // candidates sorted and scanned at once
constexpr int MAX_LEVELS = 8;
constexpr int UNROLL = 4;           // float4 loads in flight per thread
constexpr int SAMPLE_EVERY = 8;     // the planning sample reads one chunk in 8
constexpr int CPT = 4;              // float4s per thread in a streamed chunk (even)
constexpr int CH_F4 = CPT * RT;     // float4s of a streamed chunk (32 KB)
constexpr int NSTAGE = 2;           // chunks in flight in the shared-memory ring

// exp(-b / 128) for every bucket b.
struct ExpTab {
  double v[NB];
};

__device__ __forceinline__ double tab_at(const ExpTab& t, int b) { return t.v[b]; }

__device__ void init_exp_tab(ExpTab& t, int tid, int nthreads) {
  for (int i = tid; i < NB; i += nthreads) t.v[i] = exp(-(double)i * (1.0 / 128.0));
}

// The bucket masses (planning and the exact histogram) and the candidates'
// mass scan are never live at once and share storage.
struct RSmem {
  // Rows with a 16-byte aligned start are streamed through this ring by bulk
  // copies (one thread issues them, chunks in flight = NSTAGE).
  float4 ring[NSTAGE][CH_F4];
  unsigned long long full_bar[NSTAGE];   // bulk copy landed (tx bytes)
  int ring_done[NSTAGE];                 // warps done with the chunk in the slot
  int ring_issued;                       // copies issued in the current pass
  int abort_flag;                        // a bounded wait gave up
  uint32_t ring_q[RT];                   // per thread: chunks consumed so far (all equal)
  int* err;                              // the workspace status word's error field
  union {
    double mass[NB];
    double cq[SCAP];  // inclusive mass scan of at most SCAP sorted candidates
  };
  unsigned long long cand[CAP];
  ExpTab tab;
  int cnt[NB];
  double red_d[NWARP];
  double red_m[NWARP * 8 + 8];
  unsigned long long red_u[NWARP];
  long long red_l[NWARP];
  float red_f[NWARP];
  double bd[4];
  long long bl[4];
  int bi[4];
  int row_next;       // the row this CTA resolves after the current one
  int ncand;
  int tcount[RT];     // gathered keys of each thread (slot j of thread t: cand[j RT + t])
};

// ---------------------------------------------------------------- keys
// key32, ckey, ckey_value, ckey_id and bin0 come from support_keys.cuh.

// exp(x) for the far tail (x < -32), kept out of line so the loops that
// stream a row do not carry its registers.
__device__ __noinline__ double far_mass(double x) { return exp(x); }

// exp((double)s - (double)m) for an element in level-0 bucket b.
__device__ __forceinline__ double qmass_b(const ExpTab& tab, float s, double md, int b) {
  const double x = (double)s - md;
  if (b >= NB - 1) return far_mass(x);
  const double r = fma((double)b, 1.0 / 128.0, x);
  double p = 1.0 / 720.0;
  p = fma(p, r, 1.0 / 120.0);
  p = fma(p, r, 1.0 / 24.0);
  p = fma(p, r, 1.0 / 6.0);
  p = fma(p, r, 0.5);
  p = fma(p, r, 1.0);
  p = fma(p, r, 1.0);
  return tab_at(tab, b) * p;
}

__device__ __forceinline__ double qmass(const RSmem& sm, float s, float m) {
  return qmass_b(sm.tab, s, (double)m, bin0(s, m));
}

// ---------------------------------------------------------------- streaming

// Read-only streaming loads that do not allocate in L1 (most of the SM's
// on-chip memory is shared memory here, so L1 is small).
__device__ __forceinline__ float4 ld_stream4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

// L2 eviction policies for the two passes over a row: the count pass marks
// the row's lines evict-last so the exact pass that follows finds them in L2
// (148 rows in flight are about 90 MB), and the exact pass reads them
// evict-first, which hands the space back.
__device__ __forceinline__ unsigned long long l2_policy_keep() {
  unsigned long long p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ unsigned long long l2_policy_drop() {
  unsigned long long p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ float4 ld_stream4(const float4* p, unsigned long long policy) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(policy));
  return v;
}

__device__ __forceinline__ float ld_stream(const float* p) {
  float v;
  asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Apply f(value, index) to every element of the row. VEC: the row start is
// 16-byte aligned, so UNROLL float4 loads per thread are kept in flight.
template <bool VEC, bool KEEP = false, typename F>
__device__ __forceinline__ void for_each(const float* __restrict__ x, int V, F&& f) {
  if (VEC) {
    const float4* __restrict__ x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    const unsigned long long keep = KEEP ? l2_policy_keep() : 0ull;
    for (int base = 0; base < V4; base += RT * UNROLL) {
      float4 v[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int i = base + u * RT + (int)threadIdx.x;
        if (i < V4) v[u] = KEEP ? ld_stream4(x4 + i, keep) : ld_stream4(x4 + i);
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int i = base + u * RT + (int)threadIdx.x;
        if (i < V4) {
          f(v[u].x, 4 * i);
          f(v[u].y, 4 * i + 1);
          f(v[u].z, 4 * i + 2);
          f(v[u].w, 4 * i + 3);
        }
      }
    }
    for (int i = 4 * V4 + (int)threadIdx.x; i < V; i += RT) f(ld_stream(x + i), i);
  } else {
    constexpr int U = 4 * UNROLL;
    for (int base = 0; base < V; base += RT * U) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * RT + (int)threadIdx.x;
        if (i < V) v[u] = ld_stream(x + i);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * RT + (int)threadIdx.x;
        if (i < V) f(v[u], i);
      }
    }
  }
}

// ---------------------------------------------------------------- streaming through the ring
// A row whose start is 16-byte aligned is read in chunks of CH_F4 float4s
// (chunk c = float4s [c CH_F4, min(V4, (c + 1) CH_F4))) that bulk copies put
// into the shared-memory ring. Up to NSTAGE copies are in flight, so a pass's
// HBM latency is covered without holding loads in registers; every thread
// takes the float4s at offsets t, t + RT, ..., t + (CPT - 1) RT of each chunk,
// two per batch, and the warp that finishes a chunk last copies the chunk
// NSTAGE ahead into its slot. Large chunks (32 KB) amortise each chunk's wait
// and hand-off over 16 elements per thread.
//
// stream_chunks streams chunks chunk_of(0), ..., chunk_of(n - 1) and calls
// f(full, a, ia, b, ib, va, vb) for each batch: a and b two of the thread's
// float4s, ia and ib their float4 indices in the row, va and vb whether they
// lie in the row, and `full` (a type) true at compile time for every chunk but a partial
// last one. sm.ring_q[t] counts the chunks the CTA has consumed so far (the
// same on every thread); it fixes the parity of every ring barrier. Returns
// false when a bounded wait gave up: sm.abort_flag is then raised,
// STS_ERR_TIMEOUT recorded in *sm.err, and thread 0 has waited (bounded) for
// its copies in flight.
template <typename CF, typename F>
__device__ __forceinline__ bool stream_chunks(RSmem& sm, const float4* __restrict__ x4, int V4,
                                              int n, CF&& chunk_of, unsigned long long policy,
                                              F&& f) {
  int* err = sm.err;
  const int tid = (int)threadIdx.x, lane = tid & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const uint32_t q0 = sm.ring_q[tid];
  // copy chunk j into its slot (the slot's previous chunk is fully consumed)
  auto issue = [&](int j) {
    const uint32_t qq = q0 + (uint32_t)j;
    const int s = (int)(qq % NSTAGE);
    const int f0 = chunk_of(j) * CH_F4;
    const uint32_t bytes = (uint32_t)min(CH_F4, V4 - f0) * 16u;
    mbar_arrive_expect_tx(smem_u32(&sm.full_bar[s]), bytes);
    bulk_load(smem_u32(&sm.ring[s][0]), x4 + f0, bytes, smem_u32(&sm.full_bar[s]), policy);
    atomicAdd(&sm.ring_issued, 1);
  };
  if (tid == 0) {
    sm.ring_issued = 0;
    for (int j = 0; j < n && j < NSTAGE; ++j) issue(j);
  }
  bool ok = true;
  int j = 0;
  for (; j < n; ++j) {
    const uint32_t qq = q0 + (uint32_t)j;
    const int s = (int)(qq % NSTAGE);
    if (!mbar_wait(smem_u32(&sm.full_bar[s]), (qq / NSTAGE) & 1u, abort_flag, err)) {
      ok = false;
      break;
    }
    const int f0 = chunk_of(j) * CH_F4;
    const int cnt = min(CH_F4, V4 - f0);
    // the thread's float4s of the chunk, two per batch, in increasing index
    // (one copy of the batch code: the heavy passes keep their registers)
#pragma unroll 1
    for (int h = 0; h < CPT; h += 2) {
      const int ia = tid + h * RT, ib = ia + RT;
      const float4 a = sm.ring[s][ia];
      const float4 b = sm.ring[s][ib];
      if (cnt == CH_F4)
        f(std::true_type{}, a, f0 + ia, b, f0 + ib, true, true);
      else
        f(std::false_type{}, a, f0 + ia, b, f0 + ib, ia < cnt, ib < cnt);
    }
    __syncwarp();
    // the warp that finishes a chunk last refills its slot: no warp waits for
    // another one to release a slot
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&sm.ring_done[s], 1) == NWARP - 1) {
        sm.ring_done[s] = 0;
        if (j + NSTAGE < n) {
          __threadfence_block();
          fence_proxy_async_smem();  // every warp's reads of the slot before the copy
          issue(j + NSTAGE);
        }
      }
    }
  }
  if (!ok) *abort_flag = 1;
  sm.ring_q[tid] = q0 + (uint32_t)n;
  // every slot consumed before the next pass fills it; on a failed wait,
  // thread 0 waits (bounded) for the copies issued after its last chunk
  if (__syncthreads_or(!ok)) {
    if (tid == 0)
      for (int k = j; k < sm.ring_issued; ++k) {
        const uint32_t qq = q0 + (uint32_t)k;
        mbar_wait_drain(smem_u32(&sm.full_bar[qq % NSTAGE]), (qq / NSTAGE) & 1u);
      }
    __syncthreads();
    return false;
  }
  return true;
}

// Number of chunks of a row of V4 float4s.
__device__ __forceinline__ int n_chunks(int V4) { return (V4 + CH_F4 - 1) / CH_F4; }

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

// Sums of N doubles over the block in one exchange (two barriers).
template <int N>
__device__ void block_sum_multi(double (&v)[N], RSmem& sm) {
  static_assert(N <= 8, "scratch holds 8 values per warp");
#pragma unroll
  for (int k = 0; k < N; ++k)
    for (int o = 16; o; o >>= 1) v[k] += __shfl_down_sync(0xffffffffu, v[k], o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0)
#pragma unroll
    for (int k = 0; k < N; ++k) sm.red_m[w * 8 + k] = v[k];
  __syncthreads();
  if (w == 0) {
#pragma unroll
    for (int k = 0; k < N; ++k) {
      double t = l < NWARP ? sm.red_m[l * 8 + k] : 0.0;
      for (int o = 16; o; o >>= 1) t += __shfl_down_sync(0xffffffffu, t, o);
      if (l == 0) sm.red_m[NWARP * 8 + k] = t;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < N; ++k) v[k] = sm.red_m[NWARP * 8 + k];
  __syncthreads();
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

__device__ __forceinline__ int block_min_i(int v, RSmem& sm) {
  return (int)(~block_ext_u<true>(~(unsigned long long)(unsigned)v, sm));
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

// Exclusive scans of three doubles over threads in thread order, in one
// exchange.
__device__ void block_exscan_d3(const double (&v)[3], double (&pre)[3], double (&tot)[3], RSmem& sm) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  double x[3] = {v[0], v[1], v[2]};
  for (int o = 1; o < 32; o <<= 1) {
    double y[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) y[k] = __shfl_up_sync(0xffffffffu, x[k], o);
    if (l >= o)
#pragma unroll
      for (int k = 0; k < 3; ++k) x[k] += y[k];
  }
  if (l == 31)
#pragma unroll
    for (int k = 0; k < 3; ++k) sm.red_m[w * 8 + k] = x[k];
  __syncthreads();
  if (w == 0) {
    double t[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) t[k] = l < NWARP ? sm.red_m[l * 8 + k] : 0.0;
    for (int o = 1; o < 32; o <<= 1) {
      double y[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) y[k] = __shfl_up_sync(0xffffffffu, t[k], o);
      if (l >= o)
#pragma unroll
        for (int k = 0; k < 3; ++k) t[k] += y[k];
    }
    if (l < NWARP)
#pragma unroll
      for (int k = 0; k < 3; ++k) sm.red_m[l * 8 + k] = t[k];  // inclusive warp prefixes
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    pre[k] = (w > 0 ? sm.red_m[(w - 1) * 8 + k] : 0.0) + x[k] - v[k];
    tot[k] = sm.red_m[(NWARP - 1) * 8 + k];
  }
  __syncthreads();
}

// ---------------------------------------------------------------- selection

enum Crit : int { kCount = 0, kMassGE = 1, kMassGT = 2 };

constexpr double kNoQx = __builtin_nan("");

struct Cut {
  unsigned long long K;  // composite key of the last element of the prefix
  long long cnt;         // prefix length
  double mass;           // prefix mass sum exp(s - m)
  double qx = kNoQx;     // prefix sum of exp(s - m) (s - m), when the path formed it
};

__device__ __forceinline__ bool crit_ok(int crit, long long c, double mss, long long need, double target) {
  return crit == kCount ? (c >= need) : (crit == kMassGE ? (mss >= target) : (mss > target));
}

__device__ __forceinline__ void take_earlier(Cut& best, const Cut& c) {
  if (c.K > best.K) best = c;
}

// Over the NB buckets in sm.cnt / sm.mass (bucket 0 = earliest in the order),
// pick the first bucket where (above + inclusive prefix) meets the criterion,
// or the last non-empty bucket if none does. Returns it with the count and
// mass of everything before it (above included).
__device__ __noinline__ void pick_bucket(RSmem& sm, int crit, long long need, double target, long long above_cnt,
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
  int b = block_min_i(mine, sm);
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

// Level-0 histogram of the row (counts and float64 masses per bucket); also
// the total mass and the last element of the order when asked.
template <bool VEC>
__device__ __noinline__ void build_hist0(RSmem& sm, const float* __restrict__ x, int V, float m, double* Z,
                            unsigned long long* Kmin) {
  for (int i = threadIdx.x; i < NB; i += RT) {
    sm.cnt[i] = 0;
    sm.mass[i] = 0.0;
  }
  __syncthreads();
  const double md = (double)m;
  double zl = 0.0;
  unsigned long long kl = ~0ull;
  for_each<VEC>(x, V, [&](float s, int i) {
    const int b = bin0(s, m);
    const double q = qmass_b(sm.tab, s, md, b);
    atomicAdd(&sm.cnt[b], 1);
    atomicAdd(&sm.mass[b], q);
    zl += q;
    const unsigned long long K = ckey(s, i);
    kl = K < kl ? K : kl;
  });
  __syncthreads();
  if (Z) *Z = block_sum_d(zl, sm);
  if (Kmin) *Kmin = block_ext_u<false>(kl, sm);
}

// Bitonic sort of sm.cand[0, n) into descending order (composite keys are
// distinct), then the inclusive float64 scan of their masses into sm.cq[0, n)
// (thread order, deterministic). The first NW warps sort a padded run of
// N2 = 32 * NW * E keys: element i = t * E + e lives in register v[e] of
// thread t, so compare-exchange partners closer than E are in one thread,
// partners closer than 32 E are a warp shuffle away, and only the wider stages
// (log2(NW) (log2(NW) + 1) / 2 of them) go through shared memory, one barrier
// each, alternating between the two halves of sm.cand. Padding keys are 0 and
// sort last.
template <int E, int NW>
__device__ void sort_scan_regs(RSmem& sm, int n, float m) {
  constexpr int N2 = 32 * NW * E;
  static_assert(NW <= NWARP && 2 * N2 <= CAP, "two shared-stage buffers fit the candidate buffer");
  const int t = (int)threadIdx.x;
  const bool part = t < 32 * NW;  // whole warps: shuffles stay within a warp
  unsigned long long v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = t * E + e;
    v[e] = (part && i < n) ? sm.cand[i] : 0ull;
  }
  int buf = 0;
  for (int k = 2; k <= N2; k <<= 1) {
    int j = k >> 1;
    for (; j >= 32 * E; j >>= 1) {  // across warps: through shared memory
      unsigned long long* c = sm.cand + buf * N2;
      if (part)
#pragma unroll
        for (int e = 0; e < E; ++e) c[t * E + e] = v[e];
      __syncthreads();
      if (part)
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = t * E + e;
          const unsigned long long o = c[i ^ j];
          const bool keep_hi = ((i & j) == 0) == ((i & k) == 0);
          v[e] = keep_hi ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
        }
      buf ^= 1;
    }
    for (; j >= E; j >>= 1) {  // across lanes: warp shuffles
      const int lj = j / E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int i = t * E + e;
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[e], lj);
        const bool keep_hi = ((i & j) == 0) == ((i & k) == 0);
        v[e] = keep_hi ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
      }
    }
#pragma unroll
    for (int jj = E / 2; jj > 0; jj >>= 1) {  // within the thread
      if (jj >= k) continue;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int q = e ^ jj;
        if (q > e) {
          const bool desc = ((t * E + e) & k) == 0;
          const unsigned long long x0 = v[e], x1 = v[q];
          const unsigned long long hi = x0 > x1 ? x0 : x1, lo = x0 > x1 ? x1 : x0;
          v[e] = desc ? hi : lo;
          v[q] = desc ? lo : hi;
        }
      }
    }
  }
  double loc[E];
  double run = 0.0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = t * E + e;
    run += (part && i < n) ? qmass(sm, ckey_value(v[e]), m) : 0.0;
    loc[e] = run;
  }
  double tot;
  const double off = block_exscan<double>(run, sm.red_d, tot);  // its barriers end the shared stages
  if (part)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int i = t * E + e;
      sm.cand[i] = v[e];
      sm.cq[i] = off + loc[e];
    }
  __syncthreads();
}

// Sorts sm.cand[0, n) (n <= SCAP) and scans the masses into sm.cq[0, n).
__device__ __noinline__ void sort_and_scan(RSmem& sm, int n, float m) {
  n = min(n, SCAP);
  if (n <= 64)
    sort_scan_regs<2, 1>(sm, n, m);  // one warp, no shared stage
  else if (n <= 256)
    sort_scan_regs<2, 4>(sm, n, m);
  else if (n <= 1024)
    sort_scan_regs<2, NWARP>(sm, n, m);
  else if (n <= 2048)
    sort_scan_regs<4, NWARP>(sm, n, m);
  else
    sort_scan_regs<8, NWARP>(sm, n, m);
}

// First j in [lo, hi) with C(j) = base_mass + (cq[j] - cq_before) meeting a
// mass criterion; hi - 1 if none does.
__device__ __noinline__ int first_mass_hit(RSmem& sm, int lo, int hi, double base_mass, double cq_before, int crit,
                              double target) {
  int mine = CAP;
  for (int j = lo + (int)threadIdx.x; j < hi; j += RT) {
    if (crit_ok(crit, 0, base_mass + (sm.cq[j] - cq_before), 0, target)) {
      mine = j;
      break;
    }
  }
  int j = block_min_i(mine, sm);
  if (j >= hi) j = hi - 1;
  return j;
}

// Warp-cooperative append: every active lane with `take` set gets a distinct
// slot from one atomic per warp on *counter (no same-address contention).
__device__ __forceinline__ int warp_slot(int* counter, bool take) {
  const unsigned act = __activemask();
  const unsigned mask = __ballot_sync(act, take);
  if (mask == 0u) return -1;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(mask) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(counter, __popc(mask));
  base = __shfl_sync(act, base, leader);
  return take ? base + __popc(mask & ((1u << lane) - 1u)) : -1;
}

// General search: the element of the order where the criterion is first met,
// refining oversized buckets. Returns false if the refinement bound is hit.
template <bool VEC>
__device__ __noinline__ bool locate(RSmem& sm, const float* __restrict__ x, int V, float m, bool& hist_valid,
                       int crit, long long need, double target, Cut& out) {
  const double md = (double)m;
  if (!hist_valid) {
    build_hist0<VEC>(sm, x, V, m, nullptr, nullptr);
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

  for (int level = 0; set_cnt > SCAP; ++level) {
    if (level >= MAX_LEVELS) return false;
    unsigned long long kmin = ~0ull, kmax = 0ull;
    for_each<VEC>(x, V, [&](float s, int i) {
      if (bin0(s, m) != b) return;
      const unsigned long long K = ckey(s, i);
      if (refined && (K < Klo || K > Khi)) return;
      kmin = K < kmin ? K : kmin;
      kmax = K > kmax ? K : kmax;
    });
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
    for_each<VEC>(x, V, [&](float s, int i) {
      const int b0 = bin0(s, m);
      if (b0 != b) return;
      const unsigned long long K = ckey(s, i);
      if (K < Klo || K > Khi) return;
      const int sb = (int)((Khi - K) >> shift);
      atomicAdd(&sm.cnt[sb], 1);
      atomicAdd(&sm.mass[sb], qmass_b(sm.tab, s, md, b0));
    });
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

  if (threadIdx.x == 0) sm.ncand = 0;
  __syncthreads();
  for_each<VEC>(x, V, [&](float s, int i) {
    const unsigned long long K = ckey(s, i);
    const bool take = bin0(s, m) == b && !(refined && (K < Klo || K > Khi));
    const int slot = warp_slot(&sm.ncand, take);
    if (slot >= 0 && slot < CAP) sm.cand[slot] = K;
  });
  __syncthreads();
  const int n = min(sm.ncand, CAP);
  sort_and_scan(sm, n, m);
  hist_valid = false;  // the scan overwrote the bucket masses
  int jstar;
  if (crit == kCount)
    jstar = (int)(need - above_cnt - 1);
  else
    jstar = first_mass_hit(sm, 0, n, above_mass, 0.0, crit, target);
  jstar = max(0, min(jstar, n - 1));
  out.K = sm.cand[jstar];
  out.cnt = above_cnt + jstar + 1;
  out.mass = above_mass + sm.cq[jstar];
  __syncthreads();
  return true;
}

// The prefix kept by min-p: every element with key >= kt (one pass).
template <bool VEC>
__device__ __noinline__ Cut min_p_cut_pass(RSmem& sm, const float* __restrict__ x, int V, float m, uint32_t kt) {
  long long c = 0;
  double ms = 0.0;
  unsigned long long kl = ~0ull;
  for_each<VEC>(x, V, [&](float s, int i) {
    if (key32(s) >= kt) {
      ++c;
      ms += qmass(sm, s, m);
      const unsigned long long K = ckey(s, i);
      kl = K < kl ? K : kl;
    }
  });
  Cut cm;
  cm.K = block_ext_u<false>(kl, sm);
  cm.cnt = block_sum_l(c, sm);
  cm.mass = block_sum_d(ms, sm);
  return cm;
}

template <bool VEC>
__device__ __noinline__ float row_max_pass(const float* __restrict__ x, int V) {
  float lm = -INFINITY;
  for_each<VEC>(x, V, [&](float s, int) { lm = fmaxf(lm, s); });
  return lm;
}


// Gather the elements of buckets bp and bm (either may be -1) into sm.cand
// and, when kt is live, return the last element with key >= kt among the

// ---------------------------------------------------------------- exact path
// Float64 mass histogram (atomics) and the general search: used when the fast
// path below cannot prove its window holds the cut (a bucket too large for
// the sort, a crossing outside the estimated window).
template <bool VEC>
__device__ __noinline__ bool resolve_row_exact(RSmem& sm, const float* __restrict__ x, int V,
                                               float m, int k, float p, float mu, uint32_t kt,
                                               bool& hist_valid, Cut& best) {
  const bool k_on = k >= 1 && k < V, p_on = p < 1.0f, mu_on = mu > 0.0f;
  double Z;
  unsigned long long Klast;
  build_hist0<VEC>(sm, x, V, m, &Z, &Klast);
  hist_valid = true;
  best = Cut{Klast, (long long)V, Z};
  double Zk = Z;
  if (k_on) {
    Cut ck;
    if (!locate<VEC>(sm, x, V, m, hist_valid, kCount, (long long)k, 0.0, ck)) return false;
    Zk = ck.mass;
    take_earlier(best, ck);
  }
  if (p_on) {
    Cut cp;
    if (!locate<VEC>(sm, x, V, m, hist_valid, kMassGE, 0, (double)p * Zk, cp)) return false;
    take_earlier(best, cp);
  }
  if (mu_on) take_earlier(best, min_p_cut_pass<VEC>(sm, x, V, m, kt));
  return true;
}

// ---------------------------------------------------------------- fast path

// Whether element e belongs to the planning sample (with float4 streaming, one
// chunk in SAMPLE_EVERY and the scalar tail; else one block of RT elements in
// SAMPLE_EVERY): see sample_hist.
template <bool VEC>
__device__ __forceinline__ bool in_sample(int e, int V) {
  if (VEC) return e >= (V & ~3) || (((e >> 2) / CH_F4) % SAMPLE_EVERY) == 0;
  return ((e / RT) % SAMPLE_EVERY) == 0;
}

// Count-only level-0 histogram. With `sampled`, sm.cnt already holds the
// counts of the planning sample and only the other elements are added.
template <bool VEC>
__device__ __noinline__ void count_hist(RSmem& sm, const float* __restrict__ x, int V, float m,
                                        bool sampled) {
  if (!sampled) {
    for (int i = threadIdx.x; i < NB; i += RT) sm.cnt[i] = 0;
    __syncthreads();
  }
  if (VEC) {
    // every chunk, or the ones the sample skipped (chunk j + j / 7 + 1 is the
    // j-th chunk that is not a multiple of SAMPLE_EVERY)
    const float4* __restrict__ x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    const int nch = n_chunks(V4);
    const int n = sampled ? nch - (nch + SAMPLE_EVERY - 1) / SAMPLE_EVERY : nch;
    auto body = [&](auto, const float4& u, int, const float4& w, int, bool vu, bool vw) {
      if (vu) {
        atomicAdd(&sm.cnt[bin0(u.x, m)], 1);
        atomicAdd(&sm.cnt[bin0(u.y, m)], 1);
        atomicAdd(&sm.cnt[bin0(u.z, m)], 1);
        atomicAdd(&sm.cnt[bin0(u.w, m)], 1);
      }
      if (vw) {
        atomicAdd(&sm.cnt[bin0(w.x, m)], 1);
        atomicAdd(&sm.cnt[bin0(w.y, m)], 1);
        atomicAdd(&sm.cnt[bin0(w.z, m)], 1);
        atomicAdd(&sm.cnt[bin0(w.w, m)], 1);
      }
    };
    if (sampled)
      stream_chunks(sm, x4, V4, n,
                    [](int j) { return j + j / (SAMPLE_EVERY - 1) + 1; }, l2_policy_keep(), body);
    else
      stream_chunks(sm, x4, V4, n, [](int j) { return j; }, l2_policy_keep(), body);
    if (!sampled)
      for (int i = 4 * V4 + (int)threadIdx.x; i < V; i += RT)
        atomicAdd(&sm.cnt[bin0(ld_stream(x + i), m)], 1);
  } else if (!sampled) {
    for_each<false, true>(x, V, [&](float s, int) { atomicAdd(&sm.cnt[bin0(s, m)], 1); });
  } else {
    for_each<false, true>(x, V, [&](float s, int e) {
      if (!in_sample<false>(e, V)) atomicAdd(&sm.cnt[bin0(s, m)], 1);
    });
  }
  __syncthreads();
}

// Sum of counts over buckets [lo, hi).
__device__ long long count_range(RSmem& sm, int lo, int hi) {
  long long c = 0;
  for (int i = lo + (int)threadIdx.x; i < hi; i += RT) c += sm.cnt[i];
  return block_sum_l(c, sm);
}

// Results of pass 2.
struct Pass2 {
  double z, a_p, a_mu;       // total mass, mass before w_lo, mass before b_mu
  double zx, a_px, a_mux;    // the same sums of exp(s - m) (s - m) (when asked)
  long long c_p, c_mu;       // counts before w_lo and before b_mu (when counted)
  unsigned long long k_last; // last element of the order (when asked)
  bool overflow;             // a warp's gather slice overflowed
};

// Plan of pass 2, passed by value so every field lives in a register.
struct Plan2 {
  int need_last;            // last element of the order (per-thread key minimum)
  int g_lo, g_hi;           // gather buckets [g_lo, g_hi] ...
  int g2_lo, g2_hi;         // ... and [g2_lo, g2_hi] (empty ranges: lo > hi)
  int w_lo;                 // mass before w_lo is accumulated (a_p)
  int b_mu;                 // mass before b_mu is accumulated (a_mu); -1: off
  int ent;                  // also sum exp(s - m) (s - m) per region (entropy)
};

constexpr int TCAP = CAP / RT;  // private gather slots per thread, interleaved across threads

// Per-element tests in the streaming passes combine their comparisons with
// bitwise & and | rather than && and ||: the short-circuit forms compile to
// branches, which halved a pass's throughput in a streaming microbenchmark.
//
// Appends the keys of the elements flagged in gm (bit e: element e of the
// batch) to this thread's gather slots. Hits are rare, so the warp first ORs
// its lanes' flags and visits only the element positions that some lane hit
// (a warp-uniform branch each) instead of predicating all eight.
template <typename KF>
__device__ __forceinline__ void append_hits(unsigned gm, unsigned long long* tbuf, int& tfill,
                                            KF&& key_of) {
  const unsigned wm = __reduce_or_sync(0xffffffffu, gm);
  if (wm == 0u) return;
#pragma unroll
  for (int e = 0; e < 8; ++e)
    if ((wm >> e) & 1u) {
      if ((gm >> e) & 1u) {
        if (tfill < TCAP) tbuf[tfill * RT] = key_of(e);
        ++tfill;
      }
    }
}

// One pass over the row: exact float64 masses accumulated in registers, and
// the elements of up to two bucket ranges gathered into per-thread slots of
// sm.cand. The mass polynomial of E consecutive elements is evaluated as
// independent chains and summed into split accumulators, so float64 latency
// is covered. Every lane of a warp runs every batch (invalid slots masked), so
// the warp votes always see the full warp.
// TWO: the second gather range may be non-empty (false: compiled out, for the
// top-p rows without min-p, the common case).
template <bool VEC, bool NEED_Z, bool COUNTS, bool TWO = true>
__device__ __noinline__ void pass2_impl(RSmem& sm, const float* __restrict__ x, int V, float m,
                                        const Plan2 pl, Pass2& P) {
  constexpr int E = 8;
  const double md = (double)m;
  const bool need_last = pl.need_last != 0;
  const int g_lo = pl.g_lo, g_hi = pl.g_hi, g2_lo = pl.g2_lo, g2_hi = pl.g2_hi;
  const int w_lo = pl.w_lo, b_mu = pl.b_mu;
  // gather ranges as (start, span) for one unsigned compare each; an empty
  // range (lo > hi) gets a start no bucket reaches
  const unsigned g1s = g_lo <= g_hi ? (unsigned)g_lo : 0x80000000u;
  const unsigned g1n = g_lo <= g_hi ? (unsigned)(g_hi - g_lo) : 0u;
  const unsigned g2s = g2_lo <= g2_hi ? (unsigned)g2_lo : 0x80000000u;
  const unsigned g2n = g2_lo <= g2_hi ? (unsigned)(g2_hi - g2_lo) : 0u;
  unsigned long long* tbuf = sm.cand + threadIdx.x;  // this thread's slots, stride RT
  int tfill = 0;
  double z[2] = {0.0, 0.0}, ap[2] = {0.0, 0.0}, amu[2] = {0.0, 0.0};
  double zx = 0.0, apx = 0.0, amux = 0.0;  // the same sums of q (s - m) (entropy)
  const bool ent = pl.ent != 0;
  int cp = 0, cmu = 0;  // counts before w_lo and before b_mu (COUNTS)
  unsigned long long kl = ~0ull;

  // Element e < 4 of a batch is token a0 + e (valid when e < na), element
  // e >= 4 is token b0 + e - 4 (valid when e - 4 < nb); `full` (a type)
  // states at compile time that all are valid, which holds for every sweep
  // but the last. The body has no per-element branches: masses are computed
  // for all E elements and selected, the far tail (bucket NB - 1) takes one
  // warp vote per batch, the gather votes run only when some lane of the warp
  // has an element to gather, and each gather store is predicated on its
  // ballot rather than branched over.
  const bool need_mass = NEED_Z || b_mu >= 0;
  const bool need_mu = b_mu >= 0;
  auto batch = [&](auto full, const float (&sv)[E], int a0, int na, int b0, int nb) {
    auto idx = [&](int e) { return e < 4 ? a0 + e : b0 + (e - 4); };
    auto ok = [&](int e) { return decltype(full)::value || (e < 4 ? e < na : e - 4 < nb); };
    int bb[E];
#pragma unroll
    for (int e = 0; e < E; ++e) bb[e] = bin0(sv[e], m);
    if (need_mass) {
      double qq[E];
      bool far = false;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const double xx = (double)sv[e] - md;
        const double r = fma((double)bb[e], 1.0 / 128.0, xx);
        double p = 1.0 / 720.0;
        p = fma(p, r, 1.0 / 120.0);
        p = fma(p, r, 1.0 / 24.0);
        p = fma(p, r, 1.0 / 6.0);
        p = fma(p, r, 0.5);
        p = fma(p, r, 1.0);
        p = fma(p, r, 1.0);
        qq[e] = tab_at(sm.tab, bb[e]) * p;
        far |= bb[e] >= NB - 1;
      }
      if (__any_sync(0xffffffffu, far)) {
#pragma unroll
        for (int e = 0; e < E; ++e)
          if (bb[e] >= NB - 1) qq[e] = far_mass((double)sv[e] - md);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) qq[e] = ok(e) ? qq[e] : 0.0;
      // predicated adds (no selects): a region's sum only takes its elements
      if (NEED_Z)
#pragma unroll
        for (int e = 0; e < E; ++e) {
          z[e & 1] += qq[e];
          if (bb[e] < w_lo) ap[e & 1] += qq[e];
        }
      if (need_mu)
#pragma unroll
        for (int e = 0; e < E; ++e)
          if (bb[e] < b_mu) amu[e & 1] += qq[e];
      if (ent) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const double qx = ok(e) ? qq[e] * ((double)sv[e] - md) : 0.0;
          if (NEED_Z) {
            zx += qx;
            if (bb[e] < w_lo) apx += qx;
          }
          if (need_mu & (bb[e] < b_mu)) amux += qx;
        }
      }
    }
    if (COUNTS) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        cp += (int)(ok(e) & (bb[e] < w_lo));
        cmu += (int)(ok(e) & (bb[e] < b_mu));
      }
    }
    if (need_last) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const unsigned long long K = ok(e) ? ckey(sv[e], idx(e)) : ~0ull;
        kl = K < kl ? K : kl;
      }
    }
    unsigned gm = 0;  // this thread's elements in a gathered range, one bit each
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const unsigned b = (unsigned)bb[e];
      const bool g = TWO ? ok(e) & ((b - g1s <= g1n) | (b - g2s <= g2n)) : ok(e) & (b - g1s <= g1n);
      gm |= g ? 1u << e : 0u;
    }
    // each thread appends its hits to its own slots (no coordination between
    // lanes)
    append_hits(gm, tbuf, tfill, [&](int e) { return ckey(sv[e], idx(e)); });
  };

  const int tid = (int)threadIdx.x;
  int tail0 = 0;  // first token handled one per thread
  if (VEC) {
    // the row streams through the ring; a batch is two of the thread's
    // float4s of a chunk (the loads read evict-first: this is the row's last pass)
    const float4* __restrict__ x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    stream_chunks(sm, x4, V4, n_chunks(V4), [](int j) { return j; }, l2_policy_drop(),
                  [&](auto full, const float4& a4, int ia, const float4& b4, int ib, bool va,
                      bool vb) {
                    const float sv[E] = {a4.x, a4.y, a4.z, a4.w, b4.x, b4.y, b4.z, b4.w};
                    batch(full, sv, 4 * ia, va ? 4 : 0, 4 * ib, vb ? 4 : 0);
                  });
    tail0 = 4 * V4;
  }
  for (int i0 = tail0; i0 < V; i0 += RT) {
    const int i = i0 + tid;
    const bool in = i < V;
    const float t = in ? ld_stream(x + i) : 0.f;
    const float sv[E] = {t, t, t, t, t, t, t, t};
    batch(std::false_type{}, sv, i, in ? 1 : 0, i, 0);
  }
  sm.tcount[threadIdx.x] = tfill;
  {
    double sums[8] = {z[0] + z[1], ap[0] + ap[1], amu[0] + amu[1], (double)cp, (double)cmu,
                      zx, apx, amux};
    block_sum_multi<8>(sums, sm);  // counts are exact in a double
    P.z = sums[0];
    P.a_p = sums[1];
    P.a_mu = sums[2];
    P.c_p = (long long)sums[3];
    P.c_mu = (long long)sums[4];
    P.zx = sums[5];
    P.a_px = sums[6];
    P.a_mux = sums[7];
  }
  P.k_last = need_last ? block_ext_u<false>(kl, sm) : ~0ull;
  P.overflow = __syncthreads_or(tfill > TCAP) != 0;
}

// A pass that only gathers: the elements of up to two bucket ranges, tested
// by value against the ranges widened by a bucket on each side (a superset:
// the readers select the exact buckets), so no bucket index is formed.
template <bool VEC>
__device__ __noinline__ void gather_pass(RSmem& sm, const float* __restrict__ x, int V, float m,
                                         const Plan2 pl, Pass2& P) {
  constexpr int E = 8;
  auto widen = [&](int lo, int hi, float& vlo, float& vhi) {
    if (lo > hi) {
      vlo = INFINITY;
      vhi = -INFINITY;
      return;
    }
    vlo = hi >= NB - 1 ? -INFINITY : m - (float)(hi + 2) * (1.0f / BIN_SCALE);
    vhi = lo <= 0 ? INFINITY : m - (float)(lo - 1) * (1.0f / BIN_SCALE);
  };
  float l1, h1, l2, h2;
  widen(pl.g_lo, pl.g_hi, l1, h1);
  widen(pl.g2_lo, pl.g2_hi, l2, h2);
  const int tid = (int)threadIdx.x;
  unsigned long long* tbuf = sm.cand + tid;
  int tfill = 0;
  auto batch = [&](auto full, const float (&sv)[E], int a0, int na, int b0, int nb) {
    auto idx = [&](int e) { return e < 4 ? a0 + e : b0 + (e - 4); };
    auto ok = [&](int e) { return decltype(full)::value || (e < 4 ? e < na : e - 4 < nb); };
    unsigned gm = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float s = sv[e];
      const bool g = ok(e) & (((s >= l1) & (s <= h1)) | ((s >= l2) & (s <= h2)));
      gm |= g ? 1u << e : 0u;
    }
    append_hits(gm, tbuf, tfill, [&](int e) { return ckey(sv[e], idx(e)); });
  };
  int tail0 = 0;
  if (VEC) {
    const float4* __restrict__ x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    stream_chunks(sm, x4, V4, n_chunks(V4), [](int j) { return j; }, l2_policy_drop(),
                  [&](auto full, const float4& a4, int ia, const float4& b4, int ib, bool va,
                      bool vb) {
                    const float sv[E] = {a4.x, a4.y, a4.z, a4.w, b4.x, b4.y, b4.z, b4.w};
                    batch(full, sv, 4 * ia, va ? 4 : 0, 4 * ib, vb ? 4 : 0);
                  });
    tail0 = 4 * V4;
  }
  for (int i0 = tail0; i0 < V; i0 += RT) {
    const int i = i0 + tid;
    const bool in = i < V;
    const float s = in ? ld_stream(x + i) : 0.f;
    const float sv[E] = {s, s, s, s, s, s, s, s};
    batch(std::false_type{}, sv, i, in ? 1 : 0, i, 0);
  }
  sm.tcount[tid] = tfill;
  P.z = P.a_p = P.a_mu = P.zx = P.a_px = P.a_mux = 0.0;
  P.c_p = P.c_mu = 0;
  P.k_last = ~0ull;
  P.overflow = __syncthreads_or(tfill > TCAP) != 0;
}

template <bool VEC>
__device__ void pass2(RSmem& sm, const float* __restrict__ x, int V, float m, bool need_z,
                      const Plan2& pl, Pass2& P, bool counts = false) {
  if (!need_z && !counts && pl.b_mu < 0 && !pl.need_last) {  // nothing weighed or counted
    gather_pass<VEC>(sm, x, V, m, pl, P);
    return;
  }
  if (counts) {
    if (need_z)
      pass2_impl<VEC, true, true>(sm, x, V, m, pl, P);
    else
      pass2_impl<VEC, false, true>(sm, x, V, m, pl, P);
  } else {
    if (need_z) {
      if (pl.g2_lo > pl.g2_hi && pl.b_mu < 0)
        pass2_impl<VEC, true, false, false>(sm, x, V, m, pl, P);
      else
        pass2_impl<VEC, true, false>(sm, x, V, m, pl, P);
    } else {
      pass2_impl<VEC, false, false>(sm, x, V, m, pl, P);
    }
  }
}

// ---------------------------------------------------------------- min-p pass
// One pass for a row whose min-p prefix decides the support. Elements in
// buckets below g_lo are all kept: each thread stages their values in its
// own slots and weighs them in float64 eight at a time (so the float64 work
// follows the kept elements, not the row). Elements in buckets [g_lo, g_hi]
// are gathered (their keys decide which are kept). Elements after g_hi are
// dropped: they only add to a lower bound of their mass, each at least
// tab[b] exp(-1/128) = 2^(-(b + 1) log2(e) / 128), summed in fp32.
struct MuPass {
  double mass, qx;     // kept elements before g_lo: mass and sum of q (s - m)
  long long cnt;       // their number
  double rest_lower;   // lower bound of the mass of the elements after g_hi
  bool overflow;       // the gather slots overflowed
};

constexpr int MU_SLOTS = NB * 8 / 4 / RT;  // staged fp32 values per thread (the sm.mass storage)
static_assert(MU_SLOTS >= 16, "a thread stages up to 7 + 8 values");

// Level-0 bucket of s as an int and as a float (the same floor as bin0).
__device__ __forceinline__ int bin0_both(float s, float m, float& bf) {
  const float f = fminf(fmaxf(fmaf(s, -BIN_SCALE, m * BIN_SCALE), 0.0f), (float)(NB - 1));
  const float fl = __fadd_rd(f, 8388608.0f);
  bf = fl - 8388608.0f;
  return __float_as_int(fl) - 0x4B000000;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool VEC>
__device__ __noinline__ void mu_pass(RSmem& sm, const float* __restrict__ x, int V, float m,
                                     int g_lo, int g_hi, bool ent, MuPass& out) {
  constexpr int E = 8;
  constexpr float kL = 1.4426950408889634f / 128.0f;  // log2(e) / 128
  const double md = (double)m;
  const int tid = (int)threadIdx.x;
  float* stage = reinterpret_cast<float*>(sm.mass) + tid;  // slot j at stage[j RT]
  unsigned long long* tbuf = sm.cand + tid;
  int sf = 0, tfill = 0, cnt = 0;
  double mass = 0.0, qx = 0.0;
  float rest = 0.0f;
  const unsigned gs = (unsigned)g_lo, gn = (unsigned)(g_hi - g_lo);

  // weigh this thread's first n <= 8 staged values
  auto weigh = [&](int n) {
#pragma unroll
    for (int j = 0; j < E; ++j)
      if (j < n) {
        const float s = stage[j * RT];
        const double q = qmass_b(sm.tab, s, md, bin0(s, m));
        mass += q;
        if (ent) qx += q * ((double)s - md);
      }
  };

  auto batch = [&](auto full, const float (&sv)[E], int a0, int na, int b0, int nb) {
    auto idx = [&](int e) { return e < 4 ? a0 + e : b0 + (e - 4); };
    auto ok = [&](int e) { return decltype(full)::value || (e < 4 ? e < na : e - 4 < nb); };
    unsigned gm = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float bf;
      const int b = bin0_both(sv[e], m, bf);
      const bool v = ok(e);
      if (v & (b < g_lo)) {
        stage[sf * RT] = sv[e];
        ++sf;
      }
      gm |= (unsigned)(v & ((unsigned)b - gs <= gn)) << e;
      if (v & (b > g_hi)) rest += ex2_approx(-(bf + 1.0f) * kL);
    }
    if (__any_sync(0xffffffffu, sf >= E)) {  // weigh eight, keep the rest staged
      const int n = min(sf, E);
      cnt += n;
      weigh(n);
#pragma unroll
      for (int j = 0; j < E - 1; ++j)
        if (j + E < sf) stage[j * RT] = stage[(j + E) * RT];
      sf -= n;
    }
    append_hits(gm, tbuf, tfill, [&](int e) { return ckey(sv[e], idx(e)); });
  };

  int tail0 = 0;
  if (VEC) {
    const float4* __restrict__ x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    stream_chunks(sm, x4, V4, n_chunks(V4), [](int j) { return j; }, l2_policy_drop(),
                  [&](auto full, const float4& a4, int ia, const float4& b4, int ib, bool va,
                      bool vb) {
                    const float sv[E] = {a4.x, a4.y, a4.z, a4.w, b4.x, b4.y, b4.z, b4.w};
                    batch(full, sv, 4 * ia, va ? 4 : 0, 4 * ib, vb ? 4 : 0);
                  });
    tail0 = 4 * V4;
  }
  for (int i0 = tail0; i0 < V; i0 += RT * 2) {
    const int ia = i0 + tid, ib = ia + RT;
    const float a = ia < V ? ld_stream(x + ia) : 0.f, b = ib < V ? ld_stream(x + ib) : 0.f;
    const float sv[E] = {a, a, a, a, b, b, b, b};
    batch(std::false_type{}, sv, ia, ia < V ? 1 : 0, ib, ib < V ? 1 : 0);
  }
  {  // the values still staged (at most E - 1 after the last batch)
    const int n = min(sf, E);
    cnt += n;
    weigh(n);
  }
  sm.tcount[tid] = tfill;
  // each fp32 term is within 2^-22 of its value and a thread sums a few hundred:
  // 1e-4 covers both roundings, so the bound stays a lower bound
  double sums[4] = {mass, qx, (double)rest * (1.0 - 1e-4), (double)cnt};
  block_sum_multi<4>(sums, sm);
  out.mass = sums[0];
  out.qx = sums[1];
  out.rest_lower = sums[2];
  out.cnt = (long long)sums[3];
  out.overflow = __syncthreads_or(tfill > TCAP) != 0;
}

// ---------------------------------------------------------------- fp32-mass passes
// Identity rows and rows whose min-p prefix decides need no comparison of
// masses to find their support (min-p compares values), only the support's
// mass for LSE_S and, with top-p on, a certificate that the top-p crossing
// comes after the min-p prefix. Without the entropy output (and outside the
// sampler, whose inverse CDF compares masses) they are weighed in fp32:
// q = ex2((s - m) log2 e), d = s - m and the product each rounded once, eight
// terms summed in fp32 per batch and the batch sums added in float64.
//
// Error bound (u = 2^-24): the exponent is off by at most 3u |y| (three
// roundings), so a term's relative error is at most 3u |d| plus ex2.approx's
// own (a few ulp). Over a set of n terms containing the row max (d = 0,
// q = 1, so Z >= 1), sum q |d| = Z (H - ln Z) <= Z ln n with H the set's
// Shannon entropy; the relative error of the sum is therefore at most
// 3u ln(2^31) + 7u (the batch sums) = 4.3e-6 plus ex2.approx's. MASS_EPS =
// 2e-5 covers it with room for an ex2 error of 100 ulp.
constexpr double MASS_EPS = 2e-5;

struct FastPass {
  double kept, rest;           // masses of the kept elements and of the others
  long long cnt;               // kept elements
  unsigned long long k_last;   // identity rows: the last element of the order
  bool overflow;               // the gather slots overflowed (min-p rows)
};

// MODE 0 (identity): every element is kept; each thread tracks its smallest
// value and, among equal ones, its largest id (its elements come in increasing
// id order, so "<=" takes the later one), which gives the last element of the
// (s desc, id asc) order. MODE 1 (min-p): an element is kept iff s >= thr;
// kept elements with s <= hv are gathered (hv bounds the buckets that hold
// the last kept element, with a bucket of slack).
template <bool VEC, int MODE>
__device__ __noinline__ void fast_pass(RSmem& sm, const float* __restrict__ x, int V, float m,
                                       float thr, float hv, FastPass& out) {
  constexpr int E = 8;
  constexpr float kLog2e = 1.4426950408889634f;
  const int tid = (int)threadIdx.x;
  unsigned long long* tbuf = sm.cand + tid;
  int tfill = 0, cnt = 0;
  double kd = 0.0, rd = 0.0;
  float vmin = INFINITY;
  int imax = -1;

  auto batch = [&](auto full, const float (&sv)[E], int a0, int na, int b0, int nb) {
    auto idx = [&](int e) { return e < 4 ? a0 + e : b0 + (e - 4); };
    auto ok = [&](int e) { return decltype(full)::value || (e < 4 ? e < na : e - 4 < nb); };
    float bk = 0.0f, br = 0.0f;
    unsigned gm = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float q = ex2_approx((sv[e] - m) * kLog2e);
      if (MODE == 0) {
        if (ok(e)) {
          bk += q;
          if (sv[e] <= vmin) {
            vmin = sv[e];
            imax = idx(e);
          }
        }
      } else {
        const bool kept = ok(e) & (sv[e] >= thr);
        if (kept) {
          bk += q;
          ++cnt;
        } else if (ok(e)) {
          br += q;
        }
        gm |= (unsigned)(kept & (sv[e] <= hv)) << e;
      }
    }
    kd += (double)bk;
    if (MODE == 1) {
      rd += (double)br;
      append_hits(gm, tbuf, tfill, [&](int e) { return ckey(sv[e], idx(e)); });
    }
  };

  int tail0 = 0;
  if (VEC) {
    const float4* __restrict__ x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    stream_chunks(sm, x4, V4, n_chunks(V4), [](int j) { return j; }, l2_policy_drop(),
                  [&](auto full, const float4& a4, int ia, const float4& b4, int ib, bool va,
                      bool vb) {
                    const float sv[E] = {a4.x, a4.y, a4.z, a4.w, b4.x, b4.y, b4.z, b4.w};
                    batch(full, sv, 4 * ia, va ? 4 : 0, 4 * ib, vb ? 4 : 0);
                  });
    tail0 = 4 * V4;
  }
  for (int i0 = tail0; i0 < V; i0 += RT) {
    const int i = i0 + tid;
    const bool in = i < V;
    const float s = in ? ld_stream(x + i) : 0.f;
    const float sv[E] = {s, s, s, s, s, s, s, s};
    batch(std::false_type{}, sv, i, in ? 1 : 0, i, 0);
  }
  sm.tcount[tid] = tfill;
  double sums[3] = {kd, rd, (double)cnt};
  block_sum_multi<3>(sums, sm);
  out.kept = sums[0];
  out.rest = sums[1];
  out.cnt = (long long)sums[2];
  out.k_last = MODE == 0 ? block_ext_u<false>(imax >= 0 ? ckey(vmin, imax) : ~0ull, sm) : ~0ull;
  out.overflow = __syncthreads_or(tfill > TCAP) != 0;
}

// Packs the live keys of the per-warp slices densely, in slice order, into the
// storage of sm.cq (free until the sort writes its scan), so the readers below
// spread them over every thread. Returns their number (the plan bounds it by
// SCAP).
__device__ __forceinline__ unsigned long long* packed(RSmem& sm) {
  return reinterpret_cast<unsigned long long*>(sm.cq);
}

__device__ __noinline__ int pack_gathered(RSmem& sm) {
  unsigned long long* g = packed(sm);
  const int mine = min(sm.tcount[threadIdx.x], TCAP);
  long long tot;
  const int off = (int)block_exscan<long long>((long long)mine, sm.red_l, tot);
  for (int j = 0; j < mine; ++j)
    if (off + j < SCAP) g[off + j] = sm.cand[j * RT + threadIdx.x];
  __syncthreads();
  return (int)min(tot, (long long)SCAP);
}

// Move the n packed candidates whose bucket lies in [lo, hi] to
// sm.cand[0, n') (block scan, order irrelevant: they are sorted next).
// Returns n'.
__device__ __noinline__ int compact_gathered(RSmem& sm, int n, float m, int lo, int hi) {
  constexpr int PER = SCAP / RT;
  const unsigned long long* g = packed(sm);
  unsigned long long t[PER];
  int mine = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int i = j * RT + (int)threadIdx.x;
    const unsigned long long K = i < n ? g[i] : 0ull;
    const int b = bin0(ckey_value(K), m);
    t[j] = (i < n && b >= lo && b <= hi) ? K : 0ull;
    mine += t[j] != 0ull ? 1 : 0;
  }
  long long tot;
  int o = (int)block_exscan<long long>((long long)mine, sm.red_l, tot);
#pragma unroll
  for (int j = 0; j < PER; ++j)
    if (t[j] != 0ull) sm.cand[o++] = t[j];
  __syncthreads();
  return (int)tot;
}

// Exact mass and count of the n packed candidates in bucket b, and (for
// min-p) of those with key >= kt, plus the smallest such key.
__device__ __noinline__ void gathered_bucket_stats(RSmem& sm, int n, float m, int b, uint32_t kt,
                                                   double& mass, long long& cnt, double& kept_mass,
                                                   long long& kept_cnt, unsigned long long& k_min,
                                                   double& kept_qx) {
  const unsigned long long* g = packed(sm);
  double ms = 0.0, km = 0.0, kx = 0.0;
  long long c = 0, kc = 0;
  unsigned long long kmn = ~0ull;
  for (int i = threadIdx.x; i < n; i += RT) {
    const unsigned long long K = g[i];
    const float v = ckey_value(K);
    if (bin0(v, m) != b) continue;
    const double q = qmass(sm, v, m);
    ms += q;
    ++c;
    if ((uint32_t)(K >> 32) >= kt) {
      km += q;
      kx += q * ((double)v - (double)m);
      ++kc;
      kmn = K < kmn ? K : kmn;
    }
  }
  double v[5] = {ms, (double)c, km, (double)kc, kx};  // counts are exact in a double
  block_sum_multi<5>(v, sm);
  mass = v[0];
  cnt = (long long)v[1];
  kept_mass = v[2];
  kept_cnt = (long long)v[3];
  kept_qx = v[4];
  k_min = block_ext_u<false>(kmn, sm);
}

// Exact masses and counts of the n packed candidates of buckets lo..hi
// (hi - lo <= 2).
__device__ __noinline__ void window_stats(RSmem& sm, int n, float m, int lo, int hi,
                                          double (&wm)[3], long long (&wc)[3], double (&wqx)[3]) {
  const unsigned long long* g = packed(sm);
  double ms[3] = {0.0, 0.0, 0.0}, mx[3] = {0.0, 0.0, 0.0};
  long long c[3] = {0, 0, 0};
  for (int i = threadIdx.x; i < n; i += RT) {
    const float v = ckey_value(g[i]);
    const int w = bin0(v, m) - lo;
    if (w < 0 || w > hi - lo) continue;
    const double q = qmass(sm, v, m);
    const double qx = q * ((double)v - (double)m);
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      ms[u] += w == u ? q : 0.0;
      mx[u] += w == u ? qx : 0.0;
      c[u] += w == u ? 1 : 0;
    }
  }
  double v[6] = {ms[0], ms[1], ms[2], (double)c[0], (double)c[1], (double)c[2]};
  block_sum_multi<6>(v, sm);
  block_sum_multi<3>(mx, sm);
#pragma unroll
  for (int w = 0; w < 3; ++w) {
    wm[w] = v[w];
    wc[w] = (long long)v[3 + w];
    wqx[w] = mx[w];
  }
}

// Sum of exp(s - m) (s - m) over the first n keys of sm.cand (sorted): the
// part of the support's entropy sum that lies among the sorted candidates.
__device__ __noinline__ double sorted_prefix_qx(RSmem& sm, int n, float m) {
  double acc = 0.0;
  for (int j = threadIdx.x; j < n; j += RT) {
    const float v = ckey_value(sm.cand[j]);
    acc += qmass(sm, v, m) * ((double)v - (double)m);
  }
  return block_sum_d(acc, sm);
}

// Last non-empty bucket strictly before b (-1 if none).
__device__ int prev_nonempty(RSmem& sm, int b) {
  int mine = -1;
  for (int i = threadIdx.x; i < b; i += RT)
    if (sm.cnt[i] > 0) mine = i;
  return (int)block_ext_u<true>((unsigned long long)(mine + 1), sm) - 1;
}

// The estimated top-p crossing bucket from the counts alone (every element
// weighted by its bucket's mid-point mass; the far-tail bucket by 0): the first
// non-empty bucket whose inclusive estimated mass reaches p * Zhat. Returns it
// with the exact count of the elements before it, the estimated masses before
// it (e0) and of it (eb), Zhat, and sigma, the standard deviation of the
// estimate's error were the elements spread uniformly within their buckets
// (per element sd(exp(r)) = 0.00226 exp(-b / 128) for r uniform on a bucket).
struct TopPPlan {
  int b;
  long long cnt_before;
  double e0, eb, zhat, sigma;
};

__device__ __noinline__ TopPPlan plan_top_p(RSmem& sm, float p) {
  constexpr int PER = NB / RT;
  constexpr double kSdPerElement = 0.0022552;  // sd of exp(r), r ~ U(-1/128, 0]
  const int base = (int)threadIdx.x * PER;
  const double wmid = sm.bd[3];
  int c[PER];
  double q[PER];
  double loc[3] = {0.0, 0.0, 0.0};  // count, estimated mass, error variance
  int last_nz = -1;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int b = base + i;
    c[i] = sm.cnt[b];
    const double t = b < NB - 1 ? tab_at(sm.tab, b) : 0.0;
    q[i] = (double)c[i] * t * wmid;
    loc[0] += c[i];
    loc[1] += q[i];
    loc[2] += (double)c[i] * (t * kSdPerElement) * (t * kSdPerElement);
    if (c[i] > 0) last_nz = b;
  }
  double pre[3], tot[3];
  block_exscan_d3(loc, pre, tot, sm);
  const double target = (double)p * tot[1];
  int mine = NB;
  double mine_before = 0.0, mine_e0 = 0.0, mine_eb = 0.0;
  {
    double cc = pre[0], ms = pre[1];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const double before = cc, e0 = ms;
      cc += c[i];
      ms += q[i];
      if (mine == NB && c[i] > 0 && ms >= target) {
        mine = base + i;
        mine_before = before;
        mine_e0 = e0;
        mine_eb = q[i];
      }
    }
  }
  int b = block_min_i(mine, sm);
  if (b >= NB) {  // rounding kept every estimate below the target: the last non-empty bucket
    b = (int)block_ext_u<true>((unsigned long long)(unsigned)(last_nz + 1), sm) - 1;
    if (threadIdx.x == 0) {
      const double eb = (double)sm.cnt[b] * (b < NB - 1 ? tab_at(sm.tab, b) : 0.0) * wmid;
      sm.bd[0] = tot[0] - sm.cnt[b];
      sm.bd[1] = tot[1] - eb;
      sm.bd[2] = eb;
    }
  } else if (mine == b) {
    sm.bd[0] = mine_before;
    sm.bd[1] = mine_e0;
    sm.bd[2] = mine_eb;
  }
  __syncthreads();
  TopPPlan pl{b, (long long)sm.bd[0], sm.bd[1], sm.bd[2], tot[1], sqrt(tot[2])};
  __syncthreads();
  return pl;
}

// Top-k whose prefix up to the k-th element's bucket holds more than SCAP
// elements. The exact counts place the k-th element in bucket bk (with ce
// elements before it); one exact pass weighs everything before bk and gathers
// bk alone, whose sorted elements give the k-th element and the top-k mass
// Z_k = (mass before bk) + (prefix of bk). Min-p cuts earlier than the k-th
// element only when its threshold's bucket bm <= bk: within bk it is read off
// the sorted bucket, before bk one pass counts its prefix. With top-p, the
// crossing on the top-k-renormalised mass (target p Z_k, known only now) is
// placed by the exact search's locate. Returns false when bucket bk alone
// exceeds the sort (the exact search then decides).
template <bool VEC>
__device__ __noinline__ bool resolve_large_k(RSmem& sm, const float* __restrict__ x, int V, float m,
                                             int k, float p, float mu, uint32_t kt, bool ent,
                                             int bk, long long ce, Cut& best) {
  const bool p_on = p < 1.0f, mu_on = mu > 0.0f;
  if (sm.cnt[bk] > SCAP) return false;
  Plan2 pl;
  pl.need_last = 0;
  pl.g_lo = bk;
  pl.g_hi = bk;
  pl.g2_lo = 1;
  pl.g2_hi = 0;
  pl.w_lo = bk;  // a_p: the mass before bk
  pl.b_mu = -1;
  pl.ent = ent ? 1 : 0;
  Pass2 P;
  pass2<VEC>(sm, x, V, m, true, pl, P);
  if (P.overflow) return false;
  const int ng = pack_gathered(sm);
  const int n = compact_gathered(sm, ng, m, bk, bk);
  const int jk = (int)((long long)k - ce) - 1;
  if (jk < 0 || jk >= n) return false;
  sort_and_scan(sm, n, m);
  best = Cut{sm.cand[jk], (long long)k, P.a_p + sm.cq[jk]};
  const double Zk = best.mass;
  if (mu_on) {
    const int bm = bin0(key32_value(kt), m);
    if (bm == bk) {
      int mine = 0;
      for (int j = threadIdx.x; j < n; j += RT) mine += (uint32_t)(sm.cand[j] >> 32) >= kt ? 1 : 0;
      const int nk = (int)block_sum_l(mine, sm);  // kept elements of bk: a prefix of it
      if (nk >= 1)
        take_earlier(best, Cut{sm.cand[nk - 1], ce + nk, P.a_p + sm.cq[nk - 1]});
      else  // nothing of bk kept: the min-p prefix ends in an earlier bucket
        take_earlier(best, min_p_cut_pass<VEC>(sm, x, V, m, kt));
    } else if (bm < bk) {
      take_earlier(best, min_p_cut_pass<VEC>(sm, x, V, m, kt));
    }
  }
  if (ent && best.cnt > ce) best.qx = P.a_px + sorted_prefix_qx(sm, (int)(best.cnt - ce), m);
  if (p_on) {
    bool hist_valid = false;
    Cut cp;
    if (!locate<VEC>(sm, x, V, m, hist_valid, kMassGE, 0, (double)p * Zk, cp)) return false;
    take_earlier(best, cp);
  }
  __syncthreads();
  return true;
}

// Resolve a row with one count pass and one exact pass. Returns false when the
// exact path must decide instead.
template <bool VEC>
__device__ __noinline__ bool resolve_row_fast(RSmem& sm, const float* __restrict__ x, int V, float m,
                                              int k, float p, float mu, uint32_t kt, bool sampled,
                                              bool ent, bool f32m, Cut& best) {
  const bool k_on = k >= 1 && k < V, p_on = p < 1.0f, mu_on = mu > 0.0f;
  Plan2 pl;
  pl.need_last = 0;
  pl.g_lo = 1;
  pl.g_hi = 0;
  pl.g2_lo = 1;
  pl.g2_hi = 0;
  pl.w_lo = -1;
  pl.b_mu = -1;
  pl.ent = ent ? 1 : 0;
  Pass2 P;

  if (!k_on && !p_on && !mu_on) {  // identity: total mass and the last element only
    if (f32m) {
      FastPass fp;
      fast_pass<VEC, 0>(sm, x, V, m, 0.0f, 0.0f, fp);
      best = Cut{fp.k_last, (long long)V, fp.kept, 0.0};
      return true;
    }
    pl.need_last = 1;
    pass2<VEC>(sm, x, V, m, true, pl, P);
    best = Cut{P.k_last, (long long)V, P.z, P.zx};
    return true;
  }

  count_hist<VEC>(sm, x, V, m, sampled);

  if (k_on) {
    // small k: the prefix of buckets up to the k-th element's fits the buffer
    // and holds every cut that can come before the top-k cut
    int bk;
    long long ce;
    double me;
    pick_bucket(sm, kCount, (long long)k, 0.0, 0, 0.0, bk, ce, me);
    const long long incl = ce + sm.cnt[bk];
    __syncthreads();
    if (incl > SCAP) return resolve_large_k<VEC>(sm, x, V, m, k, p, mu, kt, ent, bk, ce, best);
    pl.g_lo = 0;
    pl.g_hi = bk;
    pass2<VEC>(sm, x, V, m, false, pl, P);
    if (P.overflow) return false;
    const int ng = pack_gathered(sm);
    const int n = compact_gathered(sm, ng, m, 0, bk);
    sort_and_scan(sm, n, m);
    const int jk = min(k, n) - 1;
    Cut ck{sm.cand[jk], (long long)jk + 1, sm.cq[jk]};
    best = ck;
    const double Zk = ck.mass;
    if (p_on) {
      const int jp = first_mass_hit(sm, 0, jk + 1, 0.0, 0.0, kMassGE, (double)p * Zk);
      take_earlier(best, Cut{sm.cand[jp], (long long)jp + 1, sm.cq[jp]});
    }
    if (mu_on) {
      int mine = 0;
      for (int j = threadIdx.x; j < n; j += RT) mine += (uint32_t)(sm.cand[j] >> 32) >= kt ? 1 : 0;
      const int nk = (int)block_sum_l(mine, sm);
      if (nk >= 1 && nk < n) take_earlier(best, Cut{sm.cand[nk - 1], (long long)nk, sm.cq[nk - 1]});
    }
    if (ent) best.qx = sorted_prefix_qx(sm, (int)best.cnt, m);  // the support is a sorted prefix
    __syncthreads();
    return true;
  }

  // top-k off: estimate the top-p crossing bucket from counts x mid-bucket
  // weights and gather it, with a neighbour bucket on each side where the
  // estimate comes within six sigma (plus 1e-5 Zhat for bias) of the target;
  // if the exact masses then put the crossing outside, retry once with the
  // full 3-bucket window. For min-p gather the threshold's bucket and the
  // non-empty bucket before it.
  for (int attempt = 0; attempt < 2; ++attempt) {
    long long before_win = 0, before_mu = 0;
    int lo = 0, hi = -1, bm = -1, bprev = -1;
    bool narrowed = false;
    long long gathered = 0;
    if (p_on) {
      const TopPPlan tp = plan_top_p(sm, p);
      const int bh = tp.b;
      const double t = (double)p * tp.zhat, margin = 6.0 * tp.sigma + 1e-5 * tp.zhat;
      const bool near_lo = attempt > 0 || t - tp.e0 < margin;
      const bool near_hi = attempt > 0 || tp.e0 + tp.eb - t < margin;
      lo = (near_lo && bh > 0) ? bh - 1 : bh;
      hi = (near_hi && bh < NB - 1) ? bh + 1 : bh;
      narrowed = (bh > 0 && lo == bh) || (bh < NB - 1 && hi == bh);
      const long long c_lo = lo < bh ? sm.cnt[lo] : 0, c_hi = hi > bh ? sm.cnt[hi] : 0;
      gathered += c_lo + sm.cnt[bh] + c_hi;
      before_win = tp.cnt_before - c_lo;
      pl.g_lo = lo;
      pl.g_hi = hi;
      pl.w_lo = lo;
    }
    if (mu_on) {
      bm = bin0(key32_value(kt), m);
      bprev = prev_nonempty(sm, bm);
      before_mu = count_range(sm, 0, bm);
      const int a0 = bprev >= 0 ? bprev : bm;
      gathered += sm.cnt[bm] + (a0 < bm ? sm.cnt[a0] : 0);  // buckets between are empty
      pl.g2_lo = a0;
      pl.g2_hi = bm;
      pl.b_mu = bm;
    }
    __syncthreads();
    if (gathered > SCAP) return false;  // keep the per-warp slices far from full
    pass2<VEC>(sm, x, V, m, p_on, pl, P);
    if (P.overflow) return false;
    const int ng = pack_gathered(sm);

    bool have = false;
    if (mu_on) {
      double mass, kmass, kqx;
      long long cnt, kcnt;
      unsigned long long kmin;
      gathered_bucket_stats(sm, ng, m, bm, kt, mass, cnt, kmass, kcnt, kmin, kqx);
      if (kcnt == 0 && bprev >= 0) {
        // nothing of bucket bm is kept: the min-p prefix ends with bucket bprev
        double m2, k2, x2;
        long long c2, kc2;
        gathered_bucket_stats(sm, ng, m, bprev, 0u, m2, c2, k2, kc2, kmin, x2);
      }
      best = Cut{kmin, before_mu + kcnt, P.a_mu + kmass, P.a_mux + kqx};
      have = true;
    }
    if (p_on) {
      const double target = (double)p * P.z;
      // the crossing bucket, from the exact masses of the gathered window
      double wm[3], wqx[3];
      long long wc[3];
      window_stats(sm, ng, m, lo, hi, wm, wc, wqx);
      double before = P.a_p, before_qx = P.a_px;
      long long cbefore = before_win;
      int c = -1;
      for (int w = lo; w <= hi; ++w) {
        if (before < target && target <= before + wm[w - lo]) {
          c = w;
          break;
        }
        before += wm[w - lo];
        before_qx += wqx[w - lo];
        cbefore += wc[w - lo];
      }
      if (c < 0) {  // the crossing lies outside the window
        if (narrowed) continue;
        return false;
      }
      const int n = compact_gathered(sm, ng, m, c, c);
      sort_and_scan(sm, n, m);
      const int jp = first_mass_hit(sm, 0, n, before, 0.0, kMassGE, target);
      const double qx = ent ? before_qx + sorted_prefix_qx(sm, jp + 1, m) : kNoQx;
      const Cut cp{sm.cand[jp], cbefore + jp + 1, before + sm.cq[jp], qx};
      if (have)
        take_earlier(best, cp);
      else
        best = cp;
    }
    __syncthreads();
    return true;
  }
  return false;
}

// Sum of exp(s - m) (s - m) over the support (every element whose composite
// key is >= K, the key of its last element): one pass over the row, for rows
// decided by the exact search, whose histograms carry masses only.
template <bool VEC>
__device__ __noinline__ double support_qx_pass(RSmem& sm, const float* __restrict__ x, int V,
                                               float m, unsigned long long K) {
  double acc = 0.0;
  for_each<VEC>(x, V, [&](float s, int i) {
    if (ckey(s, i) >= K) acc += qmass(sm, s, m) * ((double)s - (double)m);
  });
  return block_sum_d(acc, sm);
}

// ---------------------------------------------------------------- planned path
// The first attempt for every filtered row. A sample of the row (one sweep in
// SAMPLE_EVERY) feeds a count histogram from which the gathered range is
// planned: for top-k the buckets up to the k-th element, for min-p the
// buckets around its threshold (when top-p is on too, only if the sample puts
// the top-p crossing clearly after the min-p prefix). One pass then gathers
// that range and, for min-p, counts and weighs everything before it (float64
// masses, exact counts), and the row is decided from those. A plan the pass
// does not confirm (fewer than k elements gathered, a buffer too small, top-p
// deciding after all), and every row whose top-p crossing decides, goes to
// the fast path above, whose count pass adds the rest of the row to the
// sample's counts, and from there to the exact search: the result never
// rests on the sample, only the amount of work does.

// Count histogram of the planning sample in sm.cnt. Returns the sample size.
template <bool VEC>
__device__ __noinline__ int sample_hist(RSmem& sm, const float* __restrict__ x, int V, float m) {
  for (int i = threadIdx.x; i < NB; i += RT) sm.cnt[i] = 0;
  __syncthreads();
  const int tid = (int)threadIdx.x;
  int n = 0;  // uniform over the block
  if (VEC) {
    // chunks 0, SAMPLE_EVERY, 2 SAMPLE_EVERY, ... and the scalar tail
    const float4* __restrict__ x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    const int nch = n_chunks(V4);
    const int ns = (nch + SAMPLE_EVERY - 1) / SAMPLE_EVERY;
    stream_chunks(sm, x4, V4, ns, [](int j) { return j * SAMPLE_EVERY; }, l2_policy_keep(),
                  [&](auto, const float4& u, int, const float4& w, int, bool vu, bool vw) {
                    if (vu) {
                      atomicAdd(&sm.cnt[bin0(u.x, m)], 1);
                      atomicAdd(&sm.cnt[bin0(u.y, m)], 1);
                      atomicAdd(&sm.cnt[bin0(u.z, m)], 1);
                      atomicAdd(&sm.cnt[bin0(u.w, m)], 1);
                    }
                    if (vw) {
                      atomicAdd(&sm.cnt[bin0(w.x, m)], 1);
                      atomicAdd(&sm.cnt[bin0(w.y, m)], 1);
                      atomicAdd(&sm.cnt[bin0(w.z, m)], 1);
                      atomicAdd(&sm.cnt[bin0(w.w, m)], 1);
                    }
                  });
    for (int j = 0; j < ns; ++j) n += 4 * min(CH_F4, V4 - j * SAMPLE_EVERY * CH_F4);
    for (int i = 4 * V4 + tid; i < V; i += RT) atomicAdd(&sm.cnt[bin0(ld_stream(x + i), m)], 1);
    n += V - 4 * V4;  // the scalar tail (< 4 elements) is always in the sample
  } else {
    for (int base = 0; base < V; base += RT * SAMPLE_EVERY) {
      const int i = base + tid;
      if (i < V) atomicAdd(&sm.cnt[bin0(ld_stream(x + i), m)], 1);
      n += min(RT, V - base);
    }
  }
  __syncthreads();
  return n;
}

// Upper bound of the true count behind an estimate est = scale * (sampled
// count): five standard deviations of the sampling error plus slack.
__device__ __forceinline__ double count_upper(double est, double scale) {
  return est + 5.0 * sqrt(est * (scale - 1.0)) + 16.0;
}

// The smallest bucket whose estimated inclusive count, less five standard
// deviations of its sampling error, reaches `need` (so the prefix of buckets
// up to it holds at least `need` elements with high probability; the exact
// pass checks it). Returns -1 when the prefix's upper bound exceeds `cap` or
// no bucket qualifies.
__device__ __noinline__ int plan_prefix_count(RSmem& sm, long long need, double scale, int cap) {
  constexpr int PER = NB / RT;
  const int base = (int)threadIdx.x * PER;
  long long lc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) lc += sm.cnt[base + i];
  long long tc;
  const long long pc = block_exscan<long long>(lc, sm.red_l, tc);
  int mine = NB;
  {
    long long c = pc;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      c += sm.cnt[base + i];
      const double est = scale * (double)c;
      const double lower = scale > 1.0 ? est - 5.0 * sqrt(est * (scale - 1.0)) : est;
      if (mine == NB && sm.cnt[base + i] > 0 && lower >= (double)need) mine = base + i;
    }
  }
  const int b = block_min_i(mine, sm);
  if (b >= NB - 1) return -1;  // never plan into the clamped far-tail bucket
  if (threadIdx.x == b / PER) {
    long long c = pc;
    for (int i = base; i <= b; ++i) c += sm.cnt[i];
    sm.bl[1] = c;
  }
  __syncthreads();
  const long long incl = sm.bl[1];
  __syncthreads();
  if (count_upper(scale * (double)incl, scale) > (double)cap) return -1;
  return b;
}

// The sample's estimate of the fraction of the row's mass in buckets below b
// (every sampled element weighs its bucket's mid-point mass; the far-tail
// bucket weighs 0).
__device__ __noinline__ double estimated_mass_before(RSmem& sm, int b) {
  const double wmid = sm.bd[3];
  double v[2] = {0.0, 0.0};
  for (int i = threadIdx.x; i < NB - 1; i += RT) {
    const double w = (double)sm.cnt[i] * tab_at(sm.tab, i) * wmid;
    v[0] += w;
    v[1] += i < b ? w : 0.0;
  }
  block_sum_multi<2>(v, sm);
  return v[0] > 0.0 ? v[1] / v[0] : 1.0;
}

// Highest bucket below b holding a sampled element (0 when none does).
__device__ int sampled_before(RSmem& sm, int b) {
  int mine = -1;
  for (int i = threadIdx.x; i < b; i += RT)
    if (sm.cnt[i] > 0) mine = i;
  const int r = (int)block_ext_u<true>((unsigned long long)(mine + 1), sm) - 1;
  return r < 0 ? 0 : r;
}

// Applies f to every key this thread gathered in the pass before (its own
// slots; together the threads visit every gathered key once).
template <typename F>
__device__ __forceinline__ void for_each_gathered(RSmem& sm, F&& f) {
  const int n = min(sm.tcount[threadIdx.x], TCAP);
  for (int j = 0; j < n; ++j) f(sm.cand[j * RT + threadIdx.x]);
}

// Mass, count and smallest key of the gathered elements with key >= kt whose
// bucket lies in [lo, hi] (the min-p range of the planned pass).
__device__ __noinline__ void gathered_kept(RSmem& sm, float m, int lo, int hi, uint32_t kt,
                                           double& mass, long long& cnt, unsigned long long& k_min,
                                           double& qx) {
  double ms = 0.0, c = 0.0, mx = 0.0;
  unsigned long long kmn = ~0ull;
  for_each_gathered(sm, [&](unsigned long long K) {
    const float v = ckey_value(K);
    const int b = bin0(v, m);
    if (b < lo || b > hi || (uint32_t)(K >> 32) < kt) return;
    const double q = qmass(sm, v, m);
    ms += q;
    mx += q * ((double)v - (double)m);
    c += 1.0;
    kmn = K < kmn ? K : kmn;
  });
  double s[3] = {ms, c, mx};
  block_sum_multi<3>(s, sm);
  mass = s[0];
  cnt = (long long)s[1];
  qx = s[2];
  k_min = block_ext_u<false>(kmn, sm);
}

// On return, `sampled` tells whether sm.cnt holds the planning sample's counts
// (the fast path then counts only the rest of the row).
template <bool VEC>
__device__ __noinline__ bool resolve_row_planned(RSmem& sm, const float* __restrict__ x, int V,
                                                 float m, int k, float p, float mu, uint32_t kt,
                                                 bool ent, bool f32m, bool& sampled, Cut& best) {
  const bool k_on = k >= 1 && k < V, p_on = p < 1.0f, mu_on = mu > 0.0f;
  sampled = false;
  if (!k_on && !p_on && !mu_on) return false;  // identity rows: the fast path's single pass
  // top-p alone: no plan uses the sample, and the fast path's count pass
  // streams the whole row faster than the sample's strided chunks
  if (!k_on && !mu_on) return false;
  const int ns = sample_hist<VEC>(sm, x, V, m);
  sampled = true;
  const double scale = (double)V / (double)ns;
  Plan2 pl;
  pl.need_last = 0;
  pl.g_lo = 1;
  pl.g_hi = 0;
  pl.g2_lo = 1;
  pl.g2_hi = 0;
  pl.w_lo = -1;
  pl.b_mu = -1;
  pl.ent = ent ? 1 : 0;
  Pass2 P;

  if (k_on) {
    // every bucket up to the one that holds the k-th element, by the sample
    const int bk = plan_prefix_count(sm, (long long)k, scale, SCAP);
    if (bk < 0) return false;
    pl.g_lo = 0;
    pl.g_hi = bk;
    pass2<VEC>(sm, x, V, m, false, pl, P);
    if (P.overflow) return false;
    const int ng = pack_gathered(sm);
    const int n = compact_gathered(sm, ng, m, 0, bk);
    if (n < k || ng >= SCAP) return false;  // the prefix does not reach the k-th element
    sort_and_scan(sm, n, m);
    const int jk = k - 1;
    Cut ck{sm.cand[jk], (long long)jk + 1, sm.cq[jk]};
    best = ck;
    if (p_on) {
      const int jp = first_mass_hit(sm, 0, jk + 1, 0.0, 0.0, kMassGE, (double)p * ck.mass);
      take_earlier(best, Cut{sm.cand[jp], (long long)jp + 1, sm.cq[jp]});
    }
    if (mu_on) {
      int mine = 0;
      for (int j = threadIdx.x; j < n; j += RT) mine += (uint32_t)(sm.cand[j] >> 32) >= kt ? 1 : 0;
      const int nk = (int)block_sum_l(mine, sm);
      if (nk >= 1 && nk < n) take_earlier(best, Cut{sm.cand[nk - 1], (long long)nk, sm.cq[nk - 1]});
    }
    if (ent) best.qx = sorted_prefix_qx(sm, (int)best.cnt, m);  // the support is a sorted prefix
    __syncthreads();
    return true;
  }

  // top-k off: min-p alone, or min-p with a top-p crossing that the sample
  // puts clearly after the min-p prefix (the exact pass confirms it; rows
  // where top-p decides take the fast path, which counts the rest of the row
  // onto the sample). Everything in buckets below bm = bucket(threshold) is
  // kept and everything above it dropped; the range gathered starts at the
  // last sampled bucket before bm, which is non-empty, so it or bm holds the
  // last kept element.
  if (!mu_on) return false;
  const int bm = bin0(key32_value(kt), m);
  const int g2lo = sampled_before(sm, bm);
  if (p_on && estimated_mass_before(sm, bm + 1) > (double)p - 0.05) return false;
  if (f32m) {
    // kept iff s >= thr; the last kept element lies in buckets [g2lo, bm],
    // so the kept elements with s <= hv (one bucket of slack) are gathered
    const int glo = g2lo > 0 ? g2lo - 1 : 0;
    const double est = scale * (double)count_range(sm, glo, bm + 1);
    if (count_upper(est, scale) > 0.75 * CAP) return false;
    const float hv = m - (float)(g2lo - 1) * (1.0f / BIN_SCALE);
    FastPass fp;
    fast_pass<VEC, 1>(sm, x, V, m, key32_value(kt), hv, fp);
    if (fp.overflow) return false;
    const int ng = pack_gathered(sm);
    if (ng == 0 || ng >= SCAP) return false;
    const unsigned long long* g = packed(sm);
    unsigned long long kmn = ~0ull;
    for (int i = threadIdx.x; i < ng; i += RT) kmn = g[i] < kmn ? g[i] : kmn;
    const unsigned long long kmin = block_ext_u<false>(kmn, sm);
    // certificate against the bounds of the fp32 masses
    if (p_on && !(fp.kept * (1.0 + MASS_EPS) < (double)p * (fp.kept + fp.rest) * (1.0 - MASS_EPS)))
      return false;
    best = Cut{kmin, fp.cnt, fp.kept, 0.0};
    return true;
  }
  const double est = scale * (double)count_range(sm, g2lo, bm + 1);
  if (count_upper(est, scale) > 0.75 * CAP) return false;  // keep the warp slices far from full
  MuPass mp;
  mu_pass<VEC>(sm, x, V, m, g2lo, bm, ent, mp);
  if (mp.overflow) return false;
  double km, kx;
  long long kc;
  unsigned long long kmin;
  gathered_kept(sm, m, g2lo, bm, kt, km, kc, kmin, kx);
  if (kc == 0) return false;
  const Cut cm{kmin, mp.cnt + kc, mp.mass + km, mp.qx + kx};
  // With top-p on, the min-p prefix decides when its mass stays below p Z;
  // Z >= (its mass) + the lower bound of the dropped elements' mass
  // certifies it (otherwise the fast path decides).
  if (p_on && !(cm.mass < (double)p * (cm.mass + mp.rest_lower))) return false;
  best = cm;
  return true;
}

template <bool VEC>
__global__ void __launch_bounds__(RT, 1) resolve_kernel(const ResolveArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  RSmem& sm = *reinterpret_cast<RSmem*>(smem_raw);
  const int V = a.V;
  init_exp_tab(sm.tab, threadIdx.x, RT);
  sm.ring_q[threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    sm.bd[3] = exp(-1.0 / 256.0);  // mid-bucket weight factor
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_u32(&sm.full_bar[s]), 1);
      sm.ring_done[s] = 0;
    }
    sm.abort_flag = 0;
    sm.err = &a.hdr->err;
    fence_barrier_init();
  }
  __syncthreads();

  // A row's metadata and the first two of its partial maxima per thread are
  // loaded one row ahead, so their latency overlaps the previous row's work.
  struct Ahead {
    float part0, part1, p, mu;
    int flags, k;
  };
  auto load_ahead = [&](int row, Ahead& h) {
    h.part0 = h.part1 = -INFINITY;
    h.flags = 0;
    h.k = 0;
    h.p = 1.0f;
    h.mu = 0.0f;
    if (row >= a.rows) return;
    if (a.max_part) {
      const float* mp = a.max_part + (size_t)row * (size_t)a.n_parts;
      const int i0 = threadIdx.x, i1 = threadIdx.x + RT;
      if (i0 < a.n_parts) h.part0 = mp[i0];
      if (i1 < a.n_parts) h.part1 = mp[i1];
    }
    if (a.row_flags) h.flags = a.row_flags[row];
    h.k = a.top_k[row];
    h.p = a.top_p[row];
    h.mu = a.min_p[row];
  };
  // Rows are handed out dynamically (their costs differ several-fold by
  // metadata, and a static split leaves the launch waiting on its slowest
  // CTA): the first gridDim.x rows go one per CTA, the rest in the order CTAs
  // claim them from the header's counter. A CTA claims the row after next at
  // the start of each row, so the atomic's latency overlaps the row's work and
  // the next row's metadata can be loaded one row ahead.
  unsigned long long claim = 0;
  if (threadIdx.x == 0) sm.row_next = (int)gridDim.x + (int)atomicAdd(&a.hdr->next_row, 1ull);
  __syncthreads();
  int nxt = sm.row_next;
  auto advance = [&]() {
    if (threadIdx.x == 0) sm.row_next = (int)claim;
    __syncthreads();
    const int r2 = nxt;
    nxt = sm.row_next;
    return r2;
  };
  Ahead ahead;
  load_ahead(blockIdx.x, ahead);

  for (int r = blockIdx.x; r < a.rows; r = advance()) {
    const Ahead cur = ahead;
    if (threadIdx.x == 0) {
      const unsigned long long c = atomicAdd(&a.hdr->next_row, 1ull) + gridDim.x;
      claim = c < (unsigned long long)INT_MAX ? c : (unsigned long long)INT_MAX;
    }
    load_ahead(nxt, ahead);
    const float* __restrict__ x = a.S + (size_t)r * (size_t)a.ld;
    const bool invalid = (cur.flags & STS_ROW_INVALID) != 0;
    if (invalid) {
      if (threadIdx.x == 0) {
        const float nan = __int_as_float(0x7fc00000);
        if (a.logprob) a.logprob[r] = nan;
        if (a.entropy) a.entropy[r] = nan;
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
      __syncthreads();
      continue;
    }

    // unfiltered row max: from the projection's per-tile maxima when present
    float lm = -INFINITY;
    if (a.max_part) {
      const float* mp = a.max_part + (size_t)r * (size_t)a.n_parts;
      lm = fmaxf(cur.part0, cur.part1);
      for (int i = threadIdx.x + 2 * RT; i < a.n_parts; i += RT) lm = fmaxf(lm, mp[i]);
    } else {
      lm = row_max_pass<VEC>(x, V);
    }
    const float m = block_max_f(lm, sm);
    const double md = (double)m;

    const int k = cur.k;
    const float p = cur.p;
    const float mu = cur.mu;
    const bool k_on = k >= 1 && k < V;
    const bool p_on = p < 1.0f;
    const bool mu_on = mu > 0.0f;

    uint32_t kt = 0;
    if (mu_on) {
      if (threadIdx.x == 0) sm.bi[0] = (int)min_p_threshold_key(m, mu);
      __syncthreads();
      kt = (uint32_t)sm.bi[0];
      __syncthreads();
    }

    Cut best;
    bool hist_valid = false;
    // planned pass first; the fast path and the exact search decide the rows
    // whose plan does not hold (identity rows go straight to the fast path's
    // single pass)
    int path = (k_on || p_on || mu_on) ? kPathPlanned : kPathIdentity;
    bool sampled = false;
    const bool ent = a.entropy != nullptr;
    // fp32 masses where no mass comparison decides the output
    const bool f32m = !ent && a.mode != kModeSample;
    bool ok = resolve_row_planned<VEC>(sm, x, V, m, k, p, mu, kt, ent, f32m, sampled, best);
    if (!ok) {
      if (path == kPathPlanned) path = kPathFast;
      ok = resolve_row_fast<VEC>(sm, x, V, m, k, p, mu, kt, sampled, ent, f32m, best);
    }
    if (!ok) {
      path = kPathExact;
      ok = resolve_row_exact<VEC>(sm, x, V, m, k, p, mu, kt, hist_valid, best);
    }
    if (threadIdx.x == 0) atomicAdd(&a.hdr->path_rows[path], 1ull);
    __syncthreads();
    if (sm.abort_flag) break;  // a bounded wait gave up: STS_ERR_TIMEOUT is recorded

    if (!ok) {  // a bound of the exact search was exceeded: the row fails like an invalid one
      if (threadIdx.x == 0) {
        atomicCAS(&a.hdr->err, 0, (int)STS_ERR_OVERFLOW);
        const float nan = __int_as_float(0x7fc00000);
        if (a.logprob) a.logprob[r] = nan;
        if (a.entropy) a.entropy[r] = nan;
        if (a.row_max) a.row_max[r] = nan;
        if (a.lse_support) a.lse_support[r] = nan;
        if (a.cut_logit) a.cut_logit[r] = nan;
        if (a.cut_id) a.cut_id[r] = -1;
        if (a.sampled) a.sampled[r] = -1;
        if (a.support_size) a.support_size[r] = 0;
        if (a.flags_out) a.flags_out[r] = STS_ROW_INVALID;
      }
      if (a.mask)
        for (int i = threadIdx.x; i < V; i += RT) a.mask[(size_t)r * V + i] = 0;
      __syncthreads();
      continue;
    }

    const double lse = md + log(best.mass);
    if (ent) {
      // entropy of the renormalised support: ln Z_S - sum_S q (s - m) / Z_S,
      // q = exp(s - m); the sum comes from the deciding path, else one pass
      const double qx = isnan(best.qx) ? support_qx_pass<VEC>(sm, x, V, m, best.K) : best.qx;
      if (threadIdx.x == 0) a.entropy[r] = (float)fmax(log(best.mass) - qx / best.mass, 0.0);
    }
    if (a.mode == kModeSample) {
      Cut cs;
      const double tgt = a.u[r] * best.mass;
      const bool ok2 = locate<VEC>(sm, x, V, m, hist_valid, kMassGT, 0, tgt, cs);
      if (!ok2 || cs.K < best.K) cs = best;
      if (threadIdx.x == 0) a.sampled[r] = ckey_id(cs.K);
    }
    if (threadIdx.x == 0) {
      if (a.support_size) a.support_size[r] = (int32_t)best.cnt;
      if (a.cut_logit) a.cut_logit[r] = ckey_value(best.K);
      if (a.cut_id) a.cut_id[r] = ckey_id(best.K);
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

// Evaluates the resolver's mass function exp(s - m) and the library exp on
// the same inputs (test hook for the table-driven exponential).
__global__ void mass_probe_kernel(const float* s, float m, double* mine, double* lib, int64_t n) {
  __shared__ ExpTab tab;
  init_exp_tab(tab, threadIdx.x, blockDim.x);
  __syncthreads();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = s[i];
    mine[i] = qmass_b(tab, v, (double)m, bin0(v, m));
    lib[i] = exp((double)v - (double)m);
  }
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

static_assert(sizeof(RSmem) <= 227 * 1024, "the resolver CTA fits one SM's shared memory");
static_assert(NB == SCAP, "bucket masses and the candidates' scan share storage");
static_assert(SCAP <= CAP && SCAP == 8 * RT, "a sorted run fits the candidate buffer");

size_t resolve_smem_bytes() { return sizeof(RSmem); }

cudaError_t launch_mass_probe(const float* s, float m, double* mine, double* lib, int64_t n,
                              cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int blocks = (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  mass_probe_kernel<<<blocks, 256, 0, stream>>>(s, m, mine, lib, n);
  return cudaGetLastError();
}

cudaError_t launch_resolve(const ResolveArgs& a, int num_sms, cudaStream_t stream) {
  const size_t smem = sizeof(RSmem);
  const bool vec = (a.ld % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.S) & 15u) == 0);
  auto kern = vec ? resolve_kernel<true> : resolve_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = a.rows < num_sms ? a.rows : num_sms;
  if (grid <= 0) return cudaSuccess;
  e = cudaMemsetAsync(&a.hdr->next_row, 0, sizeof(a.hdr->next_row), stream);  // the row counter
  if (e != cudaSuccess) return e;
  kern<<<grid, RT, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace sts
