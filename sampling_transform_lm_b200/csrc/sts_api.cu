// C ABI of the scoring core: argument checks, workspace carving, tensor maps
// and the launch sequence of the forward / backward / sample / filter paths.
//
//   forward   validate rows -> per row chunk: [tcgen05 GEMM, epilogue s = z/tau
//             -> fp32 chunk of scaled logits] -> [exact per-row resolver]
//   backward  per vocabulary chunk: [recompute GEMM with the dz epilogue ->
//             bf16 dZ chunk] -> [dW slice GEMM, written once] -> [dH GEMM,
//             stored for the first chunk, TMA reduce-added after]
//
// ("Consolidate sampling-transform scoring on one shared chunked core", xorl
// PR 74: "What this PR does", item 2, chunked core with a recompute VJP; the
// "Self-review pass" single-pass vocabulary-chunked backward with write-once
// weight-gradient slices.)
#include <algorithm>
#include <cstddef>
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "gemm_sm100.cuh"
#include "sts_internal.h"

namespace sts {
namespace {

// 111 x 256 columns: for T and d multiples of 512 the dz GEMM (ceil(T/128) x
// Vc/256 tiles) and the dW GEMM (ceil(d/128) x Vc/256 tiles) then fill whole
// waves of a 148-SM part (111 = 3 x 37), and a chunk this wide needs few launches
// (six at V = 152,064; the bf16 dZ buffer is T x Vc x 2 bytes, 0.93 GB at T = 16384).
constexpr int64_t kDefaultVocabChunk = 28416;
constexpr size_t kDefaultChunkBytes = size_t(4) << 30;  // forward logits chunk budget

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool map2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
           uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  std::memset(m, 0, sizeof(*m));
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 operand, K contiguous: [rows][K] with row stride ld elements.
bool map_kmajor(CUtensorMap* m, const void* p, int64_t K, int64_t rows, int64_t ld, uint32_t box_rows) {
  return map2d(m, p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)rows, (uint64_t)ld * 2,
               64, box_rows);
}

// bf16 operand, MN contiguous: [K][MN] with row stride ld elements.
bool map_mnmajor(CUtensorMap* m, const void* p, int64_t MN, int64_t K, int64_t ld) {
  return map2d(m, p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)MN, (uint64_t)K, (uint64_t)ld * 2,
               64, 64);
}

bool map_out_f32(CUtensorMap* m, const void* p, int64_t cols, int64_t rows, int64_t ld) {
  return map2d(m, p, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (uint64_t)cols, (uint64_t)rows,
               (uint64_t)ld * 4, 32, 32);
}

bool map_out_bf16(CUtensorMap* m, const void* p, int64_t cols, int64_t rows, int64_t ld) {
  return map2d(m, p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)cols, (uint64_t)rows,
               (uint64_t)ld * 2, 64, 32);
}

template <bool AMN, bool BMN, int EPI>
cudaError_t run_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                     const GemmParams& p, int sms, cudaStream_t st) {
  auto kern = gemm_kernel<AMN, BMN, EPI>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMM_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long tiles =
      (long long)((p.M + GEMM_BM - 1) / GEMM_BM) * (long long)((p.N + GEMM_BN - 1) / GEMM_BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, st>>>(a, b, c, p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- launch accounting

std::atomic<long long> g_launches[STS_KERNEL_KINDS];

struct TimingState {
  std::mutex mu;
  bool on = false;
  struct Rec {
    int kind;
    cudaEvent_t beg, end;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  cudaEvent_t get() {
    if (used < pool.size()) return pool[used++];
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    pool.push_back(e);
    ++used;
    return e;
  }
};
TimingState g_timing;

// Brackets one kernel launch: counts it and, when timing is on, records the
// two events around it on the launch stream.
template <typename F>
cudaError_t timed_launch(int kind, cudaStream_t st, F&& launch) {
  g_launches[kind].fetch_add(1, std::memory_order_relaxed);
  cudaEvent_t b = nullptr, e = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_timing.mu);
    if (g_timing.on) {
      b = g_timing.get();
      e = g_timing.get();
    }
  }
  if (b) cudaEventRecord(b, st);
  const cudaError_t err = launch();
  if (e) {
    cudaEventRecord(e, st);
    std::lock_guard<std::mutex> lock(g_timing.mu);
    g_timing.recs.push_back({kind, b, e});
  }
  return err;
}

struct DeviceInfo {
  bool ok;
  int sms;
};

sts_status device_info(DeviceInfo& info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return STS_ERR_CUDA;
  static DeviceInfo cache[64];
  static bool have[64];
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return STS_ERR_CUDA;
  if (!have[dev]) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return STS_ERR_CUDA;
    cache[dev].ok = (prop.major == 10 && prop.minor == 0);
    cache[dev].sms = prop.multiProcessorCount;
    have[dev] = true;
  }
  info = cache[dev];
  return info.ok ? STS_OK : STS_ERR_UNSUPPORTED_ARCH;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- shapes

bool shape_ok(const sts_shape* s) {
  if (!s) return false;
  if (s->T < 1 || s->T > (int64_t(1) << 31) - 1) return false;
  if (s->V < 1 || s->V > (int64_t(1) << 31) - 1) return false;
  if (s->d < 8 || (s->d % 8) != 0 || s->d > (int64_t(1) << 20)) return false;
  if (s->vocab_chunk < 0 || (s->vocab_chunk % 256) != 0) return false;
  if (s->row_chunk < 0 || (s->row_chunk % 128) != 0) return false;
  return true;
}

int64_t logits_ld(const sts_shape* s) { return (s->V + 3) / 4 * 4; }

int64_t row_chunk(const sts_shape* s) {
  const int64_t Tpad = (s->T + 127) / 128 * 128;
  int64_t rc = s->row_chunk;
  if (rc == 0) {
    const int64_t per_row = logits_ld(s) * 4;
    rc = (int64_t)(kDefaultChunkBytes / (size_t)per_row) / 128 * 128;
    if (rc < 128) rc = 128;
  }
  return rc < Tpad ? rc : Tpad;
}

int64_t vocab_chunk(const sts_shape* s) {
  const int64_t Vpad = (s->V + 255) / 256 * 256;
  const int64_t vc = s->vocab_chunk ? s->vocab_chunk : kDefaultVocabChunk;
  return vc < Vpad ? vc : Vpad;
}

int64_t n_parts(const sts_shape* s) { return (s->V + GEMM_BN - 1) / GEMM_BN; }

struct FwdLayout {
  size_t flags_off, max_off, logits_off, total;
};

FwdLayout fwd_layout(const sts_shape* s) {
  FwdLayout L;
  L.flags_off = sizeof(WsHeader);
  L.max_off = align_up(L.flags_off + (size_t)s->T * 4, kAlign);
  L.logits_off = align_up(L.max_off + (size_t)row_chunk(s) * (size_t)n_parts(s) * 4, kAlign);
  L.total = align_up(L.logits_off + (size_t)row_chunk(s) * (size_t)logits_ld(s) * 4, kAlign);
  return L;
}

struct BwdLayout {
  size_t dz_off, ht_off, total;
  int64_t ht_ld;  // row stride of H^T (elements): T rounded up to 8 (16-byte TMA rows)
};

BwdLayout bwd_layout(const sts_shape* s) {
  BwdLayout L;
  L.dz_off = kAlign;
  L.ht_ld = (s->T + 7) / 8 * 8;
  L.ht_off = align_up(L.dz_off + (size_t)s->T * (size_t)vocab_chunk(s) * 2, kAlign);
  L.total = align_up(L.ht_off + (size_t)s->d * (size_t)L.ht_ld * 2, kAlign);
  return L;
}

// HT[j][t] = H[t][j] (bf16), 32 x 32 tiles through shared memory.
__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ H, int64_t T, int64_t d,
                                      uint16_t* __restrict__ HT, int64_t ld) {
  __shared__ uint16_t tile[32][33];
  const int64_t t0 = (int64_t)blockIdx.y * 32, j0 = (int64_t)blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t t = t0 + i, j = j0 + threadIdx.x;
    if (t < T && j < d) tile[i][threadIdx.x] = H[t * d + j];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t j = j0 + i, t = t0 + threadIdx.x;
    if (j < d && t < T) HT[j * ld + t] = tile[threadIdx.x][i];
  }
}

size_t filter_bytes(const sts_shape* s) { return align_up(sizeof(WsHeader) + (size_t)s->T * 4, kAlign); }

sts_status check_rows(const sts_shape* s, const sts_rows* r, bool need_target) {
  if (!r) return STS_ERR_NULL;
  if (r->len != s->T) return STS_ERR_SHAPE;
  if (!r->temperature || !r->top_k || !r->top_p || !r->min_p) return STS_ERR_NULL;
  if (need_target && !r->target) return STS_ERR_NULL;
  return STS_OK;
}

sts_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return STS_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return STS_ERR_WORKSPACE;
  if (ws_bytes < need) return STS_ERR_WORKSPACE;
  return STS_OK;
}

sts_status reset_header(void* ws, cudaStream_t st) {
  WsHeader* h = static_cast<WsHeader*>(ws);
  if (cudaMemsetAsync(&h->bad_row_code, 0xFF, sizeof(h->bad_row_code), st) != cudaSuccess)
    return STS_ERR_CUDA;
  // err, its padding and the path counters are contiguous
  static_assert(offsetof(WsHeader, path_rows) == offsetof(WsHeader, err) + 8, "header layout");
  if (cudaMemsetAsync(&h->err, 0, 8 + sizeof(h->path_rows), st) != cudaSuccess) return STS_ERR_CUDA;
  return STS_OK;
}

#define STS_TRY(x)                     \
  do {                                 \
    const sts_status _s = (x);         \
    if (_s != STS_OK) return _s;       \
  } while (0)

#define STS_CUDA(x)                                    \
  do {                                                 \
    if ((x) != cudaSuccess) return STS_ERR_CUDA;       \
  } while (0)

// Forward-style pass shared by sts_forward and sts_sample.
sts_status forward_impl(const sts_shape* shape, const void* H, const void* W, const sts_rows* rows,
                        float* logprob, float* entropy, const sts_saved* saved, const double* u,
                        int64_t* sampled, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!shape_ok(shape)) return STS_ERR_SHAPE;
  if (!H || !W) return STS_ERR_NULL;
  const bool fwd = (sampled == nullptr);
  STS_TRY(check_rows(shape, rows, fwd));
  if (fwd) {
    if (!logprob || !saved || !saved->row_max || !saved->lse_support || !saved->cut_logit ||
        !saved->cut_id || !saved->support_size || !saved->flags)
      return STS_ERR_NULL;
  } else if (!u) {
    return STS_ERR_NULL;
  }
  if (!aligned16(H) || !aligned16(W)) return STS_ERR_SHAPE;
  const FwdLayout L = fwd_layout(shape);
  STS_TRY(check_ws(ws, ws_bytes, L.total));
  DeviceInfo dev;
  STS_TRY(device_info(dev));

  const int64_t T = shape->T, V = shape->V, d = shape->d;
  const int64_t ld = logits_ld(shape), rc_max = row_chunk(shape);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
  int32_t* flags = fwd ? saved->flags : reinterpret_cast<int32_t*>(wsb + L.flags_off);
  float* S = reinterpret_cast<float*>(wsb + L.logits_off);
  float* max_part = reinterpret_cast<float*>(wsb + L.max_off);
  const int np = (int)n_parts(shape);

  STS_TRY(reset_header(ws, st));
  STS_CUDA(timed_launch(STS_KERNEL_VALIDATE, st, [&] {
    launch_validate(rows->target, rows->temperature, rows->top_p, rows->min_p, T, V, flags, hdr, fwd, st);
    return cudaGetLastError();
  }));

  CUtensorMap ma, mb;
  if (!map_kmajor(&ma, H, d, T, d, GEMM_BM) || !map_kmajor(&mb, W, d, V, d, GEMM_BN))
    return STS_ERR_CUDA;

  for (int64_t t0 = 0; t0 < T; t0 += rc_max) {
    const int64_t rc = (T - t0) < rc_max ? (T - t0) : rc_max;
    CUtensorMap mc;
    if (!map_out_f32(&mc, S, V, rc, ld)) return STS_ERR_CUDA;
    GemmParams p{};
    p.M = (int)rc;
    p.N = (int)V;
    p.K = (int)d;
    p.a_mn0 = (int)t0;
    p.tau = rows->temperature + t0;
    p.err = &hdr->err;
    p.max_part = max_part;
    p.max_ld = np;
    STS_CUDA(timed_launch(STS_KERNEL_LOGITS_GEMM, st, [&] {
      return run_gemm<false, false, kEpiLogits>(ma, mb, mc, p, dev.sms, st);
    }));

    ResolveArgs a{};
    a.S = S;
    a.ld = ld;
    a.rows = (int)rc;
    a.V = (int)V;
    a.mode = fwd ? kModeForward : kModeSample;
    a.target = fwd ? rows->target + t0 : nullptr;
    a.top_k = rows->top_k + t0;
    a.top_p = rows->top_p + t0;
    a.min_p = rows->min_p + t0;
    a.u = fwd ? nullptr : u + t0;
    a.row_flags = flags + t0;
    a.flags_out = flags + t0;
    if (fwd) {
      a.logprob = logprob + t0;
      a.entropy = entropy ? entropy + t0 : nullptr;
      a.row_max = saved->row_max + t0;
      a.lse_support = saved->lse_support + t0;
      a.cut_logit = saved->cut_logit + t0;
      a.cut_id = saved->cut_id + t0;
      a.support_size = saved->support_size + t0;
    } else {
      a.sampled = sampled + t0;
    }
    a.hdr = hdr;
    a.row_base = t0;
    a.max_part = max_part;
    a.n_parts = np;
    STS_CUDA(timed_launch(STS_KERNEL_RESOLVE, st, [&] { return launch_resolve(a, dev.sms, st); }));
  }
  return STS_OK;
}

// The backward over W's vocabulary rows [0, V); their ids in the full
// vocabulary start at vocab_offset (0 unless W is one rank's vocabulary shard).
sts_status backward_impl(const sts_shape* shape, const void* H, const void* W,
                         const sts_rows* rows, const sts_saved* saved, const float* grad,
                         float* dH, float* dW, int accumulate_dW, void* ws, size_t ws_bytes,
                         sts_stream_t stream, sts_slice_fn on_dw_slice, void* user, int comm_sms,
                         int64_t vocab_offset) {
  if (!shape_ok(shape)) return STS_ERR_SHAPE;
  if (comm_sms < 0) return STS_ERR_SHAPE;
  if (vocab_offset < 0 || vocab_offset + shape->V > (int64_t(1) << 31) - 1) return STS_ERR_SHAPE;
  if (!H || !W || !grad || !dH || !dW) return STS_ERR_NULL;
  STS_TRY(check_rows(shape, rows, true));
  if (!saved || !saved->lse_support || !saved->cut_logit || !saved->cut_id || !saved->flags)
    return STS_ERR_NULL;
  if (!aligned16(H) || !aligned16(W) || !aligned16(dH) || !aligned16(dW)) return STS_ERR_SHAPE;
  const BwdLayout L = bwd_layout(shape);
  STS_TRY(check_ws(ws, ws_bytes, L.total));
  DeviceInfo dev;
  STS_TRY(device_info(dev));
  if (comm_sms >= dev.sms) return STS_ERR_SHAPE;
  dev.sms -= comm_sms;  // persistent GEMMs leave these SMs to the caller's exchange kernels
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  const int64_t T = shape->T, V = shape->V, d = shape->d, Vc = vocab_chunk(shape);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
  void* dZ = wsb + L.dz_off;
  STS_TRY(reset_header(ws, st));

  // dW is formed as (dW)^T = H^T . dZ, so that its 128-row operand is
  // K-major (H^T, transposed once per call) and only the 256-wide one (dZ)
  // is read MN-major; the epilogue writes the product transposed, i.e. dW
  void* HT = wsb + L.ht_off;
  CUtensorMap m_h_k, m_w_k, m_ht_k, m_w_mn, m_dw, m_dh;
  if (!map_kmajor(&m_h_k, H, d, T, d, GEMM_BM) || !map_kmajor(&m_w_k, W, d, V, d, GEMM_BN) ||
      !map_kmajor(&m_ht_k, HT, T, d, L.ht_ld, GEMM_BM) || !map_mnmajor(&m_w_mn, W, d, V, d) ||
      !map_out_f32(&m_dw, dW, d, V, d) || !map_out_f32(&m_dh, dH, d, T, d))
    return STS_ERR_CUDA;
  STS_CUDA(timed_launch(STS_KERNEL_DW_GEMM, st, [&] {
    const dim3 grid((unsigned)((d + 31) / 32), (unsigned)((T + 31) / 32));
    transpose_bf16_kernel<<<grid, dim3(32, 8), 0, st>>>(static_cast<const uint16_t*>(H), T, d,
                                                        static_cast<uint16_t*>(HT), L.ht_ld);
    return cudaGetLastError();
  }));

  for (int64_t v0 = 0; v0 < V; v0 += Vc) {
    const int64_t w = (V - v0) < Vc ? (V - v0) : Vc;
    CUtensorMap m_dz_out, m_dz_k, m_dz_mn;
    if (!map_out_bf16(&m_dz_out, dZ, w, T, Vc) || !map_kmajor(&m_dz_k, dZ, w, T, Vc, GEMM_BM) ||
        !map_mnmajor(&m_dz_mn, dZ, w, T, Vc))
      return STS_ERR_CUDA;

    // 1. recompute the chunk's logits and form dZ in the epilogue
    GemmParams p{};
    p.M = (int)T;
    p.N = (int)w;
    p.K = (int)d;
    p.b_mn0 = (int)v0;
    p.tau = rows->temperature;
    p.lse = saved->lse_support;
    p.cut_logit = saved->cut_logit;
    p.cut_id = saved->cut_id;
    p.target = rows->target;
    p.grad = grad;
    p.flags = saved->flags;
    p.col_base = (int)(vocab_offset + v0);
    p.err = &hdr->err;
    STS_CUDA(timed_launch(STS_KERNEL_DZ_GEMM, st, [&] {
      return run_gemm<false, false, kEpiDZ>(m_h_k, m_w_k, m_dz_out, p, dev.sms, st);
    }));

    // 2. dW[v0:v0+w] = (H^T . dZ)^T: H^T K-major, dZ MN-major, the tile
    //    stored transposed; written once
    GemmParams q{};
    q.M = (int)d;
    q.N = (int)w;
    q.K = (int)T;
    q.c_y0 = (int)v0;
    q.err = &hdr->err;
    STS_CUDA(timed_launch(STS_KERNEL_DW_GEMM, st, [&] {
      return accumulate_dW
                 ? run_gemm<false, true, kEpiReduceF32T>(m_ht_k, m_dz_mn, m_dw, q, dev.sms, st)
                 : run_gemm<false, true, kEpiStoreF32T>(m_ht_k, m_dz_mn, m_dw, q, dev.sms, st);
    }));
    // the slice is final once this GEMM completes on `st`: hand it out before
    // enqueuing the work that follows, so its exchange overlaps that work
    if (on_dw_slice) on_dw_slice(user, v0, w, dW + (size_t)v0 * (size_t)d, stream);

    // 3. dH (+)= dZ . W[v0:v0+w] (W read MN-major)
    GemmParams r{};
    r.M = (int)T;
    r.N = (int)d;
    r.K = (int)w;
    r.b_k0 = (int)v0;
    r.err = &hdr->err;
    STS_CUDA(timed_launch(STS_KERNEL_DH_GEMM, st, [&] {
      return v0 == 0 ? run_gemm<false, true, kEpiStoreF32>(m_dz_k, m_w_mn, m_dh, r, dev.sms, st)
                     : run_gemm<false, true, kEpiReduceF32>(m_dz_k, m_w_mn, m_dh, r, dev.sms, st);
    }));
  }
  return STS_OK;
}

}  // namespace
}  // namespace sts

using namespace sts;

extern "C" {

int sts_abi_version(void) { return STS_ABI_VERSION; }

const char* sts_status_string(sts_status s) {
  switch (s) {
    case STS_OK: return "ok";
    case STS_ERR_NULL: return "a required pointer is NULL";
    case STS_ERR_SHAPE: return "invalid shape, alignment or metadata length";
    case STS_ERR_DTYPE: return "operands must be bf16 (fp8 heads are not supported)";
    case STS_ERR_TEMPERATURE: return "temperature must be finite and > 0";
    case STS_ERR_TOP_K: return "invalid top_k";
    case STS_ERR_TOP_P: return "top_p must be in (0, 1]";
    case STS_ERR_MIN_P: return "min_p must be in [0, 1]";
    case STS_ERR_TARGET: return "target must be in [0, V)";
    case STS_ERR_WORKSPACE: return "workspace missing, misaligned (256 B) or too small";
    case STS_ERR_OVERFLOW: return "an internal bound was exceeded";
    case STS_ERR_TIMEOUT: return "a bounded device wait gave up";
    case STS_ERR_CUDA: return "a CUDA call failed";
    case STS_ERR_UNSUPPORTED_ARCH: return "device is not sm_100 (B200)";
  }
  return "unknown status";
}

int64_t sts_vocab_chunk(const sts_shape* shape) {
  if (!shape_ok(shape)) return -1;
  return vocab_chunk(shape);
}

size_t sts_workspace_bytes(const sts_shape* shape, int pass) {
  if (!shape_ok(shape)) return 0;
  switch (pass) {
    case 0: return fwd_layout(shape).total;
    case 1: return bwd_layout(shape).total;
    case 2: return filter_bytes(shape);
  }
  return 0;
}

sts_status sts_forward(const sts_shape* shape, const void* H, const void* W, const sts_rows* rows,
                       float* logprob, float* entropy, const sts_saved* saved, void* ws,
                       size_t ws_bytes, sts_stream_t stream) {
  return forward_impl(shape, H, W, rows, logprob, entropy, saved, nullptr, nullptr, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

sts_status sts_sample(const sts_shape* shape, const void* H, const void* W, const sts_rows* rows,
                      const double* u, int64_t* sampled, void* ws, size_t ws_bytes,
                      sts_stream_t stream) {
  if (!sampled) return STS_ERR_NULL;
  return forward_impl(shape, H, W, rows, nullptr, nullptr, nullptr, u, sampled, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

sts_status sts_backward_sliced(const sts_shape* shape, const void* H, const void* W,
                               const sts_rows* rows, const sts_saved* saved, const float* grad,
                               float* dH, float* dW, int accumulate_dW, void* ws, size_t ws_bytes,
                               sts_stream_t stream, sts_slice_fn on_dw_slice, void* user,
                               int comm_sms) {
  return backward_impl(shape, H, W, rows, saved, grad, dH, dW, accumulate_dW, ws, ws_bytes, stream,
                       on_dw_slice, user, comm_sms, 0);
}

sts_status sts_backward(const sts_shape* shape, const void* H, const void* W, const sts_rows* rows,
                        const sts_saved* saved, const float* grad, float* dH, float* dW,
                        int accumulate_dW, void* ws, size_t ws_bytes, sts_stream_t stream) {
  return backward_impl(shape, H, W, rows, saved, grad, dH, dW, accumulate_dW, ws, ws_bytes, stream,
                       nullptr, nullptr, 0, 0);
}

sts_status sts_backward_shard(const sts_shape* shape, const void* H, const void* W_shard,
                              const sts_rows* rows, const sts_saved* saved, const float* grad,
                              float* dH_partial, float* dW_shard, int accumulate_dW,
                              int64_t vocab_offset, void* ws, size_t ws_bytes, sts_stream_t stream) {
  return backward_impl(shape, H, W_shard, rows, saved, grad, dH_partial, dW_shard, accumulate_dW, ws,
                       ws_bytes, stream, nullptr, nullptr, 0, vocab_offset);
}

sts_status sts_resolve_logits(const sts_shape* shape, const float* S, int64_t ld,
                              const sts_rows* rows, float* logprob, float* entropy,
                              const sts_saved* saved, void* ws, size_t ws_bytes,
                              sts_stream_t stream) {
  if (!shape_ok(shape)) return STS_ERR_SHAPE;
  if (!S || !logprob) return STS_ERR_NULL;
  if (ld < shape->V) return STS_ERR_SHAPE;
  STS_TRY(check_rows(shape, rows, true));
  if (!saved || !saved->row_max || !saved->lse_support || !saved->cut_logit || !saved->cut_id ||
      !saved->support_size || !saved->flags)
    return STS_ERR_NULL;
  STS_TRY(check_ws(ws, ws_bytes, filter_bytes(shape)));
  DeviceInfo dev;
  STS_TRY(device_info(dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  int32_t* flags = saved->flags;
  STS_TRY(reset_header(ws, st));
  STS_CUDA(timed_launch(STS_KERNEL_VALIDATE, st, [&] {
    launch_validate(rows->target, rows->temperature, rows->top_p, rows->min_p, shape->T, shape->V,
                    flags, hdr, true, st);
    return cudaGetLastError();
  }));
  ResolveArgs a{};
  a.S = S;
  a.ld = ld;
  a.rows = (int)shape->T;
  a.V = (int)shape->V;
  a.mode = kModeForward;
  a.target = rows->target;
  a.top_k = rows->top_k;
  a.top_p = rows->top_p;
  a.min_p = rows->min_p;
  a.row_flags = flags;
  a.flags_out = flags;
  a.logprob = logprob;
  a.entropy = entropy;
  a.row_max = saved->row_max;
  a.lse_support = saved->lse_support;
  a.cut_logit = saved->cut_logit;
  a.cut_id = saved->cut_id;
  a.support_size = saved->support_size;
  a.hdr = hdr;
  STS_CUDA(timed_launch(STS_KERNEL_RESOLVE, st, [&] { return launch_resolve(a, dev.sms, st); }));
  return STS_OK;
}

sts_status sts_filter_logits(const sts_shape* shape, const float* S, const sts_rows* rows,
                             int32_t* support_size, float* cut_logit, int32_t* cut_id,
                             uint8_t* mask, float* entropy, void* ws, size_t ws_bytes,
                             sts_stream_t stream) {
  if (!shape_ok(shape)) return STS_ERR_SHAPE;
  if (!S || !support_size || !cut_logit || !cut_id) return STS_ERR_NULL;
  if (!rows) return STS_ERR_NULL;
  if (rows->len != shape->T) return STS_ERR_SHAPE;
  if (!rows->top_k || !rows->top_p || !rows->min_p) return STS_ERR_NULL;
  STS_TRY(check_ws(ws, ws_bytes, filter_bytes(shape)));
  DeviceInfo dev;
  STS_TRY(device_info(dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
  int32_t* flags = reinterpret_cast<int32_t*>(wsb + sizeof(WsHeader));
  STS_TRY(reset_header(ws, st));
  STS_CUDA(timed_launch(STS_KERNEL_VALIDATE, st, [&] {
    launch_validate(nullptr, nullptr, rows->top_p, rows->min_p, shape->T, shape->V, flags, hdr, false, st);
    return cudaGetLastError();
  }));
  ResolveArgs a{};
  a.S = S;
  a.ld = shape->V;
  a.rows = (int)shape->T;
  a.V = (int)shape->V;
  a.mode = kModeFilter;
  a.top_k = rows->top_k;
  a.top_p = rows->top_p;
  a.min_p = rows->min_p;
  a.row_flags = flags;
  a.flags_out = nullptr;
  a.support_size = support_size;
  a.cut_logit = cut_logit;
  a.cut_id = cut_id;
  a.mask = mask;
  a.entropy = entropy;
  a.hdr = hdr;
  STS_CUDA(timed_launch(STS_KERNEL_RESOLVE, st, [&] { return launch_resolve(a, dev.sms, st); }));
  return STS_OK;
}

sts_status sts_scaled_logits(const sts_shape* shape, const void* H, const void* W,
                             const float* temperature, int64_t t0, int64_t nrows, int64_t v0,
                             int64_t cols, float* S_out, int64_t ld, sts_stream_t stream) {
  if (!shape_ok(shape)) return STS_ERR_SHAPE;
  if (!H || !W || !temperature || !S_out) return STS_ERR_NULL;
  if (t0 < 0 || nrows < 1 || t0 + nrows > shape->T || (t0 % GEMM_BM) != 0) return STS_ERR_SHAPE;
  if (v0 < 0 || cols < 1 || v0 + cols > shape->V || (v0 % GEMM_BN) != 0) return STS_ERR_SHAPE;
  if (ld < cols || (ld % 4) != 0 || !aligned16(S_out) || !aligned16(H) || !aligned16(W))
    return STS_ERR_SHAPE;
  DeviceInfo dev;
  STS_TRY(device_info(dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t d = shape->d;
  CUtensorMap ma, mb, mc;
  if (!map_kmajor(&ma, H, d, shape->T, d, GEMM_BM) || !map_kmajor(&mb, W, d, shape->V, d, GEMM_BN) ||
      !map_out_f32(&mc, S_out, cols, nrows, ld))
    return STS_ERR_CUDA;
  GemmParams p{};
  p.M = (int)nrows;
  p.N = (int)cols;
  p.K = (int)d;
  p.a_mn0 = (int)t0;
  p.b_mn0 = (int)v0;
  p.tau = temperature + t0;
  p.err = nullptr;  // no workspace: a bounded-wait timeout here is not reported
  STS_CUDA(timed_launch(STS_KERNEL_LOGITS_GEMM, st, [&] {
    return run_gemm<false, false, kEpiLogits>(ma, mb, mc, p, dev.sms, st);
  }));
  return STS_OK;
}

sts_status sts_path_counts(const void* ws, sts_stream_t stream, int64_t* counts) {
  if (!ws || !counts) return STS_ERR_NULL;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return STS_ERR_CUDA;
  WsHeader h;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return STS_ERR_CUDA;
  for (int i = 0; i < 4; ++i) counts[i] = (int64_t)h.path_rows[i];
  return STS_OK;
}

int64_t sts_launch_count(int kind) {
  if (kind < 0 || kind >= STS_KERNEL_KINDS) return -1;
  return (int64_t)g_launches[kind].load();
}

sts_status sts_timing_enable(int on) {
  std::lock_guard<std::mutex> lock(g_timing.mu);
  g_timing.on = on != 0;
  g_timing.recs.clear();
  g_timing.used = 0;
  return STS_OK;
}

sts_status sts_timing_read(int kind, double* total_ms, int64_t* launches) {
  if (kind < 0 || kind >= STS_KERNEL_KINDS) return STS_ERR_SHAPE;
  if (!total_ms || !launches) return STS_ERR_NULL;
  std::lock_guard<std::mutex> lock(g_timing.mu);
  double tot = 0.0;
  int64_t n = 0;
  for (const auto& r : g_timing.recs) {
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.end) != cudaSuccess) return STS_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.beg, r.end) != cudaSuccess) return STS_ERR_CUDA;
    tot += ms;
    ++n;
  }
  *total_ms = tot;
  *launches = n;
  return STS_OK;
}

sts_status sts_probe_mass_exp(const float* s, float m, double* mass, double* lib_exp, int64_t n,
                              sts_stream_t stream) {
  if (!s || !mass || !lib_exp) return STS_ERR_NULL;
  if (n < 0) return STS_ERR_SHAPE;
  DeviceInfo dev;
  STS_TRY(device_info(dev));
  STS_CUDA(launch_mass_probe(s, m, mass, lib_exp, n, reinterpret_cast<cudaStream_t>(stream)));
  return STS_OK;
}

sts_status sts_get_status(const void* ws, sts_stream_t stream, int64_t* first_bad_row) {
  if (first_bad_row) *first_bad_row = -1;
  if (!ws) return STS_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return STS_ERR_CUDA;
  WsHeader h;
  if (cudaMemcpy(&h, ws, 16, cudaMemcpyDeviceToHost) != cudaSuccess) return STS_ERR_CUDA;
  if (h.bad_row_code != ~0ull) {
    if (first_bad_row) *first_bad_row = (int64_t)(h.bad_row_code >> 32);
    return (sts_status)(h.bad_row_code & 0xFFFFFFFFull);
  }
  if (h.err) return (sts_status)h.err;
  return STS_OK;
}

}  // extern "C"
