// sts_filter_logits_noalloc: the support program on caller-given fp32 scaled
// logits, for callers that cannot allocate device memory.
//
// It runs the same two kernels as sts_filter_logits (row validation, then the
// per-row resolver), but their scratch -- a 256-byte status header and one
// int32 flag per row -- lives in the file-scope device array below instead of
// a caller-provided workspace. Nothing here calls cudaMalloc, cudaFree or any
// allocating library routine; the array is created when the library's device
// code is loaded and every GPU that loads the library keeps it until exit.
#include <mutex>

#include "sts_internal.h"

namespace sts {
namespace {

constexpr int64_t kNoAllocMaxRows = 65536;
constexpr size_t kNoAllocBytes = sizeof(WsHeader) + (size_t)kNoAllocMaxRows * sizeof(int32_t);

// Shared by every call on a device; holds the previous call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

struct NoAllocDevice {
  void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int sms = 0;
  bool arch_ok = false;
};

// Resolves, once per device and with that device current, the device address
// of the scratch array (a host-side reference to the array's name is only a
// stand-in, not a device pointer) and the SM count.
sts_status noalloc_device(NoAllocDevice& out) {
  static NoAllocDevice cache[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return STS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  NoAllocDevice& d = cache[dev];
  if (d.scratch == nullptr) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return STS_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return STS_ERR_CUDA;
    d.arch_ok = (major == 10 && minor == 0);
    d.sms = sms;
    d.scratch = p;
  }
  out = d;
  return out.arch_ok ? STS_OK : STS_ERR_UNSUPPORTED_ARCH;
}

}  // namespace
}  // namespace sts

using namespace sts;

extern "C" sts_status sts_filter_logits_noalloc(const sts_shape* shape, const float* S,
                                                const sts_rows* rows, int32_t* support_size,
                                                float* cut_logit, int32_t* cut_id, uint8_t* mask,
                                                sts_stream_t stream) {
  if (!shape || shape->T < 1 || shape->V < 1 || shape->V > (int64_t(1) << 31) - 1)
    return STS_ERR_SHAPE;
  if (shape->T > kNoAllocMaxRows) return STS_ERR_SHAPE;  // beyond the scratch array
  if (!S || !support_size || !cut_logit || !cut_id || !rows) return STS_ERR_NULL;
  if (rows->len != shape->T) return STS_ERR_SHAPE;
  if (!rows->top_k || !rows->top_p || !rows->min_p) return STS_ERR_NULL;
  NoAllocDevice dev;
  const sts_status ds = noalloc_device(dev);
  if (ds != STS_OK) return ds;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(dev.scratch);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base);
  int32_t* flags = reinterpret_cast<int32_t*>(base + sizeof(WsHeader));
  // the header must start clean on every call; the flags are fully rewritten
  if (cudaMemsetAsync(&hdr->bad_row_code, 0xFF, sizeof(hdr->bad_row_code), st) != cudaSuccess ||
      cudaMemsetAsync(&hdr->err, 0, sizeof(hdr->err), st) != cudaSuccess)
    return STS_ERR_CUDA;
  launch_validate(nullptr, nullptr, rows->top_p, rows->min_p, shape->T, shape->V, flags, hdr, false, st);
  if (cudaGetLastError() != cudaSuccess) return STS_ERR_CUDA;
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
  a.support_size = support_size;
  a.cut_logit = cut_logit;
  a.cut_id = cut_id;
  a.mask = mask;
  a.hdr = hdr;
  if (launch_resolve(a, dev.sms, st) != cudaSuccess) return STS_ERR_CUDA;
  return STS_OK;
}
