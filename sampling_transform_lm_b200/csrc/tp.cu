// Vocabulary-parallel tensor parallelism: the rank-order gather of the
// vocabulary shards' scaled logits into full rows ("Consolidate
// sampling-transform scoring on one shared chunked core", xorl PR 74, "What
// this PR does", item 2: ordinary vocabulary-parallel body TP is handled
// inside the core; chunk-local logits are gathered in rank order, hidden
// gradients summed across vocabulary ranks, weight-shard gradients local).
//
// After an all-gather, rank k's shard of every row sits in one contiguous
// block src[k] = [T][Vl]; the support program needs each row whole, so the
// blocks are interleaved: dst[r][k Vl + j] = src[k][r][j]. A pure copy: one
// read and one write of the T x (world Vl) fp32 logits, float4 wide when the
// shard width and the destination stride allow it.
#include "sts_internal.h"

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
