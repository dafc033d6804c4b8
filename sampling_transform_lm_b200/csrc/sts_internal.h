// Internal declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sts.h"

namespace sts {

// Status header at the start of every workspace (256 bytes).
//   bad_row_code: min over failing rows of (row << 32 | status); all-ones = none
//   err:          first non-row error (timeout, overflow), 0 = none
//   path_rows:    rows the resolver decided by each path (diagnostic counters)
//   next_row:     the resolver's row counter (rows handed out dynamically;
//                 zeroed before every resolver launch)
enum ResolvePath : int { kPathPlanned = 0, kPathFast = 1, kPathExact = 2, kPathIdentity = 3 };
struct WsHeader {
  unsigned long long bad_row_code;
  int err;
  int pad0;
  unsigned long long path_rows[4];
  unsigned long long next_row;
  unsigned long long reserved[25];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

constexpr size_t kAlign = 1024;
__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Resolver modes.
enum ResolveMode : int { kModeForward = 0, kModeSample = 1, kModeFilter = 2 };

struct ResolveArgs {
  const float* S;          // scaled logits of this row chunk, [rows][ld]
  int64_t ld;              // row stride of S (elements)
  int rows;                // rows in this chunk
  int V;
  int mode;
  // per-row inputs, already offset to the chunk's first row
  const int64_t* target;   // forward
  const int32_t* top_k;
  const float* top_p;
  const float* min_p;
  const double* u;         // sample
  const int32_t* row_flags;  // validation result (STS_ROW_INVALID bit)
  // outputs (chunk-offset); any may be null when the mode does not use it
  float* logprob;
  float* entropy;          // forward: entropy of the filtered distribution, or null
  float* row_max;
  float* lse_support;
  float* cut_logit;
  int32_t* cut_id;
  int32_t* support_size;
  int32_t* flags_out;
  int64_t* sampled;
  uint8_t* mask;           // [rows][V]
  WsHeader* hdr;
  int64_t row_base;        // global index of the chunk's first row (error reports)
  const float* max_part;   // [rows][n_parts] per-tile row maxima, or null (max pass)
  int n_parts;
};

// kernels / launchers (resolver.cu)
void launch_validate(const int64_t* target, const float* temperature, const float* top_p,
                     const float* min_p, int64_t T, int64_t V, int32_t* flags, WsHeader* hdr,
                     bool check_target, cudaStream_t stream);
cudaError_t launch_resolve(const ResolveArgs& a, int num_sms, cudaStream_t stream);
size_t resolve_smem_bytes();
cudaError_t launch_mass_probe(const float* s, float m, double* mine, double* lib, int64_t n,
                              cudaStream_t stream);

}  // namespace sts
