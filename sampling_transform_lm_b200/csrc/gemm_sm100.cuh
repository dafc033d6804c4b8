// Persistent tcgen05 GEMM for sm_100a with fused epilogues.
//
//   C[m, n] = epilogue( sum_k A[m, k] * B[n, k] )     bf16 in, fp32 accumulate
//
// One CTA per SM, 192 threads:
//   warp 0      TMA producer: fills a 4-stage shared-memory ring (A 128x64,
//               B 256x64 bf16 per stage, 128-byte swizzle) from tensor maps
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=256,
//               K=16) into one of two TMEM accumulators (2 x 256 columns)
//   warps 2..5  epilogue: tcgen05.ld the accumulator (warp w owns TMEM lanes
//               32*(w%4)..+31, i.e. 32 rows), apply the fused transform,
//               stage 32 rows x 128 B in swizzled shared memory and write it
//               with a TMA store (or a TMA fp32 reduce-add)
// Double-buffered accumulators let the epilogue of tile i overlap the
// main loop of tile i+1. Either operand may be K-major or MN-major in global
// memory; the MN-major forms are read through the MN-major UMMA descriptor,
// so no operand is ever transposed in memory.
//
// Epilogues (the forward and backward of the scoring core, "Consolidate
// sampling-transform scoring on one shared chunked core", xorl PR 74,
// "What this PR does", item 2):
//   kEpiLogits    s = z / tau_row (IEEE fp32 division) -> fp32
//   kEpiDZ        s = z / tau_row; p = exp(s - LSE_S) on the support, 0 off it;
//                 dz = g/tau * (1[col == y] - p) (0 for rows whose target is
//                 out of support or invalid) -> bf16. Support membership uses
//                 the forward's exact quotient (re-divided near the cut); p
//                 uses z * (1/tau) and the hardware exp2 (relative error
//                 ~2e-6, well below the bf16 rounding of dz)
//   kEpiStoreF32  acc -> fp32
//   kEpiReduceF32 acc -> fp32, added in place (TMA reduce-add)
//   kEpiStoreF32T, kEpiReduceF32T  the same into C's transpose: element
//                 (m, n) lands at row n, column m of the output, so a
//                 product computed as (dW)^T = H^T . dZ is written as dW
//                 (its 32 x 32 blocks are staged transposed in shared memory)
#pragma once

#include "sts_device.cuh"

namespace sts {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_THREADS = 192;
constexpr uint32_t GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;   // 16 KB
constexpr uint32_t GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;   // 32 KB
constexpr uint32_t GEMM_STAGE_BYTES = GEMM_A_BYTES + GEMM_B_BYTES;
constexpr uint32_t GEMM_EPI_BUF = 32 * 128;                // one warp: 32 rows x 128 B
constexpr uint32_t GEMM_EPI_BYTES = 4 * 2 * GEMM_EPI_BUF;  // 4 warps, double-buffered
constexpr uint32_t GEMM_TMEM_COLS = 512;                   // 2 accumulators x 256 fp32
constexpr size_t GEMM_SMEM_BYTES =
    1024 + GEMM_STAGES * GEMM_STAGE_BYTES + GEMM_EPI_BYTES + 256;
constexpr int GEMM_GROUP_M = 16;  // m-blocks per raster group (L2 reuse of B)

enum EpiKind : int {
  kEpiLogits = 0,
  kEpiDZ = 1,
  kEpiStoreF32 = 2,
  kEpiReduceF32 = 3,
  kEpiStoreF32T = 4,
  kEpiReduceF32T = 5
};

struct GemmParams {
  int M, N, K;
  // load coordinate origins (elements): MN origin and K origin of A and B
  int a_mn0, a_k0, b_mn0, b_k0;
  // store coordinate origin of C: x (column) and y (row)
  int c_x0, c_y0;
  // epilogue inputs, indexed by the problem row m (pointers pre-offset)
  const float* tau;
  const float* lse;
  const float* cut_logit;
  const int32_t* cut_id;
  const int64_t* target;
  const float* grad;
  const int32_t* flags;
  int col_base;  // global vocabulary id of problem column 0 (kEpiDZ)
  int* err;      // STS_ERR_TIMEOUT lands here
  float* max_part;  // kEpiLogits: per-(row, 256-column tile) max, [M][max_ld]; may be null
  int max_ld;
  // Raster: tiles run in groups of group_m m-blocks (0: GEMM_GROUP_M), every
  // n-block of a group before the next group, so a group's A panels are
  // reused from L2 across its n-blocks and each B panel across its m-blocks.
  int group_m;
};

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void gemm_tile_coords(int t, int num_m, int num_n, int group_m, int& mb,
                                                 int& nb) {
  const int per_group = group_m * num_n;
  const int g = t / per_group;
  const int first = g * group_m;
  const int gm = min(group_m, num_m - first);
  const int r = t - g * per_group;
  mb = first + r % gm;
  nb = r / gm;
}

template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_c, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);

  uint8_t* sA = smem;
  uint8_t* sB = sA + GEMM_STAGES * GEMM_A_BYTES;
  uint8_t* sE = sB + GEMM_STAGES * GEMM_B_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sE + GEMM_EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + GEMM_STAGES;
  uint64_t* tfull = bars + 2 * GEMM_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (p.M + GEMM_BM - 1) / GEMM_BM;
  const int num_n = (p.N + GEMM_BN - 1) / GEMM_BN;
  const int num_tiles = num_m * num_n;
  const int nk = (p.K + GEMM_BK - 1) / GEMM_BK;
  const int group_m = p.group_m > 0 ? p.group_m : GEMM_GROUP_M;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GEMM_STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 4);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    tma_prefetch_desc(&map_c);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t stage = 0, phase = 0;
    long long issued = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
      int mb, nb;
      gemm_tile_coords(t, num_m, num_n, group_m, mb, nb);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, GEMM_STAGE_BYTES);
          const uint32_t a_dst = smem_u32(sA + stage * GEMM_A_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * GEMM_B_BYTES);
          const int k = kb * GEMM_BK;
          if (A_MN) {
#pragma unroll
            for (int j = 0; j < GEMM_BM / 64; ++j)
              tma_load_2d(a_dst + j * 8192, &map_a, fb, p.a_mn0 + mb * GEMM_BM + j * 64, p.a_k0 + k);
          } else {
            tma_load_2d(a_dst, &map_a, fb, p.a_k0 + k, p.a_mn0 + mb * GEMM_BM);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < GEMM_BN / 64; ++j)
              tma_load_2d(b_dst + j * 8192, &map_b, fb, p.b_mn0 + nb * GEMM_BN + j * 64, p.b_k0 + k);
          } else {
            tma_load_2d(b_dst, &map_b, fb, p.b_k0 + k, p.b_mn0 + nb * GEMM_BN);
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == GEMM_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Our own loads must have landed before the CTA may exit.
    if (lane == 0) {
      for (int s = 0; s < GEMM_STAGES; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / GEMM_STAGES) * GEMM_STAGES + s;
          mbar_wait_drain(smem_u32(&full[s]), (uint32_t)((last / GEMM_STAGES) & 1));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(GEMM_BM, GEMM_BN, A_MN, B_MN);
    uint32_t stage = 0, phase = 0;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t aphase = (uint32_t)(it >> 1) & 1u;
      if (!mbar_wait(smem_u32(&tempty[buf]), aphase ^ 1u, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(buf * GEMM_BN);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + stage * GEMM_A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * GEMM_B_BYTES);
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            const uint64_t ad =
                A_MN ? desc_mnmajor_sw128(a0 + kk * 2048, 8192) : desc_kmajor_sw128(a0 + kk * 32);
            const uint64_t bd =
                B_MN ? desc_mnmajor_sw128(b0 + kk * 2048, 8192) : desc_kmajor_sw128(b0 + kk * 32);
            umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty[stage]));
        }
        __syncwarp();
        if (++stage == GEMM_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(&tfull[buf]));
      __syncwarp();
    }
    // Every MMA this thread issued must be complete before TMEM is freed.
    if (lane == 0) {
      umma_commit(smem_u32(drain));
      mbar_wait_drain(smem_u32(drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int CW = (EPI == kEpiDZ) ? 64 : 32;  // columns per 128-byte staged row
    const int q = warp & 3;                        // TMEM lane quarter of this warp
    uint8_t* stg = sE + (warp - 2) * 2 * GEMM_EPI_BUF;
    int it = 0;
    int sel = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      int mb, nb;
      gemm_tile_coords(t, num_m, num_n, group_m, mb, nb);
      const int buf = it & 1;
      const uint32_t aphase = (uint32_t)(it >> 1) & 1u;
      if (!mbar_wait(smem_u32(&tfull[buf]), aphase, abort_flag, p.err)) break;
      tc_fence_after();

      const int row0 = mb * GEMM_BM + q * 32;  // first problem row of this warp
      const int row = row0 + lane;
      const bool row_ok = row < p.M;
      const bool quarter_live = row0 < p.M;

      float tau = 1.f, lse = 0.f, cut = 0.f, coef = 0.f, rtau = 1.f, cut_lo = 0.f, cut_hi = 0.f;
      int cut_id = -1;
      long long y = -1;
      if (EPI == kEpiLogits || EPI == kEpiDZ) {
        if (row_ok) tau = p.tau[row];
      }
      if (EPI == kEpiDZ) {
        if (row_ok) {
          const int fl = p.flags[row];
          const bool inside = (fl & STS_ROW_TARGET_IN_SUPPORT) && !(fl & STS_ROW_INVALID);
          if (inside) {
            lse = p.lse[row];
            cut = p.cut_logit[row];
            cut_id = p.cut_id[row];
            y = p.target[row];
            coef = __fdiv_rn(p.grad[row], tau);
            rtau = __frcp_rn(tau);
            const float margin = fabsf(cut) * 1e-6f + 1e-30f;  // ~8 ulp of the cut
            cut_lo = cut - margin;
            cut_hi = cut + margin;
          }
        }
      }

      float tile_max = -INFINITY;
      for (int cc = 0; cc < GEMM_BN / CW; ++cc) {
        const int ncol0 = nb * GEMM_BN + cc * CW;  // first problem column of this chunk
        if (ncol0 >= p.N) break;
        float v[CW];
        {
          uint32_t r[32];
          const uint32_t taddr =
              tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * GEMM_BN + cc * CW);
          tmem_ld_32x32b_x32(taddr, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          if (CW == 64) {
            tmem_ld_32x32b_x32(taddr + 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[32 + j] = __uint_as_float(r[j]);
          }
        }
        if (EPI == kEpiLogits) {
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = __fdiv_rn(v[j], tau);
          const int valid = p.N - ncol0;  // columns past N hold zero-filled products
#pragma unroll
          for (int j = 0; j < CW; ++j)
            if (j < valid) tile_max = fmaxf(tile_max, v[j]);
        } else if (EPI == kEpiDZ) {
          if (coef != 0.f) {
            static_assert(CW % 32 == 0, "a chunk is whole 32-column halves");
            const long long col0 = (long long)p.col_base + ncol0;
            const long long yrel = y - col0;
            const int yj = (yrel >= 0 && yrel < CW) ? (int)yrel : -1;  // onehot column
            // z * (1/tau) is within 2 ulp of the forward's IEEE quotient; only
            // values that close to the cut ("near") are re-divided exactly, so
            // the membership decision is the forward's bit for bit. They are
            // rare and take a separate pass, so the main loop carries no
            // per-element branch and the exponentials of 32 columns overlap.
#pragma unroll
            for (int h = 0; h < CW; h += 32) {
              uint32_t near = 0u;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float sf = v[h + j] * rtau;
                near |= ((sf >= cut_lo) & !(sf > cut_hi) ? 1u : 0u) << j;
              }
              // the near columns one at a time (a rolled loop: one copy of the
              // exact division, and no register pressure on the main loop)
              for (uint32_t todo = near; todo != 0u; todo &= todo - 1u) {
                const int j0 = __ffs(todo) - 1;
                float z = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) z = j == j0 ? v[h + j] : z;
                const float sf = __fdiv_rn(z, tau);
                const bool member =
                    (sf > cut) || (sf == cut && col0 + h + j0 <= (long long)cut_id);
                const float pr = member ? __expf(sf - lse) : 0.f;
                const float o = coef * ((h + j0 == yj ? 1.f : 0.f) - pr);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[h + j] = j == j0 ? o : v[h + j];
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float sf = v[h + j] * rtau;
                const float pr = sf > cut_hi ? __expf(sf - lse) : 0.f;
                const float out = coef * ((h + j == yj ? 1.f : 0.f) - pr);
                v[h + j] = ((near >> j) & 1u) ? v[h + j] : out;
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < CW; ++j) v[j] = 0.f;
          }
        }

        // stage this row (128 bytes) into the swizzled buffer and store it
        const uint32_t sb = smem_u32(stg + sel * GEMM_EPI_BUF);
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        constexpr bool kT = (EPI == kEpiStoreF32T || EPI == kEpiReduceF32T);
        const uint32_t row_addr = sb + (uint32_t)lane * 128u;
        if (kT) {
          // block row j holds column ncol0 + j of the tile: lane's element goes
          // to column `lane` of that row (128-byte swizzle: 16-byte chunk
          // lane / 4 of row j sits at chunk (lane / 4) ^ (j % 8))
#pragma unroll
          for (int j = 0; j < 32; ++j)
            st_shared_f32(sb + (uint32_t)j * 128u + ((uint32_t)((lane >> 2) ^ (j & 7)) << 4) +
                              ((uint32_t)(lane & 3) << 2),
                          v[j]);
        }
#pragma unroll
        for (int c = 0; c < 8 && !kT; ++c) {
          uint32_t w0, w1, w2, w3;
          if (EPI == kEpiDZ) {
            w0 = pack_bf16x2(v[c * 8 + 0], v[c * 8 + 1]);
            w1 = pack_bf16x2(v[c * 8 + 2], v[c * 8 + 3]);
            w2 = pack_bf16x2(v[c * 8 + 4], v[c * 8 + 5]);
            w3 = pack_bf16x2(v[c * 8 + 6], v[c * 8 + 7]);
          } else {
            w0 = __float_as_uint(v[c * 4 + 0]);
            w1 = __float_as_uint(v[c * 4 + 1]);
            w2 = __float_as_uint(v[c * 4 + 2]);
            w3 = __float_as_uint(v[c * 4 + 3]);
          }
          st_shared_v4(row_addr + (uint32_t)((c ^ (lane & 7)) << 4), w0, w1, w2, w3);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && quarter_live) {
          if (EPI == kEpiReduceF32)
            tma_reduce_add_2d(&map_c, sb, p.c_x0 + ncol0, p.c_y0 + row0);
          else if (EPI == kEpiReduceF32T)
            tma_reduce_add_2d(&map_c, sb, p.c_x0 + row0, p.c_y0 + ncol0);
          else if (EPI == kEpiStoreF32T)
            tma_store_2d(&map_c, sb, p.c_x0 + row0, p.c_y0 + ncol0);
          else
            tma_store_2d(&map_c, sb, p.c_x0 + ncol0, p.c_y0 + row0);
          bulk_commit();
        }
        __syncwarp();
        sel ^= 1;
      }
      if (EPI == kEpiLogits && p.max_part != nullptr && row_ok)
        p.max_part[(size_t)row * p.max_ld + nb] = tile_max;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[buf]));
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
  }
}

}  // namespace sts
