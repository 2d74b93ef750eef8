// Batched bf16 GEMM on the tcgen05 tensor cores (sm_100a): C[b] (+)= alpha * A[b] B[b], fp32
// accumulation in TMEM, fp32 or bf16 output.  The backward pass of the hybrid attention is built
// from these products (QK^T, dO V^T, dS K, dS^T Q, P^T dO, the state and feature-map gradients),
// each with its operands in whichever layout the forward left them:
//   A is M x K, stored K-contiguous ([M][K], a_mn = 0) or M-contiguous ([K][M], a_mn = 1);
//   B is K x N, stored K-contiguous ([N][K], b_mn = 0) or N-contiguous ([K][N], b_mn = 1).
// With split > 1 the K range is cut into `split` parts computed by separate CTAs that add their
// partial tiles into C with fp32 atomics (C must hold the initial value; fp32 output only).
// With b_parts = 2 the product is A (B + B2) computed as A B + A B2 in one accumulator (B2 a
// second operand of B's shape and layout): the K loop runs twice over A, first against B, then
// against B2.
// One CTA computes one 128 x 128 tile of C: warp 0 streams 64-deep K slices of A and B through a
// kStages-deep TMA ring (128-byte swizzle; rows, columns and K past the matrix read zeros), warp 1
// issues four M128 N128 K16 MMAs per slice and owns the TMEM accumulator, warps 2-5 read the
// accumulator back (one row per thread) and store, add to, or round into C.  Short K loops use
// the 2-stage instance, whose 65 KB of shared memory lets three CTAs share an SM, so one CTA's
// epilogue overlaps the others' loads.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace rehyat {
namespace gemm {

using namespace sm100;

constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kThreads = 192;
constexpr uint32_t kTileA = kBM * kBK * 2;
constexpr uint32_t kTileB = kBN * kBK * 2;
constexpr uint32_t kStageBytes = kTileA + kTileB;
__host__ __device__ constexpr uint32_t smem_bytes(int stages) {
  return stages * kStageBytes + 1024;
}

struct Params {
  int M, N, K;
  int a_mn, b_mn;
  void* C;
  long long ldc, c_batch;  // elements
  int c_bf16, accumulate;
  float alpha;
  int split;    // K parts (>= 1); blockIdx.z = batch * split + part
  int b_parts;  // 1, or 2: C (+)= alpha A (B + B2) (split must be 1)
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Descriptor of the kk-th K16 step of a 128-row operand tile in shared memory.
//   K-contiguous tile: one box of [128 rows][64 K] (128-byte rows), step = 32 bytes.
//   M/N-contiguous tile: two boxes of [64 K][64 rows] (8 KB each, the second holding rows
//   64..127), step = 16 K-rows = 2 KB, leading byte offset = 8 KB between the two halves.
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kk, bool mn) {
  return mn ? sdesc_sw128(base + kk * 16 * 128, 64 * 128, 1024)
            : sdesc_sw128(base + kk * 32, 16, 1024);
}

// Loads the 64-deep K slice kb of the 128-row tile starting at row r0 of an operand.
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                             bool mn, int r0, int k0, int b) {
  if (mn) {
    tma_load_3d(dst, map, bar, r0, k0, b);
    tma_load_3d(dst + 64 * 128, map, bar, r0 + 64, k0, b);
  } else {
    tma_load_3d(dst, map, bar, k0, r0, b);
  }
}

// grid (ceil(N / 128), ceil(M / 128), batch * split), block 192.
template <int kStages>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, const Params p) {
  static_assert(smem_bytes(kStages) + 256 <= 232448, "shared memory over the limit");
  enum { kFull = 0, kEmpty = kStages, kDone = 2 * kStages, kNumBars };
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  const int b = blockIdx.z / p.split, part = blockIdx.z - b * p.split;
  const int k_slices = (p.K + kBK - 1) / kBK;
  const int per_part = (k_slices + p.split - 1) / p.split;
  const int kb0 = part * per_part;
  const int num_k1 = max(0, min(k_slices, kb0 + per_part) - kb0);  // slices against one B
  const int num_k = num_k1 * p.b_parts;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool leader = lane == 0;

  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 128);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ---- TMA producer ----
    if (leader) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    bool ok = true;
    int issued = 0;
    for (int kb = 0; kb < num_k; ++kb) {
      const int s = kb % kStages;
      if (kb >= kStages)
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kEmpty + s], ((kb / kStages) - 1) & 1, abort_flag));
      if (!ok) break;
      if (leader) {
        uint8_t* st = sm + s * kStageBytes;
        const int kk0 = (kb0 + kb % num_k1) * kBK;
        mbar_arrive_expect_tx(&bars[kFull + s], kStageBytes);
        load_operand(st, &tmA, &bars[kFull + s], p.a_mn, m0, kk0, b);
        load_operand(st + kTileA, kb < num_k1 ? &tmB : &tmB2, &bars[kFull + s], p.b_mn, n0, kk0, b);
      }
      __syncwarp();
      ++issued;
    }
    if (!ok) {
      for (int kb = (issued > kStages ? issued - kStages : 0); kb < issued; ++kb)
        mbar_wait_drain(&bars[kFull + kb % kStages], (kb / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer ----
    const uint32_t idesc = idesc_bf16(kBM, kBN, p.a_mn != 0, p.b_mn != 0);
    bool ok = true;
    for (int kb = 0; kb < num_k && ok; ++kb) {
      const int s = kb % kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kFull + s], (kb / kStages) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint32_t a = smem_u32(sm + s * kStageBytes);
        const uint32_t bb = a + kTileA;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_ss(tmem, operand_desc(a, kk, p.a_mn), operand_desc(bb, kk, p.b_mn), idesc,
                 (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[kEmpty + s]);
      }
      __syncwarp();
    }
    if (leader) mma_commit(&bars[kDone]);
    __syncwarp();
  } else {
    // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 = rows of the tile ----
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kDone], 0, abort_flag));
    if (ok && num_k > 0) {
      tc_fence_after();
      const int g = warp & 3;
      const int row = m0 + g * 32 + lane;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(g * 32) << 16);
      const bool row_ok = row < p.M;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        const int col0 = n0 + c * 32;
        if (!row_ok || col0 >= p.N) continue;
        const long long base = (long long)b * p.c_batch + (long long)row * p.ldc + col0;
        const int ncol = min(32, p.N - col0);
        if (p.split > 1) {
          float* C = static_cast<float*>(p.C) + base;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < ncol) atomicAdd(C + i, __uint_as_float(r[i]) * p.alpha);
        } else if (p.c_bf16) {
          __nv_bfloat16* C = static_cast<__nv_bfloat16*>(p.C) + base;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (i < ncol) {
              float x = __uint_as_float(r[i]) * p.alpha;
              if (p.accumulate) x += __bfloat162float(C[i]);
              C[i] = __float2bfloat16_rn(x);
            }
          }
        } else {
          float* C = static_cast<float*>(p.C) + base;
          if (ncol == 32) {
            float4* C4 = reinterpret_cast<float4*>(C);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 v = make_float4(__uint_as_float(r[4 * i]) * p.alpha,
                                     __uint_as_float(r[4 * i + 1]) * p.alpha,
                                     __uint_as_float(r[4 * i + 2]) * p.alpha,
                                     __uint_as_float(r[4 * i + 3]) * p.alpha);
              if (p.accumulate) {
                const float4 o = C4[i];
                v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
              }
              C4[i] = v;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (i < ncol) {
                const float x = __uint_as_float(r[i]) * p.alpha;
                C[i] = p.accumulate ? C[i] + x : x;
              }
            }
          }
        }
      }
    }
  }
  // every MMA (and its barrier arrivals) is complete once kDone has fired
  if (warp == 1) mbar_wait_drain(&bars[kDone], 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace gemm
}  // namespace rehyat
