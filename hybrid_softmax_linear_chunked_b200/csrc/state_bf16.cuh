// State kernels of the bf16 path ("ReHyAt overview" page §2.3: S = sum phi_k(k) v^T,
// Z = sum phi_k(k), S_{t+1} = S_t + sum over the frames folded after chunk t).
//
//  * fold_partial_bf16_kernel: for one fold range of key rows (the frames leaving a chunk's
//    softmax window) and one split of it, dS = phi_k(K)^T V (F x D) and dZ = phi_k(K)^T 1 on the
//    tensor cores: phi_k is computed by the CUDA cores from the TMA-loaded K tile straight into
//    shared memory in the layout of an MN-major MMA operand, and both products accumulate in
//    TMEM in fp32 over the split's 128-token tiles.
//  * state_scan_kernel: exclusive prefix over fold ranges (the state chunk c reads), written as
//    a transposed bf16 copy S_c^T [D][F] for the attention kernel's readout MMA, plus fp32 Z_c
//    (and fp32 S_c on request).
//  * state_add_kernel: S += sum of split partials, Z likewise (streaming fold, in place).
#pragma once

#include "featmap.cuh"
#include "sm100.cuh"

namespace rehyat {
namespace state {

using namespace sm100;

constexpr int kTok = 128;  // tokens per tile (MMA K)
constexpr int kHD = 128;
constexpr int kFD = 128;
constexpr int kThreads = 192;
constexpr int kTileBytes = kTok * kHD * 2;

constexpr uint32_t kOffK = 0;                          // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;      // 2 stages
constexpr uint32_t kOffPhi = kOffV + 2 * kTileBytes;    // 2 stages
constexpr uint32_t kOffOnes = kOffPhi + 2 * kTileBytes; // 16 x 128 bf16 of 1.0
constexpr int kMinG = 4;                                 // smallest supported group count
constexpr uint32_t kOffW = kOffOnes + 4096;             // W_k of the head (F * D / G fp32)
constexpr uint32_t kWBytesMax = kFD * kHD / kMinG * 4;
constexpr uint32_t kOffB = kOffW + kWBytesMax;          // bias
constexpr uint32_t kSmemBytes = kOffB + kFD * 4 + 1024;

enum Bar {
  kKFull = 0, kKEmpty = 2, kVFull = 4, kVEmpty = 6, kPhiFull = 8, kPhiEmpty = 10, kDone = 12,
  kNumBars = 13
};

struct FoldParams {
  int L, H, P;
  int T, Tc, To, kv_frame0;  // schedule (mode 0)
  int single_rows;           // mode 1: fold rows [0, single_rows) of the k/v buffer; -1 = mode 0
  int n_fold, splits;
  const float* Wk;
  const float* bk;
  float* dS;  // [BH][n_fold][splits][F][D]
  float* dZ;  // [BH][n_fold][splits][F]
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// grid (splits, n_fold, BH), block 192: warps 0-3 feature map (one token per thread), warp 4
// TMA producer, warp 5 MMA issuer (both run their loop warp-wide; lane 0 issues).
// TMEM: dS in columns [0, 128), dZ in [128, 144).
template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    fold_partial_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const FoldParams p) {
  constexpr int Dg = kHD / G, Fg = kFD / G;
  static_assert(G >= kMinG && kFD * Dg * 4 <= kWBytesMax, "W_k does not fit its shared-memory slot");
  static_assert(kSmemBytes <= 232448, "shared memory over the per-CTA limit");
  const int split = blockIdx.x, fc = blockIdx.y, bh = blockIdx.z, h = bh % p.H;
  int r0, r1;
  if (p.single_rows >= 0) {
    r0 = 0;
    r1 = p.single_rows;
  } else {
    const int w0 = max(0, fc * p.Tc - p.To), w1 = max(0, (fc + 1) * p.Tc - p.To);
    r0 = (w0 - p.kv_frame0) * p.L;
    r1 = (w1 - p.kv_frame0) * p.L;
  }
  const int n_tiles_all = (r1 - r0 + kTok - 1) / kTok;
  const int t_begin = (int)((long long)split * n_tiles_all / p.splits);
  const int t_end = (int)((long long)(split + 1) * n_tiles_all / p.splits);
  const int n_tiles = t_end - t_begin;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* dS = p.dS + (((size_t)bh * p.n_fold + fc) * p.splits + split) * kFD * kHD;
  float* dZ = p.dZ + (((size_t)bh * p.n_fold + fc) * p.splits + split) * kFD;
  if (n_tiles <= 0) {
    for (int i = tid; i < kFD * kHD; i += kThreads) dS[i] = 0.f;
    for (int i = tid; i < kFD; i += kThreads) dZ[i] = 0.f;
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  float* sW = reinterpret_cast<float*>(sm + kOffW);
  float* sB = reinterpret_cast<float*>(sm + kOffB);

  if (warp == 4) {
    tmem_alloc(&tmem_base_sh, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool many = (i == kKEmpty || i == kKEmpty + 1 || i == kPhiFull || i == kPhiFull + 1);
      mbar_init(&bars[i], many ? 128 : 1);
    }
    abort_sh = 0;
    fence_mbar_init();
  }
  {
    const float* Wh = p.Wk + (size_t)h * kFD * Dg;
    for (int i = tid; i < kFD * Dg; i += kThreads) sW[i] = Wh[i];
    for (int i = tid; i < kFD; i += kThreads) sB[i] = p.bk ? p.bk[(size_t)h * kFD + i] : 0.f;
    uint32_t* ones = reinterpret_cast<uint32_t*>(sm + kOffOnes);
    for (int i = tid; i < 1024; i += kThreads) ones[i] = 0x3F803F80u;  // bf16 pair (1.0, 1.0)
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  const bool leader = lane == 0;
  if (warp == 4) {
    // ---- producer ----
    if (leader) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    bool ok = true;
    int issued_k = 0, issued_v = 0;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i & 1;
      const int row = r0 + (t_begin + i) * kTok;
      if (i >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kKEmpty + s], ((i >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      if (leader) {
        uint8_t* dk = sm + kOffK + s * kTileBytes;
        mbar_arrive_expect_tx(&bars[kKFull + s], kTileBytes);
        tma_load_3d(dk, &tmK, &bars[kKFull + s], 0, row, bh);
        tma_load_3d(dk + kTok * 128, &tmK, &bars[kKFull + s], 64, row, bh);
      }
      __syncwarp();
      ++issued_k;
      if (i >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kVEmpty + s], ((i >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      if (leader) {
        uint8_t* dv = sm + kOffV + s * kTileBytes;
        mbar_arrive_expect_tx(&bars[kVFull + s], kTileBytes);
        tma_load_3d(dv, &tmV, &bars[kVFull + s], 0, row, bh);
        tma_load_3d(dv + kTok * 128, &tmV, &bars[kVFull + s], 64, row, bh);
      }
      __syncwarp();
      ++issued_v;
    }
    if (!ok) {
      for (int i = max(0, issued_k - 2); i < issued_k; ++i)
        mbar_wait_drain(&bars[kKFull + (i & 1)], (i >> 1) & 1);
      for (int i = max(0, issued_v - 2); i < issued_v; ++i)
        mbar_wait_drain(&bars[kVFull + (i & 1)], (i >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---- MMA issuer ----
    const uint32_t id_s = idesc_bf16(kFD, kHD, true, true);
    const uint32_t id_z = idesc_bf16(kFD, 16, true, false);
    const uint32_t ones = smem_u32(sm + kOffOnes);
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kPhiFull + s], (i >> 1) & 1, abort_flag) &&
                                       mbar_wait(&bars[kVFull + s], (i >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint32_t ph = smem_u32(sm + kOffPhi + s * kTileBytes);
        const uint32_t vb = smem_u32(sm + kOffV + s * kTileBytes);
        for (int kk = 0; kk < kTok / 16; ++kk) {
          const uint64_t a = sdesc_sw128(ph + kk * 16 * 128, kTok * 128, 1024);
          mma_ss(tmem, a, sdesc_sw128(vb + kk * 16 * 128, kTok * 128, 1024), id_s,
                 (i > 0 || kk > 0) ? 1u : 0u);
          mma_ss(tmem + 128, a,
                 sdesc_sw128(ones + (kk >> 2) * (16 * 128) + (kk & 3) * 32, 16, 1024), id_z,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars[kPhiEmpty + s]);
        mma_commit(&bars[kVEmpty + s]);
      }
      __syncwarp();
    }
    if (leader) mma_commit(&bars[kDone]);
    __syncwarp();
    mbar_wait_drain(&bars[kDone], 0);
    __syncwarp();
  } else {
    // ---- feature map warps: thread tid owns token row tid of each tile ----
    const int r = tid;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kKFull + s], (i >> 1) & 1, abort_flag));
      if (ok && i >= 2)
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kPhiEmpty + s], ((i >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      const uint8_t* krow = sm + kOffK + s * kTileBytes;
      uint8_t* prow = sm + kOffPhi + s * kTileBytes;
      const bool valid = r0 + (t_begin + i) * kTok + r < r1;
#pragma unroll 1
      for (int g = 0; g < G; ++g) {
        float x[Dg];
#pragma unroll
        for (int c8 = 0; c8 < Dg / 8; ++c8) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(krow + sw128_offset(r, g * Dg + c8 * 8, kTok));
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(b2[e]);
            x[c8 * 8 + 2 * e] = f2.x;
            x[c8 * 8 + 2 * e + 1] = f2.y;
          }
        }
#pragma unroll
        for (int c8 = 0; c8 < Fg / 8; ++c8) {
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float ph2[2];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
              const int o = c8 * 8 + 2 * e + q2;
              const int f = g * Fg + o;
              const float* w = sW + (g * Fg + o) * Dg;
              float u = sB[f];
#pragma unroll
              for (int k2 = 0; k2 < Dg; ++k2) u = fmaf(w[k2], x[k2], u);
              ph2[q2] = valid ? int_pow(softplus_fast(u), part_power(f, kFD, p.P)) : 0.f;
            }
            packed[e] = pack_bf16x2(ph2[0], ph2[1]);
          }
          *reinterpret_cast<uint4*>(prow + sw128_offset(r, g * Fg + c8 * 8, kTok)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
      fence_async_smem();
      mbar_arrive(&bars[kKEmpty + s]);
      mbar_arrive(&bars[kPhiFull + s]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kDone], 0, abort_flag));
    if (ok) {
      tc_fence_after();
      // lane r of TMEM is feature f = r: dS row f (128 columns), dZ in column 128.
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;  // warps 0-3
      float* srow = dS + (size_t)r * kHD;
#pragma unroll
      for (int cc = 0; cc < kHD / 32; ++cc) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + cc * 32, rr);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          *reinterpret_cast<float4*>(srow + cc * 32 + q4 * 4) =
              make_float4(__uint_as_float(rr[q4 * 4]), __uint_as_float(rr[q4 * 4 + 1]),
                          __uint_as_float(rr[q4 * 4 + 2]), __uint_as_float(rr[q4 * 4 + 3]));
      }
      uint32_t z16[16];
      tmem_ld16(tmem + lane_base + 128, z16);
      dZ[r] = __uint_as_float(z16[0]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Exclusive prefix over fold ranges.  grid (F/32 * D/32, BH), block (32, 8).
//   acc starts at S0/Z0 (if given) else 0; for c in 0..C-1: emit state c, then add fold c.
//   St  [BH][C][D][F] bf16 (transposed), Zc [BH][C][F] fp32, S_out [BH][C][F][D] fp32 (opt).
__global__ void __launch_bounds__(256) state_scan_kernel(
    const float* __restrict__ dS, const float* __restrict__ dZ, int n_fold, int splits, int C,
    int F, int D, const float* __restrict__ S0, const float* __restrict__ Z0,
    __nv_bfloat16* __restrict__ St, float* __restrict__ Zc, float* __restrict__ S_out,
    float* __restrict__ Z_out) {
  __shared__ float tile[32][33];
  const int bh = blockIdx.y;
  const int tiles_d = D / 32;
  const int f0 = (blockIdx.x / tiles_d) * 32, d0 = (blockIdx.x % tiles_d) * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  float acc[4];
  float accz = 0.f;
  const bool z_thread = (d0 == 0 && ty == 0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int f = f0 + ty + 8 * i;
    acc[i] = S0 ? S0[((size_t)bh * F + f) * D + d0 + tx] : 0.f;
  }
  if (z_thread) accz = Z0 ? Z0[(size_t)bh * F + f0 + tx] : 0.f;
  for (int c = 0; c < C; ++c) {
    if (St) {
#pragma unroll
      for (int i = 0; i < 4; ++i) tile[ty + 8 * i][tx] = acc[i];
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int d = d0 + ty + 8 * i;
        St[(((size_t)bh * C + c) * D + d) * F + f0 + tx] = __float2bfloat16_rn(tile[tx][ty + 8 * i]);
      }
      __syncthreads();
    }
    if (S_out) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        S_out[(((size_t)bh * C + c) * F + f0 + ty + 8 * i) * D + d0 + tx] = acc[i];
    }
    if (z_thread) {
      if (Zc) Zc[((size_t)bh * C + c) * F + f0 + tx] = accz;
      if (Z_out) Z_out[((size_t)bh * C + c) * F + f0 + tx] = accz;
    }
    if (c < n_fold) {
      for (int s = 0; s < splits; ++s) {
        const size_t base = (((size_t)bh * n_fold + c) * splits + s);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += dS[(base * F + f0 + ty + 8 * i) * D + d0 + tx];
        if (z_thread) accz += dZ[base * F + f0 + tx];
      }
    }
  }
}

// S[bh] += sum_s dS[bh][0][s], Z likewise.  grid (ceil(F*D/256), BH), block 256.
__global__ void __launch_bounds__(256) state_add_kernel(const float* __restrict__ dS,
                                                        const float* __restrict__ dZ, int splits,
                                                        int F, int D, float* __restrict__ S,
                                                        float* __restrict__ Z) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e < F * D) {
    float a = S[(size_t)bh * F * D + e];
    for (int s = 0; s < splits; ++s) a += dS[((size_t)bh * splits + s) * F * D + e];
    S[(size_t)bh * F * D + e] = a;
  }
  if (e < F) {
    float z = Z[(size_t)bh * F + e];
    for (int s = 0; s < splits; ++s) z += dZ[((size_t)bh * splits + s) * F + e];
    Z[(size_t)bh * F + e] = z;
  }
}

}  // namespace state
}  // namespace rehyat
