// State kernels of the bf16 path ("ReHyAt overview" page §2.3: S = sum phi_k(k) v^T,
// Z = sum phi_k(k), S_{t+1} = S_t + sum over the frames folded after chunk t).
//
//  * fold_partial_bf16_kernel: for one fold range of key rows (the frames leaving a chunk's
//    softmax window) and one split of it, dS = phi_k(K)^T V (F x D) and dZ = phi_k(K)^T 1 on the
//    tensor cores.  The grouped linear of phi_k is a tensor-core product too (the compact
//    block-diagonal weights of featmap.cuh, built by the CTA in shared memory); the CUDA cores
//    apply bias, softplus and powers and write phi_k straight into the shared-memory layout of an
//    MN-major MMA operand; both sums accumulate in TMEM in fp32 over the split's 128-token
//    tiles.  The compact weights leave room for two K stages, so the next K tile loads while the
//    current one is still being multiplied (the dense G = 1 matrix keeps one).
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
// warps 0-15 feature map (four per 32-lane TMEM group, 32 features each), 16 producer, 17 MMA:
// sixteen feature-map warps keep enough independent softplus chains in flight per SM
constexpr int kPhiWarps = 16;
constexpr int kPhiThreads = kPhiWarps * 32;
constexpr int kWarpProducer = kPhiWarps, kWarpMma = kPhiWarps + 1;
constexpr int kThreads = kPhiThreads + 64;
constexpr int kTileBytes = kTok * kHD * 2;

// Shared memory with kKSt K stages: 2 with the compact weights of G >= 2 (at most 64 rows,
// 16 KB per part), 1 with the dense G = 1 matrix (32 KB per part).
template <int kKSt>
struct FoldLayout {
  static constexpr uint32_t kWPart = kKSt == 2 ? 16384 : 32768;
  static constexpr uint32_t kOffK = 0;                           // kKSt stages
  static constexpr uint32_t kOffV = kOffK + kKSt * kTileBytes;    // 2 stages
  static constexpr uint32_t kOffPhi = kOffV + 2 * kTileBytes;     // 2 stages
  static constexpr uint32_t kOffW = kOffPhi + 2 * kTileBytes;     // compact W_k: hi, then lo
  static constexpr uint32_t kOffOnes = kOffW + 2 * kWPart;        // 8 rows x 128 B of bf16 1.0
  static constexpr uint32_t kOffB = kOffOnes + 1024;              // bias of phi_k, F fp32
  static constexpr uint32_t kOffPw = kOffB + kFD * 4;             // part power of each feature
  static constexpr uint32_t kSmemBytes = kOffPw + kFD + 1024;     // + alignment slack
};

// TMEM columns: U buffers [0,128) and [128,256), dS [256,384), dZ [384,400).
constexpr uint32_t kColDS = 256, kColDZ = 384;

enum Bar {
  kKFull = 0, kKEmpty = 2, kVFull = 4, kVEmpty = 6, kUFull = 8, kUEmpty = 10, kPhiFull = 12,
  kPhiEmpty = 14, kDone = 16, kNumBars = 17
};

struct FoldParams {
  int L, H, P;
  int T, Tc, To, kv_frame0;  // schedule (mode 0)
  int fold_c0;               // mode 0: chunk index of fold 0 (a segment of a longer sequence)
  int single_rows;           // mode 1: fold rows [0, single_rows) of the k/v buffer; -1 = mode 0
  // mode 1 with a carried segment: the first seg_rows of the fold range come from tmKc/tmVc at
  // row seg_row0, the remaining single_rows - seg_rows from tmK/tmV at row 0; each segment is
  // tiled on its own.  seg_rows = 0: one segment.
  int seg_rows, seg_row0;
  int kv_rows, carry_rows;  // rows per (b, h) of the main and of the carried K/V tensor maps
  int n_fold, splits;
  int G;
  const float* W;   // [H, G, F/G, D/G] fp32 weights of phi_k
  const float* bk;
  float* dS;  // [BH][n_fold][splits][F][D]
  float* dZ;  // [BH][n_fold][splits][F]
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// K-major SW128 descriptor of the kk-th 16-wide K step of a 128 x 128 bf16 tile.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_addr, int kk) {
  return sdesc_sw128(tile_addr + (kk >> 2) * (kTok * 128) + (kk & 3) * 32, 16, 1024);
}
// MN-major SW128 descriptor of the kk-th 16-row K step of a [128 rows][128 cols] bf16 tile.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_addr, int kk) {
  return sdesc_sw128(tile_addr + kk * 16 * 128, kTok * 128, 1024);
}

// grid (splits, n_fold, BH), block 320: warps 0-7 feature map (token row = TMEM lane
// 32*(warp%4) + lane; warps 0-3 take features 0-63, warps 4-7 features 64-127), warp 8 TMA
// producer, warp 9 MMA issuer (both run their loop warp-wide; lane 0 issues).
// Per 128-token tile i: U = K_i Wbd_hi^T + K_i Wbd_lo^T (grouped linear of phi_k on the tensor
// cores, fp32 in TMEM); the feature-map warps add the bias, apply softplus and the part powers,
// and write phi_k as bf16 into the MN-major A operand of dS += phi_k^T V_i and
// dZ += phi_k^T 1 (a ones matrix as B: N = 16, every row group read from the same 1 KiB).
template <int kKSt>
__global__ void __launch_bounds__(kThreads, 1)
    fold_partial_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV,
                             const __grid_constant__ CUtensorMap tmKc,
                             const __grid_constant__ CUtensorMap tmVc, const FoldParams p) {
  using Lay = FoldLayout<kKSt>;
  static_assert(Lay::kSmemBytes + 256 <= 232448, "shared memory (dynamic + static) over the limit");
  const int split = blockIdx.x, fc = blockIdx.y, bh = blockIdx.z, h = bh % p.H;
  int r0, r1;
  if (p.single_rows >= 0) {
    r0 = 0;
    r1 = p.single_rows;
  } else {
    const int c = p.fold_c0 + fc;
    const int w0 = max(0, c * p.Tc - p.To), w1 = max(0, (c + 1) * p.Tc - p.To);
    r0 = (w0 - p.kv_frame0) * p.L;
    r1 = (w1 - p.kv_frame0) * p.L;
  }
  // tiles [0, n_seg) cover the carried segment, the rest rows [r0 + seg, r1)
  const int seg = p.single_rows >= 0 ? p.seg_rows : 0;
  const int n_seg = (seg + kTok - 1) / kTok;
  const int n_tiles_all = n_seg + (r1 - r0 - seg + kTok - 1) / kTok;
  const int t_begin = (int)((long long)split * n_tiles_all / p.splits);
  const int t_end = (int)((long long)(split + 1) * n_tiles_all / p.splits);
  const int n_tiles = t_end - t_begin;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* dS = p.dS + (((size_t)bh * p.n_fold + fc) * p.splits + split) * kFD * kHD;
  float* dZ = p.dZ + (((size_t)bh * p.n_fold + fc) * p.splits + split) * kFD;
  // Launched behind the streaming attention with programmatic serialization, the fold reads
  // only the window (never written there) and overlaps the attention's last wave; every CTA
  // waits for that grid before it exits, so whatever follows the fold in the stream is ordered
  // after the attention too.  For an ordinary launch the wait returns at once.
  if (n_tiles <= 0) {
    for (int i = tid; i < kFD * kHD; i += kThreads) dS[i] = 0.f;
    for (int i = tid; i < kFD; i += kThreads) dZ[i] = 0.f;
    grid_dep_wait();
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  float* sB = reinterpret_cast<float*>(sm + Lay::kOffB);
  uint8_t* sPw = sm + Lay::kOffPw;

  if (warp == kWarpProducer) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool many = (i == kUEmpty || i == kUEmpty + 1 || i == kPhiFull || i == kPhiFull + 1);
      mbar_init(&bars[i], many ? kPhiThreads : 1);
    }
    abort_sh = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < kFD; i += kThreads) {
    sB[i] = p.bk ? p.bk[(size_t)h * kFD + i] : 0.f;
    sPw[i] = static_cast<uint8_t>(feature_power(i, kFD, p.P));
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(sm + Lay::kOffOnes);
    for (int i = tid; i < 256; i += kThreads) ones[i] = 0x3F803F80u;  // bf16 pair (1.0, 1.0)
  }
  build_compact_w(p.W + (size_t)h * kFD * kHD / p.G, kFD, kHD, p.G, sm + Lay::kOffW,
                  sm + Lay::kOffW + Lay::kWPart, tid, kThreads);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t sK0 = smem_u32(sm + Lay::kOffK), sV0 = smem_u32(sm + Lay::kOffV);
  const uint32_t sPhi = smem_u32(sm + Lay::kOffPhi), sW0 = smem_u32(sm + Lay::kOffW);
  const uint32_t sOnes = smem_u32(sm + Lay::kOffOnes);

  const bool leader = lane == 0;
  if (warp == kWarpProducer) {
    // ---- producer ----
    if (leader) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    __syncwarp();
    bool ok = true;
    int issued_k = 0, issued_v = 0;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i & 1;
      const int ti = t_begin + i;
      const bool carried = ti < n_seg;
      // the main source holds window row seg at its row r0 (mode 1 with a segment: r0 = 0)
      const int row = carried ? p.seg_row0 + ti * kTok : r0 + (ti - n_seg) * kTok;
      const CUtensorMap* mK = carried ? &tmKc : &tmK;
      const CUtensorMap* mV = carried ? &tmVc : &tmV;
      const int sk = i % kKSt;
      if (i >= kKSt)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars[kKEmpty + sk], ((i / kKSt) - 1) & 1, abort_flag));
      if (!ok) break;
      if (leader) {
        uint8_t* dk = sm + Lay::kOffK + sk * kTileBytes;
        mbar_arrive_expect_tx(&bars[kKFull + sk], kTileBytes);
        const int kv_ext = carried ? p.carry_rows : p.kv_rows;
        tma_load_3d_chk(11, dk, mK, &bars[kKFull + sk], 0, row, bh, kHD, kv_ext, gridDim.z);
        tma_load_3d_chk(11, dk + kTok * 128, mK, &bars[kKFull + sk], 64, row, bh, kHD, kv_ext,
                        gridDim.z);
      }
      __syncwarp();
      ++issued_k;
      if (i >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kVEmpty + s], ((i >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      if (leader) {
        uint8_t* dv = sm + Lay::kOffV + s * kTileBytes;
        mbar_arrive_expect_tx(&bars[kVFull + s], kTileBytes);
        const int kv_ext = carried ? p.carry_rows : p.kv_rows;
        tma_load_3d_chk(12, dv, mV, &bars[kVFull + s], 0, row, bh, kHD, kv_ext, gridDim.z);
        tma_load_3d_chk(12, dv + kTok * 128, mV, &bars[kVFull + s], 64, row, bh, kHD, kv_ext,
                        gridDim.z);
      }
      __syncwarp();
      ++issued_v;
    }
    if (!ok) {
      for (int i = max(0, issued_k - kKSt); i < issued_k; ++i)
        mbar_wait_drain(&bars[kKFull + i % kKSt], (i / kKSt) & 1);
      for (int i = max(0, issued_v - 2); i < issued_v; ++i)
        mbar_wait_drain(&bars[kVFull + (i & 1)], (i >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---- MMA issuer ----
    const CompactW cw = compact_w(kFD, kHD, p.G);
    const uint32_t id_u = idesc_bf16(kTok, cw.NT, false, false);  // K (K-major) x compact Wbd
    const uint32_t id_s = idesc_bf16(kFD, kHD, true, true);     // phi^T (MN) x V (MN)
    const uint32_t id_z = idesc_bf16(kFD, 16, true, false);     // phi^T (MN) x ones (K)
    auto wait = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, abort_flag));
    };
    auto issue_fold = [&](int i) {  // dS, dZ += tile i (phi and V in stage i & 1)
      if (leader) {
        const uint32_t vb = sV0 + (i & 1) * kTileBytes;
        const uint32_t pb = sPhi + (i & 1) * kTileBytes;
        for (int kk = 0; kk < kTok / 16; ++kk) {
          const uint64_t a = mnmajor_desc(pb, kk);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tmem + kColDS, a, mnmajor_desc(vb, kk), id_s, acc);
          // ones: SBO = 0 so both 8-row groups of the 16 B rows read the same 1 KiB
          mma_ss(tmem + kColDZ, a, sdesc_sw128(sOnes + (kk & 3) * 32, 16, 0), id_z, acc);
        }
        mma_commit(&bars[kPhiEmpty + (i & 1)]);
        mma_commit(&bars[kVEmpty + (i & 1)]);
      }
      __syncwarp();
    };
    bool ok = true;
    const int ks_per_tile = cw.KT / 16;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int s = i & 1, sk = i % kKSt;
      ok = wait(kKFull + sk, (i / kKSt) & 1);
      if (ok && i >= 2) ok = wait(kUEmpty + s, ((i >> 1) - 1) & 1);
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint32_t kb = sK0 + sk * kTileBytes;
        for (int part = 0; part < 2; ++part) {
          const uint32_t wb = sW0 + part * Lay::kWPart;
          for (int kk = 0; kk < kHD / 16; ++kk) {
            // tile t of the compact W fills U's columns [t NT, (t+1) NT)
            const int t = kk / ks_per_tile, ks = kk - t * ks_per_tile;
            mma_ss(tmem + s * 128 + t * cw.NT, kmajor_desc(kb, kk),
                   sdesc_sw128(wb + (kk >> 2) * (cw.NT * 128) + (kk & 3) * 32, 16, 1024), id_u,
                   (part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(&bars[kUFull + s]);
        mma_commit(&bars[kKEmpty + sk]);
      }
      __syncwarp();
      if (i >= 1) {
        const int ip = i - 1;
        ok = wait(kPhiFull + (ip & 1), (ip >> 1) & 1) && wait(kVFull + (ip & 1), (ip >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        issue_fold(i - 1);
      }
    }
    if (ok) {
      const int i = n_tiles - 1;
      ok = wait(kPhiFull + (i & 1), (i >> 1) & 1) && wait(kVFull + (i & 1), (i >> 1) & 1);
      if (ok) {
        tc_fence_after();
        issue_fold(i);
      }
    }
    if (leader) mma_commit(&bars[kDone]);
    __syncwarp();
    mbar_wait_drain(&bars[kDone], 0);
    __syncwarp();
  } else {
    // ---- feature-map warps: token row r = TMEM lane, feature quarter hf ----
    const int r = tid & 127, hf = tid >> 7;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t col0 = hf * 32;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kUFull + s], (i >> 1) & 1, abort_flag));
      if (ok && i >= 2)  // the fold of tile i - 2 has read this phi stage
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kPhiEmpty + s], ((i >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint8_t* prow = sm + Lay::kOffPhi + s * kTileBytes;
      const int ti = t_begin + i;
      const bool valid = ti < n_seg ? ti * kTok + r < seg : r0 + seg + (ti - n_seg) * kTok + r < r1;
#pragma unroll 1
      for (int c16 = 0; c16 < 2; ++c16) {  // 16 features per step keeps the loop body small
        const int f0 = col0 + c16 * 16;
        uint32_t uu[16];
        tmem_ld16(tmem + lane_base + s * 128 + f0, uu);
        uint32_t packed[8];
        phi16(uu, f0, sB, sPw, valid ? 1.f : 0.f, packed);
        *reinterpret_cast<uint4*>(prow + sw128_offset(r, f0, kTok)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
        *reinterpret_cast<uint4*>(prow + sw128_offset(r, f0 + 8, kTok)) =
            make_uint4(packed[4], packed[5], packed[6], packed[7]);
      }
      tc_fence_before();
      mbar_arrive(&bars[kUEmpty + s]);
      fence_async_smem();
      mbar_arrive(&bars[kPhiFull + s]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kDone], 0, abort_flag));
    // the partial slot (grid (splits, n_fold, BH)) lies inside dS / dZ
    if (ok && !bounds_ok(13, ((long long)bh * p.n_fold + fc) * p.splits + split, 0,
                         (long long)gridDim.z * p.n_fold * p.splits))
      ok = false;
    if (ok) {
      tc_fence_after();
      // lane r of TMEM is feature f = r: dS row f (this thread writes columns col0 .. col0+31),
      // dZ in column kColDZ.
      float* srow = dS + (size_t)r * kHD + col0;
      uint32_t rr[32];
      tmem_ld32(tmem + lane_base + kColDS + col0, rr);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        *reinterpret_cast<float4*>(srow + q4 * 4) =
            make_float4(__uint_as_float(rr[q4 * 4]), __uint_as_float(rr[q4 * 4 + 1]),
                        __uint_as_float(rr[q4 * 4 + 2]), __uint_as_float(rr[q4 * 4 + 3]));
      if (hf == 0) {  // warps 0-3
        uint32_t z16[16];
        tmem_ld16(tmem + lane_base + kColDZ, z16);
        dZ[r] = __uint_as_float(z16[0]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpProducer) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  grid_dep_wait();
}

// Exclusive prefix over fold ranges.  grid (F/32 * D/32, BH), block (32, 8).
//   acc starts at the sum of the n_prefix states S0[i]/Z0[i] (i in order; S0 [n_prefix][BH][F][D],
//   Z0 [n_prefix][BH][F]; none if S0 is null) else 0; for c in 0..C-1: emit state c, then add
//   fold c.
//   St  [BH][C][D][F] bf16 (transposed), Zc [BH][C][F] fp32, S_out [BH][C][F][D] fp32 (opt).
__global__ void __launch_bounds__(256) state_scan_kernel(
    const float* __restrict__ dS, const float* __restrict__ dZ, int n_fold, int splits, int C,
    int F, int D, const float* __restrict__ S0, const float* __restrict__ Z0, int n_prefix,
    __nv_bfloat16* __restrict__ St, float* __restrict__ Zc, float* __restrict__ S_out,
    float* __restrict__ Z_out) {
  // a phi_q kernel launched behind this one (it reads none of this kernel's outputs) may start
  // at once; it waits for this grid before it exits
  grid_dep_signal();
  __shared__ float tile[32][33];
  const int bh = blockIdx.y;
  const int tiles_d = D / 32;
  const int f0 = (blockIdx.x / tiles_d) * 32, d0 = (blockIdx.x % tiles_d) * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  float acc[4];
  float accz = 0.f;
  const bool z_thread = (d0 == 0 && ty == 0);
  const int BH = gridDim.y;
  const int np = S0 ? n_prefix : 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = 0.f;
  for (int r = 0; r < np; ++r) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int f = f0 + ty + 8 * i;
      acc[i] += S0[(((size_t)r * BH + bh) * F + f) * D + d0 + tx];
    }
    if (z_thread && Z0) accz += Z0[((size_t)r * BH + bh) * F + f0 + tx];
  }
  for (int c = 0; c < C; ++c) {
    // this chunk's fold partials are loaded first, so their latency overlaps the stores below
    float add[4] = {0.f, 0.f, 0.f, 0.f};
    float addz = 0.f;
    if (c < n_fold) {
      for (int s = 0; s < splits; ++s) {
        const size_t base = (((size_t)bh * n_fold + c) * splits + s);
#pragma unroll
        for (int i = 0; i < 4; ++i) add[i] += dS[(base * F + f0 + ty + 8 * i) * D + d0 + tx];
        if (z_thread) addz += dZ[base * F + f0 + tx];
      }
    }
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
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += add[i];
    accz += addz;
  }
}

// S_tot[bh] = sum over the n partial slabs dS[bh][0..n) (n = folds x splits), Z_tot likewise:
// one segment's fold total.  grid (ceil(F*D/256), BH), block 256.
__global__ void __launch_bounds__(256) state_sum_kernel(const float* __restrict__ dS,
                                                        const float* __restrict__ dZ, int n,
                                                        int F, int D, float* __restrict__ S_tot,
                                                        float* __restrict__ Z_tot) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e < F * D) {
    float a = 0.f;
    for (int s = 0; s < n; ++s) a += dS[((size_t)bh * n + s) * F * D + e];
    S_tot[(size_t)bh * F * D + e] = a;
  }
  if (e < F) {
    float z = 0.f;
    for (int s = 0; s < n; ++s) z += dZ[((size_t)bh * n + s) * F + e];
    Z_tot[(size_t)bh * F + e] = z;
  }
}

// Element e of (b, h) bh: S[bh] += sum_s dS[bh][0][s], Z likewise.
__device__ __forceinline__ void state_add_element(const float* __restrict__ dS,
                                                  const float* __restrict__ dZ, int splits, int F,
                                                  int D, float* __restrict__ S,
                                                  float* __restrict__ Z, int bh, int e) {
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

// S[bh] += sum_s dS[bh][0][s], Z likewise.  grid (ceil(F*D/256), BH), block 256.
__global__ void __launch_bounds__(256) state_add_kernel(const float* __restrict__ dS,
                                                        const float* __restrict__ dZ, int splits,
                                                        int F, int D, float* __restrict__ S,
                                                        float* __restrict__ Z) {
  state_add_element(dS, dZ, splits, F, D, S, Z, blockIdx.y, blockIdx.x * 256 + threadIdx.x);
}

// The streaming step's closing launch: the state add above (blocks [0, n_add)) and the next
// carry of K and V (the remaining blocks): per (b, h), n_vec 16-byte vectors from
// src[bh * src_stride + src_off ..] to dst[bh * n_vec ..], K then V.  grid (n_add + n_copy, BH),
// block 256.  The carry copy reads the chunk, which the attention and the fold read too; it
// writes the carry, which they read as well, so it must run after both (stream order).
struct CarryCopy {
  const uint4* k_src;
  const uint4* v_src;
  uint4* k_dst;
  uint4* v_dst;
  long long src_stride, src_off, n_vec;  // in 16-byte vectors
};

__global__ void __launch_bounds__(256) state_add_carry_kernel(const float* __restrict__ dS,
                                                              const float* __restrict__ dZ,
                                                              int splits, int F, int D,
                                                              float* __restrict__ S,
                                                              float* __restrict__ Z, int n_add,
                                                              const CarryCopy cc) {
  const int bh = blockIdx.y;
  if ((int)blockIdx.x < n_add) {
    state_add_element(dS, dZ, splits, F, D, S, Z, bh, blockIdx.x * 256 + threadIdx.x);
    return;
  }
  const long long stride = (long long)(gridDim.x - n_add) * 256;
  for (long long i = (long long)(blockIdx.x - n_add) * 256 + threadIdx.x; i < 2 * cc.n_vec;
       i += stride) {
    const bool is_v = i >= cc.n_vec;
    const long long j = is_v ? i - cc.n_vec : i;
    const uint4* src = is_v ? cc.v_src : cc.k_src;
    uint4* dst = is_v ? cc.v_dst : cc.k_dst;
    dst[bh * cc.n_vec + j] = src[bh * cc.src_stride + cc.src_off + j];
  }
}

}  // namespace state
}  // namespace rehyat
