// Feature map phi of the "ReHyAt overview" page §2.2.2 for many bf16 rows, on the tensor cores:
// u = x Wbd^T (the grouped 1x1 linear as the compact block-diagonal matrix of featmap.cuh, bf16 hi
// + lo parts built in shared memory from the fp32 weights, fp32 in TMEM) by tcgen05, then bias,
// softplus and the part powers on the CUDA cores, written as bf16 rows.  Used for phi_q of the
// query rows that read a linear state, so that the attention kernel's epilogue only has to load
// a finished phi_q tile.  The output leaves by TMA stores from shared memory: the feature-map
// warps write a tile's phi over the X stage that its MMA has consumed, the producer stores it
// and refills the stage once the store has read it.
#pragma once

#include "featmap.cuh"
#include "sm100.cuh"

namespace rehyat {
namespace phi {

using namespace sm100;

constexpr int kRows = 128;  // rows per tile (MMA M)
constexpr int kHD = 128;
constexpr int kFD = 128;
constexpr int kThreads = 320;  // warps 0-7 feature map, 8 producer, 9 MMA
constexpr int kPhiThreads = 256;
constexpr int kTileBytes = kRows * kHD * 2;

// Shared memory of the instance for G >= 2 (compact weights of at most 64 rows: 16 KB per part;
// two CTAs per SM) or for G = 1 (the full 128 x 128 matrix: 32 KB per part; one CTA per SM).
template <bool kDense>
struct Layout {
  static constexpr uint32_t kWPart = kDense ? 32768 : 16384;
  static constexpr uint32_t kOffX = 0;                          // 2 stages
  static constexpr uint32_t kOffW = kOffX + 2 * kTileBytes;      // compact W: hi, then lo
  static constexpr uint32_t kOffB = kOffW + 2 * kWPart;          // bias, F fp32
  static constexpr uint32_t kOffPw = kOffB + kFD * 4;            // part power of each feature
  static constexpr uint32_t kSmemBytes = kOffPw + kFD + 1024;    // + alignment slack
  static constexpr int kCtasPerSm = kDense ? 1 : 2;
};

// kOutFull: a tile's phi is in its X stage (256 arrivals); the stage is free again once the
// producer's store of it has read it.
enum Bar { kXFull = 0, kOutFull = 2, kUFull = 4, kUEmpty = 6, kDone = 8, kNumBars = 9 };

struct Params {
  int row0;           // first row (of each (b, h) sequence) to map
  int n_rows;         // rows to map, starting at row0
  int rows_per_bh;    // rows of each (b, h) in x and phi
  int tiles_per_cta;  // 128-row tiles per CTA (blockIdx.x picks a run of them)
  int H, P, G;
  const float* W;     // [H, G, F/G, D/G] fp32
  const float* bias;  // [H, F] or null
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// grid (ceil(n_tiles / tiles_per_cta), BH), block 320.  Feature-map thread tid owns row
// (tid & 127) = TMEM lane and features [64 (tid >> 7), +64).  tmX reads x [BH, rows_per_bh, D];
// tmPhi writes phi [BH, rows_per_bh, F] with its row extent cut at row0 + n_rows, so that the
// rows of a ragged last tile past the range are not written.
template <bool kDense>
__global__ void __launch_bounds__(kThreads, Layout<kDense>::kCtasPerSm)
    featmap_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmPhi, const Params p) {
  using Lay = Layout<kDense>;
  static_assert(Lay::kSmemBytes + 256 <= 232448 / Lay::kCtasPerSm,
                "shared memory (dynamic + static) over the limit");
  // the attention launched behind this kernel may start at once: it reads phi_q only after
  // waiting for this grid.  Launched itself behind the library's state scan, this kernel waits for
  // that grid before it exits, so that its completion implies the scan's.
  grid_dep_signal();
  const int bh = blockIdx.y, h = bh % p.H;
  const int n_tiles_all = (p.n_rows + kRows - 1) / kRows;
  const int t_begin = blockIdx.x * p.tiles_per_cta;
  const int n_tiles = min(p.tiles_per_cta, n_tiles_all - t_begin);
  if (n_tiles <= 0) {
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
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 8) {
    tmem_alloc(&tmem_base_sh, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(&bars[i], (i == kUEmpty || i == kUEmpty + 1 || i == kOutFull || i == kOutFull + 1)
                              ? kPhiThreads
                              : 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < kFD; i += kThreads) {
    sB[i] = p.bias ? p.bias[(size_t)h * kFD + i] : 0.f;
    sPw[i] = static_cast<uint8_t>(feature_power(i, kFD, p.P));
  }
  build_compact_w(p.W + (size_t)h * kFD * kHD / p.G, kFD, kHD, p.G, sm + Lay::kOffW,
                  sm + Lay::kOffW + Lay::kWPart, tid, kThreads);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const bool leader = lane == 0;

  if (warp == 8) {
    // ---- producer: loads of x, stores of phi ----
    if (leader) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmPhi);
    }
    __syncwarp();
    bool ok = true;
    int issued = 0;
    const long long out_rows = (long long)p.row0 + p.n_rows;
    // phi of tile j goes out from X stage j & 1; the stage is reusable once the store read it
    auto store_tile = [&](int j) {
      const int s = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kOutFull + s], (j >> 1) & 1, abort_flag));
      if (!ok) return;
      if (leader) {
        const uint8_t* src = sm + Lay::kOffX + s * kTileBytes;
        const int row = p.row0 + (t_begin + j) * kRows;
        tma_store_3d_chk(23, &tmPhi, src, 0, row, bh, kFD, out_rows, gridDim.y);
        tma_store_3d_chk(23, &tmPhi, src + kRows * 128, 64, row, bh, kFD, out_rows, gridDim.y);
        bulk_commit_group();
        bulk_wait_read_all();
      }
      __syncwarp();
    };
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i & 1;
      const int row = p.row0 + (t_begin + i) * kRows;
      if (i >= 2) store_tile(i - 2);
      if (!ok) break;
      if (leader) {
        uint8_t* dx = sm + Lay::kOffX + s * kTileBytes;
        mbar_arrive_expect_tx(&bars[kXFull + s], kTileBytes);
        tma_load_3d_chk(21, dx, &tmX, &bars[kXFull + s], 0, row, bh, kHD, p.rows_per_bh,
                        gridDim.y);
        tma_load_3d_chk(21, dx + kRows * 128, &tmX, &bars[kXFull + s], 64, row, bh, kHD,
                        p.rows_per_bh, gridDim.y);
      }
      __syncwarp();
      ++issued;
    }
    for (int j = max(0, n_tiles - 2); j < n_tiles && ok; ++j) store_tile(j);
    if (leader) bulk_wait_all();  // the stores are complete before the CTA exits
    if (!ok) {
      for (int i = max(0, issued - 2); i < issued; ++i)
        mbar_wait_drain(&bars[kXFull + (i & 1)], (i >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---- MMA issuer: U[s] = X_i Wbd_hi^T + X_i Wbd_lo^T, tile by tile of the compact W (its
    // completion also frees X stage s for the feature-map warps' phi) ----
    const CompactW cw = compact_w(kFD, kHD, p.G);
    const uint32_t id_u = idesc_bf16(kRows, cw.NT, false, false);
    const uint64_t dX0 = sdesc_sw128(smem_u32(sm + Lay::kOffX), 16, 1024);
    const uint64_t dW0 = sdesc_sw128(smem_u32(sm + Lay::kOffW), 16, 1024);
    auto koff = [](int kk, int rows) {
      return (uint64_t)((kk >> 2) * (rows * 128 / 16) + (kk & 3) * 2);
    };
    auto wait = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, abort_flag));
    };
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int s = i & 1;
      ok = wait(kXFull + s, (i >> 1) & 1);
      if (ok && i >= 2) ok = wait(kUEmpty + s, ((i >> 1) - 1) & 1);
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint64_t dx = dX0 + (uint64_t)(s * kTileBytes / 16);
        const int ks_per_tile = cw.KT / 16;
        for (int part = 0; part < 2; ++part) {
          const uint64_t dw = dW0 + (uint64_t)(part * Lay::kWPart / 16);
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const int t = kk / ks_per_tile, ks = kk - t * ks_per_tile;
            mma_ss(tmem + s * 128 + t * cw.NT, dx + koff(kk, kRows), dw + koff(kk, cw.NT), id_u,
                   (part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(&bars[kUFull + s]);
      }
      __syncwarp();
    }
    if (leader) mma_commit(&bars[kDone]);
    __syncwarp();
    mbar_wait_drain(&bars[kDone], 0);
    __syncwarp();
  } else {
    // ---- feature-map warps ----
    const int r = tid & 127, hf = tid >> 7;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int col0 = hf * 64;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kUFull + s], (i >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // the MMA that read X stage s is complete (U_FULL): phi of the tile goes over it, in the
      // 128B-swizzled layout of the store's two 64-feature boxes
      uint8_t* xs = sm + Lay::kOffX + s * kTileBytes;
#pragma unroll 1
      for (int c16 = 0; c16 < 4; ++c16) {
        const int f0 = col0 + c16 * 16;
        uint32_t uu[16];
        tmem_ld16(tmem + lane_base + s * 128 + f0, uu);
        uint32_t packed[8];
        phi16(uu, f0, sB, sPw, 1.f, packed);
        *reinterpret_cast<uint4*>(xs + sw128_offset(r, f0, kRows)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
        *reinterpret_cast<uint4*>(xs + sw128_offset(r, f0 + 8, kRows)) =
            make_uint4(packed[4], packed[5], packed[6], packed[7]);
      }
      tc_fence_before();
      mbar_arrive(&bars[kUEmpty + s]);
      fence_async_smem();
      mbar_arrive(&bars[kOutFull + s]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  grid_dep_wait();
}

}  // namespace phi
}  // namespace rehyat
