// Fused softmax-window backward of the hybrid attention, FlashAttention style: the scores of a
// (query tile, key tile) pair are recomputed in TMEM and never reach memory.  With the forward's
// row statistics (lse2 = log2 of the row denominator, D = dO . O, both [BH][N] fp32):
//   P = 2^(q.k log2(e)/sqrt(D) - lse2),   dS = P (dO . v - D) / sqrt(D)
//   dV += P^T dO,  dK += dS^T Q          (dkdv_kernel: one CTA per key tile of a chunk's window,
//                                          looping over the chunk's query tiles)
//   dQ += dS K                           (dq_kernel: one CTA per query tile, looping over the
//                                          window's key tiles)
// The derivative is that of the "ReHyAt overview" page's §2.2.1 output formula; the linear
// terms' gradients are separate (backward.cuh and tensor-core products).
//
// Both kernels: 320 threads.  Warps 0-7 compute: warp w owns TMEM lanes 32 (w % 4) .. + 31 (one
// row per thread) and the column half w / 4 (64 of the 128 score columns), so two warps share
// each SM sub-partition's work; warp 8 loads by TMA (and allocates TMEM), warp 9 issues the MMAs.
// Per loop step the MMA warp issues the two score products (S and dP, SS), the compute warps turn
// them into packed bf16 P / dS written back over the scores in TMEM (half h's 64 columns pack into
// TMEM columns [64 h, 64 h + 32), inside its own half, so the two halves never touch each other's
// scores), and the MMA warp issues the products that use them as the A operand (TS), whose K16
// step kk reads packed column 64 (kk / 4) + 8 (kk % 4).  Launch once per chunk (keys of the
// overlap frames belong to two chunks' windows; the launches' += on dK, dV are ordered by the
// stream).
#pragma once

#include "attn_bf16.cuh"
#include "sm100.cuh"

namespace rehyat {
namespace attn_bwd {

using namespace sm100;
using attn::kmajor_desc;
using attn::mnmajor_desc;

// Two probabilities and two dS values from two (score, dP) pairs, on paired fp32 instructions:
// p = 2^(s scale - lse2), g = (p / sqrt(D)) (dP - D).  neg_l2 and neg_d hold -lse2 and -D.
__device__ __forceinline__ void grad_pair(uint32_t s0, uint32_t s1, uint32_t d0, uint32_t d1,
                                          uint64_t sl2x2, uint64_t neg_l2, uint64_t neg_d,
                                          uint64_t isd2, uint32_t& pp, uint32_t& gg) {
  const uint64_t x = f2_fma(f2_pack(__uint_as_float(s0), __uint_as_float(s1)), sl2x2, neg_l2);
  float xa, xb;
  f2_unpack(x, xa, xb);
  const uint64_t pr = f2_pack(ex2(xa), ex2(xb));
  const uint64_t t = f2_add(f2_pack(__uint_as_float(d0), __uint_as_float(d1)), neg_d);
  const uint64_t g = f2_mul(f2_mul(pr, isd2), t);
  float pa, pb, ga, gb;
  f2_unpack(pr, pa, pb);
  f2_unpack(g, ga, gb);
  pp = pack_bf16x2(pa, pb);
  gg = pack_bf16x2(ga, gb);
}

constexpr int kThreads = 320;
constexpr int kCompute = 256;  // compute threads (warps 0-7)

// TMEM column of the packed bf16 A operand for the K16 step kk (see above).
__device__ __forceinline__ uint32_t packed_col(int kk) { return (kk >> 2) * 64 + (kk & 3) * 8; }
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 bf16 tile (two 128 x 64 boxes)
constexpr uint32_t kStatBytes = 2 * 128 * 4;

struct Params {
  int L, T, Tc, To, c;   // frames per chunk etc.; c = the chunk of this launch
  int N;                 // rows per (b, h)
  const float* lse2;     // [BH][N]
  const float* Drow;     // [BH][N]
  float scale_log2, inv_sqrt_d;
  float* dq;             // [BH][N][D] fp32, +=
  float* dk;
  float* dv;
};

struct Geometry {
  int q_row0, nq, k_row0, nw;
};

__device__ __forceinline__ Geometry geometry(const Params& p) {
  const int s = p.c * p.Tc;
  const int e = min(s + p.Tc, p.T);
  const int w = max(0, s - p.To);
  return Geometry{s * p.L, (e - s) * p.L, w * p.L, (e - w) * p.L};
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                          int row, int bh) {
  tma_load_3d(dst, map, bar, 0, row, bh);
  tma_load_3d(dst + 128 * 128, map, bar, 64, row, bh);
}

// Load 32 consecutive columns at each of two TMEM addresses with one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t (&a)[32], uint32_t tb,
                                            uint32_t (&b)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, "
      "%41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, "
      "%58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : REHYAT_R32(a, 0), REHYAT_R32(b, 0)
      : "r"(ta), "r"(tb)
      : "memory");
}
// TMA tile reduce-add of one 3-D box of fp32 from shared memory (128B-swizzled) into the tensor:
// every element is added to global memory; the parts of the box past the tensor's extents are
// not touched.  Tracked by this thread's bulk async-groups like tma_store_3d.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int c0,
                                                  int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// tma_reduce_add_3d of an fp32 tensor with, in debug-bounds builds, the inner coordinate a
// multiple of 4 elements (16 bytes) inside the row and the row and depth coordinates inside the
// tensor; a failed check is recorded and the reduction skipped.
__device__ __forceinline__ void tma_reduce_add_3d_chk(int site, const CUtensorMap* map,
                                                      const void* src, int c0, int c1, int c2,
                                                      long long ext0, long long ext1,
                                                      long long ext2) {
#ifdef REHYAT_DEBUG_BOUNDS
  const bool ok = bounds_ok(site, c0 & 3, 0, 1) & bounds_ok(site, c0, 0, ext0) &
                  bounds_ok(site, c1, 0, ext1) & bounds_ok(site, c2, 0, ext2);
  if (!ok) return;
#else
  (void)site, (void)ext0, (void)ext1, (void)ext2;
#endif
  tma_reduce_add_3d(map, src, c0, c1, c2);
}
// Writes 32 fp32 values (TMEM words; zeros when !keep) as row r of a [128 rows][32 fp32] box in the
// 128B-swizzled layout of an fp32 TMA tile (16-byte chunk j of the row at position j ^ (r % 8)).
__device__ __forceinline__ void stage_row32(uint8_t* box, int r, const uint32_t* v, bool keep) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 x = keep ? make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                        __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(box + r * 128 + ((j ^ (r & 7)) * 16)) = x;
  }
}

// ------------------------------------------------------------------------------------------
// dK, dV: CTA = one 128-key tile of chunk c's window; loop over the chunk's query tiles.
// TMEM: S^T [0,128) -> P^T, dP^T [128,256) -> dS^T, dV [256,384), dK [384,512).
// smem: K, V (resident), Q and dO in 2 stages, the query tiles' lse2 and D in 2 stages.
// ------------------------------------------------------------------------------------------
constexpr uint32_t kKOffK = 0, kKOffV = kTile, kKOffQ = 2 * kTile, kKOffO = 4 * kTile;
constexpr uint32_t kKOffStat = 6 * kTile;
constexpr uint32_t kKSmem = kKOffStat + 2 * kStatBytes + 1024;
enum KBar { kKvFull = 0, kQFull = 1, kQEmpty = 3, kSdFull = 5, kPdFull = 6, kKDone = 7, kKBars = 8 };

// grid (ceil(nw / 128), 1, BH)
__global__ void __launch_bounds__(kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                const Params p) {
  static_assert(kKSmem + 256 <= 232448, "shared memory over the limit");
  const Geometry g = geometry(p);
  const int bh = blockIdx.z;
  const int key0 = blockIdx.x * 128;  // within the window
  if (key0 >= g.nw) return;
  const int n_q = (g.nq + 127) / 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[kKBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 8) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kKBars; ++i) mbar_init(&bars[i], i == kPdFull ? kCompute : 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  float* sStat = reinterpret_cast<float*>(sm + kKOffStat);  // [stage][lse 128 | D 128]

  if (warp == 8) {
    // ---- producer ----
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmO);
      mbar_arrive_expect_tx(&bars[kKvFull], 2 * kTile);
      load_tile(sm + kKOffK, &tmK, &bars[kKvFull], g.k_row0 + key0, bh);
      load_tile(sm + kKOffV, &tmV, &bars[kKvFull], g.k_row0 + key0, bh);
    }
    __syncwarp();
    bool ok = true;
    int issued = 0;
    for (int i = 0; i < n_q; ++i) {
      const int s = i & 1;
      if (i >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kQEmpty + s], ((i >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      // the query tile's statistics; rows past the chunk get lse2 = +inf, so P = dS = 0 there
      float* st = sStat + s * 256;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int qi = i * 128 + lane * 4 + t;
        const bool valid = qi < g.nq;
        const long long idx = (long long)bh * p.N + g.q_row0 + (valid ? qi : 0);
        st[lane * 4 + t] = valid ? -p.lse2[idx] : -INFINITY;  // negated for the FMA
        st[128 + lane * 4 + t] = valid ? -p.Drow[idx] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[kQFull + s], 2 * kTile);
        load_tile(sm + kKOffQ + s * kTile, &tmQ, &bars[kQFull + s], g.q_row0 + i * 128, bh);
        load_tile(sm + kKOffO + s * kTile, &tmO, &bars[kQFull + s], g.q_row0 + i * 128, bh);
      }
      __syncwarp();
      ++issued;
    }
    if (!ok) {
      mbar_wait_drain(&bars[kKvFull], 0);
      for (int i = max(0, issued - 2); i < issued; ++i)
        mbar_wait_drain(&bars[kQFull + (i & 1)], (i >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---- MMA issuer ----
    const uint32_t id_ss = idesc_bf16(128, 128, false, false);
    const uint32_t id_ts = idesc_bf16(128, 128, false, true);
    const uint32_t sK = smem_u32(sm + kKOffK), sV = smem_u32(sm + kKOffV);
    auto wait = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, abort_flag));
    };
    bool ok = wait(kKvFull, 0);
    for (int i = 0; i < n_q && ok; ++i) {
      const int s = i & 1;
      const uint32_t sQ = smem_u32(sm + kKOffQ + s * kTile), sO = smem_u32(sm + kKOffO + s * kTile);
      ok = wait(kQFull + s, (i >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        for (int kk = 0; kk < 8; ++kk)  // S^T = K Q^T
          mma_ss(tmem, kmajor_desc(sK, kk), kmajor_desc(sQ, kk), id_ss, kk > 0 ? 1u : 0u);
        for (int kk = 0; kk < 8; ++kk)  // dP^T = V dO^T
          mma_ss(tmem + 128, kmajor_desc(sV, kk), kmajor_desc(sO, kk), id_ss, kk > 0 ? 1u : 0u);
        mma_commit(&bars[kSdFull]);
      }
      __syncwarp();
      ok = wait(kPdFull, i & 1);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        for (int kk = 0; kk < 8; ++kk)  // dV += P^T dO
          mma_ts(tmem + 256, tmem + packed_col(kk), mnmajor_desc(sO, kk), id_ts,
                 (i > 0 || kk > 0) ? 1u : 0u);
        for (int kk = 0; kk < 8; ++kk)  // dK += dS^T Q
          mma_ts(tmem + 384, tmem + 128 + packed_col(kk), mnmajor_desc(sQ, kk), id_ts,
                 (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[kQEmpty + s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&bars[kKDone]);
    __syncwarp();
    mbar_wait_drain(&bars[kKDone], 0);
    __syncwarp();
  } else {
    // ---- compute: thread = key row r of the tile, column half hc ----
    const int r = tid & 127, hc = tid >> 7;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base, tD = tmem + lane_base + 128;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t isd2 = f2_pack(p.inv_sqrt_d, p.inv_sqrt_d);
    bool ok = true;
    for (int i = 0; i < n_q; ++i) {
      const int s = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kSdFull], i & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // -lse2 and -D of the tile's 128 queries, read four at a time (same address in every lane)
      const float4* nl4 = reinterpret_cast<const float4*>(sStat + s * 256);
      const float4* nd4 = nl4 + 32;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = hc * 2 + cc;  // 32-column chunk of the scores
        uint32_t sv[32], dv[32];
        tmem_ld32x2(tS + c * 32, sv, tD + c * 32, dv);
        uint32_t pp[16], gg[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 nl = nl4[c * 8 + e4], nd = nd4[c * 8 + e4];
          grad_pair(sv[4 * e4], sv[4 * e4 + 1], dv[4 * e4], dv[4 * e4 + 1], sl2x2,
                    f2_pack(nl.x, nl.y), f2_pack(nd.x, nd.y), isd2, pp[2 * e4], gg[2 * e4]);
          grad_pair(sv[4 * e4 + 2], sv[4 * e4 + 3], dv[4 * e4 + 2], dv[4 * e4 + 3], sl2x2,
                    f2_pack(nl.z, nl.w), f2_pack(nd.z, nd.w), isd2, pp[2 * e4 + 1],
                    gg[2 * e4 + 1]);
        }
        // packed columns [64 hc + 16 cc, + 16): this half's first chunk, already read
        tmem_st16(tS + hc * 64 + cc * 16, pp);
        tmem_st16(tD + hc * 64 + cc * 16, gg);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[kPdFull]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kKDone], 0, abort_flag)) && !*abort_flag;
    // dV and dK are added into global memory by TMA reduce-adds of four 32-column fp32 boxes
    // each, staged in the Q and dO stages (free: every MMA is complete); rows past the window add
    // zeros.
    if (ok) {
      tc_fence_after();
      const bool row_ok = key0 + r < g.nw;
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        const int cc = hc * 2 + c2;
        uint32_t a[32], b[32];
        tmem_ld32x2(tmem + lane_base + 256 + cc * 32, a, tmem + lane_base + 384 + cc * 32, b);
        stage_row32(sm + kKOffQ + cc * 16384, r, a, row_ok);
        stage_row32(sm + kKOffO + cc * 16384, r, b, row_ok);
      }
    }
    // every compute thread gets here, whatever its waits returned; after an abort nothing is added
    fence_async_smem();
    named_bar_sync(1, kCompute);
    if (tid == 0 && !*abort_flag) {
      const int row = g.k_row0 + key0;
      for (int cc = 0; cc < 4; ++cc) {
        tma_reduce_add_3d_chk(41, &tmDV, sm + kKOffQ + cc * 16384, cc * 32, row, bh, 128, p.N,
                              gridDim.z);
        tma_reduce_add_3d_chk(41, &tmDK, sm + kKOffO + cc * 16384, cc * 32, row, bh, 128, p.N,
                              gridDim.z);
      }
      bulk_commit_group();
      bulk_wait_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------
// dQ: CTA = one 128-row query tile of chunk c; loop over the window's key tiles.
// TMEM: S [0,128), dP [128,256) -> dS, dQ [256,384).  smem: Q, dO (resident), K and V in 2
// stages.
// ------------------------------------------------------------------------------------------
constexpr uint32_t kQOffQ = 0, kQOffO = kTile, kQOffK = 2 * kTile, kQOffV = 4 * kTile;
constexpr uint32_t kQSmem = 6 * kTile + 1024;
enum QBar { kQoFull = 0, kKFull = 1, kKEmpty = 3, kSFull = 5, kDsFull = 6, kQDone = 7, kQBars = 8 };

// grid (ceil(nq / 128), 1, BH)
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const __grid_constant__ CUtensorMap tmDQ, const Params p) {
  static_assert(kQSmem + 256 <= 232448, "shared memory over the limit");
  const Geometry g = geometry(p);
  const int bh = blockIdx.z;
  const int q0 = blockIdx.x * 128;  // within the chunk
  if (q0 >= g.nq) return;
  const int n_k = (g.nw + 127) / 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[kQBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 8) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kQBars; ++i) mbar_init(&bars[i], i == kDsFull ? kCompute : 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 8) {
    // ---- producer ----
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bars[kQoFull], 2 * kTile);
      load_tile(sm + kQOffQ, &tmQ, &bars[kQoFull], g.q_row0 + q0, bh);
      load_tile(sm + kQOffO, &tmO, &bars[kQoFull], g.q_row0 + q0, bh);
    }
    __syncwarp();
    bool ok = true;
    int issued = 0;
    for (int j = 0; j < n_k; ++j) {
      const int s = j & 1;
      if (j >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kKEmpty + s], ((j >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[kKFull + s], 2 * kTile);
        load_tile(sm + kQOffK + s * kTile, &tmK, &bars[kKFull + s], g.k_row0 + j * 128, bh);
        load_tile(sm + kQOffV + s * kTile, &tmV, &bars[kKFull + s], g.k_row0 + j * 128, bh);
      }
      __syncwarp();
      ++issued;
    }
    if (!ok) {
      mbar_wait_drain(&bars[kQoFull], 0);
      for (int j = max(0, issued - 2); j < issued; ++j)
        mbar_wait_drain(&bars[kKFull + (j & 1)], (j >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---- MMA issuer ----
    const uint32_t id_ss = idesc_bf16(128, 128, false, false);
    const uint32_t id_ts = idesc_bf16(128, 128, false, true);
    const uint32_t sQ = smem_u32(sm + kQOffQ), sO = smem_u32(sm + kQOffO);
    auto wait = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, abort_flag));
    };
    bool ok = wait(kQoFull, 0);
    for (int j = 0; j < n_k && ok; ++j) {
      const int s = j & 1;
      const uint32_t sK = smem_u32(sm + kQOffK + s * kTile), sV = smem_u32(sm + kQOffV + s * kTile);
      ok = wait(kKFull + s, (j >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        for (int kk = 0; kk < 8; ++kk)  // S = Q K^T
          mma_ss(tmem, kmajor_desc(sQ, kk), kmajor_desc(sK, kk), id_ss, kk > 0 ? 1u : 0u);
        for (int kk = 0; kk < 8; ++kk)  // dP = dO V^T
          mma_ss(tmem + 128, kmajor_desc(sO, kk), kmajor_desc(sV, kk), id_ss, kk > 0 ? 1u : 0u);
        mma_commit(&bars[kSFull]);
      }
      __syncwarp();
      ok = wait(kDsFull, j & 1);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        for (int kk = 0; kk < 8; ++kk)  // dQ += dS K
          mma_ts(tmem + 256, tmem + 128 + packed_col(kk), mnmajor_desc(sK, kk), id_ts,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[kKEmpty + s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&bars[kQDone]);
    __syncwarp();
    mbar_wait_drain(&bars[kQDone], 0);
    __syncwarp();
  } else {
    // ---- compute: thread = query row r of the tile, column half hc ----
    const int r = tid & 127, hc = tid >> 7;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base, tD = tmem + lane_base + 128;
    const bool row_ok = q0 + r < g.nq;
    const long long row = (long long)bh * p.N + g.q_row0 + q0 + r;
    const float l2 = row_ok ? p.lse2[row] : INFINITY;
    const float Di = row_ok ? p.Drow[row] : 0.f;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t isd2 = f2_pack(p.inv_sqrt_d, p.inv_sqrt_d);
    const uint64_t neg_l2 = f2_pack(-l2, -l2), neg_d = f2_pack(-Di, -Di);
    bool ok = true;
    for (int j = 0; j < n_k; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kSFull], j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int valid = g.nw - j * 128;  // key columns of this tile inside the window
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = hc * 2 + cc;
        uint32_t sv[32], dv[32];
        tmem_ld32x2(tS + c * 32, sv, tD + c * 32, dv);
        uint32_t gg[16], pp;
        if (valid < 128) {  // the window's last key tile: keys past the window get dS = 0
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e >= valid) sv[e] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e)
          grad_pair(sv[2 * e], sv[2 * e + 1], dv[2 * e], dv[2 * e + 1], sl2x2, neg_l2, neg_d,
                    isd2, pp, gg[e]);
        tmem_st16(tD + hc * 64 + cc * 16, gg);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[kDsFull]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kQDone], 0, abort_flag)) && !*abort_flag;
    // dQ is added into global memory by TMA reduce-adds of four 32-column fp32 boxes, staged in
    // the K stages (free: every MMA is complete); rows past the chunk add zeros.
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        const int cc = hc * 2 + c2;
        uint32_t a[32];
        tmem_ld32(tmem + lane_base + 256 + cc * 32, a);
        stage_row32(sm + kQOffK + cc * 16384, r, a, row_ok);
      }
    }
    // every compute thread gets here, whatever its waits returned; after an abort nothing is added
    fence_async_smem();
    named_bar_sync(1, kCompute);
    if (tid == 0 && !*abort_flag) {
      for (int cc = 0; cc < 4; ++cc)
        tma_reduce_add_3d_chk(42, &tmDQ, sm + kQOffK + cc * 16384, cc * 32, g.q_row0 + q0, bh, 128,
                              p.N, gridDim.z);
      bulk_commit_group();
      bulk_wait_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn_bwd
}  // namespace rehyat
