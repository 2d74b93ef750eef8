// Fused hybrid attention forward, bf16 in / bf16 out, tcgen05 tensor cores (sm_100a).
//
// One CTA owns two 128-row query tiles of one temporal chunk of one (batch, head) and streams
// the chunk's softmax window (its own frames plus the To frames before it) through shared memory
// in 128-key tiles.  Per key tile j and query tile t:
//     S_t = Q_t K_j^T                          (tcgen05.mma, smem x smem -> TMEM fp32)
//     P_t = exp2(S_t * log2(e)/sqrt(D) - m_t)  (softmax warpgroup t, P written back into TMEM
//                                               over S_t as packed bf16 pairs)
//     O_t += P_t V_j                           (tcgen05.mma, A from TMEM, V MN-major in smem)
// with the running max m_t kept lazily: O_t and l_t are rescaled only when the tile max exceeds
// m_t by more than 8 (a factor 256), so exp2 arguments stay <= 8.
// Epilogue (the hybrid joint normaliser of the "ReHyAt overview" page §2.2.1 and the state
// readout of §2.3), for chunks that have a linear region: the grouped linear of phi_q runs on the
// tensor cores as U_t = Q_t Wbd^T (block-diagonal W in bf16 hi + lo parts, two MMAs into the now
// free S_t columns); the softmax warpgroup turns its U row into phi_q(q) * 2^-m (bias, softplus,
// part powers) and writes it as bf16 over its Q tile in shared memory; one more MMA adds
// phi_q 2^-m . S_c into O_t, and l_t += 2^-m phi_q . Z_c; the output is O_t / l_t.  m starts at
// 0 for chunks that have a linear region, so 2^-m <= 1 and a row can never lose both terms to
// underflow.  A tile whose 128 rows all lie in the chunk is packed as bf16 into its Q tile's
// shared memory and leaves by two TMA stores; a ragged tile's rows are stored one by one.
//
// Warp roles (320 threads): warps 0-3 softmax/epilogue of tile 0, warps 4-7 of tile 1, warp 8
// TMA producer (+ TMEM allocation), warp 9 MMA issuer.  TMEM columns: S_0 [0,128), S_1
// [128,256), O_0 [256,384), O_1 [384,512).
#pragma once

#include "featmap.cuh"
#include "sm100.cuh"

namespace rehyat {
namespace attn {

using namespace sm100;

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kHD = 128;  // head dim D
constexpr int kFD = 128;  // feature dim F
constexpr int kThreads = 320;
constexpr int kTileBytes = kBM * kHD * 2;  // one 128 x 128 bf16 tile

// dynamic shared memory layout (offsets from the 1024-aligned base)
constexpr uint32_t kOffQ0 = 0;
constexpr uint32_t kOffQ1 = kOffQ0 + kTileBytes;
constexpr uint32_t kOffK = kOffQ1 + kTileBytes;       // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;    // 2 stages
constexpr uint32_t kOffB = kOffV + 2 * kTileBytes;    // bias of phi_q, F fp32
constexpr uint32_t kOffZ = kOffB + kFD * 4;            // Z_c, F fp32
constexpr uint32_t kOffPw = kOffZ + kFD * 4;           // part power of each feature, int
constexpr uint32_t kSmemBytes = kOffPw + kFD * 4 + 1024;  // + alignment slack

enum Bar {
  kQFull = 0,
  kKFull = 1,    // 2
  kKEmpty = 3,   // 2
  kVFull = 5,    // 2
  kVEmpty = 7,   // 2
  kSFull = 9,    // 2 (per query tile)
  kPFull = 11,   // 2 (per query tile, 128 arrivals)
  kOFull = 13,   // 2 (per query tile): its last P.V is complete (one phase per CTA)
  kStFull = 15,
  kPhiFull = 16,  // 2 (per query tile, 128 arrivals)
  kRoDone = 18,   // 2
  kMmaDone = 20,
  kWbFull = 21,  // block-diagonal W_q (hi, lo) loaded into the V stages
  kUFull = 22,   // 2 (per query tile): U_t = Q_t Wbd^T complete
  kPhiqFull = 24,  // precomputed phi_q tiles loaded over the Q tiles
  kNumBars = 25
};

struct Params {
  int L;              // tokens per frame
  int T;              // frames of the query sequence
  int Tc, To;         // chunk length, overlap
  int frames_before;  // video frame index of query row 0
  int kv_frame0;      // video frame index of key/value row 0
  int H, P;
  int n_states;       // states per (b, h) in St / Z (state index = chunk index)
  int nq_rows;        // rows per (b, h) of q and out
  // Two-source window (streaming with carried frames): the first kv_split rows of the window come
  // from tmKc/tmVc starting at row carry_row0, the rest from tmK/tmV; each segment is tiled on
  // its own (its last tile ragged).  kv_split = 0: the whole window is in tmK/tmV.
  int kv_split;
  int carry_row0;
  int kv_rows, carry_rows;  // rows per (b, h) of the main and of the carried K/V tensor maps
  float scale_log2;   // log2(e) / sqrt(D)
  const float* bq;    // [H, F] or null
  const float* Z;     // [BH, n_states, F]
  __nv_bfloat16* out; // [BH, nq_rows, D]
  float* lse;         // [BH, nq_rows] or null: log2 of each row's denominator (for the backward)
  // A chunk whose tile count is odd has a lone last tile.  With n_split > 1 that tile's key window
  // is cut into n_split parts, each run by its own (short) CTA, which writes its rows'
  // unnormalised O and (m, l) here instead of the output; lone_combine_kernel merges the parts.
  // Only part 0 adds the linear-state readout.  Slot of (chunk c, bh, part):
  // (c * BH + bh) * n_split + part.  Not combined with lse.
  int n_split;
  float* part_o;      // [chunks * BH * n_split][128][D] fp32
  float* part_ml;     // [chunks * BH * n_split][128][2] fp32: m (log2 units) and l per row
};

// Rows and key window of chunk c of a launch (frames relative to the video).
struct ChunkGeom {
  int q_row0, nq;    // query rows [q_row0, q_row0 + nq) of the q/out buffers
  int k_row0, nk;    // window rows of the main K/V source (after the carried segment)
  bool has_linear;   // the chunk reads a linear state
};
__device__ __forceinline__ ChunkGeom chunk_geom(const Params& p, int c) {
  const int gs = p.frames_before + c * p.Tc;
  const int ge = min(gs + p.Tc, p.frames_before + p.T);
  const int gw = max(0, gs - p.To);
  ChunkGeom g;
  g.q_row0 = (gs - p.frames_before) * p.L;
  g.nq = (ge - gs) * p.L;
  g.k_row0 = (gw - p.kv_frame0) * p.L;
  g.nk = (ge - gw) * p.L;
  g.has_linear = gw > 0;
  return g;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}


// K-major SW128 descriptor of the kk-th 16-wide K step of a 128-row, 128-wide bf16 tile.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_addr, int kk) {
  return sdesc_sw128(tile_addr + (kk >> 2) * (kBM * 128) + (kk & 3) * 32, 16, 1024);
}
// MN-major SW128 descriptor of the kk-th 16-row K step of a [128 rows][128 cols] bf16 tile
// whose columns are the M/N dimension.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_addr, int kk) {
  return sdesc_sw128(tile_addr + kk * 16 * 128, kBM * 128, 1024);
}

// kPhiGlobal: phi_q of the query rows comes precomputed (bf16, one row per query) through tmPhi
// and is loaded over the Q tiles once their last S MMA is done; otherwise the kernel computes it
// in its epilogue from U = Q Wbd^T (tmW).
template <bool kPhiGlobal>
__global__ void __launch_bounds__(kThreads, 1)
    hybrid_attn_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV,
                            const __grid_constant__ CUtensorMap tmSt,
                            const __grid_constant__ CUtensorMap tmW,
                            const __grid_constant__ CUtensorMap tmPhi,
                            const __grid_constant__ CUtensorMap tmKc,
                            const __grid_constant__ CUtensorMap tmVc,
                            const __grid_constant__ CUtensorMap tmOut, const Params p) {
  static_assert(kSmemBytes + 256 <= 232448, "shared memory (dynamic + static) over the limit");

  // ---- chunk geometry (uniform over the CTA) ----
  // grid (slots, BH, chunks).  Within one chunk the linear CTA index walks the full tile pairs of
  // one (b, h) after another, so the CTAs in flight share few K/V windows in L2; the lone last
  // tiles of an odd tile count follow (one per (b, h), or n_split short parts of its key window
  // each).  Chunk 0, whose window is shortest, is dispatched last.
  const int c = (blockIdx.z + 1) % gridDim.z;
  const ChunkGeom geo = chunk_geom(p, c);
  const int q_row0 = geo.q_row0, nq = geo.nq, k_row0 = geo.k_row0, nk = geo.nk;
  const bool has_linear = geo.has_linear;
  const int n_full = ((nq + kBM - 1) / kBM) / 2, n_lone = ((nq + kBM - 1) / kBM) & 1;
  const int n_split = p.n_split > 1 ? p.n_split : 1;
  const int n_bh = gridDim.y;
  const int lin = blockIdx.x + gridDim.x * blockIdx.y;
  int bh, pair, part = -1;  // part >= 0: one part of the lone tile's key window
  if (lin < n_full * n_bh) {
    bh = lin / n_full;
    pair = lin - bh * n_full;
  } else if (lin < (n_full + n_lone * n_split) * n_bh) {
    const int idx = lin - n_full * n_bh;
    bh = idx / n_split;
    pair = n_full;
    if (n_split > 1) part = idx - bh * n_split;
  } else {
    return;  // a slot past this chunk's tiles (its chunk is shorter than the longest)
  }
  const int h = bh % p.H;
  const int tile_row0 = pair * 2 * kBM;
  const bool has_t1 = tile_row0 + kBM < nq;
  // key tiles: n_kc from the carried segment (rows [0, kv_split) of the window), then the rest;
  // a part covers key tiles [j0, j0 + n_kv) of them (the host keeps every part non-empty)
  const int kv_split = p.kv_split;
  const int n_kc = (kv_split + kBN - 1) / kBN;
  const int n_kv_all = n_kc + (nk - kv_split + kBN - 1) / kBN;
  const int j0 = part >= 0 ? (int)((long long)part * n_kv_all / n_split) : 0;
  const int n_kv = (part >= 0 ? (int)((long long)(part + 1) * n_kv_all / n_split) : n_kv_all) - j0;
  // the linear-state readout (phi_q . S, phi_q . Z) is added once: by the whole-window CTA or by
  // part 0
  const bool readout = has_linear && part <= 0;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* sB = reinterpret_cast<float*>(sm + kOffB);
  float* sZ = reinterpret_cast<float*>(sm + kOffZ);
  uint8_t* sPw = sm + kOffPw;

  if (warp == 8) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool many = (i == kPFull || i == kPFull + 1 || i == kPhiFull || i == kPhiFull + 1);
      mbar_init(&bars[i], many ? 128 : 1);
    }
    abort_sh = 0;
    fence_mbar_init();
  }
  if (tid < 256 && readout) {
    for (int i = tid; i < kFD; i += 256) {
      sPw[i] = static_cast<uint8_t>(feature_power(i, kFD, p.P));
      sB[i] = p.bq ? p.bq[(size_t)h * kFD + i] : 0.f;
      if (!kPhiGlobal) sZ[i] = p.Z[((size_t)bh * p.n_states + c) * kFD + i];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // A kernel launched behind this one may start once every CTA is here, filling the SMs of the
  // last wave; it must not write anything this kernel reads later (window, phi_q, S^T, Z_c).
  grid_dep_signal();

  const uint32_t sQ0 = smem_u32(sm + kOffQ0), sQ1 = smem_u32(sm + kOffQ1);
  const uint32_t sK0 = smem_u32(sm + kOffK), sK1 = sK0 + kTileBytes;
  const uint32_t sV0 = smem_u32(sm + kOffV), sV1 = sV0 + kTileBytes;

  if (warp == 8) {
    // ================================ TMA producer ================================
    // The whole warp runs the loop and waits; lane 0 issues the copies.
    const bool leader = lane == 0;
    if (leader) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bars[kQFull], has_t1 ? 2 * kTileBytes : kTileBytes);
      for (int t = 0; t < (has_t1 ? 2 : 1); ++t) {
        uint8_t* dst = sm + (t ? kOffQ1 : kOffQ0);
        const int row = q_row0 + tile_row0 + t * kBM;
        tma_load_3d_chk(1, dst, &tmQ, &bars[kQFull], 0, row, bh, kHD, p.nq_rows, n_bh);
        tma_load_3d_chk(1, dst + kBM * 128, &tmQ, &bars[kQFull], 64, row, bh, kHD, p.nq_rows,
                        n_bh);
      }
    }
    __syncwarp();
    int issued_k = 0, issued_v = 0;
    bool st_issued = false;
    bool ok = true;
    if (leader && n_kc > 0) {
      tma_prefetch_desc(&tmKc);
      tma_prefetch_desc(&tmVc);
    }
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      const int jg = j0 + j;  // key tile of the window
      const bool carried = jg < n_kc;
      const int row = carried ? p.carry_row0 + jg * kBN : k_row0 + kv_split + (jg - n_kc) * kBN;
      const CUtensorMap* mK = carried ? &tmKc : &tmK;
      const CUtensorMap* mV = carried ? &tmVc : &tmV;
      if (j >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kKEmpty + s], ((j >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      if (leader) {
        uint8_t* dk = sm + kOffK + s * kTileBytes;
        mbar_arrive_expect_tx(&bars[kKFull + s], kTileBytes);
        const int kv_ext = carried ? p.carry_rows : p.kv_rows;
        tma_load_3d_chk(2, dk, mK, &bars[kKFull + s], 0, row, bh, kHD, kv_ext, n_bh);
        tma_load_3d_chk(2, dk + kBM * 128, mK, &bars[kKFull + s], 64, row, bh, kHD, kv_ext, n_bh);
      }
      __syncwarp();
      ++issued_k;
      if (j >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kVEmpty + s], ((j >> 1) - 1) & 1, abort_flag));
      if (!ok) break;
      if (leader) {
        uint8_t* dv = sm + kOffV + s * kTileBytes;
        mbar_arrive_expect_tx(&bars[kVFull + s], kTileBytes);
        const int kv_ext = carried ? p.carry_rows : p.kv_rows;
        tma_load_3d_chk(3, dv, mV, &bars[kVFull + s], 0, row, bh, kHD, kv_ext, n_bh);
        tma_load_3d_chk(3, dv + kBM * 128, mV, &bars[kVFull + s], 64, row, bh, kHD, kv_ext, n_bh);
      }
      __syncwarp();
      ++issued_v;
    }
    if (ok && readout) {
      // S_c^T, Z_c and phi_q come from the kernels enqueued before this one.  Launched behind
      // the phi_q kernel with programmatic serialization, this kernel ran its key loop while
      // that grid was still running: wait for it (and so for everything before it) here.
      grid_dep_wait();
      if (kPhiGlobal) {  // Z_c for the epilogue; published by the phi_q barrier's arrival below
        for (int i = lane; i < kFD; i += 32) sZ[i] = p.Z[((size_t)bh * p.n_states + c) * kFD + i];
        __syncwarp();
      }
      // S_c^T goes into the K stage that the (absent) tile n_kv would use.
      const int s = n_kv & 1;
      if (n_kv >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kKEmpty + s], ((n_kv >> 1) - 1) & 1, abort_flag));
      if (ok) {
        if (leader) {
          uint8_t* dst = sm + kOffK + s * kTileBytes;
          mbar_arrive_expect_tx(&bars[kStFull], kTileBytes);
          const long long st_depth = (long long)n_bh * p.n_states;
          tma_load_3d_chk(4, dst, &tmSt, &bars[kStFull], 0, 0, bh * p.n_states + c, kFD, kHD,
                          st_depth);
          tma_load_3d_chk(4, dst + kBM * 128, &tmSt, &bars[kStFull], 64, 0, bh * p.n_states + c,
                          kFD, kHD, st_depth);
        }
        __syncwarp();
        st_issued = true;
      }
    }
    bool wb_issued = false;
    if (ok && readout && kPhiGlobal) {
      // phi_q tiles go over the Q tiles once both tiles' last S MMAs are done.
      const int last = n_kv - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kKEmpty + (last & 1)], (last >> 1) & 1, abort_flag));
      if (ok) {
        if (leader) {
          mbar_arrive_expect_tx(&bars[kPhiqFull], has_t1 ? 2 * kTileBytes : kTileBytes);
          for (int t = 0; t < (has_t1 ? 2 : 1); ++t) {
            uint8_t* dst = sm + (t ? kOffQ1 : kOffQ0);
            const int row = q_row0 + tile_row0 + t * kBM;
            tma_load_3d_chk(5, dst, &tmPhi, &bars[kPhiqFull], 0, row, bh, kFD, p.nq_rows, n_bh);
            tma_load_3d_chk(5, dst + kBM * 128, &tmPhi, &bars[kPhiqFull], 64, row, bh, kFD,
                            p.nq_rows, n_bh);
          }
        }
        __syncwarp();
        wb_issued = true;
      }
    } else if (ok && readout) {
      // Block-diagonal W_q (hi, lo) goes into the two V stages once their last P.V is done.
      for (int s = 0; s < 2 && ok; ++s) {
        const int last = (n_kv - 1) - (((n_kv - 1) & 1) != s ? 1 : 0);  // last use of stage s
        if (last >= 0)
          ok = __all_sync(0xffffffffu, mbar_wait(&bars[kVEmpty + s], (last >> 1) & 1, abort_flag));
      }
      if (ok) {
        if (leader) {
          mbar_arrive_expect_tx(&bars[kWbFull], 2 * kTileBytes);
          for (int s = 0; s < 2; ++s) {
            uint8_t* dst = sm + kOffV + s * kTileBytes;
            tma_load_3d_chk(6, dst, &tmW, &bars[kWbFull], 0, 0, h * 2 + s, kHD, kFD, 2 * p.H);
            tma_load_3d_chk(6, dst + kBM * 128, &tmW, &bars[kWbFull], 64, 0, h * 2 + s, kHD, kFD,
                            2 * p.H);
          }
        }
        __syncwarp();
        wb_issued = true;
      }
    }
    if (!ok) {
      // Abort: let every copy already issued land before the CTA can exit.
      if (wb_issued) mbar_wait_drain(&bars[kPhiGlobal ? kPhiqFull : kWbFull], 0);
      mbar_wait_drain(&bars[kQFull], 0);
      for (int j = max(0, issued_k - 2); j < issued_k; ++j)
        mbar_wait_drain(&bars[kKFull + (j & 1)], (j >> 1) & 1);
      for (int j = max(0, issued_v - 2); j < issued_v; ++j)
        mbar_wait_drain(&bars[kVFull + (j & 1)], (j >> 1) & 1);
      if (st_issued) mbar_wait_drain(&bars[kStFull], 0);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ================================ MMA issuer ================================
    // Lane 0 runs the loop alone (waits, MMAs, commits); the other lanes wait at the end.  The
    // two query tiles alternate strictly (P.V and the next S of tile 0, then of tile 1), so one
    // tile's MMAs run while the other tile's softmax works.  There is no per-step O_FULL commit:
    // S_FULL(t, j) is committed after P.V(t, j-1) was issued by this thread, so its completion
    // already tells the softmax that O_t may be rescaled.
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(kBM, kBN, false, false);
      const uint32_t id_pv = idesc_bf16(kBM, kHD, false, true);
      const int nt = has_t1 ? 2 : 1;
      auto issue_s = [&](int t, int j) {
        const uint32_t d = tmem + t * 128;
        const uint32_t qb = t ? sQ1 : sQ0;
        const uint32_t kb = (j & 1) ? sK1 : sK0;
        for (int kk = 0; kk < kHD / 16; ++kk)
          mma_ss(d, kmajor_desc(qb, kk), kmajor_desc(kb, kk), id_qk, kk > 0 ? 1u : 0u);
        mma_commit(&bars[kSFull + t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t d = tmem + 256 + t * 128;
        const uint32_t a = tmem + t * 128;
        const uint32_t vb = (j & 1) ? sV1 : sV0;
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(d, a + kk * 8, mnmajor_desc(vb, kk), id_pv, (j > 0 || kk > 0) ? 1u : 0u);
      };
      auto wait = [&](int b, uint32_t parity) { return mbar_wait(&bars[b], parity, abort_flag); };
      bool ok = wait(kQFull, 0) && wait(kKFull, 0);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < nt; ++t) issue_s(t, 0);
        mma_commit(&bars[kKEmpty]);
      }
      for (int j = 1; j < n_kv && ok; ++j) {
        const int s = j & 1, sp = (j - 1) & 1;
        ok = wait(kKFull + s, (j >> 1) & 1) && wait(kVFull + sp, ((j - 1) >> 1) & 1);
        for (int t = 0; t < nt && ok; ++t) {
          ok = wait(kPFull + t, (j - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, j - 1);
          issue_s(t, j);
        }
        if (!ok) break;
        mma_commit(&bars[kVEmpty + sp]);
        mma_commit(&bars[kKEmpty + s]);
      }
      if (ok) {
        const int j = n_kv - 1;
        ok = wait(kVFull + (j & 1), (j >> 1) & 1);
        for (int t = 0; t < nt && ok; ++t) {
          ok = wait(kPFull + t, j & 1);
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, j);
          mma_commit(&bars[kOFull + t]);  // the tile's O is final (epilogue without a state)
        }
        if (ok) mma_commit(&bars[kVEmpty + (j & 1)]);
      }
      if (ok && readout) {
        // U_t = Q_t Wbd_hi^T + Q_t Wbd_lo^T into the S_t columns (free once P_t.V is issued).
        if (!kPhiGlobal) ok = wait(kWbFull, 0);
        if (ok && !kPhiGlobal) {
          tc_fence_after();
          for (int t = 0; t < nt; ++t) {
            const uint32_t d = tmem + t * 128;
            const uint32_t qb = t ? sQ1 : sQ0;
            for (int part = 0; part < 2; ++part) {
              const uint32_t wb = part ? sV1 : sV0;
              for (int kk = 0; kk < kHD / 16; ++kk)
                mma_ss(d, kmajor_desc(qb, kk), kmajor_desc(wb, kk), id_qk,
                       (part > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bars[kUFull + t]);
          }
        }
        const uint32_t stb = (n_kv & 1) ? sK1 : sK0;
        if (ok) ok = wait(kStFull, 0);
        for (int t = 0; t < nt && ok; ++t) {
          ok = wait(kPhiFull + t, 0);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + 256 + t * 128;
          const uint32_t qb = t ? sQ1 : sQ0;
          for (int kk = 0; kk < kFD / 16; ++kk)
            mma_ss(d, kmajor_desc(qb, kk), kmajor_desc(stb, kk), id_qk, 1u);
          mma_commit(&bars[kRoDone + t]);
        }
      }
      // Every tcgen05 op (and the mbarrier arrivals it triggers) must finish before teardown.
      mma_commit(&bars[kMmaDone]);
      mbar_wait_drain(&bars[kMmaDone], 0);
    }
    __syncwarp();
  } else {
    // ============================ softmax / epilogue warpgroups ============================
    const int t = warp >> 2;          // query tile of this warpgroup
    const int r = tid & 127;          // row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + 256 + t * 128;
    const bool active = (t == 0) || has_t1;
    // a whole-window CTA's tile whose 128 rows all lie in the chunk is stored by TMA
    const bool full_tile = part < 0 && tile_row0 + t * kBM + kBM <= nq;
    if (active) {
      const float sl2 = p.scale_log2;
      float m = has_linear ? 0.f : -INFINITY;
      float l = 0.f;
      bool ok = true;
      for (int j = 0; j < n_kv; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kSFull + t], j & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        // The S row (128 fp32) is read once into registers; the row max is a tree over eight
        // partial maxima and the row sum uses four accumulators, so neither is one long
        // dependency chain.  Only a segment's last tile can be ragged (uniform branch).
        // key columns of this tile inside its segment of the window
        const int jg = j0 + j;
        const int valid = jg < n_kc ? kv_split - jg * kBN : nk - kv_split - (jg - n_kc) * kBN;
        uint32_t rr[kBN];
        tmem_ld128(tS, rr);
        if (valid < kBN) {
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (i >= valid) rr[i] = __float_as_uint(-INFINITY);
        }
        float mx;
        {
          float m8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = __uint_as_float(rr[i]);
#pragma unroll
          for (int i = 8; i + 16 <= kBN; i += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              m8[e] = max3(m8[e], __uint_as_float(rr[i + e]), __uint_as_float(rr[i + 8 + e]));
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], __uint_as_float(rr[kBN - 8 + e]));
          mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        }
        const float m_tile = mx * sl2;
        const float m_new = (m_tile > m + 8.f) ? m_tile : m;
        const bool rescale = (m_new != m) && (j > 0);
        if (__any_sync(0xffffffffu, rescale)) {
          // Rare: rescale O and l.  S_FULL for this tile was committed after the tile's previous
          // P.V, so that P.V is complete and O may be rewritten.  S is reloaded afterwards so it
          // need not stay live here.
          const float fac = rescale ? ex2(m - m_new) : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < kHD / 16; ++cc) {
            uint32_t ro[16];
            tmem_ld16(tO + cc * 16, ro);
#pragma unroll
            for (int i = 0; i < 16; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) * fac);
            tmem_st16(tO + cc * 16, ro);
          }
          l *= fac;
          tmem_ld128(tS, rr);
          if (valid < kBN) {
#pragma unroll
            for (int i = 0; i < kBN; ++i)
              if (i >= valid) rr[i] = __float_as_uint(-INFINITY);
          }
        }
        m = m_new;
        // Column pairs go through paired fp32 instructions (x = s * scale - m for two columns in
        // one FMA, the row sum in two paired accumulators); 2^x on the MUFU; bf16 pack.
        // 16 probabilities -> 8 packed columns per TMEM store.
        const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m, -m);
        uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int hh = 0; hh < kBN / 16; ++hh) {
          uint32_t pr[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(rr[hh * 16 + 2 * i]),
                                               __uint_as_float(rr[hh * 16 + 2 * i + 1])),
                                       sl2x2, negm2);
            float xa, xb;
            f2_unpack(x2, xa, xb);
            const uint64_t p2 = f2_pack(ex2(xa), ex2(xb));
            rs2[i & 1] = f2_add(rs2[i & 1], p2);
            float a, b;
            f2_unpack(p2, a, b);
            pr[i] = pack_bf16x2(a, b);
          }
          tmem_st8(tS + hh * 8, pr);
        }
        float rowsum;
        {
          float a0, a1, b0, b1;
          f2_unpack(rs2[0], a0, a1);
          f2_unpack(rs2[1], b0, b1);
          rowsum = (a0 + a1) + (b0 + b1);
        }
        l += rowsum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[kPFull + t]);
      }
      // ---- epilogue ----
      if (ok && readout && kPhiGlobal) {
        // The precomputed phi_q row sits in this row of the Q tile: scale it by 2^-m in place
        // (bf16) and form phi_q . Z_c with the same rounded values the MMA will use.
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kPhiqFull], 0, abort_flag));
        if (ok) {
          uint8_t* qrow = sm + (t ? kOffQ1 : kOffQ0);
          const float esc = ex2(-m);
          float lin[2] = {0.f, 0.f};
#pragma unroll 4
          for (int c8 = 0; c8 < kFD / 8; ++c8) {
            uint4* a4 = reinterpret_cast<uint4*>(qrow + sw128_offset(r, c8 * 8, kBM));
            uint4 v4 = *a4;
            uint32_t* w = reinterpret_cast<uint32_t*>(&v4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 b2 = *reinterpret_cast<__nv_bfloat162*>(&w[e]);
              const float2 f2 = __bfloat1622float2(b2);
              const float x0 = __bfloat162float(__float2bfloat16_rn(f2.x * esc));
              const float x1 = __bfloat162float(__float2bfloat16_rn(f2.y * esc));
              lin[0] = fmaf(x0, sZ[c8 * 8 + 2 * e], lin[0]);
              lin[1] = fmaf(x1, sZ[c8 * 8 + 2 * e + 1], lin[1]);
              w[e] = pack_bf16x2(x0, x1);
            }
            *a4 = v4;
          }
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(&bars[kPhiFull + t]);
          l += lin[0] + lin[1];
          ok = __all_sync(0xffffffffu, mbar_wait(&bars[kRoDone + t], 0, abort_flag));
        }
      } else if (ok && readout) {
        // U_FULL also means every earlier MMA of this CTA (the last P.V included) is complete.
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kUFull + t], 0, abort_flag));
        if (ok) {
          tc_fence_after();
          // phi_q(q) * 2^-m in bf16 over this row of the Q tile (its last reader, the U MMA, is
          // done); 16 features per step keeps the loop body small.
          uint8_t* qrow = sm + (t ? kOffQ1 : kOffQ0);
          const float esc = ex2(-m);
          float lin[2] = {0.f, 0.f};
#pragma unroll 1
          for (int c16 = 0; c16 < kFD / 16; ++c16) {
            const int f0 = c16 * 16;
            uint32_t uu[16];
            tmem_ld16(tS + f0, uu);
            uint32_t packed[8];
            phi16(uu, f0, sB, sPw, esc, packed);
#pragma unroll
            for (int f2 = 0; f2 < 8; ++f2) {
              const float2 pf = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&packed[f2]));
              lin[0] = fmaf(pf.x, sZ[f0 + 2 * f2], lin[0]);
              lin[1] = fmaf(pf.y, sZ[f0 + 2 * f2 + 1], lin[1]);
            }
            *reinterpret_cast<uint4*>(qrow + sw128_offset(r, f0, kBM)) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            *reinterpret_cast<uint4*>(qrow + sw128_offset(r, f0 + 8, kBM)) =
                make_uint4(packed[4], packed[5], packed[6], packed[7]);
          }
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(&bars[kPhiFull + t]);
          l += lin[0] + lin[1];
          ok = __all_sync(0xffffffffu, mbar_wait(&bars[kRoDone + t], 0, abort_flag));
        }
      } else if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kOFull + t], 0, abort_flag));
      }
      if (ok && part >= 0) {
        // one part of a lone tile's window: its rows' unnormalised O and (m, l), every row
        tc_fence_after();
        const size_t slot = ((size_t)c * n_bh + bh) * n_split + part;
        const bool store_ok = bounds_ok(8, (long long)slot, 0, (long long)gridDim.z * n_bh * n_split);
        float* po = p.part_o + (slot * kBM + r) * kHD;
#pragma unroll
        for (int cc = 0; cc < kHD / 32; ++cc) {
          uint32_t rr[32];
          tmem_ld32(tO + cc * 32, rr);
          if (store_ok) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4*>(po + cc * 32 + q4 * 4) =
                  make_float4(__uint_as_float(rr[q4 * 4]), __uint_as_float(rr[q4 * 4 + 1]),
                              __uint_as_float(rr[q4 * 4 + 2]), __uint_as_float(rr[q4 * 4 + 3]));
          }
        }
        if (store_ok)
          *reinterpret_cast<float2*>(p.part_ml + (slot * kBM + r) * 2) = make_float2(m, l);
      } else if (ok) {
        tc_fence_after();
        const int row_in_chunk = tile_row0 + t * kBM + r;
        const bool row_valid =
            row_in_chunk < nq && bounds_ok(7, q_row0 + row_in_chunk, 0, p.nq_rows);
        const float inv = 1.f / l;
        if (p.lse && row_valid)
          p.lse[(size_t)bh * p.nq_rows + q_row0 + row_in_chunk] = m + log2f(l);
        if (full_tile) {
          // A full tile leaves by two TMA stores from its Q tile's shared memory, which no MMA
          // reads any more (its readout, or without one its last S, is complete): rows packed in
          // the 128B-swizzled layout of the store's two 64-column boxes (stored below).
          uint8_t* ostage = sm + (t ? kOffQ1 : kOffQ0);
#pragma unroll
          for (int cc = 0; cc < kHD / 32; ++cc) {
            uint32_t rr[32];
            tmem_ld32(tO + cc * 32, rr);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 o4;
              o4.x = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 0]) * inv, __uint_as_float(rr[q4 * 8 + 1]) * inv);
              o4.y = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 2]) * inv, __uint_as_float(rr[q4 * 8 + 3]) * inv);
              o4.z = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 4]) * inv, __uint_as_float(rr[q4 * 8 + 5]) * inv);
              o4.w = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 6]) * inv, __uint_as_float(rr[q4 * 8 + 7]) * inv);
              *reinterpret_cast<uint4*>(ostage + sw128_offset(r, cc * 32 + q4 * 8, kBM)) = o4;
            }
          }
        } else {
          __nv_bfloat16* orow = p.out + ((size_t)bh * p.nq_rows + q_row0 + row_in_chunk) * kHD;
#pragma unroll
          for (int cc = 0; cc < kHD / 32; ++cc) {
            uint32_t rr[32];
            tmem_ld32(tO + cc * 32, rr);
            if (row_valid) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                uint4 o4;
                o4.x = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 0]) * inv, __uint_as_float(rr[q4 * 8 + 1]) * inv);
                o4.y = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 2]) * inv, __uint_as_float(rr[q4 * 8 + 3]) * inv);
                o4.z = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 4]) * inv, __uint_as_float(rr[q4 * 8 + 5]) * inv);
                o4.w = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 6]) * inv, __uint_as_float(rr[q4 * 8 + 7]) * inv);
                *reinterpret_cast<uint4*>(orow + cc * 32 + q4 * 8) = o4;
              }
            }
          }
        }
      }
      if (full_tile) {
        // every thread of the tile gets here, whatever its waits returned (a named barrier has
        // no time limit); after an abort the store is skipped
        fence_async_smem();
        named_bar_sync(1 + t, kBM);
        if (r == 0 && !*abort_flag) {
          uint8_t* ostage = sm + (t ? kOffQ1 : kOffQ0);
          const int row = q_row0 + tile_row0 + t * kBM;
          tma_store_3d_chk(32, &tmOut, ostage, 0, row, bh, kHD, p.nq_rows, n_bh);
          tma_store_3d_chk(32, &tmOut, ostage + kBM * 128, 64, row, bh, kHD, p.nq_rows, n_bh);
          bulk_commit_group();
          bulk_wait_all();  // complete before the CTA exits
        }
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merges the parts of every chunk's lone last tile (see Params::n_split):
//   out = sum_i 2^(m_i - M) O_i / sum_i 2^(m_i - M) l_i,  M = max_i m_i.
// grid (BH, chunks, 128 rows), block D = 128 (one output column per thread).
__global__ void __launch_bounds__(kHD) lone_combine_kernel(const Params p) {
  const int bh = blockIdx.x, c = blockIdx.y, r = blockIdx.z, col = threadIdx.x;
  const ChunkGeom geo = chunk_geom(p, c);
  const int n_tiles = (geo.nq + kBM - 1) / kBM;
  if (!(n_tiles & 1)) return;  // no lone tile in this chunk
  const int row_in_chunk = (n_tiles / 2) * 2 * kBM + r;
  if (row_in_chunk >= geo.nq) return;
  const size_t slot0 = ((size_t)c * gridDim.x + bh) * p.n_split;
  if (!bounds_ok(31, geo.q_row0 + row_in_chunk, 0, p.nq_rows)) return;
  float M = -INFINITY;
  for (int i = 0; i < p.n_split; ++i) M = fmaxf(M, p.part_ml[((slot0 + i) * kBM + r) * 2]);
  float num = 0.f, den = 0.f;
  for (int i = 0; i < p.n_split; ++i) {
    const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + ((slot0 + i) * kBM + r) * 2);
    const float w = ex2(ml.x - M);
    den = fmaf(w, ml.y, den);
    num = fmaf(w, p.part_o[((slot0 + i) * kBM + r) * kHD + col], num);
  }
  p.out[((size_t)bh * p.nq_rows + geo.q_row0 + row_in_chunk) * kHD + col] =
      __float2bfloat16_rn(num / den);
}

}  // namespace attn
}  // namespace rehyat
