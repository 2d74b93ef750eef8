// fp32 path (CUDA cores, exact expf/log1pf): the same hybrid attention forward for fp32 inputs,
// where bf16 tensor-core products would not reach fp32 accuracy.  Sources as for the bf16 path:
// "ReHyAt overview" page §2.2.1 (joint normaliser), §2.2.2 (phi), §2.3 (states).
//
//  * fold_partial_f32_kernel: dS = phi_k^T V, dZ = phi_k^T 1 over one fold range (phi_k already
//    computed by featmap_kernel into the workspace).
//  * state_scan_f32_kernel: exclusive prefix S_c, Z_c (fp32, [C][F][D] / [C][F]).
//  * hybrid_attn_f32_kernel: one warp per query row; keys of the softmax window in blocks of 32
//    (one key per lane), exact online softmax, then the phi_q . S_c / phi_q . Z_c readout.
#pragma once

#include <cstdint>

namespace rehyat {
namespace fp32 {

struct FoldParams {
  int L, T, Tc, To, kv_frame0;
  int single_rows;  // >= 0: fold rows [0, single_rows) of the k/v buffer
  int n_fold, F, D, nkv_rows;
  const float* phik;  // [BH][nkv_rows][F]
  const float* v;     // [BH][nkv_rows][D]
  float* dS;          // [BH][n_fold][F][D]
  float* dZ;          // [BH][n_fold][F]
};

// grid (n_fold, BH), block 256.
__global__ void __launch_bounds__(256) fold_partial_f32_kernel(const FoldParams p) {
  const int fc = blockIdx.x, bh = blockIdx.y;
  int r0, r1;
  if (p.single_rows >= 0) {
    r0 = 0;
    r1 = p.single_rows;
  } else {
    r0 = (max(0, fc * p.Tc - p.To) - p.kv_frame0) * p.L;
    r1 = (max(0, (fc + 1) * p.Tc - p.To) - p.kv_frame0) * p.L;
  }
  const float* phik = p.phik + (size_t)bh * p.nkv_rows * p.F;
  const float* v = p.v + (size_t)bh * p.nkv_rows * p.D;
  float* dS = p.dS + ((size_t)bh * p.n_fold + fc) * p.F * p.D;
  float* dZ = p.dZ + ((size_t)bh * p.n_fold + fc) * p.F;
  for (int e = threadIdx.x; e < p.F * p.D; e += 256) {
    const int f = e / p.D, d = e - f * p.D;
    float acc = 0.f;
    for (int t = r0; t < r1; ++t) acc = fmaf(phik[(size_t)t * p.F + f], v[(size_t)t * p.D + d], acc);
    dS[e] = acc;
  }
  for (int f = threadIdx.x; f < p.F; f += 256) {
    float acc = 0.f;
    for (int t = r0; t < r1; ++t) acc += phik[(size_t)t * p.F + f];
    dZ[f] = acc;
  }
}

// S_c = S0 + sum_{c' < c} dS_{c'} (S0 optional), likewise Z.  grid (ceil(F*D/256), BH).
__global__ void __launch_bounds__(256) state_scan_f32_kernel(const float* __restrict__ dS,
                                                             const float* __restrict__ dZ,
                                                             int n_fold, int C, int F, int D,
                                                             const float* __restrict__ S0,
                                                             const float* __restrict__ Z0,
                                                             float* __restrict__ Sc,
                                                             float* __restrict__ Zc) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e < F * D) {
    float acc = S0 ? S0[(size_t)bh * F * D + e] : 0.f;
    for (int c = 0; c < C; ++c) {
      Sc[((size_t)bh * C + c) * F * D + e] = acc;
      if (c < n_fold) acc += dS[((size_t)bh * n_fold + c) * F * D + e];
    }
  }
  if (e < F) {
    float acc = Z0 ? Z0[(size_t)bh * F + e] : 0.f;
    for (int c = 0; c < C; ++c) {
      Zc[((size_t)bh * C + c) * F + e] = acc;
      if (c < n_fold) acc += dZ[((size_t)bh * n_fold + c) * F + e];
    }
  }
}

struct AttnParams {
  int L, T, Tc, To, frames_before, kv_frame0;
  int D, F, nq_rows, nkv_rows, n_states;
  float scale;            // 1/sqrt(D)
  const float* q;         // [BH][nq_rows][D]
  const float* k;         // [BH][nkv_rows][D]
  const float* v;
  const float* phiq;      // [BH][nq_rows][F]
  const float* S;         // [BH][n_states][F][D]
  const float* Z;         // [BH][n_states][F]
  float* out;             // [BH][nq_rows][D]
};

constexpr int kMaxD = 256;

// grid (ceil(max rows per chunk / 4), C, BH), block 128 (warp w -> one query row).
__global__ void __launch_bounds__(128) hybrid_attn_f32_kernel(const AttnParams p) {
  __shared__ float sq[4][kMaxD];
  const int c = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gs = p.frames_before + c * p.Tc;
  const int ge = min(gs + p.Tc, p.frames_before + p.T);
  const int gw = max(0, gs - p.To);
  const int nq = (ge - gs) * p.L;
  const int rq = blockIdx.x * 4 + warp;
  if (rq >= nq) return;
  const int row = (gs - p.frames_before) * p.L + rq;
  const int k0 = (gw - p.kv_frame0) * p.L;
  const int nk = (ge - gw) * p.L;
  const bool has_linear = gw > 0;
  const int DL = p.D / 32;  // dims per lane

  const float* qr = p.q + ((size_t)bh * p.nq_rows + row) * p.D;
  for (int d = lane; d < p.D; d += 32) sq[warp][d] = qr[d];
  __syncwarp();
  const float* kb = p.k + ((size_t)bh * p.nkv_rows + k0) * p.D;
  const float* vb = p.v + ((size_t)bh * p.nkv_rows + k0) * p.D;

  float acc[kMaxD / 32];
  for (int i = 0; i < kMaxD / 32; ++i) acc[i] = 0.f;
  float m = has_linear ? 0.f : -INFINITY;
  float l = 0.f;
  for (int j0 = 0; j0 < nk; j0 += 32) {
    const int j = j0 + lane;
    float s = -INFINITY;
    if (j < nk) {
      const float* kr = kb + (size_t)j * p.D;
      float dot = 0.f;
      for (int d = 0; d < p.D; ++d) dot = fmaf(sq[warp][d], kr[d], dot);
      s = dot * p.scale;
    }
    float mx = s;
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float m_new = fmaxf(m, mx);
    const float fac = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float pj = (j < nk) ? expf(s - m_new) : 0.f;
    float ps = pj;
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * fac + ps;
    for (int i = 0; i < DL; ++i) acc[i] *= fac;
    const int cnt = min(32, nk - j0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float w = __shfl_sync(0xffffffffu, pj, jj);
      const float* vr = vb + (size_t)(j0 + jj) * p.D;
      for (int i = 0; i < DL; ++i) acc[i] = fmaf(w, vr[lane + 32 * i], acc[i]);
    }
    m = m_new;
  }
  float den = l;
  if (has_linear) {
    const float e = expf(-m);
    const float* ph = p.phiq + ((size_t)bh * p.nq_rows + row) * p.F;
    const float* S = p.S + ((size_t)bh * p.n_states + c) * p.F * p.D;
    const float* Z = p.Z + ((size_t)bh * p.n_states + c) * p.F;
    float lin[kMaxD / 32];
    for (int i = 0; i < kMaxD / 32; ++i) lin[i] = 0.f;
    float lz = 0.f;
    for (int f = 0; f < p.F; ++f) {
      const float pf = ph[f];
      lz = fmaf(pf, Z[f], lz);
      for (int i = 0; i < DL; ++i) lin[i] = fmaf(pf, S[(size_t)f * p.D + lane + 32 * i], lin[i]);
    }
    for (int i = 0; i < DL; ++i) acc[i] = fmaf(e, lin[i], acc[i]);
    den = fmaf(e, lz, den);
  }
  float* orow = p.out + ((size_t)bh * p.nq_rows + row) * p.D;
  const float inv = 1.f / den;
  for (int i = 0; i < DL; ++i) orow[lane + 32 * i] = acc[i] * inv;
}

// S[bh] += dS[bh], Z[bh] += dZ[bh] (streaming fold).  grid (ceil(F*D/256), BH).
__global__ void __launch_bounds__(256) state_add_f32_kernel(const float* __restrict__ dS,
                                                            const float* __restrict__ dZ, int F,
                                                            int D, float* __restrict__ S,
                                                            float* __restrict__ Z) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e < F * D) S[(size_t)bh * F * D + e] += dS[(size_t)bh * F * D + e];
  if (e < F) Z[(size_t)bh * F + e] += dZ[(size_t)bh * F + e];
}

}  // namespace fp32
}  // namespace rehyat
