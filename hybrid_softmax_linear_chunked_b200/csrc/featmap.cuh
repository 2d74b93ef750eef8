// Feature map phi of the "ReHyAt overview" page §2.2.2: grouped 1x1 linear (G groups, group g
// maps input dims [g*D/G, (g+1)*D/G) to features [g*F/G, (g+1)*F/G)), plus bias, split into P
// contiguous parts (the first F mod P parts one longer, numpy.array_split order), part p
// (1-based) raised to softplus(.)^p, concatenated back in order.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace rehyat {

using sm100::pack_bf16x2;

// Power applied to feature f when F features are split into P parts.
__host__ __device__ __forceinline__ int part_power(int f, int F, int P) {
  const int base = F / P, extra = F % P;
  const int big = extra * (base + 1);
  const int p = (f < big) ? f / (base + 1) : extra + (f - big) / base;
  return p + 1;
}

// Entry of the per-feature table the kernels keep: the part power, or 0 for the elu + 1 map
// (kernels receive P = 0 for it; a power of 0 never occurs in the polynomial map).
__host__ __device__ __forceinline__ int feature_power(int f, int F, int P) {
  return P == 0 ? 0 : part_power(f, F, P);
}

// elu(u) + 1: u + 1 for u > 0, e^u otherwise.
__device__ __forceinline__ float elu1_fast(float u) { return u > 0.f ? u + 1.f : __expf(u); }
__device__ __forceinline__ float elu1_accurate(float u) { return u > 0.f ? u + 1.f : expf(u); }

__device__ __forceinline__ float int_pow(float x, int p) {
  float r = x;
  for (int i = 1; i < p; ++i) r *= x;
  return r;
}

// x^p by selects, for 1 <= p <= 4.
__device__ __forceinline__ float pow_upto4(float x, int p) {
  const float x2 = x * x;
  float r = x;
  r = (p == 2) ? x2 : r;
  r = (p == 3) ? x2 * x : r;
  r = (p == 4) ? x2 * x2 : r;
  return r;
}

// softplus(u) = max(u, 0) + log1p(e^{-|u|}) with the CUDA math library's expf/log1pf.
__device__ __forceinline__ float softplus_accurate(float u) {
  return fmaxf(u, 0.f) + log1pf(expf(-fabsf(u)));
}

// Same function with the fast hardware exp/log.  log1p(y) for y = e^{-|u|} in (0, 1] uses the
// first terms of its Taylor series y - y^2/2 + y^3/3 below y = 2^-7 (truncation < y^4/4, i.e.
// relative 1.2e-7) and log(1 + y) above it, where 1 + y >= 1.0078 keeps rounding of the sum
// below 1e-5 relative.  Accurate to well within bf16 rounding.
__device__ __forceinline__ float softplus_fast(float u) {
  const float y = __expf(-fabsf(u));
  const float l = (y < 0.0078125f) ? y * (1.f - y * (0.5f - y * (1.f / 3.f))) : __logf(1.f + y);
  return fmaxf(u, 0.f) + l;
}

// log2(1 + y) = y r(y) for y in [0, 1], with r(y) = log2(1 + y) / y a quintic fitted for minimax
// relative error on [0, 1] by iteratively reweighted least squares (softplus_poly_fit.py beside
// this file): 8.6e-6 relative in fp32 Horner form, against the 2^-9 rounding of the bf16 result.
constexpr float kL1pC0 = 1.44268286f;
constexpr float kL1pC1 = -0.720426023f;
constexpr float kL1pC2 = 0.469173372f;
constexpr float kL1pC3 = -0.303034991f;
constexpr float kL1pC4 = 0.146032020f;
constexpr float kL1pC5 = -0.0344357193f;
constexpr float kLog2e = 1.44269504f;
constexpr float kLn2 = 0.693147181f;

// softplus in log2 units for a pair of lanes: with t = u log2(e),
//     softplus(u) = ln2 * s,   s = max(t, 0) + log2(1 + 2^-|t|),
// 2^-|t| on the MUFU (one op per element) and log2(1 + y) by the quintic on the FMA pipe.
__device__ __forceinline__ uint64_t softplus_log2_x2(uint64_t t2) {
  using namespace sm100;
  float ta, tb;
  f2_unpack(t2, ta, tb);
  const uint64_t y2 = f2_pack(ex2(-fabsf(ta)), ex2(-fabsf(tb)));
  uint64_t r2 = f2_fma(f2_pack(kL1pC5, kL1pC5), y2, f2_pack(kL1pC4, kL1pC4));
  r2 = f2_fma(r2, y2, f2_pack(kL1pC3, kL1pC3));
  r2 = f2_fma(r2, y2, f2_pack(kL1pC2, kL1pC2));
  r2 = f2_fma(r2, y2, f2_pack(kL1pC1, kL1pC1));
  r2 = f2_fma(r2, y2, f2_pack(kL1pC0, kL1pC0));
  return f2_fma(r2, y2, f2_pack(fmaxf(ta, 0.f), fmaxf(tb, 0.f)));
}

// phi of 16 consecutive features f0 .. f0+15 from their grouped-linear outputs u (fp32 bits):
// softplus(u + bias)^p, with p the feature's part power (pw[], non-decreasing in f), times
// `scale`, packed as 8 bf16 pairs.  Parts are contiguous, so a 16-feature chunk nearly always
// has a single power p: that case (a uniform branch) folds ln2^p and the scale into one factor,
// phi = s^p * (ln2^p * scale), in paired instructions.
__device__ __forceinline__ void phi16(const uint32_t* u, int f0, const float* bias,
                                      const uint8_t* pw, float scale, uint32_t* packed) {
  using namespace sm100;
  const int p_first = pw[f0], p_last = pw[f0 + 15];
  if (p_last == 0) {  // elu + 1 map (the whole table is 0)
    float ph[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) ph[i] = elu1_fast(__uint_as_float(u[i]) + bias[f0 + i]);
#pragma unroll
    for (int i = 0; i < 8; ++i) packed[i] = pack_bf16x2(ph[2 * i] * scale, ph[2 * i + 1] * scale);
    return;
  }
  const uint64_t l2e2 = f2_pack(kLog2e, kLog2e);
  uint64_t s2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 b = *reinterpret_cast<const float2*>(bias + f0 + 2 * i);
    const uint64_t x2 = f2_add(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])),
                               f2_pack(b.x, b.y));
    s2[i] = softplus_log2_x2(f2_mul(x2, l2e2));
  }
  if (p_first == p_last && p_first <= 3) {
    const float c = p_first == 1 ? kLn2 * scale
                  : p_first == 2 ? (kLn2 * kLn2) * scale
                                 : (kLn2 * kLn2 * kLn2) * scale;
    const uint64_t c2 = f2_pack(c, c);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint64_t v2 = s2[i];
      if (p_first == 2) v2 = f2_mul(v2, v2);
      if (p_first == 3) v2 = f2_mul(f2_mul(v2, v2), v2);
      float a, b;
      f2_unpack(f2_mul(v2, c2), a, b);
      packed[i] = pack_bf16x2(a, b);
    }
    return;
  }
  float ph[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f2_unpack(s2[i], ph[2 * i], ph[2 * i + 1]);
    ph[2 * i] *= kLn2;
    ph[2 * i + 1] *= kLn2;
  }
  if (p_last <= 4) {
#pragma unroll
    for (int i = 0; i < 16; ++i) ph[i] = pow_upto4(ph[i], pw[f0 + i]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) ph[i] = int_pow(ph[i], pw[f0 + i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) packed[i] = pack_bf16x2(ph[2 * i] * scale, ph[2 * i + 1] * scale);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Standalone feature map: x [BH, n, D] -> phi [BH, n, F].  One thread per token; the head's W
// and bias are staged in shared memory (read as broadcasts).  The x row is staged through a
// per-thread slice of shared memory loaded cooperatively (coalesced) so global traffic is one
// read of x and one write of phi.
//   grid (ceil(n / 128), BH), block 128, dynamic smem: W (G*F/G*D/G floats) + F floats bias +
//   128 * (D + 1) floats of x staging.
template <typename Tin, typename Tout, bool kAccurate>
__global__ void __launch_bounds__(128) featmap_kernel(const Tin* __restrict__ x,
                                                      const float* __restrict__ W,
                                                      const float* __restrict__ bias,
                                                      Tout* __restrict__ phi, int n, int H, int D,
                                                      int F, int G, int P) {
  extern __shared__ float fm_smem[];
  const int Dg = D / G, Fg = F / G;
  float* sW = fm_smem;                 // [G][Fg][Dg]
  float* sB = sW + G * Fg * Dg;        // [F]
  float* sX = sB + F;                  // [128][D + 1]
  const int bh = blockIdx.y, h = bh % H;
  const int row0 = blockIdx.x * 128;
  const float* Wh = W + (size_t)h * G * Fg * Dg;
  for (int i = threadIdx.x; i < G * Fg * Dg; i += 128) sW[i] = Wh[i];
  for (int i = threadIdx.x; i < F; i += 128) sB[i] = bias ? bias[(size_t)h * F + i] : 0.f;
  const Tin* xb = x + ((size_t)bh * n + row0) * D;
  const int rows = min(128, n - row0);
  for (int i = threadIdx.x; i < rows * D; i += 128) {
    const int r = i / D, c = i - r * D;
    sX[r * (D + 1) + c] = to_f32<Tin>(xb[i]);
  }
  __syncthreads();
  const int r = threadIdx.x;
  if (r >= rows) return;
  const float* xr = sX + r * (D + 1);
  Tout* out = phi + ((size_t)bh * n + row0 + r) * F;
  for (int g = 0; g < G; ++g) {
    for (int o = 0; o < Fg; ++o) {
      const int f = g * Fg + o;
      const float* w = sW + (g * Fg + o) * Dg;
      float u = sB[f];
      for (int i = 0; i < Dg; ++i) u = fmaf(w[i], xr[g * Dg + i], u);
      if (P == 0) {
        out[f] = from_f32<Tout>(kAccurate ? elu1_accurate(u) : elu1_fast(u));
      } else {
        const float sp = kAccurate ? softplus_accurate(u) : softplus_fast(u);
        out[f] = from_f32<Tout>(int_pow(sp, part_power(f, F, P)));
      }
    }
  }
}

// Compact tensor-core form of the grouped linear u = x Wbd^T, built in shared memory by the CTA
// that uses it.  The block-diagonal F x D matrix Wbd is covered by TG = min(G, F/16) diagonal
// tiles of NT = F/TG rows (features) by KT = D/TG columns (input dims): tile t is rows
// [t NT, (t+1) NT) x columns [t KT, (t+1) KT) of Wbd, and every group's block lies inside one
// tile (a 16 x 16 tile holds two 8 x 8 blocks when G = 16).  The tiles are stored side by side
// as one [NT][D] bf16 matrix in the 128-byte-swizzled K-major layout of an MMA B operand (row n,
// column d = tile t's column d - t KT), twice: hi = bf16(w) and lo = bf16(w - hi).  u's columns
// [t NT, (t+1) NT) are then the MMAs of tile t's KT / 16 K steps with N = NT: D / 16 MMAs per
// part whatever G is, against 8 full-width ones for the dense matrix.
struct CompactW {
  int TG, NT, KT;
};
__host__ __device__ __forceinline__ CompactW compact_w(int F, int D, int G) {
  const int tg = G < F / 16 ? G : F / 16;
  return {tg, F / tg, D / tg};
}
// Bytes of one part (hi or lo) of the compact matrix.
__host__ __device__ __forceinline__ int compact_w_bytes(int F, int D, int G) {
  return compact_w(F, D, G).NT * D * 2;
}

// Writes both parts of head h's compact matrix (W of that head: [G][F/G][D/G] fp32) into shared
// memory at hi and lo (1024-byte aligned); threads tid = 0 .. nthreads-1 share the work.  The
// caller makes the stores visible to the tensor cores (fence.proxy.async + a CTA barrier).
__device__ __forceinline__ void build_compact_w(const float* __restrict__ W, int F, int D, int G,
                                                uint8_t* hi, uint8_t* lo, int tid, int nthreads) {
  const CompactW cw = compact_w(F, D, G);
  const int Fg = F / G, Dg = D / G;
  for (int e = tid; e < cw.NT * D; e += nthreads) {
    const int n = e / D, d = e - n * D;
    const int f = (d / cw.KT) * cw.NT + n;  // feature of row n in the tile that column d is in
    const int g = f / Fg;
    const float w = (d / Dg == g) ? W[f * Dg + (d - g * Dg)] : 0.f;
    const __nv_bfloat16 wh = __float2bfloat16_rn(w);
    const __nv_bfloat16 wl = __float2bfloat16_rn(w - __bfloat162float(wh));
    const uint32_t off = sm100::sw128_offset(n, d, cw.NT);
    *reinterpret_cast<__nv_bfloat16*>(hi + off) = wh;
    *reinterpret_cast<__nv_bfloat16*>(lo + off) = wl;
  }
}

// Block-diagonal form of the grouped linear for the tensor cores: for head h, the dense
// F x D matrix Wbd[f][d] = W[g][f - g F/G][d - g D/G] when d lies in f's group g, else 0, split
// into bf16 hi = bf16(Wbd) and lo = bf16(Wbd - hi) so that x.Wbd^T from two bf16 MMAs with fp32
// accumulation carries about 16 mantissa bits of W.
//   out [H][2][F][D] bf16 (hi at [h][0], lo at [h][1]).
//   grid (ceil(F*D / 2048), H), block 256: each thread writes 8 consecutive d of one f.
__global__ void __launch_bounds__(256) blockdiag_weights_kernel(const float* __restrict__ W, int D,
                                                                int F, int G,
                                                                __nv_bfloat16* __restrict__ out) {
  const int h = blockIdx.y;
  const int Dg = D / G, Fg = F / G;
  const int e0 = (blockIdx.x * 256 + threadIdx.x) * 8;
  if (e0 >= F * D) return;
  const int f = e0 / D, d0 = e0 - f * D;  // D % 8 == 0, so the 8 elements share f
  const int g = f / Fg;
  const float* Wrow = W + (size_t)h * F * Dg + (size_t)f * Dg;
  uint32_t hi2[4], lo2[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float w[2], r[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int d = d0 + 2 * q + e;
      w[e] = (d / Dg == g) ? Wrow[d - g * Dg] : 0.f;
      r[e] = w[e] - __bfloat162float(__float2bfloat16_rn(w[e]));
    }
    __nv_bfloat162 hv = __floats2bfloat162_rn(w[0], w[1]);
    __nv_bfloat162 lv = __floats2bfloat162_rn(r[0], r[1]);
    hi2[q] = *reinterpret_cast<uint32_t*>(&hv);
    lo2[q] = *reinterpret_cast<uint32_t*>(&lv);
  }
  __nv_bfloat16* hi = out + (size_t)h * 2 * F * D;
  *reinterpret_cast<uint4*>(hi + e0) = make_uint4(hi2[0], hi2[1], hi2[2], hi2[3]);
  *reinterpret_cast<uint4*>(hi + (size_t)F * D + e0) = make_uint4(lo2[0], lo2[1], lo2[2], lo2[3]);
}

}  // namespace rehyat
