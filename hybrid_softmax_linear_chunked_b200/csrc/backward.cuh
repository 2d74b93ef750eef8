// Backward pass of the hybrid attention: the element-wise and reduction steps between the tensor-
// core products (gemm_bf16.cuh).  The gradients are the derivative of the "ReHyAt overview"
// page's §2.2.1 output formula (softmax part + linear part) / (softmax + linear normaliser),
// written with the row statistics the forward saves (lse2 = log2 of the row's denominator in
// the units where key j weighs 2^(q.k_j log2(e) / sqrt(D))):
//   P_ij  = 2^(s_ij log2(e)/sqrt(D) - lse2_i)    softmax weight of key j, normalised
//   lam_i = 2^(-lse2_i)                          normalised weight of the linear term
//   D_i   = dO_i . O_i
//   dS_ij = P_ij (dO_i . v_j - D_i) / sqrt(D)    gradient of the raw logit q_i . k_j
//   dphi_q_i = lam_i (S_c dO_i - D_i Z_c)        (S_c dO_i = the row of dO S_c^T)
//   R_c = sum_{i in c} lam_i phi_q_i dO_i^T,  r_c = sum_{i in c} lam_i D_i phi_q_i
//   for a key in the frames first linear for chunk c: dphi_k = R~_c v - r~_c, dv += R~_c^T phi_k,
//   with R~_c = sum_{c' >= c} R_c' (r~ likewise)
//   du = dphi * f'(u) (f the feature map's activation), then dx, dW, db through the grouped
//   linear.
#pragma once

#include <cuda_bf16.h>

#include "featmap.cuh"

namespace rehyat {
namespace bwd {

// D_i = dO_i . O_i and lam_i = 2^-lse2_i, one warp per row of D = 128 bf16.
//   grid (ceil(rows / 8), 1), block 256; rows = BH * N.
__global__ void __launch_bounds__(256) rowstats_kernel(const __nv_bfloat16* __restrict__ dO,
                                                       const __nv_bfloat16* __restrict__ O,
                                                       const float* __restrict__ lse2,
                                                       long long rows, int D,
                                                       float* __restrict__ Drow,
                                                       float* __restrict__ lam) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int d = lane * 2; d < D; d += 64) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(dO + row * D + d);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(O + row * D + d);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    acc = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, acc));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    Drow[row] = acc;
    lam[row] = exp2f(-lse2[row]);
  }
}

// dphi_q = lam (G - D Z_c) for the nq rows of one chunk (G = dO S_c^T, fp32 [BH][nq][F]), into
// dphi [BH][N][F] rows from row0; also phi_s = lam phi_q (bf16 [BH][nq][F]) for R_c.
//   grid (nq, BH), block F.
__global__ void phiq_grad_kernel(const float* __restrict__ G, int nq, int F, long long N,
                                 long long row0, const float* __restrict__ lam,
                                 const float* __restrict__ Drow, const float* __restrict__ Zc,
                                 long long z_bh_stride, const __nv_bfloat16* __restrict__ phiq,
                                 float* __restrict__ dphi, __nv_bfloat16* __restrict__ phi_s) {
  const int i = blockIdx.x, bh = blockIdx.y, f = threadIdx.x;
  const long long srow = (long long)bh * N + row0 + i;
  const float lm = lam[srow], Di = Drow[srow];
  const float g = G[((long long)bh * nq + i) * F + f];
  dphi[srow * F + f] = lm * (g - Di * Zc[(long long)bh * z_bh_stride + f]);
  phi_s[((long long)bh * nq + i) * F + f] =
      __float2bfloat16_rn(lm * __bfloat162float(phiq[srow * F + f]));
}

// Partial sums of r_c = sum_i lam_i D_i phi_q_i over blocks of kRBlock rows of one chunk:
// rpart [BH][nblk][F].  grid (nblk, BH), block F.
constexpr int kRBlock = 64;
__global__ void rpart_kernel(int nq, int F, long long N, long long row0,
                             const float* __restrict__ lam, const float* __restrict__ Drow,
                             const __nv_bfloat16* __restrict__ phiq, float* __restrict__ rpart,
                             int nblk) {
  const int blk = blockIdx.x, bh = blockIdx.y, f = threadIdx.x;
  float acc = 0.f;
  const int i1 = min(nq, (blk + 1) * kRBlock);
  for (int i = blk * kRBlock; i < i1; ++i) {
    const long long srow = (long long)bh * N + row0 + i;
    acc = fmaf(lam[srow] * Drow[srow], __bfloat162float(phiq[srow * F + f]), acc);
  }
  rpart[((long long)bh * nblk + blk) * F + f] = acc;
}

// r_c = the sum of its rpart blocks ([C][BH][nblk][F], zeros for chunks without a linear
// region), into r [BH][C][F].  grid (C, BH), block F.
__global__ void rreduce_kernel(const float* __restrict__ rpart, int nblk, int F,
                               float* __restrict__ r) {
  const int c = blockIdx.x, bh = blockIdx.y, BH = gridDim.y, C = gridDim.x, f = threadIdx.x;
  float acc = 0.f;
  for (int b = 0; b < nblk; ++b) acc += rpart[(((long long)c * BH + bh) * nblk + b) * F + f];
  r[((long long)bh * C + c) * F + f] = acc;
}

// Suffix sums over chunks: Rt_c = sum_{c' >= c} R_c' (bf16 [BH][C][F][D], R fp32, chunks
// without a linear region hold zeros) and rt_c = sum_{c' >= c} r_c' (fp32 [BH][C][F], in place
// over r).
//   grid (ceil(F*D / 256), BH), block 256.
__global__ void suffix_kernel(const float* __restrict__ R, int C, int F, int D,
                              __nv_bfloat16* __restrict__ Rt, float* __restrict__ rt) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const long long FD = (long long)F * D;
  if (e < FD) {
    float acc = 0.f;
    for (int c = C - 1; c >= 0; --c) {
      const long long o = ((long long)bh * C + c) * FD + e;
      acc += R[o];
      Rt[o] = __float2bfloat16_rn(acc);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x < F) {
    float acc = 0.f;
    for (int c = C - 1; c >= 0; --c) {
      acc += rt[((long long)bh * C + c) * F + threadIdx.x];
      rt[((long long)bh * C + c) * F + threadIdx.x] = acc;
    }
  }
}

// du = (g - rsub) * f'(u + bias) for rows [row0, row1) of every (b, h) (others untouched), where
// g is the incoming gradient of phi (fp32 [BH][N][F]) and rsub (fp32 [BH][C][F] or null) is
// subtracted with chunk index cidx(row) = (frame + To) / Tc + 1 (the first chunk that reads the
// key linearly).  f' of the polynomial map on part p: p softplus^(p-1) sigmoid; of elu + 1:
// 1 (u > 0) or e^u (P = 0).  du in bf16 [BH][N][F] for the products that follow.
//   grid (ceil((row1 - row0) / kFeatRows), BH), block F; each block takes kFeatRows rows.
constexpr int kFeatRows = 16;
__global__ void feat_grad_kernel(const float* __restrict__ U, const float* __restrict__ bias,
                                 int H, const float* __restrict__ g,
                                 const float* __restrict__ rsub, int C, int L, int Tc, int To,
                                 int F, int P, long long N, long long row0, long long row1,
                                 __nv_bfloat16* __restrict__ du) {
  const int bh = blockIdx.y, f = threadIdx.x, h = bh % H;
  const float b = bias ? bias[(long long)h * F + f] : 0.f;
  const int p = P == 0 ? 0 : part_power(f, F, P);  // this thread's feature: one power
  const long long r0 = row0 + (long long)blockIdx.x * kFeatRows;
  const long long r1 = min(row1, r0 + kFeatRows);
  for (long long row = r0; row < r1; ++row) {
    const long long o = ((long long)bh * N + row) * F + f;
    const float u = U[o] + b;
    float gv = g[o];
    if (rsub) {
      const int c = (int)((row / L + To) / Tc) + 1;
      gv -= rsub[((long long)bh * C + c) * F + f];
    }
    float fp;
    if (p == 0) {
      fp = u > 0.f ? 1.f : __expf(u);
    } else {
      const float sig = __fdividef(1.f, 1.f + __expf(-u));
      fp = sig;
      if (p > 1) fp = (float)p * int_pow(softplus_fast(u), p - 1) * sig;
    }
    du[o] = __float2bfloat16_rn(gv * fp);
  }
}

// Column sums of du (bf16 [BH][N][F]) over blocks of 256 rows of [row0, row1):
// part [BH][nblk][F].  grid (nblk, BH), block F.
__global__ void colsum_part_kernel(const __nv_bfloat16* __restrict__ du, int F, long long N,
                                   long long row0, long long row1, float* __restrict__ part,
                                   int nblk) {
  const int blk = blockIdx.x, bh = blockIdx.y, f = threadIdx.x;
  const long long r0 = row0 + (long long)blk * 256;
  const long long r1 = min(row1, r0 + 256);
  float acc = 0.f;
  for (long long r = r0; r < r1; ++r) acc += __bfloat162float(du[((long long)bh * N + r) * F + f]);
  part[((long long)bh * nblk + blk) * F + f] = acc;
}

// db[h][f] += the partial sums of every batch b and row block, in a fixed order.
//   grid (H), block F.
__global__ void bias_grad_kernel(const float* __restrict__ part, int B, int H, int F, int nblk,
                                 float* __restrict__ db) {
  const int h = blockIdx.x, f = threadIdx.x;
  float acc = 0.f;
  for (int b = 0; b < B; ++b)
    for (int k = 0; k < nblk; ++k) acc += part[((long long)(b * H + h) * nblk + k) * F + f];
  db[(long long)h * F + f] += acc;
}

// dW[h][g][o][i] += dWbd[h][g Fg + o][g Dg + i]: the diagonal blocks of the block-diagonal
// weight gradient.  grid (ceil(F*Dg / 256), H), block 256.
__global__ void blockdiag_grad_kernel(const float* __restrict__ dWbd, int D, int F, int G,
                                      float* __restrict__ dW) {
  const int h = blockIdx.y;
  const int Fg = F / G, Dg = D / G;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // over F * Dg
  if (e >= F * Dg) return;
  const int f = e / Dg, i = e - f * Dg, g = f / Fg;
  dW[(long long)h * F * Dg + e] += dWbd[((long long)h * F + f) * D + g * Dg + i];
}

}  // namespace bwd
}  // namespace rehyat

