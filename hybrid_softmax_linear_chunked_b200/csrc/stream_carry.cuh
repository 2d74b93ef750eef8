// Window assembly for the streaming step with carried frames ("ReHyAt overview" page §2.3 and
// §5.2: between chunks only S, Z and the overlap frames are kept).  The caller keeps the last
// `cap` frames of K and V it has seen (the carry, right-aligned); each call builds the softmax
// window [last ov carried frames | the chunk] and the next carry [the last cap frames of
// (carry ++ chunk)] in one pass of 16-byte copies, per (b, h):
//   window rows [0, ov L)           <- carry rows [(cap - ov) L, cap L)
//   window rows [ov L, (ov + cf) L) <- chunk rows [0, cf L)
//   new carry frame f (0 <= f < cap) <- chunk frame f - (cap - cf) if f >= cap - cf,
//                                       else carry frame f + cf
// The new carry goes to a separate buffer (the old one is still being read).  With
// window_out = 0 only the new carry is written (the kernels read the window in place).
#pragma once

#include <cstdint>

namespace rehyat {
namespace carry {

struct Params {
  int L;          // rows per frame
  int ov, cf;     // overlap frames taken from the carry, chunk frames
  int cap;        // carried frames
  int row_vec;    // 16-byte vectors per row
  int window_out; // 1: also write the window
  const uint4* carry;   // [BH][cap L][row]
  const uint4* chunk;   // [BH][cf L][row]
  uint4* window;        // [BH][(ov + cf) L][row]
  uint4* carry_new;     // [BH][cap L][row]
};

// grid (x, BH), block 256; threads stride over the (window + new carry) vectors of one (b, h).
__global__ void __launch_bounds__(256) gather_kernel(const Params p) {
  const long long bh = blockIdx.y;
  const long long L = p.L;
  const long long win_rows = p.window_out ? (long long)(p.ov + p.cf) * L : 0LL;
  const long long cap_rows = (long long)p.cap * L;
  const long long chunk_rows = (long long)p.cf * L;
  const long long total = (win_rows + cap_rows) * p.row_vec;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / p.row_vec;
    const int c = (int)(i - row * p.row_vec);
    long long src_row;
    const uint4* src;
    uint4* dst;
    if (row < win_rows) {
      dst = p.window + (bh * win_rows + row) * p.row_vec + c;
      if (row < (long long)p.ov * L) {
        src = p.carry;
        src_row = bh * cap_rows + (long long)(p.cap - p.ov) * L + row;
      } else {
        src = p.chunk;
        src_row = bh * chunk_rows + row - (long long)p.ov * L;
      }
    } else {
      const long long r = row - win_rows;
      const int f = (int)(r / L);
      const long long rr = r - (long long)f * L;
      dst = p.carry_new + (bh * cap_rows + r) * p.row_vec + c;
      if (f >= p.cap - p.cf) {
        src = p.chunk;
        src_row = bh * chunk_rows + (long long)(f - (p.cap - p.cf)) * L + rr;
      } else {
        src = p.carry;
        src_row = bh * cap_rows + (long long)(f + p.cf) * L + rr;
      }
    }
    *dst = src[src_row * p.row_vec + c];
  }
}

}  // namespace carry
}  // namespace rehyat
