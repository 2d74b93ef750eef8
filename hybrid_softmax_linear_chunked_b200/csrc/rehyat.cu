// librehyat.so: host side of the C ABI declared in include/rehyat.h.  Argument checks, workspace
// carving, TMA tensor-map encoding and kernel launches; every kernel of the library is compiled
// in this one translation unit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/rehyat.h"
#include "attn_bf16.cuh"
#include "attn_bwd_bf16.cuh"
#include "featmap.cuh"
#include "fp32_path.cuh"
#include "backward.cuh"
#include "gemm_bf16.cuh"
#include "phi_bf16.cuh"
#include "sm100.cuh"
#include "state_bf16.cuh"
#include "stream_carry.cuh"

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(REHYAT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return REHYAT_OK;
}

#define RH_TRY(expr)                 \
  do {                               \
    int rh_status_ = (expr);         \
    if (rh_status_ != REHYAT_OK) return rh_status_; \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The kernels take the part count P with P = 0 standing for the elu + 1 map.
int kernel_P(const rehyat_dims& d) { return d.phi == REHYAT_PHI_ELU1 ? 0 : d.P; }

int check_dims(const rehyat_dims& d, rehyat_dtype dt) {
  if (d.B < 1 || d.H < 1 || d.D < 1 || d.F < 1 || d.G < 1 || d.P < 1)
    return fail(REHYAT_ERR_ARG, "dims must be positive (B=%d H=%d D=%d F=%d G=%d P=%d)", d.B, d.H,
                d.D, d.F, d.G, d.P);
  if (d.D % d.G || d.F % d.G)
    return fail(REHYAT_ERR_ARG, "G=%d must divide D=%d and F=%d", d.G, d.D, d.F);
  if (d.P > d.F) return fail(REHYAT_ERR_ARG, "P=%d exceeds F=%d", d.P, d.F);
  if (d.phi != REHYAT_PHI_POLY && d.phi != REHYAT_PHI_ELU1)
    return fail(REHYAT_ERR_ARG, "unknown feature map kind phi=%d", d.phi);
  if (dt != REHYAT_F32 && dt != REHYAT_BF16) return fail(REHYAT_ERR_DTYPE, "unknown dtype %d", (int)dt);
  return REHYAT_OK;
}

// Shapes the attention / state kernels support (the standalone feature map is more general).
int check_path_shape(const rehyat_dims& d, rehyat_dtype dt) {
  if (dt == REHYAT_BF16) {
    if (d.D != 128 || d.F != 128)
      return fail(REHYAT_ERR_SHAPE, "bf16 path needs D = F = 128 (got D=%d F=%d)", d.D, d.F);
  } else {
    if (d.D % 32 || d.D > rehyat::fp32::kMaxD || d.F > 256)
      return fail(REHYAT_ERR_SHAPE, "fp32 path needs D %% 32 == 0, D <= 256, F <= 256 (D=%d F=%d)",
                  d.D, d.F);
  }
  return REHYAT_OK;
}

int check_sched(int T, int L, int Tc, int To) {
  if (T < 1 || L < 1) return fail(REHYAT_ERR_ARG, "need T >= 1 and frame_tokens >= 1 (T=%d L=%d)", T, L);
  if (Tc < 1 || To < 0) return fail(REHYAT_ERR_ARG, "need Tc >= 1 and To >= 0 (Tc=%d To=%d)", Tc, To);
  if ((long long)T * L > (1LL << 30)) return fail(REHYAT_ERR_ARG, "sequence too long");
  return REHYAT_OK;
}

// ---------------------------------------------------------------------------------------------
// TMA tensor maps
// ---------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || !p || q != cudaDriverEntryPointSuccess)
      return fail(REHYAT_ERR_CUDA, "cuTensorMapEncodeTiled not available");
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  *out = fn;
  return REHYAT_OK;
}

// bf16 [outer][rows][cols] tensor, loaded as 128-row x 64-column boxes with 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, int cols, long long rows, long long outer) {
  EncodeTiledFn enc;
  RH_TRY(get_encoder(&enc));
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * 2 * (cuuint64_t)rows};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(REHYAT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return REHYAT_OK;
}

// fp32 [outer][rows][cols] tensor, boxes of 32 columns (128 bytes) by 128 rows, 128-byte swizzle:
// the target of the backward's TMA reduce-adds.
int make_map_f32(CUtensorMap* m, const void* base, int cols, long long rows, long long outer) {
  EncodeTiledFn enc;
  RH_TRY(get_encoder(&enc));
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)cols * 4 * (cuuint64_t)rows};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(REHYAT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return REHYAT_OK;
}

// bf16 [outer][rows][cols] tensor with explicit strides (elements), box {box_cols, box_rows, 1}.
int make_map_strided(CUtensorMap* m, const void* base, long long cols, long long rows,
                     long long outer, long long row_stride, long long outer_stride, int box_cols,
                     int box_rows) {
  EncodeTiledFn enc;
  RH_TRY(get_encoder(&enc));
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)outer_stride * 2};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(REHYAT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return REHYAT_OK;
}

// A bf16 matrix operand of a batched GEMM: element (i, j) of batch b at
// ptr + b * batch_stride + i * ld + j, i.e. ld is the stride of the leading (non-contiguous)
// index, in elements.
struct Operand {
  const void* ptr;
  long long ld, batch_stride;
  bool mn;  // false: K contiguous; true: M (for A) or N (for B) contiguous
};

// C[b] (+)= alpha A[b] B[b] with A M x K, B K x N (layouts per Operand::mn), C [M][N] with row
// stride ldc.  Strides and bases must be 16-byte aligned (multiples of 8 elements).  With B2
// (same shape and layout as B, no split) the product is A (B + B2), summed in the accumulator.
int launch_gemm(int M, int N, int K, int batch, const Operand& A, const Operand& B, void* C,
                long long ldc, long long c_batch, bool c_bf16, bool accumulate, float alpha,
                cudaStream_t st, int split = 1, const Operand* B2 = nullptr) {
  if (split < 1 || (split > 1 && (c_bf16 || !accumulate)))
    return fail(REHYAT_ERR_ARG, "split-K GEMM needs fp32 output accumulated into C");
  if (B2 && (split > 1 || B2->mn != B.mn))
    return fail(REHYAT_ERR_ARG, "a two-part B needs split = 1 and one layout");
  if (M < 1 || N < 1 || K < 1 || batch < 1) return fail(REHYAT_ERR_ARG, "empty GEMM");
  if ((A.ld | A.batch_stride | B.ld | B.batch_stride) & 7)
    return fail(REHYAT_ERR_ALIGN, "GEMM operand strides must be multiples of 8 elements");
  if (!aligned16(A.ptr) || !aligned16(B.ptr) || !aligned16(C) || (!c_bf16 && ((ldc | c_batch) & 3)))
    return fail(REHYAT_ERR_ALIGN, "GEMM pointers must be 16-byte aligned");
  if (B2 && (!aligned16(B2->ptr) || ((B2->ld | B2->batch_stride) & 7)))
    return fail(REHYAT_ERR_ALIGN, "GEMM pointers must be 16-byte aligned");
  CUtensorMap ma, mb, mb2;
  if (A.mn) RH_TRY(make_map_strided(&ma, A.ptr, M, K, batch, A.ld, A.batch_stride, 64, 64));
  else RH_TRY(make_map_strided(&ma, A.ptr, K, M, batch, A.ld, A.batch_stride, 64, 128));
  if (B.mn) RH_TRY(make_map_strided(&mb, B.ptr, N, K, batch, B.ld, B.batch_stride, 64, 64));
  else RH_TRY(make_map_strided(&mb, B.ptr, K, N, batch, B.ld, B.batch_stride, 64, 128));
  if (B2) {
    if (B2->mn) RH_TRY(make_map_strided(&mb2, B2->ptr, N, K, batch, B2->ld, B2->batch_stride, 64, 64));
    else RH_TRY(make_map_strided(&mb2, B2->ptr, K, N, batch, B2->ld, B2->batch_stride, 64, 128));
  } else {
    mb2 = mb;
  }
  rehyat::gemm::Params gp{};
  gp.M = M; gp.N = N; gp.K = K; gp.a_mn = A.mn; gp.b_mn = B.mn;
  gp.C = C; gp.ldc = ldc; gp.c_batch = c_batch; gp.c_bf16 = c_bf16; gp.accumulate = accumulate;
  gp.alpha = alpha;
  gp.split = split;
  gp.b_parts = B2 ? 2 : 1;
  // a K loop of at most four 64-deep slices per CTA runs on the 2-stage ring (three CTAs per SM)
  const int slices = (int)((((K + 63) / 64) + split - 1) / split) * gp.b_parts;
  const bool short_k = slices <= 4;
  auto k = short_k ? rehyat::gemm::gemm_bf16_kernel<2> : rehyat::gemm::gemm_bf16_kernel<4>;
  const uint32_t smem = rehyat::gemm::smem_bytes(short_k ? 2 : 4);
  RH_TRY(cuda_check(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem), "gemm attr"));
  dim3 grid((N + 127) / 128, (M + 127) / 128, batch * split);
  k<<<grid, rehyat::gemm::kThreads, smem, st>>>(ma, mb, mb2, gp);
  return cuda_check(cudaGetLastError(), "gemm launch");
}

// ---------------------------------------------------------------------------------------------
// Workspace plans
// ---------------------------------------------------------------------------------------------
struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  }
};

int fold_splits(int BH, int n_fold, long long rows_per_fold) {
  if (n_fold <= 0) return 1;
  const long long tiles = (rows_per_fold + 127) / 128;
  // one wave of the one-CTA-per-SM fold kernel: long loops amortise each CTA's set-up
  long long want = 148LL / ((long long)BH * n_fold);
  long long s = want < 1 ? 1 : want;
  const long long max_s = tiles / 2 > 0 ? tiles / 2 : 1;
  if (s > max_s) s = max_s;
  if (s > 16) s = 16;
  return (int)s;
}

// Token splits of one fold range in the whole-sequence forward (and its segments): a function
// of the range's length only, about 18 tiles of 128 tokens per split and at most 16, so that
// every (b, h) is folded in the same order whatever other (b, h) share the call (a head-sharded
// run reproduces the one-call result bit for bit).
int fold_splits_shape(long long rows_per_fold) {
  const long long tiles = (rows_per_fold + 127) / 128;
  long long s = (tiles + 8) / 18;
  if (s < 1) s = 1;
  if (s > 16) s = 16;
  return (int)s;
}

// Parts a chunk's lone last tile is cut into (its key window spread over that many short CTAs,
// which fill the attention's last wave instead of forming a wave of their own), at most
// kMaxLoneSplit; every part keeps at least one key tile.
constexpr int kMaxLoneSplit = 4;
int lone_split_count(int min_key_tiles) {
  int k = kMaxLoneSplit;
  if (k > min_key_tiles) k = min_key_tiles;
  return k < 1 ? 1 : k;
}
// Scratch for the parts of the lone tiles of `n_chunks` chunks: O [128][D] and (m, l) per row.
size_t lone_part_bytes(size_t BH, int n_chunks, int D) {
  return BH * n_chunks * kMaxLoneSplit * 128 * ((size_t)D + 2) * 4;
}

// Lone-tile split of an attention launch over chunks [0, n_chunks) whose chunk c owns frames
// [frames_before + c*Tc, min(frames_before + (c+1)*Tc, frames_before + T)) and reads a window
// reaching To frames back: parts per lone tile (1 when no chunk has one, or when not allowed) and
// the grid's slot count per (b, h).
struct LoneSplit {
  int n_split, slots;
};
LoneSplit lone_split_plan(int T, int L, int Tc, int To, int frames_before, int n_chunks,
                          bool allow) {
  int max_tiles = 0, min_key = 1 << 30;
  bool any_lone = false;
  for (int c = 0; c < n_chunks; ++c) {
    const int gs = frames_before + c * Tc;
    const int ge = gs + Tc < frames_before + T ? gs + Tc : frames_before + T;
    const int gw = gs - To > 0 ? gs - To : 0;
    const int tiles = ((ge - gs) * L + 127) / 128;
    if (tiles > max_tiles) max_tiles = tiles;
    if (tiles & 1) {
      any_lone = true;
      const int key_tiles = ((ge - gw) * L + 127) / 128;
      if (key_tiles < min_key) min_key = key_tiles;
    }
  }
  LoneSplit r;
  r.n_split = (allow && any_lone) ? lone_split_count(min_key) : 1;
  r.slots = max_tiles / 2 + (any_lone ? r.n_split : 0);
  return r;
}

struct ForwardPlan {
  int C, n_fold, splits;
  size_t dS, dZ, St, Zc, Wqbd, Wkbd, phiq_bf16, phiq, phik, Sc, part, total;
};

ForwardPlan plan_forward(const rehyat_dims& d, rehyat_dtype dt, int T, int L, int Tc, int To) {
  ForwardPlan p{};
  const size_t BH = (size_t)d.B * d.H;
  p.C = (T + Tc - 1) / Tc;
  p.n_fold = p.C - 1;
  Carve cv;
  if (dt == REHYAT_BF16) {
    p.splits = fold_splits_shape((long long)Tc * L);
    const size_t nf = p.n_fold > 0 ? p.n_fold : 0;
    p.dS = cv.take(BH * nf * p.splits * d.F * d.D * 4);
    p.dZ = cv.take(BH * nf * p.splits * d.F * 4);
    p.St = cv.take(BH * p.C * d.D * d.F * 2);
    p.Zc = cv.take(BH * p.C * d.F * 4);
    p.Wqbd = cv.take((size_t)d.H * 2 * d.F * d.D * 2);
    p.Wkbd = cv.take((size_t)d.H * 2 * d.F * d.D * 2);
    p.phiq_bf16 = cv.take(BH * (size_t)T * L * d.F * 2);
    p.part = cv.take(lone_part_bytes(BH, p.C, d.D));
  } else {
    p.splits = 1;
    const size_t N = (size_t)T * L;
    const size_t nf = p.n_fold > 0 ? p.n_fold : 0;
    p.phiq = cv.take(BH * N * d.F * 4);
    p.phik = cv.take(BH * N * d.F * 4);
    p.dS = cv.take(BH * nf * d.F * d.D * 4);
    p.dZ = cv.take(BH * nf * d.F * 4);
    p.Sc = cv.take(BH * p.C * d.F * d.D * 4);
    p.Zc = cv.take(BH * p.C * d.F * 4);
  }
  p.total = cv.off;
  return p;
}

struct ChunkPlan {
  int o, nq, nkv, fold_rows, splits;
  size_t St, dS, dZ, Wqbd, Wkbd, phiq_bf16, phiq, phik, part, total;
};

ChunkPlan plan_chunk(const rehyat_dims& d, rehyat_dtype dt, int L, int frames_before,
                     int chunk_frames, int To, int To_next) {
  ChunkPlan p{};
  const size_t BH = (size_t)d.B * d.H;
  p.o = To < frames_before ? To : frames_before;
  p.nq = chunk_frames * L;
  p.nkv = (p.o + chunk_frames) * L;
  const int w = frames_before - p.o;
  int w_next = frames_before + chunk_frames - To_next;
  if (w_next < 0) w_next = 0;
  p.fold_rows = (w_next - w) * L;
  if (p.fold_rows < 0) p.fold_rows = 0;
  Carve cv;
  if (dt == REHYAT_BF16) {
    // the split count depends only on the chunk length so that one workspace size fits every
    // call of a stream
    p.splits = fold_splits((int)BH, 1, (long long)chunk_frames * L);
    p.St = cv.take(BH * d.D * d.F * 2);
    p.dS = cv.take(BH * p.splits * d.F * d.D * 4);
    p.dZ = cv.take(BH * p.splits * d.F * 4);
    p.Wqbd = cv.take((size_t)d.H * 2 * d.F * d.D * 2);
    p.Wkbd = cv.take((size_t)d.H * 2 * d.F * d.D * 2);
    p.phiq_bf16 = cv.take(BH * (size_t)p.nq * d.F * 2);
    p.part = cv.take(lone_part_bytes(BH, 1, d.D));
  } else {
    p.splits = 1;
    const size_t max_kv = (size_t)(To + chunk_frames) * L;
    p.phiq = cv.take(BH * (size_t)p.nq * d.F * 4);
    p.phik = cv.take(BH * max_kv * d.F * 4);
    p.dS = cv.take(BH * d.F * d.D * 4);
    p.dZ = cv.take(BH * d.F * 4);
  }
  p.total = cv.off;
  return p;
}

// A segment of chunks [c0, c1) of a T-frame sequence (context parallelism): its query frames
// [s0, s1), key/value frames [h0, s1) (the overlap halo first), its folds [c0, min(c1, C-1)).
struct SegPlan {
  int C, s0, s1, h0, n_local, n_fold, splits;
  long long nq_rows, nkv_rows;
  size_t dS, dZ, St, Zc, Wqbd, Wkbd, phiq_bf16, part, total;
};

SegPlan plan_segment(const rehyat_dims& d, int T, int L, int Tc, int To, int c0, int c1) {
  SegPlan p{};
  const size_t BH = (size_t)d.B * d.H;
  p.C = (T + Tc - 1) / Tc;
  p.s0 = c0 * Tc;
  p.s1 = c1 * Tc < T ? c1 * Tc : T;
  p.h0 = p.s0 - To > 0 ? p.s0 - To : 0;
  p.n_local = c1 - c0;
  const int fold_end = c1 < p.C - 1 ? c1 : p.C - 1;
  p.n_fold = fold_end > c0 ? fold_end - c0 : 0;
  p.nq_rows = (long long)(p.s1 - p.s0) * L;
  p.nkv_rows = (long long)(p.s1 - p.h0) * L;
  p.splits = fold_splits_shape((long long)Tc * L);
  Carve cv;
  const size_t nf = p.n_fold;
  p.dS = cv.take(BH * nf * p.splits * d.F * d.D * 4);
  p.dZ = cv.take(BH * nf * p.splits * d.F * 4);
  p.St = cv.take(BH * p.n_local * d.D * d.F * 2);
  p.Zc = cv.take(BH * p.n_local * d.F * 4);
  p.Wqbd = cv.take((size_t)d.H * 2 * d.F * d.D * 2);
  p.Wkbd = cv.take((size_t)d.H * 2 * d.F * d.D * 2);
  p.phiq_bf16 = cv.take(BH * (size_t)p.nq_rows * d.F * 2);
  p.part = cv.take(lone_part_bytes(BH, p.n_local, d.D));
  p.total = cv.off;
  return p;
}

// Streaming with carried frames: the chunk step's own workspace, then (fp32 only) the assembled K
// and V windows, then the next carry of K and V (used when the chunk is shorter than the carry).
// The bf16 kernels read the window straight from the carry and the chunk.
struct CarryPlan {
  size_t step, step_bytes, kwin, vwin, kcar, vcar, total;
};

CarryPlan plan_carry(const rehyat_dims& d, rehyat_dtype dt, int L, int chunk_frames, int To,
                     int cap) {
  CarryPlan p{};
  const size_t es = dt == REHYAT_BF16 ? 2 : 4;
  const size_t BH = (size_t)d.B * d.H;
  Carve cv;
  p.step_bytes = plan_chunk(d, dt, L, To, chunk_frames, To, To).total;
  p.step = cv.take(p.step_bytes);
  if (dt != REHYAT_BF16) {
    p.kwin = cv.take(BH * (size_t)(To + chunk_frames) * L * d.D * es);
    p.vwin = cv.take(BH * (size_t)(To + chunk_frames) * L * d.D * es);
  }
  p.kcar = cv.take(BH * (size_t)cap * L * d.D * es);
  p.vcar = cv.take(BH * (size_t)cap * L * d.D * es);
  p.total = cv.off;
  return p;
}

// ---------------------------------------------------------------------------------------------
// Launch helpers
// ---------------------------------------------------------------------------------------------
int launch_featmap(const rehyat_dims& d, rehyat_dtype dt, int n, const void* x, const float* W,
                   const float* b, void* phi, cudaStream_t st) {
  const size_t smem = ((size_t)d.F * d.D / d.G + d.F + 128 * (size_t)(d.D + 1)) * 4;
  if (smem > 227 * 1024)
    return fail(REHYAT_ERR_SHAPE, "feature map of D=%d F=%d G=%d needs %zu B of shared memory", d.D,
                d.F, d.G, smem);
  dim3 grid((n + 127) / 128, d.B * d.H);
  if (dt == REHYAT_BF16) {
    auto k = rehyat::featmap_kernel<__nv_bfloat16, __nv_bfloat16, false>;
    RH_TRY(cuda_check(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem), "featmap attr"));
    k<<<grid, 128, smem, st>>>(static_cast<const __nv_bfloat16*>(x), W, b,
                               static_cast<__nv_bfloat16*>(phi), n, d.H, d.D, d.F, d.G, kernel_P(d));
  } else {
    auto k = rehyat::featmap_kernel<float, float, true>;
    RH_TRY(cuda_check(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem), "featmap attr"));
    k<<<grid, 128, smem, st>>>(static_cast<const float*>(x), W, b, static_cast<float*>(phi), n,
                               d.H, d.D, d.F, d.G, kernel_P(d));
  }
  return cuda_check(cudaGetLastError(), "featmap launch");
}

template <bool kPhiGlobal>
int launch_attn_bf16(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& ms, const CUtensorMap& mw, const CUtensorMap& mphi,
                     const rehyat::attn::Params& ap, dim3 grid, cudaStream_t st,
                     const CUtensorMap* mkc = nullptr, const CUtensorMap* mvc = nullptr,
                     bool behind_phiq = false) {
  auto k = rehyat::attn::hybrid_attn_bf16_kernel<kPhiGlobal>;
  RH_TRY(cuda_check(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)rehyat::attn::kSmemBytes),
                    "attn attr"));
  // behind_phiq: the launch before this one, in the same call, is the library's phi_q kernel
  // (everything before that had finished when it started).  The kernel reads what earlier
  // launches wrote (S^T, Z_c, phi_q) only after waiting for that grid, so it is launched with
  // programmatic stream serialization and its key loop overlaps the phi_q kernel.  A caller's
  // own work right before an attention launch is never overlapped.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(rehyat::attn::kThreads);
  cfg.dynamicSmemBytes = rehyat::attn::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (kPhiGlobal && behind_phiq) ? 1 : 0;
  const CUtensorMap kc = mkc ? *mkc : mk, vc = mvc ? *mvc : mv;
  // the output [grid.y (b, h)][nq_rows][D] for the full query tiles' TMA stores
  CUtensorMap mo;
  RH_TRY(make_map(&mo, ap.out, rehyat::attn::kHD, ap.nq_rows, grid.y));
  return cuda_check(cudaLaunchKernelEx(&cfg, k, mq, mk, mv, ms, mw, mphi, kc, vc, mo, ap),
                    "attention launch");
}

// Merges the parts of the lone last tiles of a split attention launch into its output.
int launch_lone_combine(const rehyat::attn::Params& ap, int BH, int n_chunks, cudaStream_t st) {
  rehyat::attn::lone_combine_kernel<<<dim3(BH, n_chunks, 128), rehyat::attn::kHD, 0, st>>>(ap);
  return cuda_check(cudaGetLastError(), "lone-tile combine launch");
}

// phi of rows [row0, row0 + n_rows) of every (b, h) sequence of x (rows_per_bh rows each) into
// phi ([BH][rows_per_bh][F] bf16) on the tensor cores; W are the fp32 weights [H][G][F/G][D/G]
// (each CTA builds its head's compact block-diagonal matrix in shared memory).
template <bool kDense>
int launch_featmap_tc_inst(const rehyat_dims& d, const CUtensorMap& mx, const CUtensorMap& mphi,
                           int n_rows, rehyat::phi::Params pp, cudaStream_t st, bool behind_scan) {
  using Lay = rehyat::phi::Layout<kDense>;
  const int BH = d.B * d.H;
  const int n_tiles = (n_rows + 127) / 128;
  // one wave: as many CTAs per (b, h) as fit on the 148 SMs
  const int slots = 148 * Lay::kCtasPerSm;
  const int ctas_per_bh = BH < slots ? slots / BH : 1;
  int per_cta = (n_tiles + ctas_per_bh - 1) / ctas_per_bh;
  if (per_cta < 1) per_cta = 1;
  if (per_cta > n_tiles) per_cta = n_tiles;
  pp.tiles_per_cta = per_cta;
  auto k = rehyat::phi::featmap_tc_kernel<kDense>;
  RH_TRY(cuda_check(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lay::kSmemBytes),
                    "featmap_tc attr"));
  // behind_scan: the launch before this one, in the same call, is the library's state scan, whose
  // outputs this kernel does not read: launched with programmatic stream serialization, it starts
  // at once and waits for the scan's grid before it exits.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((n_tiles + per_cta - 1) / per_cta, BH);
  cfg.blockDim = dim3(rehyat::phi::kThreads);
  cfg.dynamicSmemBytes = Lay::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = behind_scan ? 1 : 0;
  return cuda_check(cudaLaunchKernelEx(&cfg, k, mx, mphi, pp), "featmap_tc launch");
}

int launch_featmap_tc(const rehyat_dims& d, const void* x, int rows_per_bh, int row0, int n_rows,
                      const float* W, const float* bias, __nv_bfloat16* phi, cudaStream_t st,
                      bool behind_scan = false) {
  if (n_rows <= 0) return REHYAT_OK;
  const long long BH = (long long)d.B * d.H;
  CUtensorMap mx, mphi;
  RH_TRY(make_map(&mx, x, d.D, rows_per_bh, BH));
  // phi rows [row0, row0 + n_rows) of each (b, h): the map's row extent ends there, so a ragged
  // last tile's store writes nothing past the range
  RH_TRY(make_map_strided(&mphi, phi, d.F, (long long)row0 + n_rows, BH, d.F,
                          (long long)rows_per_bh * d.F, 64, 128));
  rehyat::phi::Params pp{};
  pp.row0 = row0; pp.n_rows = n_rows; pp.rows_per_bh = rows_per_bh;
  pp.H = d.H; pp.P = kernel_P(d); pp.G = d.G; pp.W = W; pp.bias = bias;
  // the G = 1 matrix is dense (32 KB per part): its instance runs one CTA per SM
  if (rehyat::compact_w(d.F, d.D, d.G).NT > 64)
    return launch_featmap_tc_inst<true>(d, mx, mphi, n_rows, pp, st, behind_scan);
  return launch_featmap_tc_inst<false>(d, mx, mphi, n_rows, pp, st, behind_scan);
}

// behind_attention: launch with programmatic stream serialization right after an attention
// launch, so the fold starts once every attention CTA is resident (the kernel waits for the
// attention grid before it exits).
template <int kKSt>
int launch_fold_inst(const CUtensorMap& mk, const CUtensorMap& mv,
                     const rehyat::state::FoldParams& fp, dim3 grid, cudaStream_t st,
                     const CUtensorMap* mkc, const CUtensorMap* mvc, bool behind_attention) {
  using Lay = rehyat::state::FoldLayout<kKSt>;
  auto k = rehyat::state::fold_partial_bf16_kernel<kKSt>;
  RH_TRY(cuda_check(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lay::kSmemBytes),
                    "fold attr"));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(rehyat::state::kThreads);
  cfg.dynamicSmemBytes = Lay::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = behind_attention ? 1 : 0;
  const CUtensorMap kc = mkc ? *mkc : mk, vc = mvc ? *mvc : mv;
  return cuda_check(cudaLaunchKernelEx(&cfg, k, mk, mv, kc, vc, fp), "fold launch");
}

// The fold kernel over `grid` (splits, folds, BH); fp.W / fp.G are the fp32 weights of phi_k.
int launch_fold_bf16(const CUtensorMap& mk, const CUtensorMap& mv,
                     const rehyat::state::FoldParams& fp, dim3 grid, cudaStream_t st,
                     const CUtensorMap* mkc = nullptr, const CUtensorMap* mvc = nullptr,
                     bool behind_attention = false) {
  // two K stages unless the weights are the dense G = 1 matrix
  if (rehyat::compact_w(rehyat::state::kFD, rehyat::state::kHD, fp.G).NT > 64)
    return launch_fold_inst<1>(mk, mv, fp, grid, st, mkc, mvc, behind_attention);
  return launch_fold_inst<2>(mk, mv, fp, grid, st, mkc, mvc, behind_attention);
}

// Block-diagonal bf16 hi/lo weights of one feature map into `out` ([H][2][F][D] bf16) and the
// tensor map the kernels load them with.
int prepare_blockdiag(const rehyat_dims& d, const float* W, __nv_bfloat16* out, CUtensorMap* map,
                      cudaStream_t st) {
  rehyat::blockdiag_weights_kernel<<<dim3((d.F * d.D + 2047) / 2048, d.H), 256, 0, st>>>(
      W, d.D, d.F, d.G, out);
  RH_TRY(cuda_check(cudaGetLastError(), "block-diagonal weights launch"));
  return make_map(map, out, d.D, d.F, 2LL * d.H);
}

// S0/Z0: n_prefix stacked initial states ([n_prefix][BH][F][D], [n_prefix][BH][F]) summed in
// order, or null for zero.
int launch_scan_bf16(const rehyat_dims& d, const float* dS, const float* dZ, int n_fold,
                     int splits, int C, const float* S0, const float* Z0, __nv_bfloat16* St,
                     float* Zc, float* S_out, float* Z_out, cudaStream_t st, int n_prefix = 1) {
  dim3 grid((d.F / 32) * (d.D / 32), d.B * d.H);
  rehyat::state::state_scan_kernel<<<grid, dim3(32, 8), 0, st>>>(
      dS, dZ, n_fold, splits, C, d.F, d.D, S0, Z0, n_prefix, St, Zc, S_out, Z_out);
  return cuda_check(cudaGetLastError(), "scan launch");
}

// Enqueue the bf16 fold partials of the forward schedule and their scan.
int forward_states_bf16(const rehyat_dims& d, int T, int L, int Tc, int To, const void* k,
                        const void* v, const float* Wk, const float* bk, const ForwardPlan& pl,
                        uint8_t* ws, __nv_bfloat16* St, float* Zc, float* S_out, float* Z_out,
                        cudaStream_t st) {
  const long long N = (long long)T * L;
  const int BH = d.B * d.H;
  float* dS = reinterpret_cast<float*>(ws + pl.dS);
  float* dZ = reinterpret_cast<float*>(ws + pl.dZ);
  if (pl.n_fold > 0) {
    CUtensorMap mk, mv;
    RH_TRY(make_map(&mk, k, d.D, N, BH));
    RH_TRY(make_map(&mv, v, d.D, N, BH));
    rehyat::state::FoldParams fp{};
    fp.L = L; fp.H = d.H; fp.P = kernel_P(d); fp.T = T; fp.Tc = Tc; fp.To = To; fp.kv_frame0 = 0;
    fp.single_rows = -1; fp.n_fold = pl.n_fold; fp.splits = pl.splits;
    fp.kv_rows = fp.carry_rows = (int)N;
    fp.G = d.G; fp.W = Wk; fp.bk = bk; fp.dS = dS; fp.dZ = dZ;
    RH_TRY(launch_fold_bf16(mk, mv, fp, dim3(pl.splits, pl.n_fold, BH), st));
  }
  return launch_scan_bf16(d, dS, dZ, pl.n_fold, pl.splits, pl.C, nullptr, nullptr, St, Zc, S_out,
                          Z_out, st);
}

int forward_states_f32(const rehyat_dims& d, int T, int L, int Tc, int To, const void* k,
                       const void* v, const float* Wk, const float* bk, const ForwardPlan& pl,
                       uint8_t* ws, float* Sc, float* Zc, cudaStream_t st) {
  const int N = T * L;
  float* phik = reinterpret_cast<float*>(ws + pl.phik);
  float* dS = reinterpret_cast<float*>(ws + pl.dS);
  float* dZ = reinterpret_cast<float*>(ws + pl.dZ);
  RH_TRY(launch_featmap(d, REHYAT_F32, N, k, Wk, bk, phik, st));
  if (pl.n_fold > 0) {
    rehyat::fp32::FoldParams fp{};
    fp.L = L; fp.T = T; fp.Tc = Tc; fp.To = To; fp.kv_frame0 = 0; fp.single_rows = -1;
    fp.n_fold = pl.n_fold; fp.F = d.F; fp.D = d.D; fp.nkv_rows = N;
    fp.phik = phik; fp.v = static_cast<const float*>(v); fp.dS = dS; fp.dZ = dZ;
    rehyat::fp32::fold_partial_f32_kernel<<<dim3(pl.n_fold, d.B * d.H), 256, 0, st>>>(fp);
    RH_TRY(cuda_check(cudaGetLastError(), "fold f32 launch"));
  }
  rehyat::fp32::state_scan_f32_kernel<<<dim3((d.F * d.D + 255) / 256, d.B * d.H), 256, 0, st>>>(
      dS, dZ, pl.n_fold, pl.C, d.F, d.D, nullptr, nullptr, Sc, Zc);
  return cuda_check(cudaGetLastError(), "scan f32 launch");
}

// ---------------------------------------------------------------------------------------------
// Library-owned scratch for rehyat_chunk_forward_static (callers that cannot allocate device
// memory themselves).  A fixed array in the module's device memory: every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits.
// ---------------------------------------------------------------------------------------------
constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mutex;
void* g_static_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device.  The host-side name of the array is
// only a stand-in, so the address is looked up once per device (with that device current) and
// cached.
int static_scratch_for_current_device(void** out) {
  int dev = -1;
  RH_TRY(cuda_check(cudaGetDevice(&dev), "cudaGetDevice"));
  if (dev < 0 || dev >= kMaxDevices) return fail(REHYAT_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_ptr[dev]) {
    void* p = nullptr;
    RH_TRY(cuda_check(cudaGetSymbolAddress(&p, g_static_scratch), "cudaGetSymbolAddress(scratch)"));
    g_static_scratch_ptr[dev] = p;
  }
  *out = g_static_scratch_ptr[dev];
  return REHYAT_OK;
}

// Debug-bounds self test: writes 1 to buf[0, n) and then tries buf[bad_index] through the store
// check (index inside [0, n)), which a debug-bounds build records and skips.  The caller's buffer
// has room past n, so the write would stay inside it even if the check were missing.
__global__ void __launch_bounds__(256) bounds_selftest_kernel(float* buf, long long n,
                                                              long long bad_index) {
  const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
  if (i < n) buf[i] = 1.f;
  if (i == 0 && rehyat::sm100::bounds_ok(99, bad_index, 0, n)) buf[bad_index] = 2.f;
}

// Exercises the error path of the bounded mbarrier wait: every warp waits on a barrier that
// nothing arrives on.  The first wait to pass `limit_ns` raises the CTA's abort flag and sets
// the device error word; the other warps see the flag and return too.
__global__ void __launch_bounds__(64) wait_timeout_selftest_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    rehyat::sm100::mbar_init(&bar, 1);
    abort_sh = 0;
    rehyat::sm100::fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &abort_sh;
  rehyat::sm100::mbar_wait(&bar, 0, abort_flag, limit_ns);
  __syncthreads();
}

}  // namespace

// =============================================================================================
// C ABI
// =============================================================================================
// ---------------------------------------------------------------------------------------------
// Backward workspace: the forward's (states, phi_q), then the backward's own buffers.
// ---------------------------------------------------------------------------------------------
struct BackwardPlan {
  ForwardPlan fwd;
  int C, c_lin, nq_max, nw_max, nblk_r, nblk_b;
  size_t fwd_off, fwd_bytes, phik, Drow, lam, GB, phis, dphiq, dphik, U, DU, RB, Rt, rpart, rt,
      dWbd, dbpart, total;
};

BackwardPlan plan_backward(const rehyat_dims& d, int T, int L, int Tc, int To) {
  BackwardPlan p{};
  p.fwd = plan_forward(d, REHYAT_BF16, T, L, Tc, To);
  const size_t BH = (size_t)d.B * d.H, N = (size_t)T * L, F = d.F, D = d.D;
  p.C = (T + Tc - 1) / Tc;
  p.c_lin = To / Tc + 1;  // first chunk with a linear region
  p.nq_max = (Tc < T ? Tc : T) * L;
  p.nw_max = ((Tc + To) < T ? (Tc + To) : T) * L;
  p.nblk_r = (p.nq_max + rehyat::bwd::kRBlock - 1) / rehyat::bwd::kRBlock;
  p.nblk_b = (int)((N + 255) / 256);
  Carve cv;
  p.fwd_off = cv.take(p.fwd.total);
  p.fwd_bytes = p.fwd.total;
  p.phik = cv.take(BH * N * F * 2);
  p.Drow = cv.take(BH * N * 4);
  p.lam = cv.take(BH * N * 4);
  p.GB = cv.take(BH * p.nq_max * F * 4);
  p.phis = cv.take(BH * p.nq_max * F * 2);
  p.dphiq = cv.take(BH * N * F * 4);
  p.dphik = cv.take(BH * N * F * 4);
  p.U = cv.take(BH * N * F * 4);
  p.DU = cv.take(BH * N * F * 2);
  p.RB = cv.take(BH * p.C * F * D * 4);
  p.Rt = cv.take(BH * p.C * F * D * 2);
  p.rpart = cv.take((size_t)p.C * BH * p.nblk_r * F * 4);
  p.rt = cv.take(BH * p.C * F * 4);
  p.dWbd = cv.take((size_t)d.H * F * D * 4);
  p.dbpart = cv.take(BH * p.nblk_b * F * 4);
  p.total = cv.off;
  return p;
}

// Feature-map backward of rows [r0, r1) of every (b, h): U = x Wbd^T, du = (g - rsub) f'(U + b),
// dx += du Wbd, dW += diag blocks of du^T x, db += column sums of du.
int feature_backward(const rehyat_dims& d, long long N, long long r0, long long r1,
                     const void* x, const __nv_bfloat16* Wbd, const float* bias, const float* g,
                     const float* rsub, int C, int L, int Tc, int To, const BackwardPlan& pl,
                     uint8_t* ws, float* dx, float* dW, float* db, cudaStream_t st) {
  if (r1 <= r0) return REHYAT_OK;
  const long long rows = r1 - r0, F = d.F, D = d.D;
  const int H = d.H, BH = d.B * d.H;
  float* U = reinterpret_cast<float*>(ws + pl.U);
  __nv_bfloat16* DU = reinterpret_cast<__nv_bfloat16*>(ws + pl.DU);
  float* dWbd = reinterpret_cast<float*>(ws + pl.dWbd);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  for (int b = 0; b < d.B; ++b) {
    const long long bo = (long long)b * H * N;  // first row of batch b
    // U = x (Wbd_hi + Wbd_lo)^T, both parts in one accumulator
    const Operand lo{Wbd + F * D, D, 2 * F * D, false};
    RH_TRY(launch_gemm((int)rows, (int)F, (int)D, H, Operand{xb + (bo + r0) * D, D, N * D, false},
                       Operand{Wbd, D, 2 * F * D, false}, U + (bo + r0) * F, F, N * F, false,
                       false, 1.f, st, 1, &lo));
  }
  rehyat::bwd::feat_grad_kernel<<<
      dim3((unsigned)((rows + rehyat::bwd::kFeatRows - 1) / rehyat::bwd::kFeatRows), BH), d.F, 0,
      st>>>(U, bias, H, g, rsub, C, L, Tc, To, d.F, kernel_P(d), N, r0, r1, DU);
  RH_TRY(cuda_check(cudaGetLastError(), "feature gradient launch"));
  RH_TRY(cuda_check(cudaMemsetAsync(dWbd, 0, (size_t)H * F * D * 4, st), "memset"));
  for (int b = 0; b < d.B; ++b) {
    const long long bo = (long long)b * H * N;
    // dx += du (Wbd_hi + Wbd_lo), both parts in one accumulator
    const Operand lo{Wbd + F * D, D, 2 * F * D, true};
    RH_TRY(launch_gemm((int)rows, (int)D, (int)F, H, Operand{DU + (bo + r0) * F, F, N * F, false},
                       Operand{Wbd, D, 2 * F * D, true}, dx + (bo + r0) * D, D, N * D, false,
                       true, 1.f, st, 1, &lo));
    // dWbd += du^T x over this batch's rows
    RH_TRY(launch_gemm((int)F, (int)D, (int)rows, H, Operand{DU + (bo + r0) * F, F, N * F, true},
                       Operand{xb + (bo + r0) * D, D, N * D, true}, dWbd, D, F * D, false, true,
                       1.f, st, 16));
  }
  rehyat::bwd::blockdiag_grad_kernel<<<dim3((unsigned)((F * (D / d.G) + 255) / 256), H), 256, 0,
                                       st>>>(dWbd, d.D, d.F, d.G, dW);
  RH_TRY(cuda_check(cudaGetLastError(), "weight gradient launch"));
  float* part = reinterpret_cast<float*>(ws + pl.dbpart);
  const int nblk = (int)((rows + 255) / 256);
  rehyat::bwd::colsum_part_kernel<<<dim3(nblk, BH), d.F, 0, st>>>(DU, d.F, N, r0, r1, part, nblk);
  RH_TRY(cuda_check(cudaGetLastError(), "bias gradient launch"));
  rehyat::bwd::bias_grad_kernel<<<H, d.F, 0, st>>>(part, d.B, H, d.F, nblk, db);
  return cuda_check(cudaGetLastError(), "bias gradient launch");
}

extern "C" {

const char* rehyat_last_error(void) { return g_msg; }

int rehyat_debug_bounds(void) {
#ifdef REHYAT_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

int rehyat_version(void) { return 102; }

int rehyat_featmap(rehyat_dims d, rehyat_dtype dt, int n_tokens, const void* x, const float* W,
                   const float* bias, void* phi, void* stream) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  if (n_tokens < 1) return fail(REHYAT_ERR_ARG, "n_tokens must be >= 1");
  if (!x || !W || !phi) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(phi)) return fail(REHYAT_ERR_ALIGN, "x/phi not 16-byte aligned");
  return launch_featmap(d, dt, n_tokens, x, W, bias, phi, static_cast<cudaStream_t>(stream));
}

int rehyat_forward_workspace_size(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens,
                                  int Tc, int To, size_t* bytes) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(T, frame_tokens, Tc, To));
  if (!bytes) return fail(REHYAT_ERR_ARG, "null bytes pointer");
  *bytes = plan_forward(d, dt, T, frame_tokens, Tc, To).total;
  return REHYAT_OK;
}

static int forward_common_checks(const rehyat_dims& d, rehyat_dtype dt, int T, int L, int Tc,
                                 int To, const void* workspace, size_t ws_bytes,
                                 ForwardPlan* pl) {
  RH_TRY(check_dims(d, dt));
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(T, L, Tc, To));
  *pl = plan_forward(d, dt, T, L, Tc, To);
  if (!workspace || ws_bytes < pl->total)
    return fail(REHYAT_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", pl->total, ws_bytes);
  if (!aligned16(workspace)) return fail(REHYAT_ERR_ALIGN, "workspace not 16-byte aligned");
  return REHYAT_OK;
}

int rehyat_forward_states(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                          const void* k, const void* v, const float* Wk, const float* bk,
                          void* workspace, size_t ws_bytes, void* stream) {
  g_msg[0] = 0;
  ForwardPlan pl;
  RH_TRY(forward_common_checks(d, dt, T, L, Tc, To, workspace, ws_bytes, &pl));
  if (!k || !v || !Wk) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(k) || !aligned16(v)) return fail(REHYAT_ERR_ALIGN, "k/v not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (dt == REHYAT_BF16)
    return forward_states_bf16(d, T, L, Tc, To, k, v, Wk, bk, pl, ws,
                               reinterpret_cast<__nv_bfloat16*>(ws + pl.St),
                               reinterpret_cast<float*>(ws + pl.Zc), nullptr, nullptr, st);
  return forward_states_f32(d, T, L, Tc, To, k, v, Wk, bk, pl, ws,
                            reinterpret_cast<float*>(ws + pl.Sc),
                            reinterpret_cast<float*>(ws + pl.Zc), st);
}

// behind_scan: the caller enqueued rehyat_forward_states right before (the phi_q kernel then
// starts under the state scan, which it does not read).
static int forward_phiq_impl(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                             const void* q, const float* Wq, const float* bq, void* workspace,
                             size_t ws_bytes, void* stream, bool behind_scan);

int rehyat_forward_phiq(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                        const void* q, const float* Wq, const float* bq, void* workspace,
                        size_t ws_bytes, void* stream) {
  return forward_phiq_impl(d, dt, T, L, Tc, To, q, Wq, bq, workspace, ws_bytes, stream, false);
}

static int forward_phiq_impl(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                             const void* q, const float* Wq, const float* bq, void* workspace,
                             size_t ws_bytes, void* stream, bool behind_scan) {
  g_msg[0] = 0;
  ForwardPlan pl;
  RH_TRY(forward_common_checks(d, dt, T, L, Tc, To, workspace, ws_bytes, &pl));
  if (!q || !Wq) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q)) return fail(REHYAT_ERR_ALIGN, "q not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const long long N = (long long)T * L;
  if (dt == REHYAT_BF16) {
    // phi_q of every query row whose chunk has a linear region: chunks c >= To / Tc + 1
    const long long row_lin = (long long)(To / Tc + 1) * Tc * L;
    if (row_lin < N)
      RH_TRY(launch_featmap_tc(d, q, (int)N, (int)row_lin, (int)(N - row_lin), Wq, bq,
                               reinterpret_cast<__nv_bfloat16*>(ws + pl.phiq_bf16), st,
                               behind_scan));
    return REHYAT_OK;
  }
  return launch_featmap(d, REHYAT_F32, (int)N, q, Wq, bq, ws + pl.phiq, st);
}

static int forward_attend_impl(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                               const void* q, const void* k, const void* v, void* out,
                               float* lse, const void* workspace, size_t ws_bytes, void* stream,
                               bool behind_phiq);

int rehyat_forward_attend(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                          const void* q, const void* k, const void* v, void* out,
                          const void* workspace, size_t ws_bytes, void* stream) {
  return forward_attend_impl(d, dt, T, L, Tc, To, q, k, v, out, nullptr, workspace, ws_bytes,
                             stream, false);
}

// behind_phiq: the caller enqueued rehyat_forward_phiq right before (the attention then overlaps
// the phi_q kernel).
static int forward_attend_impl(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                               const void* q, const void* k, const void* v, void* out,
                               float* lse, const void* workspace, size_t ws_bytes,
                               void* stream, bool behind_phiq) {
  g_msg[0] = 0;
  ForwardPlan pl;
  RH_TRY(forward_common_checks(d, dt, T, L, Tc, To, workspace, ws_bytes, &pl));
  if (!q || !k || !v || !out) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(REHYAT_ERR_ALIGN, "q/k/v/out not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(const_cast<void*>(workspace));
  const int BH = d.B * d.H;
  const long long N = (long long)T * L;
  const int rows_per_chunk = (Tc < T ? Tc : T) * L;
  if (dt == REHYAT_BF16) {
    CUtensorMap mq, mk, mv, ms, mphi;
    RH_TRY(make_map(&mq, q, d.D, N, BH));
    RH_TRY(make_map(&mk, k, d.D, N, BH));
    RH_TRY(make_map(&mv, v, d.D, N, BH));
    RH_TRY(make_map(&ms, ws + pl.St, d.F, d.D, (long long)BH * pl.C));
    RH_TRY(make_map(&mphi, ws + pl.phiq_bf16, d.F, N, BH));
    rehyat::attn::Params ap{};
    ap.L = L; ap.T = T; ap.Tc = Tc; ap.To = To; ap.frames_before = 0; ap.kv_frame0 = 0;
    ap.H = d.H; ap.P = kernel_P(d); ap.n_states = pl.C; ap.nq_rows = (int)N;
    ap.kv_rows = ap.carry_rows = (int)N;
    ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d.D));
    ap.bq = nullptr;  // phi_q comes finished from the workspace
    ap.Z = reinterpret_cast<const float*>(ws + pl.Zc);
    ap.out = static_cast<__nv_bfloat16*>(out);
    ap.lse = lse;
    // lone last tiles run as parts of their key window (not when row statistics are kept)
    const LoneSplit ls = lone_split_plan(T, L, Tc, To, 0, pl.C, lse == nullptr);
    ap.n_split = ls.n_split;
    ap.part_o = reinterpret_cast<float*>(ws + pl.part);
    ap.part_ml = ap.part_o + (size_t)BH * pl.C * kMaxLoneSplit * 128 * d.D;
    RH_TRY(launch_attn_bf16<true>(mq, mk, mv, ms, mq, mphi, ap, dim3(ls.slots, BH, pl.C), st,
                                  nullptr, nullptr, behind_phiq));
    if (ap.n_split > 1) RH_TRY(launch_lone_combine(ap, BH, pl.C, st));
    return REHYAT_OK;
  }
  rehyat::fp32::AttnParams ap{};
  ap.L = L; ap.T = T; ap.Tc = Tc; ap.To = To; ap.frames_before = 0; ap.kv_frame0 = 0;
  ap.D = d.D; ap.F = d.F; ap.nq_rows = (int)N; ap.nkv_rows = (int)N; ap.n_states = pl.C;
  ap.scale = (float)(1.0 / std::sqrt((double)d.D));
  ap.q = static_cast<const float*>(q); ap.k = static_cast<const float*>(k);
  ap.v = static_cast<const float*>(v); ap.phiq = reinterpret_cast<const float*>(ws + pl.phiq);
  ap.S = reinterpret_cast<const float*>(ws + pl.Sc);
  ap.Z = reinterpret_cast<const float*>(ws + pl.Zc);
  ap.out = static_cast<float*>(out);
  rehyat::fp32::hybrid_attn_f32_kernel<<<dim3((rows_per_chunk + 3) / 4, pl.C, BH), 128, 0, st>>>(ap);
  return cuda_check(cudaGetLastError(), "attention f32 launch");
}

int rehyat_forward(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To, const void* q,
                   const void* k, const void* v, const float* Wq, const float* bq,
                   const float* Wk, const float* bk, void* out, void* workspace,
                   size_t ws_bytes, void* stream) {
  g_msg[0] = 0;
  // every argument is checked before the first phase enqueues anything
  ForwardPlan pl;
  RH_TRY(forward_common_checks(d, dt, T, L, Tc, To, workspace, ws_bytes, &pl));
  if (!q || !k || !v || !Wq || !Wk || !out) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(REHYAT_ERR_ALIGN, "q/k/v/out not 16-byte aligned");
  RH_TRY(rehyat_forward_states(d, dt, T, L, Tc, To, k, v, Wk, bk, workspace, ws_bytes, stream));
  RH_TRY(forward_phiq_impl(d, dt, T, L, Tc, To, q, Wq, bq, workspace, ws_bytes, stream, true));
  return forward_attend_impl(d, dt, T, L, Tc, To, q, k, v, out, nullptr, workspace, ws_bytes,
                             stream, true);
}

int rehyat_forward_train(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                         const void* q, const void* k, const void* v, const float* Wq,
                         const float* bq, const float* Wk, const float* bk, void* out, float* lse,
                         void* workspace, size_t ws_bytes, void* stream) {
  g_msg[0] = 0;
  if (dt != REHYAT_BF16) return fail(REHYAT_ERR_DTYPE, "the training forward is bf16 only");
  ForwardPlan pl;
  RH_TRY(forward_common_checks(d, dt, T, L, Tc, To, workspace, ws_bytes, &pl));
  if (!q || !k || !v || !Wq || !Wk || !out || !lse) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(REHYAT_ERR_ALIGN, "q/k/v/out not 16-byte aligned");
  RH_TRY(rehyat_forward_states(d, dt, T, L, Tc, To, k, v, Wk, bk, workspace, ws_bytes, stream));
  RH_TRY(forward_phiq_impl(d, dt, T, L, Tc, To, q, Wq, bq, workspace, ws_bytes, stream, true));
  return forward_attend_impl(d, dt, T, L, Tc, To, q, k, v, out, lse, workspace, ws_bytes, stream,
                             true);
}

int rehyat_backward_workspace_size(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                                   size_t* bytes) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  if (dt != REHYAT_BF16) return fail(REHYAT_ERR_DTYPE, "the backward pass is bf16 only");
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(T, L, Tc, To));
  if (!bytes) return fail(REHYAT_ERR_ARG, "null bytes pointer");
  *bytes = plan_backward(d, T, L, Tc, To).total;
  return REHYAT_OK;
}

int rehyat_backward(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To, const void* q,
                    const void* k, const void* v, const float* Wq, const float* bq,
                    const float* Wk, const float* bk, const void* out, const float* lse,
                    const void* dout, float* dq, float* dk, float* dv, float* dWq, float* dbq,
                    float* dWk, float* dbk, void* workspace, size_t ws_bytes, void* stream) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  if (dt != REHYAT_BF16) return fail(REHYAT_ERR_DTYPE, "the backward pass is bf16 only");
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(T, L, Tc, To));
  if (L % 8) return fail(REHYAT_ERR_SHAPE, "the backward needs frame_tokens %% 8 == 0 (got %d)", L);
  if (!q || !k || !v || !Wq || !Wk || !out || !lse || !dout || !dq || !dk || !dv || !dWq ||
      !dbq || !dWk || !dbk)
    return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(REHYAT_ERR_ALIGN, "tensors must be 16-byte aligned");
  const BackwardPlan pl = plan_backward(d, T, L, Tc, To);
  if (!workspace || ws_bytes < pl.total)
    return fail(REHYAT_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", pl.total, ws_bytes);
  if (!aligned16(workspace)) return fail(REHYAT_ERR_ALIGN, "workspace not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* fw = ws + pl.fwd_off;
  const int BH = d.B * d.H;
  const long long N = (long long)T * L, F = d.F, D = d.D;
  const int C = pl.C;
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
  const __nv_bfloat16* dob = static_cast<const __nv_bfloat16*>(dout);
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  auto b16 = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  const size_t ND = (size_t)BH * N * D * 4;
  const size_t WB = (size_t)d.H * F * (D / d.G) * 4;
  RH_TRY(cuda_check(cudaMemsetAsync(dq, 0, ND, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(dk, 0, ND, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(dv, 0, ND, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(dWq, 0, WB, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(dWk, 0, WB, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(dbq, 0, (size_t)d.H * F * 4, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(dbk, 0, (size_t)d.H * F * 4, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(ws + pl.RB, 0, (size_t)BH * C * F * D * 4, st), "memset"));
  RH_TRY(cuda_check(cudaMemsetAsync(ws + pl.rpart, 0, (size_t)C * BH * pl.nblk_r * F * 4, st),
                    "memset"));

  // states S_c (transposed, bf16), Z_c and phi_q of the rows that read a state, as the forward
  RH_TRY(rehyat_forward_states(d, dt, T, L, Tc, To, k, v, Wk, bk, fw, pl.fwd_bytes, stream));
  RH_TRY(rehyat_forward_phiq(d, dt, T, L, Tc, To, q, Wq, bq, fw, pl.fwd_bytes, stream));
  // the block-diagonal weights (bf16 hi, lo) of both feature maps for the gradient GEMMs
  {
    CUtensorMap unused;
    RH_TRY(prepare_blockdiag(d, Wq, reinterpret_cast<__nv_bfloat16*>(fw + pl.fwd.Wqbd), &unused,
                             st));
    RH_TRY(prepare_blockdiag(d, Wk, reinterpret_cast<__nv_bfloat16*>(fw + pl.fwd.Wkbd), &unused,
                             st));
  }
  const __nv_bfloat16* St = reinterpret_cast<const __nv_bfloat16*>(fw + pl.fwd.St);
  const float* Zc = reinterpret_cast<const float*>(fw + pl.fwd.Zc);
  const __nv_bfloat16* phiq = reinterpret_cast<const __nv_bfloat16*>(fw + pl.fwd.phiq_bf16);
  const __nv_bfloat16* Wqbd = reinterpret_cast<const __nv_bfloat16*>(fw + pl.fwd.Wqbd);
  const __nv_bfloat16* Wkbd = reinterpret_cast<const __nv_bfloat16*>(fw + pl.fwd.Wkbd);
  // the key rows that some later chunk reads linearly: [0, w_{C-1} L)
  const long long wl = (long long)((C - 1) * Tc - To > 0 ? (C - 1) * Tc - To : 0) * L;
  if (wl > 0) RH_TRY(launch_featmap_tc(d, k, (int)N, 0, (int)wl, Wk, bk, b16(pl.phik), st));
  rehyat::bwd::rowstats_kernel<<<(unsigned)((BH * N + 7) / 8), 256, 0, st>>>(
      dob, static_cast<const __nv_bfloat16*>(out), lse, BH * N, d.D, f32(pl.Drow), f32(pl.lam));
  RH_TRY(cuda_check(cudaGetLastError(), "row statistics launch"));

  const float sl2 = (float)(1.4426950408889634 / std::sqrt((double)d.D));
  const float isd = (float)(1.0 / std::sqrt((double)d.D));
  CUtensorMap mq, mk, mv, mo, mdq, mdk, mdv;
  RH_TRY(make_map(&mq, q, d.D, N, BH));
  RH_TRY(make_map(&mk, k, d.D, N, BH));
  RH_TRY(make_map(&mv, v, d.D, N, BH));
  RH_TRY(make_map(&mo, dout, d.D, N, BH));
  RH_TRY(make_map_f32(&mdq, dq, d.D, N, BH));
  RH_TRY(make_map_f32(&mdk, dk, d.D, N, BH));
  RH_TRY(make_map_f32(&mdv, dv, d.D, N, BH));
  for (int c = 0; c < C; ++c) {
    const int s = c * Tc, e = (s + Tc < T ? s + Tc : T), w = (s - To > 0 ? s - To : 0);
    const long long nq = (long long)(e - s) * L, nw = (long long)(e - w) * L;
    const long long r0 = (long long)s * L;
    // the softmax window's gradients, scores recomputed in TMEM: dK, dV per key tile, dQ per
    // query tile
    {
      rehyat::attn_bwd::Params bp{};
      bp.L = L; bp.T = T; bp.Tc = Tc; bp.To = To; bp.c = c; bp.N = (int)N;
      bp.lse2 = lse; bp.Drow = f32(pl.Drow); bp.scale_log2 = sl2; bp.inv_sqrt_d = isd;
      bp.dq = dq; bp.dk = dk; bp.dv = dv;
      auto kkv = rehyat::attn_bwd::dkdv_kernel;
      auto kq = rehyat::attn_bwd::dq_kernel;
      RH_TRY(cuda_check(cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)rehyat::attn_bwd::kKSmem), "dkdv attr"));
      RH_TRY(cuda_check(cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)rehyat::attn_bwd::kQSmem), "dq attr"));
      kkv<<<dim3((unsigned)((nw + 127) / 128), 1, BH), rehyat::attn_bwd::kThreads,
            rehyat::attn_bwd::kKSmem, st>>>(mq, mk, mv, mo, mdk, mdv, bp);
      RH_TRY(cuda_check(cudaGetLastError(), "dkdv launch"));
      kq<<<dim3((unsigned)((nq + 127) / 128), 1, BH), rehyat::attn_bwd::kThreads,
           rehyat::attn_bwd::kQSmem, st>>>(mq, mk, mv, mo, mdq, bp);
      RH_TRY(cuda_check(cudaGetLastError(), "dq launch"));
    }
    if (w > 0) {
      // G = dO_c S_c^T; dphi_q = lam (G - D Z_c); R_c = (lam phi_q)^T dO_c; r_c partials
      RH_TRY(launch_gemm((int)nq, (int)F, (int)D, BH, Operand{dob + r0 * D, D, N * D, false},
                         Operand{St + (long long)c * D * F, F, (long long)C * D * F, true},
                         f32(pl.GB), F, nq * F, false, false, 1.f, st));
      rehyat::bwd::phiq_grad_kernel<<<dim3((unsigned)nq, BH), d.F, 0, st>>>(
          f32(pl.GB), (int)nq, d.F, N, r0, f32(pl.lam), f32(pl.Drow), Zc + (long long)c * F,
          (long long)C * F, phiq, f32(pl.dphiq), b16(pl.phis));
      RH_TRY(cuda_check(cudaGetLastError(), "phi_q gradient launch"));
      RH_TRY(launch_gemm((int)F, (int)D, (int)nq, BH, Operand{b16(pl.phis), F, nq * F, true},
                         Operand{dob + r0 * D, D, N * D, true},
                         f32(pl.RB) + (long long)c * F * D, D, (long long)C * F * D, false, true,
                         1.f, st, 8));
      const int nblk = (int)((nq + rehyat::bwd::kRBlock - 1) / rehyat::bwd::kRBlock);
      rehyat::bwd::rpart_kernel<<<dim3(nblk, BH), d.F, 0, st>>>(
          (int)nq, d.F, N, r0, f32(pl.lam), f32(pl.Drow), phiq,
          f32(pl.rpart) + (long long)c * BH * pl.nblk_r * F, pl.nblk_r);
      RH_TRY(cuda_check(cudaGetLastError(), "r partial launch"));
    }
  }
  if (wl > 0) {
    rehyat::bwd::rreduce_kernel<<<dim3(C, BH), d.F, 0, st>>>(f32(pl.rpart), pl.nblk_r, d.F,
                                                             f32(pl.rt));
    RH_TRY(cuda_check(cudaGetLastError(), "r reduce launch"));
    rehyat::bwd::suffix_kernel<<<dim3((unsigned)((F * D + 255) / 256), BH), 256, 0, st>>>(
        f32(pl.RB), C, d.F, d.D, b16(pl.Rt), f32(pl.rt));
    RH_TRY(cuda_check(cudaGetLastError(), "suffix launch"));
    // keys folded after chunk c (frames [w_c, w_{c+1})) are read linearly from chunk c + 1 on
    for (int c = 0; c + 1 < C; ++c) {
      const int w0 = (c * Tc - To > 0 ? c * Tc - To : 0);
      const int w1 = ((c + 1) * Tc - To > 0 ? (c + 1) * Tc - To : 0);
      if (w1 <= w0) continue;
      const long long g0 = (long long)w0 * L, ng = (long long)(w1 - w0) * L;
      const __nv_bfloat16* Rt1 = b16(pl.Rt) + (long long)(c + 1) * F * D;
      // dphi_k = V_g Rt^T (r~ is subtracted with the activation derivative); dv_g += phi_k Rt
      RH_TRY(launch_gemm((int)ng, (int)F, (int)D, BH, Operand{vb + g0 * D, D, N * D, false},
                         Operand{Rt1, D, (long long)C * F * D, false}, f32(pl.dphik) + g0 * F, F,
                         N * F, false, false, 1.f, st));
      RH_TRY(launch_gemm((int)ng, (int)D, (int)F, BH,
                         Operand{b16(pl.phik) + g0 * F, F, N * F, false},
                         Operand{Rt1, D, (long long)C * F * D, true}, dv + g0 * D, D, N * D,
                         false, true, 1.f, st));
    }
  }
  // through the feature maps: q rows of chunks with a linear region, k rows read linearly
  const long long rq0 = (long long)pl.c_lin * Tc * L;
  if (rq0 < N)
    RH_TRY(feature_backward(d, N, rq0, N, q, Wqbd, bq, f32(pl.dphiq), nullptr, C, L, Tc, To, pl,
                            ws, dq, dWq, dbq, st));
  if (wl > 0)
    RH_TRY(feature_backward(d, N, 0, wl, k, Wkbd, bk, f32(pl.dphik), f32(pl.rt), C, L, Tc, To,
                            pl, ws, dk, dWk, dbk, st));
  return REHYAT_OK;
}

int rehyat_chunk_workspace_size(rehyat_dims d, rehyat_dtype dt, int frame_tokens,
                                int chunk_frames, int To, size_t* bytes) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(chunk_frames, frame_tokens, 1, To));
  if (!bytes) return fail(REHYAT_ERR_ARG, "null bytes pointer");
  *bytes = plan_chunk(d, dt, frame_tokens, To, chunk_frames, To, To).total;
  return REHYAT_OK;
}

int rehyat_chunk_forward(rehyat_dims d, rehyat_dtype dt, int L, int frames_before,
                         int chunk_frames, int To, const void* q, const void* k_win,
                         const void* v_win, const float* Wq, const float* bq, const float* Wk,
                         const float* bk, float* S, float* Z, void* out, void* workspace,
                         size_t ws_bytes, void* stream) {
  return rehyat_chunk_forward_sched(d, dt, L, frames_before, chunk_frames, To, To, q, k_win,
                                    v_win, Wq, bq, Wk, bk, S, Z, out, workspace, ws_bytes,
                                    stream);
}

// Where a bf16 chunk step's softmax window lives: window rows [0, split) in the carried frames
// (kc, vc with carry_rows rows per (b, h); window row 0 at row carry_row0), the rest in (k, v)
// (rows per (b, h); window row `split` at row 0).  split = 0: the whole window is (k, v).
struct WindowSrc {
  const void* k;
  const void* v;
  long long rows;
  const void* kc;
  const void* vc;
  long long carry_rows;
  int split, carry_row0;
};

// One bf16 chunk step ("ReHyAt overview" page §2.2-§2.3 and §5.2): S^T copy, phi_q, the
// attention with the state readout, then the fold of the frames leaving the window into S, Z.
// With `cc`, the next carry of K and V is copied in the same closing launch as the state add.
static int chunk_step_bf16(const rehyat_dims& d, int L, int frames_before, int chunk_frames,
                           int To, const ChunkPlan& pl, const void* q, const WindowSrc& w,
                           const float* Wq, const float* bq, const float* Wk, const float* bk,
                           float* S, float* Z, void* out, uint8_t* ws, cudaStream_t st,
                           const rehyat::state::CarryCopy* cc = nullptr) {
  const int BH = d.B * d.H;
  __nv_bfloat16* St = reinterpret_cast<__nv_bfloat16*>(ws + pl.St);
  float* dS = reinterpret_cast<float*>(ws + pl.dS);
  float* dZ = reinterpret_cast<float*>(ws + pl.dZ);
  // S^T in bf16 for the readout MMA (C = 1, no folds: a transposed copy of S)
  RH_TRY(launch_scan_bf16(d, dS, dZ, 0, 1, 1, S, Z, St, nullptr, nullptr, nullptr, st));
  CUtensorMap mq, mk, mv, mkc, mvc, ms;
  RH_TRY(make_map(&mq, q, d.D, pl.nq, BH));
  RH_TRY(make_map(&mk, w.k, d.D, w.rows, BH));
  RH_TRY(make_map(&mv, w.v, d.D, w.rows, BH));
  if (w.split > 0) {
    RH_TRY(make_map(&mkc, w.kc, d.D, w.carry_rows, BH));
    RH_TRY(make_map(&mvc, w.vc, d.D, w.carry_rows, BH));
  } else {
    mkc = mk;
    mvc = mv;
  }
  RH_TRY(make_map(&ms, St, d.F, d.D, BH));
  __nv_bfloat16* phiq = reinterpret_cast<__nv_bfloat16*>(ws + pl.phiq_bf16);
  // phi_q right before the attention, which overlaps it
  if (frames_before - pl.o > 0)  // the chunk reads a linear state; it starts under the S^T copy
    RH_TRY(launch_featmap_tc(d, q, pl.nq, 0, pl.nq, Wq, bq, phiq, st, true));
  CUtensorMap mphi;
  RH_TRY(make_map(&mphi, phiq, d.F, pl.nq, BH));
  rehyat::attn::Params ap{};
  ap.L = L; ap.T = chunk_frames; ap.Tc = chunk_frames; ap.To = To;
  ap.frames_before = frames_before;
  // the main source's row 0 is window row `split`
  ap.kv_frame0 = frames_before - pl.o + w.split / L;
  ap.kv_split = w.split; ap.carry_row0 = w.carry_row0;
  ap.kv_rows = (int)w.rows;
  ap.carry_rows = (int)(w.split > 0 ? w.carry_rows : w.rows);
  ap.H = d.H; ap.P = kernel_P(d); ap.n_states = 1; ap.nq_rows = pl.nq;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d.D));
  ap.bq = bq; ap.Z = Z; ap.out = static_cast<__nv_bfloat16*>(out);
  // the lone last tile (odd tile count) runs as parts of its key window
  const int q_tiles = (pl.nq + 127) / 128;
  const int key_tiles = (int)((w.split + 127) / 128 + (pl.nkv - w.split + 127) / 128);
  ap.n_split = (q_tiles & 1) ? lone_split_count(key_tiles) : 1;
  ap.part_o = reinterpret_cast<float*>(ws + pl.part);
  ap.part_ml = ap.part_o + (size_t)BH * kMaxLoneSplit * 128 * d.D;
  // (the weight map is unused: phi_q comes finished from the workspace)
  RH_TRY(launch_attn_bf16<true>(mq, mk, mv, ms, mq, mphi, ap,
                                dim3(q_tiles / 2 + ((q_tiles & 1) ? ap.n_split : 0), BH, 1), st,
                                &mkc, &mvc, true));
  if (pl.fold_rows > 0) {
    // the fold reads only the window and writes its own partials: it runs in the attention's
    // last wave; the state update after it waits for both
    rehyat::state::FoldParams fp{};
    fp.L = L; fp.H = d.H; fp.P = kernel_P(d); fp.single_rows = pl.fold_rows; fp.n_fold = 1;
    fp.kv_rows = (int)w.rows;
    fp.carry_rows = (int)(w.split > 0 ? w.carry_rows : w.rows);
    fp.seg_rows = pl.fold_rows < w.split ? pl.fold_rows : w.split;
    fp.seg_row0 = w.carry_row0;
    fp.splits = pl.splits; fp.G = d.G; fp.W = Wk; fp.bk = bk; fp.dS = dS; fp.dZ = dZ;
    RH_TRY(launch_fold_bf16(mk, mv, fp, dim3(pl.splits, 1, BH), st, &mkc, &mvc, true));
  }
  if (ap.n_split > 1) RH_TRY(launch_lone_combine(ap, BH, 1, st));
  const int n_add = pl.fold_rows > 0 ? (d.F * d.D + 255) / 256 : 0;
  if (cc && cc->n_vec > 0) {
    long long n_copy = (2 * cc->n_vec + 255) / 256;
    if (n_copy > 16) n_copy = 16;
    rehyat::state::state_add_carry_kernel<<<dim3((unsigned)(n_add + n_copy), BH), 256, 0, st>>>(
        dS, dZ, pl.splits, d.F, d.D, S, Z, n_add, *cc);
    return cuda_check(cudaGetLastError(), "state add and carry launch");
  }
  if (n_add > 0) {
    rehyat::state::state_add_kernel<<<dim3(n_add, BH), 256, 0, st>>>(dS, dZ, pl.splits, d.F, d.D,
                                                                     S, Z);
    RH_TRY(cuda_check(cudaGetLastError(), "state add launch"));
  }
  return REHYAT_OK;
}

// Argument checks shared by the window-buffer and the carried-frame chunk steps.
static int check_step(const rehyat_dims& d, rehyat_dtype dt, int L, int frames_before,
                      int chunk_frames, int To, int To_next) {
  RH_TRY(check_dims(d, dt));
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(chunk_frames, L, 1, To));
  if (frames_before < 0) return fail(REHYAT_ERR_ARG, "frames_before must be >= 0");
  if (To_next < 0) return fail(REHYAT_ERR_ARG, "To_next must be >= 0");
  const int o = To < frames_before ? To : frames_before;
  const int seen = frames_before + chunk_frames;
  if ((To_next < seen ? To_next : seen) > o + chunk_frames)
    return fail(REHYAT_ERR_ARG,
                "To_next=%d reaches before this window (%d frames): those frames are already "
                "folded into S", To_next, o + chunk_frames);
  return REHYAT_OK;
}

int rehyat_chunk_forward_sched(rehyat_dims d, rehyat_dtype dt, int L, int frames_before,
                               int chunk_frames, int To, int To_next, const void* q,
                               const void* k_win, const void* v_win, const float* Wq,
                               const float* bq, const float* Wk, const float* bk, float* S,
                               float* Z, void* out, void* workspace, size_t ws_bytes,
                               void* stream) {
  g_msg[0] = 0;
  RH_TRY(check_step(d, dt, L, frames_before, chunk_frames, To, To_next));
  if (!q || !k_win || !v_win || !Wq || !Wk || !S || !Z || !out)
    return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k_win) || !aligned16(v_win) || !aligned16(out))
    return fail(REHYAT_ERR_ALIGN, "q/k_win/v_win/out not 16-byte aligned");
  const ChunkPlan pl = plan_chunk(d, dt, L, frames_before, chunk_frames, To, To_next);
  const size_t need = plan_chunk(d, dt, L, To, chunk_frames, To, To).total;
  if (!workspace || ws_bytes < need || ws_bytes < pl.total)
    return fail(REHYAT_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, ws_bytes);
  if (!aligned16(workspace)) return fail(REHYAT_ERR_ALIGN, "workspace not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int BH = d.B * d.H;

  if (dt == REHYAT_BF16) {
    const WindowSrc w{k_win, v_win, pl.nkv, nullptr, nullptr, 0, 0, 0};
    return chunk_step_bf16(d, L, frames_before, chunk_frames, To, pl, q, w, Wq, bq, Wk, bk, S, Z,
                           out, ws, st);
  }
  // fp32
  float* phiq = reinterpret_cast<float*>(ws + pl.phiq);
  float* phik = reinterpret_cast<float*>(ws + pl.phik);
  float* dS = reinterpret_cast<float*>(ws + pl.dS);
  float* dZ = reinterpret_cast<float*>(ws + pl.dZ);
  RH_TRY(launch_featmap(d, REHYAT_F32, pl.nq, q, Wq, bq, phiq, st));
  rehyat::fp32::AttnParams ap{};
  ap.L = L; ap.T = chunk_frames; ap.Tc = chunk_frames; ap.To = To;
  ap.frames_before = frames_before; ap.kv_frame0 = frames_before - pl.o;
  ap.D = d.D; ap.F = d.F; ap.nq_rows = pl.nq; ap.nkv_rows = pl.nkv; ap.n_states = 1;
  ap.scale = (float)(1.0 / std::sqrt((double)d.D));
  ap.q = static_cast<const float*>(q); ap.k = static_cast<const float*>(k_win);
  ap.v = static_cast<const float*>(v_win); ap.phiq = phiq; ap.S = S; ap.Z = Z;
  ap.out = static_cast<float*>(out);
  rehyat::fp32::hybrid_attn_f32_kernel<<<dim3((pl.nq + 3) / 4, 1, BH), 128, 0, st>>>(ap);
  RH_TRY(cuda_check(cudaGetLastError(), "attention f32 launch"));
  if (pl.fold_rows > 0) {
    RH_TRY(launch_featmap(d, REHYAT_F32, pl.nkv, k_win, Wk, bk, phik, st));
    rehyat::fp32::FoldParams fp{};
    fp.single_rows = pl.fold_rows; fp.n_fold = 1; fp.F = d.F; fp.D = d.D; fp.nkv_rows = pl.nkv;
    fp.phik = phik; fp.v = static_cast<const float*>(v_win); fp.dS = dS; fp.dZ = dZ;
    rehyat::fp32::fold_partial_f32_kernel<<<dim3(1, BH), 256, 0, st>>>(fp);
    RH_TRY(cuda_check(cudaGetLastError(), "fold f32 launch"));
    rehyat::fp32::state_add_f32_kernel<<<dim3((d.F * d.D + 255) / 256, BH), 256, 0, st>>>(
        dS, dZ, d.F, d.D, S, Z);
    RH_TRY(cuda_check(cudaGetLastError(), "state add f32 launch"));
  }
  return REHYAT_OK;
}

int rehyat_chunk_carry_workspace_size(rehyat_dims d, rehyat_dtype dt, int frame_tokens,
                                      int chunk_frames, int To, int carry_frames,
                                      size_t* bytes) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(chunk_frames, frame_tokens, 1, To));
  if (carry_frames < To) return fail(REHYAT_ERR_ARG, "carry_frames %d < To %d", carry_frames, To);
  if (!bytes) return fail(REHYAT_ERR_ARG, "null bytes pointer");
  *bytes = plan_carry(d, dt, frame_tokens, chunk_frames, To, carry_frames).total;
  return REHYAT_OK;
}

int rehyat_chunk_forward_carry(rehyat_dims d, rehyat_dtype dt, int L, int frames_before,
                               int chunk_frames, int To, int To_next, int carry_frames,
                               const void* q, const void* k, const void* v, const float* Wq,
                               const float* bq, const float* Wk, const float* bk, float* S,
                               float* Z, void* k_carry, void* v_carry, void* out,
                               void* workspace, size_t ws_bytes, void* stream) {
  g_msg[0] = 0;
  RH_TRY(check_step(d, dt, L, frames_before, chunk_frames, To, To_next));
  if (carry_frames < To) return fail(REHYAT_ERR_ARG, "carry_frames %d < To %d", carry_frames, To);
  if (!q || !k || !v || !Wq || !Wk || !S || !Z || !out ||
      (carry_frames > 0 && (!k_carry || !v_carry)))
    return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_carry) ||
      !aligned16(v_carry) || !aligned16(out))
    return fail(REHYAT_ERR_ALIGN, "q/k/v/k_carry/v_carry/out not 16-byte aligned");
  // the step's workspace is sized for this call's To; the caller's workspace comes from
  // rehyat_chunk_carry_workspace_size with the largest chunk_frames and To
  const CarryPlan pl = plan_carry(d, dt, L, chunk_frames, To, carry_frames);
  if (!workspace || ws_bytes < pl.total)
    return fail(REHYAT_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", pl.total, ws_bytes);
  if (!aligned16(workspace)) return fail(REHYAT_ERR_ALIGN, "workspace not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int BH = d.B * d.H;
  const int ov = To < frames_before ? To : frames_before;
  const size_t es = dt == REHYAT_BF16 ? 2 : 4;
  const size_t frame_bytes = (size_t)L * d.D * es;  // one frame of one (b, h)
  rehyat::carry::Params cp{};
  cp.L = L; cp.ov = ov; cp.cf = chunk_frames; cp.cap = carry_frames;
  cp.row_vec = (int)(d.D * es / 16);
  // gather launch: window (fp32 only) and next carry of K, then of V
  auto gather = [&](bool window) -> int {
    cp.window_out = window ? 1 : 0;
    const long long vecs =
        ((window ? (long long)(ov + chunk_frames) : 0LL) + carry_frames) * L * cp.row_vec;
    long long gx = (vecs + 255) / 256;
    const long long max_gx = (8LL * 148 + BH - 1) / BH;
    if (gx > max_gx) gx = max_gx;
    if (gx < 1) gx = 1;
    for (int t = 0; t < 2; ++t) {
      cp.carry = static_cast<const uint4*>(t ? v_carry : k_carry);
      cp.chunk = static_cast<const uint4*>(t ? v : k);
      cp.window = window ? reinterpret_cast<uint4*>(ws + (t ? pl.vwin : pl.kwin)) : nullptr;
      cp.carry_new = reinterpret_cast<uint4*>(ws + (t ? pl.vcar : pl.kcar));
      rehyat::carry::gather_kernel<<<dim3((unsigned)gx, BH), 256, 0, st>>>(cp);
      RH_TRY(cuda_check(cudaGetLastError(), "window gather launch"));
    }
    return REHYAT_OK;
  };
  auto copy_back = [&]() -> int {
    const size_t car_bytes = (size_t)BH * carry_frames * frame_bytes;
    if (!car_bytes) return REHYAT_OK;
    RH_TRY(cuda_check(cudaMemcpyAsync(k_carry, ws + pl.kcar, car_bytes, cudaMemcpyDeviceToDevice, st),
                      "carry copy"));
    RH_TRY(cuda_check(cudaMemcpyAsync(v_carry, ws + pl.vcar, car_bytes, cudaMemcpyDeviceToDevice, st),
                      "carry copy"));
    return REHYAT_OK;
  };

  if (dt == REHYAT_BF16) {
    // The kernels read the window straight from the carry (its last ov frames) and the chunk.
    const ChunkPlan cpl = plan_chunk(d, dt, L, frames_before, chunk_frames, To, To_next);
    if (cpl.total > pl.step_bytes)
      return fail(REHYAT_ERR_WORKSPACE, "chunk step needs %zu bytes, plan holds %zu", cpl.total,
                  pl.step_bytes);
    const WindowSrc w{k, v, (long long)chunk_frames * L, k_carry, v_carry,
                      (long long)carry_frames * L, ov * L, (carry_frames - ov) * L};
    // the next carry, after every read of the old one (stream order): the last carry_frames
    // frames of (carry ++ chunk); a chunk at least that long supplies all of them, copied in
    // the step's closing launch
    if (chunk_frames >= carry_frames) {
      const long long fv = (long long)(frame_bytes / 16);  // 16-byte vectors per frame
      const rehyat::state::CarryCopy cc{static_cast<const uint4*>(k), static_cast<const uint4*>(v),
                                        static_cast<uint4*>(k_carry), static_cast<uint4*>(v_carry),
                                        chunk_frames * fv, (chunk_frames - carry_frames) * fv,
                                        carry_frames * fv};
      return chunk_step_bf16(d, L, frames_before, chunk_frames, To, cpl, q, w, Wq, bq, Wk, bk, S,
                             Z, out, ws + pl.step, st, &cc);
    }
    RH_TRY(chunk_step_bf16(d, L, frames_before, chunk_frames, To, cpl, q, w, Wq, bq, Wk, bk, S, Z,
                           out, ws + pl.step, st));
    RH_TRY(gather(false));
    return copy_back();
  }
  // fp32: assemble the window, run the window-buffer step, then replace the carry
  RH_TRY(gather(true));
  RH_TRY(rehyat_chunk_forward_sched(d, dt, L, frames_before, chunk_frames, To, To_next, q,
                                    ws + pl.kwin, ws + pl.vwin, Wq, bq, Wk, bk, S, Z, out,
                                    ws + pl.step, pl.step_bytes, stream));
  return copy_back();
}

static int segment_checks(const rehyat_dims& d, rehyat_dtype dt, int T, int L, int Tc, int To,
                          int c0, int c1, const void* workspace, size_t ws_bytes, SegPlan* pl) {
  RH_TRY(check_dims(d, dt));
  if (dt != REHYAT_BF16) return fail(REHYAT_ERR_DTYPE, "segments are bf16 only");
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(T, L, Tc, To));
  const int C = (T + Tc - 1) / Tc;
  if (c0 < 0 || c1 <= c0 || c1 > C)
    return fail(REHYAT_ERR_ARG, "segment [%d, %d) is not inside chunks [0, %d)", c0, c1, C);
  *pl = plan_segment(d, T, L, Tc, To, c0, c1);
  if (workspace || ws_bytes) {
    if (!workspace || ws_bytes < pl->total)
      return fail(REHYAT_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", pl->total, ws_bytes);
    if (!aligned16(workspace)) return fail(REHYAT_ERR_ALIGN, "workspace not 16-byte aligned");
  }
  return REHYAT_OK;
}

int rehyat_segment_workspace_size(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc,
                                  int To, int c0, int c1, size_t* bytes) {
  g_msg[0] = 0;
  SegPlan pl;
  RH_TRY(segment_checks(d, dt, T, frame_tokens, Tc, To, c0, c1, nullptr, 0, &pl));
  if (!bytes) return fail(REHYAT_ERR_ARG, "null bytes pointer");
  *bytes = pl.total;
  return REHYAT_OK;
}

int rehyat_segment_states(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To, int c0,
                          int c1, const void* k_seg, const void* v_seg, const float* Wk,
                          const float* bk, float* S_seg, float* Z_seg, void* workspace,
                          size_t ws_bytes, void* stream) {
  g_msg[0] = 0;
  SegPlan pl;
  if (!workspace) return fail(REHYAT_ERR_WORKSPACE, "null workspace");
  RH_TRY(segment_checks(d, dt, T, L, Tc, To, c0, c1, workspace, ws_bytes, &pl));
  if (!k_seg || !v_seg || !Wk || !S_seg || !Z_seg) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(k_seg) || !aligned16(v_seg))
    return fail(REHYAT_ERR_ALIGN, "k_seg/v_seg not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int BH = d.B * d.H;
  float* dS = reinterpret_cast<float*>(ws + pl.dS);
  float* dZ = reinterpret_cast<float*>(ws + pl.dZ);
  if (pl.n_fold > 0) {
    CUtensorMap mk, mv;
    RH_TRY(make_map(&mk, k_seg, d.D, pl.nkv_rows, BH));
    RH_TRY(make_map(&mv, v_seg, d.D, pl.nkv_rows, BH));
    rehyat::state::FoldParams fp{};
    fp.L = L; fp.H = d.H; fp.P = kernel_P(d); fp.T = T; fp.Tc = Tc; fp.To = To;
    fp.kv_frame0 = pl.h0; fp.fold_c0 = c0;
    fp.single_rows = -1; fp.n_fold = pl.n_fold; fp.splits = pl.splits;
    fp.kv_rows = fp.carry_rows = (int)pl.nkv_rows;
    fp.G = d.G; fp.W = Wk; fp.bk = bk; fp.dS = dS; fp.dZ = dZ;
    RH_TRY(launch_fold_bf16(mk, mv, fp, dim3(pl.splits, pl.n_fold, BH), st));
  }
  rehyat::state::state_sum_kernel<<<dim3((d.F * d.D + 255) / 256, BH), 256, 0, st>>>(
      dS, dZ, pl.n_fold * pl.splits, d.F, d.D, S_seg, Z_seg);
  return cuda_check(cudaGetLastError(), "segment sum launch");
}

int rehyat_segment_attend(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To, int c0,
                          int c1, const void* q_seg, const void* k_seg, const void* v_seg,
                          const float* Wq, const float* bq, int n_prefix, const float* S_prefix,
                          const float* Z_prefix, void* out_seg, void* workspace, size_t ws_bytes,
                          void* stream) {
  g_msg[0] = 0;
  SegPlan pl;
  if (!workspace) return fail(REHYAT_ERR_WORKSPACE, "null workspace");
  RH_TRY(segment_checks(d, dt, T, L, Tc, To, c0, c1, workspace, ws_bytes, &pl));
  if (!q_seg || !k_seg || !v_seg || !Wq || !out_seg) return fail(REHYAT_ERR_ARG, "null pointer");
  if (n_prefix < 0) return fail(REHYAT_ERR_ARG, "n_prefix must be >= 0");
  if (n_prefix > 0 && (!S_prefix || !Z_prefix))
    return fail(REHYAT_ERR_ARG, "null S_prefix/Z_prefix with n_prefix = %d", n_prefix);
  if (!aligned16(q_seg) || !aligned16(k_seg) || !aligned16(v_seg) || !aligned16(out_seg))
    return fail(REHYAT_ERR_ALIGN, "q_seg/k_seg/v_seg/out_seg not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int BH = d.B * d.H;
  // the state each local chunk reads: the earlier segments' sums, then this segment's folds
  RH_TRY(launch_scan_bf16(d, reinterpret_cast<const float*>(ws + pl.dS),
                          reinterpret_cast<const float*>(ws + pl.dZ), pl.n_fold, pl.splits,
                          pl.n_local, n_prefix > 0 ? S_prefix : nullptr,
                          n_prefix > 0 ? Z_prefix : nullptr,
                          reinterpret_cast<__nv_bfloat16*>(ws + pl.St),
                          reinterpret_cast<float*>(ws + pl.Zc), nullptr, nullptr, st,
                          n_prefix));
  // phi_q of the rows whose chunk reads a linear state (chunk c with c*Tc > To)
  int c_lin = To / Tc + 1;
  if (c_lin < c0) c_lin = c0;
  const long long row_lin = (long long)(c_lin - c0) * Tc * L;
  __nv_bfloat16* phiq = reinterpret_cast<__nv_bfloat16*>(ws + pl.phiq_bf16);
  if (row_lin < pl.nq_rows)
    RH_TRY(launch_featmap_tc(d, q_seg, (int)pl.nq_rows, (int)row_lin,
                             (int)(pl.nq_rows - row_lin), Wq, bq, phiq, st));
  CUtensorMap mq, mk, mv, ms, mphi;
  RH_TRY(make_map(&mq, q_seg, d.D, pl.nq_rows, BH));
  RH_TRY(make_map(&mk, k_seg, d.D, pl.nkv_rows, BH));
  RH_TRY(make_map(&mv, v_seg, d.D, pl.nkv_rows, BH));
  RH_TRY(make_map(&ms, ws + pl.St, d.F, d.D, (long long)BH * pl.n_local));
  RH_TRY(make_map(&mphi, phiq, d.F, pl.nq_rows, BH));
  rehyat::attn::Params ap{};
  ap.L = L; ap.T = pl.s1 - pl.s0; ap.Tc = Tc; ap.To = To;
  ap.frames_before = pl.s0; ap.kv_frame0 = pl.h0;
  ap.kv_rows = ap.carry_rows = (int)pl.nkv_rows;
  ap.H = d.H; ap.P = kernel_P(d); ap.n_states = pl.n_local; ap.nq_rows = (int)pl.nq_rows;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d.D));
  ap.bq = nullptr;  // phi_q comes finished from the workspace
  ap.Z = reinterpret_cast<const float*>(ws + pl.Zc);
  ap.out = static_cast<__nv_bfloat16*>(out_seg);
  const LoneSplit ls = lone_split_plan(ap.T, L, Tc, To, pl.s0, pl.n_local, true);
  ap.n_split = ls.n_split;
  ap.part_o = reinterpret_cast<float*>(ws + pl.part);
  ap.part_ml = ap.part_o + (size_t)BH * pl.n_local * kMaxLoneSplit * 128 * d.D;
  RH_TRY(launch_attn_bf16<true>(mq, mk, mv, ms, mq, mphi, ap, dim3(ls.slots, BH, pl.n_local), st,
                                nullptr, nullptr, true));
  if (ap.n_split > 1) RH_TRY(launch_lone_combine(ap, BH, pl.n_local, st));
  return REHYAT_OK;
}

int rehyat_chunk_forward_static(rehyat_dims d, rehyat_dtype dt, int L, int frames_before,
                                int chunk_frames, int To, const void* q, const void* k_win,
                                const void* v_win, const float* Wq, const float* bq,
                                const float* Wk, const float* bk, float* S, float* Z, void* out,
                                void* stream) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  if (dt != REHYAT_BF16) return fail(REHYAT_ERR_DTYPE, "the static-scratch call is bf16 only");
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(chunk_frames, L, 1, To));
  if (frames_before < 0) return fail(REHYAT_ERR_ARG, "frames_before must be >= 0");
  if (!q || !k_win || !v_win || !Wq || !Wk || !S || !Z || !out)
    return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k_win) || !aligned16(v_win) || !aligned16(out))
    return fail(REHYAT_ERR_ALIGN, "q/k_win/v_win/out not 16-byte aligned");
  // Same plan as rehyat_chunk_forward, with the fold split count lowered until the scratch fits.
  ChunkPlan pl = plan_chunk(d, dt, L, frames_before, chunk_frames, To, To);
  const size_t BH = (size_t)d.B * d.H;
  const size_t st_bytes = round_up(BH * d.D * d.F * 2, 256);
  const size_t wbd_bytes = round_up((size_t)d.H * 2 * d.F * d.D * 2, 256);
  // S^T, the block-diagonal W_q the attention's epilogue reads (the fold builds its compact
  // W_k itself), the fold partials
  auto total_for = [&](int splits) {
    return st_bytes + wbd_bytes + round_up(BH * splits * d.F * d.D * 4, 256) +
           round_up(BH * splits * d.F * 4, 256);
  };
  int splits = pl.splits;
  while (splits > 1 && total_for(splits) > kStaticScratchBytes) --splits;
  if (total_for(splits) > kStaticScratchBytes)
    return fail(REHYAT_ERR_WORKSPACE,
                "B*H=%zu needs %zu bytes of scratch; the library's static scratch holds %zu",
                BH, total_for(splits), kStaticScratchBytes);
  void* scratch = nullptr;
  RH_TRY(static_scratch_for_current_device(&scratch));
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  __nv_bfloat16* St = reinterpret_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* Wqbd = reinterpret_cast<__nv_bfloat16*>(ws + st_bytes);
  float* dS = reinterpret_cast<float*>(ws + st_bytes + wbd_bytes);
  float* dZ = reinterpret_cast<float*>(ws + st_bytes + wbd_bytes +
                                       round_up(BH * splits * d.F * d.D * 4, 256));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nbh = d.B * d.H;
  // Nothing in the scratch has to start at zero: every byte a kernel reads was written earlier
  // in this call (S^T by the scan, every split's partial by the fold kernel).
  RH_TRY(launch_scan_bf16(d, dS, dZ, 0, 1, 1, S, Z, St, nullptr, nullptr, nullptr, st));
  CUtensorMap mq, mk, mv, ms, mwq;
  RH_TRY(make_map(&mq, q, d.D, pl.nq, nbh));
  RH_TRY(make_map(&mk, k_win, d.D, pl.nkv, nbh));
  RH_TRY(make_map(&mv, v_win, d.D, pl.nkv, nbh));
  RH_TRY(make_map(&ms, St, d.F, d.D, nbh));
  RH_TRY(prepare_blockdiag(d, Wq, Wqbd, &mwq, st));
  rehyat::attn::Params ap{};
  ap.L = L; ap.T = chunk_frames; ap.Tc = chunk_frames; ap.To = To;
  ap.frames_before = frames_before; ap.kv_frame0 = frames_before - pl.o;
  ap.H = d.H; ap.P = kernel_P(d); ap.n_states = 1; ap.nq_rows = pl.nq;
  ap.kv_rows = ap.carry_rows = pl.nkv;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d.D));
  ap.bq = bq; ap.Z = Z; ap.out = static_cast<__nv_bfloat16*>(out);
  RH_TRY(launch_attn_bf16<false>(mq, mk, mv, ms, mwq, mq, ap, dim3((pl.nq + 255) / 256, nbh, 1),
                                 st));
  if (pl.fold_rows > 0) {
    rehyat::state::FoldParams fp{};
    fp.L = L; fp.H = d.H; fp.P = kernel_P(d); fp.single_rows = pl.fold_rows; fp.n_fold = 1;
    fp.kv_rows = fp.carry_rows = pl.nkv;
    fp.splits = splits; fp.G = d.G; fp.W = Wk; fp.bk = bk; fp.dS = dS; fp.dZ = dZ;
    RH_TRY(launch_fold_bf16(mk, mv, fp, dim3(splits, 1, nbh), st));
    rehyat::state::state_add_kernel<<<dim3((d.F * d.D + 255) / 256, nbh), 256, 0, st>>>(
        dS, dZ, splits, d.F, d.D, S, Z);
    RH_TRY(cuda_check(cudaGetLastError(), "state add launch"));
  }
  return REHYAT_OK;
}

int rehyat_chunk_states(rehyat_dims d, rehyat_dtype dt, int T, int L, int Tc, int To,
                        const void* k, const void* v, const float* Wk, const float* bk,
                        float* S_out, float* Z_out, void* workspace, size_t ws_bytes,
                        void* stream) {
  g_msg[0] = 0;
  RH_TRY(check_dims(d, dt));
  RH_TRY(check_path_shape(d, dt));
  RH_TRY(check_sched(T, L, Tc, To));
  if (!k || !v || !Wk || !S_out || !Z_out) return fail(REHYAT_ERR_ARG, "null pointer");
  if (!aligned16(k) || !aligned16(v)) return fail(REHYAT_ERR_ALIGN, "k/v not 16-byte aligned");
  const ForwardPlan pl = plan_forward(d, dt, T, L, Tc, To);
  if (!workspace || ws_bytes < pl.total)
    return fail(REHYAT_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", pl.total, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (dt == REHYAT_BF16)
    return forward_states_bf16(d, T, L, Tc, To, k, v, Wk, bk, pl, ws, nullptr, nullptr, S_out,
                               Z_out, st);
  return forward_states_f32(d, T, L, Tc, To, k, v, Wk, bk, pl, ws, S_out, Z_out, st);
}

int rehyat_gemm_bf16(int M, int N, int K, int batch, const void* A, long long lda,
                     long long a_batch, int a_mn, const void* B, long long ldb, long long b_batch,
                     int b_mn, void* C, long long ldc, long long c_batch, int c_bf16,
                     int accumulate, float alpha, void* stream) {
  g_msg[0] = 0;
  if (!A || !B || !C) return fail(REHYAT_ERR_ARG, "null pointer");
  return launch_gemm(M, N, K, batch, Operand{A, lda, a_batch, a_mn != 0},
                     Operand{B, ldb, b_batch, b_mn != 0}, C, ldc, c_batch, c_bf16 != 0,
                     accumulate != 0, alpha, static_cast<cudaStream_t>(stream));
}

int rehyat_selftest_wait_timeout(long long limit_ns, void* stream) {
  g_msg[0] = 0;
  if (limit_ns < 1000 || limit_ns > 2000000000LL)
    return fail(REHYAT_ERR_ARG, "limit_ns %lld outside [1e3, 2e9]", limit_ns);
  wait_timeout_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_ns));
  return cuda_check(cudaGetLastError(), "wait_timeout_selftest_kernel launch");
}

int rehyat_selftest_bounds(float* buf, long long n, long long bad_index, void* stream) {
  g_msg[0] = 0;
#ifndef REHYAT_DEBUG_BOUNDS
  (void)buf, (void)n, (void)bad_index, (void)stream;
  return fail(REHYAT_ERR_ARG, "not a debug-bounds build (compile with REHYAT_DEBUG_BOUNDS)");
#else
  if (!buf || n < 1 || n > (1LL << 30)) return fail(REHYAT_ERR_ARG, "need buf and 1 <= n <= 2^30");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned blocks = (unsigned)((n + 256) / 256);
  bounds_selftest_kernel<<<blocks, 256, 0, st>>>(buf, n, bad_index);
  return cuda_check(cudaGetLastError(), "bounds self-test launch");
#endif
}

int rehyat_sync_status(void* stream) {
  g_msg[0] = 0;
  RH_TRY(cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "stream sync"));
  int err = 0;
  RH_TRY(cuda_check(cudaMemcpyFromSymbol(&err, rehyat::sm100::g_device_error, sizeof(int)),
                    "read device error word"));
  if (err) {
    const int zero = 0;
    cudaMemcpyToSymbol(rehyat::sm100::g_device_error, &zero, sizeof(int));
    if (err == 2) {
      long long info[3] = {0, 0, 0};
      cudaMemcpyFromSymbol(info, rehyat::sm100::g_bounds_info, sizeof(info));
      return fail(REHYAT_ERR_BOUNDS,
                  "bounds check %lld failed: value %lld, limit %lld (access redirected or skipped)",
                  info[0], info[1], info[2]);
    }
    return fail(REHYAT_ERR_TIMEOUT, "a kernel wait timed out (device error %d)", err);
  }
  return REHYAT_OK;
}

}  // extern "C"
