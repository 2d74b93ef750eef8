/*
 * rehyat.h - C ABI of librehyat.so: the forward pass of ReHyAt chunk-wise recurrent hybrid
 * attention on NVIDIA B200 (sm_100a).
 *
 * What is computed (sources: "ReHyAt overview" page, maplevalley.com.cn news 2180822, §2.2.1
 * hybrid output, §2.2.2 feature map, §2.3 recurrence and states, §5.2 streaming loop; and
 * "Neuer Ansatz zur effizienten Videogenerierung mit ReHyAt", mind-verse.de, sections
 * "Temporär segmentierte hybride Aufmerksamkeit" and "Rekurrente Formulierung"):
 *
 *   A video of T latent frames with L = frame_tokens tokens per frame is a token sequence of
 *   N = T*L rows, frame-major.  Frames are grouped into temporal chunks of Tc frames; chunk c
 *   owns query frames [c*Tc, e_c), e_c = min((c+1)*Tc, T).  A query of chunk c attends
 *     - with exact softmax weights exp(q.k/sqrt(D)) to the key frames [w_c, e_c),
 *       w_c = max(0, c*Tc - To)  (its own chunk, bidirectional, plus To frames before it);
 *     - with linear weights phi_q(q).phi_k(k) to every earlier key frame [0, w_c), read from
 *       the running states S_c = sum phi_k(k) v^T (F x D) and Z_c = sum phi_k(k) (F);
 *     - not at all to later frames;
 *   and the two parts share one normaliser:
 *     o = (sum_{j in window} e^{q.k_j/sqrt(D)} v_j + phi_q(q)^T S_c)
 *       / (sum_{j in window} e^{q.k_j/sqrt(D)}     + phi_q(q)^T Z_c).
 *   After chunk c the frames that leave the window, [w_c, w_{c+1}), are folded into (S, Z).
 *
 *   phi(x) (separate weights for q and k): u = grouped 1x1 linear of x (G groups; group g maps
 *   x[g*D/G, (g+1)*D/G) to u[g*F/G, (g+1)*F/G) with W[g] of shape (F/G, D/G)) plus bias; u is
 *   split into P contiguous parts (the first F mod P parts one longer) and part p (1-based)
 *   becomes softplus(u_p)^p; the parts are concatenated back in order.
 *
 * Conventions for every call:
 *   - Tensors are dense, row-major, per (b, h) contiguous: a "[B,H,n,D]" tensor holds row r of
 *     head h of batch b at element ((b*H + h)*n + r)*D.  Device pointers unless stated.
 *   - q, k, v, out, phi, the states and the workspace must be 16-byte aligned.
 *   - Weights W are fp32 [H, G, F/G, D/G]; biases fp32 [H, F] or NULL (zero).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only enqueues work
 *     on it: the library never allocates device memory, never synchronises, and keeps no state
 *     between calls other than the device error word read by rehyat_sync_status().
 *   - The caller owns every buffer.  Buffers may not overlap, except where stated.  Sizes come
 *     from the integer arguments; the library cannot see how large a buffer really is, so a
 *     buffer smaller than its documented shape is read or written past its end.  (The Python
 *     binding compares every tensor's shape with the shape its call implies.)
 *   - dtype REHYAT_BF16: q, k, v, out (and phi) are bf16; arithmetic is bf16 tensor-core
 *     products with fp32 accumulation, fp32 softmax and fp32 states.  Requires D = F = 128.
 *     dtype REHYAT_F32: everything fp32 on CUDA cores; requires D % 32 == 0, D <= 256,
 *     F <= 256.
 *   - Return value: REHYAT_OK or a negative rehyat_status; rehyat_last_error() then gives a
 *     message (per host thread).  A bad argument is reported before anything is enqueued.
 */
#ifndef REHYAT_H
#define REHYAT_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  REHYAT_OK = 0,
  REHYAT_ERR_ARG = -1,       /* null pointer, non-positive size, Tc < 1, To < 0, P out of range */
  REHYAT_ERR_SHAPE = -2,     /* D, F, G combination not supported for the dtype */
  REHYAT_ERR_DTYPE = -3,     /* unknown dtype */
  REHYAT_ERR_WORKSPACE = -4, /* workspace NULL or smaller than the *_workspace_size query */
  REHYAT_ERR_CUDA = -5,      /* a CUDA runtime call or a launch failed */
  REHYAT_ERR_TIMEOUT = -6,   /* a kernel's bounded wait gave up (from rehyat_sync_status) */
  REHYAT_ERR_ALIGN = -7,     /* a pointer is not 16-byte aligned */
  REHYAT_ERR_BOUNDS = -8     /* debug-bounds builds: a TMA coordinate or store index was out of
                                range (from rehyat_sync_status); the access was redirected to a
                                legal coordinate or skipped, so results are not to be trusted */
} rehyat_status;

typedef enum { REHYAT_F32 = 0, REHYAT_BF16 = 1 } rehyat_dtype;

/* Which feature map phi follows the grouped linear u = x W_g^T + b:
 *   REHYAT_PHI_POLY: split u into P contiguous parts, part p (1-based) -> softplus(u_p)^p
 *                    (the polynomial map of the "ReHyAt overview" page §2.2.2);
 *   REHYAT_PHI_ELU1: elu(u) + 1 (the linear-attention map of the same page §2.1.2; with
 *                    G = D groups of 1 x 1 weights all 1 and no bias it is elu(x) + 1 of the
 *                    raw token, as printed there).  P is then ignored. */
typedef enum { REHYAT_PHI_POLY = 0, REHYAT_PHI_ELU1 = 1 } rehyat_phi;

/* Problem dimensions shared by all calls: batch B, heads H, head dim D, feature count F of phi,
 * group count G of its grouped linear (D % G == 0, F % G == 0), polynomial parts P (1..F), and
 * the feature map kind `phi` (a rehyat_phi; 0, the polynomial map, when zero-initialised). */
typedef struct {
  int B, H, D, F, G, P;
  int phi;
} rehyat_dims;

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char* rehyat_last_error(void);

/* ABI version of this library (major*100 + minor). */
int rehyat_version(void);

/* 1 if this library was built with REHYAT_DEBUG_BOUNDS (the package build's debug-bounds
 * variant, librehyat_debug.so), else 0.  Such a build checks, before every TMA tile load of the
 * forward kernels (attention, fold, phi_q), that the coordinates lie in the tensor (inner
 * coordinate a multiple of 16 bytes inside the row, first row no more than one box outside,
 * depth inside), and before every global store of those kernels (outputs, partial sums, lone-tile
 * parts) that the index lies in its buffer.  A failed check does not trap: it records the first
 * failure (site, value, limit) in the device error word, redirects the copy to coordinate
 * (0, 0, 0) or skips the store, and rehyat_sync_status() returns REHYAT_ERR_BOUNDS. */
int rehyat_debug_bounds(void);

/* Feature map phi of the "ReHyAt overview" page §2.2.2, standalone.
 *   x    [B,H,n_tokens,D] (dtype), W [H,G,F/G,D/G] fp32, bias [H,F] fp32 or NULL,
 *   phi  [B,H,n_tokens,F] (dtype), written.
 * Any D, F, G, P that satisfy the dims rules (no D = F = 128 requirement here). */
int rehyat_featmap(rehyat_dims d, rehyat_dtype dt, int n_tokens, const void* x, const float* W,
                   const float* bias, void* phi, void* stream);

/* Workspace bytes rehyat_forward needs for these sizes (written to *bytes). */
int rehyat_forward_workspace_size(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens,
                                  int Tc, int To, size_t* bytes);

/* Hybrid attention over a whole sequence (every chunk of the §2.2.1 schedule in one call; the
 * §2.3 states are formed as prefix sums of per-chunk folds, so chunks run in parallel).
 *   q, k, v  [B,H,T*frame_tokens,D] (dtype);  Wq/bq, Wk/bk: phi_q and phi_k parameters;
 *   out      [B,H,T*frame_tokens,D] (dtype), written;
 *   workspace: device scratch of at least rehyat_forward_workspace_size() bytes. */
int rehyat_forward(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                   const void* q, const void* k, const void* v, const float* Wq, const float* bq,
                   const float* Wk, const float* bk, void* out, void* workspace,
                   size_t ws_bytes, void* stream);

/* rehyat_forward in three phases on the same workspace (rehyat_forward is exactly
 * rehyat_forward_states, rehyat_forward_phiq, rehyat_forward_attend in that order):
 *   _states: the §2.3 folds of every chunk and their prefix sums (the state each chunk reads),
 *            written into the workspace; reads k, v and phi_k's parameters;
 *   _phiq:   phi_q of every query row whose chunk reads a linear state, into the workspace;
 *   _attend: the hybrid output of every chunk from q, k, v and the workspace.
 * The workspace must not change between the calls.  Useful to reuse the states of one (k, v)
 * across several query sets, and to time the phases separately. */
int rehyat_forward_states(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                          const void* k, const void* v, const float* Wk, const float* bk,
                          void* workspace, size_t ws_bytes, void* stream);
int rehyat_forward_phiq(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                        const void* q, const float* Wq, const float* bq, void* workspace,
                        size_t ws_bytes, void* stream);
int rehyat_forward_attend(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                          const void* q, const void* k, const void* v, void* out,
                          const void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes rehyat_chunk_forward needs for one chunk of chunk_frames frames. */
int rehyat_chunk_workspace_size(rehyat_dims d, rehyat_dtype dt, int frame_tokens,
                                int chunk_frames, int To, size_t* bytes);

/* One step of the streaming loop of the "ReHyAt overview" page §5.2: the chunk whose first
 * frame is frame `frames_before` of the video, `chunk_frames` frames long.
 *   o = min(To, frames_before) overlap frames precede it in the softmax window.
 *   q      [B,H,chunk_frames*L,D]              the chunk's queries;
 *   k_win, v_win [B,H,(o+chunk_frames)*L,D]    the overlap frames followed by the chunk's own;
 *   S [B,H,F,D] fp32, Z [B,H,F] fp32 (in/out)  the states holding every frame before the
 *                                              window (zeros for the first chunk);
 *   out    [B,H,chunk_frames*L,D]              written.
 * After the output, the window frames the next chunk no longer sees (the first
 * max(0, frames_before + chunk_frames - To) - (frames_before - o) of them, assuming the next
 * chunk uses the same To) are folded into S and Z in place.  Memory use does not depend on how
 * many chunks came before. */
int rehyat_chunk_forward(rehyat_dims d, rehyat_dtype dt, int frame_tokens, int frames_before,
                         int chunk_frames, int To, const void* q, const void* k_win,
                         const void* v_win, const float* Wq, const float* bq, const float* Wk,
                         const float* bk, float* S, float* Z, void* out, void* workspace,
                         size_t ws_bytes, void* stream);

/* The streaming step with the overlap frames kept by the library: the caller passes only the
 * chunk (k, v [B,H,chunk_frames*L,D]) and a carry buffer per tensor (k_carry, v_carry
 * [B,H,carry_frames*L,D], inout, same dtype): the last carry_frames frames of K and V seen so
 * far, right-aligned (after f frames, only the last min(f, carry_frames) are meaningful).  The
 * result is that of rehyat_chunk_forward_sched (To_next as there) on the window [the last
 * min(To, frames_before) carried frames | the chunk]; bf16 kernels read that window in place
 * from the carry and the chunk, fp32 assembles it in the workspace.  Afterwards the carry holds
 * the last carry_frames frames of (carry ++ chunk).  Needs To <= carry_frames; a
 * zero-initialised carry is fine for the first call.  The state between calls is then S, Z and
 * the carry: the method's recurrent state (page §2.3).  Workspace:
 * rehyat_chunk_carry_workspace_size with the largest chunk_frames and To of the stream. */
int rehyat_chunk_carry_workspace_size(rehyat_dims d, rehyat_dtype dt, int frame_tokens,
                                      int chunk_frames, int To, int carry_frames, size_t* bytes);
int rehyat_chunk_forward_carry(rehyat_dims d, rehyat_dtype dt, int frame_tokens,
                               int frames_before, int chunk_frames, int To, int To_next,
                               int carry_frames, const void* q, const void* k, const void* v,
                               const float* Wq, const float* bq, const float* Wk,
                               const float* bk, float* S, float* Z, void* k_carry,
                               void* v_carry, void* out, void* workspace, size_t ws_bytes,
                               void* stream);

/* rehyat_chunk_forward for a variable chunk schedule ("ReHyAt overview" page §5.2: a longer
 * chunk for key frames such as the first, more overlap where motion is strong): chunk_frames
 * and To may change from call to call, and To_next is the overlap the NEXT call will use.
 * After the output, the window frames that the next window no longer holds, [w_c, w_{c+1}) with
 * w_c = frames_before - min(To, frames_before) and w_{c+1} = max(0, frames_before +
 * chunk_frames - To_next), are folded into S and Z.  REHYAT_ERR_ARG if To_next < 0 or if the
 * next window would reach frames this call's window does not hold (min(To_next,
 * frames_before + chunk_frames) > min(To, frames_before) + chunk_frames: they were folded
 * before).  The workspace must have the size rehyat_chunk_workspace_size gives for the largest
 * chunk_frames and To of the schedule.  rehyat_chunk_forward is this call with To_next = To. */
int rehyat_chunk_forward_sched(rehyat_dims d, rehyat_dtype dt, int frame_tokens,
                               int frames_before, int chunk_frames, int To, int To_next,
                               const void* q, const void* k_win, const void* v_win,
                               const float* Wq, const float* bq, const float* Wk,
                               const float* bk, float* S, float* Z, void* out, void* workspace,
                               size_t ws_bytes, void* stream);

/* rehyat_chunk_forward for callers that cannot allocate device memory: no workspace argument.
 * The pages have no counterpart of this call; it exists for callers such as a plugin inside a
 * host framework that owns every allocation, or a code path that must not call cudaMalloc
 * (for example while another component is capturing or replaying work).  Same arguments and
 * results as rehyat_chunk_forward (bf16 only); the scratch it needs lives in a fixed 16 MiB
 * array inside the library's device memory, which every GPU that loads the library keeps for
 * the life of the process.
 *   - The first call on a device looks up that array's device address (once per device, with
 *     the device current); make that first call before any stream capture.
 *   - Returns REHYAT_ERR_WORKSPACE, before anything is enqueued, when the scratch does not fit
 *     the array.  With one fold split it needs B*H*(6*F*D + 4*F) + 4*H*F*D bytes (S^T, the
 *     fold partials and one block-diagonal weight copy, each part rounded up to 256 B): at
 *     D = F = 128 that is 98,816 bytes per (b, h) plus 65,536 per head, so B*H <= 156 at
 *     H = 12 and B <= 169 at H = 1.  When the token splits rehyat_chunk_forward would use for
 *     the fold do not fit, fewer are used (down to one).
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - Every call shares the one array, whatever the stream: calls whose work overlaps on the
 *     GPU race on it and must be ordered by the caller (same stream, or events).
 *   - Nothing in the array needs to start at zero; it keeps the last call's contents. */
int rehyat_chunk_forward_static(rehyat_dims d, rehyat_dtype dt, int frame_tokens,
                                int frames_before, int chunk_frames, int To, const void* q,
                                const void* k_win, const void* v_win, const float* Wq,
                                const float* bq, const float* Wk, const float* bk, float* S,
                                float* Z, void* out, void* stream);

/* The states every chunk of rehyat_forward reads (§2.3), for inspection and testing:
 *   S_out [B,H,C,F,D] fp32 and Z_out [B,H,C,F] fp32 with C = ceil(T/Tc); S_out[..,c,..] is the
 *   sum over key frames [0, w_c) of phi_k(k) v^T.  Same workspace as rehyat_forward. */
int rehyat_chunk_states(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                        const void* k, const void* v, const float* Wk, const float* bk,
                        float* S_out, float* Z_out, void* workspace, size_t ws_bytes,
                        void* stream);

/* ---- training: the forward that keeps its row statistics, and the backward pass ----
 * The pages train the feature maps by distillation and then fine-tune ("ReHyAt overview" §3.1.1,
 * §3.1.2); both need the gradients of the §2.2.1 output formula.  bf16 only (D = F = 128).
 *
 * rehyat_forward_train: rehyat_forward plus lse [B,H,T*L] fp32: for every query row, log2 of
 *   its denominator (softmax sum plus linear term) in the units where key j weighs
 *   2^(q.k_j log2(e) / sqrt(D)).  Same workspace as rehyat_forward.
 * rehyat_backward: given q, k, v, the weights, the forward's out and lse, and dout = dL/dout
 *   [B,H,T*L,D] bf16, writes dq, dk, dv [B,H,T*L,D] fp32, dWq, dWk [H,G,F/G,D/G] fp32 and dbq,
 *   dbk [H,F] fp32 (summed over the batch; written even when bq / bk are NULL).  Needs
 *   frame_tokens % 8 == 0 (REHYAT_ERR_SHAPE otherwise) and a workspace of
 *   rehyat_backward_workspace_size bytes (it holds one chunk's score matrices: about
 *   12 B * B*H * (Tc*L) * ((Tc+To)*L) plus O(B*H*T*L*F)). */
int rehyat_forward_train(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                         const void* q, const void* k, const void* v, const float* Wq,
                         const float* bq, const float* Wk, const float* bk, void* out, float* lse,
                         void* workspace, size_t ws_bytes, void* stream);
int rehyat_backward_workspace_size(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens,
                                   int Tc, int To, size_t* bytes);
int rehyat_backward(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                    const void* q, const void* k, const void* v, const float* Wq,
                    const float* bq, const float* Wk, const float* bk, const void* out,
                    const float* lse, const void* dout, float* dq, float* dk, float* dv,
                    float* dWq, float* dbq, float* dWk, float* dbk, void* workspace,
                    size_t ws_bytes, void* stream);

/* Batched bf16 GEMM on the tensor cores (the building block of the backward pass; no
 * counterpart on the pages): for b < batch, C[b] = alpha * A[b] B[b] (accumulate = 0) or
 * C[b] += alpha * A[b] B[b] (accumulate = 1), fp32 accumulation, C fp32 (c_bf16 = 0) or bf16.
 *   A is M x K: element (m, k) of batch b at A + b*a_batch + m*lda + k (a_mn = 0) or
 *               A + b*a_batch + k*lda + m (a_mn = 1); bf16.
 *   B is K x N: element (k, n) at B + b*b_batch + n*ldb + k (b_mn = 0) or
 *               B + b*b_batch + k*ldb + n (b_mn = 1); bf16.
 *   C [M][N] per batch: element (m, n) at C + b*c_batch + m*ldc + n.
 * Strides in elements; A, B strides multiples of 8, fp32 ldc a multiple of 4, pointers 16-byte
 * aligned (REHYAT_ERR_ALIGN otherwise).  Enqueued on `stream`; allocates nothing. */
int rehyat_gemm_bf16(int M, int N, int K, int batch, const void* A, long long lda,
                     long long a_batch, int a_mn, const void* B, long long ldb, long long b_batch,
                     int b_mn, void* C, long long ldc, long long c_batch, int c_bf16,
                     int accumulate, float alpha, void* stream);

/* Context parallelism over chunk ranges ("ReHyAt overview" page §2.3: the state a chunk reads
 * is a sum over the folds of all chunks before it, so a sequence splits into contiguous chunk
 * ranges whose only coupling is that sum and the To overlap frames).  A segment is the chunks
 * [c0, c1) of a bf16 sequence of T frames (0 <= c0 < c1 <= ceil(T/Tc)):
 *   query frames [s0, s1) with s0 = c0*Tc, s1 = min(c1*Tc, T);
 *   key/value frames [h0, s1) with h0 = max(0, s0 - To) (the To halo frames before s0 included).
 *   q_seg [B,H,(s1-s0)*L,D], k_seg, v_seg [B,H,(s1-h0)*L,D], out_seg [B,H,(s1-s0)*L,D] bf16.
 * Two phases on one workspace (sized by rehyat_segment_workspace_size, unchanged in between):
 *   _states: the folds of the segment's chunks (every fold c' in [c0, min(c1, C-1)), frames
 *            [w_c', w_c'+1)) into the workspace, and their sum into S_seg [B,H,F,D] and
 *            Z_seg [B,H,F] (fp32, caller-owned; zeros when the segment folds nothing);
 *   _attend: the outputs of the segment's chunks.  S_prefix [n_prefix][B,H,F,D] and Z_prefix
 *            [n_prefix][B,H,F] hold the S_seg/Z_seg of every segment before this one (n_prefix
 *            of them, in sequence order; n_prefix = 0 and null pointers for the first segment);
 *            they are summed in that order into the state of chunk c0.
 * Between the phases a multi-GPU caller gathers every rank's S_seg/Z_seg; nothing else crosses
 * ranks except the halo frames of k and v.  With one segment (c0 = 0, c1 = C, n_prefix = 0) the
 * result equals rehyat_forward up to the order of fp32 additions in the states.  bf16 only
 * (REHYAT_ERR_DTYPE otherwise).  Enqueued on `stream`; allocates nothing. */
int rehyat_segment_workspace_size(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc,
                                  int To, int c0, int c1, size_t* bytes);
int rehyat_segment_states(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                          int c0, int c1, const void* k_seg, const void* v_seg, const float* Wk,
                          const float* bk, float* S_seg, float* Z_seg, void* workspace,
                          size_t ws_bytes, void* stream);
int rehyat_segment_attend(rehyat_dims d, rehyat_dtype dt, int T, int frame_tokens, int Tc, int To,
                          int c0, int c1, const void* q_seg, const void* k_seg, const void* v_seg,
                          const float* Wq, const float* bq, int n_prefix, const float* S_prefix,
                          const float* Z_prefix, void* out_seg, void* workspace, size_t ws_bytes,
                          void* stream);

/* Failure-path self test (no counterpart on the pages): enqueue on `stream` one small kernel whose
 * warps wait on an mbarrier that nothing arrives on, with the same bounded wait the other
 * kernels use but a limit of `limit_ns` nanoseconds (1e3 .. 2e9).  The wait gives up, the kernel
 * sets the device error word and returns, so the next rehyat_sync_status() on that stream
 * returns REHYAT_ERR_TIMEOUT (and clears the word); the context stays usable.  Returns
 * REHYAT_ERR_ARG for a limit out of range, REHYAT_ERR_CUDA if the launch fails. */
int rehyat_selftest_wait_timeout(long long limit_ns, void* stream);

/* Exercises the bounds checks of a debug-bounds build: a kernel writes 1.0 to buf[0, n) and then
 * attempts buf[bad_index] through a store check against [0, n).  With bad_index outside [0, n)
 * the check records the failure and skips the store, and the next rehyat_sync_status() returns
 * REHYAT_ERR_BOUNDS.  buf [n + slack] fp32 device memory: give room past n for bad_index, so the
 * write stays inside the buffer even if the check were absent.  Returns REHYAT_ERR_ARG in a
 * build without the checks (rehyat_debug_bounds() == 0) or for n outside [1, 2^30]. */
int rehyat_selftest_bounds(float* buf, long long n, long long bad_index, void* stream);

/* Synchronise `stream` and report device-side failures of earlier calls: REHYAT_ERR_TIMEOUT if
 * a kernel's bounded wait gave up, REHYAT_ERR_BOUNDS if a bounds check of a debug-bounds build
 * failed (the error word is then cleared), REHYAT_ERR_CUDA if the stream reports a CUDA error,
 * else REHYAT_OK. */
int rehyat_sync_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* REHYAT_H */
