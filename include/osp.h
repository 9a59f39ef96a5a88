/*
 * osp.h — C ABI of libosp.so: spacetime attention for video diffusion transformers on
 * NVIDIA B200 (sm_100a).
 *
 * The library computes, on one GPU, the attention hot path that the Open-Sora Plan and
 * CogVideoX pages describe:
 *   - 3D RoPE over the (t, h, w) latent token grid ("CogVideoX: Text-to-Video Diffusion
 *     Models with an Expert Transformer", section 2.2 "3D-RoPE"; "Open Video Models",
 *     The Breakthrough: separate rotation frequencies per axis);
 *   - dense 3D full attention over text + video tokens (CogVideoX section 2 and section 2.2
 *     "3D Full Attention");
 *   - Skiparse sparse attention, Single Skip and Group Skip with sparse ratio k
 *     ("Open-Sora Plan: Open-Source Large Video Generation Model", section 2.2.2);
 *   - video -> text cross-attention (Open-Sora Plan section 2.2.1), and Skiparse with a text
 *     prefix joined to every set;
 *   - the factorized 2D + 1D attention CogVideoX compares against (section 2.2, Table 8) and
 *     frame-causal attention (the Sora page);
 *   - packed batches of videos of different shapes, with per-sample RoPE grids and
 *     block-diagonal attention (CogVideoX section 3.1 "Multi-Resolution Frame Pack");
 *   - the backward pass of dense, Skiparse, frame-causal and factorized attention (training).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Layout. Every q/k/v/o tensor is contiguous BSHD bf16: [B][N][heads][head_dim], where
 *    N = text_len + T*H*W. Text tokens come first; video token v = text_len + (t*H + h)*W + w
 *    (row-major over the grid, w fastest).
 *  Pointers. All tensor pointers are DEVICE pointers owned by the caller, 16-byte aligned.
 *    The library never frees or retains them beyond the call's stream work.
 *  Sizes. The library sizes every access from the shape arguments alone and cannot see the
 *    allocations behind the pointers: each buffer must hold at least the elements its entry
 *    point documents for that shape.  A smaller buffer is out-of-bounds device access (the
 *    index-checked debug build skips such accesses and reports OSP_ERR_BOUNDS through
 *    osp_check_status; the release build does not check).
 *  Streams. `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *    enqueues work on that stream and returns; results are ready when the stream is.
 *  Errors. Every entry point returns an osp_status. On a non-zero return nothing has been
 *    enqueued and osp_get_last_error() describes the problem. Device-side faults of the
 *    bounded-wait kind (OSP_ERR_TIMEOUT) are reported later by osp_check_status().
 *  Scratch. On first use per device the library allocates (cudaMalloc) one small status
 *    word and caches it until process exit. Attention calls whose last partial wave of work
 *    is split over several KV ranges (see osp_attn_full) take a stream-ordered workspace
 *    (a few MB) from a library-owned per-device memory pool created on first use; freed
 *    blocks stay cached in that pool, so steady-state calls do not allocate from the driver.
 *  Threads. Entry points may be called from several host threads; the last-error message is
 *    per thread.
 */
#ifndef OSP_H_
#define OSP_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  OSP_OK = 0,
  OSP_ERR_INVALID_ARG = 1,  /* null pointer, bad dimension, RoPE split not summing to head_dim */
  OSP_ERR_UNSUPPORTED = 2,  /* head_dim not in {64, 96, 128}; text tokens in gather/scatter; ... */
  OSP_ERR_DIVISIBILITY = 3, /* T*H*W mod k != 0 (Single Skip) or mod k*k != 0 (Group Skip) */
  OSP_ERR_CUDA = 4,         /* a CUDA runtime/driver call or a kernel launch failed */
  OSP_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (see osp_check_status) */
  OSP_ERR_BOUNDS = 6        /* a device-side index check failed (see osp_check_status) */
} osp_status;

/* Skiparse modes ("Open-Sora Plan", section 2.2.2).
 *  OSP_SKIP_SINGLE: set g = video tokens {s*k + g : 0 <= s < T*H*W/k}.
 *  OSP_SKIP_GROUP:  groups of k adjacent tokens; set g = groups whose index is g mod k,
 *                   i.e. slot s = o*k + r of set g is token o*k*k + g*k + r.
 * Each set lists its tokens in ascending order ("slot" = position within the set). */
enum { OSP_SKIP_SINGLE = 0, OSP_SKIP_GROUP = 1 };

/* Problem shape. N = text_len + T*H*W tokens per sample. */
typedef struct {
  int32_t B;         /* batch size, >= 1 */
  int32_t text_len;  /* text tokens before the video tokens, >= 0 */
  int32_t T, H, W;   /* latent token grid, each >= 1 */
  int32_t heads;     /* attention heads, >= 1 */
  int32_t head_dim;  /* channels per head; RoPE needs it even, attention needs 64, 96 or 128 */
} osp_shape;

/* 3D RoPE parameters ("CogVideoX" section 2.2 "3D-RoPE"): channels [0, d_t) rotate with t,
 * [d_t, d_t+d_h) with h, [d_t+d_h, head_dim) with w. Inside a chunk of size d_a, channel pair
 * (2j, 2j+1) rotates by angle pos * theta^(-2j/d_a) (RoFormer). Positions are raw integer grid
 * indices (extrapolation, CogVideoX section 3.1). Text tokens are not rotated. */
typedef struct {
  int32_t d_t, d_h, d_w;  /* each even and >= 0 (0: that axis is not rotated); sum == head_dim */
  double theta;           /* frequency base, > 0 (10000 on the pages) */
} osp_rope;

/* Packed batches ("CogVideoX" section 3.1 "Multi-Resolution Frame Pack": videos of different
 * durations and resolutions share one batch, after Patch'n Pack).  A packed tensor is
 * [total][heads][head_dim] bf16, the samples' rows one after another; sample i is its text_len
 * text tokens followed by its T*H*W video tokens (row-major, w fastest).  Offsets ("bounds") are
 * HOST arrays of n + 1 int32 values: bounds[0] = 0, non-decreasing, sample i owning rows
 * [bounds[i], bounds[i+1]). */
#define OSP_MAX_SEGMENTS 256   /* samples per packed call */

typedef struct {
  int32_t text_len;  /* >= 0 */
  int32_t T, H, W;   /* >= 1 each */
} osp_sample_grid;

/* 3D RoPE of q and k.
 *  q, k:          [B][N][heads][head_dim] bf16, device.
 *  q_out, k_out:  same shape; may equal q / k (in place) but must not overlap them otherwise.
 *  Text tokens are copied unchanged (nothing is written for them when out == in).
 *  Arithmetic: fp64 rotation of the bf16 inputs (fp64 cos/sin), rounded once to bf16 (RNE):
 *    outputs are the correctly rounded rotation up to the last bits of fp64 cos/sin.
 *  Errors: OSP_ERR_INVALID_ARG (null, bad shape or split), OSP_ERR_CUDA (launch failed). */
int osp_rope3d(const void* q, const void* k, void* q_out, void* k_out, const osp_shape* shape,
               const osp_rope* rope, void* stream);

/* Dense 3D full attention ("CogVideoX" section 2.2 "3D Full Attention"): for every sample b
 * and head h, O = softmax(Q K^T * scale) V over all N tokens (text and video), bidirectional.
 *  q, k, v: [B][N][heads][head_dim] bf16, device (apply osp_rope3d first for 3D RoPE).
 *  o:       same shape, bf16, device; must not overlap q, k or v.
 *  softmax_scale: <= 0 selects 1/sqrt(head_dim).
 *  Arithmetic: bf16 operands on tcgen05 tensor cores, fp32 accumulation in tensor memory,
 *    fp32 online softmax, probabilities rounded to bf16 for the PV product, O rounded to bf16.
 *  Work split: the (sample, head, 256-query block) units run one per SM; when the last wave
 *    would leave SMs idle, its units are split into 2-8 KV ranges whose fp32 partials are merged
 *    exactly (log-sum-exp) by a second kernel. Results then differ from the unsplit order only
 *    in fp32 summation order. OSP_SPLIT_KV=0 in the environment disables the split.
 *  Errors: OSP_ERR_INVALID_ARG, OSP_ERR_UNSUPPORTED (head_dim not 64/96/128), OSP_ERR_CUDA. */
int osp_attn_full(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                  float softmax_scale, void* stream);

/* Video -> text cross-attention ("Open-Sora Plan" section 2.2.1: every block attends from the
 * video tokens to the mT5 text embeddings): for every sample b and head h,
 *   O = softmax(Q K^T * scale) V  with Q the video tokens and K, V the text tokens.
 *  q, o:  [B][T*H*W][heads][head_dim] bf16, device (video tokens only; o must not overlap q, k, v).
 *  k, v:  [B][text_len][heads][head_dim] bf16, device (text_len >= 1 key/value tokens).
 *  No RoPE is involved (text tokens have no grid position). Same kernel, arithmetic, scale
 *  convention and work split as osp_attn_full.
 *  Errors: OSP_ERR_INVALID_ARG (null, text_len < 1), OSP_ERR_UNSUPPORTED, OSP_ERR_CUDA. */
int osp_attn_cross(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                   float softmax_scale, void* stream);

/* Factorized "2D + 1D" attention ("CogVideoX" section 2.2 and Table 8: separate spatial and
 * temporal attention, the baseline 3D full attention replaces; the Sora page, "Video DiT
 * Diffusion Model": Local Spatial Attention and Causal Time Attention).  Video tokens only:
 * shape->text_len must be 0 (OSP_ERR_UNSUPPORTED otherwise); q, k, v, o as osp_attn_full.
 *
 * osp_attn_spatial: token (t, h, w) attends to the H*W tokens of frame t (block-diagonal over
 *   frames). Runs osp_attn_full's kernel on the B*T frames (same arithmetic and work split). */
int osp_attn_spatial(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                     float softmax_scale, void* stream);

/* osp_attn_temporal: token (t, h, w) attends to the tokens (t', h, w) of its spatial position,
 *   every t' (causal = 0) or t' <= t (causal = 1).
 *   T <= 64: a shared-memory-staged kernel with mma.sync tiles (the sets are too small for
 *   128-row tensor-memory tiles; the work is bound by HBM traffic), P rounded to bf16, fp32
 *   accumulation.  T > 64: the osp_skiparse_attn kernel with the position's tokens as Single
 *   Skip set pos, k = H*W (causal: with the osp_attn_frame_causal mask on one-token blocks).
 *   Errors: OSP_ERR_INVALID_ARG (causal not 0/1, ...), OSP_ERR_UNSUPPORTED (text, head_dim),
 *   OSP_ERR_CUDA. */
int osp_attn_temporal(const void* q, const void* k, const void* v, void* o, const osp_shape* shape, int32_t causal,
                      float softmax_scale, void* stream);

/* Frame-causal attention (the Sora page, "Long-Time Consistency Strategies": during generation of
 * frame i the model attends to all previous frames): over N = text_len + T*H*W tokens, query
 * token r attends to the first limit(r) tokens, limit = text_len for a text token and
 * text_len + (t + 1)*H*W for a token of frame t (text is one block before frame 0; it sees
 * itself, every video token sees it).  q, k, v, o as osp_attn_full; same kernel and arithmetic,
 * with key tiles past a query block's last limit skipped; no KV-range split.
 *  Errors: as osp_attn_full. */
int osp_attn_frame_causal(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                          float softmax_scale, void* stream);

/* Training: forward with saved statistics, and the backward pass (Open-Sora Plan section 2.2.2:
 * the model is trained with Skiparse attention).  sparse_k == 1: dense attention over
 * N = text_len + T*H*W tokens (as osp_attn_full); sparse_k > 1: Skiparse Single / Group Skip
 * (as osp_skiparse_attn, Group Skip needs k | 128), text_len > 0 joining the text prefix to
 * every set (a text query sees all N tokens, a video query of set g the text and set g).
 *
 * osp_attn_forward_train: o as the corresponding inference call (same kernel, arithmetic and work
 *   split), plus lse, the log2-domain log-sum-exp of every query row's scaled scores:
 *   lse[((b*G + g)*heads + h)*n_pad + s] = log2(sum_j exp2(score_sj * scale * log2(e))) for slot s
 *   of set g (G = 1 and slot = token for dense; G = k for Skiparse), n = N / G,
 *   n_pad = ceil(n / 128) * 128.  lse: device fp32 array of B * G * heads * n_pad values (the
 *   padding entries are not written), 16-byte aligned; it is an opaque input of the backward.
 *   Skiparse with text_len > 0: n = T*H*W / k for the video rows' block, which is followed by the
 *   text rows' lse[B*k*heads*n_pad + (b*heads + h)*L_pad + t], L_pad = ceil(text_len / 128) * 128
 *   (B * (k * heads * n_pad + heads * L_pad) values). */
int osp_attn_forward_train(const void* q, const void* k, const void* v, void* o, float* lse, const osp_shape* shape,
                           int32_t sparse_k, int32_t mode, float softmax_scale, void* stream);

/* osp_attn_backward: gradients of the attention output o with respect to q, k, v, given the
 *   upstream gradient dout (same shape as o) and the forward's o and lse:
 *     dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)), dQ = scale * dS K,
 *     dK = scale * dS^T Q, per (sample, set, head), with P = exp2(S * scale * log2(e) - lse).
 *   dq, dk, dv: [B][N][heads][head_dim] bf16, device, written completely; must not overlap the
 *   inputs.  Arithmetic: tcgen05 tensor cores, bf16 operands (P and dS rounded to bf16), fp32
 *   accumulation in tensor memory, outputs rounded to bf16.  Scratch: rowsum(dO * O) in a
 *   stream-ordered block (B * G * heads * n_pad floats) from the library's memory pool.
 *   Three kernel launches: row sums, dK/dV, and dQ (head_dim 96, 128), or at head_dim 64 the
 *   row sums, dK/dV with dQ accumulated into an fp32 scratch block (B * G * heads * n_pad * 64
 *   floats, same pool) by bulk reduce-adds, and a finalize that rounds dQ to bf16; the order of
 *   those fp32 additions follows the CTAs' timing, so dQ at head_dim 64 can differ from run to
 *   run in its last bits (dK, dV and the other head dims are reproducible).
 *   Skiparse with text_len > 0: the video queries' part runs over B*k gathered samples of
 *   [set g's n rows; the text rows] (queries: the first n), the text queries' part over the
 *   natural samples (queries: the first text_len rows); dK and dV of a row sum their fp32
 *   contributions (sets 0..k-1, then the text queries) before one rounding to bf16.  Scratch:
 *   the gathered q, k, v, o, dout and dq (bf16) and dk, dv (fp32) of B*k*(n + text_len) rows,
 *   and the text queries' fp32 dk, dv of B*N rows, from the same pool.
 *  Errors: as the forward, OSP_ERR_CUDA. */
int osp_attn_backward(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                      void* dq, void* dk, void* dv, const osp_shape* shape, int32_t sparse_k, int32_t mode,
                      float softmax_scale, void* stream);

/* Training with the frame-causal mask (osp_attn_frame_causal): the forward with its saved lse
 * (dense layout, G = 1: lse[(b*heads + h)*n_pad + token], n_pad = ceil(N / 128) * 128) and the
 * backward, with the same arithmetic as osp_attn_forward_train / osp_attn_backward and P zero
 * outside the mask.  The dK/dV kernel skips query tiles that cannot see its keys and the dQ kernel
 * key tiles past its queries' limit.
 *  Errors: as osp_attn_frame_causal, OSP_ERR_CUDA. */
int osp_attn_frame_causal_train(const void* q, const void* k, const void* v, void* o, float* lse,
                                const osp_shape* shape, float softmax_scale, void* stream);
int osp_attn_frame_causal_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                   const float* lse, void* dq, void* dk, void* dv, const osp_shape* shape,
                                   float softmax_scale, void* stream);

/* Training of the factorized (2D + 1D) attention (osp_attn_spatial, osp_attn_temporal): the
 * forward with its saved lse and the backward, with the arithmetic of osp_attn_forward_train /
 * osp_attn_backward.  Video tokens only (text_len 0); q, k, v, o, dout, dq, dk, dv as
 * osp_attn_backward (written completely, no overlap with the inputs).
 *
 * osp_attn_spatial_train / _backward: the dense kernels on the B*T frames, each of H*W tokens;
 *   lse[((b*T + t)*heads + h)*n_pad + (h'*W + w)], n_pad = ceil(H*W / 128) * 128.
 * osp_attn_temporal_train / _backward: the Skiparse kernels with spatial position pos = h*W + w
 *   as Single Skip set pos, k = H*W (slot t = frame t; causal = 1: P zero where t' > t, through
 *   the block-causal mask with one-slot blocks); lse[((b*H*W + pos)*heads + h)*n_pad + t],
 *   n_pad = ceil(T / 128) * 128.  With T <= 64 the training forward and the backward run per-set
 *   kernels instead (one warp per (sample, position, head) set, mma.sync tiles of 16 rows, bound
 *   by HBM traffic; the environment variable OSP_TEMPORAL_BWD=0 selects the tile kernels), with
 *   the same rounding points: P and dS in bf16 before their products, fp32 accumulation, bf16
 *   outputs; the forward writes the lse slots t < T of each set's row.
 *  Errors: OSP_ERR_INVALID_ARG (null or unaligned pointer, causal not 0/1), OSP_ERR_UNSUPPORTED
 *  (text, head_dim, too many frames or positions), OSP_ERR_CUDA. */
int osp_attn_spatial_train(const void* q, const void* k, const void* v, void* o, float* lse, const osp_shape* shape,
                           float softmax_scale, void* stream);
int osp_attn_spatial_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, const osp_shape* shape,
                              float softmax_scale, void* stream);
int osp_attn_temporal_train(const void* q, const void* k, const void* v, void* o, float* lse, const osp_shape* shape,
                            int32_t causal, float softmax_scale, void* stream);
int osp_attn_temporal_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                               const float* lse, void* dq, void* dk, void* dv, const osp_shape* shape, int32_t causal,
                               float softmax_scale, void* stream);

/* 3D RoPE of a packed batch (CogVideoX section 3.1: every video keeps its own position grid,
 * starting at (0, 0, 0); extrapolation, never rescaled).
 *  samples:       HOST array of n_samples (1 .. OSP_MAX_SEGMENTS) sample grids, read during the call.
 *  q, k:          packed [sum_i (text_len_i + T_i*H_i*W_i)][heads][head_dim] bf16, device.
 *  q_out, k_out:  same shape; may equal q / k. Text rows are copied (skipped in place).
 *  Arithmetic as osp_rope3d: sample i's rows equal what osp_rope3d gives for that sample alone.
 *  Errors: OSP_ERR_INVALID_ARG (null, n_samples out of range, bad grid or split), OSP_ERR_CUDA. */
int osp_rope3d_packed(const void* q, const void* k, void* q_out, void* k_out, const osp_sample_grid* samples,
                      int32_t n_samples, int32_t heads, int32_t head_dim, const osp_rope* rope, void* stream);

/* Block-diagonal attention over a packed batch (CogVideoX section 3.1; Patch'n Pack masks
 * attention to each example): query row r of sample i attends to the key/value rows of sample
 * i only, per head, O = softmax(Q_i K_i^T * scale) V_i.
 *  q_bounds:  HOST, n_seg + 1 offsets of the samples' rows in q and o.
 *  kv_bounds: HOST, n_seg + 1 offsets in k and v, or NULL for q_bounds (self-attention within
 *             each sample; with different bounds: per-sample cross-attention, e.g. each video's
 *             queries against its own prompt's text tokens).
 *  q, o:      [q_bounds[n_seg]][heads][head_dim] bf16, device; o must not overlap q, k, v.
 *  k, v:      [kv_bounds[n_seg]][heads][head_dim] bf16, device.
 *  n_seg:     1 .. OSP_MAX_SEGMENTS. A sample with query rows needs >= 1 key row; samples with
 *             no query rows are skipped.
 *  softmax_scale: <= 0 selects 1/sqrt(head_dim).
 *  Same kernel and arithmetic as osp_attn_full; work units (sample, head, 256-query block) are
 *  never split over KV ranges here. The bounds are copied into the launch's parameters, so the
 *  host arrays may be reused as soon as the call returns.
 *  Errors: OSP_ERR_INVALID_ARG (null, bad bounds, a sample with queries but no keys),
 *  OSP_ERR_UNSUPPORTED (head_dim, n_seg > OSP_MAX_SEGMENTS, > 2^30 rows), OSP_ERR_CUDA. */
int osp_attn_packed(const void* q, const void* k, const void* v, void* o, const int32_t* q_bounds,
                    const int32_t* kv_bounds, int32_t n_seg, int32_t heads, int32_t head_dim,
                    float softmax_scale, void* stream);

/* Training a model on packed batches (CogVideoX section 3.1: Multi-Resolution Frame Pack trains on
 * mixed-shape batches): osp_attn_packed's self-attention (each sample attends to its own rows)
 * with the row log-sum-exp saved, and its backward pass.
 *  bounds:  HOST, n_seg + 1 offsets of the samples' rows in every tensor (as q_bounds above).
 *  lse:     fp32, device, 16-byte aligned, [heads][osp_attn_packed_lse_rows(bounds, n_seg)];
 *           sample i's rows start at the start of its 256-row blocks (the sum of
 *           ceil(len_j / 256) * 256 over j < i); row r of sample i holds m + log2(l) of its scaled
 *           scores (log2 domain); padding slots are not written.
 *  osp_attn_packed_train: o = osp_attn_packed(q, k, v, bounds, NULL) bit for bit, plus lse.
 *  osp_attn_packed_backward: dq, dk, dv [bounds[n_seg]][heads][head_dim] bf16, device (not
 *    overlapping the inputs), from q, k, v, o, dout and the lse of osp_attn_packed_train: each
 *    sample's own attention backward, the arithmetic of osp_attn_backward (P and dS rounded to
 *    bf16, fp32 accumulation); the call takes a stream-ordered workspace from the library's pool
 *    (row sums, and at head_dim 64 an fp32 dQ accumulator of heads * lse_rows * 64 floats).
 *  osp_attn_packed_lse_rows: the lse row count per head (>= 0), or -OSP_ERR_INVALID_ARG for bad
 *    bounds.
 *  Errors: OSP_ERR_INVALID_ARG (null or unaligned pointer, bad bounds), OSP_ERR_UNSUPPORTED
 *  (head_dim, n_seg > OSP_MAX_SEGMENTS), OSP_ERR_CUDA. */
int osp_attn_packed_lse_rows(const int32_t* bounds, int32_t n_seg);
int osp_attn_packed_train(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* bounds,
                          int32_t n_seg, int32_t heads, int32_t head_dim, float softmax_scale, void* stream);
int osp_attn_packed_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, const int32_t* bounds, int32_t n_seg,
                             int32_t heads, int32_t head_dim, float softmax_scale, void* stream);

/* Skiparse gather ("Open-Sora Plan" section 2.2.2: sequence cut to 1/k, batch grown k-fold):
 *   x_out[b*k + g][s] = RoPE(x[b][token(g, s)])   for q and k (RoPE skipped if rope == NULL),
 *   v_out[b*k + g][s] = v[b][token(g, s)]         (exact copy).
 *  q, k, v:     [B][T*H*W][heads][head_dim] bf16, device; shape->text_len must be 0.
 *               k/k_out and v/v_out may be NULL together (that tensor is skipped).
 *  *_out:       [B*k][T*H*W/k][heads][head_dim] bf16, device, not overlapping the inputs.
 *  Errors: OSP_ERR_INVALID_ARG (k < 1, bad mode, null q/q_out), OSP_ERR_UNSUPPORTED
 *  (text_len != 0), OSP_ERR_DIVISIBILITY, OSP_ERR_CUDA. */
int osp_skiparse_gather(const void* q, const void* k, const void* v, void* q_out, void* k_out,
                        void* v_out, const osp_shape* shape, int32_t sparse_k, int32_t mode,
                        const osp_rope* rope, void* stream);

/* Inverse of the gather for one tensor: o[b][token(g, s)] = o_perm[b*k + g][s] (exact copy).
 *  o_perm: [B*k][T*H*W/k][heads][head_dim] bf16, device; o: [B][T*H*W][heads][head_dim].
 *  Errors as for osp_skiparse_gather. */
int osp_skiparse_scatter(const void* o_perm, void* o, const osp_shape* shape, int32_t sparse_k,
                         int32_t mode, void* stream);

/* Fused Skiparse attention: every video token attends only to the tokens of its own set
 * ("Open-Sora Plan" section 2.2.2). The set structure is folded into the kernel's tile
 * address map, so no permuted copy of q/k/v/o is ever written.
 *  q, k, v, o: [B][text_len + T*H*W][heads][head_dim] bf16, device, natural token order.
 *  Text prefix (text_len > 0; the pages give no joint text + Skiparse scheme, so the text tokens
 *    are read as global tokens): a video token of set g attends to every text token and to the
 *    video tokens of set g; a text token attends to every token of its sample.  Two launches of
 *    the same kernel (video queries with the text rows prepended to every set's KV range, then
 *    the text queries over all rows).
 *  Group Skip additionally needs k to divide 128 (a power of two up to 128).
 *  Same arithmetic and scale convention as osp_attn_full. k == 1 is dense attention.
 *  Errors: OSP_ERR_INVALID_ARG, OSP_ERR_UNSUPPORTED, OSP_ERR_DIVISIBILITY, OSP_ERR_CUDA. */
int osp_skiparse_attn(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                      int32_t sparse_k, int32_t mode, float softmax_scale, void* stream);

/* Skiparse index map: dev_out[g*(n_video/k) + s] = token(g, s), int32, device, n_video entries.
 *  Errors: OSP_ERR_INVALID_ARG, OSP_ERR_DIVISIBILITY, OSP_ERR_CUDA. */
int osp_skiparse_index_map(int32_t n_video, int32_t sparse_k, int32_t mode, int32_t* dev_out,
                           void* stream);

/* Dense 3D full attention exactly like osp_attn_full, for callers that cannot allocate device
 * memory. The pages have no counterpart: this exists only for how the library is called.
 * Who needs it: callers whose device memory is entirely owned by another allocator (a
 * framework's caching pool or a serving runtime that reserves the GPU's memory up front), and
 * latency-critical callers, for whom cudaMalloc's implicit device synchronisation would stall
 * every stream. osp_attn_full allocates one status word with cudaMalloc on its first call per
 * device; this entry point never calls cudaMalloc, cudaFree or any allocating routine.
 *  Scratch: the kernel's only scratch, its 4-byte status word, lives in a file-scope
 *    __device__ array of 256 bytes (the maximum; every problem size needs the same 4 bytes, and
 *    a call whose scratch would exceed the array is rejected with OSP_ERR_UNSUPPORTED). Every
 *    GPU that loads the library holds the array until the process exits.
 *  First call per device: looks up the array's device address (cudaGetSymbolAddress) with that
 *    device current and caches it; make that first call before any stream capture (a first
 *    call on a capturing stream returns OSP_ERR_CUDA and says so). Device ordinals 0..63 only
 *    (a higher ordinal returns OSP_ERR_UNSUPPORTED).
 *  Sharing: all calls on a device share the array, and each call clears the status word on
 *    `stream` before its kernel. Calls that overlap on the GPU (different streams) race on it.
 *  Errors: as osp_attn_full (OSP_ERR_INVALID_ARG, OSP_ERR_UNSUPPORTED, OSP_ERR_CUDA). A
 *    bounded-wait timeout inside the kernel is recorded in the static word; osp_check_status
 *    reports it (OSP_ERR_TIMEOUT, output invalid) and clears it, allocating nothing.
 *  Arguments, layout and arithmetic are those of osp_attn_full, without its split of the last
 *    wave (which needs a workspace): results are bit-identical whenever osp_attn_full does not
 *    split, and otherwise differ only in fp32 summation order. */
int osp_attn_full_noalloc(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                          float softmax_scale, void* stream);

/* Synchronises `stream`, then reads and clears this device's status words: the library's own
 * word and, once osp_attn_full_noalloc has run on the device, that entry point's static word.
 * A word that does not exist yet has never been written and is skipped, so this call allocates
 * nothing.
 * Returns OSP_OK, OSP_ERR_TIMEOUT (a kernel's bounded wait gave up; its output is invalid),
 * OSP_ERR_BOUNDS, or OSP_ERR_CUDA (the synchronisation or the read failed). */
int osp_check_status(void* stream);

/* Message for the last non-zero return on the calling thread ("" if none). The pointer stays
 * valid until the next call on the same thread. */
const char* osp_get_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int osp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OSP_H_ */
