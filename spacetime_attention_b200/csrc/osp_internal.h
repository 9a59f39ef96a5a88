// Internal declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/osp.h"
#include "osp_device.cuh"

namespace osp {

constexpr int kMaxSegments = OSP_MAX_SEGMENTS;

// Sets the calling thread's last-error message; returns `code`.
int set_error(int code, const char* fmt, ...);

// OSP_ERR_CUDA with the kernel's name if the last launch failed, else OSP_OK.
int check_launch(const char* what);

// SM count of the current device (cached per device).
int device_sm_count();

// Per-device status word (allocated on first use, kept until exit).
unsigned* device_status_word();
// The status words of the current device that exist, without creating any: the library's
// (nullptr before its first use) and osp_attn_full_noalloc's static word (nullptr before that
// entry point's first call on this device).
unsigned* device_status_word_if_present();
unsigned* noalloc_status_word_if_present();

// Bounded-wait limit for the attention kernels, in nanoseconds (OSP_WAIT_TIMEOUT_MS, default
// 2000 ms; read on every launch).
uint64_t wait_timeout_ns();

// Test knob (OSP_DEBUG_WITHHOLD_Q=1, read on every launch): the attention kernel never loads Q,
// so its bounded waits run out and the launch reports OSP_ERR_TIMEOUT through osp_check_status.
int debug_withhold_q();

// Per-device memory pool of the library's stream-ordered workspaces (created on first use; keeps
// freed blocks cached until process exit).
cudaMemPool_t workspace_pool();

// Split-KV of the last partial wave of attention CTAs (OSP_SPLIT_KV=0 disables; read per launch).
int split_kv_enabled();

// Sets the dynamic shared-memory limit of kernel `func` to `bytes` on the current device, once per
// (device, kernel), from any host thread.  OSP_ERR_CUDA naming `name` on failure.
int ensure_smem_attr(const void* func, int bytes, const char* name);

// Debug builds only (kernels compiled with OSP_BOUNDS_CHECK=1): the kernels' index-check limits
// are divided by OSP_DEBUG_BOUNDS_DIV (default 1), so a test can make the checks fire without
// any out-of-range access (the checked access is skipped).  Read per launch.
unsigned bounds_check_divisor();

// Attention CTAs running several work items in turn (OSP_PERSIST, read per launch): 1 (default)
// for short KV ranges, 0 never, 2 always (where the launch allows it).
int persist_mode();

int rope3d_launch(const void* q, const void* k, void* q_out, void* k_out, const osp_shape& s,
                  const osp_rope& rope, cudaStream_t stream);
int skiparse_gather_launch(const void* const src[3], void* const dst[3], int n_tensors, const osp_shape& s,
                           int k, int mode, const osp_rope* rope, cudaStream_t stream);
int skiparse_scatter_launch(const void* o_perm, void* o, const osp_shape& s, int k, int mode,
                            cudaStream_t stream);
int index_map_launch(int n_video, int k, int mode, int32_t* out, cudaStream_t stream);

// Attention over `G` token sets per sample (G = 1: dense over all N tokens; G = k: Skiparse).
//   layout: 0 dense, OSP_SKIP_SINGLE + 1, OSP_SKIP_GROUP + 1
int attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s, int layout,
                     int sparse_k, float scale, cudaStream_t stream);

// Cross-attention: queries are the T*H*W video tokens of q, keys/values the text_len tokens of
// k and v; o has q's shape.
int cross_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s, float scale,
                           cudaStream_t stream);

// Skiparse with a joined text prefix (text_len > 0, k > 1): video queries of set g attend to the
// text rows and set g; text queries attend to every row.  Two launches of the attention kernel.
// lse (training forward, may be null): the video queries' rows in set-slot order,
// [B*G][heads][ceil(n/128)*128] (n = T*H*W / G), followed by the text queries' rows,
// [B][heads][ceil(text_len/128)*128].
int skiparse_text_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s,
                                   int sparse_k, int mode, float scale, cudaStream_t stream, float* lse = nullptr);
// Backward of the above from its o and lse: a per-set pass over [set rows; text rows] samples
// (video queries) and a pass of the text queries over all tokens, summed in fp32.
int skiparse_text_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                  const float* lse, void* dq, void* dk, void* dv, const osp_shape& s, int sparse_k,
                                  int mode, float scale, cudaStream_t stream);

// Frame-causal attention (dense layout): token r attends to the text block and the frames up to its own.
int frame_causal_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s,
                                  float scale, cudaStream_t stream);

// Causal temporal attention for any T: Single Skip sets (k = H*W) with a token-causal mask.
int causal_temporal_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s,
                                     float scale, cudaStream_t stream);

// Temporal attention of 2D + 1D (T <= 64): sets of T tokens at stride H*W, optionally causal in t.
// T <= 64: one warp per (sample, position, head) set; lse (optional, training forward): the row
// log-sum-exp in the layout of the tile kernels' lse.
int temporal_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s, int causal,
                              float scale, cudaStream_t stream, float* lse = nullptr);

// Backward of temporal attention for T <= 64 (one warp per set): dq, dk, dv from q, k, v, o,
// dout and the training forward's lse ([B*H*W][heads][ceil(T/128)*128], log2 domain).
int temporal_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, const osp_shape& s, int causal,
                             float scale, cudaStream_t stream);

// TMA map over a BSHD tensor for the attention kernels' 128-row x 64-channel SW128 tiles, viewed
// per layout (0 dense, 1 Single Skip, 2 Group Skip); batch_rows = rows between samples (< 0: N).
int make_attn_tmap(CUtensorMap* tm, const void* ptr, const osp_shape& s, int N, int layout, int k,
                   long long batch_rows = -1);

// Training forward: attention as attention_launch (layout 0 dense, or Skiparse) that also writes
// the row log-sum-exp (log2 domain of the scaled scores) to lse, [B*G][heads][ceil(n/128)*128].
int attention_forward_lse_launch(const void* q, const void* k, const void* v, void* o, float* lse,
                                 const osp_shape& s, int layout, int sparse_k, float scale, cudaStream_t stream,
                                 bool frame_causal = false, int causal_block = 0);

// Backward pass of attention_forward_lse_launch: dq, dk, dv from q, k, v, o, dout and lse.
// q_limit >= 0 (dense layout): only the first q_limit rows of each sample are queries (their
// lse in rows of ceil(q_limit / 128) * 128); dq is written for those rows only, dk and dv carry
// their contributions.  dkdv_f32: dk and dv are fp32 arrays, written unrounded.
int attention_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, const osp_shape& s, int layout,
                              int sparse_k, float scale, cudaStream_t stream, bool frame_causal = false,
                              int causal_block = 0, int q_limit = -1, bool dkdv_f32 = false);

// Packed batch (block-diagonal attention): segment i owns q/o rows [q_bounds[i], q_bounds[i+1])
// and k/v rows [kv_bounds[i], kv_bounds[i+1]); host arrays of n_seg + 1 validated offsets.
// lse (optional, training forward of self-attention): [heads][packed_lse_rows], sample i's rows
// from the start of its 256-row blocks.
int packed_attention_launch(const void* q, const void* k, const void* v, void* o, const int32_t* q_bounds,
                            const int32_t* kv_bounds, int n_seg, int heads, int head_dim, float scale,
                            cudaStream_t stream, float* lse = nullptr);
// Rows of a packed batch's lse per head: sum over samples of ceil(len / 256) * 256.
int packed_lse_rows(const int32_t* bounds, int n_seg);
// Backward of packed self-attention (each sample's own attention) from the training forward's lse.
int packed_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                           const float* lse, void* dq, void* dk, void* dv, const int32_t* bounds, int n_seg,
                           int heads, int head_dim, float scale, cudaStream_t stream);

// 3D RoPE of a packed batch: sample i is text_len_i unrotated tokens then its own T_i x H_i x W_i grid.
int rope3d_packed_launch(const void* q, const void* k, void* q_out, void* k_out, const osp_sample_grid* samples,
                         int n_samples, int heads, int head_dim, const osp_rope& rope, cudaStream_t stream);

}  // namespace osp
