// Host side of the attention forward (tcgen05 kernel in attn_fwd_kernel.cuh): TMA tensor maps,
// the split of the work into items (split-KV tail, items in turn), workspace, launches, and the
// entry points of dense, Skiparse, cross, frame-causal, joined-text and packed attention.

#include <cuda.h>

#include <mutex>
#include <type_traits>

#include "attn_fwd_kernel.cuh"

namespace osp {
namespace {

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// Tensor map over a BSHD [B][N][heads][D] bf16 tensor, viewed per `layout`:
//   dense:  (heads*D, N, B)                    box (64, 128, 1)
//   single: (heads*D, k, N/k, B)               box (64, 1, 128, 1)   token = s*k + g
//   group:  (heads*D, k, k, N/(k*k), B)         box (64, k, 1, 128/k, 1)  token = (o*k + g)*k + r
// The channel axis merges heads and head_dim; a box starts at channel h*D + 64c.
// batch_rows: rows between samples (default N); a view of part of each sample (the text rows,
// or the video rows from an offset pointer) keeps the full sample stride.
int make_tmap(CUtensorMap* tm, const void* ptr, const osp_shape& s, int N, int layout, int k,
              long long batch_rows = -1, int box_ch = 64,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return set_error(OSP_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t HD = (cuuint64_t)s.heads * s.head_dim;
  const cuuint64_t row = HD * 2;  // bytes per token
  const cuuint64_t bstride = row * (cuuint64_t)(batch_rows < 0 ? N : batch_rows);
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5], estr[5] = {1, 1, 1, 1, 1};
  cuuint32_t rank;
  if (layout == 0) {
    rank = 3;
    dims[0] = HD; dims[1] = (cuuint64_t)N; dims[2] = (cuuint64_t)s.B;
    strides[0] = row; strides[1] = bstride;
    box[0] = (cuuint32_t)box_ch; box[1] = kBM; box[2] = 1;
  } else if (layout == 1) {
    rank = 4;
    dims[0] = HD; dims[1] = (cuuint64_t)k; dims[2] = (cuuint64_t)(N / k); dims[3] = (cuuint64_t)s.B;
    strides[0] = row; strides[1] = row * k; strides[2] = bstride;
    box[0] = (cuuint32_t)box_ch; box[1] = 1; box[2] = kBM; box[3] = 1;
  } else {
    rank = 5;
    dims[0] = HD; dims[1] = (cuuint64_t)k; dims[2] = (cuuint64_t)k; dims[3] = (cuuint64_t)(N / (k * k));
    dims[4] = (cuuint64_t)s.B;
    strides[0] = row; strides[1] = row * k; strides[2] = row * k * k; strides[3] = bstride;
    box[0] = (cuuint32_t)box_ch; box[1] = (cuuint32_t)k; box[2] = 1; box[3] = (cuuint32_t)(kBM / k); box[4] = 1;
  }
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(OSP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return OSP_OK;
}

// Output maps of the TMA-store epilogue: the same view of o as make_tmap gives of q, plus at
// d = 96 a 32-channel box (64-byte swizzle) for each head's channels 64 .. 95.  Used at d >= 96,
// where a thread's row is 192-256 bytes of strided stores; at d = 64 (softmax-bound, 128-byte
// rows) the per-row stores measured faster (CogVideoX-2B grid: dense -1.5 %, spatial -8 % and
// cross-attention -5 % through the staging tile).
int make_out_maps(OutMaps* om, const void* o, const osp_shape& s, int N, int layout, int k,
                  long long batch_rows = -1) {
  *om = OutMaps{};
  if (s.head_dim < 96) return OSP_OK;
  int rc = make_tmap(&om->o, o, s, N, layout, k, batch_rows);
  if (rc == OSP_OK && s.head_dim == 96)
    rc = make_tmap(&om->tail, o, s, N, layout, k, batch_rows, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  om->use = rc == OSP_OK ? 1 : 0;
  return rc;
}

template <int D, int kMode, bool kLoop = false>
int launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
             const SegParam<kMode>& seg, const OutMaps& om, dim3 grid, cudaStream_t stream) {
  constexpr int smem = Cfg<D>::kSmemBytes;
  // The warpgroup register split only adds up if the kernel is launched with exactly
  // kRegsLaunch registers per thread; otherwise setmaxnreg.inc could never be satisfied.
  static const int regs = [] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, kMode, kLoop>) == cudaSuccess ? fa.numRegs : -1;
  }();
  if (regs < 0) return set_error(OSP_ERR_CUDA, "cudaFuncGetAttributes(attn_fwd_kernel<%d>) failed", D);
  if ((uint32_t)regs != kRegsLaunch)
    return set_error(OSP_ERR_CUDA, "attn_fwd_kernel<%d> compiled to %d registers per thread, expected %u", D, regs,
                     kRegsLaunch);
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(attn_fwd_kernel<D, kMode, kLoop>), smem, "attn_fwd_kernel");
  if (rc) return rc;
  attn_fwd_kernel<D, kMode, kLoop><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p, seg, om);
  return check_launch("attn_fwd_kernel");
}

}  // namespace

int make_attn_tmap(CUtensorMap* tm, const void* ptr, const osp_shape& s, int N, int layout, int k,
                   long long batch_rows) {
  return make_tmap(tm, ptr, s, N, layout, k, batch_rows);
}

namespace {

// Attention launch with an explicit status word (the kernel's only global scratch).
// N_kv: tokens per sample of k and v; < 0 means the same sequence as q (self-attention).
// Runs the attention kernel over `units` work units of n_kv_tiles KV tiles each: the split of
// the last partial wave over KV ranges (when allowed), its workspace and the combine kernel.
template <int kMode>
int run_units(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, AttnParams& p,
              const SegParam<kMode>& extra, const OutMaps& om, long long units, int n_kv_tiles, bool allow_split,
              int head_dim, cudaStream_t stream) {
  if (units > (1LL << 30)) return set_error(OSP_ERR_UNSUPPORTED, "%lld attention work units is too many", units);
  p.n_full = (int)units;
  p.n_split = 1;
  // Split-KV for the last partial wave (one CTA per SM): its R units are split into KV ranges so
  // that about one wave of CTAs runs them.  Needs a workspace, so only where allocation is allowed.
  const int sms = device_sm_count();
  const int rem = (int)(units % sms);
  if (allow_split && split_kv_enabled() && rem > 0) {
    const int ns = std::min(std::min(sms / rem, n_kv_tiles / 2), 8);
    if (ns >= 2) {
      p.n_full = (int)(units - rem);
      p.n_split = ns;
    }
  }
  void* ws = nullptr;
  if (p.n_split > 1) {
    const size_t rows = (size_t)(units - p.n_full) * p.n_split * 2 * kBM;
    const size_t bytes = rows * (size_t)head_dim * sizeof(float) + rows * sizeof(float2);
    cudaMemPool_t pool = workspace_pool();
    if (!pool || cudaMallocFromPoolAsync(&ws, bytes, pool, stream) != cudaSuccess)
      return set_error(OSP_ERR_CUDA, "stream-ordered workspace allocation (%zu bytes) failed", bytes);
    p.ws_o = static_cast<float*>(ws);
    p.ws_ml = reinterpret_cast<float2*>(p.ws_o + rows * (size_t)head_dim);
    p.ws_rows = rows;
  }
  // debug builds: the index checks' limits (a test divisor shrinks them to exercise the checks)
  const unsigned long long div = (unsigned long long)bounds_check_divisor();
  p.o_elems /= div;
  p.lse_elems /= div;
  p.ws_rows /= div;
  const long long ctas = p.n_full + (units - p.n_full) * p.n_split;
  p.n_items = (int)ctas;
  // Short KV ranges: one CTA per SM runs items in turn, so an item's Q load and first QK^T
  // overlap the previous item's softmax and epilogue (a fixed cost per item that a few KV tiles
  // do not amortise).  Not with a split tail (its items differ in kind) or packed batches.
  long long grid_ctas = ctas;
  const int persist = persist_mode();
  if (kMode != kModePacked && p.n_split == 1 &&
      ((persist == 1 && n_kv_tiles <= kPersistMaxTiles && ctas >= 2LL * sms) || persist == 2))
    grid_ctas = std::min<long long>(ctas, sms);
  const bool loop = grid_ctas < ctas;
  dim3 grid((unsigned)grid_ctas);
  int rc;
  switch (head_dim) {
    case 64:
      rc = loop ? launch_d<64, kMode, true>(tq, tk, tv, p, extra, om, grid, stream)
                : launch_d<64, kMode, false>(tq, tk, tv, p, extra, om, grid, stream);
      break;
    case 96:
      rc = loop ? launch_d<96, kMode, true>(tq, tk, tv, p, extra, om, grid, stream)
                : launch_d<96, kMode, false>(tq, tk, tv, p, extra, om, grid, stream);
      break;
    case 128:
      rc = loop ? launch_d<128, kMode, true>(tq, tk, tv, p, extra, om, grid, stream)
                : launch_d<128, kMode, false>(tq, tk, tv, p, extra, om, grid, stream);
      break;
    default: rc = set_error(OSP_ERR_UNSUPPORTED, "head_dim %d not in {64, 96, 128}", head_dim);
  }
  if (rc == OSP_OK && p.n_split > 1) {
    const int su = (int)(units - p.n_full);
    const unsigned blocks = (unsigned)(((size_t)su * 2 * kBM + 7) / 8);
    switch (head_dim) {
      case 64: attn_combine_kernel<64><<<blocks, 256, 0, stream>>>(p, su); break;
      case 96: attn_combine_kernel<96><<<blocks, 256, 0, stream>>>(p, su); break;
      default: attn_combine_kernel<128><<<blocks, 256, 0, stream>>>(p, su); break;
    }
    rc = check_launch("attn_combine_kernel");
  }
  if (ws) cudaFreeAsync(ws, stream);
  return rc;
}

AttnParams base_params(const osp_shape& s, int layout, int sparse_k, float scale, void* o, unsigned* status) {
  AttnParams p{};
  p.heads = s.heads;
  p.G = (layout == 0) ? 1 : sparse_k;
  p.k = (layout == 0) ? 1 : sparse_k;
  p.layout = layout;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.status = status;
  p.timeout_ns = wait_timeout_ns();
  p.debug_withhold_q = debug_withhold_q();
  return p;
}

// frame_causal: the block-causal mask over a set's slots: s's text block, then blocks of
// causal_block slots (a frame, H*W, when 0).
int launch_with_status(const void* q, const void* k, const void* v, void* o, const osp_shape& s, int layout,
                       int sparse_k, float scale, cudaStream_t stream, unsigned* status, bool allow_split,
                       int N_kv = -1, bool frame_causal = false, float* lse = nullptr, int causal_block = 0) {
  const int N = (N_kv < 0) ? s.text_len + s.T * s.H * s.W : s.T * s.H * s.W;   // q / o tokens per sample
  if (N_kv < 0) N_kv = N;
  AttnParams p = base_params(s, layout, sparse_k, scale, o, status);
  const int G = p.G;
  const int n = N / G;
  p.n_q = n;
  p.n_kv = N_kv / G;
  p.N_q = N;
  // rows per causal block: a frame (H*W) by default; 1 makes the mask token-causal within a set
  p.frame_hw = frame_causal ? (causal_block > 0 ? causal_block : s.H * s.W) : 0;
  p.text_len = s.text_len;
  p.lse = lse;
  p.lse_stride = (n + kBM - 1) / kBM * kBM;
  p.o_elems = (unsigned long long)s.B * N * s.heads * s.head_dim;
  p.lse_elems = lse ? (unsigned long long)s.B * G * s.heads * p.lse_stride : 0;
  if (frame_causal) allow_split = false;   // a KV range could hold no visible key for some rows
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap(&tq, q, s, N, layout, p.k)) != OSP_OK) return rc;
  if ((rc = make_tmap(&tk, k, s, N_kv, layout, p.k)) != OSP_OK) return rc;
  if ((rc = make_tmap(&tv, v, s, N_kv, layout, p.k)) != OSP_OK) return rc;
  OutMaps om;
  if ((rc = make_out_maps(&om, o, s, N, layout, p.k)) != OSP_OK) return rc;
  const long long qblocks = (n + 2 * kBM - 1) / (2 * kBM);
  p.qblocks = (int)qblocks;
  const long long units = qblocks * s.heads * (long long)s.B * G;
  const int n_kv_tiles = (p.n_kv + kBN - 1) / kBN;
  if (frame_causal)
    return run_units<kModeFrameCausal>(tq, tk, tv, p, NoSegTable{}, om, units, n_kv_tiles, false, s.head_dim, stream);
  return run_units<kModePlain>(tq, tk, tv, p, NoSegTable{}, om, units, n_kv_tiles, allow_split, s.head_dim, stream);
}

}  // namespace

int attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s, int layout,
                     int sparse_k, float scale, cudaStream_t stream) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  return launch_with_status(q, k, v, o, s, layout, sparse_k, scale, stream, status, true);
}

int cross_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s, float scale,
                           cudaStream_t stream) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  return launch_with_status(q, k, v, o, s, 0, 1, scale, stream, status, true, s.text_len);
}

int skiparse_text_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s,
                                   int sparse_k, int mode, float scale, cudaStream_t stream, float* lse) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  const int L = s.text_len, Nv = s.T * s.H * s.W, N = L + Nv;
  const size_t row = (size_t)s.heads * s.head_dim * 2;
  const osp_shape sv{s.B, 0, s.T, s.H, s.W, s.heads, s.head_dim};   // the video part of each sample
  int rc;
  // 1) video queries: set g attends to the text rows, then to the set's own rows
  {
    const int layout = mode + 1;
    AttnParams p = base_params(sv, layout, sparse_k, scale, o, status);
    const int n = Nv / sparse_k;
    p.n_q = p.n_kv = n;
    p.N_q = N;
    p.text_len = L;
    p.q_row_base = L;
    p.o_elems = (unsigned long long)s.B * N * s.heads * s.head_dim;
    p.lse = lse;
    p.lse_stride = (n + kBM - 1) / kBM * kBM;
    p.lse_elems = lse ? (unsigned long long)s.B * sparse_k * s.heads * p.lse_stride : 0;
    CUtensorMap tq, tk, tv;
    TextMaps tm{};
    const char* qv = static_cast<const char*>(q) + L * row;
    const char* kv = static_cast<const char*>(k) + L * row;
    const char* vv = static_cast<const char*>(v) + L * row;
    if ((rc = make_tmap(&tq, qv, sv, Nv, layout, sparse_k, N)) != OSP_OK) return rc;
    if ((rc = make_tmap(&tk, kv, sv, Nv, layout, sparse_k, N)) != OSP_OK) return rc;
    if ((rc = make_tmap(&tv, vv, sv, Nv, layout, sparse_k, N)) != OSP_OK) return rc;
    if ((rc = make_tmap(&tm.k, k, s, L, 0, 1, N)) != OSP_OK) return rc;
    if ((rc = make_tmap(&tm.v, v, s, L, 0, 1, N)) != OSP_OK) return rc;
    OutMaps om;
    if ((rc = make_out_maps(&om, static_cast<char*>(o) + L * row, sv, Nv, layout, sparse_k, N)) != OSP_OK) return rc;
    const long long qblocks = (n + 2 * kBM - 1) / (2 * kBM);
    p.qblocks = (int)qblocks;
    const long long units = qblocks * s.heads * (long long)s.B * sparse_k;
    const int n_kv_tiles = (n + kBN - 1) / kBN + (L + kBN - 1) / kBN;
    rc = run_units<kModeSkipText>(tq, tk, tv, p, tm, om, units, n_kv_tiles, true, s.head_dim, stream);
    if (rc) return rc;
  }
  if (L == 0) return OSP_OK;
  // 2) text queries: every text token attends to all N tokens of its sample
  AttnParams p = base_params(s, 0, 1, scale, o, status);
  p.n_q = L;
  p.n_kv = N;
  p.N_q = N;
  p.o_elems = (unsigned long long)s.B * N * s.heads * s.head_dim;
  if (lse) {   // after the video rows' block
    const long long n_pad = (Nv / sparse_k + kBM - 1) / kBM * kBM;
    p.lse = lse + (size_t)s.B * sparse_k * s.heads * n_pad;
    p.lse_stride = (L + kBM - 1) / kBM * kBM;
    p.lse_elems = (unsigned long long)s.B * s.heads * p.lse_stride;
  }
  CUtensorMap tq, tk, tv;
  if ((rc = make_tmap(&tq, q, s, L, 0, 1, N)) != OSP_OK) return rc;
  if ((rc = make_tmap(&tk, k, s, N, 0, 1)) != OSP_OK) return rc;
  if ((rc = make_tmap(&tv, v, s, N, 0, 1)) != OSP_OK) return rc;
  OutMaps om;
  if ((rc = make_out_maps(&om, o, s, L, 0, 1, N)) != OSP_OK) return rc;
  const long long qblocks = (L + 2 * kBM - 1) / (2 * kBM);
  p.qblocks = (int)qblocks;
  const long long units = qblocks * s.heads * (long long)s.B;
  return run_units<kModePlain>(tq, tk, tv, p, NoSegTable{}, om, units, (N + kBN - 1) / kBN, true, s.head_dim,
                               stream);
}

int attention_forward_lse_launch(const void* q, const void* k, const void* v, void* o, float* lse,
                                 const osp_shape& s, int layout, int sparse_k, float scale, cudaStream_t stream,
                                 bool frame_causal, int causal_block) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  return launch_with_status(q, k, v, o, s, layout, sparse_k, scale, stream, status, true, -1, frame_causal, lse,
                            causal_block);
}

int frame_causal_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s,
                                  float scale, cudaStream_t stream) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  return launch_with_status(q, k, v, o, s, 0, 1, scale, stream, status, false, -1, true);
}

int causal_temporal_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s,
                                     float scale, cudaStream_t stream) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  // spatial position pos is Single Skip set pos with k = H*W (slot t = frame t); the frame-causal
  // mask with one-row blocks lets slot t see slots 0..t
  return launch_with_status(q, k, v, o, s, OSP_SKIP_SINGLE + 1, s.H * s.W, scale, stream, status, false, -1, true,
                            nullptr, 1);
}

int packed_attention_launch(const void* q, const void* k, const void* v, void* o, const int32_t* q_bounds,
                            const int32_t* kv_bounds, int n_seg, int heads, int head_dim, float scale,
                            cudaStream_t stream, float* lse) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  SegTable seg{};
  seg.n_seg = n_seg;
  long long blocks = 0;
  for (int i = 0; i <= n_seg; ++i) {
    seg.q[i] = q_bounds[i];
    seg.kv[i] = kv_bounds[i];
    seg.blk[i] = (int)blocks;
    if (i < n_seg) blocks += (q_bounds[i + 1] - q_bounds[i] + 2 * kBM - 1) / (2 * kBM);
  }
  const long long units = blocks * heads;
  if (units == 0) return OSP_OK;   // no query rows at all
  if (units > (1LL << 30)) return set_error(OSP_ERR_UNSUPPORTED, "%lld attention work units is too many", units);
  const int n_q_total = q_bounds[n_seg], n_kv_total = kv_bounds[n_seg];
  AttnParams p{};
  p.N_q = n_q_total;
  p.heads = heads;
  p.G = 1;
  p.k = 1;
  p.layout = 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.status = status;
  p.timeout_ns = wait_timeout_ns();
  p.debug_withhold_q = debug_withhold_q();
  p.qblocks = 1;
  p.n_full = (int)units;
  p.n_split = 1;
  p.n_items = (int)units;
  p.o_elems = (unsigned long long)n_q_total * heads * head_dim / (unsigned long long)bounds_check_divisor();
  // training forward: lse [heads][blocks * 256], sample i's rows from blk[i] * 256
  p.lse = lse;
  p.lse_stride = (int)(blocks * 2 * kBM);
  p.lse_elems = lse ? (unsigned long long)heads * p.lse_stride / (unsigned long long)bounds_check_divisor() : 0;
  // the packed tensors are one sample of n_q_total (q, o) / n_kv_total (k, v) rows
  const osp_shape sh{1, 0, 1, 1, 1, heads, head_dim};
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap(&tq, q, sh, n_q_total, 0, 1)) != OSP_OK) return rc;
  if ((rc = make_tmap(&tk, k, sh, n_kv_total, 0, 1)) != OSP_OK) return rc;
  if ((rc = make_tmap(&tv, v, sh, n_kv_total, 0, 1)) != OSP_OK) return rc;
  const dim3 grid((unsigned)units);
  switch (head_dim) {
    case 64: return launch_d<64, kModePacked>(tq, tk, tv, p, seg, OutMaps{}, grid, stream);
    case 96: return launch_d<96, kModePacked>(tq, tk, tv, p, seg, OutMaps{}, grid, stream);
    case 128: return launch_d<128, kModePacked>(tq, tk, tv, p, seg, OutMaps{}, grid, stream);
    default: return set_error(OSP_ERR_UNSUPPORTED, "head_dim %d not in {64, 96, 128}", head_dim);
  }
}

// ------------------------------------------------------------------------------------------
// Allocation-free dense attention (osp_attn_full_noalloc)
// ------------------------------------------------------------------------------------------
// The attention kernel's only global scratch is its status word, into which its bounded waits
// report a timeout.  osp_attn_full keeps that word in memory the library obtains with cudaMalloc
// on first use.  This variant keeps it in the file-scope device array below instead, so a call
// allocates nothing.  Every GPU that loads the library holds the array until the process exits.
// In host code `g_noalloc_scratch` names a host-side shadow, not device memory: the kernel gets
// the device address obtained with cudaGetSymbolAddress, once per device.
constexpr size_t kNoAllocScratchBytes = 256;   // maximum scratch a call may use
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Scratch bytes the kernel needs for a problem: its status word, whatever the shape.
size_t noalloc_scratch_bytes(const osp_shape&) { return sizeof(unsigned); }

// Device address of g_noalloc_scratch on the current device; looked up on the first call per
// device (with that device current) and cached.  The lookup is refused while `stream` is being
// captured, so that a first call inside a capture fails with a message saying so.
int noalloc_scratch_address(void** out, cudaStream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
    return set_error(OSP_ERR_CUDA, "osp_attn_full_noalloc: no usable current CUDA device");
  if (dev >= kNoAllocMaxDevices)
    return set_error(OSP_ERR_UNSUPPORTED, "osp_attn_full_noalloc: device ordinal %d is beyond its limit of %d devices",
                     dev, kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone)
      return set_error(OSP_ERR_CUDA, "osp_attn_full_noalloc: the first call on device %d must come before any "
                       "stream capture (it looks up the static scratch's address)", dev);
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return set_error(OSP_ERR_CUDA, "osp_attn_full_noalloc: cudaGetSymbolAddress failed: %s",
                       cudaGetErrorString(e));
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return OSP_OK;
}

}  // namespace

unsigned* noalloc_status_word_if_present() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  return static_cast<unsigned*>(g_noalloc_addr[dev]);
}

}  // namespace osp

extern "C" int osp_attn_full_noalloc(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                                     float softmax_scale, void* stream) {
  using namespace osp;
  set_error(OSP_OK, "");
  if (!shape) return set_error(OSP_ERR_INVALID_ARG, "shape is NULL");
  const osp_shape& s = *shape;
  if (s.B < 1 || s.text_len < 0 || s.T < 1 || s.H < 1 || s.W < 1 || s.heads < 1)
    return set_error(OSP_ERR_INVALID_ARG, "bad shape: B=%d text_len=%d T=%d H=%d W=%d heads=%d", s.B, s.text_len,
                     s.T, s.H, s.W, s.heads);
  if (s.head_dim != 64 && s.head_dim != 96 && s.head_dim != 128)
    return set_error(OSP_ERR_UNSUPPORTED, "attention head_dim %d not in {64, 96, 128}", s.head_dim);
  if ((long long)s.text_len + (long long)s.T * s.H * s.W > (1LL << 30))
    return set_error(OSP_ERR_UNSUPPORTED, "sequence length too large");
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  const uintptr_t a = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                      reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
  if (a & 15u) return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t need = noalloc_scratch_bytes(s);
  if (need > kNoAllocScratchBytes)
    return set_error(OSP_ERR_UNSUPPORTED, "osp_attn_full_noalloc needs %zu bytes of scratch, more than its %zu-byte "
                     "static array", need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = noalloc_scratch_address(&scratch, st);
  if (rc) return rc;
  // the array keeps the previous call's contents: the status word must start at zero
  if (cudaMemsetAsync(scratch, 0, need, st) != cudaSuccess)
    return set_error(OSP_ERR_CUDA, "osp_attn_full_noalloc: clearing the scratch word failed");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)s.head_dim);
  return launch_with_status(q, k, v, o, s, 0, 1, softmax_scale, st, static_cast<unsigned*>(scratch), false);
}
