// 3D RoPE and the Skiparse k-fold permutation (gather / scatter), fused into one streaming
// kernel, plus the Skiparse index-map kernel.
//
// Sources: "CogVideoX: Text-to-Video Diffusion Models with an Expert Transformer" section 2.2
// "3D-RoPE" (one 1D RoPE per axis on its own channel share, concatenated) and section 3.1
// (raw integer positions, extrapolated); RoFormer for the pairwise rotation with frequencies
// theta^(-2j/d_axis); "Open-Sora Plan" section 2.2.2 for the Skiparse sets and the k-fold batch.
//
// Work decomposition: a CTA owns a tile of whole token rows (heads * head_dim contiguous bf16,
// 1-8 KB each), so every load and store is a coalesced 16-byte vector.  Per tile it first
// computes each row's source/destination row and (t, h, w) position, then one cos/sin pair
// per (row, channel pair) into shared memory, then streams the rows of every tensor.

#include <type_traits>

#include "osp_internal.h"

namespace osp {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxPairs = 128;   // head_dim <= 256

// identity: RoPE in natural order; gather / scatter: the Skiparse k-fold permutation;
// packed: RoPE of a packed batch (identity order, every sample with its own grid)
enum MapKind { kMapIdentity = 0, kMapGather = 1, kMapScatter = 2, kMapPacked = 3 };

struct PermuteParams {
  const uint4* src[3];
  uint4* dst[3];
  int n_tensors;
  unsigned rope_mask;      // bit i: rotate tensor i
  long long rows;          // rows to process (per tensor)
  int vpr;                 // 16-byte vectors per row = heads * head_dim / 8
  int head_dim;
  int N;                   // tokens per sample in the natural-order tensor
  int text_len;
  int H, W;
  int sparse_k, mode;      // Skiparse (gather / scatter only)
  int d_t, d_h, d_w;
  double log2_theta;
  int rows_per_tile;
  long long n_tiles;
  // 16-byte vectors in each source / destination tensor and the status word, for the debug
  // build's index checks
  unsigned long long src_vecs, dst_vecs;
  unsigned* status;
};

// Samples of a packed batch: sample i owns rows [start[i], start[i+1]), its first text[i] rows
// are text, the rest an H[i] x W[i]-wide grid.  A kernel parameter (copied at launch).
struct PackTable {
  int n;
  int start[kMaxSegments + 1];
  int text[kMaxSegments];
  int H[kMaxSegments];
  int W[kMaxSegments];
};
struct NoPackTable {};
template <int MAP>
using PackParam = typename std::conditional<MAP == kMapPacked, PackTable, NoPackTable>::type;

// Token index of slot s of set g (Open-Sora Plan section 2.2.2; reading in osp.h).
__device__ __forceinline__ int skiparse_token(int g, int s, int k, int mode) {
  if (mode == OSP_SKIP_SINGLE) return s * k + g;
  const int o = s / k, r = s - o * k;
  return (o * k + g) * k + r;
}

// fp64 -> bf16 with a single round-to-nearest-even: first fp64 -> fp32 rounded to odd (truncate,
// then set the last bit if anything was dropped; Boldo & Melquiond, "When double rounding is odd"),
// then fp32 -> bf16 RNE.  fp32 keeps 16 more significand bits than bf16, so the second rounding
// sees the exact tie/no-tie information.
__device__ __forceinline__ uint32_t bf16_rn_from_f64(double x) {
  const float t = __double2float_rz(x);
  uint32_t b = __float_as_uint(t);
  if ((double)t != x) b |= 1u;
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(b)));
}

template <int MAP>
__global__ void __launch_bounds__(kThreads) permute_rope_kernel(const PermuteParams p,
                                                                const __grid_constant__ PackParam<MAP> tab) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* omega = reinterpret_cast<double*>(smem_raw);                       // [head_dim/2]
  long long* src_row = reinterpret_cast<long long*>(omega + kMaxPairs);      // [rows_per_tile]
  long long* dst_row = src_row + p.rows_per_tile;                            // [rows_per_tile]
  int* vid = reinterpret_cast<int*>(dst_row + p.rows_per_tile);              // video index or -1
  int4* tpos = reinterpret_cast<int4*>(vid + ((p.rows_per_tile + 3) & ~3));  // (t, h, w) per row
  double2* cs = reinterpret_cast<double2*>(tpos + p.rows_per_tile);          // [tile][pairs]
  uint16_t* colpair = reinterpret_cast<uint16_t*>(cs + p.rows_per_tile * (p.head_dim >> 1));  // [vpr]

  const int npairs = p.head_dim >> 1;
  // Frequencies of every channel pair: pair j of a chunk of size d_a -> theta^(-2j/d_a).
  for (int i = threadIdx.x; i < npairs; i += kThreads) {
    const int c = 2 * i;
    int j, da;
    if (c < p.d_t) { j = i; da = p.d_t; }
    else if (c < p.d_t + p.d_h) { j = i - p.d_t / 2; da = p.d_h; }
    else { j = i - (p.d_t + p.d_h) / 2; da = p.d_w; }
    omega[i] = exp2(-(2.0 * j / da) * p.log2_theta);
  }
  // first channel pair of every 16-byte column of a token row (8 channels = 4 pairs per column)
  for (int c = threadIdx.x; c < p.vpr; c += kThreads) colpair[c] = (uint16_t)((c % (p.head_dim >> 3)) * 4);
  const int per_set = (MAP == kMapIdentity) ? 0 : p.N / p.sparse_k;

  for (long long tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
    __syncthreads();  // previous tile's table fully consumed (and omega ready on the first pass)
    const long long row0 = tile * p.rows_per_tile;
    const int nrows = (int)min((long long)p.rows_per_tile, p.rows - row0);
    for (int i = threadIdx.x; i < nrows; i += kThreads) {
      const long long r = row0 + i;
      long long s_row, d_row;
      int token, text_len = p.text_len, H = p.H, W = p.W;
      if constexpr (MAP == kMapIdentity) {
        s_row = d_row = r;
        token = (int)(r % p.N);
      } else if constexpr (MAP == kMapPacked) {
        // sample of row r: the largest s with start[s] <= r (starts strictly increase)
        int lo = 0, hi = tab.n;
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (tab.start[mid] <= r) lo = mid;
          else hi = mid;
        }
        s_row = d_row = r;
        token = (int)(r - tab.start[lo]);
        text_len = tab.text[lo];
        H = tab.H[lo];
        W = tab.W[lo];
      } else {
        const long long bk = r / per_set;           // b*k + g
        const int s = (int)(r - bk * per_set);
        const int g = (int)(bk % p.sparse_k);
        const long long b = bk / p.sparse_k;
        token = skiparse_token(g, s, p.sparse_k, p.mode);
        if (MAP == kMapGather) { s_row = b * p.N + token; d_row = r; }
        else { s_row = r; d_row = b * p.N + token; }
      }
      src_row[i] = s_row;
      dst_row[i] = d_row;
      const int v = token - text_len;  // < 0 for text tokens
      vid[i] = v;
      if (v >= 0) tpos[i] = make_int4(v / (H * W), (v / W) % H, v % W, 0);
    }
    __syncthreads();
    if (p.rope_mask) {
      for (int idx = threadIdx.x; idx < nrows * npairs; idx += kThreads) {
        const int i = idx / npairs, pr = idx - i * npairs;
        const int v = vid[i];
        double2 c_s = make_double2(1.0, 0.0);
        if (v >= 0) {
          const int c = 2 * pr;
          const int4 tp = tpos[i];
          const int pos = c < p.d_t ? tp.x : (c < p.d_t + p.d_h ? tp.y : tp.z);
          double sn, cn;
          sincos((double)pos * omega[pr], &sn, &cn);
          c_s = make_double2(cn, sn);
        }
        cs[idx] = c_s;
      }
      __syncthreads();
    }
    // Flattened (row, 16-byte column) walk over the tile: thread i starts at vector i and
    // advances by kThreads vectors; (row, col) is stepped incrementally (no division per vector).
    const int drow = kThreads / p.vpr, dcol = kThreads - drow * p.vpr;
    const int total = nrows * p.vpr;
    for (int t = 0; t < p.n_tensors; ++t) {
      const uint4* __restrict__ src = p.src[t];
      uint4* dst = p.dst[t];
      const bool rot = (p.rope_mask >> t) & 1u;
      const bool inplace = (const void*)src == (const void*)dst;
      int row = threadIdx.x / p.vpr, col = threadIdx.x - (threadIdx.x / p.vpr) * p.vpr;
      for (int base = threadIdx.x; base < total; base += 4 * kThreads) {
        uint4 val[4];
        int rowi[4], coli[4];
        bool live[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // 4 independent 16-byte loads in flight per thread
          rowi[u] = row;
          coli[u] = col;
          live[u] = base + u * kThreads < total && !(inplace && vid[row] < 0);  // text row in place: skip
          live[u] = live[u] && index_ok(src_row[row] * p.vpr + col, p.src_vecs, p.status) &&
                    index_ok(dst_row[row] * p.vpr + col, p.dst_vecs, p.status);
          if (live[u]) val[u] = src[src_row[row] * p.vpr + col];
          col += dcol;
          row += drow;
          if (col >= p.vpr) { col -= p.vpr; ++row; }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (!live[u]) continue;
          if (rot && vid[rowi[u]] >= 0) {
            const double2* tab = cs + rowi[u] * npairs + colpair[coli[u]];
            uint32_t w[4] = {val[u].x, val[u].y, val[u].z, val[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              // bf16 -> fp64 is exact; the rotation runs in fp64 and is rounded once to bf16
              const double x = (double)__uint_as_float(w[e] << 16);
              const double y = (double)__uint_as_float(w[e] & 0xFFFF0000u);
              const double2 c_s = tab[e];
              const double xr = fma(x, c_s.x, -y * c_s.y);
              const double yr = fma(x, c_s.y, y * c_s.x);
              w[e] = bf16_rn_from_f64(xr) | (bf16_rn_from_f64(yr) << 16);
            }
            val[u] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          dst[dst_row[rowi[u]] * p.vpr + coli[u]] = val[u];
        }
      }
    }
  }
}

__global__ void index_map_kernel(int n_video, int k, int mode, int* out) {
  const int per_set = n_video / k;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_video; i += gridDim.x * blockDim.x) {
    const int g = i / per_set, s = i - g * per_set;
    out[i] = skiparse_token(g, s, k, mode);
  }
}

int launch_permute(int map, PermuteParams& p, cudaStream_t stream, const PackTable* tab = nullptr) {
  // every tensor of a call has the natural-order row count on one side and `rows` on the other
  const unsigned long long nat = (unsigned long long)p.rows * p.vpr;
  p.src_vecs = p.dst_vecs = nat / bounds_check_divisor();
  p.status = device_status_word();
  if (!p.status) return OSP_ERR_CUDA;
  const int npairs = p.head_dim / 2;
  // ~4096 vectors (64 KB of one tensor) per tile, at most 64 rows, and the cos/sin table within
  // 40 KB of shared memory
  const int table_rows = (40 * 1024) / (npairs * (int)sizeof(double2));
  p.rows_per_tile = (int)std::max(1, std::min(std::min(64, table_rows), (4096 + p.vpr - 1) / p.vpr));
  p.n_tiles = (p.rows + p.rows_per_tile - 1) / p.rows_per_tile;
  const size_t smem = kMaxPairs * sizeof(double) + 2 * p.rows_per_tile * sizeof(long long) +
                      ((p.rows_per_tile + 3) & ~3) * sizeof(int) + p.rows_per_tile * sizeof(int4) +
                      (size_t)p.rows_per_tile * npairs * sizeof(double2) + (size_t)p.vpr * sizeof(uint16_t);
  const int sms = device_sm_count();
  const long long grid = std::min<long long>(p.n_tiles, (long long)sms * 8);
  if (grid <= 0) return OSP_OK;
  switch (map) {
    case kMapIdentity:
      permute_rope_kernel<kMapIdentity><<<(unsigned)grid, kThreads, smem, stream>>>(p, NoPackTable{});
      break;
    case kMapGather:
      permute_rope_kernel<kMapGather><<<(unsigned)grid, kThreads, smem, stream>>>(p, NoPackTable{});
      break;
    case kMapPacked:
      permute_rope_kernel<kMapPacked><<<(unsigned)grid, kThreads, smem, stream>>>(p, *tab);
      break;
    default:
      permute_rope_kernel<kMapScatter><<<(unsigned)grid, kThreads, smem, stream>>>(p, NoPackTable{});
      break;
  }
  return check_launch("permute_rope_kernel");
}

void fill_rope(PermuteParams& p, const osp_rope* rope) {
  if (rope) {
    p.d_t = rope->d_t;
    p.d_h = rope->d_h;
    p.d_w = rope->d_w;
    p.log2_theta = std::log2(rope->theta);
  } else {
    p.d_t = p.head_dim;
    p.d_h = p.d_w = 0;
    p.log2_theta = 0.0;
  }
}

}  // namespace

int rope3d_launch(const void* q, const void* k, void* q_out, void* k_out, const osp_shape& s,
                  const osp_rope& rope, cudaStream_t stream) {
  PermuteParams p{};
  p.src[0] = static_cast<const uint4*>(q);
  p.dst[0] = static_cast<uint4*>(q_out);
  p.src[1] = static_cast<const uint4*>(k);
  p.dst[1] = static_cast<uint4*>(k_out);
  p.n_tensors = 2;
  p.rope_mask = 3u;
  p.head_dim = s.head_dim;
  p.N = s.text_len + s.T * s.H * s.W;
  p.rows = (long long)s.B * p.N;
  p.vpr = s.heads * s.head_dim / 8;
  p.text_len = s.text_len;
  p.H = s.H;
  p.W = s.W;
  p.sparse_k = 1;
  p.mode = 0;
  fill_rope(p, &rope);
  return launch_permute(kMapIdentity, p, stream);
}

int rope3d_packed_launch(const void* q, const void* k, void* q_out, void* k_out, const osp_sample_grid* samples,
                         int n_samples, int heads, int head_dim, const osp_rope& rope, cudaStream_t stream) {
  PackTable tab{};
  tab.n = n_samples;
  long long rows = 0;
  for (int i = 0; i < n_samples; ++i) {
    tab.start[i] = (int)rows;
    tab.text[i] = samples[i].text_len;
    tab.H[i] = samples[i].H;
    tab.W[i] = samples[i].W;
    rows += (long long)samples[i].text_len + (long long)samples[i].T * samples[i].H * samples[i].W;
  }
  tab.start[n_samples] = (int)rows;
  PermuteParams p{};
  p.src[0] = static_cast<const uint4*>(q);
  p.dst[0] = static_cast<uint4*>(q_out);
  p.src[1] = static_cast<const uint4*>(k);
  p.dst[1] = static_cast<uint4*>(k_out);
  p.n_tensors = 2;
  p.rope_mask = 3u;
  p.head_dim = head_dim;
  p.N = (int)rows;
  p.rows = rows;
  p.vpr = heads * head_dim / 8;
  p.H = p.W = 1;
  p.sparse_k = 1;
  fill_rope(p, &rope);
  return launch_permute(kMapPacked, p, stream, &tab);
}

int skiparse_gather_launch(const void* const src[3], void* const dst[3], int n_tensors, const osp_shape& s,
                           int k, int mode, const osp_rope* rope, cudaStream_t stream) {
  PermuteParams p{};
  for (int i = 0; i < n_tensors; ++i) {
    p.src[i] = static_cast<const uint4*>(src[i]);
    p.dst[i] = static_cast<uint4*>(dst[i]);
  }
  p.n_tensors = n_tensors;
  p.rope_mask = rope ? (n_tensors >= 2 ? 3u : 1u) : 0u;
  p.head_dim = s.head_dim;
  p.N = s.T * s.H * s.W;
  p.rows = (long long)s.B * p.N;
  p.vpr = s.heads * s.head_dim / 8;
  p.text_len = 0;
  p.H = s.H;
  p.W = s.W;
  p.sparse_k = k;
  p.mode = mode;
  fill_rope(p, rope);
  return launch_permute(kMapGather, p, stream);
}

int skiparse_scatter_launch(const void* o_perm, void* o, const osp_shape& s, int k, int mode,
                            cudaStream_t stream) {
  PermuteParams p{};
  p.src[0] = static_cast<const uint4*>(o_perm);
  p.dst[0] = static_cast<uint4*>(o);
  p.n_tensors = 1;
  p.rope_mask = 0u;
  p.head_dim = s.head_dim;
  p.N = s.T * s.H * s.W;
  p.rows = (long long)s.B * p.N;
  p.vpr = s.heads * s.head_dim / 8;
  p.text_len = 0;
  p.H = s.H;
  p.W = s.W;
  p.sparse_k = k;
  p.mode = mode;
  fill_rope(p, nullptr);
  return launch_permute(kMapScatter, p, stream);
}

int index_map_launch(int n_video, int k, int mode, int32_t* out, cudaStream_t stream) {
  const int threads = 256;
  const int blocks = std::max(1, std::min((n_video + threads - 1) / threads, device_sm_count() * 4));
  index_map_kernel<<<blocks, threads, 0, stream>>>(n_video, k, mode, out);
  return check_launch("index_map_kernel");
}

}  // namespace osp
