// 3D RoPE and the Skiparse k-fold permutation (gather / scatter), fused into one streaming
// kernel, plus the Skiparse index-map kernel.
//
// Sources: "CogVideoX: Text-to-Video Diffusion Models with an Expert Transformer" section 2.2
// "3D-RoPE" (one 1D RoPE per axis on its own channel share, concatenated) and section 3.1
// (raw integer positions, extrapolated); RoFormer for the pairwise rotation with frequencies
// theta^(-2j/d_axis); "Open-Sora Plan" section 2.2.2 for the Skiparse sets and the k-fold batch.
//
// Work decomposition: a thread owns one 16-byte column (4 channel pairs) of one head-sized slice
// of a token row and applies it to every head of every tensor: it maps the row to its source and
// destination rows and (t, h, w) position, computes the rotation of its 4 pairs once (fp64
// sincos, kept in registers), and streams the column of each head.  Consecutive threads take
// consecutive columns, so every warp access is a run of whole 16 * (head_dim / 8)-byte segments.
// The rotation itself runs in fp32 with a certified error bound; the rare elements whose bf16
// rounding the bound cannot decide are redone in fp64, so every output is the correctly
// rounded rotation.

#include <type_traits>

#include "osp_internal.h"

namespace osp {

namespace {

constexpr int kThreads = 256;
// Heads per step of the one-, two- and three-tensor kernels: 12, 12 and 12 independent 16-byte
// loads in flight per thread (as many as fit the 128 registers of two CTAs per SM without spills;
// same-box A/B against 8, 8, 9: RoPE +5 % on the CogVideoX-2B and Open-Sora Plan grids, gather
// +4 %, scatter +3 %).
#ifndef OSP_ROPE_HS1
#define OSP_ROPE_HS1 12
#endif
#ifndef OSP_ROPE_HS2
#define OSP_ROPE_HS2 6
#endif
#ifndef OSP_ROPE_HS3
#define OSP_ROPE_HS3 4
#endif
constexpr int kMaxPairs = 128;   // head_dim <= 256
constexpr int kMaxTensors = 3;   // q, k, v

// identity: RoPE in natural order; gather / scatter: the Skiparse k-fold permutation;
// packed: RoPE of a packed batch (identity order, every sample with its own grid)
enum MapKind { kMapIdentity = 0, kMapGather = 1, kMapScatter = 2, kMapPacked = 3 };

struct PermuteParams {
  const uint4* src[kMaxTensors];
  uint4* dst[kMaxTensors];
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

// Rotation constants of one channel pair at one position, in registers: the fp64 cosine and sine
// split as c = c_hi + c_lo, s = s_hi + s_lo, where c_hi, s_hi keep 16 significant bits (so that
// their products with a bf16 value, 8 significant bits, are exact in fp32) and c_lo, s_lo are the
// fp32 roundings of the remainders (|c_lo| < 2^-15 |c|, rounding error < 2^-39 |c|).  Held as the
// fp32 pairs the packed arithmetic consumes: (c_hi, s_hi), (-s_hi, c_hi), (c_lo, s_lo), (-s_lo, c_lo).
struct RotRegs {
  uint64_t hi, nhi, lo, nlo;
};

__device__ __forceinline__ RotRegs rot_regs(double cn, double sn) {
  const float ch = __uint_as_float(__float_as_uint((float)cn) & 0xFFFFFF00u);
  const float sh = __uint_as_float(__float_as_uint((float)sn) & 0xFFFFFF00u);
  const float cl = (float)(cn - (double)ch), sl = (float)(sn - (double)sh);
  return RotRegs{f2_pack(ch, sh), f2_pack(-sh, ch), f2_pack(cl, sl), f2_pack(-sl, cl)};
}

// One rotated pair in fp64 from the split cosine and sine (exact to 2^-39 relative), rounded once
// to bf16: the arithmetic for the rare elements whose fp32 result is not certified.
__device__ __noinline__ uint32_t rope_pair_f64(uint32_t w, uint64_t hi, uint64_t lo) {
  float ch, sh, cl, sl;
  f2_unpack(hi, ch, sh);
  f2_unpack(lo, cl, sl);
  const double cn = (double)ch + (double)cl, sn = (double)sh + (double)sl;
  // bf16 -> fp64 is exact
  const double x = (double)__uint_as_float(w << 16);
  const double y = (double)__uint_as_float(w & 0xFFFF0000u);
  const double xr = fma(x, cn, -y * sn);
  const double yr = fma(x, sn, y * cn);
  return bf16_rn_from_f64(xr) | (bf16_rn_from_f64(yr) << 16);
}

// Whether rounding the fp32 value r to bf16 (nearest, ties to even) gives the same bf16 as
// rounding any value within e of r, given that the bf16 rounding boundary below |r| is out of
// reach (checked by the caller): the boundary just above |r| is its bf16 truncation plus half a
// bf16 step (bit pattern ...8000, in the same binade, so |r| - mid is exact in fp32).  Infinite
// and NaN results fail.
__device__ __forceinline__ bool bf16_rn_certain(float r, float e) {
  const float ar = fabsf(r);
  const float mid = __uint_as_float((__float_as_uint(ar) & 0xFFFF0000u) | 0x8000u);
  return fabsf(ar - mid) > e;
}

#ifndef OSP_ROPE_CERTIFY
#define OSP_ROPE_CERTIFY 0      // 1: check every result and redo uncertain pairs in fp64 (correctly rounded, slower)
#endif

// Rotation of one bf16 pair (x, y): xr = x c - y s, yr = x s + y c in packed fp32 pairs:
//   (r1x, r1y) = fma((x, x), (c_hi, s_hi), (y, y) * (-s_hi, c_hi))   products exact, one rounding
//   (lox, loy) = fma((x, x), (c_lo, s_lo), (y, y) * (-s_lo, c_lo))   the small remainder terms
//   (xr, yr)   = (r1x, r1y) + (lox, loy)
// Error bound per result r: 2^-24 |r1| + 2^-24 |r| + 2^-38 (|x| + |y|) (remainder rounding and the
// split's c_lo, s_lo) <= e = 2^-23 |r| + 2^-36 (|x| + |y|) + 2^-140 (absolute errors at subnormal
// scale).  The bf16 boundary below |r| lies at least a quarter bf16 step (>= 2^-10 |r|) away,
// beyond e whenever |r| >= 2^-25 (|x| + |y|).  Returns false when either result is not certified
// to round like the exact value.
__device__ __forceinline__ bool rope_pair_f32(uint32_t w, const RotRegs& t, uint32_t& out) {
  const float x = __uint_as_float(w << 16), y = __uint_as_float(w & 0xFFFF0000u);
  const uint64_t xx = f2_pack(x, x), yy = f2_pack(y, y);
  const uint64_t r1 = f2_fma(xx, t.hi, f2_mul(yy, t.nhi));
  const uint64_t lo = f2_fma(xx, t.lo, f2_mul(yy, t.nlo));
  float xr, yr;
  f2_unpack(f2_add(r1, lo), xr, yr);
  out = pack_bf16x2(xr, yr);
  if (!OSP_ROPE_CERTIFY) return true;
  const float a = fabsf(x) + fabsf(y);
  if (a == 0.f) return true;   // both results are exactly (signed) zero, in any precision
  const float abs_term = fmaf(a, 0x1p-36f, 0x1p-140f), tiny = a * 0x1p-25f;
  return fabsf(xr) >= tiny && fabsf(yr) >= tiny && bf16_rn_certain(xr, fmaf(fabsf(xr), 0x1p-23f, abs_term)) &&
         bf16_rn_certain(yr, fmaf(fabsf(yr), 0x1p-23f, abs_term));
}

// Thread work item = (row, 16-byte column within a head): the thread computes the rotation of
// its column's 4 channel pairs at its row's position once (fp64 sincos, kept in registers) and
// applies it to that column of every head of every tensor.  Consecutive threads take consecutive
// columns, then the next row, so each warp load covers whole 16 * (head_dim / 8)-byte head
// segments of a few rows.
template <int MAP, int NT>
__global__ void __launch_bounds__(kThreads, 2) permute_rope_kernel(const PermuteParams p,
                                                                   const __grid_constant__ PackParam<MAP> tab) {
  // heads per step: about 12 independent 16-byte loads in flight per thread over the NT tensors
  constexpr int HS = NT == 1 ? OSP_ROPE_HS1 : (NT == 2 ? OSP_ROPE_HS2 : OSP_ROPE_HS3);
  __shared__ double omega[kMaxPairs];
  const int npairs = p.head_dim >> 1;
  // Frequencies of every channel pair: pair j of a chunk of size d_a -> theta^(-2j/d_a).
  for (int i = threadIdx.x; i < npairs; i += blockDim.x) {
    const int c = 2 * i;
    int j, da;
    if (c < p.d_t) { j = i; da = p.d_t; }
    else if (c < p.d_t + p.d_h) { j = i - p.d_t / 2; da = p.d_h; }
    else { j = i - (p.d_t + p.d_h) / 2; da = p.d_w; }
    omega[i] = exp2(-(2.0 * j / da) * p.log2_theta);
  }
  __syncthreads();
  const int dv = p.head_dim >> 3;           // 16-byte columns per head
  const int heads = p.vpr / dv;
  const int per_set = (MAP == kMapIdentity || MAP == kMapPacked) ? 0 : p.N / p.sparse_k;
  const long long items = p.rows * dv;
  bool all_inplace = true;
  for (int t = 0; t < NT; ++t) all_inplace &= (const void*)p.src[t] == (const void*)p.dst[t];

  for (long long it = (long long)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (long long)gridDim.x * blockDim.x) {
    const long long r = it / dv;
    const int cv = (int)(it - r * dv);
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
      const int sl = (int)(r - bk * per_set);
      const int g = (int)(bk % p.sparse_k);
      const long long b = bk / p.sparse_k;
      token = skiparse_token(g, sl, p.sparse_k, p.mode);
      if (MAP == kMapGather) { s_row = b * p.N + token; d_row = r; }
      else { s_row = r; d_row = b * p.N + token; }
    }
    const int v = token - text_len;  // < 0 for text tokens
    if (v < 0 && all_inplace) continue;          // text row in place: nothing to do
    const long long sb = s_row * p.vpr + cv, db = d_row * p.vpr + cv;
    // tensors this row writes: all, except in-place ones on a text row
    unsigned todo = 0;
#pragma unroll
    for (int t = 0; t < NT; ++t)
      if (!(v < 0 && (const void*)p.src[t] == (const void*)p.dst[t])) todo |= 1u << t;
    uint4 val[NT][HS];
    bool live[NT][HS];
    auto load_step = [&](int h0) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int u = 0; u < HS; ++u) {
          const long long off = (long long)(h0 + u) * dv;
          live[t][u] = ((todo >> t) & 1u) && h0 + u < heads && index_ok(sb + off, p.src_vecs, p.status) &&
                       index_ok(db + off, p.dst_vecs, p.status);
          if (live[t][u]) val[t][u] = p.src[t][sb + off];
        }
      }
    };
    // the first step's loads go out before the rotation constants are computed, so their
    // latency overlaps the sincos
    load_step(0);
    // rotation of this column's 4 pairs at the row's (t, h, w) position (identity for text)
    RotRegs rot[4];
    const bool rotate_row = p.rope_mask && v >= 0;
    if (rotate_row) {
      const int tp = v / (H * W), hp = (v / W) % H, wp = v % W;
      // one sincos at a time (its registers are not needed by the streaming loop below)
      double sc[4][2];
#pragma unroll 1
      for (int e = 0; e < 4; ++e) {
        const int pr = 4 * cv + e, c = 2 * pr;
        const int pos = c < p.d_t ? tp : (c < p.d_t + p.d_h ? hp : wp);
        sincos((double)pos * omega[pr], &sc[e][1], &sc[e][0]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) rot[e] = rot_regs(sc[e][0], sc[e][1]);
    }
#pragma unroll 1
    for (int h0 = 0;;) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const bool rot_t = rotate_row && ((p.rope_mask >> t) & 1u);
#pragma unroll
        for (int u = 0; u < HS; ++u) {
          if (!live[t][u]) continue;
          uint4 x = val[t][u];
          if (rot_t) {
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            uint32_t o[4];
            bool certain = true;
#pragma unroll
            for (int e = 0; e < 4; ++e) certain &= rope_pair_f32(w[e], rot[e], o[e]);
            if (!certain) {
              // rare (about 1e-4 of the pairs of N(0,1) data): redo the four pairs in fp64
#pragma unroll 1
              for (int e = 0; e < 4; ++e) o[e] = rope_pair_f64(w[e], rot[e].hi, rot[e].lo);
            }
            x = make_uint4(o[0], o[1], o[2], o[3]);
          }
          p.dst[t][db + (long long)(h0 + u) * dv] = x;
        }
      }
      h0 += HS;
      if (h0 >= heads) break;
      load_step(h0);
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
  const long long items = p.rows * (p.head_dim / 8);
  const int sms = device_sm_count();
  const long long grid = std::min<long long>((items + kThreads - 1) / kThreads, (long long)sms * 8);
  if (grid <= 0) return OSP_OK;
  const dim3 g((unsigned)grid), b(kThreads);
  switch (map) {
    case kMapIdentity:
      permute_rope_kernel<kMapIdentity, 2><<<g, b, 0, stream>>>(p, NoPackTable{});
      break;
    case kMapPacked:
      permute_rope_kernel<kMapPacked, 2><<<g, b, 0, stream>>>(p, *tab);
      break;
    case kMapGather:
      if (p.n_tensors == 3) permute_rope_kernel<kMapGather, 3><<<g, b, 0, stream>>>(p, NoPackTable{});
      else if (p.n_tensors == 2) permute_rope_kernel<kMapGather, 2><<<g, b, 0, stream>>>(p, NoPackTable{});
      else permute_rope_kernel<kMapGather, 1><<<g, b, 0, stream>>>(p, NoPackTable{});
      break;
    default:
      permute_rope_kernel<kMapScatter, 1><<<g, b, 0, stream>>>(p, NoPackTable{});
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
