// Backward pass of Skiparse attention with a joined text prefix.
//
// Source: "Open-Sora Plan: Open-Source Large Video Generation Model", section 2.2.2 (Skiparse
// attention; the text tokens are joined to every sparse set) and the chain rule of softmax
// attention.  In a sample of N = L + Nv tokens (L text, Nv video), a text query sees all N
// tokens, and a video query of set g sees the L text tokens and the n = Nv / k tokens of set g.
// The gradients split along the queries:
//   video queries of set g: a dense backward over the sample [set g's n rows in slot order;
//     the L text rows] whose first n rows are the queries.  It yields dQ of set g's rows whole,
//     and dK, dV contributions to set g's rows and to the text rows;
//   text queries: a dense backward over the natural sample whose first L rows are the queries.
//     It yields dQ of the text rows whole, and dK, dV contributions to all N rows.
// dK and dV of a text row sum the contributions of the k sets and of the text queries, those of
// a video row the contributions of its set and of the text queries; both passes leave them in
// fp32 and text_bwd_combine_kernel adds them in a fixed order (sets 0..k-1, then the text
// queries) and rounds once to bf16.  Both passes run the tcgen05 kernels of attn_bwd.cu; the
// [set rows; text rows] samples are gathered here (video queries' Q, dO, O, their keys' K, V),
// since a set's keys and the text keys then form one run of rows.

#include "osp_internal.h"

namespace osp {

namespace {

// Video token (0-based within the video part) of slot s of set g, and the inverse.
__device__ __forceinline__ int set_slot_token(int mode, int s, int g, int k) {
  if (mode == OSP_SKIP_SINGLE) return s * k + g;
  const int o = s / k;   // Group Skip: k*k-token blocks, set g takes row g of each
  return (o * k + g) * k + (s - o * k);
}
__device__ __forceinline__ void token_set_slot(int mode, int t, int k, int* g, int* s) {
  if (mode == OSP_SKIP_SINGLE) {
    *g = t % k;
    *s = t / k;
  } else {
    const int kk = k * k, ob = t / kk, rem = t - ob * kk;
    *g = rem / k;
    *s = ob * k + (rem - *g * k);
  }
}

struct TextBwdDims {
  int B, G, L, n, N;     // samples, sets (= k), text rows, rows per set, tokens per sample
  int mode, k;
  int vpr;               // 16-byte vectors per token row (heads * head_dim * 2 / 16)
  unsigned* status;
  unsigned long long aug_rows, nat_rows;   // rows of the gathered / natural tensors (debug checks)
};

// One warp per row of the [B*G][n + L] samples: row a < n is set g's slot a (a video query and
// key), row a >= n is text token a - n (a key only; its Q and dO rows are zero, O is not read).
__global__ void __launch_bounds__(256) text_bwd_gather_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                              const uint4* __restrict__ v, const uint4* __restrict__ o,
                                                              const uint4* __restrict__ dout, uint4* qa, uint4* ka,
                                                              uint4* va, uint4* oa, uint4* doa, TextBwdDims d,
                                                              long long rows) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int a = (int)(r % (d.n + d.L));
    const long long bg = r / (d.n + d.L);
    const int b = (int)(bg / d.G), g = (int)(bg % d.G);
    const bool video = a < d.n;
    const int tok = video ? d.L + set_slot_token(d.mode, a, g, d.k) : a - d.n;
    const size_t src = ((size_t)b * d.N + tok) * d.vpr, dst = (size_t)r * d.vpr;
    if (!index_ok((size_t)b * d.N + tok, d.nat_rows, d.status) || !index_ok(r, d.aug_rows, d.status)) continue;
    for (int i = lane; i < d.vpr; i += 32) {
      ka[dst + i] = k[src + i];
      va[dst + i] = v[src + i];
      if (video) {
        qa[dst + i] = q[src + i];
        doa[dst + i] = dout[src + i];
        oa[dst + i] = o[src + i];
      } else {
        qa[dst + i] = make_uint4(0, 0, 0, 0);
        doa[dst + i] = make_uint4(0, 0, 0, 0);
      }
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// One warp per natural token row (b, t): dK, dV = the rounded sum of the fp32 contributions;
// a video row also takes dQ (bf16) from its set's sample.  wpr = 4-float vectors per row.
__global__ void __launch_bounds__(256) text_bwd_combine_kernel(const float4* __restrict__ dka,
                                                               const float4* __restrict__ dva,
                                                               const float4* __restrict__ dkt,
                                                               const float4* __restrict__ dvt,
                                                               const uint2* __restrict__ dqa, uint2* dq, uint2* dk,
                                                               uint2* dv, TextBwdDims d, long long rows) {
  const int lane = threadIdx.x & 31;
  const int wpr = d.vpr * 2;   // 4-element vectors per row
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int t = (int)(r % d.N);
    const long long b = r / d.N;
    const size_t nat = (size_t)r * wpr;
    if (!index_ok(r, d.nat_rows, d.status)) continue;
    if (t < d.L) {
      for (int i = lane; i < wpr; i += 32) {
        float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
        for (int g = 0; g < d.G; ++g) {
          const size_t arow = (size_t)(b * d.G + g) * (d.n + d.L) + d.n + t;
          if (!index_ok(arow, d.aug_rows, d.status)) break;
          const size_t ar = arow * wpr + i;
          const float4 xk = dka[ar], xv = dva[ar];
          sk = make_float4(sk.x + xk.x, sk.y + xk.y, sk.z + xk.z, sk.w + xk.w);
          sv = make_float4(sv.x + xv.x, sv.y + xv.y, sv.z + xv.z, sv.w + xv.w);
        }
        const float4 tk = dkt[nat + i], tv = dvt[nat + i];
        dk[nat + i] = make_uint2(pack_bf16_rn(sk.x + tk.x, sk.y + tk.y), pack_bf16_rn(sk.z + tk.z, sk.w + tk.w));
        dv[nat + i] = make_uint2(pack_bf16_rn(sv.x + tv.x, sv.y + tv.y), pack_bf16_rn(sv.z + tv.z, sv.w + tv.w));
      }
    } else {
      int g, s;
      token_set_slot(d.mode, t - d.L, d.k, &g, &s);
      const size_t arow = (size_t)(b * d.G + g) * (d.n + d.L) + s;
      if (!index_ok(arow, d.aug_rows, d.status)) continue;
      const size_t ar = arow * wpr;
      for (int i = lane; i < wpr; i += 32) {
        const float4 xk = dka[ar + i], xv = dva[ar + i], tk = dkt[nat + i], tv = dvt[nat + i];
        dk[nat + i] = make_uint2(pack_bf16_rn(xk.x + tk.x, xk.y + tk.y), pack_bf16_rn(xk.z + tk.z, xk.w + tk.w));
        dv[nat + i] = make_uint2(pack_bf16_rn(xv.x + tv.x, xv.y + tv.y), pack_bf16_rn(xv.z + tv.z, xv.w + tv.w));
        dq[nat + i] = dqa[ar + i];
      }
    }
  }
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

int skiparse_text_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                  const float* lse, void* dq, void* dk, void* dv, const osp_shape& s, int sparse_k,
                                  int mode, float scale, cudaStream_t stream) {
  const int L = s.text_len, Nv = s.T * s.H * s.W, N = L + Nv, G = sparse_k, n = Nv / G;
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  const size_t row_elems = (size_t)s.heads * s.head_dim;
  const size_t aug_rows = (size_t)s.B * G * (n + L), nat_rows = (size_t)s.B * N;
  TextBwdDims d{s.B, G, L, n, N, mode, sparse_k, s.heads * s.head_dim * 2 / 16, status,
                aug_rows / bounds_check_divisor(), nat_rows / bounds_check_divisor()};
  const size_t bf_aug = align256(aug_rows * row_elems * 2), f_aug = align256(aug_rows * row_elems * 4);
  const size_t f_nat = align256(nat_rows * row_elems * 4);
  // Q, K, V, O, dO and dQ of the [set; text] samples (bf16), their dK and dV (fp32), the text
  // queries' dK and dV contributions (fp32, natural order)
  const size_t bytes = 6 * bf_aug + 2 * f_aug + 2 * f_nat;
  cudaMemPool_t pool = workspace_pool();
  void* ws = nullptr;
  if (!pool || cudaMallocFromPoolAsync(&ws, bytes, pool, stream) != cudaSuccess)
    return set_error(OSP_ERR_CUDA, "stream-ordered workspace allocation (%zu bytes) failed", bytes);
  char* w = static_cast<char*>(ws);
  void *qa = w, *ka = w + bf_aug, *va = w + 2 * bf_aug, *oa = w + 3 * bf_aug, *doa = w + 4 * bf_aug,
       *dqa = w + 5 * bf_aug;
  float* dka = reinterpret_cast<float*>(w + 6 * bf_aug);
  float* dva = reinterpret_cast<float*>(w + 6 * bf_aug + f_aug);
  float* dkt = reinterpret_cast<float*>(w + 6 * bf_aug + 2 * f_aug);
  float* dvt = reinterpret_cast<float*>(w + 6 * bf_aug + 2 * f_aug + f_nat);
  const unsigned grid_cap = (unsigned)device_sm_count() * 16;
  int rc = OSP_OK;
  {
    const long long rows = (long long)aug_rows;
    const unsigned blocks = (unsigned)std::min<long long>((rows + 7) / 8, grid_cap);
    text_bwd_gather_kernel<<<blocks, 256, 0, stream>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v),
        static_cast<const uint4*>(o), static_cast<const uint4*>(dout), static_cast<uint4*>(qa),
        static_cast<uint4*>(ka), static_cast<uint4*>(va), static_cast<uint4*>(oa), static_cast<uint4*>(doa), d, rows);
    rc = check_launch("text_bwd_gather_kernel");
  }
  // video queries: B*G dense samples of n + L rows, the first n of them queries; their lse is the
  // forward's set-slot block
  if (rc == OSP_OK) {
    const osp_shape sa{s.B * G, 0, 1, 1, n + L, s.heads, s.head_dim};
    rc = attention_backward_launch(qa, ka, va, oa, doa, lse, dqa, dka, dva, sa, 0, 1, scale, stream, false, 0, n,
                                   true);
  }
  // text queries: the natural samples, the first L rows queries; their lse follows the video block
  if (rc == OSP_OK) {
    const size_t n_pad = (size_t)(n + 127) / 128 * 128;
    const float* lse_t = lse + (size_t)s.B * G * s.heads * n_pad;
    rc = attention_backward_launch(q, k, v, o, dout, lse_t, dq, dkt, dvt, s, 0, 1, scale, stream, false, 0, L, true);
  }
  if (rc == OSP_OK) {
    const long long rows = (long long)nat_rows;
    const unsigned blocks = (unsigned)std::min<long long>((rows + 7) / 8, grid_cap);
    text_bwd_combine_kernel<<<blocks, 256, 0, stream>>>(
        reinterpret_cast<const float4*>(dka), reinterpret_cast<const float4*>(dva),
        reinterpret_cast<const float4*>(dkt), reinterpret_cast<const float4*>(dvt), static_cast<const uint2*>(dqa), static_cast<uint2*>(dq), static_cast<uint2*>(dk),
        static_cast<uint2*>(dv), d, rows);
    rc = check_launch("text_bwd_combine_kernel");
  }
  cudaFreeAsync(ws, stream);
  return rc;
}

}  // namespace osp
