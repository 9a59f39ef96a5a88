// Temporal attention of the factorized "2D + 1D" scheme: token (t, h, w) attends to the tokens
// (t', h, w) of the same spatial position, every t' or (causal) t' <= t.
//
// Sources: "CogVideoX: Text-to-Video Diffusion Models with an Expert Transformer", section 2.2
// (separated spatial and temporal attention of earlier video models) and Table 8 (3D full vs
// 2D + 1D attention); the Sora page, "Video DiT Diffusion Model" (Causal Time Attention).
//
// The work is many independent tiny problems: one (sample, spatial position, head) set of T
// tokens (T <= 64) at a stride of H*W rows, T x T scores over head_dim channels.  Per token and
// head it reads q, k, v and writes o once (8 * head_dim bytes) for 4 * T * head_dim flops:
// 6.5 flop/byte at T = 13, d = 64, far below the balance point, so the kernel is bound by HBM.
// The design therefore follows the memory: each warp owns one set at a time and stages its
// q/k/v rows in shared memory with 16-byte cp.async copies; many resident warps (one staging
// buffer each, ~100 KB of shared memory per CTA, two CTAs per SM) keep enough copies in flight,
// which measured faster than fewer warps with double buffers.  The small contractions run on mma.sync
// (m16n8k16, bf16 in, fp32 accumulate) so that the arithmetic costs a few dozen instructions
// per set instead of thousands of scalar FMAs.  The 128-row tcgen05 tiles of the main kernel
// would leave more than 85 % of every tile empty here.

#include "osp_internal.h"

// Staging buffers per warp (2: the next set's copies overlap the current set's arithmetic) and
// the shared memory a CTA may take (bounds the warps per CTA).  Measured on B200 (GB/s, CogVideoX
// / Open-Sora Plan / long grids): 1 buffer, 100 KB: 5270 / 5260 / 5740; 2 buffers, 200 KB:
// 5160 / 3930 / 5620.
#ifndef OSP_TEMPORAL_BUFS
#define OSP_TEMPORAL_BUFS 1
#endif
#ifndef OSP_TEMPORAL_SMEM_KB
#define OSP_TEMPORAL_SMEM_KB 100
#endif

namespace osp {

namespace {

struct TemporalParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* o;
  int T, HW, heads;
  long long n_sets;     // B * HW * heads, set s = (b * HW + pos) * heads + h
  float scale_log2;
  int causal;
  int warps;            // warps per CTA (each with its own staging buffers)
  unsigned long long elems;   // elements of each tensor (debug index checks)
  unsigned* status;
  // training forward (optional): row log-sum-exp lse[set * lse_stride + t] = m + log2(l) in the
  // log2 domain of the scaled scores, the layout the backward kernels read
  float* lse;
  int lse_stride;
  unsigned long long lse_elems;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool fill) {
  // src-size 0 writes 16 zero bytes and reads nothing
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(fill ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D, int MT>
struct TemporalCfg {
  static constexpr int kRows = 16 * MT;              // token rows per set, padded
  static constexpr int kRowBytes = D * 2 + 16;       // padded row: conflict-free ldmatrix
  static constexpr int kTensorBytes = kRows * kRowBytes;
  static constexpr int kBufBytes = 3 * kTensorBytes; // q, k, v
  static constexpr int kBufs = OSP_TEMPORAL_BUFS;
  static constexpr int kWarpBytes = kBufs * kBufBytes;
};

template <int D, int MT>
__global__ void __launch_bounds__(256) attn_temporal_kernel(const TemporalParams p) {
  using C = TemporalCfg<D, MT>;
  constexpr int kChunks = D / 8;                     // 16-byte chunks per row
  extern __shared__ __align__(128) unsigned char smem_t[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t wbase = smem_u32(smem_t) + (uint32_t)(warp * C::kWarpBytes);
  const long long step = (long long)gridDim.x * p.warps;
  long long set = (long long)blockIdx.x * p.warps + warp;
  const int g = lane >> 2, c = lane & 3;

  // global element offset of row t = 0 of a set (the host checks n_sets < 2^31); row t adds
  // t * tstride
  const long long tstride = (long long)p.HW * p.heads * D;
  auto set_base = [&](long long s) -> long long {
    const int si = (int)s;
    const int h = si % p.heads, bp = si / p.heads;
    const int pos = bp % p.HW, b = bp / p.HW;
    return ((long long)b * p.T * p.HW + pos) * p.heads * D + (long long)h * D;
  };
  auto prefetch = [&](long long s, int buf) {
    const uint32_t base = wbase + (uint32_t)(buf * C::kBufBytes);
    const long long sb = set_base(s);
    for (int ch = lane; ch < C::kRows * kChunks; ch += 32) {
      const int r = ch / kChunks, cc = ch - r * kChunks;
      const bool live = r < p.T && index_ok(sb + r * tstride + cc * 8 + 7, p.elems, p.status);
      const long long off = live ? sb + r * tstride + cc * 8 : 0;
      const uint32_t dst = base + (uint32_t)(r * C::kRowBytes + cc * 16);
      cp_async16(dst, p.q + off, live);
      cp_async16(dst + C::kTensorBytes, p.k + off, live);
      cp_async16(dst + 2 * C::kTensorBytes, p.v + off, live);
    }
    cp_async_commit();
  };

  int buf = 0;
  if (C::kBufs == 2 && set < p.n_sets) prefetch(set, 0);
  for (; set < p.n_sets; set += step, buf ^= (C::kBufs - 1)) {
    if constexpr (C::kBufs == 2) {
      const bool more = set + step < p.n_sets;
      if (more) prefetch(set + step, buf ^ 1);
      if (more) cp_async_wait<1>();
      else cp_async_wait<0>();
    } else {
      prefetch(set, 0);
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint32_t sq = wbase + (uint32_t)(buf * C::kBufBytes);
    const uint32_t sk = sq + C::kTensorBytes, sv = sq + 2 * C::kTensorBytes;

#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      // ---- S = Q K^T for query rows mt*16 .. mt*16+15, all kRows keys
      float s[2 * MT][4];
#pragma unroll
      for (int nt = 0; nt < 2 * MT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(sq + (uint32_t)((mt * 16 + (lane & 15)) * C::kRowBytes + (kk * 16 + (lane >> 4) * 8) * 2), a[0], a[1],
                a[2], a[3]);
#pragma unroll
        for (int n2 = 0; n2 < MT; ++n2) {   // 16 keys per ldmatrix.x4
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sk + (uint32_t)((n2 * 16 + (lane & 7) + ((lane >> 4) << 3)) * C::kRowBytes +
                                  (kk * 16 + ((lane >> 3) & 1) * 8) * 2),
                  b0, b1, b2, b3);
          mma_bf16_16816(s[2 * n2], a, b0, b1);
          mma_bf16_16816(s[2 * n2 + 1], a, b2, b3);
        }
      }
      // ---- mask, row max, exponentials, row sums (rows r0 = mt*16 + g and r1 = r0 + 8)
      const int r0 = mt * 16 + g, r1 = r0 + 8;
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2 * MT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = nt * 8 + 2 * c + e;
          const bool ok0 = key < p.T && (!p.causal || key <= r0);
          const bool ok1 = key < p.T && (!p.causal || key <= r1);
          s[nt][e] = ok0 ? s[nt][e] * p.scale_log2 : -INFINITY;
          s[nt][2 + e] = ok1 ? s[nt][2 + e] * p.scale_log2 : -INFINITY;
          m0 = fmaxf(m0, s[nt][e]);
          m1 = fmaxf(m1, s[nt][2 + e]);
        }
      }
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
      // rows past T with the causal mask still see key 0, so m is finite on every row
      float l0 = 0.f, l1 = 0.f;
      uint32_t pa[MT][4];   // P as A fragments, one per 16 keys
#pragma unroll
      for (int nt = 0; nt < 2 * MT; ++nt) {
        const float e0 = ex2_approx(s[nt][0] - m0), e1 = ex2_approx(s[nt][1] - m0);
        const float e2 = ex2_approx(s[nt][2] - m1), e3 = ex2_approx(s[nt][3] - m1);
        l0 += e0 + e1;
        l1 += e2 + e3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(e0, e1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(e2, e3);
      }
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if (p.lse && c == 0) {   // one lane of the four holding each row
        const unsigned long long lb = (unsigned long long)set * p.lse_stride;
        if (r0 < p.T && index_ok(lb + r0, p.lse_elems, p.status)) p.lse[lb + r0] = m0 + __log2f(l0);
        if (r1 < p.T && index_ok(lb + r1, p.lse_elems, p.status)) p.lse[lb + r1] = m1 + __log2f(l1);
      }
      // ---- O = P V
      float o[D / 8][4];
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < MT; ++kk) {
        // A fragment of keys kk*16..+15: (row g, keys 2c..) from n-tile 2kk, (row g+8) likewise,
        // then the same rows for keys +8 from n-tile 2kk+1
        const uint32_t a[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
#pragma unroll
        for (int n2 = 0; n2 < D / 16; ++n2) {   // 16 channels per ldmatrix.x4.trans
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sv + (uint32_t)((kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * C::kRowBytes +
                                    (n2 * 16 + (lane >> 4) * 8) * 2),
                    b0, b1, b2, b3);
          mma_bf16_16816(o[2 * n2], a, b0, b1);
          mma_bf16_16816(o[2 * n2 + 1], a, b2, b3);
        }
      }
      // ---- normalise and park the bf16 rows in the (consumed) Q rows of this m-tile
      const float i0 = 1.f / l0, i1 = 1.f / l1;
      __syncwarp();
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        const uint32_t col = (uint32_t)((nt * 8 + 2 * c) * 2);
        const uint32_t w0 = pack_bf16x2(o[nt][0] * i0, o[nt][1] * i0);
        const uint32_t w1 = pack_bf16x2(o[nt][2] * i1, o[nt][3] * i1);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(sq + (uint32_t)(r0 * C::kRowBytes) + col), "r"(w0) : "memory");
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(sq + (uint32_t)(r1 * C::kRowBytes) + col), "r"(w1) : "memory");
      }
    }
    __syncwarp();
    // ---- coalesced 16-byte stores of the T output rows
    const long long ob = set_base(set);
    for (int ch = lane; ch < p.T * kChunks; ch += 32) {
      const int r = ch / kChunks, cc = ch - r * kChunks;
      uint4 val;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                   : "r"(sq + (uint32_t)(r * C::kRowBytes + cc * 16)));
      if (index_ok(ob + r * tstride + cc * 8 + 7, p.elems, p.status))
        *reinterpret_cast<uint4*>(p.o + ob + r * tstride + cc * 8) = val;
    }
    __syncwarp();   // this buffer is refilled by the prefetch two sets later
  }
}

template <int D, int MT>
int launch_temporal_t(TemporalParams& p, cudaStream_t stream) {
  using C = TemporalCfg<D, MT>;
  // as many warps per CTA (<= 8) as fit the shared-memory budget
  p.warps = std::max(1, std::min(8, (OSP_TEMPORAL_SMEM_KB * 1024) / C::kWarpBytes));
  const int smem = p.warps * C::kWarpBytes;
  const int rc = ensure_smem_attr(reinterpret_cast<const void*>(attn_temporal_kernel<D, MT>), smem,
                                  "attn_temporal_kernel");
  if (rc) return rc;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_temporal_kernel<D, MT>, p.warps * 32, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const long long ctas_needed = (p.n_sets + p.warps - 1) / p.warps;
  const long long grid = std::min<long long>(ctas_needed, (long long)device_sm_count() * per_sm);
  attn_temporal_kernel<D, MT><<<(unsigned)grid, p.warps * 32, smem, stream>>>(p);
  return check_launch("attn_temporal_kernel");
}

template <int D>
int launch_temporal_d(TemporalParams& p, cudaStream_t stream) {
  switch ((p.T + 15) / 16) {
    case 1: return launch_temporal_t<D, 1>(p, stream);
    case 2: return launch_temporal_t<D, 2>(p, stream);
    case 3: return launch_temporal_t<D, 3>(p, stream);
    default: return launch_temporal_t<D, 4>(p, stream);
  }
}

// ------------------------------------------------------------------------------------------
// Backward of the temporal attention for T <= 64: one warp per set, as the forward.
//
// Per set the warp stages q, k, v, o and dO (T rows each) and the set's saved lse, forms
// Dv_i = rowsum(dO_i * O_i), then runs two passes over the same mma.sync fragment patterns as
// the forward (C = X Y^T from rows of X and Y; C = A Z with A the packed bf16 fragments of a
// score tile and Z rows read transposed):
//   keys major   (16 keys at a time):  S^T = K Q^T, dP^T = V dO^T, P^T = exp2(S^T * c - lse),
//                                      dS^T = P^T * (dP^T - Dv); dV = P^T dO, dK = dS^T Q * scale;
//   queries major (16 queries at a time): S, dP, P, dS as above; dQ = dS K * scale.
// The second pass recomputes S and dP instead of transposing P / dS through shared memory: the
// products are small next to the 16 * head_dim bytes that every token and head moves through HBM
// (q, k, v, o, dO read; dQ, dK, dV written).
// ------------------------------------------------------------------------------------------
#ifndef OSP_TEMPORAL_BWD_SMEM_KB
#define OSP_TEMPORAL_BWD_SMEM_KB 100
#endif

struct TemporalBwdParams {
  const __nv_bfloat16 *q, *k, *v, *o, *dout;
  const float* lse;
  __nv_bfloat16 *dq, *dk, *dv;
  int T, HW, heads;
  long long n_sets;     // B * HW * heads, set s = (b * HW + pos) * heads + h
  int lse_stride;       // floats between the lse rows of consecutive sets
  float scale, scale_log2;
  int causal;
  int warps;
  unsigned long long elems, lse_elems;
  unsigned* status;
};

template <int D, int MT>
struct TemporalBwdCfg {
  static constexpr int kRows = 16 * MT;
  static constexpr int kRowBytes = D * 2 + 16;
  static constexpr int kTensorBytes = kRows * kRowBytes;
  static constexpr int kOutOff = 5 * kTensorBytes;             // q, k, v, o, dO, then 16 output rows
  static constexpr int kVecOff = kOutOff + 16 * kRowBytes;      // lse[kRows], Dv[kRows] (fp32)
  static constexpr int kWarpBytes = kVecOff + 2 * kRows * 4;
};

// acc[2*MT] (16 x kRows, C layout) = rows x0 .. x0+15 of X times the kRows rows of Y, transposed
template <int D, int MT>
__device__ __forceinline__ void tb_rows_by_rows(uint32_t X, int x0, uint32_t Y, int lane, float (&acc)[2 * MT][4]) {
  using C = TemporalBwdCfg<D, MT>;
#pragma unroll
  for (int nt = 0; nt < 2 * MT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(X + (uint32_t)((x0 + (lane & 15)) * C::kRowBytes + (kk * 16 + (lane >> 4) * 8) * 2), a[0], a[1], a[2],
            a[3]);
#pragma unroll
    for (int n2 = 0; n2 < MT; ++n2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(Y + (uint32_t)((n2 * 16 + (lane & 7) + ((lane >> 4) << 3)) * C::kRowBytes +
                             (kk * 16 + ((lane >> 3) & 1) * 8) * 2),
              b0, b1, b2, b3);
      mma_bf16_16816(acc[2 * n2], a, b0, b1);
      mma_bf16_16816(acc[2 * n2 + 1], a, b2, b3);
    }
  }
}

// out (16 x D, C layout) = A (16 x kRows, packed bf16 fragments) times the kRows rows of Z
template <int D, int MT>
__device__ __forceinline__ void tb_frag_by_rows(const uint32_t (&a)[MT][4], uint32_t Z, int lane,
                                                float (&out)[D / 8][4]) {
  using C = TemporalBwdCfg<D, MT>;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) out[nt][0] = out[nt][1] = out[nt][2] = out[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < MT; ++kk) {
#pragma unroll
    for (int n2 = 0; n2 < D / 16; ++n2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(Z + (uint32_t)((kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * C::kRowBytes +
                               (n2 * 16 + (lane >> 4) * 8) * 2),
                b0, b1, b2, b3);
      mma_bf16_16816(out[2 * n2], a[kk], b0, b1);
      mma_bf16_16816(out[2 * n2 + 1], a[kk], b2, b3);
    }
  }
}

// Writes a 16 x D fp32 C-layout tile, times mul, as bf16 rows r0 .. r0+15 (< T) of dst.
template <int D, int MT>
__device__ __forceinline__ void tb_store_rows(const float (&acc)[D / 8][4], float mul, uint32_t so, int lane, int r0,
                                              int T, long long base, long long tstride, __nv_bfloat16* dst,
                                              const TemporalBwdParams& p) {
  using C = TemporalBwdCfg<D, MT>;
  constexpr int kChunks = D / 8;
  const int g = lane >> 2, c = lane & 3;
  __syncwarp();
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const uint32_t col = (uint32_t)((nt * 8 + 2 * c) * 2);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(so + (uint32_t)(g * C::kRowBytes) + col),
                 "r"(pack_bf16x2(acc[nt][0] * mul, acc[nt][1] * mul))
                 : "memory");
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(so + (uint32_t)((g + 8) * C::kRowBytes) + col),
                 "r"(pack_bf16x2(acc[nt][2] * mul, acc[nt][3] * mul))
                 : "memory");
  }
  __syncwarp();
  const int rows = min(16, T - r0);
  for (int ch = lane; ch < rows * kChunks; ch += 32) {
    const int r = ch / kChunks, cc = ch - r * kChunks;
    uint4 val;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                 : "r"(so + (uint32_t)(r * C::kRowBytes + cc * 16)));
    const long long off = base + (long long)(r0 + r) * tstride + cc * 8;
    if (index_ok(off + 7, p.elems, p.status)) *reinterpret_cast<uint4*>(dst + off) = val;
  }
}

template <int D, int MT>
__global__ void __launch_bounds__(256) attn_temporal_bwd_kernel(const TemporalBwdParams p) {
  using C = TemporalBwdCfg<D, MT>;
  constexpr int kChunks = D / 8;
  extern __shared__ __align__(128) unsigned char smem_tb[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sq = smem_u32(smem_tb) + (uint32_t)(warp * C::kWarpBytes);
  const uint32_t sk = sq + C::kTensorBytes, sv = sq + 2 * C::kTensorBytes, so_in = sq + 3 * C::kTensorBytes,
                 sdo = sq + 4 * C::kTensorBytes, sout = sq + C::kOutOff;
  float* vec = reinterpret_cast<float*>(smem_tb + warp * C::kWarpBytes + C::kVecOff);
  float* s_lse = vec;
  float* s_dv = vec + C::kRows;
  const int g = lane >> 2, c = lane & 3;
  const long long tstride = (long long)p.HW * p.heads * D;
  const long long step = (long long)gridDim.x * p.warps;

  for (long long set = (long long)blockIdx.x * p.warps + warp; set < p.n_sets; set += step) {
    const int si = (int)set;
    const int h = si % p.heads, bp = si / p.heads;
    const int pos = bp % p.HW, b = bp / p.HW;
    const long long base = ((long long)b * p.T * p.HW + pos) * p.heads * D + (long long)h * D;
    // ---- stage the set's q, k, v, o, dO rows (zero past T) and its lse
    for (int ch = lane; ch < C::kRows * kChunks; ch += 32) {
      const int r = ch / kChunks, cc = ch - r * kChunks;
      const bool live = r < p.T && index_ok(base + r * tstride + cc * 8 + 7, p.elems, p.status);
      const long long off = live ? base + r * tstride + cc * 8 : 0;
      const uint32_t dst = sq + (uint32_t)(r * C::kRowBytes + cc * 16);
      cp_async16(dst, p.q + off, live);
      cp_async16(dst + C::kTensorBytes, p.k + off, live);
      cp_async16(dst + 2 * C::kTensorBytes, p.v + off, live);
      cp_async16(dst + 3 * C::kTensorBytes, p.o + off, live);
      cp_async16(dst + 4 * C::kTensorBytes, p.dout + off, live);
    }
    cp_async_commit();
    for (int t = lane; t < C::kRows; t += 32) {
      const unsigned long long li = (unsigned long long)set * p.lse_stride + t;
      s_lse[t] = (t < p.T && index_ok(li, p.lse_elems, p.status)) ? p.lse[li] : 0.f;
    }
    cp_async_wait<0>();
    __syncwarp();
    // ---- Dv = rowsum(dO * O): four lanes per row, D / 4 channels each (zero rows past T)
#pragma unroll
    for (int i = 0; i < C::kRows / 8; ++i) {
      const int r = i * 8 + g;
      float acc = 0.f;
#pragma unroll
      for (int v4 = 0; v4 < D / 32; ++v4) {
        const uint32_t off = (uint32_t)(r * C::kRowBytes + (c * (D / 4) + v4 * 8) * 2);
        uint4 a, d;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w)
                     : "r"(so_in + off));
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(d.x), "=r"(d.y), "=r"(d.z), "=r"(d.w)
                     : "r"(sdo + off));
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[e]));
          const float2 df = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dw[e]));
          acc = fmaf(af.x, df.x, acc);
          acc = fmaf(af.y, df.y, acc);
        }
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (c == 0) s_dv[r] = acc;
    }
    __syncwarp();

    // ---- keys major: dV and dK of keys kt*16 .. kt*16+15
#pragma unroll 1
    for (int kt = 0; kt < MT; ++kt) {
      if (kt * 16 >= p.T) break;
      uint32_t pa[MT][4], da[MT][4];
      {
        float st[2 * MT][4], dpt[2 * MT][4];
        tb_rows_by_rows<D, MT>(sk, kt * 16, sq, lane, st);
        tb_rows_by_rows<D, MT>(sv, kt * 16, sdo, lane, dpt);
        const int j0 = kt * 16 + g, j1 = j0 + 8;
#pragma unroll
        for (int nt = 0; nt < 2 * MT; ++nt) {
          float pe[4], de[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = nt * 8 + 2 * c + (e & 1);   // query (column)
            const int j = (e < 2) ? j0 : j1;          // key (row)
            const bool ok = i < p.T && j < p.T && (!p.causal || j <= i);
            const float pv = ok ? ex2_approx(st[nt][e] * p.scale_log2 - s_lse[i]) : 0.f;
            pe[e] = pv;
            de[e] = pv * (dpt[nt][e] - s_dv[i]);
          }
          pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(pe[0], pe[1]);
          pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(pe[2], pe[3]);
          da[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(de[0], de[1]);
          da[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(de[2], de[3]);
        }
      }
      {
        float acc[D / 8][4];
        tb_frag_by_rows<D, MT>(pa, sdo, lane, acc);
        tb_store_rows<D, MT>(acc, 1.f, sout, lane, kt * 16, p.T, base, tstride, p.dv, p);
        tb_frag_by_rows<D, MT>(da, sq, lane, acc);
        tb_store_rows<D, MT>(acc, p.scale, sout, lane, kt * 16, p.T, base, tstride, p.dk, p);
      }
    }
    // ---- queries major: dQ of queries mt*16 .. mt*16+15
#pragma unroll 1
    for (int mt = 0; mt < MT; ++mt) {
      if (mt * 16 >= p.T) break;
      uint32_t da[MT][4];
      {
        float s[2 * MT][4], dp[2 * MT][4];
        tb_rows_by_rows<D, MT>(sq, mt * 16, sk, lane, s);
        tb_rows_by_rows<D, MT>(sdo, mt * 16, sv, lane, dp);
        const int i0 = mt * 16 + g, i1 = i0 + 8;
#pragma unroll
        for (int nt = 0; nt < 2 * MT; ++nt) {
          float de[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = nt * 8 + 2 * c + (e & 1);   // key (column)
            const int i = (e < 2) ? i0 : i1;          // query (row)
            const bool ok = i < p.T && j < p.T && (!p.causal || j <= i);
            const float pv = ok ? ex2_approx(s[nt][e] * p.scale_log2 - s_lse[i]) : 0.f;
            de[e] = pv * (dp[nt][e] - s_dv[i]);
          }
          da[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(de[0], de[1]);
          da[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(de[2], de[3]);
        }
      }
      float acc[D / 8][4];
      tb_frag_by_rows<D, MT>(da, sk, lane, acc);
      tb_store_rows<D, MT>(acc, p.scale, sout, lane, mt * 16, p.T, base, tstride, p.dq, p);
    }
    __syncwarp();   // the staging area is refilled for the next set
  }
}

template <int D, int MT>
int launch_temporal_bwd_t(TemporalBwdParams& p, cudaStream_t stream) {
  using C = TemporalBwdCfg<D, MT>;
  p.warps = std::max(1, std::min(8, (OSP_TEMPORAL_BWD_SMEM_KB * 1024) / C::kWarpBytes));
  const int smem = p.warps * C::kWarpBytes;
  const int rc = ensure_smem_attr(reinterpret_cast<const void*>(attn_temporal_bwd_kernel<D, MT>), smem,
                                  "attn_temporal_bwd_kernel");
  if (rc) return rc;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_temporal_bwd_kernel<D, MT>, p.warps * 32, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const long long ctas_needed = (p.n_sets + p.warps - 1) / p.warps;
  const long long grid = std::min<long long>(ctas_needed, (long long)device_sm_count() * per_sm);
  attn_temporal_bwd_kernel<D, MT><<<(unsigned)grid, p.warps * 32, smem, stream>>>(p);
  return check_launch("attn_temporal_bwd_kernel");
}

template <int D>
int launch_temporal_bwd_d(TemporalBwdParams& p, cudaStream_t stream) {
  switch ((p.T + 15) / 16) {
    case 1: return launch_temporal_bwd_t<D, 1>(p, stream);
    case 2: return launch_temporal_bwd_t<D, 2>(p, stream);
    case 3: return launch_temporal_bwd_t<D, 3>(p, stream);
    default: return launch_temporal_bwd_t<D, 4>(p, stream);
  }
}

}  // namespace

int temporal_attention_launch(const void* q, const void* k, const void* v, void* o, const osp_shape& s, int causal,
                              float scale, cudaStream_t stream, float* lse) {
  if (s.T > 64) return set_error(OSP_ERR_UNSUPPORTED, "the per-set temporal kernel takes T <= 64 (got %d)", s.T);
  TemporalParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.T = s.T;
  p.HW = s.H * s.W;
  p.heads = s.heads;
  p.n_sets = (long long)s.B * p.HW * s.heads;
  if (p.n_sets > 0x7fffffffLL) return set_error(OSP_ERR_UNSUPPORTED, "%lld temporal sets is too many", p.n_sets);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal;
  p.elems = (unsigned long long)s.B * s.T * p.HW * s.heads * s.head_dim / bounds_check_divisor();
  p.lse = lse;
  p.lse_stride = (s.T + 127) / 128 * 128;   // the layout of the tile kernels' lse (one row per set)
  p.lse_elems = (unsigned long long)p.n_sets * p.lse_stride / bounds_check_divisor();
  p.status = device_status_word();
  if (!p.status) return OSP_ERR_CUDA;
  switch (s.head_dim) {
    case 64: return launch_temporal_d<64>(p, stream);
    case 96: return launch_temporal_d<96>(p, stream);
    case 128: return launch_temporal_d<128>(p, stream);
    default: return set_error(OSP_ERR_UNSUPPORTED, "head_dim %d not in {64, 96, 128}", s.head_dim);
  }
}

int temporal_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, const osp_shape& s, int causal,
                             float scale, cudaStream_t stream) {
  if (s.T > 64) return set_error(OSP_ERR_UNSUPPORTED, "the per-set temporal backward takes T <= 64 (got %d)", s.T);
  TemporalBwdParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.lse = lse;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.T = s.T;
  p.HW = s.H * s.W;
  p.heads = s.heads;
  p.n_sets = (long long)s.B * p.HW * s.heads;
  if (p.n_sets > 0x7fffffffLL) return set_error(OSP_ERR_UNSUPPORTED, "%lld temporal sets is too many", p.n_sets);
  p.lse_stride = (s.T + 127) / 128 * 128;   // the training forward's lse rows (one per set and head)
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal;
  const unsigned long long div = (unsigned long long)bounds_check_divisor();
  p.elems = (unsigned long long)s.B * s.T * p.HW * s.heads * s.head_dim / div;
  p.lse_elems = (unsigned long long)p.n_sets * p.lse_stride / div;
  p.status = device_status_word();
  if (!p.status) return OSP_ERR_CUDA;
  switch (s.head_dim) {
    case 64: return launch_temporal_bwd_d<64>(p, stream);
    case 96: return launch_temporal_bwd_d<96>(p, stream);
    case 128: return launch_temporal_bwd_d<128>(p, stream);
    default: return set_error(OSP_ERR_UNSUPPORTED, "head_dim %d not in {64, 96, 128}", s.head_dim);
  }
}

}  // namespace osp
