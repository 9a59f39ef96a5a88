// Backward pass of dense and Skiparse attention on tcgen05 tensor cores.
//
// Source: "Open-Sora Plan: Open-Source Large Video Generation Model", section 2.2.2 (the model
// is trained with Skiparse attention); the gradients are the chain rule of softmax attention.
// For one (sample, set, head) with S = Q K^T * scale, P = softmax(S), O = P V and upstream dO:
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Dv),  Dv = rowsum(dO * O),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
// P is rebuilt from the forward pass's row log-sum-exp: P = exp2(S * scale * log2(e) - lse).
//
// Three kernels:
//   attn_bwd_dvec_kernel  Dv per query row (fp32), written in set-slot order like lse;
//   attn_bwd_dkdv_kernel  one CTA per 128-key tile: K, V stay in shared memory while the set's
//                         query tiles stream through; S^T = K Q^T and dP^T = V dO^T land in
//                         tensor memory with the keys on the lanes, the compute warps turn them
//                         into P^T and dS^T (bf16, written back over S^T / dP^T), and
//                         dV += P^T dO, dK += dS^T Q accumulate in tensor memory;
//   attn_bwd_dq_kernel    one CTA per 128-query tile: Q, dO stay resident while the key tiles
//                         stream; S = Q K^T, dP = dO V^T, dS (bf16, over dP), dQ += dS K.
// Rows are addressed through the same TMA maps as the forward kernel, so Skiparse sets are
// never gathered.  Every wait is bounded (status word + abort flag, as in the forward kernel).

#include <type_traits>

#include "osp_internal.h"

namespace osp {

namespace {

constexpr int kBT = 128;                 // rows per tile (queries or keys)
constexpr int kChunkBytes = 128 * 128;   // 128 rows x 64 bf16 channels, one SW128 atom wide
// warps 0-7 compute (warp w: tensor-memory lane quarter w % 4, column half w / 4; two warps per
// SM sub-partition keep its MUFU busy), 8 TMA producer, 9 issues the score products (S, dP),
// 10 the accumulating products (dV, dK or dQ): the sub-tile products are short, and one issuing
// thread for all of them left the tensor pipe waiting on issue.
constexpr int kBwdThreads = 352;
constexpr int kComputeThreads = 256;
constexpr int kProdWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kAccWarp = 10;
// dK/dV kernel: four compute warps per SM sub-partition, each turning 16 of a sub-tile's 64
// query columns into P and dS (OSP_BWD_WIDE=0: two per sub-partition, 32 columns each).  More
// warps per sub-partition keep its MUFU and issue slots busy while each warp waits on tensor
// memory or on a barrier; a warp's chain (load, exponentials, pack, store) is half as long.
#ifndef OSP_BWD_WIDE
#define OSP_BWD_WIDE 1
#endif
constexpr int kDkCols = OSP_BWD_WIDE ? 16 : 32;          // query columns per compute warp and sub-tile
constexpr int kDkComputeWarps = 4 * (64 / kDkCols);      // 16 or 8
constexpr int kDkComputeThreads = 32 * kDkComputeWarps;
constexpr int kDkProdWarp = kDkComputeWarps, kDkMmaWarp = kDkComputeWarps + 1, kDkAccWarp = kDkComputeWarps + 2,
              kDkRedWarp = kDkComputeWarps + 3;
// One thread issues every product of the dK/dV kernel (1), or the score products and the
// accumulating products come from two warps with a buffer-free barrier between them (0); -1
// (default): one issuer at d = 64 and 128, two at d = 96 (same-box A/B with one issuer: d = 128
// +4 %, d = 64 +1 %, d = 96 -2 %).
#ifndef OSP_BWD_ONE_ISSUER
#define OSP_BWD_ONE_ISSUER -1
#endif
#ifndef OSP_BWD_FUSE_DQ
#define OSP_BWD_FUSE_DQ 1                // d = 64: dQ accumulated by the dK/dV kernel (no dQ kernel)
#endif
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
// The streamed 128-row tiles are processed as two 64-row sub-tiles, and the score buffers are
// double-buffered across sub-tiles so that the products of sub-tile t+1 run on the tensor core
// while the compute warps turn sub-tile t into P / dS.  Tensor-memory columns: buffer b holds S
// (or S^T) at 128b .. 128b+63 and dP (dP^T) at 128b+64 .. 128b+127; accumulators at 256 and 384.
constexpr int kSub = 64;
constexpr uint32_t kColAcc0 = 256;   // dV (dK kernel) or dQ (dQ kernel); dK at BwdCfg::kColDk
__device__ __forceinline__ uint32_t col_s(int buf) { return 128u * buf; }
__device__ __forceinline__ uint32_t col_dp(int buf) { return 128u * buf + 64u; }
// descriptor offset (16-byte units) of the second 64-row sub-tile of a 128-row SW128 tile
// (eight 1024-byte groups of 8 rows), for both K-major and MN-major use
constexpr uint64_t kSubDescOff = (64 * 128) >> 4;

template <int D>
struct BwdCfg {
  static constexpr int kChunks = (D + 63) / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  // Fused dQ (d = 64, where two 64-column tensor-memory buffers are free next to dV and dK): the
  // dK/dV kernel also computes dQ_i = dS_i K for every query tile it streams, from dS^T written to
  // shared memory by the compute warps, and adds it into an fp32 accumulator with one bulk
  // reduce-add per tile; the dQ kernel (which recomputes S, dP and P) is not launched.
  static constexpr bool kFuseDq = (D == 64) && OSP_BWD_FUSE_DQ;
  // Fused dQ: K and V also sit in tensor memory (32 columns each, packed bf16 pairs of channels,
  // key = lane), so the score products S^T = K Q^T and dP^T = V dO^T read only their B operand
  // from shared memory.  Both operands from shared memory cost an M = 128, N = 64, K = 16 product
  // about 60 cycles of shared-memory reads (6 KB at 128 B per cycle) against 32 of math; with A in
  // tensor memory it is bound by its math.  The dQ buffer is then single (its second copy's
  // columns hold K and V).
  static constexpr bool kKvTmem = kFuseDq;
  // d = 96: dK's accumulator moves up to columns 352 .. 447 (next to dV at 256), which leaves
  // 448 .. 495 for K, so S^T = K Q^T also takes A from tensor memory (V does not fit; dP^T keeps
  // both operands in shared memory)
  static constexpr bool kKTmem = (D == 96);
  static constexpr uint32_t kColDk = (D == 96) ? 352u : 384u;
  static constexpr bool kOneIssuer = OSP_BWD_ONE_ISSUER < 0 ? (D != 96) : (OSP_BWD_ONE_ISSUER != 0);
  // dK/dV kernel: compute warps, producer, two MMA issuers and (fused dQ) the reduce warp
  static constexpr int kThreads = 32 * (kDkComputeWarps + (kFuseDq ? 4 : 3));
  static constexpr int kResOff = 0;                                 // two resident tiles
  static constexpr int kStageOff = 2 * kTileBytes;                  // stages of two tiles each
  static constexpr int kVecOff = kStageOff + kStages * 2 * kTileBytes;
  static constexpr int kVecBytes = 2 * kBT * 4;                     // lse + Dv of one query tile
  // fused dQ: dS^T of a query tile (bf16, two 64-query SW128 chunks) double-buffered, and the
  // fp32 staging tile of dQ (row-major [128][D]) read by the bulk reduce
  static constexpr int kDsOff = (kVecOff + kStages * kVecBytes + 1023) / 1024 * 1024;
  static constexpr int kDsBytes = kFuseDq ? 2 * 2 * kChunkBytes : 0;
  static constexpr int kStgOff = kDsOff + kDsBytes;
  static constexpr int kStgBytes = kFuseDq ? kBT * D * 4 : 0;
  static constexpr int kBarOff = kStgOff + kStgBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;
};

struct BwdParams {
  int n;            // rows per set (queries = keys)
  int N;            // tokens per sample of the natural-order tensors
  int heads, G, k, layout;
  int n_tiles;      // ceil(n / 128)
  int vec_stride;   // floats per (sample*set, head) row of lse / Dv (n rounded up to 128)
  // Queries: the first q_rows rows of each set (q_tiles = ceil(q_rows / 128) tiles); n and
  // n_tiles unless only a prefix of the rows are queries (the text queries of a joined-text call)
  int q_rows, q_tiles;
  float scale_log2;
  float scale;
  const float* lse;
  float* dvec;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dk32;      // non-null: dK and dV are written unrounded, fp32, here and in dv32 (not dk, dv)
  float* dv32;
  float* dq_acc;    // fused dQ: fp32 [B*G][heads][vec_stride][D], zeroed before the dK/dV kernel
  unsigned long long dq_acc_elems;
  unsigned* status;
  unsigned long long timeout_ns;
  unsigned long long elems, vec_elems;   // elements of each BSHD tensor / of lse and Dv (debug checks)
  // Frame-causal mask (dense layout; 0 = off): blocks are [text], [frame 0], [frame 1], ...
  // (frame_hw tokens each after text_len text tokens); query r sees keys of blocks <= its own.
  int frame_hw;
  int text_len;
};

// Packed batch (block-diagonal self-attention, every sample its own set): sample i owns packed
// rows [row[i], row[i+1]), its lse / Dv / dQ-accumulator rows start at vrow[i] (the training
// forward's 256-row blocks), and tile[i] counts the 128-row tiles of the samples before it (a
// kernel's CTAs are heads * tile[n_seg]).  Passed by value as a kernel parameter.
struct BwdSegTable {
  int n_seg;
  int row[kMaxSegments + 1];
  int vrow[kMaxSegments + 1];
  int tile[kMaxSegments + 1];
};
struct NoBwdSeg {};
template <bool kPk>
using BwdSegParam = typename std::conditional<kPk, BwdSegTable, NoBwdSeg>::type;

// The (sample*set, head, 128-row tile) a CTA works on, the set's rows n (tiles n_tiles), the
// packed row its rows start at, and the first lse / Dv row of the (set, head).
struct BwdUnit {
  int tile, h, bg, b, g, n, n_tiles, row_base;
  size_t vec_row;
};
template <bool kPk>
__device__ __forceinline__ BwdUnit bwd_unit(const BwdParams& p, const BwdSegParam<kPk>& seg, int cta, bool reverse,
                                            int tiles_per_set = 0) {
  BwdUnit u;
  if constexpr (kPk) {
    // sample: the largest i < n_seg with heads * tile[i] <= cta (empty samples own no CTA)
    int lo = 0, hi = seg.n_seg;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.heads * seg.tile[mid] <= cta) lo = mid;
      else hi = mid;
    }
    const int nt = seg.tile[lo + 1] - seg.tile[lo];
    const int local = cta - p.heads * seg.tile[lo];
    u.h = local / nt;
    const int t = local - u.h * nt;
    u.tile = reverse ? nt - 1 - t : t;
    u.bg = u.b = u.g = 0;
    u.n = seg.row[lo + 1] - seg.row[lo];
    u.n_tiles = nt;
    u.row_base = seg.row[lo];
    u.vec_row = (size_t)u.h * p.vec_stride + seg.vrow[lo];
  } else {
    const int tps = tiles_per_set > 0 ? tiles_per_set : p.n_tiles;   // CTAs per (set, head)
    const int t = cta % tps;
    u.tile = reverse ? tps - 1 - t : t;
    const int hb = cta / tps;
    u.h = hb % p.heads;
    u.bg = hb / p.heads;
    u.b = u.bg / p.G;
    u.g = u.bg % p.G;
    u.n = p.n;
    u.n_tiles = p.n_tiles;
    u.row_base = 0;
    u.vec_row = ((size_t)u.bg * p.heads + u.h) * p.vec_stride;
  }
  return u;
}

// First token of the block that token x belongs to (block 0: the text prefix; block 1 + f: frame f).
__device__ __forceinline__ int causal_block_start(int x, int text_len, int hw) {
  return x < text_len ? 0 : text_len + (x - text_len) / hw * hw;
}
// Keys visible to query r: the tokens of blocks 0 .. block(r).
__device__ __forceinline__ int causal_limit(int r, int text_len, int hw) {
  return r < text_len ? text_len : text_len + ((r - text_len) / hw + 1) * hw;
}
// Bit e set when query q0 + e (e < 32) may see a key whose block starts at token kstart.  Block
// indices never decrease along the sequence, so block(q) >= block(key) exactly when q >= kstart.
__device__ __forceinline__ uint32_t causal_columns(int q0, int kstart) {
  const int sh = kstart - q0;
  return sh <= 0 ? 0xffffffffu : (sh >= 32 ? 0u : (0xffffffffu << sh));
}

__device__ __forceinline__ int bwd_slot_token(int layout, int s, int g, int k) {
  if (layout == 0) return s;
  if (layout == 1) return s * k + g;
  const int o = s / k;
  return (o * k + g) * k + (s - o * k);
}

__device__ __forceinline__ void bwd_load_tile(const CUtensorMap* tm, uint32_t dst, uint32_t bar, int layout,
                                              int chan, int row0, int g, int b, int k) {
  if (layout == 0) tma_load_3d(dst, tm, bar, chan, row0, b);
  else if (layout == 1) tma_load_4d(dst, tm, bar, chan, g, row0, b);
  else tma_load_5d(dst, tm, bar, chan, 0, g, row0 / k, b);
}

// Packed bf16 P / dS columns: compute warp half h owns the 32 columns 32h .. 32h + 31 of a
// 64-column sub-tile buffer and writes their 16 packed columns at 32h .. 32h + 15, i.e. over its
// own consumed S / dP columns, so the two warps sharing a lane quarter never touch each other's
// unread columns.  The tensor-memory A operand of K-step kk (16 rows of P / dS) starts at:
__device__ __forceinline__ uint32_t packed_col(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }
// 32-lane x 16-column tensor-memory load and 8-column store (one lane per thread)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
// 32-lane x N-column tensor-memory loads (N = 16 or 32) and stores of N packed columns (8, 16)
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 16) tmem_ld16(taddr, r);
  else tmem_ld32(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 8) tmem_st8(taddr, r);
  else tmem_st16(taddr, r);
}
// The same for the dK/dV kernel's compute warps of kDkCols columns: K-step kk (queries 16kk ..
// 16kk + 15) lies in warp column group 16kk / kDkCols, which packs its columns from its first.
__device__ __forceinline__ uint32_t packed_col_dk(int kk) {
  return (uint32_t)(kDkCols * ((16 * kk) / kDkCols) + ((16 * kk) % kDkCols) / 2);
}

__device__ __forceinline__ bool bwd_warp_wait(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------------------------------------
// Dv = rowsum(dO * O), one thread per (sample, token, head) row, stored at the row's set slot
// ------------------------------------------------------------------------------------------
template <int D, bool kPk = false>
__global__ void __launch_bounds__(256) attn_bwd_dvec_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            const BwdParams p, long long rows,
                                                            const __grid_constant__ BwdSegParam<kPk> seg) {
  for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < rows;
       r += (long long)gridDim.x * blockDim.x) {
    const int h = (int)(r % p.heads);
    const long long bt = r / p.heads;
    const int token = (int)(bt % p.N);
    const int b = (int)(bt / p.N);
    if (!index_ok(r * D + D - 1, p.elems, p.status)) continue;
    const uint4* a = reinterpret_cast<const uint4*>(o + r * D);
    const uint4* c = reinterpret_cast<const uint4*>(dout + r * D);
    float acc = 0.f;
#pragma unroll
    for (int v = 0; v < D / 8; ++v) {
      const uint4 x = a[v], y = c[v];
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(xs[e] << 16), __uint_as_float(ys[e] << 16), acc);
        acc = fmaf(__uint_as_float(xs[e] & 0xFFFF0000u), __uint_as_float(ys[e] & 0xFFFF0000u), acc);
      }
    }
    if constexpr (kPk) {   // packed row -> its sample's lse / Dv row
      int lo = 0, hi = seg.n_seg;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (seg.row[mid] <= token) lo = mid;
        else hi = mid;
      }
      const size_t vi = (size_t)h * p.vec_stride + seg.vrow[lo] + (token - seg.row[lo]);
      if (index_ok(vi, p.vec_elems, p.status)) p.dvec[vi] = acc;
      continue;
    }
    int g = 0, slot = token;
    if (p.layout == 0 && slot >= p.q_rows) continue;   // not a query row (joined-text's text queries)
    if (p.layout == 1) {
      g = token % p.k;
      slot = token / p.k;
    } else if (p.layout == 2) {
      const int kk = p.k * p.k, ob = token / kk, rem = token - ob * kk;
      g = rem / p.k;
      slot = ob * p.k + (rem - g * p.k);
    }
    const size_t vi = ((size_t)(b * p.G + g) * p.heads + h) * p.vec_stride + slot;
    if (index_ok(vi, p.vec_elems, p.status)) p.dvec[vi] = acc;
  }
}

// P and dS of one 32-column chunk for one TMEM lane (the thread's row).
//   s, dp: raw scores / dP of the chunk; lse, dv: per-column (kCols) or per-row values.
//   valid: columns [0, valid) of the chunk are real; vis: bit e clear masks column e out.
// Per-column lse / Dv are read four columns at a time (16-byte shared loads, 16-byte aligned
// pointers): every lane reads the same columns, and one broadcast load per four columns instead
// of one per column keeps the shared-memory pipe, which the tensor core's operand reads also
// use, free.
template <bool kPerColumn, bool kMask, int kN>
__device__ __forceinline__ void bwd_chunk_body(const uint32_t (&s)[kN], const uint32_t (&dp)[kN], float sl2,
                                               const float* lse_col, const float* dv_col, float lse_row,
                                               float dv_row, int valid, uint32_t (&pk)[kN / 2],
                                               uint32_t (&dk)[kN / 2], uint32_t vis) {
#pragma unroll
  for (int e = 0; e < kN; e += 4) {
    float l[4], dd[4];
    if constexpr (kPerColumn) {
      const float4 l4 = reinterpret_cast<const float4*>(lse_col)[e >> 2];
      const float4 d4 = reinterpret_cast<const float4*>(dv_col)[e >> 2];
      l[0] = l4.x; l[1] = l4.y; l[2] = l4.z; l[3] = l4.w;
      dd[0] = d4.x; dd[1] = d4.y; dd[2] = d4.z; dd[3] = d4.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        l[u] = lse_row;
        dd[u] = dv_row;
      }
    }
    float pv[4], dsv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      pv[u] = ex2_approx(fmaf(__uint_as_float(s[e + u]), sl2, -l[u]));
      dsv[u] = pv[u] * (__uint_as_float(dp[e + u]) - dd[u]);
      if constexpr (kMask) {
        const bool ok = e + u < valid && ((vis >> (e + u)) & 1u);
        pv[u] = ok ? pv[u] : 0.f;
        dsv[u] = ok ? dsv[u] : 0.f;
      }
    }
    pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
    pk[(e >> 1) + 1] = pack_bf16x2(pv[2], pv[3]);
    dk[e >> 1] = pack_bf16x2(dsv[0], dsv[1]);
    dk[(e >> 1) + 1] = pack_bf16x2(dsv[2], dsv[3]);
  }
}

template <bool kPerColumn, int kN>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&s)[kN], const uint32_t (&dp)[kN], float sl2,
                                          const float* lse_col, const float* dv_col, float lse_row, float dv_row,
                                          int valid, uint32_t (&pk)[kN / 2], uint32_t (&dk)[kN / 2],
                                          uint32_t vis = 0xffffffffu) {
  constexpr uint32_t kAll = kN >= 32 ? 0xffffffffu : ((1u << kN) - 1u);
  if (valid >= kN && (vis & kAll) == kAll)   // every column real and visible: no per-element mask
    bwd_chunk_body<kPerColumn, false, kN>(s, dp, sl2, lse_col, dv_col, lse_row, dv_row, valid, pk, dk, vis);
  else
    bwd_chunk_body<kPerColumn, true, kN>(s, dp, sl2, lse_col, dv_col, lse_row, dv_row, valid, pk, dk, vis);
}

// Writes one 128-row tile's fp32 accumulator row (TMEM columns [col, col + D)) as bf16, scaled.
// part = 0 / 1: only the even / odd 32-column chunks (two warps share a row); -1: all.
template <int D>
__device__ __forceinline__ void bwd_store_row(uint32_t taddr, float scale, __nv_bfloat16* dst, bool live,
                                              int part = -1) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    if (part >= 0 && (cc & 1) != part) continue;
    uint32_t r[32];
    tmem_ld32(taddr + 32 * cc, r);
    tmem_wait_ld();
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * scale, __uint_as_float(r[2 * e + 1]) * scale);
    if (live) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
      for (int v = 0; v < 4; ++v) d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
  }
}

// fp32 variant: the row's D accumulator columns times scale, unrounded
template <int D>
__device__ __forceinline__ void bwd_store_row_f32(uint32_t taddr, float scale, float* dst, bool live,
                                                  int part = -1) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    if (part >= 0 && (cc & 1) != part) continue;
    uint32_t r[32];
    tmem_ld32(taddr + 32 * cc, r);
    tmem_wait_ld();
    if (live) {
      float4* d4 = reinterpret_cast<float4*>(dst + 32 * cc);
#pragma unroll
      for (int v = 0; v < 8; ++v)
        d4[v] = make_float4(__uint_as_float(r[4 * v]) * scale, __uint_as_float(r[4 * v + 1]) * scale,
                            __uint_as_float(r[4 * v + 2]) * scale, __uint_as_float(r[4 * v + 3]) * scale);
    }
  }
}

// ------------------------------------------------------------------------------------------
// dK, dV: one CTA per (sample*set, head, 128-key tile)
// ------------------------------------------------------------------------------------------
// kKeysMajor = true: the kernel's "resident" tiles are K, V and the streamed ones Q, dO.
template <int D, bool kPk = false>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                         const BwdParams p, const __grid_constant__ BwdSegParam<kPk> seg) {
  using C = BwdCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const int B_RES = 0, B_FULL = 1, B_EMPTY = 1 + kStages, B_SFULL = 1 + 2 * kStages, B_PREADY = B_SFULL + 2,
            B_DONE = B_PREADY + 2, B_FIN = B_DONE + 1, B_BUFFREE = B_FIN + 1, B_FIN2 = B_BUFFREE + 2;
  // fused dQ: dS buffer free (dQ product of the tile two back done) [2], dQ product done [2], dQ
  // tensor-memory buffer read out [2], staging tile written, staging tile read by the reduce
  const int B_DSFREE = B_FIN2 + 1, B_DQFULL = B_DSFREE + 2, B_DQTFREE = B_DQFULL + 2, B_STGFULL = B_DQTFREE + 2,
            B_STGFREE = B_STGFULL + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // fused dQ: its tensor-memory buffer (64 columns next to dV at 256), and K, V (32 columns each
  // after dK at 384)
  constexpr uint32_t kColDq = 320, kColK = 448, kColV = 480;
  const int B_KVT = B_STGFREE + 1;   // K and V are in tensor memory

  const BwdUnit un = bwd_unit<kPk>(p, seg, (int)blockIdx.x, false);
  const int tile = un.tile, h = un.h, b = un.b, g = un.g;
  const int n_rows = un.n, rb = un.row_base;   // the set's rows; its first packed row (packed batches)
  const int kv0 = tile * kBT;
  // query tiles i0 .. n_tiles-1 (frame-causal: the first query that may see key kv0 opens the range)
  const int i0 = p.frame_hw ? causal_block_start(kv0, p.text_len, p.frame_hw) / kBT : 0;
  const int nq = (kPk ? un.n_tiles : p.q_tiles) - i0;
  const int q_rows = kPk ? n_rows : p.q_rows;   // query rows of the set (a prefix of its rows)
  const int chan0 = h * D;
  const size_t vec_row = un.vec_row;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_RES), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(B_SFULL + u), 1);
      mbar_init(bar(B_PREADY + u), kDkComputeThreads);
    }
    mbar_init(bar(B_DONE), 1);
    mbar_init(bar(B_FIN), 1);
    mbar_init(bar(B_BUFFREE + 0), 1);
    mbar_init(bar(B_BUFFREE + 1), 1);
    mbar_init(bar(B_FIN2), 1);
    if constexpr (C::kFuseDq) {
      for (int u = 0; u < 2; ++u) mbar_init(bar(B_DSFREE + u), 1);
      mbar_init(bar(B_DQFULL), 1);
      mbar_init(bar(B_DQTFREE), kDkComputeThreads);
      mbar_init(bar(B_STGFULL), kDkComputeThreads);
      mbar_init(bar(B_STGFREE), 1);
    }
    if constexpr (C::kKvTmem || C::kKTmem) mbar_init(bar(B_KVT), kDkComputeThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kDkProdWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  if (warp == kDkMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
  auto sDs = [&](int b) { return sbase + C::kDsOff + (uint32_t)(b * 2 * kChunkBytes); };   // fused dQ: dS^T
  const uint32_t sStg = sbase + C::kStgOff;                                              // fused dQ: staging
  auto sRes = [&](int i) { return sbase + C::kResOff + (uint32_t)(i * C::kTileBytes); };           // K, V
  auto sStr = [&](int s, int i) { return sbase + C::kStageOff + (uint32_t)((2 * s + i) * C::kTileBytes); };  // Q, dO
  auto sVec = [&](int s) { return sbase + C::kVecOff + (uint32_t)(s * C::kVecBytes); };

  if (warp == kDkProdWarp) {
    // ------------------------------------------------------------------ TMA producer
    const bool leader = elect_one_sync();
    int issued = 0;
    if (leader) {
      mbar_arrive_expect_tx(bar(B_RES), 2 * C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c) {
        bwd_load_tile(&tm_k, sRes(0) + c * kChunkBytes, bar(B_RES), p.layout, chan0 + 64 * c, rb + kv0, g, b, p.k);
        bwd_load_tile(&tm_v, sRes(1) + c * kChunkBytes, bar(B_RES), p.layout, chan0 + 64 * c, rb + kv0, g, b, p.k);
      }
    }
    for (int il = 0; il < nq; ++il) {
      const int s = il % kStages, i = i0 + il;
      if (il >= kStages && !bwd_warp_wait(bar(B_EMPTY + s), ((il / kStages) - 1) & 1, wc)) break;
      if (leader) {
        // the tile's lse / Dv slices (skipped, with their bytes, if a debug index check fails)
        const bool vec_ok = index_ok(vec_row + (size_t)i * kBT + kBT - 1, p.vec_elems, p.status);
        mbar_arrive_expect_tx(bar(B_FULL + s), 2 * C::kTileBytes + (vec_ok ? C::kVecBytes : 0));
        for (int c = 0; c < C::kChunks; ++c) {
          bwd_load_tile(&tm_q, sStr(s, 0) + c * kChunkBytes, bar(B_FULL + s), p.layout, chan0 + 64 * c,
                        rb + i * kBT, g, b, p.k);
          bwd_load_tile(&tm_do, sStr(s, 1) + c * kChunkBytes, bar(B_FULL + s), p.layout, chan0 + 64 * c,
                        rb + i * kBT, g, b, p.k);
        }
        if (vec_ok) {
          bulk_load(sVec(s), p.lse + vec_row + (size_t)i * kBT, kBT * 4, bar(B_FULL + s));
          bulk_load(sVec(s) + kBT * 4, p.dvec + vec_row + (size_t)i * kBT, kBT * 4, bar(B_FULL + s));
        }
      }
      issued = il + 1;
    }
    // every load issued lands before the CTA may exit
    mbar_drain(bar(B_RES), 0, p.timeout_ns);
    for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
      mbar_drain(bar(B_FULL + t % kStages), (t / kStages) & 1, p.timeout_ns);
    __syncwarp();
  } else if (warp == kDkMmaWarp || warp == kDkAccWarp) {
    // ------------------------------------------------------------------ MMA issuers
    const bool leader = elect_one_sync();
    constexpr uint32_t idesc_ss = idesc_bf16_f32(kBT, kSub, false);  // M = 128 keys, N = 64 queries, K-major
    constexpr uint32_t idesc_ts = idesc_bf16_f32(kBT, D, true);      // M = 128, N = D, B MN-major
    constexpr uint64_t kTileStep = (uint64_t)(C::kTileBytes >> 4);
    const uint64_t dK = sdesc_sw128(sRes(0), 16, 1024), dV = sdesc_sw128(sRes(1), 16, 1024);
    const uint64_t dQk = sdesc_sw128(sStr(0, 0), 16, 1024);             // Q as K-major B (N = queries)
    const uint64_t dQmn = sdesc_sw128(sStr(0, 0), kChunkBytes, 1024);   // Q as MN-major B (N = channels)
    const uint64_t dOk = sdesc_sw128(sStr(0, 1), 16, 1024);
    const uint64_t dOmn = sdesc_sw128(sStr(0, 1), kChunkBytes, 1024);
    // stage s's tiles sit 2*s tiles after stage 0's
    auto stage_off = [&](int s) { return (uint64_t)(2 * s) * kTileStep; };
    // D_t = A K-major (128 rows x D) times B K-major (128 rows x D)^T
    auto issue_ss = [&](uint32_t d_col, uint64_t a0, uint64_t b0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
        if (leader) mma_ss(tmem + d_col, a0 + off, b0 + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
    };
    // D_t (+)= A (tensor memory, packed bf16, 128 x 64) times B MN-major (64 rows x D)
    auto issue_ts = [&](uint32_t d_col, uint32_t a_col, uint64_t b0, bool acc) {
#pragma unroll
      for (int kk = 0; kk < kSub / 16; ++kk)
        if (leader) mma_ts(tmem + d_col, tmem + a_col + packed_col_dk(kk), b0 + (uint64_t)(128 * kk), idesc_ts,
                           (acc || kk > 0) ? 1u : 0u);
    };
    // Sub-tile t = 2i + hh is rows 64hh .. 64hh+63 of query tile i, in score buffer t & 1.
    // Warp 9 issues S^T / dP^T of sub-tile t once warp 10's products of sub-tile t-2 (the last
    // readers of buffer t & 1) have completed; warp 10 issues dV / dK of sub-tile t once the
    // compute warps have written P^T / dS^T.
    const int n_sub = 2 * nq;
    // D_t = A (tensor memory: K or V, packed channel pairs, 8 columns per 16 channels) times B
    // K-major (64 query rows x D)^T
    auto issue_ts_kv = [&](uint32_t d_col, uint32_t a_col, uint64_t b0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
        if (leader) mma_ts(tmem + d_col, tmem + a_col + 8u * kk, b0 + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
    };
    // fused dQ: dQ_i = dS_i K, A = dS_i^T from shared memory (MN-major: rows = keys, queries
    // contiguous in two 64-query SW128 chunks 16 KB apart), B = the resident K (MN-major, N = D)
    constexpr uint32_t idesc_dq = idesc_bf16_f32(kBT, D, true, true);
    const uint64_t dKres_mn = sdesc_sw128(sRes(0), kChunkBytes, 1024);
    auto issue_scores = [&](int t) {   // S^T and dP^T of sub-tile t into score buffer t & 1
      const int hh = t & 1, s = (t >> 1) % kStages;
      const uint64_t sub = stage_off(s) + (hh ? kSubDescOff : 0);
      if constexpr (C::kKvTmem) {
        issue_ts_kv(col_s(t & 1), kColK, dQk + sub);    // S^T = K Q_sub^T
        issue_ts_kv(col_dp(t & 1), kColV, dOk + sub);   // dP^T = V dO_sub^T
      } else if constexpr (C::kKTmem) {
        issue_ts_kv(col_s(t & 1), kColK, dQk + sub);
        issue_ss(col_dp(t & 1), dV, dOk + sub);
      } else {
        issue_ss(col_s(t & 1), dK, dQk + sub);
        issue_ss(col_dp(t & 1), dV, dOk + sub);
      }
      if (leader) tc_commit(bar(B_SFULL + (t & 1)));
    };
    auto issue_accum = [&](int t) {   // dV, dK of sub-tile t from score buffer t & 1
      const int hh = t & 1, s = (t >> 1) % kStages;
      const uint64_t sub = stage_off(s) + (hh ? kSubDescOff : 0);
      issue_ts(kColAcc0, col_s(t & 1), dOmn + sub, t > 0);    // dV += P^T dO_sub
      issue_ts(C::kColDk, col_dp(t & 1), dQmn + sub, t > 0);   // dK += dS^T Q_sub
    };
    auto issue_dq = [&](int i) -> bool {   // dQ of local tile i, after its second sub-tile
      const int b = i & 1;
      // the tensor-memory buffer's previous tile (i - 1) has been read out
      if (i >= 1 && !bwd_warp_wait(bar(B_DQTFREE), (i - 1) & 1, wc)) return false;
      tc_fence_after();
      const uint64_t da = sdesc_sw128(sDs(b), kChunkBytes, 1024);
#pragma unroll
      for (int kk = 0; kk < kBT / 16; ++kk)   // 16 keys (two 8-row groups, 2 KB) per step
        if (leader) mma_ss(tmem + kColDq, da + (uint64_t)(128 * kk), dKres_mn + (uint64_t)(128 * kk), idesc_dq,
                           kk > 0 ? 1u : 0u);
      if (leader) tc_commit(bar(B_DQFULL));
      if (leader) tc_commit(bar(B_DSFREE + b));
      return true;
    };
    if (C::kOneIssuer && warp == kDkMmaWarp) {
      // one thread issues every product: the first two sub-tiles' scores, then per sub-tile t its
      // dV and dK, the scores of t + 2 into the buffer those just read (the tensor pipe runs one
      // thread's products in order), and after a tile's second sub-tile its dQ
      bool ok = bwd_warp_wait(bar(B_RES), 0, wc);
      if constexpr (C::kKvTmem || C::kKTmem) ok = ok && bwd_warp_wait(bar(B_KVT), 0, wc);
      if (ok && n_sub > 0) ok = bwd_warp_wait(bar(B_FULL + 0), 0, wc);
      for (int t = 0; ok && t < n_sub && t < 2; ++t) {
        tc_fence_after();
        issue_scores(t);
      }
      for (int t = 0; ok && t < n_sub; ++t) {
        const int i = t >> 1, hh = t & 1, s = i % kStages;
        if (!bwd_warp_wait(bar(B_PREADY + (t & 1)), (t >> 1) & 1, wc)) break;
        tc_fence_after();
        issue_accum(t);
        if (hh == 1 && leader) tc_commit(bar(B_EMPTY + s));   // tile i's Q and dO are consumed
        const int tn = t + 2;
        if (tn < n_sub) {
          const int in = tn >> 1;
          if ((tn & 1) == 0 && !bwd_warp_wait(bar(B_FULL + in % kStages), (in / kStages) & 1, wc)) break;
          tc_fence_after();
          issue_scores(tn);
        }
        if constexpr (C::kFuseDq) {
          if (hh == 1 && !issue_dq(i)) break;
        }
        if (t == n_sub - 1 && leader) tc_commit(bar(B_DONE));
      }
      if (leader) tc_commit(bar(B_FIN));
      mbar_drain(bar(B_FIN), 0, p.timeout_ns);
    } else if (C::kOneIssuer) {
      // (the accumulating-product warp has nothing to issue when one thread issues everything)
    } else if (warp == kDkMmaWarp) {
      bool ok = bwd_warp_wait(bar(B_RES), 0, wc);
      if constexpr (C::kKvTmem || C::kKTmem) ok = ok && bwd_warp_wait(bar(B_KVT), 0, wc);
      for (int t = 0; ok && t < n_sub; ++t) {
        const int i = t >> 1, hh = t & 1, s = i % kStages;
        if (hh == 0 && !bwd_warp_wait(bar(B_FULL + s), (i / kStages) & 1, wc)) break;
        if (t >= 2 && !bwd_warp_wait(bar(B_BUFFREE + (t & 1)), ((t - 2) >> 1) & 1, wc)) break;
        tc_fence_after();
        issue_scores(t);
      }
      if (leader) tc_commit(bar(B_FIN));
      mbar_drain(bar(B_FIN), 0, p.timeout_ns);
    } else {
      for (int t = 0; t < n_sub; ++t) {
        const int i = t >> 1, hh = t & 1, s = i % kStages;
        if (!bwd_warp_wait(bar(B_PREADY + (t & 1)), (t >> 1) & 1, wc)) break;
        tc_fence_after();
        issue_accum(t);
        if (leader) tc_commit(bar(B_BUFFREE + (t & 1)));      // buffer t & 1 may be overwritten
        if (hh == 1 && leader) tc_commit(bar(B_EMPTY + s));   // both halves of tile i consumed
        if constexpr (C::kFuseDq) {
          if (hh == 1 && !issue_dq(i)) break;
        }
        if (t == n_sub - 1 && leader) tc_commit(bar(B_DONE));
      }
      if (leader) tc_commit(bar(B_FIN2));
      mbar_drain(bar(B_FIN2), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == kDkRedWarp) {
    // ------------------------------------------------------------------ fused dQ: bulk reduce-add
    // of each query tile's fp32 dQ (staged in shared memory by the compute warps) into the
    // accumulator rows of this (sample*set, head); the staging tile is released once read
    if constexpr (C::kFuseDq) {
      const bool leader = elect_one_sync();
      for (int il = 0; il < nq; ++il) {
        if (!bwd_warp_wait(bar(B_STGFULL), il & 1, wc)) break;
        const size_t row0 = vec_row + (size_t)(i0 + il) * kBT;
        if (leader && index_ok((row0 + kBT) * D - 1, p.dq_acc_elems, p.status)) {
          bulk_reduce_add_f32(p.dq_acc + row0 * D, sStg, kBT * D * 4);
          bulk_wait_read();
        }
        __syncwarp();
        if (leader) mbar_arrive(bar(B_STGFREE));
      }
      if (leader) bulk_wait_all();
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ compute warps 0-7
    constexpr int kN = kDkCols;                              // query columns of this warp per sub-tile
    constexpr int kGroups = kSub / kN;                       // column groups of a lane quarter
    const int quarter = warp & 3, cg = warp >> 2;            // lane quarter, column group
    const int row = quarter * 32 + lane;                    // key row = tensor-memory lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    const int kstart = p.frame_hw ? causal_block_start(kv0 + row, p.text_len, p.frame_hw) : 0;   // its block's start
    // fused dQ: reads this warp's 32 x kN block (query rows of its lane quarter, columns kN cg ..)
    // of dQ of local tile ix out of tensor memory and writes it into the staging tile: row-major
    // fp32, with the eight 16-byte chunks of each 32-float half row permuted by XOR (row & 7) so
    // that a warp's stores spread over all banks.  The accumulator rows keep that permutation
    // (it depends on the row alone, so every key tile's contribution lands on the same element);
    // the finalize kernel undoes it.
    auto drain_dq = [&](int ix) -> bool {
      if (!bwd_warp_wait(bar(B_DQFULL), ix & 1, wc)) return false;
      tc_fence_after();
      uint32_t r[kN];
      tmem_ldn<kN>(tmem + lane_base + kColDq + (uint32_t)(kN * cg), r);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_DQTFREE));
      if (ix >= 1 && !bwd_warp_wait(bar(B_STGFREE), (ix - 1) & 1, wc)) return false;
      // this warp's floats kN cg .. kN cg + kN - 1: half row (kN cg) / 32, its chunks from (kN cg % 32) / 4
      const uint32_t rowb = sStg + (uint32_t)(row * D * 4 + ((kN * cg) / 32) * 128);
      const int c0 = ((kN * cg) % 32) / 4;
#pragma unroll
      for (int c = 0; c < kN / 4; ++c) {
        const uint32_t pc = (uint32_t)((c0 + c) ^ (row & 7));
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowb + 16u * pc), "r"(r[4 * c]),
                     "r"(r[4 * c + 1]), "r"(r[4 * c + 2]), "r"(r[4 * c + 3])
                     : "memory");
      }
      fence_proxy_async_smem();   // visible to the bulk reduce issued after STGFULL
      mbar_arrive(bar(B_STGFULL));
      return true;
    };
    if constexpr (C::kKvTmem) {
      // K (column groups 0, 1) or V (2, 3): this row's channels 32 (cg & 1) .. + 31, i.e. its
      // 16-byte SW128 chunks 4 (cg & 1) .. + 3, as packed pairs into tensor-memory columns
      // 16 (cg & 1) .. + 15 of the K or V block
      ok = bwd_warp_wait(bar(B_RES), 0, wc);
      if (ok) {
        const uint32_t src = sRes(cg >> 1) + (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
        uint32_t r[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t c = (uint32_t)((4 * (cg & 1) + v) ^ (row & 7));
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(r[4 * v]), "=r"(r[4 * v + 1]), "=r"(r[4 * v + 2]), "=r"(r[4 * v + 3])
                       : "r"(src + 16u * c));
        }
        tmem_st16(tmem + lane_base + ((cg >> 1) ? kColV : kColK) + 16u * (uint32_t)(cg & 1), r);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_KVT));
      }
    } else if constexpr (C::kKTmem) {
      // K only (d = 96): column groups 0 .. 2 take this row's 16-byte chunks 4 cg .. 4 cg + 3
      // (channels 32 cg ..; chunk c lies in SW128 block c / 8) into columns 16 cg .. + 15
      ok = bwd_warp_wait(bar(B_RES), 0, wc);
      if (ok) {
        if (cg < 3) {
          uint32_t r[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int c = 4 * cg + v;
            const uint32_t src = sRes(0) + (uint32_t)((c >> 3) * kChunkBytes + (row >> 3) * 1024 + (row & 7) * 128) +
                                 16u * (uint32_t)((c & 7) ^ (row & 7));
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(r[4 * v]), "=r"(r[4 * v + 1]), "=r"(r[4 * v + 2]), "=r"(r[4 * v + 3])
                         : "r"(src));
          }
          tmem_st16(tmem + lane_base + kColK + 16u * (uint32_t)cg, r);
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar(B_KVT));
      }
    }
    for (int t = 0; ok && t < 2 * nq; ++t) {
      const int il = t >> 1, i = i0 + il, hh = t & 1, bb = t & 1;
      if (!bwd_warp_wait(bar(B_SFULL + bb), (t >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const float* vec = reinterpret_cast<const float*>(smem + C::kVecOff + (il % kStages) * C::kVecBytes) +
                         kSub * hh + kN * cg;
      const int qa = i * kBT + kSub * hh + kN * cg;   // this warp's first query column
      // a key row past the set's end (zero-fill, or in a packed batch the next sample's keys) gets
      // no valid column: its P and dS are zero, so the fused dQ product sums real keys only
      const int valid_q = (kv0 + row < n_rows) ? q_rows - qa : 0;
      const uint32_t vis = p.frame_hw ? causal_columns(qa, kstart) : 0xffffffffu;
      const uint32_t tS = tmem + lane_base + col_s(bb) + (uint32_t)(kN * cg);
      const uint32_t tP = tmem + lane_base + col_dp(bb) + (uint32_t)(kN * cg);
      uint32_t s[kN], dp[kN];
      tmem_ldn<kN>(tS, s);
      tmem_ldn<kN>(tP, dp);
      tmem_wait_ld();
      uint32_t pk[kN / 2], dk[kN / 2];
      bwd_chunk<true, kN>(s, dp, p.scale_log2, vec, vec + kBT, 0.f, 0.f, valid_q, pk, dk, vis);
      // P^T and dS^T over this warp's consumed S^T / dP^T columns (its first kN / 2)
      tmem_stn<kN / 2>(tS, pk);
      tmem_stn<kN / 2>(tP, dk);
      if constexpr (C::kFuseDq) {
        // dS^T row (this key) for queries 64hh + kN cg .. into the dS buffer of tile il: SW128
        // chunk hh, 16-byte column c = (kN / 8) cg + v XOR (row & 7), 8-row groups 1 KB apart
        const int b = il & 1;
        if (hh == 0 && il >= 2 && !bwd_warp_wait(bar(B_DSFREE + b), ((il >> 1) - 1) & 1, wc)) { ok = false; break; }
        const uint32_t base = sDs(b) + (uint32_t)(hh * kChunkBytes) + (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
#pragma unroll
        for (int v = 0; v < kN / 8; ++v) {
          const uint32_t c = (uint32_t)(((kN / 8) * cg + v) ^ (row & 7));
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + 16u * c), "r"(dk[4 * v]),
                       "r"(dk[4 * v + 1]), "r"(dk[4 * v + 2]), "r"(dk[4 * v + 3])
                       : "memory");
        }
        fence_proxy_async_smem();   // visible to the dQ product issued after P_ready
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PREADY + bb));
      if constexpr (C::kFuseDq) {
        if (hh == 1 && il >= 1 && !drain_dq(il - 1)) { ok = false; break; }
      }
    }
    if constexpr (C::kFuseDq) {
      if (ok && nq > 0) ok = drain_dq(nq - 1);
    }
    if (ok && bwd_warp_wait(bar(B_DONE), 0, wc)) {
      tc_fence_after();
      const int j = kv0 + row;
      const bool live = j < n_rows;
      const int token = rb + bwd_slot_token(p.layout, live ? j : 0, g, p.k);
      const size_t off = (((size_t)b * p.N + token) * p.heads + h) * D;
      const bool store = live && index_ok(off + D - 1, p.elems, p.status);
      // the first half of a quarter's column groups writes dV, the second dK; with two groups
      // per half they split the 32-column chunks by parity
      const bool is_dk = cg >= kGroups / 2;
      const int part = kGroups > 2 ? (cg & 1) : -1;
      if (p.dk32) {
        if (!is_dk) bwd_store_row_f32<D>(tmem + lane_base + kColAcc0, 1.f, p.dv32 + off, store, part);
        else bwd_store_row_f32<D>(tmem + lane_base + C::kColDk, p.scale, p.dk32 + off, store, part);
      } else if (!is_dk) {
        bwd_store_row<D>(tmem + lane_base + kColAcc0, 1.f, p.dv + off, store, part);
      } else {
        bwd_store_row<D>(tmem + lane_base + C::kColDk, p.scale, p.dk + off, store, part);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kDkMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// dQ: one CTA per (sample*set, head, 128-query tile)
// ------------------------------------------------------------------------------------------
template <int D, bool kPk = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const BwdParams p, const __grid_constant__ BwdSegParam<kPk> seg) {
  using C = BwdCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const int B_RES = 0, B_FULL = 1, B_EMPTY = 1 + kStages, B_SFULL = 1 + 2 * kStages, B_PREADY = B_SFULL + 2,
            B_DONE = B_PREADY + 2, B_FIN = B_DONE + 1, B_BUFFREE = B_FIN + 1, B_FIN2 = B_BUFFREE + 2;
  const int B_QT = B_FIN2 + 1;   // Q and dO are in tensor memory
  // Q and dO also sit in tensor memory (packed channel pairs, query = lane) after the dQ
  // accumulator, so the score products S = Q K^T and dP = dO V^T read only K / V from shared memory
  constexpr uint32_t kColQ = 384, kColDo = 448;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // frame-causal: a head's query tiles in reverse, so that those seeing the most keys start first
  const BwdUnit un = bwd_unit<kPk>(p, seg, (int)blockIdx.x, p.frame_hw != 0, kPk ? 0 : p.q_tiles);
  const int tile = un.tile, h = un.h, b = un.b, g = un.g;
  const int n_rows = un.n, rb = un.row_base;   // the set's rows; its first packed row (packed batches)
  const int q_rows = kPk ? n_rows : p.q_rows;  // its query rows
  const int q0 = tile * kBT;
  // key tiles 0 .. nk-1 (frame-causal: up to the last key the tile's last query may see)
  const int nk = p.frame_hw
                     ? (min(n_rows, causal_limit(min(q0 + kBT, n_rows) - 1, p.text_len, p.frame_hw)) + kBT - 1) / kBT
                     : un.n_tiles;
  const int chan0 = h * D;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_RES), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(B_SFULL + u), 1);
      mbar_init(bar(B_PREADY + u), kComputeThreads);
    }
    mbar_init(bar(B_DONE), 1);
    mbar_init(bar(B_FIN), 1);
    mbar_init(bar(B_BUFFREE + 0), 1);
    mbar_init(bar(B_BUFFREE + 1), 1);
    mbar_init(bar(B_FIN2), 1);
    mbar_init(bar(B_QT), kComputeThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProdWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
  auto sRes = [&](int i) { return sbase + C::kResOff + (uint32_t)(i * C::kTileBytes); };           // Q, dO
  auto sStr = [&](int s, int i) { return sbase + C::kStageOff + (uint32_t)((2 * s + i) * C::kTileBytes); };  // K, V

  if (warp == kProdWarp) {
    const bool leader = elect_one_sync();
    int issued = 0;
    if (leader) {
      mbar_arrive_expect_tx(bar(B_RES), 2 * C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c) {
        bwd_load_tile(&tm_q, sRes(0) + c * kChunkBytes, bar(B_RES), p.layout, chan0 + 64 * c, rb + q0, g, b, p.k);
        bwd_load_tile(&tm_do, sRes(1) + c * kChunkBytes, bar(B_RES), p.layout, chan0 + 64 * c, rb + q0, g, b, p.k);
      }
    }
    for (int j = 0; j < nk; ++j) {
      const int s = j % kStages;
      if (j >= kStages && !bwd_warp_wait(bar(B_EMPTY + s), ((j / kStages) - 1) & 1, wc)) break;
      if (leader) {
        mbar_arrive_expect_tx(bar(B_FULL + s), 2 * C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c) {
          bwd_load_tile(&tm_k, sStr(s, 0) + c * kChunkBytes, bar(B_FULL + s), p.layout, chan0 + 64 * c,
                        rb + j * kBT, g, b, p.k);
          bwd_load_tile(&tm_v, sStr(s, 1) + c * kChunkBytes, bar(B_FULL + s), p.layout, chan0 + 64 * c,
                        rb + j * kBT, g, b, p.k);
        }
      }
      issued = j + 1;
    }
    mbar_drain(bar(B_RES), 0, p.timeout_ns);
    for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
      mbar_drain(bar(B_FULL + t % kStages), (t / kStages) & 1, p.timeout_ns);
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kAccWarp) {
    const bool leader = elect_one_sync();
    constexpr uint32_t idesc_ss = idesc_bf16_f32(kBT, kSub, false);  // M = 128 queries, N = 64 keys
    constexpr uint32_t idesc_ts = idesc_bf16_f32(kBT, D, true);
    constexpr uint64_t kTileStep = (uint64_t)(C::kTileBytes >> 4);
    const uint64_t dQ = sdesc_sw128(sRes(0), 16, 1024), dO = sdesc_sw128(sRes(1), 16, 1024);
    const uint64_t dKk = sdesc_sw128(sStr(0, 0), 16, 1024);             // K as K-major B (N = keys)
    const uint64_t dKmn = sdesc_sw128(sStr(0, 0), kChunkBytes, 1024);   // K as MN-major B (N = channels)
    const uint64_t dVk = sdesc_sw128(sStr(0, 1), 16, 1024);
    auto stage_off = [&](int s) { return (uint64_t)(2 * s) * kTileStep; };
    auto issue_ss = [&](uint32_t d_col, uint64_t a0, uint64_t b0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
        if (leader) mma_ss(tmem + d_col, a0 + off, b0 + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
    };
    auto issue_ts = [&](uint32_t d_col, uint32_t a_col, uint64_t b0, bool acc) {
#pragma unroll
      for (int kk = 0; kk < kSub / 16; ++kk)
        if (leader) mma_ts(tmem + d_col, tmem + a_col + packed_col(kk), b0 + (uint64_t)(128 * kk), idesc_ts,
                           (acc || kk > 0) ? 1u : 0u);
    };
    // sub-tile t = 2j + hh: keys 64hh .. 64hh+63 of key tile j, score buffer t & 1; the two
    // issuing warps split as in the dK/dV kernel
    // D_t = A (tensor memory: Q or dO, 8 columns per 16 channels) times B K-major (64 keys x D)^T
    auto issue_ts_q = [&](uint32_t d_col, uint32_t a_col, uint64_t b0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
        if (leader) mma_ts(tmem + d_col, tmem + a_col + 8u * kk, b0 + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
    };
    (void)dQ;
    (void)dO;
    const int n_sub = 2 * nk;
    auto issue_scores = [&](int t) {   // S and dP of sub-tile t into score buffer t & 1
      const int hh = t & 1, s = (t >> 1) % kStages;
      const uint64_t sub = stage_off(s) + (hh ? kSubDescOff : 0);
      issue_ts_q(col_s(t & 1), kColQ, dKk + sub);     // S = Q K_sub^T
      issue_ts_q(col_dp(t & 1), kColDo, dVk + sub);   // dP = dO V_sub^T
      if (leader) tc_commit(bar(B_SFULL + (t & 1)));
    };
    auto issue_accum = [&](int t) {   // dQ += dS K_sub, dS from score buffer t & 1
      const int hh = t & 1, s = (t >> 1) % kStages;
      issue_ts(kColAcc0, col_dp(t & 1), dKmn + stage_off(s) + (hh ? kSubDescOff : 0), t > 0);
    };
    // (one thread issuing both, as in the dK/dV kernel, measured -5 % at d = 96 and -0.6 % at
    // d = 128 here)
    if (warp == kMmaWarp) {
      bool ok = bwd_warp_wait(bar(B_RES), 0, wc) && bwd_warp_wait(bar(B_QT), 0, wc);
      for (int t = 0; ok && t < n_sub; ++t) {
        const int j = t >> 1, hh = t & 1, s = j % kStages;
        if (hh == 0 && !bwd_warp_wait(bar(B_FULL + s), (j / kStages) & 1, wc)) break;
        if (t >= 2 && !bwd_warp_wait(bar(B_BUFFREE + (t & 1)), ((t - 2) >> 1) & 1, wc)) break;
        tc_fence_after();
        issue_scores(t);
      }
      if (leader) tc_commit(bar(B_FIN));
      mbar_drain(bar(B_FIN), 0, p.timeout_ns);
    } else {
      for (int t = 0; t < n_sub; ++t) {
        const int j = t >> 1, hh = t & 1, s = j % kStages;
        if (!bwd_warp_wait(bar(B_PREADY + (t & 1)), (t >> 1) & 1, wc)) break;
        tc_fence_after();
        issue_accum(t);
        if (leader) tc_commit(bar(B_BUFFREE + (t & 1)));
        if (hh == 1 && leader) tc_commit(bar(B_EMPTY + s));
        if (t == n_sub - 1 && leader) tc_commit(bar(B_DONE));
      }
      if (leader) tc_commit(bar(B_FIN2));
      mbar_drain(bar(B_FIN2), 0, p.timeout_ns);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;                    // query row = tensor-memory lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int qs = q0 + row;
    const bool live = qs < q_rows;
    const size_t vec_row = un.vec_row;
    const bool vin = live && index_ok(vec_row + qs, p.vec_elems, p.status);
    const float lse_r = vin ? p.lse[vec_row + qs] : 0.f;
    const float dv_r = vin ? p.dvec[vec_row + qs] : 0.f;
    // Q (half 0) or dO (half 1): this row's D channels, SW128 chunks of 64 channels, as packed
    // pairs into the tensor-memory block
    bool ok = bwd_warp_wait(bar(B_RES), 0, wc);
    if (ok) {
      uint32_t r[D / 2];
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {   // 16-byte chunk c: channels 8c .. 8c + 7
        const uint32_t src = sRes(half) + (uint32_t)((c >> 3) * kChunkBytes + (row >> 3) * 1024 + (row & 7) * 128) +
                             16u * (uint32_t)((c & 7) ^ (row & 7));
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r[4 * c]), "=r"(r[4 * c + 1]), "=r"(r[4 * c + 2]), "=r"(r[4 * c + 3])
                     : "r"(src));
      }
      const uint32_t dst = tmem + lane_base + (half ? kColDo : kColQ);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tmem_st32(dst + 32u * c, *reinterpret_cast<const uint32_t(*)[32]>(&r[32 * c]));
      if constexpr (D % 64) tmem_st16(dst + 32u * (D / 64), *reinterpret_cast<const uint32_t(*)[16]>(&r[32 * (D / 64)]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_QT));
    }
    const int klim = p.frame_hw ? min(n_rows, causal_limit(qs, p.text_len, p.frame_hw)) : n_rows;   // keys it sees
    for (int t = 0; ok && t < 2 * nk; ++t) {
      const int j = t >> 1, hh = t & 1, bb = t & 1;
      if (!bwd_warp_wait(bar(B_SFULL + bb), (t >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const int valid_k = klim - (j * kBT + kSub * hh + 32 * half);   // of this warp's 32 key columns
      const uint32_t tS = tmem + lane_base + col_s(bb) + 32 * half, tP = tmem + lane_base + col_dp(bb) + 32 * half;
      uint32_t s[32], dp[32];
      tmem_ld32(tS, s);
      tmem_ld32(tP, dp);
      tmem_wait_ld();
      uint32_t pk[16], dk[16];
      bwd_chunk<false>(s, dp, p.scale_log2, nullptr, nullptr, lse_r, dv_r, live ? valid_k : 0, pk, dk);
      tmem_st16(tP, dk);    // dS over this warp's consumed dP columns
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PREADY + bb));
    }
    if (ok && bwd_warp_wait(bar(B_DONE), 0, wc)) {
      tc_fence_after();
      const int token = rb + bwd_slot_token(p.layout, live ? qs : 0, g, p.k);
      const size_t off = (((size_t)b * p.N + token) * p.heads + h) * D;
      const bool store = live && index_ok(off + D - 1, p.elems, p.status);
      bwd_store_row<D>(tmem + lane_base + kColAcc0, p.scale, p.dq + off, store, half);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// fused dQ: dq = bf16(scale * dq_acc), from the accumulator's set-slot rows to natural token order
// ------------------------------------------------------------------------------------------
template <int D, bool kPk = false>
__global__ void __launch_bounds__(256) attn_bwd_dq_finalize_kernel(const BwdParams p, long long rows,
                                                                   const __grid_constant__ BwdSegParam<kPk> seg) {
  constexpr int V = D / 8;   // 16-byte output vectors (8 channels) per row
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < rows * V;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long r = idx / V;
    const int v = (int)(idx - r * V);
    int slot, h, token, b = 0;
    size_t vrow;   // the (set, head)'s first accumulator row
    if constexpr (kPk) {   // r = packed row * heads + h
      h = (int)(r % p.heads);
      token = (int)(r / p.heads);
      int lo = 0, hi = seg.n_seg;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (seg.row[mid] <= token) lo = mid;
        else hi = mid;
      }
      slot = token - seg.row[lo];
      vrow = (size_t)h * p.vec_stride + seg.vrow[lo];
    } else {
      slot = (int)(r % p.q_rows);
      const long long bh = r / p.q_rows;
      h = (int)(bh % p.heads);
      const int bg = (int)(bh / p.heads);
      b = bg / p.G;
      vrow = ((size_t)bg * p.heads + h) * p.vec_stride;
      token = bwd_slot_token(p.layout, slot, bg % p.G, p.k);
    }
    // logical 16-byte chunks 2v, 2v + 1 of the row; within each 32-float half (8 chunks) the
    // dK/dV kernel stored chunk c at c ^ (slot & 7)
    const int c0 = 2 * v, hc = c0 & ~7;
    const size_t rbase = (vrow + slot) * D;
    const size_t src = rbase + 4 * (hc + ((c0 & 7) ^ (slot & 7)));
    const size_t src1 = rbase + 4 * (hc + (((c0 + 1) & 7) ^ (slot & 7)));
    const size_t dst = (((size_t)b * p.N + token) * p.heads + h) * D + 8 * v;
    if (!index_ok(rbase + D - 1, p.dq_acc_elems, p.status) || !index_ok(dst + 7, p.elems, p.status)) continue;
    const float4 x = *reinterpret_cast<const float4*>(p.dq_acc + src);
    const float4 y = *reinterpret_cast<const float4*>(p.dq_acc + src1);
    const float sc = p.scale;
    *reinterpret_cast<uint4*>(p.dq + dst) =
        make_uint4(pack_bf16x2(x.x * sc, x.y * sc), pack_bf16x2(x.z * sc, x.w * sc), pack_bf16x2(y.x * sc, y.y * sc),
                   pack_bf16x2(y.z * sc, y.w * sc));
  }
}

template <int D, bool kPk = false>
int launch_bwd_d(const void* o, const void* dout, const CUtensorMap& tq, const CUtensorMap& tk,
                 const CUtensorMap& tv, const CUtensorMap& tdo, const BwdParams& p, long long rows, long long ctas,
                 cudaStream_t stream, const BwdSegParam<kPk>& seg = BwdSegParam<kPk>{}) {
  constexpr int smem = BwdCfg<D>::kSmemBytes;
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(attn_bwd_dkdv_kernel<D, kPk>), smem,
                            "attn_bwd_dkdv_kernel");
  if (rc || (rc = ensure_smem_attr(reinterpret_cast<const void*>(attn_bwd_dq_kernel<D, kPk>), smem,
                                   "attn_bwd_dq_kernel")))
    return rc;
  const long long dblocks = std::min<long long>((rows + 255) / 256, (long long)device_sm_count() * 16);
  attn_bwd_dvec_kernel<D, kPk><<<(unsigned)dblocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                                      static_cast<const __nv_bfloat16*>(dout), p, rows,
                                                                      seg);
  rc = check_launch("attn_bwd_dvec_kernel");
  if (rc) return rc;
  if (ctas <= 0) return OSP_OK;   // no rows at all
  attn_bwd_dkdv_kernel<D, kPk><<<(unsigned)ctas, BwdCfg<D>::kThreads, smem, stream>>>(tq, tk, tv, tdo, p, seg);
  if ((rc = check_launch("attn_bwd_dkdv_kernel"))) return rc;
  if constexpr (BwdCfg<D>::kFuseDq) {
    // (sample*set, head, query slot) rows: B * G * heads * q_rows (all rows unless a prefix)
    const long long qrows = kPk ? rows : rows / p.n * p.q_rows;
    const long long fblocks = std::min<long long>((qrows * (D / 8) + 255) / 256, (long long)device_sm_count() * 16);
    if (fblocks > 0)
      attn_bwd_dq_finalize_kernel<D, kPk><<<(unsigned)fblocks, 256, 0, stream>>>(p, qrows, seg);
    return check_launch("attn_bwd_dq_finalize_kernel");
  }
  const long long dq_ctas = kPk ? ctas : ctas / p.n_tiles * p.q_tiles;   // query tiles
  attn_bwd_dq_kernel<D, kPk><<<(unsigned)dq_ctas, kBwdThreads, smem, stream>>>(tq, tk, tv, tdo, p, seg);
  return check_launch("attn_bwd_dq_kernel");
}

}  // namespace

int attention_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, const osp_shape& s, int layout,
                              int sparse_k, float scale, cudaStream_t stream, bool frame_causal,
                              int causal_block, int q_limit, bool dkdv_f32) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  const int N = s.text_len + s.T * s.H * s.W;
  const int G = (layout == 0) ? 1 : sparse_k;
  const int n = N / G;
  BwdParams p{};
  p.n = n;
  p.N = N;
  p.heads = s.heads;
  p.G = G;
  p.k = (layout == 0) ? 1 : sparse_k;
  p.layout = layout;
  p.n_tiles = (n + kBT - 1) / kBT;
  // queries: all n rows of each set, or (dense layout) its first q_limit rows
  p.q_rows = (layout == 0 && q_limit >= 0 && q_limit < n) ? q_limit : n;
  p.q_tiles = (p.q_rows + kBT - 1) / kBT;
  p.vec_stride = p.q_tiles * kBT;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scale = scale;
  p.lse = lse;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  if (dkdv_f32) {
    p.dk32 = static_cast<float*>(dk);
    p.dv32 = static_cast<float*>(dv);
  } else {
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
  }
  p.status = status;
  p.timeout_ns = wait_timeout_ns();
  p.elems = (unsigned long long)s.B * N * s.heads * s.head_dim / bounds_check_divisor();
  p.frame_hw = frame_causal ? (causal_block > 0 ? causal_block : s.H * s.W) : 0;
  p.text_len = s.text_len;
  p.vec_elems = (unsigned long long)s.B * G * s.heads * p.vec_stride / bounds_check_divisor();
  const long long ctas = (long long)p.n_tiles * s.heads * s.B * G;
  if (ctas > (1LL << 30)) return set_error(OSP_ERR_UNSUPPORTED, "%lld backward work units is too many", ctas);
  CUtensorMap tq, tk, tv, tdo;
  int rc;
  if ((rc = make_attn_tmap(&tq, q, s, N, layout, p.k)) != OSP_OK) return rc;
  if ((rc = make_attn_tmap(&tk, k, s, N, layout, p.k)) != OSP_OK) return rc;
  if ((rc = make_attn_tmap(&tv, v, s, N, layout, p.k)) != OSP_OK) return rc;
  if ((rc = make_attn_tmap(&tdo, dout, s, N, layout, p.k)) != OSP_OK) return rc;
  // Dv scratch, [B*G][heads][vec_stride] fp32, from the library's stream-ordered pool; cleared so
  // that the padding slots past n hold zeros
  const size_t vec_bytes = (size_t)s.B * G * s.heads * p.vec_stride * sizeof(float);
  void* ws = nullptr;
  cudaMemPool_t pool = workspace_pool();
  if (!pool || cudaMallocFromPoolAsync(&ws, vec_bytes, pool, stream) != cudaSuccess)
    return set_error(OSP_ERR_CUDA, "stream-ordered workspace allocation (%zu bytes) failed", vec_bytes);
  if (cudaMemsetAsync(ws, 0, vec_bytes, stream) != cudaSuccess) {
    cudaFreeAsync(ws, stream);
    return set_error(OSP_ERR_CUDA, "clearing the backward workspace failed");
  }
  p.dvec = static_cast<float*>(ws);
  // fused dQ (d = 64): the fp32 dQ accumulator [B*G][heads][vec_stride][D], zeroed
  void* acc = nullptr;
  if (s.head_dim == 64 && BwdCfg<64>::kFuseDq) {
    const size_t acc_bytes = (size_t)s.B * G * s.heads * p.vec_stride * s.head_dim * sizeof(float);
    if (cudaMallocFromPoolAsync(&acc, acc_bytes, pool, stream) != cudaSuccess) {
      cudaFreeAsync(ws, stream);
      return set_error(OSP_ERR_CUDA, "stream-ordered workspace allocation (%zu bytes) failed", acc_bytes);
    }
    if (cudaMemsetAsync(acc, 0, acc_bytes, stream) != cudaSuccess) {
      cudaFreeAsync(acc, stream);
      cudaFreeAsync(ws, stream);
      return set_error(OSP_ERR_CUDA, "clearing the backward workspace failed");
    }
    p.dq_acc = static_cast<float*>(acc);
    p.dq_acc_elems = (unsigned long long)(acc_bytes / sizeof(float)) / bounds_check_divisor();
  }
  const long long rows = (long long)s.B * N * s.heads;
  switch (s.head_dim) {
    case 64: rc = launch_bwd_d<64>(o, dout, tq, tk, tv, tdo, p, rows, ctas, stream); break;
    case 96: rc = launch_bwd_d<96>(o, dout, tq, tk, tv, tdo, p, rows, ctas, stream); break;
    case 128: rc = launch_bwd_d<128>(o, dout, tq, tk, tv, tdo, p, rows, ctas, stream); break;
    default: rc = set_error(OSP_ERR_UNSUPPORTED, "head_dim %d not in {64, 96, 128}", s.head_dim);
  }
  if (acc) cudaFreeAsync(acc, stream);
  cudaFreeAsync(ws, stream);
  return rc;
}

int packed_lse_rows(const int32_t* bounds, int n_seg) {
  long long rows = 0;
  for (int i = 0; i < n_seg; ++i) rows += (bounds[i + 1] - bounds[i] + 255) / 256 * 256;
  return (int)rows;
}

int packed_backward_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                           const float* lse, void* dq, void* dk, void* dv, const int32_t* bounds, int n_seg,
                           int heads, int head_dim, float scale, cudaStream_t stream) {
  unsigned* status = device_status_word();
  if (!status) return OSP_ERR_CUDA;
  const int N = bounds[n_seg];
  BwdSegTable seg{};
  seg.n_seg = n_seg;
  long long tiles = 0, vrows = 0;
  for (int i = 0; i <= n_seg; ++i) {
    seg.row[i] = bounds[i];
    seg.vrow[i] = (int)vrows;
    seg.tile[i] = (int)tiles;
    if (i < n_seg) {
      const int len = bounds[i + 1] - bounds[i];
      tiles += (len + kBT - 1) / kBT;
      vrows += (len + 255) / 256 * 256;   // the training forward's 256-row blocks
    }
  }
  BwdParams p{};
  p.N = N;
  p.heads = heads;
  p.G = 1;
  p.k = 1;
  p.layout = 0;
  p.n = N;                                // unused per CTA (each sample's own rows); for the host checks
  p.n_tiles = (int)tiles;
  p.q_rows = N;
  p.q_tiles = (int)tiles;
  p.vec_stride = (int)vrows;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scale = scale;
  p.lse = lse;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.status = status;
  p.timeout_ns = wait_timeout_ns();
  p.elems = (unsigned long long)N * heads * head_dim / bounds_check_divisor();
  p.vec_elems = (unsigned long long)heads * p.vec_stride / bounds_check_divisor();
  const long long ctas = tiles * heads;
  if (ctas > (1LL << 30)) return set_error(OSP_ERR_UNSUPPORTED, "%lld backward work units is too many", ctas);
  if (N == 0) return OSP_OK;
  const osp_shape sh{1, 0, 1, 1, 1, heads, head_dim};   // one sample of N packed rows
  CUtensorMap tq, tk, tv, tdo;
  int rc;
  if ((rc = make_attn_tmap(&tq, q, sh, N, 0, 1)) != OSP_OK) return rc;
  if ((rc = make_attn_tmap(&tk, k, sh, N, 0, 1)) != OSP_OK) return rc;
  if ((rc = make_attn_tmap(&tv, v, sh, N, 0, 1)) != OSP_OK) return rc;
  if ((rc = make_attn_tmap(&tdo, dout, sh, N, 0, 1)) != OSP_OK) return rc;
  const size_t vec_bytes = (size_t)heads * p.vec_stride * sizeof(float);
  void* ws = nullptr;
  cudaMemPool_t pool = workspace_pool();
  if (!pool || cudaMallocFromPoolAsync(&ws, vec_bytes, pool, stream) != cudaSuccess)
    return set_error(OSP_ERR_CUDA, "stream-ordered workspace allocation (%zu bytes) failed", vec_bytes);
  if (cudaMemsetAsync(ws, 0, vec_bytes, stream) != cudaSuccess) {
    cudaFreeAsync(ws, stream);
    return set_error(OSP_ERR_CUDA, "clearing the backward workspace failed");
  }
  p.dvec = static_cast<float*>(ws);
  void* acc = nullptr;
  if (head_dim == 64 && BwdCfg<64>::kFuseDq) {
    const size_t acc_bytes = (size_t)heads * p.vec_stride * head_dim * sizeof(float);
    if (cudaMallocFromPoolAsync(&acc, acc_bytes, pool, stream) != cudaSuccess) {
      cudaFreeAsync(ws, stream);
      return set_error(OSP_ERR_CUDA, "stream-ordered workspace allocation (%zu bytes) failed", acc_bytes);
    }
    if (cudaMemsetAsync(acc, 0, acc_bytes, stream) != cudaSuccess) {
      cudaFreeAsync(acc, stream);
      cudaFreeAsync(ws, stream);
      return set_error(OSP_ERR_CUDA, "clearing the backward workspace failed");
    }
    p.dq_acc = static_cast<float*>(acc);
    p.dq_acc_elems = (unsigned long long)(acc_bytes / sizeof(float)) / bounds_check_divisor();
  }
  const long long rows = (long long)N * heads;
  switch (head_dim) {
    case 64: rc = launch_bwd_d<64, true>(o, dout, tq, tk, tv, tdo, p, rows, ctas, stream, seg); break;
    case 96: rc = launch_bwd_d<96, true>(o, dout, tq, tk, tv, tdo, p, rows, ctas, stream, seg); break;
    case 128: rc = launch_bwd_d<128, true>(o, dout, tq, tk, tv, tdo, p, rows, ctas, stream, seg); break;
    default: rc = set_error(OSP_ERR_UNSUPPORTED, "head_dim %d not in {64, 96, 128}", head_dim);
  }
  if (acc) cudaFreeAsync(acc, stream);
  cudaFreeAsync(ws, stream);
  return rc;
}

}  // namespace osp
