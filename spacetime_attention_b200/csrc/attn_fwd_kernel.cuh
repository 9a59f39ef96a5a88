// Device code of the attention forward kernel (included once, by attn_fwd.cu, which holds the
// host-side launchers).  Kept in its own file so that a capture of the kernel's counters can
// be tied to this text alone.
//
// Flash-style attention forward for sm_100a on tcgen05 tensor cores.
//
// Computes, per (sample b, head h, token set g), O = softmax(Q K^T * scale) V over the set's n
// tokens: the whole sequence for 3D full attention ("CogVideoX" section 2.2 "3D Full
// Attention"), or one Skiparse set ("Open-Sora Plan" section 2.2.2).  The Skiparse sets are
// folded into the TMA tensor maps: a Single Skip set is a strided view of the token axis and a
// Group Skip set a 2-level view, so the k-fold permuted tensor never exists in memory.
//
// CTA = 2 query tiles of 128 rows sharing one K/V stream (384 threads, 3 warpgroups):
//   warps 0-3  softmax for query tile 0 (thread = one query row = one TMEM lane)
//   warps 4-7  softmax for query tile 1
//   warp 8     TMA producer: Q once, then K/V tiles into a ring of shared-memory stages
//   warp 9     tensor-memory allocator and MMA issuer (one elected thread)
//   warps 10-11 idle (they complete the third warpgroup for the register split)
// Registers: launched at 168 per thread (384 x 168 = 64,512); the producer/MMA warpgroup drops
// to 104 and the two softmax warpgroups rise to 200 (2 x 128 x 200 + 128 x 104 = 64,512).
// Tensor memory (512 columns x 128 lanes x 32 bit): S0 [0,128), S1 [128,256) fp32 scores,
// O0 [256, 256+D), O1 [384, 384+D) fp32 output accumulators.  The softmax overwrites the first
// 64 columns of S_i with P_i in bf16 pairs, and the PV product reads P_i from tensor memory as
// its A operand, so probabilities never touch shared memory.
// MMA issue order per KV tile j: PV0(j), S0(j+1), PV1(j), S1(j+1): while one softmax group
// works on its scores the tensor core runs the other group's two products.
// Online softmax keeps a per-row running max m and sum l in registers; O is rescaled only when
// the max grows by more than 2^8 (the final O/l uses the same stale max on both sides, so the
// result is exact), which removes most TMEM round trips of O.
// Every mbarrier wait is bounded: on timeout the CTA raises a shared abort flag, records
// kDevTimeout in the device status word, drains its in-flight TMA loads and MMAs, frees its
// tensor memory and exits.

#pragma once

#include <cuda.h>

#include <type_traits>

#include "osp_internal.h"

namespace osp {
namespace {

constexpr int kBM = 128;               // query rows per tile
constexpr int kBN = 128;               // keys per KV tile
constexpr int kChunkBytes = 128 * 128; // 128 rows x 64 bf16 channels (one 128-byte swizzle atom wide)
constexpr int kThreads = 384;
constexpr uint32_t kRegsLaunch = 168;   // ptxas' count for __launch_bounds__(384, 1)
constexpr uint32_t kRegsSoftmax = 200;
constexpr uint32_t kRegsSupport = 104;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsSupport == kThreads * kRegsLaunch,
              "register split must equal the launch allocation");
#ifndef OSP_MMA_WARP
#define OSP_MMA_WARP 9          // warp 8 loads; the MMA warp is 9, 10 or 11 (the idle ones fill the warpgroup)
#endif
#ifndef OSP_SPLIT_MMA
#define OSP_SPLIT_MMA 2         // separate-P layout: 1 = QK^T on warp 10, PV on warp 9;
#endif                          // 2 = QK^T on warp 10, PV of tile 0 on warp 9, of tile 1 on warp 11
#ifndef OSP_SPLIT_MMA_TILES
#define OSP_SPLIT_MMA_TILES 1   // P inside S at d = 96: tile 0's MMAs on warp 9, tile 1's on warp 11
#endif
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = OSP_MMA_WARP;
constexpr int kQkWarp = 10;
constexpr int kPv1Warp = 11;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kPersistMaxTiles = 32;       // KV tiles per item up to which CTAs run items in turn

// Tuning switches (compile-time; the defaults are the measured best on B200: alternating the
// softmax groups cost 4 % at d=64; the polynomial share pays only at d=128, where MUFU and the
// tensor core are balanced: 1 pair in 16 there, +6 %).
#ifndef OSP_SOFTMAX_TURNS
#define OSP_SOFTMAX_TURNS 0     // 1: the two softmax groups alternate their exponential phases
#endif
#ifndef OSP_POLY16_D64
#define OSP_POLY16_D64 0        // exp2 pairs (of 16) on the FMA pipe at d = 64
#endif
#ifndef OSP_POLY16_D96
#define OSP_POLY16_D96 0
#endif
#ifndef OSP_POLY16_D128
#define OSP_POLY16_D128 1
#endif
#ifndef OSP_F32X2
#define OSP_F32X2 1             // packed fp32 pairs for the scale/subtract and the row sum
#endif

template <int D>
struct Cfg {
  static constexpr int kChunks = (D + 63) / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (D == 64) ? 4 : 2;
  // d <= 64: S0, S1, O0, O1 and separate P0, P1 buffers fit the 512 TMEM columns, so the softmax
  // releases S as soon as it is in registers and QK^T of the next tile overlaps the exponentials.
  // Larger d: P aliases the first 64 columns of S.
  static constexpr bool kSepP = (D <= 64);
  // Of every 16 exponential pairs, this many run as a polynomial on the FMA/ALU pipes instead of
  // MUFU (whose 16 ex2/clk/SM bound the softmax at small d); the rest use ex2.approx.
  static constexpr int kPolyPer16 = (D <= 64) ? OSP_POLY16_D64 : (D <= 96 ? OSP_POLY16_D96 : OSP_POLY16_D128);
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  // Output staging for the TMA-store epilogue, per query tile: one 64-channel SW128 chunk (16 KB),
  // through which a row's 64-channel parts go in turn (rounds); at d = 96 the second round holds
  // the last 32 channels as a 64-byte-swizzled 128 x 64-byte tile, stored with a 32-channel box
  // so that no box reaches into the next head's channels.
  static constexpr int kStgTileBytes = (D >= 96) ? kChunkBytes : 0;   // d = 64 keeps per-row stores
  static constexpr int kStgOff = kVOff + kStages * kTileBytes;
  static constexpr int kStgRounds = kChunks;
  static constexpr int kBarOff = kStgOff + 2 * kStgTileBytes;
  // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_ready[2],
  // o_full[2], mma_done, s_free[2], turn[2], ..., stg_full[2], stg_free[2]
  static constexpr int kNumBars = 1 + 4 * kStages + 16 + 4;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 32 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

// Output tensor maps for the TMA-store epilogue (the same view of o as the query map's of q);
// use = 0 keeps per-thread row stores (packed batches).  tail: d = 96's channels 64 .. 95.
struct OutMaps {
  CUtensorMap o;
  CUtensorMap tail;
  int use;
};

struct AttnParams {
  int n_q;        // query rows per set
  int n_kv;       // key / value rows per set (= n_q for self-attention)
  int N_q;        // tokens per sample of the natural-order q and o tensors
  int heads;
  int G;          // sets per sample
  int k;          // sparse ratio (1 for dense)
  int layout;     // 0 dense, 1 Single Skip, 2 Group Skip
  float scale_log2;
  __nv_bfloat16* o;
  unsigned* status;
  unsigned long long timeout_ns;
  int debug_withhold_q;   // test knob: never load Q, so every consumer's bounded wait runs out
  // Frame-causal mask (dense layout only; 0 = off): query token r attends to the first
  // limit(r) keys, limit = text_len for a text token and text_len + (t + 1) * frame_hw for a
  // token of frame t.  Query blocks then run heaviest (latest) first.
  int frame_hw;
  int text_len;
  // Skiparse with a joined text prefix (mode kModeSkipText): every set's KV range is the
  // text_len text rows (ceil(text_len / 128) tiles from the text maps) followed by the set's own
  // tiles; the set's query tokens sit q_row_base (= text_len) rows into each sample.
  int q_row_base;
  // Optional row log-sum-exp for the backward pass (plain mode): lse[(b*G + g)*heads + h][slot]
  // = m + log2(l) in the log2 domain of the scaled scores, rows lse_stride apart.
  float* lse;
  int lse_stride;
  // element counts of the buffers written, for the debug build's index checks
  unsigned long long o_elems, lse_elems, ws_rows;
  // Work items (1-D grid): units are (sample*set, head, query block) with the query block fastest.
  // CTAs [0, n_full) process whole units; every later unit is split into n_split KV ranges whose
  // CTAs write fp32 partials (unnormalised O, running max m, row sum l) to ws_o / ws_ml, merged
  // by attn_combine_kernel.
  int qblocks;            // 256-row query blocks per (sample*set, head)
  int n_full;
  int n_split;
  int n_items;            // work items (whole units, then split parts); CTA c runs items c, c + grid, ...
  float* ws_o;            // [split units][n_split][256][D]
  float2* ws_ml;          // [split units][n_split][256]
};

// Packed batch of samples of different lengths (block-diagonal attention).  Segment i owns query
// rows [q[i], q[i+1]) and key rows [kv[i], kv[i+1]) of the packed tensors and the work units
// [heads * blk[i], heads * blk[i+1]) (one per head and 256-row query block, block fastest).
// Passed by value as a kernel parameter, so a launch carries its own table.
struct SegTable {
  int n_seg;
  int blk[kMaxSegments + 1];
  int q[kMaxSegments + 1];
  int kv[kMaxSegments + 1];
};
struct NoSegTable {};
// Tensor maps of the text rows of k and v (dense view, text_len rows per sample) for Skiparse
// with a joined text prefix.
struct TextMaps {
  CUtensorMap k;
  CUtensorMap v;
};
// Kernel variants: plain (dense / Skiparse / cross), packed batch, frame-causal mask, Skiparse
// with a joined text prefix.
enum AttnMode { kModePlain = 0, kModePacked = 1, kModeFrameCausal = 2, kModeSkipText = 3 };
template <int kMode>
using SegParam = typename std::conditional<
    kMode == kModePacked, SegTable, typename std::conditional<kMode == kModeSkipText, TextMaps, NoSegTable>::type>::type;

__device__ __forceinline__ void load_tile(const CUtensorMap* tm, uint32_t dst, uint32_t bar, int layout,
                                          int chan, int row0, int g, int b, int k) {
  if (layout == 0) tma_load_3d(dst, tm, bar, chan, row0, b);
  else if (layout == 1) tma_load_4d(dst, tm, bar, chan, g, row0, b);
  else tma_load_5d(dst, tm, bar, chan, 0, g, row0 / k, b);
}

// Keys visible to query token r under the frame-causal mask (text block, then one block per frame).
__device__ __forceinline__ int frame_causal_limit(int r, int text_len, int hw) {
  return r < text_len ? text_len : text_len + ((r - text_len) / hw + 1) * hw;
}

// Natural token index of slot s of set g.
__device__ __forceinline__ int slot_token(int layout, int s, int g, int k) {
  if (layout == 0) return s;
  if (layout == 1) return s * k + g;
  const int o = s / k;
  return (o * k + g) * k + (s - o * k);
}

// exp2 of two values on the FMA and ALU pipes: 2^x = 2^n * 2^f with n = round(x) (added to the
// exponent field) and f = x - n in [-1/2, 1/2]; 2^f is the degree-3 minimax polynomial derived
// by docs/exp2_poly.py (Remez, relative error 7.5e-5, far below the bf16 step of P).  Inputs
// are clamped at -125 so that the exponent field cannot underflow (2^-125 is negligible next to
// the row maximum's 1).
__device__ __forceinline__ void ex2_poly2(uint64_t x2, float& e0, float& e1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound holds round(x) in its low bits
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = f2_add(xc, f2_pack(kRound, kRound));
  const uint64_t n = f2_add(t, f2_pack(-kRound, -kRound));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), xc);
  uint64_t q = f2_fma(f2_pack(5.517166853e-02f, 5.517166853e-02f), f, f2_pack(2.426111251e-01f, 2.426111251e-01f));
  q = f2_fma(q, f, f2_pack(6.932609677e-01f, 6.932609677e-01f));
  q = f2_fma(q, f, f2_pack(9.999280572e-01f, 9.999280572e-01f));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  e0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// p = exp2(s * sl2 - m) for the 128 scores of one row, packed to bf16 pairs; returns the row sum.
// kPoly: whether the polynomial takes its share (never on a tile with masked (-inf) columns).
#ifndef OSP_EXP_BATCH
#define OSP_EXP_BATCH 8         // exponential pairs issued before any result is consumed
#endif

// p = exp2(s * sl2 - m) for the 128 scores of one row, packed to bf16 pairs; returns the row sum.
// The pairs are processed in batches: all exponentials of a batch are issued before any result
// is consumed, and the row sum uses four independent accumulators, so MUFU latency overlaps
// instead of serialising the loop.  kPoly: whether the polynomial takes its share (never on a
// tile with masked (-inf) columns).
template <int kPolyPer16, bool kPoly>
__device__ __forceinline__ float softmax_exp_row(const float (&sv)[128], float sl2, float m, uint32_t (&pk)[64]) {
  constexpr int kB = OSP_EXP_BATCH;
  const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m, -m);
  uint64_t sum2[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
  for (int c0 = 0; c0 < 64; c0 += kB) {
    float e[2 * kB];
#pragma unroll
    for (int t = 0; t < kB; ++t) {
      const int c = c0 + t;
      const uint64_t x2 = f2_fma(f2_pack(sv[2 * c], sv[2 * c + 1]), scale2, negm2);
      if (kPoly && (c % 16) < kPolyPer16) {
        ex2_poly2(x2, e[2 * t], e[2 * t + 1]);
      } else {
        float x0, x1;
        f2_unpack(x2, x0, x1);
        e[2 * t] = ex2_approx(x0);
        e[2 * t + 1] = ex2_approx(x1);
      }
    }
#pragma unroll
    for (int t = 0; t < kB; ++t) {
      sum2[t & 3] = f2_add(sum2[t & 3], f2_pack(e[2 * t], e[2 * t + 1]));
      pk[c0 + t] = pack_bf16x2(e[2 * t], e[2 * t + 1]);
    }
  }
  const uint64_t s01 = f2_add(sum2[0], sum2[1]), s23 = f2_add(sum2[2], sum2[3]);
  float lo, hi;
  f2_unpack(f2_add(s01, s23), lo, hi);
  return lo + hi;
}

// Warp-uniform bounded wait (tcgen05.ld/st that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// kLoop: the CTA runs work items blockIdx.x, blockIdx.x + gridDim.x, ... (grid smaller than the
// item count); otherwise exactly item blockIdx.x, and every cross-item wait folds away.
template <int D, int kMode, bool kLoop>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p,
                    const __grid_constant__ SegParam<kMode> seg, const __grid_constant__ OutMaps om) {
  constexpr bool kPacked = kMode == kModePacked;
  constexpr bool kFrameCausal = kMode == kModeFrameCausal;
  constexpr bool kSkipText = kMode == kModeSkipText;
  using C = Cfg<D>;
  constexpr int S = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 1 + S, B_VFULL = 1 + 2 * S, B_VEMPTY = 1 + 3 * S;
  const int B_SFULL = 1 + 4 * S, B_PREADY = B_SFULL + 2, B_OFULL = B_PREADY + 2, B_MMADONE = B_OFULL + 2;
  const int B_SFREE = B_MMADONE + 1;  // separate-P layout: softmax has S_i in registers
  const int B_TURN = B_SFREE + 2;     // softmax i may start its exponentials (MUFU hand-off)
  const int B_QKDONE = B_TURN + 2;    // split MMA issue: the QK^T warp's final commit
  const int B_PV1DONE = B_QKDONE + 1; // split MMA issue: the tile-1 PV warp's final commit
  // A CTA may run several work items in turn (grid smaller than the item count):
  const int B_QEMPTY = B_PV1DONE + 1; // Q may be overwritten: every QK^T of the item has completed
  const int B_OFREE = B_QEMPTY + 1;   // [2] the softmax has read O_i out (the next item may overwrite it)
  const int B_STGFULL = B_OFREE + 2;  // [2] tile i's rows are in its output staging tile
  const int B_STGFREE = B_STGFULL + 2; // [2] the TMA store has read tile i's staging tile
  constexpr bool kSplitMma = C::kSepP && OSP_SPLIT_MMA > 0;
  constexpr bool kSplitPv = C::kSepP && OSP_SPLIT_MMA > 1;
  // per-tile issuers (9 and 11) pay at d = 96 (+2 %); at d = 128 the tensor pipe is the bottleneck
  // and interleaving the two tiles' MMA streams delays each tile (-7 %)
  constexpr bool kSplitTiles = !C::kSepP && D == 96 && OSP_SPLIT_MMA_TILES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* seg_slot = reinterpret_cast<int*>(tmem_slot + 2);   // packed batches: this CTA's segment
  // debug builds: a row of tile i failed its output index check (its staged store is skipped)
  volatile int* stg_bad = reinterpret_cast<volatile int*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work item -> unit (sample*set, head, query block) and KV tile range [kv_lo, kv_lo + n_kv).
  // q_row0 / kv_row0 offset the rows of a packed segment; nq / nkv are the set's query and key
  // rows.  Recomputed where needed (cheap integer math) rather than kept live across the main loops.
  struct Work { int unit, part, h, b, g, q0, kv_lo, n_kv, q_row0, kv_row0, nq, nkv, q_out0; };
  auto decode = [&](int item) {
    Work w;
    w.unit = item;
    w.part = -1;
    int qb;
    if constexpr (kPacked) {
      const int sg = *seg_slot;
      const int nqb = seg.blk[sg + 1] - seg.blk[sg];
      const int local = w.unit - p.heads * seg.blk[sg];
      w.h = local / nqb;
      qb = local - w.h * nqb;
      w.b = 0;
      w.g = 0;
      w.q_row0 = seg.q[sg];
      w.q_out0 = w.q_row0;
      w.kv_row0 = seg.kv[sg];
      w.nq = seg.q[sg + 1] - w.q_row0;
      w.nkv = seg.kv[sg + 1] - w.kv_row0;
    } else {
      if (w.unit >= p.n_full) {
        const int t = w.unit - p.n_full;
        w.unit = p.n_full + t / p.n_split;
        w.part = t % p.n_split;
      }
      qb = w.unit % p.qblocks;
      const int hb = w.unit / p.qblocks;
      w.h = hb % p.heads;
      const int bg = hb / p.heads;
      w.b = bg / p.G;
      w.g = bg % p.G;
      w.q_row0 = 0;
      w.q_out0 = p.q_row_base;   // the maps start at the set's rows; outputs sit past the text
      w.kv_row0 = 0;
      w.nq = p.n_q;
      w.nkv = p.n_kv;
    }
    if constexpr (kFrameCausal) {
      qb = p.qblocks - 1 - qb;   // latest (longest) query blocks first
      // keys up to the limit of the block's last query row
      const int last = min(qb * (2 * kBM) + 2 * kBM, w.nq) - 1;
      w.nkv = min(w.nkv, frame_causal_limit(last, p.text_len, p.frame_hw));
    }
    w.q0 = qb * (2 * kBM);
    const int n_kv_all = (w.nkv + kBN - 1) / kBN + (kSkipText ? (p.text_len + kBN - 1) / kBN : 0);
    w.kv_lo = w.part < 0 ? 0 : (int)((long long)w.part * n_kv_all / p.n_split);
    w.n_kv = (w.part < 0 ? n_kv_all : (int)((long long)(w.part + 1) * n_kv_all / p.n_split)) - w.kv_lo;
    return w;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), kSplitTiles ? 2 : 1);   // per-tile issuers both release K
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), (kSplitPv || kSplitTiles) ? 2 : 1);   // both PV issuers release V
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PREADY + i), 128);
      mbar_init(bar(B_OFULL + i), 1);
    }
    mbar_init(bar(B_MMADONE), 1);
    mbar_init(bar(B_SFREE + 0), 128);
    mbar_init(bar(B_SFREE + 1), 128);
    mbar_init(bar(B_QKDONE), 1);
    mbar_init(bar(B_PV1DONE), 1);
    mbar_init(bar(B_QEMPTY), kSplitTiles ? 2 : 1);   // each QK^T issuing warp commits once per item
    mbar_init(bar(B_OFREE + 0), 128);
    mbar_init(bar(B_OFREE + 1), 128);
    mbar_init(bar(B_TURN + 0), 128);
    mbar_init(bar(B_TURN + 1), 128);
    if constexpr (D >= 96)
      for (int t = 0; t < 2; ++t) {
        mbar_init(bar(B_STGFULL + t), 128);
        mbar_init(bar(B_STGFREE + t), 1);
      }
    *abort_flag = 0;
    stg_bad[0] = stg_bad[1] = 0;
    fence_mbar_init();
  }
  if constexpr (kPacked) {
    if (warp == 0) {
      // segment of this CTA's unit: the number of i in [1, n_seg] with heads * blk[i] <= unit
      // (blk is non-decreasing and unit < heads * blk[n_seg]); 32 lanes test 8 entries each
      int c = 0;
#pragma unroll
      for (int t = 0; t < (kMaxSegments + 31) / 32; ++t) {
        const int i = 1 + lane + 32 * t;
        if (i <= seg.n_seg && p.heads * seg.blk[i] <= (int)blockIdx.x) ++c;
      }
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) *seg_slot = c;
    }
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if constexpr (kSkipText) {
      prefetch_tmap(&seg.k);
      prefetch_tmap(&seg.v);
    }
    if (D >= 96 && om.use) {
      prefetch_tmap(&om.o);
      if (D == 96) prefetch_tmap(&om.tail);
    }
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
  // KV tile jj of this unit's range: with a joined text prefix the first tiles come from the
  // text maps (dense rows), the rest from the set's own map.
  auto load_kv_tile = [&](const CUtensorMap& tm, const SegParam<kMode>& sp, uint32_t dst, uint32_t mbar, int chan,
                          int jj, const Work& w, bool is_k) {
    if constexpr (kSkipText) {
      const int ntt = (p.text_len + kBN - 1) / kBN;
      if (jj < ntt) {
        tma_load_3d(dst, is_k ? &sp.k : &sp.v, mbar, chan, jj * kBN, w.b);
        return;
      }
      jj -= ntt;
    }
    load_tile(&tm, dst, mbar, p.layout, chan, w.kv_row0 + jj * kBN, w.g, w.b, p.k);
  };

  auto sQ = [&](int i) { return sbase + C::kQOff + (uint32_t)(i * C::kTileBytes); };
  auto sK = [&](int s) { return sbase + C::kKOff + (uint32_t)(s * C::kTileBytes); };
  auto sV = [&](int s) { return sbase + C::kVOff + (uint32_t)(s * C::kTileBytes); };
  auto colS = [](int i) { return i ? 128u : 0u; };
  auto colO = [](int i) { return i ? (C::kSepP ? 320u : 384u) : 256u; };
  auto colP = [](int i) { return C::kSepP ? (i ? 448u : 384u) : (i ? 128u : 0u); };

  if (warp >= kLoadWarp) {
   // each warpgroup's register budget change dominates its own role code
   regs_dec<kRegsSupport>();
   // The producer and MMA warps run their loops with all 32 lanes converged (so addresses and
   // descriptors stay warp-uniform) and one elected lane issues the TMA / tcgen05 instructions.
   const bool leader = elect_one_sync();
   if (warp == kLoadWarp) {
    // ------------------------------------------------------------------ TMA producer
    {
      // K / V tiles are counted over all of this CTA's items (the rings continue across items)
      int k_issued = 0, v_issued = 0, q_issued = 0, jb = 0;
      const bool q_armed = !p.debug_withhold_q;
      bool ok = true;
      for (int item = blockIdx.x, ub = 0; ok && (kLoop ? item < p.n_items : ub == 0); item += gridDim.x, ++ub) {
        const Work w = decode(item);
        const int c0 = w.h * D;
        // the previous item's Q may be overwritten once its last QK^T has completed
        if (ub > 0 && !warp_wait(bar(B_QEMPTY), (ub - 1) & 1, wc)) break;
        if (leader && q_armed) {
          mbar_arrive_expect_tx(bar(B_QFULL), 2 * C::kTileBytes);
          for (int i = 0; i < 2; ++i)
            for (int c = 0; c < C::kChunks; ++c)
              load_tile(&tm_q, sQ(i) + c * kChunkBytes, bar(B_QFULL), p.layout, c0 + 64 * c,
                        w.q_row0 + w.q0 + i * kBM, w.g, w.b, p.k);
        }
        q_issued = ub + 1;
        for (int j = 0; j < w.n_kv; ++j) {
          const int jg = jb + j, s = jg % S, u = jg / S;
          if (jg >= S && !warp_wait(bar(B_KEMPTY + s), (u - 1) & 1, wc)) { ok = false; break; }
          if (leader) {
            mbar_arrive_expect_tx(bar(B_KFULL + s), C::kTileBytes);
            for (int c = 0; c < C::kChunks; ++c)
              load_kv_tile(tm_k, seg, sK(s) + c * kChunkBytes, bar(B_KFULL + s), c0 + 64 * c, w.kv_lo + j, w, true);
          }
          k_issued = jg + 1;
          if (jg >= S && !warp_wait(bar(B_VEMPTY + s), (u - 1) & 1, wc)) { ok = false; break; }
          if (leader) {
            mbar_arrive_expect_tx(bar(B_VFULL + s), C::kTileBytes);
            for (int c = 0; c < C::kChunks; ++c)
              load_kv_tile(tm_v, seg, sV(s) + c * kChunkBytes, bar(B_VFULL + s), c0 + 64 * c, w.kv_lo + j, w, false);
          }
          v_issued = jg + 1;
        }
        jb += w.n_kv;
      }
      // Drain: every load issued has landed before the CTA may exit.  A Q load is issued only
      // after the previous one was consumed, and only the last S tiles of each ring can still be
      // in flight.
      if (q_armed && q_issued > 0) mbar_drain(bar(B_QFULL), (q_issued - 1) & 1, p.timeout_ns);
      for (int t = (k_issued > S ? k_issued - S : 0); t < k_issued; ++t)
        mbar_drain(bar(B_KFULL + t % S), (t / S) & 1, p.timeout_ns);
      for (int t = (v_issued > S ? v_issued - S : 0); t < v_issued; ++t)
        mbar_drain(bar(B_VFULL + t % S), (t / S) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == kMmaWarp || (kSplitMma && warp == kQkWarp) || ((kSplitPv || kSplitTiles) && warp == kPv1Warp)) {
    // ------------------------------------------------------------------ MMA issuer
    {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
      // Descriptors are built once; a K step moves the start address (bits [0,14), 16-byte units)
      // within the tile, so each MMA only adds a small constant to a precomputed base.
      // Tiles of one kind are contiguous, kTileBytes apart, so tile t's descriptor is the first
      // one's plus t * kTileBytes / 16.
      const uint64_t dq = sdesc_sw128(sQ(0), 16, 1024), dk = sdesc_sw128(sK(0), 16, 1024);
      const uint64_t dv = sdesc_sw128(sV(0), kChunkBytes, 1024);
      constexpr uint64_t kTileStep = (uint64_t)(C::kTileBytes >> 4);
      // S_i = Q_i K^T: both operands K-major (channels contiguous), 16 channels per MMA: step kk
      // starts (kk / 4) 64-channel chunks and (kk % 4) * 32 bytes into the tile.
      auto issue_s = [&](int i, int s) {
        const uint64_t a0 = dq + (uint64_t)i * kTileStep, b0 = dk + (uint64_t)s * kTileStep;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          if (leader) mma_ss(tmem + colS(i), a0 + off, b0 + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_i += P_i V: P_i from tensor memory (bf16 pairs, 64 columns), V MN-major (channels
      // contiguous), 16 keys (2048 bytes of V) per MMA.
      auto issue_pv = [&](int i, int s, bool acc) {
        const uint64_t b0 = dv + (uint64_t)s * kTileStep;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          if (leader)
            mma_ts(tmem + colO(i), tmem + colP(i) + 8u * kk, b0 + (uint64_t)(128 * kk), idesc_pv,
                   (acc || kk > 0) ? 1u : 0u);
        }
      };
      // which MMAs this warp issues (one warp issues all of them unless the issue is split)
      const bool do_qk = !kSplitMma || warp == kQkWarp;
      const bool do_pv0 = !kSplitMma || warp == kMmaWarp;
      const bool do_pv1 = !kSplitMma || (kSplitPv ? warp == kPv1Warp : warp == kMmaWarp);
      // KV tiles are counted over all of this CTA's items (jg = jb + j), as by the producer and
      // the softmax warps; per-item barriers (Q full / empty, O free) by the item count ub.
      int jb = 0;
      bool ok = true;
      for (int item = blockIdx.x, ub = 0; ok && (kLoop ? item < p.n_items : ub == 0); item += gridDim.x, ++ub) {
        const int n_kv = decode(item).n_kv;
        const int s0 = jb % S;
        // Q and the item's first K tile, for the warps that issue QK^T (a PV-only warp never reads
        // them and must not wait on phases it could fall behind on)
        if ((!C::kSepP || do_qk) &&
            (!warp_wait(bar(B_QFULL), ub & 1, wc) || !warp_wait(bar(B_KFULL + s0), (jb / S) & 1, wc))) {
          ok = false;
          break;
        }
        if (C::kSepP) {
          // Order per KV tile j: S0(j+1) as soon as softmax 0 holds S0(j) in registers, S1(j+1)
          // likewise, then PV0(j), PV1(j) as their P tiles arrive.  O_full[i] completes after every
          // PV_i(j): the softmax waits on it before overwriting P_i and before touching O_i.
          tc_fence_after();
          if (do_qk) {
            // S_i of the previous item's last tile must be out of tensor memory
            if (ub > 0 && !warp_wait(bar(B_SFREE + 0), (jb - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            issue_s(0, s0);
            if (leader) tc_commit(bar(B_SFULL + 0));
            if (ub > 0 && !warp_wait(bar(B_SFREE + 1), (jb - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            issue_s(1, s0);
            if (leader) tc_commit(bar(B_SFULL + 1));
            if (leader) tc_commit(bar(B_KEMPTY + s0));
            if (n_kv == 1 && leader) tc_commit(bar(B_QEMPTY));
          }
          for (int j = 0; j < n_kv; ++j) {
            const int jg = jb + j, s = jg % S, u = jg / S;
            const bool more = j + 1 < n_kv;
            const int s1 = (jg + 1) % S, u1 = (jg + 1) / S;
            if (do_qk && more) {
              if (!warp_wait(bar(B_KFULL + s1), u1 & 1, wc)) { ok = false; break; }
              if (!warp_wait(bar(B_SFREE + 0), jg & 1, wc)) { ok = false; break; }
              tc_fence_after();
              issue_s(0, s1);
              if (leader) tc_commit(bar(B_SFULL + 0));
              if (!warp_wait(bar(B_SFREE + 1), jg & 1, wc)) { ok = false; break; }
              tc_fence_after();
              issue_s(1, s1);
              if (leader) tc_commit(bar(B_SFULL + 1));
              if (leader) tc_commit(bar(B_KEMPTY + s1));
              if (j + 2 == n_kv && leader) tc_commit(bar(B_QEMPTY));
            }
            if (do_pv0 || do_pv1) {
              if (!warp_wait(bar(B_VFULL + s), u & 1, wc)) { ok = false; break; }
            }
            if (do_pv0) {
              if (!warp_wait(bar(B_PREADY + 0), jg & 1, wc)) { ok = false; break; }
              // the first PV of an item overwrites O_0: the previous item's epilogue has read it
              if (j == 0 && ub > 0 && !warp_wait(bar(B_OFREE + 0), (ub - 1) & 1, wc)) { ok = false; break; }
              tc_fence_after();
              issue_pv(0, s, j > 0);
              if (leader) tc_commit(bar(B_OFULL + 0));
              if (kSplitPv && leader) tc_commit(bar(B_VEMPTY + s));
            }
            if (do_pv1) {
              if (!warp_wait(bar(B_PREADY + 1), jg & 1, wc)) { ok = false; break; }
              if (j == 0 && ub > 0 && !warp_wait(bar(B_OFREE + 1), (ub - 1) & 1, wc)) { ok = false; break; }
              tc_fence_after();
              issue_pv(1, s, j > 0);
              if (leader) tc_commit(bar(B_OFULL + 1));
              if (leader) tc_commit(bar(B_VEMPTY + s));
            }
          }
        } else if (kSplitTiles) {
          // P inside S: per tile, PV_i(j) must precede S_i(j+1) (the tensor pipe runs one thread's
          // MMAs in order); the two tiles are independent, so each has its own issuing warp.
          // The first S_i of an item follows the previous item's last PV_i in this warp's order.
          const int ti = (warp == kPv1Warp) ? 1 : 0;
          tc_fence_after();
          issue_s(ti, s0);
          if (leader) tc_commit(bar(B_SFULL + ti));
          if (leader) tc_commit(bar(B_KEMPTY + s0));
          if (n_kv == 1 && leader) tc_commit(bar(B_QEMPTY));
          for (int j = 0; j < n_kv; ++j) {
            const int jg = jb + j, s = jg % S, u = jg / S;
            const bool more = j + 1 < n_kv;
            const int s1 = (jg + 1) % S, u1 = (jg + 1) / S;
            if (!warp_wait(bar(B_VFULL + s), u & 1, wc)) { ok = false; break; }
            if (more && !warp_wait(bar(B_KFULL + s1), u1 & 1, wc)) { ok = false; break; }
            if (!warp_wait(bar(B_PREADY + ti), jg & 1, wc)) { ok = false; break; }
            if (j == 0 && ub > 0 && !warp_wait(bar(B_OFREE + ti), (ub - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            issue_pv(ti, s, j > 0);
            if (leader) tc_commit(bar(B_VEMPTY + s));
            if (more) {
              issue_s(ti, s1);
              if (leader) tc_commit(bar(B_SFULL + ti));
              if (leader) tc_commit(bar(B_KEMPTY + s1));
              if (j + 2 == n_kv && leader) tc_commit(bar(B_QEMPTY));
            } else {
              if (leader) tc_commit(bar(B_OFULL + ti));
            }
          }
        } else {
          tc_fence_after();
          issue_s(0, s0);
          if (leader) tc_commit(bar(B_SFULL + 0));
          issue_s(1, s0);
          if (leader) tc_commit(bar(B_SFULL + 1));
          if (leader) tc_commit(bar(B_KEMPTY + s0));
          if (n_kv == 1 && leader) tc_commit(bar(B_QEMPTY));
          for (int j = 0; j < n_kv; ++j) {
            const int jg = jb + j, s = jg % S, u = jg / S;
            const bool more = j + 1 < n_kv;
            const int s1 = (jg + 1) % S, u1 = (jg + 1) / S;
            if (!warp_wait(bar(B_VFULL + s), u & 1, wc)) { ok = false; break; }
            if (more && !warp_wait(bar(B_KFULL + s1), u1 & 1, wc)) { ok = false; break; }
            if (!warp_wait(bar(B_PREADY + 0), jg & 1, wc)) { ok = false; break; }
            if (j == 0 && ub > 0 && !warp_wait(bar(B_OFREE + 0), (ub - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            issue_pv(0, s, j > 0);
            if (more) {
              issue_s(0, s1);
              if (leader) tc_commit(bar(B_SFULL + 0));
            } else {
              if (leader) tc_commit(bar(B_OFULL + 0));
            }
            if (!warp_wait(bar(B_PREADY + 1), jg & 1, wc)) { ok = false; break; }
            if (j == 0 && ub > 0 && !warp_wait(bar(B_OFREE + 1), (ub - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            issue_pv(1, s, j > 0);
            if (leader) tc_commit(bar(B_VEMPTY + s));
            if (more) {
              issue_s(1, s1);
              if (leader) tc_commit(bar(B_SFULL + 1));
              if (leader) tc_commit(bar(B_KEMPTY + s1));
              if (j + 2 == n_kv && leader) tc_commit(bar(B_QEMPTY));
            } else {
              if (leader) tc_commit(bar(B_OFULL + 1));
            }
          }
        }
        jb += n_kv;
      }
      // Drain: all issued MMAs complete before tensor memory is freed.
      const int done_bar = (kSplitMma && warp == kQkWarp) ? B_QKDONE
                         : ((kSplitPv || kSplitTiles) && warp == kPv1Warp) ? B_PV1DONE : B_MMADONE;
      if (leader) tc_commit(bar(done_bar));
      mbar_drain(bar(done_bar), 0, p.timeout_ns);
    }
    __syncwarp();
   }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax / epilogue
    const int i = warp >> 2;                       // query tile
    const int quarter = warp & 3;                  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;           // row within the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + colS(i);
    const uint32_t tO = tmem + lane_base + colO(i);
    const uint32_t tP = tmem + lane_base + colP(i);
    const float sl2 = p.scale_log2;
    bool ok = true;
    int jb = 0;            // KV tiles of this CTA's earlier items
    int stg_rounds = 0;    // output staging rounds of this tile so far (TMA-store epilogue)
    for (int item = blockIdx.x, ub = 0; ok && (kLoop ? item < p.n_items : ub == 0); item += gridDim.x, ++ub) {
    const Work wk = decode(item);
    const int n_kv = wk.n_kv;
    float m = -INFINITY, l = 0.f;
    int lim = wk.nkv;                                // keys this row may see
    if constexpr (kFrameCausal)
      lim = min(lim, frame_causal_limit(wk.q0 + i * kBM + row, p.text_len, p.frame_hw));
    const int valid0 = lim - wk.kv_lo * kBN;         // valid keys from this item's first KV tile on
    for (int j = 0; j < n_kv; ++j) {
      const int jg = jb + j;
      if (!warp_wait(bar(B_SFULL + i), jg & 1, wc)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_wait_ld();
      if constexpr (C::kSepP) {
        tc_fence_before();
        mbar_arrive(bar(B_SFREE + i));   // S_i may now be overwritten by the next QK^T
      }
      float sv[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(sr[c]);
      int valid = valid0 - j * kBN;
      if constexpr (kSkipText) {
        // text tiles (ragged last one), then the set's tiles (ragged last one)
        const int jj = wk.kv_lo + j, ntt = (p.text_len + kBN - 1) / kBN;
        valid = jj < ntt ? p.text_len - jj * kBN : wk.nkv - (jj - ntt) * kBN;
      }
      const bool masked = valid < kBN;
      if (masked) {
        // only the 32-column chunks that reach past the last valid key (a uniform branch for the
        // warp unless the limit is per row); masking all 128 columns cost 1-3 % on short items
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (valid < 32 * q + 32) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * q + e >= valid) sv[32 * q + e] = -INFINITY;
          }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        mx0 = fmax3(mx0, sv[c], sv[c + 1]);
        mx1 = fmax3(mx1, sv[c + 2], sv[c + 3]);
        mx2 = fmax3(mx2, sv[c + 4], sv[c + 5]);
        mx3 = fmax3(mx3, sv[c + 6], sv[c + 7]);
      }
      const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sl2;
      const float m_cand = fmaxf(m, mx);
      const bool rescale = m_cand > m + kRescaleThreshold;
      float alpha = 1.f;
      if (rescale) {
        alpha = ex2_approx(m - m_cand);
        m = m_cand;
      }
      // The two softmax groups take turns on MUFU: group 0 runs the exponentials of tile j after
      // group 1 finished those of tile j-1, group 1 after group 0 finished tile j.  Each group's
      // load / max / store phases overlap the other group's exponentials.
      if (OSP_SOFTMAX_TURNS && (i == 1 || jg > 0)) {
        if (!warp_wait(bar(B_TURN + i), (uint32_t)((i == 0 ? jg - 1 : jg) & 1), wc)) { ok = false; break; }
      }
      uint32_t pk[64];
      // Masked columns (-inf) never take the polynomial.  With no polynomial share one inlined
      // copy of the loop can serve both kinds of tile: measured +3 to +9 % at d = 96 and on
      // short items at d = 64 (items in turn), -4 % on the d = 64 single-item kernel, which
      // keeps two copies.
      constexpr bool kOneExpCopy = C::kPolyPer16 == 0 && (D == 96 || kLoop);
      const float rs = kOneExpCopy || !masked ? softmax_exp_row<C::kPolyPer16, true>(sv, sl2, m, pk)
                                              : softmax_exp_row<C::kPolyPer16, false>(sv, sl2, m, pk);
      if (OSP_SOFTMAX_TURNS) mbar_arrive(bar(B_TURN + (1 - i)));
      l = l * alpha + rs;
      // P_i (and O_i) are free once PV_i(j-1) has completed (separate-P layout; with P inside S
      // the MMA warp already ordered it)
      if constexpr (C::kSepP) {
        if (j > 0 && !warp_wait(bar(B_OFULL + i), (jg - 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st32(tP + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
      tmem_st32(tP + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + 32 * cc, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PREADY + i));
    }
    if (!ok) break;
    // O_i complete: per tile in the separate-P layout, once per item otherwise
    if (!warp_wait(bar(B_OFULL + i), C::kSepP ? (uint32_t)((jb + n_kv - 1) & 1) : (uint32_t)(ub & 1), wc)) {
      ok = false;
      break;
    }
    {
      tc_fence_after();
      const Work w = decode(item);
      const int unit = w.unit, part = w.part, h = w.h, b = w.b, g = w.g;
      const float inv_l = 1.f / l;
      const int slot = w.q0 + i * kBM + row;
      const bool live = slot < w.nq;
      if (part < 0 && p.lse && live) {
        // packed batches: [heads][sum of the samples' 256-row blocks], sample sg at row blk[sg] * 256
        size_t li;
        if constexpr (kPacked) li = (size_t)h * p.lse_stride + (size_t)seg.blk[*seg_slot] * (2 * kBM) + slot;
        else li = ((size_t)(b * p.G + g) * p.heads + h) * p.lse_stride + slot;
        if (index_ok(li, p.lse_elems, p.status)) p.lse[li] = m + __log2f(l);
      }
      if (part >= 0) {
        // split unit: unnormalised fp32 O (relative to m) and (m, l) for the combine kernel
        const size_t prow = ((size_t)(unit - p.n_full) * p.n_split + part) * (2 * kBM) + i * kBM + row;
        const bool in = live && index_ok(prow, p.ws_rows, p.status);
        float4* wo = reinterpret_cast<float4*>(p.ws_o + prow * D);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * cc, o);
          tmem_wait_ld();
          if (in) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              wo[8 * cc + v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                           __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
          }
        }
        if (in) p.ws_ml[prow] = make_float2(m, l);
      } else if (D >= 96 && !kPacked && om.use) {
        // TMA-store epilogue: the tile's rows go through a shared staging tile in the box layout
        // of the output map (the query map's view of o), and one thread stores the box; rows past
        // the set's end lie outside the map's extent and are not written.  Compiled for d >= 96
        // only (at d = 64 its presence alone slowed the softmax loop).
        if constexpr (D >= 96) {
        const uint32_t stg = sbase + C::kStgOff + (uint32_t)(i * C::kStgTileBytes);
        const uint32_t rb = stg + (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
        const bool issuer = (warp & 3) == 0 && lane == 0;
        for (int rd = 0; rd < C::kStgRounds; ++rd) {
          // the previous store from this staging tile has been read out
          if (stg_rounds > 0 && !warp_wait(bar(B_STGFREE + i), (uint32_t)((stg_rounds - 1) & 1), wc)) {
            ok = false;
            break;
          }
          const bool tail = D == 96 && rd == 1;   // channels 64 .. 95: 64-byte rows, SW64
          for (int cx = 0; cx < (tail ? 1 : 2); ++cx) {
            uint32_t o[32];
            tmem_ld32(tO + 64 * rd + 32 * cx, o);
            tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t pw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                pw[e] = pack_bf16x2(__uint_as_float(o[8 * v + 2 * e]) * inv_l, __uint_as_float(o[8 * v + 2 * e + 1]) * inv_l);
              // 16-byte chunk: SW128 chunk (4 cx + v) ^ (row & 7) of a 128-byte row, or SW64 chunk
              // v ^ ((row >> 1) & 3) of a 64-byte row
              const uint32_t addr = tail ? stg + (uint32_t)(row * 64) + 16u * (uint32_t)(v ^ ((row >> 1) & 3))
                                         : rb + 16u * (uint32_t)((4 * cx + v) ^ (row & 7));
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pw[0]), "r"(pw[1]),
                           "r"(pw[2]), "r"(pw[3])
                           : "memory");
            }
          }
#if OSP_BOUNDS_CHECK
          if (rd == 0 && live) {   // the row's natural-order output elements, as the per-row stores check them
            const int token = w.q_out0 + slot_token(p.layout, slot, g, p.k);
            const size_t ooff = (((size_t)b * p.N_q + token) * p.heads + h) * D;
            if (!index_ok(ooff + D - 1, p.o_elems, p.status)) stg_bad[i] = 1;
          }
#endif
          fence_proxy_async_smem();
          mbar_arrive(bar(B_STGFULL + i));
          if (issuer) {
            if (!mbar_wait(bar(B_STGFULL + i), (uint32_t)(stg_rounds & 1), wc)) {
              ok = false;
            } else {
              if (!stg_bad[i]) {
                const int row0 = w.q0 + i * kBM, chan = h * D + 64 * rd;
                const CUtensorMap* m = (D == 96 && rd == 1) ? &om.tail : &om.o;
                if (p.layout == 0) tma_store_3d(m, stg, chan, row0, b);
                else if (p.layout == 1) tma_store_4d(m, stg, chan, g, row0, b);
                else tma_store_5d(m, stg, chan, 0, g, row0 / p.k, b);
                bulk_commit();
                bulk_wait_read();
              }
              if (rd == C::kStgRounds - 1) stg_bad[i] = 0;
              mbar_arrive(bar(B_STGFREE + i));
            }
          }
          ++stg_rounds;
          if (!__all_sync(0xffffffffu, ok)) break;
        }
        if (!ok) break;
        }
      } else {
      const int token = w.q_out0 + slot_token(p.layout, live ? slot : 0, g, p.k);
      const size_t ooff = (((size_t)b * p.N_q + token) * p.heads + h) * D;
      const bool store = live && index_ok(ooff + D - 1, p.o_elems, p.status);
      uint4* dst = reinterpret_cast<uint4*>(p.o + ooff);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * cc, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (store) {
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[4 * cc + v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      }
    }
    tc_fence_before();
    mbar_arrive(bar(B_OFREE + i));   // O_i is read out: the next item's first PV may overwrite it
    jb += n_kv;
    }   // items
    if constexpr (D >= 96)
      if ((warp & 3) == 0 && lane == 0) bulk_wait_all();   // this tile's output stores are complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merges the n_split partials of every split unit: with m_s, l_s, O_s (O_s unnormalised,
// relative to 2^m_s, m in log2 units), M = max m_s, w_s = 2^(m_s - M):
//   O = sum_s w_s O_s / sum_s w_s l_s.
// One warp per query row; lanes cover the head's D channels.
template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p, int n_units) {
  constexpr int kPer = D / 32;
  const int wid = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (wid >= n_units * 2 * kBM) return;
  const int su = wid / (2 * kBM), r = wid % (2 * kBM);
  const int unit = p.n_full + su;
  const int qb = unit % p.qblocks, hb = unit / p.qblocks;
  const int h = hb % p.heads, bg = hb / p.heads;
  const int b = bg / p.G, g = bg % p.G;
  const int slot = qb * 2 * kBM + r;
  if (slot >= p.n_q) return;
  if (!index_ok(((size_t)su * p.n_split + p.n_split - 1) * (2 * kBM) + r, p.ws_rows, p.status)) return;
  float mmax = -INFINITY;
  for (int s = 0; s < p.n_split; ++s)
    mmax = fmaxf(mmax, p.ws_ml[((size_t)su * p.n_split + s) * (2 * kBM) + r].x);
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float lsum = 0.f;
  for (int s = 0; s < p.n_split; ++s) {
    const size_t prow = ((size_t)su * p.n_split + s) * (2 * kBM) + r;
    const float2 ml = p.ws_ml[prow];
    const float wgt = exp2f(ml.x - mmax);
    lsum += wgt * ml.y;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] += wgt * p.ws_o[prow * D + e * 32 + lane];
  }
  const float inv = 1.f / lsum;
  if (p.lse && lane == 0) {
    const size_t li = ((size_t)(b * p.G + g) * p.heads + h) * p.lse_stride + slot;
    if (index_ok(li, p.lse_elems, p.status)) p.lse[li] = mmax + __log2f(lsum);
  }
  const int token = p.q_row_base + slot_token(p.layout, slot, g, p.k);
  const size_t ooff = (((size_t)b * p.N_q + token) * p.heads + h) * D;
  if (!index_ok(ooff + D - 1, p.o_elems, p.status)) return;
  __nv_bfloat16* dst = p.o + ooff;
#pragma unroll
  for (int e = 0; e < kPer; ++e) dst[e * 32 + lane] = __float2bfloat16_rn(acc[e] * inv);
}

}  // namespace
}  // namespace osp
