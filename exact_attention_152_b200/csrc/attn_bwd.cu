// Exact attention backward for B200 (sm_100a): dQ, dK, dV from Q, K, V, O, dO
// and the forward's log-sum-exp, with the score matrix recomputed tile by tile
// on the tensor cores (tcgen05, accumulators in Tensor Memory) and never stored.
//
// What is computed (the pages name the backward pass as what FlashAttention 4
// still lacks -- FlashAttention 4 page, ja.linux-konsole.com, sections
// "重要ポイント" and "互換性と現状"; "FlashAttention-4：非対称ハードウェアスケーリング…" (sns.style),
// section 二 -- and give no formula): the chain rule through the forward
// definition of include/attn.h, per (b, h), query row i, visible key j:
//
//   P_ij  = exp(scale * <q_i, k_j> - LSE_i)
//   dP_ij = <dO_i, v_j>,   D_i = <dO_i, O_i>,   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i
//   dK_j  = scale * sum_i dS_ij q_i
//   dQ_i  = scale * sum_j dS_ij k_j
//
// Design (this library's, for sm_100a):
//  * Three launches: a row-sum kernel for D (and dQ's fp32 accumulator is
//    zeroed), the main kernel, and a kernel that scales and rounds dQ to BF16
//    (column intervals add the mask summaries and, when the workspace has
//    room, a one-CTA plan that orders the CTAs longest first).  D and the dQ
//    accumulator live in a caller-provided workspace.
//  * Main kernel: one CTA per (b, key/value head, 128-key block).  K and V of
//    the block stay in shared memory; the CTA walks every query tile (128
//    rows) of every query head that reads this key/value head (with a key
//    band such as causal, only the tiles whose queries see one of the block's
//    keys), loading Q (two stages) and dO (one stage, refilled between the
//    tile's dV GEMM and the next tile's dP^T GEMM) by TMA.  Shared memory at
//    d = 128: K, V, two Q stages, dO, dS and the dQ drain's staging, 32 KiB
//    each.
//  * Per query tile, five BF16 GEMMs on the tensor cores, all with M = 128
//    keys or queries:
//        S^T  = K Q^T          (keys x queries, TMEM columns [0, 128))
//        dP^T = V dO^T         (TMEM columns [128, 256))
//        dV  += P^T dO         (A = P^T straight from TMEM; TMEM [256, 256+d))
//        dK  += dS^T Q         (A = dS^T from TMEM;          TMEM [256+d, 256+2d))
//        dQ_i = dS K           (A = dS from shared memory, MN-major; TMEM [128, 128+d))
//    Because the tiles are computed transposed (keys on the TMEM lanes), P^T
//    and dS^T are the A operands of the dV and dK GEMMs as they stand.
//  * Warps 0-7 turn S^T and dP^T into P^T and dS^T (one key row per thread,
//    half of the query columns per warp).  S^T is taken into registers first
//    and its columns handed back at once, so the next tile's S^T GEMM runs
//    while the exponentials are computed; P^T and dS^T go back to TMEM as
//    BF16 pairs in the dP^T columns (each 32-query chunk as 16 columns of P^T
//    then 16 of dS^T), where dQ accumulates once dK has read them.  dS also
//    goes to shared memory for the dQ GEMM.  Warps 8-11 drain each dQ tile
//    from TMEM into the fp32 accumulator with TMA reduce-adds, 32 columns at a
//    time through two alternating staging slots.  Warp 12 loads (TMA), warp
//    13 issues the MMAs from one thread, in the order
//        S(0) dP(0) | S(t+1) | dV(t) dK(t) | dQ(t) | dP(t+1) | ...
//    so the tensor pipe has the next tile's S^T to compute while the
//    element-wise warps work on this one.
//  * Variants (template arguments): key band (causal, sliding windows) or
//    column intervals (attn_bwd_colmask; the query tiles every key of the
//    block hides form at most two ranges per head and are stepped over), and
//    packed variable-length batches (attn_bwd_varlen; per-sequence offsets,
//    ragged dK/dV stores).  Masked scores are cleared by one bit test each
//    against a per-key keep word.
//  * Every wait is bounded; a timeout sets this file's status word and the CTA
//    leaves its loops and exits cleanly.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "exp2.cuh"
#include "host_common.h"
#include "sm100.cuh"
#include "tmap.h"

namespace eab {

// Column-interval mask summaries (attn_fwd.cu): for each of the BHm mask rows
// and each 128-key block, two int4 -- (max lo1, min hi1, max lo2, min hi2) and
// (min lo1, max hi1, min lo2, max hi2), an empty interval counting as
// (INT_MAX, INT_MIN) -- written to sum ([BHm, ceil(Nk / 128), 2] int4).
int launch_colmask_summary(const int* mask, void* sum, long long BHm, int Nk, cudaStream_t stream);

namespace bwd {

constexpr int kBlockK = 128;  // keys per CTA (TMEM lanes of S^T, dP^T, dV, dK)
constexpr int kBlockQ = 128;  // queries per tile
constexpr int kWarpDrain = 8;
constexpr int kWarpLoad = 12;
constexpr int kWarpMma = 13;
constexpr int kNumThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kUnbounded = 1 << 30;  // "no bound" for a side of the key band
// mask kinds (kernel template argument): none; the key band i - wl <= j <= i + wr
// (causal: wl unbounded, wr = 0); the band plus column intervals (each key j
// hidden from query rows [lo1_j, hi1_j) and [lo2_j, hi2_j))
constexpr int kMaskNone = 0;
constexpr int kMaskBand = 1;
constexpr int kMaskCols = 2;

constexpr unsigned int kStatusTimeout = kStatusWordTimeout;
constexpr unsigned int kStatusSmemAlign = 4u;  // mapped to kStatusWordLaunch on the host

__device__ unsigned int g_status_bwd;

template <int D>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;       // 128 rows x 64 bf16
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;      // 2 stages
  static constexpr int kOffDO = 4 * kTileBytes;     // 1 stage: refilled between dV and the next dP^T
  static constexpr int kOffDS = 5 * kTileBytes;     // dS, 128 queries x 128 keys, MN-major
  static constexpr int kDSBytes = 2 * kBoxBytes;
  // dQ drain staging: per drain warp two 4 KiB slots (32 rows x 32 fp32)
  static constexpr int kOffStage = kOffDS + kDSBytes;
  static constexpr int kStageBytes = 4 * 2 * 4096;
  static constexpr int kOffRow = kOffStage + kStageBytes;  // per stage: LSE*log2e [128], D [128]
  static constexpr int kRowBytes = 2 * 2 * kBlockQ * 4;
  static constexpr int kNumBars = 16;
  static constexpr int kOffBar = kOffRow + kRowBytes;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr uint32_t kTmemDP = 128;
  static constexpr uint32_t kTmemDV = 256;
  static constexpr uint32_t kTmemDK = 256 + D;
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct BwdParams {
  const float* lse;    // [B*H, Nq], natural log (packed: [H, total_q])
  const float* dsum;   // D = rowsum(dO * O), [B*H, Nq] (packed: [total_q, H])
  float* dq_acc;       // [B*H, Nq, d] fp32 (packed: [total_q, H, d]), zeroed before the launch
  const int* cu_q;     // packed variable-length batch: sequence starts (B + 1), else null
  const int* cu_k;
  __nv_bfloat16* dk;   // packed outputs, for rows stored one by one at a sequence's end
  __nv_bfloat16* dv;
  // column intervals (kMaskCols): per key (lo1, hi1, lo2, hi2), [B * mask_heads, Nk];
  // per 128-key block two summaries, [B * mask_heads, n_kblocks, 2]
  const int4* colmask;
  const int4* colsum;
  int mask_heads;      // 1 or H
  // column intervals: CTA order, longest first within groups of key/value
  // heads (colmask_bwd_plan_kernel); null: the order of blockIdx
  const int* uperm;
  uint64_t timeout_ns;
  int Nq, Nk, H, group, n_kblocks, n_qtiles;  // packed: Nq, Nk = total_q, total_k
  int wl, wr;          // key band i - wl <= j <= i + wr (kUnbounded: no bound)
  float scale_log2;    // scale * log2(e)
  float scale;
};

template <int D>
struct Smem {
  uint8_t* base;
  uint32_t sbase;
  __device__ __forceinline__ uint32_t k() const { return sbase + Cfg<D>::kOffK; }
  __device__ __forceinline__ uint32_t v() const { return sbase + Cfg<D>::kOffV; }
  __device__ __forceinline__ uint32_t q(int s) const { return sbase + Cfg<D>::kOffQ + s * Cfg<D>::kTileBytes; }
  __device__ __forceinline__ uint32_t dout() const { return sbase + Cfg<D>::kOffDO; }
  __device__ __forceinline__ uint32_t ds() const { return sbase + Cfg<D>::kOffDS; }
  // -LSE * log2(e) of the stage's 128 query rows, then their D
  __device__ __forceinline__ float* lse2(int s) const {
    return reinterpret_cast<float*>(base + Cfg<D>::kOffRow) + s * 2 * kBlockQ;
  }
  __device__ __forceinline__ float* dsum(int s) const { return lse2(s) + kBlockQ; }
  __device__ __forceinline__ uint32_t bar(int i) const { return sbase + Cfg<D>::kOffBar + 8 * i; }
  __device__ __forceinline__ uint32_t kv_full() const { return bar(0); }
  __device__ __forceinline__ uint32_t q_full(int s) const { return bar(1 + s); }
  __device__ __forceinline__ uint32_t q_empty(int s) const { return bar(3 + s); }
  __device__ __forceinline__ uint32_t s_full() const { return bar(5); }
  __device__ __forceinline__ uint32_t dp_full() const { return bar(6); }
  __device__ __forceinline__ uint32_t p_ready() const { return bar(7); }
  __device__ __forceinline__ uint32_t dq_full() const { return bar(8); }
  __device__ __forceinline__ uint32_t dq_free() const { return bar(9); }
  __device__ __forceinline__ uint32_t done() const { return bar(10); }
  // the dQ GEMM has read dS from shared memory (the next dS may be written)
  __device__ __forceinline__ uint32_t ds_free() const { return bar(11); }
  // dS of the current tile is in shared memory (the dQ GEMM may start)
  __device__ __forceinline__ uint32_t ds_ready() const { return bar(12); }
  // the element-wise warps hold the tile's S^T in registers (its columns may
  // take the next tile's S^T)
  __device__ __forceinline__ uint32_t s_free() const { return bar(13); }
  // dO of the tile is in shared memory / has been read by dP^T and dV
  __device__ __forceinline__ uint32_t do_full() const { return bar(14); }
  __device__ __forceinline__ uint32_t do_empty() const { return bar(15); }
  __device__ __forceinline__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(base + Cfg<D>::kOffMisc);
  }
};

// The work of one CTA: key block j of key/value head bh_kv; iterations walk the
// group's query heads, and within each the query tiles i_lo .. i_lo +
// tiles_per_head - 1 that can see one of the block's keys.
struct Work {
  int bh_kv, j, b, hkv, i_lo, tiles_per_head, n_it;
  bool packed;   // a compile-time constant per kernel instance
  bool force;    // column intervals hide every tile: visit (head 0, i_lo) fully masked
  int Nq, Nk;    // packed: the sequence's lengths
  int q0, k0;    // packed: the sequence's first rows
  int n_qtiles;  // query tiles of the problem
  // lengths and first rows of this CTA's problem (dense: the launch's, from 0)
  __device__ __forceinline__ int nq(const BwdParams& p) const { return packed ? Nq : p.Nq; }
  __device__ __forceinline__ int nk(const BwdParams& p) const { return packed ? Nk : p.Nk; }
  __device__ __forceinline__ int row_q0() const { return packed ? q0 : 0; }
  __device__ __forceinline__ int row_k0() const { return packed ? k0 : 0; }
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const bool ok = mbar_wait(bar, parity, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// MMA issue (one thread), fully unrolled with immediate descriptor offsets.
// ---------------------------------------------------------------------------
template <int D, int KK>
struct Mma {
  // K-major A and B, K = d: 32 bytes per K step in a 128-byte row, a new
  // 64-column box every 4 steps (S^T = K Q^T, dP^T = V dO^T).
  __device__ __forceinline__ static void kmajor(uint32_t d, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                                uint32_t b_hi, uint32_t idesc) {
    if constexpr (KK < D / 16) {
      constexpr uint32_t off = ((KK >> 2) * Cfg<D>::kBoxBytes + (KK & 3) * 32) >> 4;
      mma_ss_imm<off, off, KK == 0 ? 0u : 1u>(d, a_lo, a_hi, b_lo, b_hi, idesc);
      Mma<D, KK + 1>::kmajor(d, a_lo, a_hi, b_lo, b_hi, idesc);
    }
  }
  // A and B both MN-major, K = 128 keys, 2048 bytes per K step: dQ = dS K.
  __device__ __forceinline__ static void mnmajor(uint32_t d, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                                 uint32_t b_hi, uint32_t idesc) {
    if constexpr (KK < kBlockK / 16) {
      constexpr uint32_t off = (KK * 2048) >> 4;
      mma_ss_imm<off, off, KK == 0 ? 0u : 1u>(d, a_lo, a_hi, b_lo, b_hi, idesc);
      Mma<D, KK + 1>::mnmajor(d, a_lo, a_hi, b_lo, b_hi, idesc);
    }
  }
};

// A from TMEM, B MN-major (rows of 16 queries = 2048 bytes per K step): dV
// (SUB = 0, A = P^T) and dK (SUB = 16, A = dS^T).  The element-wise warps write
// queries [64h + 32c, 64h + 32c + 32) as 16 columns of BF16 pairs at
// 64h + 32c + SUB, so the K step of queries [16KK, 16KK + 16) reads 8 columns
// at 64 (KK / 4) + 32 ((KK / 2) % 2) + 8 (KK % 2) + SUB.
template <int D, int KK, uint32_t SUB>
struct MmaTs {
  __device__ __forceinline__ static void run(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                             uint32_t idesc, uint32_t acc) {
    if constexpr (KK < kBlockQ / 16) {
      constexpr uint32_t a_off = (KK >> 2) * 64 + ((KK >> 1) & 1) * 32 + (KK & 1) * 8 + SUB;
      constexpr uint32_t b_off = (KK * 2048) >> 4;
      mma_ts_imm<a_off, b_off>(d, a_tmem, b_lo, b_hi, idesc, KK == 0 ? acc : 1u);
      MmaTs<D, KK + 1, SUB>::run(d, a_tmem, b_lo, b_hi, idesc, acc);
    }
  }
};

// Which (query head, query tile) iteration `it` works on.  Without column
// intervals: head it / tiles_per_head, tile i_lo + it % tiles_per_head.  With
// them, the query tiles of one head that every key of this block hides form at
// most two ranges (one per interval, from the block's summary), which the walk
// steps over; every role walks the same sequence, so they agree on it.
struct Walk {
  int hh, t;           // query head within the group, query tile
  int a1, b1, a2, b2;  // hidden tiles [a1, b1] and [a2, b2] of head hh (a > b: none)
};

// mask row of query head hh of the CTA's group
__device__ __forceinline__ int mask_row(const BwdParams& prm, const Work& w, int hh) {
  return w.b * prm.mask_heads + (prm.mask_heads == 1 ? 0 : w.hkv * prm.group + hh);
}

// Tiles t whose rows [128t, min(128t + 128, Nq)) lie inside [lo, hi) for every
// key of the block: lo = the block's max lo, hi = its min hi.
__device__ __forceinline__ void hidden_range(int lo, int hi, int Nq, int n_qtiles, int* a, int* b) {
  const long long first = lo <= 0 ? 0 : (static_cast<long long>(lo) + kBlockQ - 1) / kBlockQ;
  const long long last = hi >= Nq ? n_qtiles - 1 : static_cast<long long>(hi) / kBlockQ - 1;
  *a = static_cast<int>(first < n_qtiles ? first : n_qtiles);
  *b = static_cast<int>(last < n_qtiles - 1 ? last : n_qtiles - 1);
}

__device__ __forceinline__ void walk_head(Walk& k, const BwdParams& prm, const Work& w, int n_qtiles) {
  const int4 a = __ldg(prm.colsum + (static_cast<size_t>(mask_row(prm, w, k.hh)) * prm.n_kblocks + w.j) * 2);
  hidden_range(a.x, a.y, prm.Nq, n_qtiles, &k.a1, &k.b1);
  hidden_range(a.z, a.w, prm.Nq, n_qtiles, &k.a2, &k.b2);
}

// Visible tiles of head hh in [i_lo, i_hi]: the range minus the two hidden ones.
__device__ __forceinline__ int visible_count(const Walk& k, int i_lo, int i_hi) {
  auto inter = [](int a, int b, int c, int e) { const int lo = max(a, c), hi = min(b, e); return hi >= lo ? hi - lo + 1 : 0; };
  const int both = inter(max(k.a1, k.a2), min(k.b1, k.b2), i_lo, i_hi);
  return (i_hi - i_lo + 1) - inter(k.a1, k.b1, i_lo, i_hi) - inter(k.a2, k.b2, i_lo, i_hi) + both;
}

// Move (hh, t) forward to the first visible tile at or after it.
template <int MASK>
__device__ __forceinline__ void walk_settle(Walk& k, const BwdParams& prm, const Work& w, int n_qtiles) {
  if constexpr (MASK == kMaskCols) {
    if (w.force) return;
    const int i_hi = w.i_lo + w.tiles_per_head - 1;
    for (int guard = 0; guard <= prm.group; ++guard) {
      for (int rep = 0; rep < 2; ++rep) {
        if (k.t >= k.a1 && k.t <= k.b1) k.t = k.b1 + 1;
        if (k.t >= k.a2 && k.t <= k.b2) k.t = k.b2 + 1;
      }
      if (k.t <= i_hi || k.hh + 1 >= prm.group) break;
      ++k.hh;
      k.t = w.i_lo;
      walk_head(k, prm, w, n_qtiles);
    }
  } else {
    if (k.t >= w.i_lo + w.tiles_per_head) {
      ++k.hh;
      k.t = w.i_lo;
    }
  }
}

template <int MASK>
__device__ __forceinline__ void walk_start(Walk& k, const BwdParams& prm, const Work& w, int n_qtiles) {
  k.hh = 0;
  k.t = w.i_lo;
  k.a1 = k.a2 = 1;
  k.b1 = k.b2 = 0;
  if constexpr (MASK == kMaskCols) {
    if (!w.force) walk_head(k, prm, w, n_qtiles);
  }
  walk_settle<MASK>(k, prm, w, n_qtiles);
}

template <int MASK>
__device__ __forceinline__ void walk_next(Walk& k, const BwdParams& prm, const Work& w, int n_qtiles) {
  ++k.t;
  walk_settle<MASK>(k, prm, w, n_qtiles);
}

// Positions [lo, hi) of the 32 starting at base, as bits (bit i: base + i).
__device__ __forceinline__ uint32_t span_bits(long long lo, long long hi, long long base) {
  const long long a = max(lo - base, 0LL);
  const long long b = min(hi - base, 32LL);
  if (b <= a) return 0u;
  const uint32_t upto = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  return upto & ~((1u << a) - 1u);
}

// Tensor-map coordinates (column, row, head) in the map's dimension order:
// dense maps are [BH, N, d], packed maps [total, H, d].
__device__ __forceinline__ void load_rows(uint32_t dst, const CUtensorMap* tm, int col, int row, int head,
                                          bool packed, uint32_t bar) {
  if (packed) tma_load_3d(dst, tm, col, head, row, bar);
  else tma_load_3d(dst, tm, col, row, head, bar);
}


// ---------------------------------------------------------------------------
// The query tiles a CTA iterates over (w.bh_kv, w.j, w.b, w.hkv and the packed
// fields set): with a key band, the tiles whose queries i see a key j of the
// block, i - wl <= j <= i + wr; with column intervals, those minus the tiles
// every key of the block hides, per query head of the group.  A block no
// query sees still runs one fully masked tile, so dK = dV = 0 come out of TMEM.
template <int MASK>
__device__ __forceinline__ void work_extent(const BwdParams& prm, Work& w, int n_qtiles) {
  w.n_qtiles = n_qtiles;
  w.force = false;
  w.i_lo = 0;
  w.tiles_per_head = n_qtiles;
  if (MASK != kMaskNone) {
    const long long j0 = static_cast<long long>(w.j) * kBlockK;
    long long lo = 0, hi = n_qtiles - 1;
    if (prm.wr < kUnbounded && j0 - prm.wr > 0) lo = (j0 - prm.wr) / kBlockQ;
    if (prm.wl < kUnbounded) {
      const long long last = (j0 + kBlockK - 1 + prm.wl) / kBlockQ;
      if (last < hi) hi = last;
    }
    if (lo > hi) lo = hi = (lo < n_qtiles - 1 ? lo : n_qtiles - 1);
    w.i_lo = static_cast<int>(lo);
    w.tiles_per_head = static_cast<int>(hi - lo + 1);
  }
  w.n_it = prm.group * w.tiles_per_head;
  if constexpr (MASK == kMaskCols) {
    const int i_hi = w.i_lo + w.tiles_per_head - 1;
    int n = 0;
    Walk k;
    for (k.hh = 0; k.hh < prm.group; ++k.hh) {
      walk_head(k, prm, w, n_qtiles);
      n += visible_count(k, w.i_lo, i_hi);
    }
    w.force = n == 0;
    w.n_it = n > 0 ? n : 1;
  }
}

// Producer warp: K, V once; then Q, dO (TMA) and LSE, D (plain loads) per tile.
// ---------------------------------------------------------------------------
template <int D, int MASK>
__device__ __forceinline__ void producer_role(const Smem<D>& sm, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              const CUtensorMap* tm_do, const BwdParams& prm,
                                              const Work& w, int lane) {
  using C = Cfg<D>;
  if (lane == 0) {
    mbar_arrive_expect_tx(sm.kv_full(), 2 * C::kTileBytes);
#pragma unroll
    for (int b = 0; b < C::kBoxes; ++b) {
      const int kh = w.packed ? w.hkv : w.bh_kv;
      load_rows(sm.k() + b * C::kBoxBytes, tm_k, b * 64, w.row_k0() + w.j * kBlockK, kh, w.packed,
                sm.kv_full());
      load_rows(sm.v() + b * C::kBoxBytes, tm_v, b * 64, w.row_k0() + w.j * kBlockK, kh, w.packed,
                sm.kv_full());
    }
  }
  bool ok = true;
  int it = 0, n_q = 0, n_do = 0;  // tiles whose Q / dO loads were issued
  Walk wk;
  walk_start<MASK>(wk, prm, w, w.n_qtiles);
  for (; it < w.n_it; ++it) {
    if (it > 0) walk_next<MASK>(wk, prm, w, w.n_qtiles);
    const int s = it & 1;
    const uint32_t ph = (it >> 1) & 1;
    ok = warp_wait(sm.q_empty(s), ph ^ 1u, prm.timeout_ns);
    if (!ok) break;
    const int h = w.hkv * prm.group + wk.hh;  // query head within the batch entry
    const int bh = w.b * prm.H + h;
    const int q0 = wk.t * kBlockQ;
    const int qh = w.packed ? h : bh;
    // Q first (its transaction count raised without arriving), then the rows
    // below, so the copy does not wait behind their global loads; every lane
    // arrives once its rows are in shared memory
    if (lane == 0) {
      mbar_expect_tx(sm.q_full(s), C::kTileBytes);
#pragma unroll
      for (int b = 0; b < C::kBoxes; ++b)
        load_rows(sm.q(s) + b * C::kBoxBytes, tm_q, b * 64, w.row_q0() + q0, qh, w.packed, sm.q_full(s));
    }
    // -LSE * log2(e) per query row (rows past the sequence: -inf, so P = 0
    // there), and D.  Dense: both [B*H, Nq]; packed: LSE [H, total_q], D
    // [total_q, H].
    float* nl = sm.lse2(s);
    float* dd = sm.dsum(s);
    if (w.packed) {
      const size_t lse0 = static_cast<size_t>(h) * prm.Nq + w.q0;
      const size_t d0 = static_cast<size_t>(w.q0) * prm.H + h;
#pragma unroll
      for (int r = lane; r < kBlockQ; r += 32) {
        const int q = q0 + r;
        const bool in = q < w.Nq;
        nl[r] = in ? -prm.lse[lse0 + q] * kLog2e : -INFINITY;
        dd[r] = in ? prm.dsum[d0 + static_cast<size_t>(q) * prm.H] : 0.0f;
      }
    } else {
#pragma unroll
      for (int r = lane; r < kBlockQ; r += 32) {
        const int q = q0 + r;
        const bool in = q < prm.Nq;
        const size_t row = static_cast<size_t>(bh) * prm.Nq + q;
        nl[r] = in ? -prm.lse[row] * kLog2e : -INFINITY;
        dd[r] = in ? prm.dsum[row] : 0.0f;
      }
    }
    mbar_arrive(sm.q_full(s));
    ++n_q;
    // dO, single-buffered: once the previous tile's dV has read it
    ok = warp_wait(sm.do_empty(), (it & 1) ^ 1u, prm.timeout_ns);
    if (!ok) break;
    if (lane == 0) {
      mbar_arrive_expect_tx(sm.do_full(), C::kTileBytes);
#pragma unroll
      for (int b = 0; b < C::kBoxes; ++b)
        load_rows(sm.dout() + b * C::kBoxBytes, tm_do, b * 64, w.row_q0() + q0, qh, w.packed, sm.do_full());
    }
    ++n_do;
  }
  // never leave with a copy in flight: the last two Q loads and the last dO load
  if (lane == 0) {
    mbar_wait(sm.kv_full(), 0, prm.timeout_ns);
    for (int i = n_q > 2 ? n_q - 2 : 0; i < n_q; ++i)
      mbar_wait(sm.q_full(i & 1), (i >> 1) & 1, prm.timeout_ns);
    if (n_do > 0) mbar_wait(sm.do_full(), (n_do - 1) & 1, prm.timeout_ns);
    if (!ok) atomicOr(&g_status_bwd, kStatusTimeout);
  }
}

// ---------------------------------------------------------------------------
// MMA issuer: one thread.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void mma_role(const Smem<D>& sm, uint32_t tmem, const Work& w,
                                         uint64_t timeout) {
  using C = Cfg<D>;
  constexpr uint32_t id_sq = idesc_bf16_f32(kBlockK, kBlockQ, false, false);  // S^T, dP^T
  constexpr uint32_t id_kv = idesc_bf16_f32(kBlockK, D, false, true);         // dV, dK
  constexpr uint32_t id_q = idesc_bf16_f32(kBlockQ, D, true, true);           // dQ
  const uint64_t dk_ = sdesc_sw128(sm.k(), 16, 1024), dv_ = sdesc_sw128(sm.v(), 16, 1024);
  const uint64_t dq_ = sdesc_sw128(sm.q(0), 16, 1024), do_ = sdesc_sw128(sm.dout(), 16, 1024);
  // MN-major views: Q, dO and K as B operands along d; dS as the A operand
  const uint64_t qmn = sdesc_sw128(sm.q(0), C::kBoxBytes, 1024);
  const uint64_t domn = sdesc_sw128(sm.dout(), C::kBoxBytes, 1024);
  const uint64_t kmn = sdesc_sw128(sm.k(), C::kBoxBytes, 1024);
  const uint64_t dsmn = sdesc_sw128(sm.ds(), Cfg<D>::kBoxBytes, 1024);
  auto lo = [](uint64_t x) { return static_cast<uint32_t>(x); };
  auto hi = [](uint64_t x) { return static_cast<uint32_t>(x >> 32); };
  constexpr uint32_t kStageStep = C::kTileBytes >> 4;

  bool ok = mbar_wait(sm.kv_full(), 0, timeout) && mbar_wait(sm.q_full(0), 0, timeout);
  if (ok) {
    tc_fence_after();
    // the first tile's S^T = K Q^T and dP^T = V dO^T
    Mma<D, 0>::kmajor(tmem, lo(dk_), hi(dk_), lo(dq_), hi(dq_), id_sq);
    tc_commit(sm.s_full());
    ok = mbar_wait(sm.do_full(), 0, timeout);
  }
  if (ok) {
    tc_fence_after();
    Mma<D, 0>::kmajor(tmem + C::kTmemDP, lo(dv_), hi(dv_), lo(do_), hi(do_), id_sq);
    tc_commit(sm.dp_full());
  }
  for (int it = 0; ok && it < w.n_it; ++it) {
    const int s = it & 1, sn = s ^ 1;
    const bool next = it + 1 < w.n_it;
    if (next) {
      // the next tile's S^T, as soon as the element-wise warps hold this one's
      // in registers: it runs while they compute the exponentials
      ok = mbar_wait(sm.q_full(sn), ((it + 1) >> 1) & 1, timeout) && mbar_wait(sm.s_free(), it & 1, timeout);
      if (!ok) break;
      tc_fence_after();
      Mma<D, 0>::kmajor(tmem, lo(dk_), hi(dk_), lo(dq_) + sn * kStageStep, hi(dq_), id_sq);
      tc_commit(sm.s_full());
    }
    ok = mbar_wait(sm.p_ready(), it & 1, timeout);
    if (!ok) break;
    tc_fence_after();
    const uint32_t acc = it > 0 ? 1u : 0u;
    MmaTs<D, 0, 0>::run(tmem + C::kTmemDV, tmem + C::kTmemDP, lo(domn), hi(domn), id_kv, acc);
    tc_commit(sm.do_empty());  // dO may be refilled once dV has read it
    MmaTs<D, 0, 16>::run(tmem + C::kTmemDK, tmem + C::kTmemDP, lo(qmn) + s * kStageStep, hi(qmn), id_kv, acc);
    tc_commit(sm.q_empty(s));
    ok = mbar_wait(sm.ds_ready(), it & 1, timeout);
    if (!ok) break;
    tc_fence_after();
    // dQ into the dP^T columns, whose P^T and dS^T the two GEMMs above read
    // first (MMAs from one thread execute in issue order)
    Mma<D, 0>::mnmajor(tmem + C::kTmemDP, lo(dsmn), hi(dsmn), lo(kmn), hi(kmn), id_q);
    tc_commit(sm.dq_full());
    tc_commit(sm.ds_free());
    if (next) {
      // the next tile's dP^T, once dQ has left those columns and its dO is in
      ok = mbar_wait(sm.dq_free(), it & 1, timeout) && mbar_wait(sm.do_full(), (it + 1) & 1, timeout);
      if (!ok) break;
      tc_fence_after();
      Mma<D, 0>::kmajor(tmem + C::kTmemDP, lo(dv_), hi(dv_), lo(do_), hi(do_), id_sq);
      tc_commit(sm.dp_full());
    }
  }
  tc_commit(sm.done());
  mbar_wait(sm.done(), 0, timeout);
  if (!ok) atomicOr(&g_status_bwd, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// Warps 0-7: P^T and dS^T from S^T and dP^T.  Warp (c, q) owns TMEM lanes
// 32q..32q+31 (keys) and query columns [64c, 64c+64).
// ---------------------------------------------------------------------------
template <int D, int MASK>
__device__ __forceinline__ bool softmax_grad_role(const Smem<D>& sm, uint32_t tmem,
                                                  const BwdParams& prm, const Work& w) {
  using C = Cfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3, c = warp >> 2;
  const int r = q4 * 32 + lane;          // key row within the block
  const int key = w.j * kBlockK + r;
  const bool key_in = key < w.nk(prm);
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  const uint32_t tS = tmem + lane_off + c * 64;
  const uint32_t tP = tmem + lane_off + C::kTmemDP + c * 64;
  uint8_t* ds_row = sm.base + C::kOffDS + c * C::kBoxBytes + r * 128;
  bool ok = true;
  Walk wk;
  walk_start<MASK>(wk, prm, w, w.n_qtiles);
  int4 kiv = make_int4(0, 0, 0, 0);  // this thread's key intervals (column mask)
  int kiv_head = -1;
  for (int it = 0; it < w.n_it; ++it) {
    if (it > 0) walk_next<MASK>(wk, prm, w, w.n_qtiles);
    if (MASK == kMaskCols && wk.hh != kiv_head) {
      kiv_head = wk.hh;
      kiv = key_in ? __ldg(prm.colmask + static_cast<size_t>(mask_row(prm, w, wk.hh)) * prm.Nk + key)
                   : make_int4(0, 0, 0, 0);
    }
    const int s = it & 1;
    // q_full orders the producer's LSE / D rows of this stage before the reads
    // below (long complete by now); it cannot run two phases ahead, since the
    // stage is refilled only after this tile's p_ready.
    ok = warp_wait(sm.q_full(s), (it >> 1) & 1, prm.timeout_ns) &&
         warp_wait(sm.s_full(), it & 1, prm.timeout_ns);
    if (!ok) break;
    tc_fence_after();
    // this warp's 64 columns of S^T into registers; then the columns are free
    // for the next tile's S^T GEMM
    uint32_t sv[2][32];
    tmem_ld32(tS, sv[0]);
    tmem_ld32(tS + 32, sv[1]);
    tmem_ld_wait();
    reg_fence32(sv[0]);
    reg_fence32(sv[1]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.s_free());
    const int q_base = wk.t * kBlockQ + c * 64;  // first query of this warp's columns
    // masking: key tail, a band edge crossing this warp's 32 keys x 64 queries,
    // or a key interval meeting the warp's queries
    const int k_lo = w.j * kBlockK + q4 * 32;
    bool masked = !key_in || (MASK != kMaskNone && (k_lo + 31 - q_base > prm.wr || q_base + 63 - k_lo > prm.wl));
    if (MASK == kMaskCols) {
      const bool meets = (kiv.x < q_base + 64 && kiv.y > q_base && kiv.x < kiv.y) ||
                         (kiv.z < q_base + 64 && kiv.w > q_base && kiv.z < kiv.w);
      masked = masked || meets;
    }
    const float4* nl4 = reinterpret_cast<const float4*>(sm.lse2(s) + c * 64);
    const float4* dd4 = reinterpret_cast<const float4*>(sm.dsum(s) + c * 64);
    const float2 sl2 = make_float2(prm.scale_log2, prm.scale_log2);
    // P = exp2(scale log2(e) S - LSE log2(e)) in fp32, in place of S
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      // the queries of these 32 columns this key is visible to (bit c: query
      // q_base + 32k + c): inside the band key - wr <= q <= key + wl and outside
      // the key's column intervals; one bit test per score below instead of
      // the comparisons themselves
      uint32_t keep = 0xffffffffu;
      if (masked) {
        const long long base = q_base + 32 * k;
        keep = key_in ? span_bits(MASK != kMaskNone ? static_cast<long long>(key) - prm.wr : base,
                                  MASK != kMaskNone ? static_cast<long long>(key) + prm.wl + 1 : base + 32,
                                  base)
                      : 0u;
        if (MASK == kMaskCols) keep &= ~(span_bits(kiv.x, kiv.y, base) | span_bits(kiv.z, kiv.w, base));
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) {  // query columns 32k + 4g .. 32k + 4g + 3
        const float4 nl = nl4[8 * k + g];
        float2 xa = ffma2(make_float2(__uint_as_float(sv[k][4 * g]), __uint_as_float(sv[k][4 * g + 1])), sl2,
                          make_float2(nl.x, nl.y));
        float2 xb = ffma2(make_float2(__uint_as_float(sv[k][4 * g + 2]), __uint_as_float(sv[k][4 * g + 3])),
                          sl2, make_float2(nl.z, nl.w));
        if (masked) {
          const uint32_t kw = keep >> (4 * g);
          if (!(kw & 1u)) xa.x = -INFINITY;
          if (!(kw & 2u)) xa.y = -INFINITY;
          if (!(kw & 4u)) xb.x = -INFINITY;
          if (!(kw & 8u)) xb.y = -INFINITY;
        }
        float2 pa, pb;
        if ((g & 3) == 0) {  // a quarter of the exponentials on the FMA pipe
          pa = ex2_poly2(xa);
          pb = ex2_poly2(xb);
        } else {
          pa = make_float2(ex2_mufu(xa.x), ex2_mufu(xa.y));
          pb = make_float2(ex2_mufu(xb.x), ex2_mufu(xb.y));
        }
        sv[k][4 * g] = __float_as_uint(pa.x);
        sv[k][4 * g + 1] = __float_as_uint(pa.y);
        sv[k][4 * g + 2] = __float_as_uint(pb.x);
        sv[k][4 * g + 3] = __float_as_uint(pb.y);
      }
    }
    // dS = P (dP - D); P^T and dS^T back into the dP^T columns this warp has
    // just read, 16 columns each per 32-query chunk
    ok = warp_wait(sm.dp_full(), it & 1, prm.timeout_ns);
    if (!ok) break;
    tc_fence_after();
    uint32_t dsk[2][16];  // this thread's dS row (BF16 pairs), written to shared memory last
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint32_t pv[32];
      tmem_ld32(tP + 32 * k, pv);
      tmem_ld_wait();
      reg_fence32(pv);
      uint32_t pp[16];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float4 dv = dd4[8 * k + g];
        const float2 pa = make_float2(__uint_as_float(sv[k][4 * g]), __uint_as_float(sv[k][4 * g + 1]));
        const float2 pb = make_float2(__uint_as_float(sv[k][4 * g + 2]), __uint_as_float(sv[k][4 * g + 3]));
        const float2 da = fmul2(pa, fsub2(make_float2(__uint_as_float(pv[4 * g]), __uint_as_float(pv[4 * g + 1])),
                                          make_float2(dv.x, dv.y)));
        const float2 db = fmul2(pb, fsub2(make_float2(__uint_as_float(pv[4 * g + 2]),
                                                      __uint_as_float(pv[4 * g + 3])),
                                          make_float2(dv.z, dv.w)));
        pp[2 * g] = pack_bf16x2(pa.x, pa.y);
        pp[2 * g + 1] = pack_bf16x2(pb.x, pb.y);
        dsk[k][2 * g] = pack_bf16x2(da.x, da.y);
        dsk[k][2 * g + 1] = pack_bf16x2(db.x, db.y);
      }
      tmem_st16(tP + 32 * k, pp);
      tmem_st16(tP + 32 * k + 16, dsk[k]);
    }
    // P^T and dS^T are in TMEM: the dV and dK GEMMs may start
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.p_ready());
    // dS for the dQ GEMM, once the previous dQ GEMM has read the buffer: key
    // row r of the 64-query block c, 16-byte chunks, 128-byte swizzle
    if (it > 0 && !warp_wait(sm.ds_free(), (it - 1) & 1, prm.timeout_ns)) {
      ok = false;
      break;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int chunk = (4 * k + i) ^ (r & 7);
        *reinterpret_cast<uint4*>(ds_row + chunk * 16) =
            make_uint4(dsk[k][4 * i], dsk[k][4 * i + 1], dsk[k][4 * i + 2], dsk[k][4 * i + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.ds_ready());
  }
  return ok;
}

// Warps 8-11: dQ tile (queries on the TMEM lanes) -> fp32 accumulator by TMA
// reduce-add.  Each warp stages its 32 rows in 32-column x 32-row boxes
// (128-byte swizzle, 4 KiB) through two alternating slots of its own 8 KiB of
// staging; a slot is refilled once the reduction issued from it two boxes
// earlier has read it, so the next reduction is always queued behind the
// current one, across tiles too.  The reductions are bound by the SM's write
// path to L2 (about 25 bytes per clock), so they run on their own buffer,
// overlapping everything else.  TMEM is released (dq_free) as soon as the
// whole tile is in registers, so the next dP^T GEMM overlaps the reductions.
template <int D, int MASK>
__device__ __forceinline__ bool dq_drain_role(const Smem<D>& sm, uint32_t tmem, const CUtensorMap* tm_dq,
                                              const BwdParams& prm, const Work& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3;
  const uint32_t tQ = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + Cfg<D>::kTmemDP;
  uint8_t* stage = sm.base + Cfg<D>::kOffStage + q4 * 8192;
  const uint32_t stage_s = smem_u32(stage);
  constexpr int kBoxes = D / 32;
  bool ok = true;
  Walk wk;
  walk_start<MASK>(wk, prm, w, w.n_qtiles);
  for (int it = 0; it < w.n_it; ++it) {
    if (it > 0) walk_next<MASK>(wk, prm, w, w.n_qtiles);
    ok = warp_wait(sm.dq_full(), it & 1, prm.timeout_ns);
    if (!ok) break;
    tc_fence_after();
    const int h = w.hkv * prm.group + wk.hh;
    const int qh = w.packed ? h : w.b * prm.H + h;
    // rows past a packed sequence's end reduce exact zeros (P = 0 there) into
    // the next sequence's rows, which leaves them unchanged
    const int row0 = w.row_q0() + wk.t * kBlockQ + q4 * 32;
    // all of this warp's dQ columns into registers, then TMEM is free
    uint32_t v[kBoxes][32];
#pragma unroll
    for (int bx = 0; bx < kBoxes; ++bx) tmem_ld32(tQ + 32 * bx, v[bx]);
    tmem_ld_wait();
#pragma unroll
    for (int bx = 0; bx < kBoxes; ++bx) reg_fence32(v[bx]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.dq_free());
#pragma unroll
    for (int bx = 0; bx < kBoxes; ++bx) {
      const uint32_t slot = static_cast<uint32_t>(bx & 1) * 4096u;
      // the reduction issued from this slot two boxes ago has read it
      if (lane == 0) bulk_wait_group_read1();
      __syncwarp();
      uint8_t* row = stage + slot + lane * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(row + ((c ^ (lane & 7)) * 16)) =
            make_uint4(v[bx][4 * c], v[bx][4 * c + 1], v[bx][4 * c + 2], v[bx][4 * c + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (w.packed)
          tma_reduce_add_3d(tm_dq, stage_s + slot, 32 * bx, qh, row0);
        else
          tma_reduce_add_3d(tm_dq, stage_s + slot, 32 * bx, row0, qh);
        bulk_commit_group();
      }
    }
  }
  if (lane == 0) bulk_wait_group0();  // every reduction complete before the CTA exits
  return ok;
}

// Warps 0-7 after the last tile: dV and scale * dK -> BF16 -> shared memory ->
// TMA store.  d = 128: warp (c, q) stores output columns [64c, 64c+64) of both;
// d = 64: warp (0, q) stores dV, warp (1, q) stores dK.
template <int D>
__device__ __forceinline__ bool epilogue(const Smem<D>& sm, uint32_t tmem, const CUtensorMap* tm_dk,
                                         const CUtensorMap* tm_dv, const BwdParams& prm,
                                         const Work& w, bool ok) {
  using C = Cfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3, c = warp >> 2;
  ok = ok && warp_wait(sm.done(), 0, prm.timeout_ns);
  if (!ok) return false;
  tc_fence_after();
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  constexpr int kBoxesPerWarp = D == 128 ? 2 : 1;
  // a packed sequence ending inside this warp's 32 rows: a TMA store would
  // write into the next sequence, so each row stores itself
  const bool ragged = w.packed && w.j * kBlockK + q4 * 32 + 32 > w.Nk;
#pragma unroll
  for (int bx = 0; bx < kBoxesPerWarp; ++bx) {
    // which tensor and which 64 columns
    const bool is_k = D == 128 ? bx == 1 : c == 1;
    const int col0 = D == 128 ? c * 64 : 0;
    const uint32_t src = tmem + lane_off + (is_k ? C::kTmemDK : C::kTmemDV) + col0;
    const float mul = is_k ? prm.scale : 1.0f;
    // staging: 4 KiB per (warp, box) inside the Q stages (free by now)
    uint8_t* stage = sm.base + C::kOffQ + (warp * kBoxesPerWarp + bx) * 4096;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v[32];
      tmem_ld32(src + 32 * h, v);
      tmem_ld_wait();
      reg_fence32(v);
      uint32_t wv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        wv[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
      if (ragged) {
        const int key = w.j * kBlockK + q4 * 32 + lane;
        if (key < w.Nk) {
          const int hkv_all = prm.H / prm.group;
          __nv_bfloat16* out = (is_k ? prm.dk : prm.dv) +
                               (static_cast<size_t>(w.k0 + key) * hkv_all + w.hkv) * D + col0 + 32 * h;
          uint4* dst = reinterpret_cast<uint4*>(out);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int chunk = (4 * h + i) ^ (lane & 7);
          *reinterpret_cast<uint4*>(stage + lane * 128 + chunk * 16) =
              make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    const int row0 = w.j * kBlockK + q4 * 32;
    if (lane == 0 && !ragged && row0 < w.nk(prm)) {
      if (w.packed)
        tma_store_3d(is_k ? tm_dk : tm_dv, smem_u32(stage), col0, w.hkv, w.k0 + row0);
      else
        tma_store_3d(is_k ? tm_dk : tm_dv, smem_u32(stage), col0, row0, w.bh_kv);
      bulk_commit_group();
    }
  }
  if (lane == 0) bulk_wait_group0();
  return true;
}

template <int D, int MASK, bool PACKED>
__global__ void __launch_bounds__(kNumThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ BwdParams prm) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzled tiles need 1 KiB-aligned shared memory; there is no
  // room for alignment slack, so a misaligned window is reported, not used.
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(&g_status_bwd, kStatusSmemAlign);
    return;
  }
  Smem<D> sm;
  sm.base = smem_raw;
  sm.sbase = smem_u32(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  Work w;
  const int cta = (MASK == kMaskCols && prm.uperm != nullptr) ? __ldg(prm.uperm + blockIdx.x)
                                                              : static_cast<int>(blockIdx.x);
  w.bh_kv = cta / prm.n_kblocks;
  w.j = cta % prm.n_kblocks;
  const int hkv_per_b = prm.H / prm.group;
  w.b = w.bh_kv / hkv_per_b;
  w.hkv = w.bh_kv % hkv_per_b;
  // a compile-time constant in each instance, so the dense kernel carries none
  // of the packed layout's bookkeeping
  w.packed = PACKED;
  if (PACKED) {
    // packed variable-length batch: sequence b owns query rows cu_q[b] ..
    // cu_q[b+1]-1 and key rows cu_k[b] .. cu_k[b+1]-1.  Offsets that do not
    // describe sequences inside the tensors, or a key length beyond the grid,
    // are reported and the CTA does nothing (every access stays in bounds).
    const int a = __ldg(prm.cu_q + w.b), e = __ldg(prm.cu_q + w.b + 1);
    const int c = __ldg(prm.cu_k + w.b), f = __ldg(prm.cu_k + w.b + 1);
    if (a < 0 || e < a || e > prm.Nq || c < 0 || f < c || f > prm.Nk ||
        f - c > prm.n_kblocks * kBlockK) {
      if (threadIdx.x == 0 && w.j == 0 && w.hkv == 0) atomicOr(&g_status_bwd, kStatusWordBadSeqlens);
      return;
    }
    w.Nq = e - a;
    w.Nk = f - c;
    w.q0 = a;
    w.k0 = c;
    if (w.j * kBlockK >= w.Nk) return;  // this sequence has no key in the block
  } else {
    w.Nq = w.Nk = w.q0 = w.k0 = 0;  // unused: the launch's sizes apply
  }
  // query tiles (packed: at least one -- a sequence without queries still runs
  // one fully masked tile, so dK = dV = 0 come out of TMEM)
  const int n_qtiles = PACKED ? (w.Nq > 0 ? (w.Nq + kBlockQ - 1) / kBlockQ : 1) : prm.n_qtiles;
  work_extent<MASK>(prm, w, n_qtiles);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) {
      const uint32_t b = sm.bar(i);
      uint32_t count = 1;
      if (b == sm.q_full(0) || b == sm.q_full(1)) count = 32;  // every producer lane
      if (b == sm.p_ready() || b == sm.ds_ready() || b == sm.s_free()) count = 8;
      if (b == sm.dq_free()) count = 4;
      mbar_init(b, count);
    }
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(sm.tmem_slot()), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();

  // register split of the 512 x 128 launch budget: element-wise warpgroups 152
  // (P of 64 queries in fp32 while dP^T is read), the drain 160 (a whole dQ
  // row in registers), load/MMA 48 (2 x 128 x 152 + 128 x 160 + 128 x 48 = 65536)
  if (warp < kWarpDrain) {
    setmaxnreg_inc<152>();
    bool ok = softmax_grad_role<D, MASK>(sm, tmem, prm, w);
    ok = epilogue<D>(sm, tmem, &tm_dk, &tm_dv, prm, w, ok);
    if (!ok && lane == 0) atomicOr(&g_status_bwd, kStatusTimeout);
  } else if (warp < kWarpLoad) {
    setmaxnreg_inc<160>();
    const bool ok = dq_drain_role<D, MASK>(sm, tmem, &tm_dq, prm, w);
    if (!ok && lane == 0) atomicOr(&g_status_bwd, kStatusTimeout);
  } else {
    setmaxnreg_dec<48>();
    if (warp == kWarpLoad) {
      producer_role<D, MASK>(sm, &tm_q, &tm_k, &tm_v, &tm_do, prm, w, lane);
    } else if (warp == kWarpMma) {
      if (lane == 0) mma_role<D>(sm, tmem, w, prm.timeout_ns);
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// D_i = <dO_i, O_i> in fp32, one warp per row.
template <int D>
__global__ void row_dot_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                               float* __restrict__ dsum, size_t rows) {
  const int lane = threadIdx.x & 31;
  const size_t warps = static_cast<size_t>(gridDim.x) * (blockDim.x >> 5);
  for (size_t row = blockIdx.x * static_cast<size_t>(blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    float acc = 0.0f;
#pragma unroll
    for (int c = lane * 2; c < D; c += 64) {
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(o + row * D + c);
      const __nv_bfloat162 g = *reinterpret_cast<const __nv_bfloat162*>(dout + row * D + c);
      acc = fmaf(__low2float(a), __low2float(g), acc);
      acc = fmaf(__high2float(a), __high2float(g), acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dsum[row] = acc;
  }
}

// CTA order for column intervals: for every CTA (key/value head, key block)
// the query tiles it will visit (work_extent, as its prologue computes it),
// then a counting sort by (group of hgroup key/value heads, that number, most
// first): uperm[i] is the CTA index the i-th launched CTA takes.  A group's
// Q, dO and dQ accumulator are sized to stay in L2 together; longest first
// within it evens out the end of the launch.  CTAs of equal key keep no
// particular order; the results do not depend on it.  One CTA.
constexpr int kPlanThreads = 1024;
constexpr int kPlanMaxUnits = 8192;
constexpr int kPlanMaxBins = 4096;

__global__ void __launch_bounds__(kPlanThreads) colmask_bwd_plan_kernel(const BwdParams prm, int* __restrict__ uperm,
                                                                        int n_units, int hgroup, int max_n) {
  __shared__ uint16_t ubin[kPlanMaxUnits];
  __shared__ int off[kPlanMaxBins];
  __shared__ int wsum[kPlanThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int n_bh = n_units / prm.n_kblocks;
  const int n_bins = ((n_bh + hgroup - 1) / hgroup) * (max_n + 1);
  for (int i = t; i < n_bins; i += kPlanThreads) off[i] = 0;
  __syncthreads();
  const int hkv_per_b = prm.H / prm.group;
  for (int u = t; u < n_units; u += kPlanThreads) {
    Work w;
    w.bh_kv = u / prm.n_kblocks;
    w.j = u % prm.n_kblocks;
    w.b = w.bh_kv / hkv_per_b;
    w.hkv = w.bh_kv % hkv_per_b;
    w.packed = false;
    w.Nq = w.Nk = w.q0 = w.k0 = 0;
    work_extent<kMaskCols>(prm, w, prm.n_qtiles);
    const int bin = (w.bh_kv / hgroup) * (max_n + 1) + max_n - min(w.n_it, max_n);
    ubin[u] = static_cast<uint16_t>(bin);
    atomicAdd(&off[bin], 1);
  }
  __syncthreads();
  // exclusive prefix sum of the bin sizes: thread t owns bins [b0, b1)
  const int per = (n_bins + kPlanThreads - 1) / kPlanThreads;
  const int b0 = min(t * per, n_bins), b1 = min(b0 + per, n_bins);
  int run = 0;
  for (int b = b0; b < b1; ++b) run += off[b];
  int incl = run;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = wsum[lane];
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += v;
    }
    wsum[lane] = wi - w;
  }
  __syncthreads();
  int base = wsum[warp] + incl - run;
  for (int b = b0; b < b1; ++b) {
    const int c = off[b];
    off[b] = base;
    base += c;
  }
  __syncthreads();
  for (int u = t; u < n_units; u += kPlanThreads) uperm[atomicAdd(&off[ubin[u]], 1)] = u;
}

// dQ = BF16(scale * accumulator), 4 elements per thread per step.
__global__ void dq_finish_kernel(const float4* __restrict__ acc, uint2* __restrict__ dq, float scale,
                                 size_t n4) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = acc[i];
    dq[i] = make_uint2(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale));
  }
}

template <int D, int MASK, bool PACKED>
int launch_main(const CUtensorMap* maps, const BwdParams& prm, int grid, cudaStream_t stream) {
  auto kern = attn_bwd_kernel<D, MASK, PACKED>;
  static std::once_flag once[kMaxDeviceCount];
  static cudaError_t err[kMaxDeviceCount];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::call_once(once[dev], [&] {
    err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmemBytes);
  });
  if (err[dev] != cudaSuccess) return cuda_fail(err[dev], "cudaFuncSetAttribute");
  kern<<<grid, kNumThreads, Cfg<D>::kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4],
                                                          maps[5], maps[6], prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_bwd_kernel launch");
  return ATTN_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

size_t workspace_bytes(long long BH, long long Nq, int d) {
  return align256(static_cast<size_t>(BH) * Nq * 4) + static_cast<size_t>(BH) * Nq * d * 4;
}

// D rows, the main kernel and dQ's conversion, shared by the dense and packed
// entries once the tensor maps and parameters are set up.
int run_bwd(const CUtensorMap* maps, BwdParams& prm, const void* o, const void* dout, void* dq,
            size_t rows, int d, bool mask, int grid, cudaStream_t stream) {
  const bool cols = prm.colmask != nullptr;
  cudaError_t e = cudaMemsetAsync(prm.dq_acc, 0, rows * d * 4, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  {
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((rows + 7) / 8, 148 * 16));
    float* dsum = const_cast<float*>(prm.dsum);
    if (d == 128)
      row_dot_kernel<128><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                      static_cast<const __nv_bfloat16*>(dout), dsum, rows);
    else
      row_dot_kernel<64><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                     static_cast<const __nv_bfloat16*>(dout), dsum, rows);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "row_dot_kernel launch");
  }
  int rc;
  const bool packed = prm.cu_q != nullptr;
  if (d == 128) {
    if (cols)
      rc = launch_main<128, kMaskCols, false>(maps, prm, grid, stream);
    else if (packed)
      rc = mask ? launch_main<128, kMaskBand, true>(maps, prm, grid, stream)
                : launch_main<128, kMaskNone, true>(maps, prm, grid, stream);
    else
      rc = mask ? launch_main<128, kMaskBand, false>(maps, prm, grid, stream)
                : launch_main<128, kMaskNone, false>(maps, prm, grid, stream);
  } else {
    if (cols)
      rc = launch_main<64, kMaskCols, false>(maps, prm, grid, stream);
    else if (packed)
      rc = mask ? launch_main<64, kMaskBand, true>(maps, prm, grid, stream)
                : launch_main<64, kMaskNone, true>(maps, prm, grid, stream);
    else
      rc = mask ? launch_main<64, kMaskBand, false>(maps, prm, grid, stream)
                : launch_main<64, kMaskNone, false>(maps, prm, grid, stream);
  }
  if (rc != ATTN_OK) return rc;
  const size_t n4 = rows * d / 4;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n4 + 255) / 256, 148 * 32));
  dq_finish_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(prm.dq_acc),
                                               static_cast<uint2*>(dq), prm.scale, n4);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "dq_finish_kernel launch");
  return ATTN_OK;
}

// window_left / window_right: the key band of the forward (-1 = no bound).
// Column intervals of attn_bwd_colmask: int32 [B, Hm, Nk, 4]; their block
// summaries go to the end of the workspace.
struct ColMaskArgs {
  const int* mask;
  int Hm;
};

// Column intervals: attn_bwd's workspace, the block summaries (together the
// minimum), then room for the CTA plan, one int per (head, key block) (an
// upper bound: the CTAs are per key/value head).
size_t colmask_workspace_bytes(long long BH, long long Nq, int d, long long BHm, long long Nk) {
  return align256(workspace_bytes(BH, Nq, d)) + static_cast<size_t>(BHm * ((Nk + kBlockK - 1) / kBlockK)) * 32;
}
size_t colmask_plan_bytes(long long BH, long long Nk) {
  return (static_cast<size_t>(BH * ((Nk + kBlockK - 1) / kBlockK)) * 4 + 15) & ~static_cast<size_t>(15);
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
             int H, int Hkv, int Nq, int Nk, int d, float scale, int window_left, int window_right,
             cudaStream_t stream, const ColMaskArgs* cm = nullptr) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (H > 0 && (Hkv == 0 || H % Hkv != 0)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H, BHkv = static_cast<long long>(B) * Hkv;
  if (BH > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  const size_t q_bytes = static_cast<size_t>(BH) * Nq * d * 2;
  const size_t kv_bytes = static_cast<size_t>(BHkv) * Nk * d * 2;
  if (BH == 0 || (Nq == 0 && Nk == 0)) return ATTN_OK;
  const bool any_q = Nq > 0, any_k = Nk > 0;
  if ((any_q && (!q || !o || !dout || !lse || !dq)) || (any_k && (!k || !v || !dk || !dv)))
    return ATTN_ERR_INVALID_ARG;
  if (cm && cm->Hm != 1 && cm->Hm != H) return ATTN_ERR_INVALID_ARG;
  const long long BHm = cm ? static_cast<long long>(B) * cm->Hm : 0;
  size_t need = cm ? colmask_workspace_bytes(BH, Nq, d, BHm, Nk) : workspace_bytes(BH, Nq, d);
  if (any_q && any_k && (!workspace || ws_bytes < need)) return ATTN_ERR_INVALID_ARG;
  // column intervals: the longest-first CTA plan when the workspace has room for it
  int plan_hgroup = 0, plan_max_n = 0;
  long long plan_units = 0;
  if (cm && any_q && any_k) {
    const long long n_kb = (static_cast<long long>(Nk) + kBlockK - 1) / kBlockK;
    const long long n_qt = (static_cast<long long>(Nq) + kBlockQ - 1) / kBlockQ;
    const long long group = H / Hkv, hkv_per_b = Hkv;
    // key/value heads per group: the largest divisor of a batch entry's whose
    // query heads' Q, dO (BF16) and fp32 dQ accumulator fit in ~48 MiB
    const long long per_kv = group * static_cast<long long>(Nq) * d * 8;
    long long g = 1;
    for (long long c = 1; c <= hkv_per_b; ++c)
      if (hkv_per_b % c == 0 && c * per_kv <= (48LL << 20)) g = c;
    plan_units = BHkv * n_kb;
    const long long max_n = group * n_qt;
    const long long bins = ((BHkv + g - 1) / g) * (max_n + 1);
    if (plan_units <= kPlanMaxUnits && bins <= kPlanMaxBins && ws_bytes >= need + plan_units * 4) {
      plan_hgroup = static_cast<int>(g);
      plan_max_n = static_cast<int>(max_n);
      need += static_cast<size_t>(plan_units) * 4;  // the region written
    }
  }
  if (cm && any_k && (!cm->mask || misaligned(cm->mask, 16))) return ATTN_ERR_INVALID_ARG;
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16) ||
      misaligned(dout, 16) || misaligned(dq, 16) || misaligned(dk, 16) || misaligned(dv, 16) ||
      misaligned(lse, 4) || misaligned(workspace, 256))
    return ATTN_ERR_INVALID_ARG;
  // outputs may not overlap each other, any input, or the workspace
  const size_t lse_bytes = static_cast<size_t>(BH) * Nq * 4;
  const size_t mask_bytes = static_cast<size_t>(BHm) * Nk * 16;
  const void* ins[7] = {q, k, v, o, dout, lse, cm ? cm->mask : nullptr};
  const size_t in_bytes[7] = {q_bytes, kv_bytes, kv_bytes, q_bytes, q_bytes, lse_bytes, mask_bytes};
  void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {q_bytes, kv_bytes, kv_bytes, any_q && any_k ? need : 0};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 7; ++b)
      if (ranges_overlap(outs[a], out_bytes[a], ins[b], in_bytes[b])) return ATTN_ERR_INVALID_ARG;
    for (int b = a + 1; b < 4; ++b)
      if (ranges_overlap(outs[a], out_bytes[a], outs[b], out_bytes[b])) return ATTN_ERR_INVALID_ARG;
  }
  const long long n_kblocks = (Nk + kBlockK - 1) / kBlockK;
  if (n_kblocks * BHkv > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != ATTN_OK) return rc;

  cudaError_t e;
  // no keys: every gradient is 0 (O = 0 does not depend on the inputs);
  // no queries: dK = dV = 0
  if (!any_k || !any_q) {
    if (any_q && (e = cudaMemsetAsync(dq, 0, q_bytes, stream)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    if (any_k && (e = cudaMemsetAsync(dk, 0, kv_bytes, stream)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    if (any_k && (e = cudaMemsetAsync(dv, 0, kv_bytes, stream)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    return ATTN_OK;
  }

  CUtensorMap maps[7];
  const int bh = static_cast<int>(BH), bhkv = static_cast<int>(BHkv);
  if (!make_tmap_bf16_3d(&maps[0], q, bh, Nq, d, kBlockQ, &t_last_error) ||
      !make_tmap_bf16_3d(&maps[1], k, bhkv, Nk, d, kBlockK, &t_last_error) ||
      !make_tmap_bf16_3d(&maps[2], v, bhkv, Nk, d, kBlockK, &t_last_error) ||
      !make_tmap_bf16_3d(&maps[3], dout, bh, Nq, d, kBlockQ, &t_last_error) ||
      !make_tmap_bf16_3d(&maps[4], dk, bhkv, Nk, d, 32, &t_last_error) ||
      !make_tmap_bf16_3d(&maps[5], dv, bhkv, Nk, d, 32, &t_last_error))
    return ATTN_ERR_CUDA;

  float* dsum = static_cast<float*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           align256(static_cast<size_t>(BH) * Nq * 4));
  if (!make_tmap_f32_3d(&maps[6], dq_acc, bh, Nq, d, 32, &t_last_error)) return ATTN_ERR_CUDA;

  BwdParams prm = {};
  prm.lse = lse;
  prm.dsum = dsum;
  prm.dq_acc = dq_acc;
  prm.timeout_ns = kWaitTimeoutNs;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.H = H;
  prm.group = H / Hkv;
  prm.n_kblocks = static_cast<int>(n_kblocks);
  prm.n_qtiles = (Nq + kBlockQ - 1) / kBlockQ;
  prm.wl = window_left < 0 ? kUnbounded : std::min(window_left, kUnbounded);
  prm.wr = window_right < 0 ? kUnbounded : std::min(window_right, kUnbounded);
  const bool mask = prm.wl < kUnbounded || prm.wr < kUnbounded;
  prm.scale_log2 = scale * kLog2e;
  prm.scale = scale;
  if (cm) {
    void* sum = static_cast<uint8_t*>(workspace) + align256(workspace_bytes(BH, Nq, d));
    prm.colmask = reinterpret_cast<const int4*>(cm->mask);
    prm.colsum = static_cast<const int4*>(sum);
    prm.mask_heads = cm->Hm;
    rc = launch_colmask_summary(cm->mask, sum, BHm, Nk, stream);
    if (rc != ATTN_OK) return rc;
    if (plan_hgroup > 0) {
      int* uperm = reinterpret_cast<int*>(static_cast<uint8_t*>(sum) + static_cast<size_t>(BHm * n_kblocks) * 32);
      colmask_bwd_plan_kernel<<<1, kPlanThreads, 0, stream>>>(prm, uperm, static_cast<int>(plan_units), plan_hgroup,
                                                              plan_max_n);
      const cudaError_t pe = cudaGetLastError();
      if (pe != cudaSuccess) return cuda_fail(pe, "colmask_bwd_plan_kernel launch");
      prm.uperm = uperm;
    }
  }
  return run_bwd(maps, prm, o, dout, dq, static_cast<size_t>(BH) * Nq, d, mask,
                 static_cast<int>(n_kblocks * BHkv), stream);
}

// Packed variable-length batch: q, o, dout, dq [total_q, H, d]; k, v, dk, dv
// [total_k, Hkv, d]; lse [H, total_q]; device offsets cu_q, cu_k.  Positions
// count from 0 within each sequence (the band is applied to them).
int bwd_varlen_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                    const int* cu_q, const int* cu_k, int num_seqs, int max_seqlen_k, int total_q,
                    int total_k, int H, int Hkv, int d, float scale, int window_left,
                    int window_right, cudaStream_t stream) {
  if (num_seqs < 0 || max_seqlen_k < 0 || total_q < 0 || total_k < 0 || H < 0 || Hkv < 0)
    return ATTN_ERR_INVALID_ARG;
  if (H > 0 && (Hkv == 0 || H % Hkv != 0)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_k > total_k) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (num_seqs == 0 || H == 0 || (total_q == 0 && total_k == 0)) return ATTN_OK;
  const bool any_q = total_q > 0, any_k = total_k > 0;
  if (any_k && max_seqlen_k == 0) return ATTN_ERR_INVALID_ARG;  // keys exist but no sequence may hold one
  if ((any_q && (!q || !o || !dout || !lse || !dq)) || (any_k && (!k || !v || !dk || !dv)) ||
      !cu_q || !cu_k)
    return ATTN_ERR_INVALID_ARG;
  const size_t need = workspace_bytes(H, total_q, d);
  if (any_q && any_k && (!workspace || ws_bytes < need)) return ATTN_ERR_INVALID_ARG;
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16) ||
      misaligned(dout, 16) || misaligned(dq, 16) || misaligned(dk, 16) || misaligned(dv, 16) ||
      misaligned(lse, 4) || misaligned(workspace, 256) || misaligned(cu_q, 4) || misaligned(cu_k, 4))
    return ATTN_ERR_INVALID_ARG;
  const size_t q_bytes = static_cast<size_t>(total_q) * H * d * 2;
  const size_t kv_bytes = static_cast<size_t>(total_k) * Hkv * d * 2;
  const size_t lse_bytes = static_cast<size_t>(total_q) * H * 4;
  const size_t cu_bytes = (static_cast<size_t>(num_seqs) + 1) * 4;
  const void* ins[8] = {q, k, v, o, dout, lse, cu_q, cu_k};
  const size_t in_bytes[8] = {q_bytes, kv_bytes, kv_bytes, q_bytes, q_bytes, lse_bytes, cu_bytes, cu_bytes};
  void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {q_bytes, kv_bytes, kv_bytes, any_q && any_k ? need : 0};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 8; ++b)
      if (ranges_overlap(outs[a], out_bytes[a], ins[b], in_bytes[b])) return ATTN_ERR_INVALID_ARG;
    for (int b = a + 1; b < 4; ++b)
      if (ranges_overlap(outs[a], out_bytes[a], outs[b], out_bytes[b])) return ATTN_ERR_INVALID_ARG;
  }
  const long long n_kblocks = (static_cast<long long>(max_seqlen_k) + kBlockK - 1) / kBlockK;
  const long long BHkv = static_cast<long long>(num_seqs) * Hkv;
  if (static_cast<long long>(num_seqs) * H > 0x7fffffffLL || n_kblocks * BHkv > 0x7fffffffLL)
    return ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != ATTN_OK) return rc;

  cudaError_t e;
  if (!any_k || !any_q) {
    if (any_q && (e = cudaMemsetAsync(dq, 0, q_bytes, stream)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    if (any_k && (e = cudaMemsetAsync(dk, 0, kv_bytes, stream)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    if (any_k && (e = cudaMemsetAsync(dv, 0, kv_bytes, stream)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    return ATTN_OK;
  }
  CUtensorMap maps[7];
  float* dsum = static_cast<float*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           align256(static_cast<size_t>(H) * total_q * 4));
  if (!make_tmap_bf16_packed(&maps[0], q, total_q, H, d, kBlockQ, &t_last_error) ||
      !make_tmap_bf16_packed(&maps[1], k, total_k, Hkv, d, kBlockK, &t_last_error) ||
      !make_tmap_bf16_packed(&maps[2], v, total_k, Hkv, d, kBlockK, &t_last_error) ||
      !make_tmap_bf16_packed(&maps[3], dout, total_q, H, d, kBlockQ, &t_last_error) ||
      !make_tmap_bf16_packed(&maps[4], dk, total_k, Hkv, d, 32, &t_last_error) ||
      !make_tmap_bf16_packed(&maps[5], dv, total_k, Hkv, d, 32, &t_last_error) ||
      !make_tmap_f32_packed(&maps[6], dq_acc, total_q, H, d, 32, &t_last_error))
    return ATTN_ERR_CUDA;

  BwdParams prm = {};
  prm.lse = lse;
  prm.dsum = dsum;
  prm.dq_acc = dq_acc;
  prm.cu_q = cu_q;
  prm.cu_k = cu_k;
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.timeout_ns = kWaitTimeoutNs;
  prm.Nq = total_q;
  prm.Nk = total_k;
  prm.H = H;
  prm.group = H / Hkv;
  prm.n_kblocks = static_cast<int>(n_kblocks);
  prm.n_qtiles = 0;  // per sequence
  prm.wl = window_left < 0 ? kUnbounded : std::min(window_left, kUnbounded);
  prm.wr = window_right < 0 ? kUnbounded : std::min(window_right, kUnbounded);
  const bool mask = prm.wl < kUnbounded || prm.wr < kUnbounded;
  prm.scale_log2 = scale * kLog2e;
  prm.scale = scale;
  return run_bwd(maps, prm, o, dout, dq, static_cast<size_t>(total_q) * H, d, mask,
                 static_cast<int>(n_kblocks * BHkv), stream);
}

// attn_bwd_noalloc: the same computation with its workspace in a file-scope
// device array, so the call itself allocates no memory.
constexpr size_t kStaticScratchBytes = size_t(96) << 20;  // 96 MiB per device
__device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];

// Device address of g_bwd_scratch in the current context.  The address
// belongs to the copy of this module loaded into one context: a new context on
// the same device (after cudaDeviceReset, or one the caller made current) loads
// the module again, possibly elsewhere.  So the address is cached per device
// together with the unique ID of the context it was looked up in, and looked up
// again (cudaGetSymbolAddress: a lookup, no allocation) whenever that ID
// changes or cannot be read (current_context_id, host_common.h).
int static_scratch(void** ptr) {
  static std::mutex mu;
  static void* addr[kMaxDeviceCount];
  static unsigned long long ctx_id[kMaxDeviceCount];
  static bool cached[kMaxDeviceCount];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDeviceCount) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  unsigned long long id = 0;
  if (current_context_id(&id) && cached[dev] && ctx_id[dev] == id) {
    *ptr = addr[dev];
    return ATTN_OK;
  }
  void* a = nullptr;
  e = cudaGetSymbolAddress(&a, g_bwd_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
  addr[dev] = a;
  // the lookup made the device's context current if none was: read its ID now
  cached[dev] = current_context_id(&ctx_id[dev]);
  *ptr = a;
  return ATTN_OK;
}

}  // namespace bwd

int bwd_status_take(cudaStream_t stream, unsigned int* status) {
  unsigned int st = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&st, bwd::g_status_bwd, sizeof(st), 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return cuda_fail(e, "read backward status word");
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbolAsync(bwd::g_status_bwd, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, "clear backward status word");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  // a misaligned shared-memory window is a launch problem, reported as CUDA
  if (st & bwd::kStatusSmemAlign) {
    t_last_error = "attn_bwd_kernel: dynamic shared memory not 1 KiB aligned";
    st = (st & ~bwd::kStatusSmemAlign) | kStatusWordLaunch;
  }
  *status = st;
  return ATTN_OK;
}

}  // namespace eab

extern "C" {

size_t attn_bwd_workspace_size(int B, int H, int Nq, int d) {
  if (B < 0 || H < 0 || Nq < 0 || (d != 64 && d != 128)) return 0;
  return eab::bwd::workspace_bytes(static_cast<long long>(B) * H, Nq, d);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, void* workspace,
             size_t workspace_bytes, int B, int H, int Hkv, int Nq, int Nk, int d, float scale,
             int causal, cudaStream_t stream) {
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (causal && Nq != Nk) return ATTN_ERR_UNSUPPORTED;
  return eab::bwd::bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv,
                            Nq, Nk, d, scale, -1, causal ? 0 : -1, stream);
}

int attn_bwd_window(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, int B, int H, int Hkv, int Nq, int Nk, int d,
                    float scale, int window_left, int window_right, cudaStream_t stream) {
  return eab::bwd::bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv,
                            Nq, Nk, d, scale, window_left, window_right, stream);
}

size_t attn_bwd_colmask_workspace_size(int B, int H, int Nq, int d, int Hm, int Nk) {
  if (B < 0 || H < 0 || Nq < 0 || Hm < 0 || Nk < 0 || (d != 64 && d != 128)) return 0;
  return eab::bwd::colmask_workspace_bytes(static_cast<long long>(B) * H, Nq, d,
                                           static_cast<long long>(B) * Hm, Nk) +
         eab::bwd::colmask_plan_bytes(static_cast<long long>(B) * H, Nk);
}

int attn_bwd_colmask(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, void* workspace,
                     size_t workspace_bytes, int B, int H, int Hkv, int Nq, int Nk, int d, float scale,
                     int causal, const int* mask, int Hm, cudaStream_t stream) {
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  const eab::bwd::ColMaskArgs cm = {mask, Hm};
  return eab::bwd::bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv,
                            Nq, Nk, d, scale, -1, causal ? 0 : -1, stream, &cm);
}

int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, const int* cu_seqlens_q, const int* cu_seqlens_k,
                    int num_seqs, int max_seqlen_k, int total_q, int total_k, int H, int Hkv, int d,
                    float scale, int window_left, int window_right, cudaStream_t stream) {
  return eab::bwd::bwd_varlen_impl(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes,
                                   cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_k, total_q,
                                   total_k, H, Hkv, d, scale, window_left, window_right, stream);
}

int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int B, int H, int Hkv, int Nq,
                     int Nk, int d, float scale, int causal, cudaStream_t stream) {
  // sizes beyond the static scratch are refused before anything else happens
  if (B >= 0 && H >= 0 && Nq >= 0 && (d == 64 || d == 128) &&
      eab::bwd::workspace_bytes(static_cast<long long>(B) * H, Nq, d) > eab::bwd::kStaticScratchBytes)
    return ATTN_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (causal && Nq != Nk) return ATTN_ERR_UNSUPPORTED;
  void* ws = nullptr;
  const int rc = eab::bwd::static_scratch(&ws);
  if (rc != ATTN_OK) return rc;
  return eab::bwd::bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, ws, eab::bwd::kStaticScratchBytes, B, H,
                            Hkv, Nq, Nk, d, scale, -1, causal ? 0 : -1, stream);
}

}  // extern "C"
