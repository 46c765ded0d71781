// Exact attention forward for B200 (sm_100a): TMA producer, tcgen05 MMAs with
// accumulators in Tensor Memory, online softmax with adaptive rescaling and a
// MUFU / FMA-pipe split of exp2, causal tile skipping.  Plus the C-ABI entry
// points declared in include/attn.h.
//
// Method (what the pages describe; they print no formulas or code):
//  * Tiling through on-chip memory so the Nq x Nk score matrix never reaches
//    device memory, with a running per-row max and sum (online softmax):
//    "Flash Attention（Flash Attention）" (jisaku.com glossary), sections "タイリングによるSRAMの活用"
//    and "オンライン・ソフトマックスと再計算"; FlashAttention 4 page
//    (ja.linux-konsole.com), section "なぜアテンションカーネルがまだLLMのコストを
//    支配しているのか".
//  * Warp roles -- load, tensor-core MMA, softmax, rescale, store -- each with
//    its own asynchronous pipeline: FlashAttention 4 page, section
//    "FlashAttention 4の新機能".
//  * exp2 partly evaluated as a cubic polynomial on the FMA pipe to relieve the
//    few SFUs: same page, section "CUDAコアによるソフトウェアの指数演算";
//    "FlashAttention-4：非対称ハードウェアスケーリング…" (sns.style), section 二.
//  * Rescaling only when the new max is sufficiently larger than the old one:
//    FlashAttention 4 page, section "よりスマートなオンラインソフトマックス再スケーリング".
//  * Fully asynchronous MMA with Tensor Memory: "FlashAttention-4：非対称ハードウェア
//    スケーリング…" (sns.style), section 二.
//
// Design (this library's, for sm_100a):
//  * One CTA owns two 128-row query tiles of one (b, h) -- 256 rows -- and
//    streams the head's K/V tiles (128 keys each) through a ring of shared
//    memory stages filled by TMA.  Q, K and V are read through 3-D tensor maps
//    [B*H, N, d] so out-of-range rows of one head read as zeros, never as the
//    next head's data.
//  * 12 warps.  Warps 0-7 do softmax, correction and epilogue, one thread per
//    query row: tile t uses warpgroup t (warps 4t..4t+3), and warp (t, q) owns
//    TMEM lanes 32q..32q+31 (its 32 rows) with all 128 key columns of each S
//    tile and all d output columns.  A row's scores sit in one thread's
//    registers, so its max needs no exchange between threads.  Warp 8: TMA
//    producer.  Warp 9: TMEM allocation and the single MMA-issuing thread.
//    Warps 10-11 idle (they complete the third warpgroup for the setmaxnreg
//    split 232 / 40).
//  * Tensor Memory (512 columns): S0 [0,128), S1 [128,256), O0 and O1 after
//    column 256.  P (BF16 pairs; E4M3 quadruples) overwrites the first columns
//    of its tile's S and is the A operand of O += P V straight from TMEM, so P
//    never touches shared memory.
//  * The MMA thread issues, per KV tile j:  O0 += P0 V_{j-1};  S0 = Q0 K_j^T;
//    O1 += P1 V_{j-1};  S1 = Q1 K_j^T.  Each O += P V is issued in four
//    chunks of 32 keys, each as soon as the softmax warps have stored that
//    chunk of P, so only the last chunk sits between a tile's softmax and its
//    next S.  The
//    commit that announces S_t(j) also covers O_t += P_t V_{j-1}, so when a
//    softmax warp sees S_t(j) its O_t is final up to tile j-1 and it can
//    rescale O_t in place without another wait.
//  * MMAs are issued from fully unrolled code with descriptor offsets as
//    immediates: the tensor core queues about one MMA ahead, so every cycle
//    the issuing thread spends between MMAs is a cycle the tensor core idles.
//    For the same reason the issuer looks at the barrier of its next MMA group
//    (non-blocking) before issuing the current one, and K_j / V_{j-1} arrive
//    on a single barrier per step.
//  * Masks: the key tail, a key band i - wl <= j <= i + wr (causal, sliding
//    windows), and column intervals (attn_fwd_colmask: each key hidden from up
//    to two query-row intervals).  KV tiles outside the band are never
//    visited; under column intervals a per-CTA bitmap, built from per-block
//    summaries, lists the tiles some row sees, and a one-CTA plan kernel
//    orders the CTAs by those counts, longest first within each mask row.  A
//    warp whose 64 x 32 block is cut by a mask folds it into two 32-bit keep
//    words per row and tests one bit per score.
//  * Every wait is bounded (see sm100.cuh); a timeout sets the per-device
//    status word and the CTA leaves its loops and exits cleanly.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "attn.h"
#include "exp2.cuh"
#include "sm100.cuh"
#include "host_common.h"
#include "tmap.h"

namespace eab {

constexpr int kBlockM = 128;  // query rows per tile  (= TMEM lanes)
constexpr int kBlockN = 128;  // keys per KV tile
constexpr int kRowsPerCta = 2 * kBlockM;
// 3 warpgroups: one softmax warpgroup per query tile (warps 4t .. 4t+3) and one
// for the TMA producer (warp 8), the MMA issuer (warp 9) and two idle warps
// that complete the group for the register split.
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
constexpr int kNumThreads = 384;
// setmaxnreg split of the 384 x 168 launch budget: 256 x 232 + 128 x 40 = 64512.
// The host refuses to launch a build whose register count at launch is lower
// (setmaxnreg.inc would wait for registers that are not there).
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 232;
constexpr int kProducerRegs = 40;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kProducerRegs <= kNumThreads * kLaunchRegs,
              "register split exceeds the launch budget");
constexpr int kPChunks = 4;  // P published in chunks of 32 keys
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s per pipeline wait
constexpr float kDefaultThreshold = 8.0f;           // powers of two
constexpr int kDefaultPoly16 = 4;                   // exp2 columns (of 16) on the FMA pipe
// E4M3 P: the exponent is raised by kP8Offset powers of two and the rescale
// threshold lowered to kP8Tau, so P stays within [0, 2^(kP8Tau + kP8Offset)] =
// [0, 256] (E4M3 saturates at 448) while small weights keep 4 more binades
// above E4M3's smallest subnormal.  Both cancel in O / l; LSE subtracts the offset.
constexpr float kP8Offset = 4.0f;
constexpr float kP8Tau = 4.0f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

constexpr unsigned int kStatusTimeout = kStatusWordTimeout;
constexpr unsigned int kStatusBadSeqlens = kStatusWordBadSeqlens;
// "no bound" for a side of the key band; large enough for any sequence, small
// enough that row +- bound stays inside int.
constexpr int kUnbounded = 1 << 30;

// Mask kinds (kernel template argument).  kMaskBand: the key band
// i - wl <= j <= i + wr (causal is wl unbounded, wr = 0).  kMaskCols: the band
// plus a column-interval mask -- per key column j up to two query-row
// intervals [lo1, hi1) and [lo2, hi2) that do not see key j -- with key blocks
// that hide all of a CTA's rows skipped altogether.
constexpr int kMaskNone = 0;
constexpr int kMaskBand = 1;
constexpr int kMaskCols = 2;
constexpr int kMaxMaskBlocks = 65536;  // key blocks per sequence under a column-interval mask

// Per-device status word (each device holds its own copy of module globals).
__device__ unsigned int g_status;

// F8: Q, K, V (and P) in E4M3 bytes instead of BF16.
template <int D, bool F8>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(!F8 || D == 128, "E4M3 inputs: d = 128 (one 128-byte row)");
  static constexpr int kElem = F8 ? 1 : 2;          // bytes per element
  static constexpr int kBoxCols = 128 / kElem;      // elements per 128-byte swizzle row
  static constexpr int kBoxes = D / kBoxCols;       // 128-byte swizzle boxes across d
  static constexpr int kBoxBytes = kBlockM * 128;   // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kKStep = 32 / kElem;         // MMA K per instruction (32 bytes)
  static constexpr int kStages = F8 ? 6 : (D == 64 ? 8 : 4);  // K/V ring depth
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  // BF16 O of one tile (128 rows x d) is staged for its TMA store in that
  // tile's Q buffer when it fits (BF16 inputs: same size); E4M3 Q tiles are
  // half as large, so O gets its own area after the K/V ring.
  static constexpr int kOTileBytes = kBlockM * D * 2;
  static constexpr int kOffO = F8 ? kOffKV + kStages * kTileBytes : kOffQ;
  static constexpr int kOffBar = F8 ? kOffO + 2 * kOTileBytes : kOffKV + kStages * kTileBytes;
  static constexpr int kNumKvSteps = 4;  // step barriers, used round robin
  static constexpr int kNumBars = 2 + kStages + kNumKvSteps + 2 + 2 * kPChunks + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffSeq = (kOffMisc + 16 + 15) / 16 * 16;  // this CTA's SeqView
  static constexpr int kSeqBytes = 64;
  // column-interval mask: one bit per 128-key block, set when the block is
  // visited (kMaxMaskBlocks blocks = 8M keys)
  static constexpr int kOffVis = kOffSeq + kSeqBytes;
  static constexpr int kVisBytes = kMaxMaskBlocks / 8;
  static constexpr int kSmemBytes = kOffVis + kVisBytes + 1024;  // + slack for 1 KiB alignment
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static constexpr uint32_t kTmemO = 256;
};

struct FwdParams {
  float* lse;
  unsigned long long* rescale_count;
  __nv_bfloat16* o;  // output base (packed layout: ragged row blocks are stored directly)
  const int* cu_q;   // packed variable-length batch: sequence starts (num_seqs + 1), else null
  const int* cu_k;
  uint64_t timeout_ns;
  int Nq, Nk;        // dense: sequence lengths; packed: total_q, total_k
  int BH, n_qblocks; // grid = BH * n_qblocks (packed: BH = num_seqs * H)
  int H, group;      // query heads per batch; query heads per key/value head
  int wl, wr;        // key band: i - wl <= j <= i + wr (kUnbounded: no bound)
  int grouped;       // causal band: heads in L2-sized groups, heaviest blocks first
  int hgroup;        // heads scheduled together (their K/V fit in L2)
  float scale_log2;  // scale * log2(e) (E4M3: times the Q and K scale factors)
  float tau;         // rescale threshold, powers of two
  float o_scale;     // multiplies O / l (E4M3: the V scale factor; else 1)
  // column-interval mask (kMaskCols): per key column (lo1, hi1, lo2, hi2),
  // [B * mask_heads, Nk]; per 128-key block two summaries,
  // [B * mask_heads, n_kblocks, 2] (see colmask_summary_kernel)
  const int4* colmask;
  const int4* colsum;
  int mask_heads;    // 1 (one mask for all heads of a batch entry) or H
  int n_kblocks;     // key blocks per head: ceil(Nk / 128)
  // column-interval mask: CTA order by (mask row, query block) units, most
  // visited key blocks first (colmask_plan_kernel); null: the order below
  const int* uperm;
};

// Where one CTA's sequence lives: lengths, first packed row (packed layout),
// tensor-map head coordinates and the KV tile range it visits.
struct SeqView {
  int Nq, Nk;        // this sequence's lengths
  int q0, k0;        // first row of the sequence in the packed layout (0 dense)
  int head_q, head_kv;  // tensor-map head coordinate of Q/O and of K/V
  int j_lo, n_kv;    // KV tiles visited: n_kv of them from j_lo on (consecutive
                     // unless a column-interval mask skips some)
  int mrow;          // column-interval mask: row of [B * mask_heads] to use
  bool packed;
  float* lse_row0;   // LSE of this sequence's row 0 (null: not computed)
};

// Tensor-map coordinates (column, row, head) -> the map's dimension order:
// dense maps are [BH, N, d], packed maps [total, H, d].
__device__ __forceinline__ void tma_load_rows(uint32_t dst, const CUtensorMap* tm, int col, int row,
                                              int head, bool packed, uint32_t bar) {
  if (packed) tma_load_3d(dst, tm, col, head, row, bar);
  else tma_load_3d(dst, tm, col, row, head, bar);
}

// Column-interval mask, block summaries (colmask_summary_kernel):
//   a = (max lo1, min hi1, max lo2, min hi2) over the block's keys, with an
//       empty interval counting as (INT_MAX, INT_MIN): one interval of every
//       key hides rows [r0, r1) iff a.x <= r0 && a.y >= r1 (or a.z / a.w);
//   b = (min lo1, max hi1, min lo2, max hi2): no key's interval meets [r0, r1)
//       iff b.y <= r0 || b.x >= r1 (and likewise b.z / b.w).
__device__ __forceinline__ bool cols_hide_all(const FwdParams& prm, int mrow, int blk, int r0,
                                              int r1) {
  const int4 a = __ldg(prm.colsum + (static_cast<size_t>(mrow) * prm.n_kblocks + blk) * 2);
  return (a.x <= r0 && a.y >= r1) || (a.z <= r0 && a.w >= r1);
}
__device__ __forceinline__ bool cols_touch(const FwdParams& prm, int mrow, int blk, int r0,
                                           int r1) {
  const int4 b = __ldg(prm.colsum + (static_cast<size_t>(mrow) * prm.n_kblocks + blk) * 2 + 1);
  return !(b.y <= r0 || b.x >= r1) || !(b.w <= r0 || b.z >= r1);
}

// KV tiles [j_lo, j_hi) that hold a key of the band for some of the rows of
// query block qb; a block whose band holds none still visits one tile (fully
// masked: O = 0, LSE = -inf).
template <int MASK>
__device__ __forceinline__ void kv_band_range(const FwdParams& prm, int Nq, int Nk, int qb, int* lo,
                                              int* hi) {
  const int n_all = max((Nk + kBlockN - 1) / kBlockN, 1);
  int j_lo = 0, j_hi = n_all;
  if (MASK != kMaskNone) {
    // rows and bounds are below 2^31 and 2^30: the sums stay inside 64 bits
    const long long r_lo = static_cast<long long>(qb) * kRowsPerCta;
    const long long r_end = r_lo + kRowsPerCta < Nq ? r_lo + kRowsPerCta : Nq;
    const long long r_hi = r_end - 1;
    if (prm.wr < kUnbounded) {
      const long long last = (r_hi + prm.wr) / kBlockN + 1;
      if (last < j_hi) j_hi = static_cast<int>(last);
    }
    if (prm.wl < kUnbounded && r_lo - prm.wl > 0) j_lo = static_cast<int>((r_lo - prm.wl) / kBlockN);
    if (j_lo >= j_hi) {
      j_lo = min(j_lo, n_all - 1);
      j_hi = j_lo + 1;
    }
  }
  *lo = j_lo;
  *hi = j_hi;
}

// Query rows [r0, r1) of a CTA's block qb (r1 clipped to the sequence).
__device__ __forceinline__ int cta_row_end(int qb, int Nq) {
  const long long e = static_cast<long long>(qb) * kRowsPerCta + kRowsPerCta;
  return e < Nq ? static_cast<int>(e) : Nq;
}

// KV tile visited after tile blk (first: blk = j_lo - 1).  Column-interval
// mask: the next set bit of the CTA's visited-block bitmap in shared memory
// (written once by warp 0; every role reads the same bits, so they agree on
// the sequence without communicating).  The caller asks only for tiles that
// exist (n_kv of them), so the search ends inside the bitmap.
template <int MASK>
__device__ __forceinline__ int next_block(const uint32_t* vis, int blk) {
  ++blk;
  if constexpr (MASK == kMaskCols) {
    int wi = blk >> 5;
    uint32_t bits = vis[wi] & (0xffffffffu << (blk & 31));
    while (bits == 0u && wi < kMaxMaskBlocks / 32 - 1) bits = vis[++wi];
    blk = wi * 32 + __ffs(bits) - 1;
  }
  return blk;
}

// Positions [lo, hi) of the 32 starting at base, as bits (bit i: base + i).
__device__ __forceinline__ uint32_t span_bits(long long lo, long long hi, long long base) {
  const long long a = max(lo - base, 0LL);
  const long long b = min(hi - base, 32LL);
  if (b <= a) return 0u;
  const uint32_t upto = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  return upto & ~((1u << a) - 1u);
}

// ---------------------------------------------------------------------------
// Shared-memory / barrier map of one CTA
// ---------------------------------------------------------------------------
template <int D, bool F8>
struct Smem {
  uint8_t* base;
  uint32_t sbase;
  __device__ __forceinline__ uint32_t q(int t) const { return sbase + Cfg<D, F8>::kOffQ + t * Cfg<D, F8>::kTileBytes; }
  __device__ __forceinline__ uint32_t kv(int s) const { return sbase + Cfg<D, F8>::kOffKV + s * Cfg<D, F8>::kTileBytes; }
  __device__ __forceinline__ uint32_t bar(int i) const { return sbase + Cfg<D, F8>::kOffBar + 8 * i; }
  __device__ __forceinline__ uint32_t q_full(int t) const { return bar(t); }
  // K/V slot s free again (its last reader, an MMA, has completed)
  __device__ __forceinline__ uint32_t kv_empty(int s) const { return bar(2 + s); }
  // MMA step j (0 .. n_kv): V(j-1) and K(j) both resident.  One barrier per
  // step instead of one per tile halves the MMA thread's waits on data.
  __device__ __forceinline__ uint32_t kvp(int j) const {
    return bar(2 + Cfg<D, F8>::kStages + (j % Cfg<D, F8>::kNumKvSteps));
  }
  __device__ __forceinline__ uint32_t s_full(int t) const {
    return bar(2 + Cfg<D, F8>::kStages + Cfg<D, F8>::kNumKvSteps + t);
  }
  // chunk k of P_t (keys [32k, 32k+32)) written to TMEM by all 4 warps of the
  // tile (chunk 0 also marks O_t as rescaled)
  __device__ __forceinline__ uint32_t p_full(int t, int k) const {
    return bar(4 + Cfg<D, F8>::kStages + Cfg<D, F8>::kNumKvSteps + kPChunks * t + k);
  }
  __device__ __forceinline__ uint32_t o_full(int t) const {
    return bar(4 + Cfg<D, F8>::kStages + Cfg<D, F8>::kNumKvSteps + 2 * kPChunks + t);
  }
  __device__ __forceinline__ uint32_t mma_done() const {
    return bar(6 + Cfg<D, F8>::kStages + Cfg<D, F8>::kNumKvSteps + 2 * kPChunks);
  }
  __device__ __forceinline__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(base + Cfg<D, F8>::kOffMisc);
  }
  // kept in shared memory rather than registers: the softmax warps need most of
  // it only in the epilogue
  __device__ __forceinline__ SeqView* seq() const {
    return reinterpret_cast<SeqView*>(base + Cfg<D, F8>::kOffSeq);
  }
  __device__ __forceinline__ uint32_t* vis() const {
    return reinterpret_cast<uint32_t*>(base + Cfg<D, F8>::kOffVis);
  }
};

// Warp-uniform bounded wait: every lane waits, and the warp agrees on the
// outcome so warp-collective tcgen05 instructions are never split.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const bool ok = mbar_wait(bar, parity, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// Producer: one thread, TMA loads of Q0, K0, Q1, V0, K1, V1, ...
// ---------------------------------------------------------------------------
template <int D, int MASK, bool F8>
__device__ __forceinline__ void producer_role(const Smem<D, F8>& sm, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              const SeqView& sv, const FwdParams& prm, int qb,
                                              uint64_t timeout) {
  using C = Cfg<D, F8>;
  uint32_t it = 0;
  auto load_q = [&](int t) {
    mbar_arrive_expect_tx(sm.q_full(t), C::kTileBytes);
#pragma unroll
    for (int b = 0; b < C::kBoxes; ++b)
      tma_load_rows(sm.q(t) + b * C::kBoxBytes, tm_q, b * C::kBoxCols, sv.q0 + qb * kRowsPerCta + t * kBlockM,
                    sv.head_q, sv.packed, sm.q_full(t));
  };
  auto wait_slot = [&](uint32_t& slot) -> bool {
    slot = it % C::kStages;
    const uint32_t phase = (it / C::kStages) & 1u;
    ++it;
    return mbar_wait(sm.kv_empty(slot), phase ^ 1u, timeout);
  };
  auto issue_kv = [&](const CUtensorMap* tm, int j, uint32_t slot, uint32_t pbar) {
#pragma unroll
    for (int b = 0; b < C::kBoxes; ++b)
      tma_load_rows(sm.kv(slot) + b * C::kBoxBytes, tm, b * C::kBoxCols, sv.k0 + j * kBlockN, sv.head_kv,
                    sv.packed, pbar);
  };

  const uint32_t* vis = sm.vis();
  int blk = next_block<MASK>(vis, sv.j_lo - 1);
  uint32_t s_k = 0, s_v = 0;
  load_q(0);
  bool ok = wait_slot(s_k);
  if (ok) {
    mbar_arrive_expect_tx(sm.kvp(0), C::kTileBytes);
    issue_kv(tm_k, blk, s_k, sm.kvp(0));
  }
  load_q(1);
  int prev = blk;
  int steps = ok ? 1 : 0;
  for (int j = 1; ok && j < sv.n_kv; ++j) {
    blk = next_block<MASK>(vis, blk);
    // V(j-1) and K(j) complete one barrier together
    ok = wait_slot(s_v) && wait_slot(s_k);
    if (!ok) break;
    mbar_arrive_expect_tx(sm.kvp(j), 2 * C::kTileBytes);
    issue_kv(tm_v, prev, s_v, sm.kvp(j));
    issue_kv(tm_k, blk, s_k, sm.kvp(j));
    prev = blk;
    ++steps;
  }
  if (ok) {
    ok = wait_slot(s_v);
    if (ok) {
      mbar_arrive_expect_tx(sm.kvp(sv.n_kv), C::kTileBytes);
      issue_kv(tm_v, prev, s_v, sm.kvp(sv.n_kv));
      ++steps;
    }
  }

  // Never leave the CTA with a copy in flight: wait for the latest steps
  // (immediate on the normal path).
  for (int i = steps > C::kNumKvSteps ? steps - C::kNumKvSteps : 0; i < steps; ++i)
    mbar_wait(sm.kvp(i), (i / C::kNumKvSteps) & 1, timeout);
  mbar_wait(sm.q_full(0), 0, timeout);
  mbar_wait(sm.q_full(1), 0, timeout);
  if (!ok) atomicOr(&g_status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// MMA issuer: one thread.
// ---------------------------------------------------------------------------
template <int D, bool F8, int KK>
struct MmaUnroll {
  // S = Q K^T, K steps KK .. : 32 bytes along the 128-byte row, a new box
  // every 4 steps (BF16: 16 elements per step; E4M3: 32).
  __device__ __forceinline__ static void s(uint32_t d, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                           uint32_t b_hi, uint32_t idesc) {
    if constexpr (KK < D / Cfg<D, F8>::kKStep) {
      constexpr uint32_t off = ((KK >> 2) * Cfg<D, F8>::kBoxBytes + (KK & 3) * 32) >> 4;
      if constexpr (F8)
        mma_ss_imm_f8<off, off, KK == 0 ? 0u : 1u>(d, a_lo, a_hi, b_lo, b_hi, idesc);
      else
        mma_ss_imm<off, off, KK == 0 ? 0u : 1u>(d, a_lo, a_hi, b_lo, b_hi, idesc);
      MmaUnroll<D, F8, KK + 1>::s(d, a_lo, a_hi, b_lo, b_hi, idesc);
    }
  }
  // O += P V for P chunk CH (keys [32CH, 32CH+32)).  P of key pair / quad c
  // sits in TMEM column c of the tile (BF16: two keys per column, E4M3: four),
  // so K step s reads columns [8s, 8s+8) either way.  BF16: 16 keys per step,
  // steps 2CH and 2CH+1, V rows of 16 keys = 2048 bytes per 64-column box.
  // E4M3: 32 keys per step, step CH, V rows of 32 keys = 4096 bytes.  KK
  // counts the steps of the chunk.
  template <int CH>
  __device__ __forceinline__ static void o(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                           uint32_t idesc, uint32_t acc) {
    constexpr int kSteps = F8 ? 1 : 2;
    if constexpr (KK < kSteps) {
      constexpr int step = CH * kSteps + KK;
      constexpr uint32_t a_off = step * 8;
      constexpr uint32_t b_off = (step * (F8 ? 4096 : 2048)) >> 4;
      if constexpr (F8)
        mma_ts_imm_f8<a_off, b_off>(d, a_tmem, b_lo, b_hi, idesc, (CH == 0 && KK == 0) ? acc : 1u);
      else
        mma_ts_imm<a_off, b_off>(d, a_tmem, b_lo, b_hi, idesc, (CH == 0 && KK == 0) ? acc : 1u);
      MmaUnroll<D, F8, KK + 1>::template o<CH>(d, a_tmem, b_lo, b_hi, idesc, acc);
    }
  }
};

// ---------------------------------------------------------------------------
// MMA issuer: one thread.  The tensor core queues only about one MMA ahead of
// the issuing thread, and a look at an mbarrier costs this thread ~50 cycles
// alone and over 100 while TMA and the MMAs keep shared memory busy, so every
// blocking look between two MMA groups idles the tensor core.  The thread
// therefore starts a non-blocking look (test_wait) at the barrier the NEXT
// group needs before it issues the current group, and only falls back to a
// bounded blocking wait if that look failed.  Data for a step, V_{j-1} and
// K_j, arrives on one barrier per step.
// ---------------------------------------------------------------------------
template <int D, bool F8>
__device__ __forceinline__ void mma_role(const Smem<D, F8>& sm, uint32_t tmem, int n_kv,
                                         uint64_t timeout) {
  using C = Cfg<D, F8>;
  constexpr uint32_t idesc_s = F8 ? idesc_e4m3_f32(kBlockM, kBlockN, false, false)
                                  : idesc_bf16_f32(kBlockM, kBlockN, false, false);
  constexpr uint32_t idesc_o = F8 ? idesc_e4m3_f32(kBlockM, D, false, true)
                                  : idesc_bf16_f32(kBlockM, D, false, true);
  uint32_t it = 0;  // position in the K0, V0, K1, V1, ... ring order

  auto next_slot = [&](uint32_t& slot) {
    slot = it % C::kStages;
    ++it;
  };
  auto wait_step = [&](int j) -> bool { return mbar_wait(sm.kvp(j), (j / C::kNumKvSteps) & 1, timeout); };
  // descriptors as 32-bit halves; stage and tile offsets go into the low word
  const uint64_t dq = sdesc_sw128(sm.q(0), 16, 1024);
  const uint64_t dk = sdesc_sw128(sm.kv(0), 16, 1024);
  const uint64_t dv = sdesc_sw128(sm.kv(0), C::kBoxBytes, 1024);
  const uint32_t q_lo = static_cast<uint32_t>(dq), q_hi = static_cast<uint32_t>(dq >> 32);
  const uint32_t k_lo = static_cast<uint32_t>(dk), k_hi = static_cast<uint32_t>(dk >> 32);
  const uint32_t v_lo = static_cast<uint32_t>(dv), v_hi = static_cast<uint32_t>(dv >> 32);
  constexpr uint32_t kTileStep = C::kTileBytes >> 4;
  auto mma_s = [&](int t, uint32_t slot) {
    MmaUnroll<D, F8, 0>::s(tmem + t * kBlockM, q_lo + t * kTileStep, q_hi, k_lo + slot * kTileStep,
                       k_hi, idesc_s);
  };
  // settle a look taken earlier: block only if it failed
  auto settle = [&](bool seen, uint32_t bar, uint32_t par) -> bool {
    return seen || mbar_wait(bar, par, timeout);
  };
  // O_t += P_t V in four chunks; the next chunk's barrier is looked at before
  // the current chunk is issued.  `pre` is the look at chunk 0 taken earlier
  // (while the previous S group was issued).
  auto mma_o = [&](int t, uint32_t slot, bool acc, uint32_t par, bool pre) -> bool {
    const uint32_t d = tmem + C::kTmemO + t * D, a = tmem + t * kBlockM;
    const uint32_t b_lo = v_lo + slot * kTileStep;
    if (!settle(pre, sm.p_full(t, 0), par)) return false;
    tc_fence_after();
    bool nx = mbar_test(sm.p_full(t, 1), par);
    MmaUnroll<D, F8, 0>::template o<0>(d, a, b_lo, v_hi, idesc_o, acc ? 1u : 0u);
    if (!settle(nx, sm.p_full(t, 1), par)) return false;
    tc_fence_after();
    nx = mbar_test(sm.p_full(t, 2), par);
    MmaUnroll<D, F8, 0>::template o<1>(d, a, b_lo, v_hi, idesc_o, 1u);
    if (!settle(nx, sm.p_full(t, 2), par)) return false;
    tc_fence_after();
    nx = mbar_test(sm.p_full(t, 3), par);
    MmaUnroll<D, F8, 0>::template o<2>(d, a, b_lo, v_hi, idesc_o, 1u);
    if (!settle(nx, sm.p_full(t, 3), par)) return false;
    tc_fence_after();
    MmaUnroll<D, F8, 0>::template o<3>(d, a, b_lo, v_hi, idesc_o, 1u);
    return true;
  };

  uint32_t sK = 0, sV = 0;
  next_slot(sK);
  bool ok = mbar_wait(sm.q_full(0), 0, timeout) && wait_step(0);
  if (ok) {
    tc_fence_after();
    mma_s(0, sK);
    tc_commit(sm.s_full(0));
    ok = mbar_wait(sm.q_full(1), 0, timeout);
  }
  bool pk = false, pp = false;
  if (ok) {
    tc_fence_after();
    if (n_kv > 1) pk = mbar_test(sm.kvp(1), 0);
    pp = mbar_test(sm.p_full(0, 0), 0);
    mma_s(1, sK);
    tc_commit(sm.s_full(1));
    tc_commit(sm.kv_empty(sK));
  }
  for (int j = 1; ok && j < n_kv; ++j) {
    const uint32_t par = (j - 1) & 1;
    next_slot(sV);
    next_slot(sK);
    ok = settle(pk, sm.kvp(j), (j / C::kNumKvSteps) & 1);
    if (!ok) break;
    ok = mma_o(0, sV, j > 1, par, pp);
    if (!ok) break;
    pp = mbar_test(sm.p_full(1, 0), par);
    mma_s(0, sK);
    tc_commit(sm.s_full(0));
    ok = mma_o(1, sV, j > 1, par, pp);
    if (!ok) break;
    tc_commit(sm.kv_empty(sV));
    // the next step's K/V and chunk 0 of P0, looked at while S1 is issued
    pk = mbar_test(sm.kvp(j + 1), ((j + 1) / C::kNumKvSteps) & 1);
    pp = mbar_test(sm.p_full(0, 0), j & 1);
    mma_s(1, sK);
    tc_commit(sm.s_full(1));
    tc_commit(sm.kv_empty(sK));
  }
  if (ok) {
    const uint32_t par = (n_kv - 1) & 1;
    next_slot(sV);
    ok = settle(n_kv > 1 ? pk : false, sm.kvp(n_kv), (n_kv / C::kNumKvSteps) & 1) && mma_o(0, sV, n_kv > 1, par, pp);
    if (ok) {
      tc_commit(sm.o_full(0));
      ok = mma_o(1, sV, n_kv > 1, par, false);
    }
    if (ok) {
      tc_commit(sm.o_full(1));
      tc_commit(sm.kv_empty(sV));
    }
  }
  // Everything issued must be finished before TMEM is released.
  tc_commit(sm.mma_done());
  mbar_wait(sm.mma_done(), 0, timeout);
  if (!ok) atomicOr(&g_status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// Softmax + correction + epilogue, one thread per query row.  Tile t has the
// four warps of warpgroup t: warp (t, q) owns TMEM lanes 32q..32q+31 (its 32
// rows), all 128 key columns of every S tile and all d output columns.  A
// warp waits only on pipeline mbarriers (bounded), never on another warp, so a
// failed wait simply ends its loop; the MMA thread then gives up on the P
// barrier that warp no longer signals.
// ---------------------------------------------------------------------------
template <int D, int MASK, int POLY16, bool F8>
__device__ __forceinline__ void softmax_role(const Smem<D, F8>& sm, uint32_t tmem,
                                             const CUtensorMap* tm_o, const FwdParams& prm,
                                             const SeqView& sv, int qb) {
  using C = Cfg<D, F8>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = warp >> 2;        // query tile of this CTA
  const int q4 = warp & 3;        // TMEM lane quarter this warp may access
  const int r = q4 * 32 + lane;   // row within the tile (= TMEM lane)
  const int tile_row0 = qb * kRowsPerCta + t * kBlockM;
  const int row = tile_row0 + r;
  const int rw0 = tile_row0 + q4 * 32;  // first row of this warp
  const int Nk = sv.Nk;
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  const uint32_t tS = tmem + lane_off + t * kBlockM;
  const uint32_t tO = tmem + lane_off + C::kTmemO + t * D;
  const uint64_t timeout = prm.timeout_ns;

  // scale <= 0: apply it first, then run with an effective scale of 1 (the
  // fast path folds a positive scale into one FFMA per score).
  const bool prescale = !(prm.scale_log2 > 0.0f);
  const float sl = prescale ? 1.0f : prm.scale_log2;
  float m_run = -INFINITY;  // running reference max, log2 units of scaled scores
  float l_run = 0.0f;       // running sum of 2^(score - m_run)
  bool ok = true;

  int blk = sv.j_lo - 1;
  for (int j = 0; j < sv.n_kv; ++j) {
    blk = next_block<MASK>(sm.vis(), blk);
    const int kv0 = blk * kBlockN;
    // mask needed: key tail, a band edge crossing this warp's 32 x 128 block,
    // or a column interval meeting the warp's rows
    bool masked = kv0 + kBlockN > Nk ||
                  (MASK != kMaskNone && (kv0 + kBlockN - 1 - rw0 > prm.wr || rw0 + 31 - kv0 > prm.wl));
    // column-interval mask: bit c of hid[k] = key kv0 + 32k + c hidden from this row
    uint32_t hid[4] = {0u, 0u, 0u, 0u};
    if constexpr (MASK == kMaskCols) {
      if (cols_touch(prm, sv.mrow, blk, rw0, rw0 + 32)) {
        masked = true;
        // lane l reads keys kv0 + 32k + l (coalesced).  A 32-key chunk whose
        // keys all carry the same intervals (a chunk inside one document)
        // hides a row from all 32 keys or from none, so each lane tests its
        // own row.  Otherwise each key becomes the set of the warp's 32 rows
        // it is hidden from, and ballots transpose those into per-row words
        // (bit c of row r's word k: key 32k + c).
        const int4* cm = prm.colmask + static_cast<size_t>(sv.mrow) * Nk + kv0;
        const int n_in = min(kBlockN, Nk - kv0);
        const int4 none = make_int4(0, 0, 0, 0);
        int4 iv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) iv[k] = 32 * k + lane < n_in ? __ldg(cm + 32 * k + lane) : none;
        const int row_l = rw0 + lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int4 i0 = make_int4(__shfl_sync(0xffffffffu, iv[k].x, 0), __shfl_sync(0xffffffffu, iv[k].y, 0),
                                    __shfl_sync(0xffffffffu, iv[k].z, 0), __shfl_sync(0xffffffffu, iv[k].w, 0));
          const bool same = iv[k].x == i0.x && iv[k].y == i0.y && iv[k].z == i0.z && iv[k].w == i0.w;
          if (__all_sync(0xffffffffu, same)) {
            const bool h = (row_l >= i0.x && row_l < i0.y) || (row_l >= i0.z && row_l < i0.w);
            hid[k] = h ? 0xffffffffu : 0u;
          } else {
            const uint32_t cb = span_bits(iv[k].x, iv[k].y, rw0) | span_bits(iv[k].z, iv[k].w, rw0);
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) {
              const uint32_t w = __ballot_sync(0xffffffffu, (cb >> rr) & 1u);
              if (lane == rr) hid[k] = w;
            }
          }
        }
      }
    }
    // the keys this row sees among the tile's 128, as four 32-bit words: below
    // Nk, inside the band, and not hidden by a column interval (one bit test
    // per score below instead of the comparisons themselves)
    uint32_t keep[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
    if (masked) {
      const long long klo = MASK != kMaskNone ? static_cast<long long>(row) - prm.wl : 0;
      const long long khi = MASK != kMaskNone ? min(static_cast<long long>(row) + prm.wr + 1, static_cast<long long>(Nk))
                                              : static_cast<long long>(Nk);
#pragma unroll
      for (int k = 0; k < 4; ++k) keep[k] = span_bits(klo, khi, kv0 + 32 * k) & ~hid[k];
    }
    ok = warp_wait(sm.s_full(t), j & 1, timeout);
    if (!ok) break;
    tc_fence_after();

    // the row's 128 scores: two loads, one wait
    float x[128];
    {
      uint32_t s[128];
      tmem_ld64(tS, s);
      tmem_ld64(tS + 64, s + 64);
      tmem_ld_wait();
      reg_fence64(s);
      reg_fence64(s + 64);
#pragma unroll
      for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(s[c]);
    }
    if (prescale) {
#pragma unroll
      for (int c = 0; c < 128; ++c) x[c] *= prm.scale_log2;
    }
    if (masked) {
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (!((keep[c >> 5] >> (c & 31)) & 1u)) x[c] = -INFINITY;
    }

    // the tile's row max: eight independent chains of three-input maxima
    float mx[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) mx[a] = fmaxf(x[2 * a], x[2 * a + 1]);
#pragma unroll
    for (int c = 16; c < 128; c += 16) {
#pragma unroll
      for (int a = 0; a < 8; ++a) mx[a] = fmax3(mx[a], x[c + 2 * a], x[c + 2 * a + 1]);
    }
    const float m_tile =
        fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sl;

    // adaptive rescaling: move the reference only on a jump beyond tau
    const bool resc = m_tile > m_run + prm.tau;
    float alpha = 1.0f;
    if (resc) {
      alpha = ex2_mufu(m_run - m_tile);  // 0 on the first tile
      m_run = m_tile;
    }
    l_run *= alpha;

    // Correction: rescale the row's O accumulator (final up to tile j-1, see
    // the MMA order) by alpha before O += P V_j is issued.
    if (j > 0 && __any_sync(0xffffffffu, resc)) {
      if (prm.rescale_count) {
        const unsigned n = __popc(__ballot_sync(0xffffffffu, resc));
        if (lane == 0) atomicAdd(prm.rescale_count, static_cast<unsigned long long>(n));
      }
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_ld_wait();
        reg_fence32(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
        tmem_st32(tO + cc * 32, o);
      }
    }

    // P = 2^(x*sl - m), 32 keys at a time -> BF16 pairs (E4M3 quadruples) in
    // the tile's first TMEM columns, whose scores are already in registers.
    // Chunk k is announced on its own barrier so its O += P V can start while
    // the next chunk is being exponentiated.
    constexpr float kOff = F8 ? kP8Offset : 0.0f;
    const float neg_m = (m_run == -INFINITY) ? 0.0f : kOff - m_run;
    const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(neg_m, neg_m);
    float2 sum2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
#pragma unroll
    for (int k = 0; k < kPChunks; ++k) {
      uint32_t p[16];
      float2 prev = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int c = 32 * k + 2 * i;
        const float2 u = ffma2(make_float2(x[c], x[c + 1]), sl2, nm2);
        float2 e;
        if ((c & 15) < POLY16) {
          e = ex2_poly2(u);
        } else {
          e.x = ex2_mufu(u.x);
          e.y = ex2_mufu(u.y);
        }
        sum2[i & 3] = fadd2(sum2[i & 3], e);
        if constexpr (F8) {
          // four E4M3 per TMEM column, key 4w in the low byte of word w
          if (i & 1) p[i >> 1] = pack_e4m3x4(prev.x, prev.y, e.x, e.y);
          prev = e;
        } else {
          p[i] = pack_bf16x2(e.x, e.y);
        }
      }
      if constexpr (F8)
        tmem_st8(tS + 8 * k, p);
      else
        tmem_st16(tS + 16 * k, p);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.p_full(t, k));
    }
    const float2 s01 = fadd2(sum2[0], sum2[1]), s23 = fadd2(sum2[2], sum2[3]);
    const float2 s03 = fadd2(s01, s23);
    l_run += s03.x + s03.y;
  }

  // Epilogue.
  const bool ok2 = ok && warp_wait(sm.o_full(t), 0, timeout);
  uint8_t* sOt = sm.base + C::kOffO + t * C::kOTileBytes;
  const bool ragged = sv.packed && rw0 + 32 > sv.Nq;
  if (ok2) {
    tc_fence_after();
    // O / l -> BF16 -> the tile's O staging (BF16 inputs: the tile's Q buffer,
    // whose last reader, the final S MMA, finished before the last O MMA) in
    // the 128-byte swizzled layout the O tensor map expects.
    const float inv_l = l_run > 0.0f ? prm.o_scale / l_run : 0.0f;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      tmem_ld32(tO + cc * 32, o);
      tmem_ld_wait();
      reg_fence32(o);
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
      const int col0 = cc * 32;  // first output column of this chunk
      if (ragged) {
        // the warp's 32 rows cross the end of a packed sequence: a TMA store
        // would write into the next sequence, so each row stores itself
        if (row < sv.Nq) {
          uint4* dst = reinterpret_cast<uint4*>(
              prm.o + (static_cast<size_t>(sv.q0 + row) * prm.H + sv.head_q) * D + col0);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      } else {
        uint8_t* rowp = sOt + (col0 >> 6) * C::kBoxBytes + r * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int chunk = (((col0 & 63) >> 3) + i) ^ (r & 7);
          *reinterpret_cast<uint4*>(rowp + chunk * 16) =
              make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
    }
    fence_proxy_async_smem();
  }
  __syncwarp();
  // each warp stores its 32 rows, one 64-column box at a time
  if (ok2 && !ragged && lane == 0 && rw0 < sv.Nq) {
#pragma unroll
    for (int box = 0; box < D / 64; ++box) {
      const uint32_t src = smem_u32(sOt + box * C::kBoxBytes + q4 * 32 * 128);
      if (sv.packed) tma_store_3d(tm_o, src, box * 64, sv.head_q, sv.q0 + rw0);
      else tma_store_3d(tm_o, src, box * 64, rw0, sv.head_q);
    }
    bulk_commit_group();
    bulk_wait_group_read0();
  }
  if (ok2 && sv.lse_row0 != nullptr && row < sv.Nq) {
    // P carried 2^kOff: LSE = ln 2 * (m - kOff + log2 l)
    const float m_use = (m_run == -INFINITY) ? 0.0f : m_run - (F8 ? kP8Offset : 0.0f);
    sv.lse_row0[row] = (m_use + log2f(l_run)) * kLn2;
  }
  if (!ok2 && lane == 0) atomicOr(&g_status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// The kernel.  Grid: one CTA per (b*h, 256-row query block).
// ---------------------------------------------------------------------------
template <int D, int MASK, int POLY16, bool F8>
__global__ void __launch_bounds__(kNumThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const __grid_constant__ FwdParams prm) {
  using C = Cfg<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  Smem<D, F8> sm;
  {
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    sm.base = smem_raw + pad;
    sm.sbase = raw + pad;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Tile order.  Default: head-major, so the CTAs resident at one time share a
  // few heads' K/V in L2.  Causal band: heads in groups of hgroup (sized on the
  // host so a group's K/V fits in L2), and within a group the heaviest query
  // blocks first, so short blocks fill the tail of each group while the next
  // group starts.
  const int tile = blockIdx.x;
  int bh, qb;
  if (MASK == kMaskCols && prm.uperm != nullptr) {
    // the planned order: CTA i takes unit uperm[i / hper] (a mask row and a
    // query block) for the i % hper-th query head reading that mask row
    const int hper = prm.mask_heads == 1 ? prm.H : 1;
    const int u = __ldg(prm.uperm + blockIdx.x / hper);
    const int mrow = u / prm.n_qblocks;
    qb = u % prm.n_qblocks;
    bh = prm.mask_heads == 1 ? mrow * prm.H + static_cast<int>(blockIdx.x % hper) : mrow;
  } else if (prm.grouped) {
    const int per_group = prm.hgroup * prm.n_qblocks;
    const int g = tile / per_group, w = tile % per_group;
    const int gsize = min(prm.hgroup, prm.BH - g * prm.hgroup);
    qb = prm.n_qblocks - 1 - w / gsize;
    bh = g * prm.hgroup + w % gsize;
  } else {
    bh = tile / prm.n_qblocks;
    qb = tile % prm.n_qblocks;
  }
  // grouped-query attention: query head h reads key/value head h / group of the
  // same batch entry (group = 1: one key/value head per query head)
  const int hq = bh % prm.H, seq = bh / prm.H;
  SeqView sv;
  static_assert(sizeof(SeqView) <= Cfg<D, F8>::kSeqBytes, "SeqView slot");
  sv.packed = prm.cu_q != nullptr;
  if (sv.packed) {
    // packed variable-length batch: sequence `seq` owns rows cu_q[seq] ..
    // cu_q[seq+1]-1 of the [total, H, d] tensors.  Offsets that do not describe
    // sequences inside the tensors, or a sequence longer than the grid covers,
    // are reported and the CTA does nothing (every access stays in bounds).
    const int a = __ldg(prm.cu_q + seq), b = __ldg(prm.cu_q + seq + 1);
    const int c = __ldg(prm.cu_k + seq), e = __ldg(prm.cu_k + seq + 1);
    if (a < 0 || b < a || b > prm.Nq || c < 0 || e < c || e > prm.Nk ||
        b - a > prm.n_qblocks * kRowsPerCta) {
      if (threadIdx.x == 0 && qb == 0) atomicOr(&g_status, kStatusBadSeqlens);
      return;
    }
    sv.Nq = b - a;
    sv.Nk = e - c;
    sv.q0 = a;
    sv.k0 = c;
    sv.head_q = hq;
    sv.head_kv = hq / prm.group;
    sv.lse_row0 = prm.lse ? prm.lse + static_cast<size_t>(hq) * prm.Nq + a : nullptr;
    if (qb * kRowsPerCta >= sv.Nq) return;  // this sequence is shorter than the grid
  } else {
    sv.Nq = prm.Nq;
    sv.Nk = prm.Nk;
    sv.q0 = 0;
    sv.k0 = 0;
    sv.head_q = bh;
    sv.head_kv = seq * (prm.H / prm.group) + hq / prm.group;
    sv.lse_row0 = prm.lse ? prm.lse + static_cast<size_t>(bh) * prm.Nq : nullptr;
  }
  {
    // KV tiles that hold a visible key for some row of this block; a block with
    // none (an empty band, an empty key set) still runs one fully masked tile,
    // which yields O = 0 and LSE = -inf.
    int j_lo, j_hi;
    kv_band_range<MASK>(prm, sv.Nq, sv.Nk, qb, &j_lo, &j_hi);
    sv.j_lo = j_lo;
    sv.n_kv = j_hi - j_lo;
    sv.mrow = 0;
    if constexpr (MASK == kMaskCols) {
      // the bitmap of tiles that some row of this block sees (warp 0, 32 tiles
      // a step, bit b of word w = tile 32w + b); none: visit tile j_lo fully
      // masked, as for an empty band
      sv.mrow = seq * prm.mask_heads + (prm.mask_heads == 1 ? 0 : hq);
      if (warp == 0) {
        const int r0 = qb * kRowsPerCta, r1 = cta_row_end(qb, sv.Nq);
        uint32_t* vis = sm.vis();
        int cnt = 0;
#pragma unroll 4
        for (int w = j_lo >> 5; w <= (j_hi - 1) >> 5; ++w) {
          const int blk = w * 32 + lane;
          const bool v = blk >= j_lo && blk < j_hi && !cols_hide_all(prm, sv.mrow, blk, r0, r1);
          const uint32_t word = __ballot_sync(0xffffffffu, v);
          if (lane == 0) vis[w] = word;
          cnt += __popc(word);
        }
        if (cnt == 0 && lane == 0) vis[j_lo >> 5] = 1u << (j_lo & 31);
        sv.n_kv = cnt > 0 ? cnt : 1;
      }
    }
  }
  if (threadIdx.x == 0) *sm.seq() = sv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) {
      const uint32_t b = sm.bar(i);
      // p_full: one arrival per softmax warp of the tile (4); everything else: one.
      const bool pf = b >= sm.p_full(0, 0) && b <= sm.p_full(1, kPChunks - 1);
      mbar_init(b, pf ? 4u : 1u);
    }
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(sm.tmem_slot()), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();
  const SeqView& seqv = *sm.seq();

  if (warp >= kWarpLoad) {
    // warpgroup 2: TMA producer (warp 8), MMA issuer (warp 9), two idle warps
    setmaxnreg_dec<kProducerRegs>();
    if (warp == kWarpLoad) {
      if (lane == 0) producer_role<D, MASK, F8>(sm, &tm_q, &tm_k, &tm_v, seqv, prm, qb, prm.timeout_ns);
      __syncwarp();
    } else if (warp == kWarpMma) {
      if (lane == 0) mma_role<D, F8>(sm, tmem, seqv.n_kv, prm.timeout_ns);
      __syncwarp();
    }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    softmax_role<D, MASK, POLY16, F8>(sm, tmem, &tm_o, prm, seqv, qb);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Nk == 0: no visible key -> O = 0 (memset by the host), LSE = -inf.
__global__ void fill_neg_inf_kernel(float* p, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = -INFINITY;
}

// Column-interval mask summaries: one 128-thread CTA per (mask row, key block)
// reduces the block's intervals to the two int4 that cols_hide_all and
// cols_touch read.  Keys past Nk take no part; an empty interval (lo >= hi)
// counts as (INT_MAX, INT_MIN), so it neither hides a row nor meets one.
__global__ void __launch_bounds__(128) colmask_summary_kernel(const int4* __restrict__ mask,
                                                              int4* __restrict__ sum, int Nk,
                                                              int n_kblocks) {
  const int blk = static_cast<int>(blockIdx.x % static_cast<unsigned>(n_kblocks));
  const size_t mrow = blockIdx.x / static_cast<unsigned>(n_kblocks);
  const int key = blk * kBlockN + static_cast<int>(threadIdx.x);
  // a: max lo1, min hi1, max lo2, min hi2;  b: min lo1, max hi1, min lo2, max hi2
  int a[4] = {INT_MIN, INT_MAX, INT_MIN, INT_MAX};
  int b[4] = {INT_MAX, INT_MIN, INT_MAX, INT_MIN};
  if (key < Nk) {
    const int4 iv = mask[mrow * Nk + key];
    const bool e1 = iv.x >= iv.y, e2 = iv.z >= iv.w;
    a[0] = b[0] = e1 ? INT_MAX : iv.x;
    a[1] = b[1] = e1 ? INT_MIN : iv.y;
    a[2] = b[2] = e2 ? INT_MAX : iv.z;
    a[3] = b[3] = e2 ? INT_MIN : iv.w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int oa = __shfl_xor_sync(0xffffffffu, a[i], off);
      const int ob = __shfl_xor_sync(0xffffffffu, b[i], off);
      a[i] = (i & 1) ? min(a[i], oa) : max(a[i], oa);
      b[i] = (i & 1) ? max(b[i], ob) : min(b[i], ob);
    }
  }
  __shared__ int red[4][8];
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      red[warp][i] = a[i];
      red[warp][4 + i] = b[i];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 1; w < 4; ++w) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = (i & 1) ? min(a[i], red[w][i]) : max(a[i], red[w][i]);
        b[i] = (i & 1) ? max(b[i], red[w][4 + i]) : min(b[i], red[w][4 + i]);
      }
    }
    int4* dst = sum + (mrow * n_kblocks + blk) * 2;
    dst[0] = make_int4(a[0], a[1], a[2], a[3]);
    dst[1] = make_int4(b[0], b[1], b[2], b[3]);
  }
}

// CTA order for column-interval masks, longest first within each mask row.
// For every (mask row, query block) unit the number of key blocks the
// attention kernel will visit (the band range and block-summary test of its
// prologue: one warp per unit, lanes over the blocks), then a counting sort of
// the units by (mask row, that number, most first): uperm[i] is the unit of
// the i-th group of CTAs.  Keeping the mask rows apart keeps the K/V of one
// batch entry's heads (mask row shared by all heads) or of one head (a mask
// per head) in flight together, so L2 holds them.  Units of equal key keep
// no particular order; the results do not depend on it.
constexpr int kPlanThreads = 1024;
constexpr int kPlanMaxUnits = 8192;   // per-unit bins in shared memory
constexpr int kPlanMaxBins = 4096;    // mask rows x (counts 0 .. n_kblocks)

__global__ void __launch_bounds__(kPlanThreads) colmask_plan_kernel(const FwdParams prm, int* __restrict__ uperm,
                                                                    int n_units) {
  __shared__ uint16_t ubin[kPlanMaxUnits];
  __shared__ int off[kPlanMaxBins];
  __shared__ int wsum[kPlanThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int n_bins = (n_units / prm.n_qblocks) * (prm.n_kblocks + 1);
  for (int i = t; i < n_bins; i += kPlanThreads) off[i] = 0;
  __syncthreads();
  for (int u = warp; u < n_units; u += kPlanThreads / 32) {
    const int mrow = u / prm.n_qblocks, qb = u % prm.n_qblocks;
    int j_lo, j_hi;
    kv_band_range<kMaskCols>(prm, prm.Nq, prm.Nk, qb, &j_lo, &j_hi);
    const int r0 = qb * kRowsPerCta, r1 = cta_row_end(qb, prm.Nq);
    int cnt = 0;
    for (int b = j_lo + lane; b < j_hi; b += 32) cnt += cols_hide_all(prm, mrow, b, r0, r1) ? 0 : 1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) {
      // mask row first, then most visited first
      const int bin = mrow * (prm.n_kblocks + 1) + prm.n_kblocks - min(cnt, prm.n_kblocks);
      ubin[u] = static_cast<uint16_t>(bin);
      atomicAdd(&off[bin], 1);
    }
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

int launch_colmask_summary(const int* mask, void* sum, long long BHm, int Nk, cudaStream_t stream) {
  const int n_kblocks = (Nk + kBlockN - 1) / kBlockN;
  const unsigned grid = static_cast<unsigned>(BHm * n_kblocks);
  if (grid == 0) return ATTN_OK;
  colmask_summary_kernel<<<grid, 128, 0, stream>>>(reinterpret_cast<const int4*>(mask),
                                                   static_cast<int4*>(sum), Nk, n_kblocks);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "colmask_summary_kernel launch");
  return ATTN_OK;
}

// One thread waits on a barrier that nothing signals; the bounded wait gives
// up and records a timeout.  Exercises the failure path without any fault.
__global__ void selftest_timeout_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    if (!mbar_wait(smem_u32(&bar), 0, timeout_ns)) atomicOr(&g_status, kStatusTimeout);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = kMaxDeviceCount;

template <int D, int MASK, int POLY16, bool F8 = false>
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const CUtensorMap& to, const FwdParams& prm, cudaStream_t stream) {
  auto kern = attn_fwd_kernel<D, MASK, POLY16, F8>;
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static int launch_regs[kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg<D, F8>::kSmemBytes);
    cudaFuncAttributes fa;
    if (attr_err[dev] == cudaSuccess) attr_err[dev] = cudaFuncGetAttributes(&fa, kern);
    if (attr_err[dev] == cudaSuccess) launch_regs[dev] = fa.numRegs;
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "cudaFuncSetAttribute");
  // the warpgroups' setmaxnreg shares must fit in the registers the block is
  // launched with, or setmaxnreg.inc would never be granted
  if (launch_regs[dev] * kNumThreads < 2 * 128 * kSoftmaxRegs + 128 * kProducerRegs) {
    t_last_error = "attn_fwd_kernel: built with " + std::to_string(launch_regs[dev]) +
                   " registers per thread, below the setmaxnreg split";
    return ATTN_ERR_CUDA;
  }
  const unsigned grid = static_cast<unsigned>(prm.BH) * static_cast<unsigned>(prm.n_qblocks);
  kern<<<grid, kNumThreads, Cfg<D, F8>::kSmemBytes, stream>>>(tq, tk, tv, to, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_kernel launch");
  return ATTN_OK;
}

template <int D, int MASK>
int dispatch_exp(int exp_mode, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const CUtensorMap& to, const FwdParams& prm, cudaStream_t stream) {
  switch (exp_mode) {
    case 0: return launch_fwd<D, MASK, 0>(tq, tk, tv, to, prm, stream);
    case 1: return launch_fwd<D, MASK, kDefaultPoly16>(tq, tk, tv, to, prm, stream);
    default: return launch_fwd<D, MASK, 16>(tq, tk, tv, to, prm, stream);
  }
}



// Key band from the C-ABI's (window_left, window_right), -1 = no bound.
bool band_from_window(int window_left, int window_right, int* wl, int* wr) {
  if (window_left < -1 || window_right < -1) return false;
  *wl = window_left < 0 ? kUnbounded : std::min(window_left, kUnbounded);
  *wr = window_right < 0 ? kUnbounded : std::min(window_right, kUnbounded);
  return true;
}

// Heads scheduled together under the causal order: as many as keep their K/V
// within ~48 MB of the 126 MB L2 (several query heads of a GQA group share one
// K/V head).
int heads_per_l2_group(double keys_per_head, int d, int group, long long BH) {
  const double kv_head_bytes = 2.0 * keys_per_head * d * 2.0 / group;
  const double budget = 48.0 * 1024 * 1024;
  const long long g = static_cast<long long>(budget / std::max(kv_head_bytes, 1.0));
  return static_cast<int>(std::max(1LL, std::min(g, BH)));
}

int launch_any(int d, int exp_mode, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const CUtensorMap& to, const FwdParams& prm,
               cudaStream_t stream) {
  if (prm.colmask != nullptr) {  // default exp2 split only
    return d == 128 ? launch_fwd<128, kMaskCols, kDefaultPoly16>(tq, tk, tv, to, prm, stream)
                    : launch_fwd<64, kMaskCols, kDefaultPoly16>(tq, tk, tv, to, prm, stream);
  }
  const bool mask = prm.wl < kUnbounded || prm.wr < kUnbounded;
  if (d == 128) {
    return mask ? dispatch_exp<128, kMaskBand>(exp_mode, tq, tk, tv, to, prm, stream)
                : dispatch_exp<128, kMaskNone>(exp_mode, tq, tk, tv, to, prm, stream);
  }
  return mask ? dispatch_exp<64, kMaskBand>(exp_mode, tq, tk, tv, to, prm, stream)
              : dispatch_exp<64, kMaskNone>(exp_mode, tq, tk, tv, to, prm, stream);
}

// No key at all: O = 0, LSE = -inf.
int fill_empty(void* o, size_t o_bytes, float* lse, size_t n_lse, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(o, 0, o_bytes, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if (lse && n_lse) {
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n_lse + 255) / 256, 4096));
    fill_neg_inf_kernel<<<blocks, 256, 0, stream>>>(lse, n_lse);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "fill_neg_inf_kernel launch");
  }
  return ATTN_OK;
}


// Outputs may not overlap any input or each other.
bool outputs_overlap(const void* q, size_t q_bytes, const void* k, const void* v, size_t kv_bytes,
                     const void* o, size_t o_bytes, const void* lse, size_t lse_bytes) {
  return ranges_overlap(o, o_bytes, q, q_bytes) || ranges_overlap(o, o_bytes, k, kv_bytes) ||
         ranges_overlap(o, o_bytes, v, kv_bytes) || ranges_overlap(lse, lse_bytes, q, q_bytes) ||
         ranges_overlap(lse, lse_bytes, k, kv_bytes) || ranges_overlap(lse, lse_bytes, v, kv_bytes) ||
         ranges_overlap(lse, lse_bytes, o, o_bytes);
}

// Column-interval mask of attn_fwd_colmask: int32 [B, Hm, Nk, 4] and the
// caller's workspace for the per-block summaries.
struct ColMaskArgs {
  const int* mask;
  int Hm;
  void* workspace;
  size_t workspace_bytes;
};

// Column-interval workspace: the block summaries (required), then room for the
// CTA plan of colmask_plan_kernel, one int per (mask row, 256-row query block)
// for up to 4 Nk query rows (a call whose plan does not fit keeps the fixed
// CTA order).
size_t colmask_summary_bytes(long long BHm, int Nk) {
  const long long n_kblocks = (static_cast<long long>(Nk) + kBlockN - 1) / kBlockN;
  return static_cast<size_t>(BHm * n_kblocks) * 2 * sizeof(int4);
}
size_t colmask_workspace_bytes(long long BHm, int Nk) {
  const long long plan_units = BHm * ((4LL * Nk + kRowsPerCta - 1) / kRowsPerCta);
  return colmask_summary_bytes(BHm, Nk) + ((static_cast<size_t>(plan_units) * 4 + 15) & ~static_cast<size_t>(15));
}

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int Hkv, int Nq, int Nk, int d, float scale, int window_left, int window_right,
             float tau, int exp_mode, unsigned long long* rescale_count, cudaStream_t stream,
             const ColMaskArgs* cm = nullptr) {
  int wl = 0, wr = 0;
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (H > 0 && (Hkv == 0 || H % Hkv != 0)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (!band_from_window(window_left, window_right, &wl, &wr)) return ATTN_ERR_INVALID_ARG;
  if (!(tau >= 0.0f && tau <= 64.0f)) return ATTN_ERR_UNSUPPORTED;
  if (exp_mode < 0 || exp_mode > 2) return ATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0 || Nq == 0) return ATTN_OK;  // nothing to compute
  if (BH > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (!o || (Nk > 0 && (!q || !k || !v))) return ATTN_ERR_INVALID_ARG;
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16) ||
      misaligned(lse, 4) || misaligned(rescale_count, 8))
    return ATTN_ERR_INVALID_ARG;
  const size_t o_bytes = static_cast<size_t>(BH) * Nq * d * 2;
  const long long BHkv = static_cast<long long>(B) * Hkv;
  const size_t kv_bytes = static_cast<size_t>(BHkv) * Nk * d * 2;
  const size_t lse_bytes = lse ? static_cast<size_t>(BH) * Nq * 4 : 0;
  if (outputs_overlap(q, o_bytes, k, v, kv_bytes, o, o_bytes, lse, lse_bytes))
    return ATTN_ERR_INVALID_ARG;
  const long long n_qblocks = (Nq + kRowsPerCta - 1) / kRowsPerCta;
  if (n_qblocks * BH > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  long long BHm = 0;
  size_t mask_bytes = 0, ws_need = 0;
  bool plan = false;  // longest-first CTA order (colmask_plan_kernel)
  if (cm) {
    if (cm->Hm != 1 && cm->Hm != H) return ATTN_ERR_INVALID_ARG;
    BHm = static_cast<long long>(B) * cm->Hm;
    mask_bytes = static_cast<size_t>(BHm) * Nk * sizeof(int4);
    ws_need = colmask_summary_bytes(BHm, Nk);
    const long long units = BHm * n_qblocks;
    const long long n_kb = (static_cast<long long>(Nk) + kBlockN - 1) / kBlockN;
    plan = units > 0 && units <= kPlanMaxUnits && BHm * (n_kb + 1) <= kPlanMaxBins &&
           cm->workspace_bytes >= ws_need + static_cast<size_t>(units) * 4;
    if (plan) ws_need += static_cast<size_t>(units) * 4;  // the region written
    if (Nk > 0 && (!cm->mask || !cm->workspace)) return ATTN_ERR_INVALID_ARG;
    if (misaligned(cm->mask, 16) || misaligned(cm->workspace, 16)) return ATTN_ERR_INVALID_ARG;
    if (cm->workspace_bytes < ws_need) return ATTN_ERR_INVALID_ARG;
    if (BHm * ((Nk + kBlockN - 1) / kBlockN) > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    if ((static_cast<long long>(Nk) + kBlockN - 1) / kBlockN > kMaxMaskBlocks) return ATTN_ERR_UNSUPPORTED;
    // the workspace is written: it may overlap no input or output
    const void* ws = cm->workspace;
    if (ranges_overlap(ws, ws_need, q, o_bytes) || ranges_overlap(ws, ws_need, k, kv_bytes) ||
        ranges_overlap(ws, ws_need, v, kv_bytes) || ranges_overlap(ws, ws_need, o, o_bytes) ||
        ranges_overlap(ws, ws_need, lse, lse_bytes) ||
        ranges_overlap(ws, ws_need, cm->mask, mask_bytes) ||
        ranges_overlap(o, o_bytes, cm->mask, mask_bytes) ||
        ranges_overlap(lse, lse_bytes, cm->mask, mask_bytes))
      return ATTN_ERR_INVALID_ARG;
  }
  int rc = check_device();
  if (rc != ATTN_OK) return rc;

  if (Nk == 0) return fill_empty(o, o_bytes, lse, static_cast<size_t>(BH) * Nq, stream);

  CUtensorMap tq, tk, tv, to;
  const int bh = static_cast<int>(BH);
  if (!make_tmap_bf16_3d(&tq, q, bh, Nq, d, kBlockM, &t_last_error) ||
      !make_tmap_bf16_3d(&tk, k, static_cast<int>(BHkv), Nk, d, kBlockN, &t_last_error) ||
      !make_tmap_bf16_3d(&tv, v, static_cast<int>(BHkv), Nk, d, kBlockN, &t_last_error) ||
      !make_tmap_bf16_3d(&to, o, bh, Nq, d, 32, &t_last_error))
    return ATTN_ERR_CUDA;

  FwdParams prm = {};
  prm.lse = lse;
  prm.rescale_count = rescale_count;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.timeout_ns = kWaitTimeoutNs;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.BH = bh;
  prm.H = H;
  prm.group = H / Hkv;
  prm.wl = wl;
  prm.wr = wr;
  prm.grouped = (wl == kUnbounded && wr == 0) ? 1 : 0;
  prm.hgroup = heads_per_l2_group(Nk, d, prm.group, BH);
  prm.n_qblocks = static_cast<int>(n_qblocks);
  prm.scale_log2 = scale * kLog2e;
  prm.tau = tau;
  prm.o_scale = 1.0f;
  if (cm) {
    prm.colmask = reinterpret_cast<const int4*>(cm->mask);
    prm.colsum = static_cast<const int4*>(cm->workspace);
    prm.mask_heads = cm->Hm;
    prm.n_kblocks = (Nk + kBlockN - 1) / kBlockN;
    const int rc2 = launch_colmask_summary(cm->mask, cm->workspace, BHm, Nk, stream);
    if (rc2 != ATTN_OK) return rc2;
    if (plan) {
      int* uperm = reinterpret_cast<int*>(static_cast<uint8_t*>(cm->workspace) + colmask_summary_bytes(BHm, Nk));
      colmask_plan_kernel<<<1, kPlanThreads, 0, stream>>>(prm, uperm, static_cast<int>(BHm * n_qblocks));
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail(e, "colmask_plan_kernel launch");
      prm.uperm = uperm;
    }
  }
  return launch_any(d, exp_mode, tq, tk, tv, to, prm, stream);
}

int varlen_impl(const void* q, const void* k, const void* v, void* o, float* lse,
                const int* cu_q, const int* cu_k, int num_seqs, int max_seqlen_q, int total_q,
                int total_k, int H, int Hkv, int d, float scale, int window_left,
                int window_right, cudaStream_t stream) {
  int wl = 0, wr = 0;
  if (num_seqs < 0 || max_seqlen_q < 0 || total_q < 0 || total_k < 0 || H < 0 || Hkv < 0)
    return ATTN_ERR_INVALID_ARG;
  if (H > 0 && (Hkv == 0 || H % Hkv != 0)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (!band_from_window(window_left, window_right, &wl, &wr)) return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q > total_q) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (num_seqs == 0 || H == 0 || total_q == 0) return ATTN_OK;  // nothing to compute
  if (max_seqlen_q == 0) return ATTN_ERR_INVALID_ARG;  // rows exist but no sequence may hold one
  if (!o || !q || !cu_q || !cu_k || (total_k > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16) ||
      misaligned(lse, 4) || misaligned(cu_q, 4) || misaligned(cu_k, 4))
    return ATTN_ERR_INVALID_ARG;
  const size_t q_bytes = static_cast<size_t>(total_q) * H * d * 2;
  const size_t kv_bytes = static_cast<size_t>(total_k) * Hkv * d * 2;
  const size_t lse_bytes = lse ? static_cast<size_t>(total_q) * H * 4 : 0;
  if (outputs_overlap(q, q_bytes, k, v, kv_bytes, o, q_bytes, lse, lse_bytes) ||
      ranges_overlap(o, q_bytes, cu_q, (num_seqs + 1) * 4ull) ||
      ranges_overlap(o, q_bytes, cu_k, (num_seqs + 1) * 4ull) ||
      ranges_overlap(lse, lse_bytes, cu_q, (num_seqs + 1) * 4ull) ||
      ranges_overlap(lse, lse_bytes, cu_k, (num_seqs + 1) * 4ull))
    return ATTN_ERR_INVALID_ARG;
  const long long BH = static_cast<long long>(num_seqs) * H;
  const long long n_qblocks = (max_seqlen_q + kRowsPerCta - 1) / kRowsPerCta;
  if (BH > 0x7fffffffLL || n_qblocks * BH > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != ATTN_OK) return rc;

  if (total_k == 0) return fill_empty(o, q_bytes, lse, static_cast<size_t>(total_q) * H, stream);

  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16_packed(&tq, q, total_q, H, d, kBlockM, &t_last_error) ||
      !make_tmap_bf16_packed(&tk, k, total_k, Hkv, d, kBlockN, &t_last_error) ||
      !make_tmap_bf16_packed(&tv, v, total_k, Hkv, d, kBlockN, &t_last_error) ||
      !make_tmap_bf16_packed(&to, o, total_q, H, d, 32, &t_last_error))
    return ATTN_ERR_CUDA;

  FwdParams prm = {};
  prm.lse = lse;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.cu_q = cu_q;
  prm.cu_k = cu_k;
  prm.timeout_ns = kWaitTimeoutNs;
  prm.Nq = total_q;
  prm.Nk = total_k;
  prm.BH = static_cast<int>(BH);
  prm.H = H;
  prm.group = H / Hkv;
  prm.wl = wl;
  prm.wr = wr;
  prm.grouped = (wl == kUnbounded && wr == 0) ? 1 : 0;
  // L2 grouping sized by the longest sequence (max_seqlen_q bounds the causal
  // key count; the average would let groups of long sequences overflow L2)
  prm.hgroup = heads_per_l2_group(static_cast<double>(std::min(max_seqlen_q, total_k)), d, prm.group, BH);
  prm.n_qblocks = static_cast<int>(n_qblocks);
  prm.scale_log2 = scale * kLog2e;
  prm.tau = kDefaultThreshold;
  prm.o_scale = 1.0f;
  return launch_any(d, 1, tq, tk, tv, to, prm, stream);
}

int fp8_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
             int Nq, int Nk, int d, float scale, float q_descale, float k_descale, float v_descale,
             int causal, cudaStream_t stream) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (H > 0 && (Hkv == 0 || H % Hkv != 0)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !std::isfinite(q_descale) || !std::isfinite(k_descale) ||
      !std::isfinite(v_descale))
    return ATTN_ERR_INVALID_ARG;
  const float s_eff = scale * q_descale * k_descale;
  if (!std::isfinite(s_eff)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (causal && Nq != Nk) return ATTN_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0 || Nq == 0) return ATTN_OK;
  if (BH > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (!o || (Nk > 0 && (!q || !k || !v))) return ATTN_ERR_INVALID_ARG;
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16) ||
      misaligned(lse, 4))
    return ATTN_ERR_INVALID_ARG;
  const long long BHkv = static_cast<long long>(B) * Hkv;
  const size_t q_bytes = static_cast<size_t>(BH) * Nq * d;
  const size_t kv_bytes = static_cast<size_t>(BHkv) * Nk * d;
  const size_t o_bytes = static_cast<size_t>(BH) * Nq * d * 2;
  const size_t lse_bytes = lse ? static_cast<size_t>(BH) * Nq * 4 : 0;
  if (ranges_overlap(o, o_bytes, q, q_bytes) || ranges_overlap(o, o_bytes, k, kv_bytes) ||
      ranges_overlap(o, o_bytes, v, kv_bytes) || ranges_overlap(lse, lse_bytes, q, q_bytes) ||
      ranges_overlap(lse, lse_bytes, k, kv_bytes) || ranges_overlap(lse, lse_bytes, v, kv_bytes) ||
      ranges_overlap(lse, lse_bytes, o, o_bytes))
    return ATTN_ERR_INVALID_ARG;
  const long long n_qblocks = (Nq + kRowsPerCta - 1) / kRowsPerCta;
  if (n_qblocks * BH > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != ATTN_OK) return rc;
  if (Nk == 0) return fill_empty(o, o_bytes, lse, static_cast<size_t>(BH) * Nq, stream);

  CUtensorMap tq, tk, tv, to;
  const int bh = static_cast<int>(BH);
  if (!make_tmap_u8_3d(&tq, q, bh, Nq, d, kBlockM, &t_last_error) ||
      !make_tmap_u8_3d(&tk, k, static_cast<int>(BHkv), Nk, d, kBlockN, &t_last_error) ||
      !make_tmap_u8_3d(&tv, v, static_cast<int>(BHkv), Nk, d, kBlockN, &t_last_error) ||
      !make_tmap_bf16_3d(&to, o, bh, Nq, d, 32, &t_last_error))
    return ATTN_ERR_CUDA;

  FwdParams prm = {};
  prm.lse = lse;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.timeout_ns = kWaitTimeoutNs;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.BH = bh;
  prm.H = H;
  prm.group = H / Hkv;
  prm.wl = kUnbounded;
  prm.wr = causal ? 0 : kUnbounded;
  prm.grouped = causal;
  prm.hgroup = heads_per_l2_group(Nk / 2.0, d, prm.group, BH);  // one byte per element
  prm.n_qblocks = static_cast<int>(n_qblocks);
  prm.scale_log2 = s_eff * kLog2e;
  prm.tau = kP8Tau;
  prm.o_scale = v_descale;
  return causal ? launch_fwd<128, kMaskBand, kDefaultPoly16, true>(tq, tk, tv, to, prm, stream)
                : launch_fwd<128, kMaskNone, kDefaultPoly16, true>(tq, tk, tv, to, prm, stream);
}

}  // namespace eab

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int Nq, int Nk, int d, float scale, int causal, cudaStream_t stream) {
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (causal && Nq != Nk) return ATTN_ERR_UNSUPPORTED;
  return eab::fwd_impl(q, k, v, o, lse, B, H, H, Nq, Nk, d, scale, -1, causal ? 0 : -1,
                       eab::kDefaultThreshold, 1, nullptr, stream);
}

int attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int Hkv, int Nq, int Nk, int d, float scale, int causal, cudaStream_t stream) {
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (causal && Nq != Nk) return ATTN_ERR_UNSUPPORTED;
  return eab::fwd_impl(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, -1, causal ? 0 : -1,
                       eab::kDefaultThreshold, 1, nullptr, stream);
}

int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int Hkv, int Nq, int Nk, int d, float scale, int window_left,
                    int window_right, cudaStream_t stream) {
  return eab::fwd_impl(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, window_left, window_right,
                       eab::kDefaultThreshold, 1, nullptr, stream);
}

size_t attn_colmask_workspace_size(int B, int Hm, int Nk) {
  if (B < 0 || Hm < 0 || Nk < 0) return 0;
  return eab::colmask_workspace_bytes(static_cast<long long>(B) * Hm, Nk);
}

int attn_fwd_colmask(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     const int* mask, int Hm, void* workspace, size_t workspace_bytes,
                     cudaStream_t stream) {
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  const eab::ColMaskArgs cm = {mask, Hm, workspace, workspace_bytes};
  return eab::fwd_impl(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, -1, causal ? 0 : -1,
                       eab::kDefaultThreshold, 1, nullptr, stream, &cm);
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                    int max_seqlen_q, int total_q, int total_k, int H, int Hkv, int d,
                    float scale, int window_left, int window_right, cudaStream_t stream) {
  return eab::varlen_impl(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q,
                          total_q, total_k, H, Hkv, d, scale, window_left, window_right, stream);
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int Hkv, int Nq, int Nk, int d, float scale, float q_descale, float k_descale,
                 float v_descale, int causal, cudaStream_t stream) {
  return eab::fp8_impl(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, q_descale, k_descale,
                       v_descale, causal, stream);
}

int attn_fwd_config(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int Nq, int Nk, int d, float scale, int causal,
                    float rescale_threshold, int exp_mode, unsigned long long* rescale_count,
                    cudaStream_t stream) {
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (causal && Nq != Nk) return ATTN_ERR_UNSUPPORTED;
  return eab::fwd_impl(q, k, v, o, lse, B, H, H, Nq, Nk, d, scale, -1, causal ? 0 : -1,
                       rescale_threshold, exp_mode, rescale_count, stream);
}

int attn_status_sync(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return eab::cuda_fail(e, "cudaStreamSynchronize");
  unsigned int st = 0;
  e = cudaMemcpyFromSymbolAsync(&st, eab::g_status, sizeof(st), 0, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return eab::cuda_fail(e, "read status word");
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbolAsync(eab::g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return eab::cuda_fail(e, "clear status word");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return eab::cuda_fail(e, "cudaStreamSynchronize");
  unsigned int st_bwd = 0;
  const int rc = eab::bwd_status_take(stream, &st_bwd);
  if (rc != ATTN_OK) return rc;
  st |= st_bwd;
  if (st & eab::kStatusWordTimeout) return ATTN_ERR_TIMEOUT;
  if (st & eab::kStatusWordLaunch) return ATTN_ERR_CUDA;
  if (st & eab::kStatusWordBadSeqlens) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

const char* attn_status_string(int code) {
  switch (code) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "device pipeline wait timed out";
    default: return "unknown status";
  }
}

const char* attn_last_error(void) { return eab::t_last_error.c_str(); }

int attn_selftest_timeout(unsigned int timeout_us, cudaStream_t stream) {
  if (timeout_us < 1 || timeout_us > 10000000u) return ATTN_ERR_INVALID_ARG;
  int rc = eab::check_device();
  if (rc != ATTN_OK) return rc;
  eab::selftest_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(timeout_us) * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return eab::cuda_fail(e, "selftest_timeout_kernel launch");
  return ATTN_OK;
}

}  // extern "C"
