/*
 * libattn -- exact scaled dot-product attention, forward pass, for NVIDIA B200
 * (sm_100a).  C ABI: plain pointers, sizes and a CUDA stream; no C++ or
 * framework types cross this boundary.
 *
 * What is computed.  FlashAttention 4: LLM向けのより高速でメモリ効率の良いアテンション
 * (ja.linux-konsole.com), section "はじめに": attention multiplies the queries Q
 * with the keys K, normalises with a softmax and multiplies by the values V.
 * "Flash Attention（Flash Attention）" (jisaku.com glossary), section "タイリングによるSRAMの活用" and
 * "オンライン・ソフトマックスと再計算": the work is tiled through on-chip memory
 * with a running per-row max and sum, so the Nq x Nk score matrix never reaches
 * device memory; FAQ Q3 on the same page: the result equals standard attention
 * up to floating-point rounding.  The pages print no formula and never mention
 * the scale, causal masking or the log-sum-exp; this library defines, per
 * (b, h) and query row i:
 *
 *     s_ij   = scale * <q_i, k_j>            for j in K(i)
 *     K(i)   = {0..Nk-1}, or {0..i} when causal (requires Nq == Nk)
 *     O_i    = sum_j softmax_j(s_ij) * v_j
 *     LSE_i  = log(sum_j exp(s_ij))           natural logarithm
 *     K(i) empty (Nk == 0): O_i = 0, LSE_i = -inf
 *
 * Layout.  q, k, v, o are BF16, contiguous, row-major [B, H, N, d] with d
 * fastest (N = Nq for q and o, N = Nk for k and v).  lse is FP32 [B, H, Nq].
 * Arithmetic: BF16 products, FP32 accumulation and softmax, O rounded to BF16
 * (round to nearest even) once at the end.
 *
 * Ownership.  Every pointer is a DEVICE pointer owned by the caller.  The
 * library never allocates, frees or retains them.  o and lse must not overlap
 * q, k, v or each other.
 *
 * Asynchrony.  attn_fwd() validates its arguments on the host, enqueues the
 * work on `stream` (NULL = the legacy default stream) and returns without
 * synchronising.  Outputs are valid once the stream reaches that point.
 *
 * Errors.  Argument errors are detected on the host before anything is
 * enqueued and nothing is launched.  A device-side failure (a pipeline wait
 * that exceeded its time limit) sets a per-device status word, reported and
 * cleared by attn_status_sync().
 */
#ifndef EXACT_ATTENTION_152_B200_ATTN_H
#define EXACT_ATTENTION_152_B200_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

#include <stddef.h>

/* Same definition as the CUDA runtime's (an opaque driver stream handle). */
typedef struct CUstream_st *cudaStream_t;

enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null pointer with non-empty problem, negative size,
                               non-finite scale, misaligned pointer (q,k,v,o need
                               16-byte alignment, lse 4-byte), overlapping outputs */
  ATTN_ERR_UNSUPPORTED = 2, /* d not in {64,128}, causal with Nq != Nk, device is
                               not compute capability 10.0, exp_mode/threshold out
                               of range */
  ATTN_ERR_CUDA = 3,        /* CUDA runtime/driver failure (text: attn_last_error) */
  ATTN_ERR_TIMEOUT = 4      /* a device pipeline wait exceeded its limit */
};

/*
 * Forward attention (see the definition above).
 *   q, k, v  : device, BF16 [B,H,Nq,d], [B,H,Nk,d], [B,H,Nk,d]
 *   o        : device, BF16 [B,H,Nq,d], written
 *   lse      : device, FP32 [B,H,Nq], written; may be NULL (not computed)
 *   B,H,Nq,Nk: >= 0; a problem with B*H*Nq == 0 is a no-op (pointers may be NULL)
 *   d        : head dimension, 64 or 128
 *   scale    : any finite float (0 gives uniform weights); not defaulted here
 *   causal   : 0 or 1; 1 requires Nq == Nk
 *   stream   : CUDA stream to enqueue on
 * Returns ATTN_OK or an error code; on error nothing was enqueued.
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
             int Nq, int Nk, int d, float scale, int causal, cudaStream_t stream);

/*
 * Grouped-query / multi-query attention (same contract as attn_fwd otherwise).
 * The pages list GQA/MQA among what FlashAttention 4's forward still lacks
 * (FlashAttention 4 page, ja.linux-konsole.com, sections "重要ポイント" and
 * "互換性と現状"): several query heads share one key/value head.
 *   q, o : [B, H, Nq, d];   k, v : [B, Hkv, Nk, d];   lse : [B, H, Nq]
 *   Hkv  : key/value heads, 1 <= Hkv <= H with H % Hkv == 0 (Hkv == 1 is
 *          multi-query attention, Hkv == H is attn_fwd)
 * Query head h of batch b attends to key/value head h / (H / Hkv) of batch b.
 * H % Hkv != 0 or Hkv <= 0 with H > 0 returns ATTN_ERR_INVALID_ARG.
 */
int attn_fwd_gqa(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                 int Hkv, int Nq, int Nk, int d, float scale, int causal, cudaStream_t stream);

/*
 * Sliding-window (local) attention: each query sees a band of keys around its
 * own position.  The pages only name richer masks than causal ("AIの「脳の回転」
 * を1.8倍高速化？FlashAttentionの秘密", gipyeong-lee.github.io, section
 * "今後はどうなるか？", pointing to FlashMask); this library's reading is
 *
 *     K(i) = { j : 0 <= j < Nk,  i - window_left <= j <= i + window_right }
 *
 * with -1 for "no bound on that side": (-1, -1) is attn_fwd non-causal,
 * (-1, 0) is causal, (w, 0) is causal attention over the last w+1 keys.
 * Positions of queries and keys both count from 0, so Nq != Nk is allowed; a
 * row whose band holds no key gets O = 0, LSE = -inf.
 *   q, o : [B, H, Nq, d];  k, v : [B, Hkv, Nk, d];  lse : [B, H, Nq] (may be NULL)
 *   Hkv  : as attn_fwd_gqa (Hkv == H: one key/value head per query head)
 *   window_left, window_right : >= -1; anything below -1 is ATTN_ERR_INVALID_ARG
 * Only KV tiles that hold a visible key are read.
 */
int attn_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                    int H, int Hkv, int Nq, int Nk, int d, float scale, int window_left,
                    int window_right, cudaStream_t stream);

/*
 * Column-interval ("FlashMask-style") masks.  The same page that points to
 * FlashMask ("AIの「脳の回転」を1.8倍高速化？FlashAttentionの秘密",
 * gipyeong-lee.github.io, section "今後はどうなるか？") names it only as an
 * extension that handles masks more precisely; it gives no representation.
 * This library's reading: for every key column j, up to two intervals of query
 * rows that do not see key j,
 *
 *     K(i) = { j : 0 <= j < Nk,  not (lo1_j <= i < hi1_j),  not (lo2_j <= i < hi2_j),
 *                 and j <= i if causal }
 *
 * which holds document (block-diagonal) masks, prefix-LM masks, shared-prefix
 * masks and bands in O(Nk) memory.  An interval with lo >= hi is empty.  A row
 * that sees no key gets O = 0, LSE = -inf.
 *   q, o : [B, H, Nq, d];  k, v : [B, Hkv, Nk, d];  lse : [B, H, Nq] (may be NULL)
 *   Hkv, d, scale : as attn_fwd_gqa;  causal : 0 or 1 (j <= i, any Nq, Nk)
 *   mask : DEVICE int32 [B, Hm, Nk, 4], each key's (lo1, hi1, lo2, hi2), 16-byte
 *          aligned; Hm == 1 (one mask per batch entry, shared by all heads) or
 *          Hm == H (one per query head).  Read only.
 *   workspace : DEVICE, 16-byte aligned, owned by the caller; give it
 *          attn_colmask_workspace_size(B, Hm, Nk) bytes.  The call overwrites
 *          it with per-128-key-block summaries of the mask (32 bytes per mask
 *          row and key block: the minimum accepted) and, where the workspace
 *          has room for one int per mask row and 256-row query block (the size
 *          function allows for Nq <= 4 Nk; up to 8192 such units, and mask
 *          rows x (key blocks + 1) up to 4096), with an
 *          order of the attention kernel's CTAs.  It may not overlap any other
 *          argument.  Calls on different streams need different workspaces.
 * The call launches two or three kernels on `stream`: the block summaries;
 * when the workspace has room for it, a one-CTA kernel that orders the query
 * blocks of each mask row by the number of key blocks they visit, longest
 * first (the order changes no result); then the attention kernel, which skips every 128-key
 * block that hides all 256 query rows of a CTA and masks element-wise only in
 * blocks whose intervals meet a warp's 32 rows.  Errors as attn_fwd_gqa, plus ATTN_ERR_INVALID_ARG for a NULL
 * or misaligned mask or workspace, a workspace that is too small or overlaps
 * another argument, or Hm not in {1, H}, and ATTN_ERR_UNSUPPORTED for more than
 * 65536 key blocks of 128 (8M keys: the kernel keeps one bit per key block).
 */
size_t attn_colmask_workspace_size(int B, int Hm, int Nk);
int attn_fwd_colmask(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                     int H, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     const int *mask, int Hm, void *workspace, size_t workspace_bytes,
                     cudaStream_t stream);

/*
 * Variable-length batch: sequences of different lengths packed back to back,
 * with no padding (FlashAttention 4 page, ja.linux-konsole.com, section
 * "互換性と現状", lists this among what FA4's forward lacks).
 *   q, o : BF16 [total_q, H, d]    k, v : BF16 [total_k, Hkv, d]   (d fastest)
 *   lse  : FP32 [H, total_q], may be NULL
 *   cu_seqlens_q, cu_seqlens_k : DEVICE int32 arrays of num_seqs + 1 entries;
 *       sequence s owns query rows cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 and
 *       key/value rows cu_seqlens_k[s] .. cu_seqlens_k[s+1]-1 (non-decreasing,
 *       starting at >= 0, ending at <= total_q / total_k; a sequence may be
 *       empty, and its query and key lengths may differ)
 *   max_seqlen_q : an upper bound on every sequence's query length (sizes the
 *       grid), 1 <= max_seqlen_q <= total_q when total_q > 0
 *   H, Hkv, d, scale : as attn_fwd_gqa
 *   window_left, window_right : the band of attn_fwd_window over positions
 *       counted from 0 within each sequence; (-1, 0) is causal, (-1, -1) none
 * Each sequence is attended independently: no query sees another sequence's
 * keys.  The offsets live on the device and are not read by the host: offsets
 * that break the rules above (or a sequence longer than max_seqlen_q rounded up
 * to 256) make the kernel skip that sequence and record the fact, which the next
 * attn_status_sync() returns as ATTN_ERR_INVALID_ARG; no access goes outside
 * the tensors.  All other errors are detected on the host as for attn_fwd.
 */
int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                    const int *cu_seqlens_q, const int *cu_seqlens_k, int num_seqs,
                    int max_seqlen_q, int total_q, int total_k, int H, int Hkv, int d,
                    float scale, int window_left, int window_right, cudaStream_t stream);

/*
 * FP8 forward: Q, K, V given as E4M3 bytes (OCP E4M3FN: 4 exponent bits with
 * bias 7, 3 mantissa bits, largest finite value 448) with one scale factor per
 * tensor, so the attended values are q_descale * Q8, k_descale * K8 and
 * v_descale * V8.  The pages name the FP8 forward among FlashAttention 3's
 * improvements ("Flash Attention（Flash Attention）", jisaku.com glossary,
 * sections "ハードウェアへの影響と推奨スペック" and "FlashAttention-3とFP8の時代");
 * the definition is that of
 * attn_fwd on those values:
 *
 *     s_ij = scale * q_descale * k_descale * <Q8_i, K8_j>
 *     O_i  = v_descale * sum_j softmax_j(s_ij) * V8_j,   LSE_i as in attn_fwd
 *
 * Q.K^T and P.V run on the tensor cores in E4M3 (kind::f8f6f4) with FP32
 * accumulation; P is rounded to E4M3 for P.V (O's error is therefore of the
 * order of E4M3's 2^-4 relative rounding of the weights, not BF16's 2^-9).
 *   q : [B, H, Nq, d] bytes;  k, v : [B, Hkv, Nk, d] bytes;  d must be 128
 *   o : BF16 [B, H, Nq, d];   lse : FP32 [B, H, Nq] (may be NULL)
 *   q_descale, k_descale, v_descale : finite floats
 *   Hkv, causal and everything else as attn_fwd_gqa.
 */
int attn_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                 int Hkv, int Nq, int Nk, int d, float scale, float q_descale, float k_descale,
                 float v_descale, int causal, cudaStream_t stream);

/*
 * attn_fwd with the kernel's two softmax knobs exposed (same contract otherwise).
 *
 *   rescale_threshold : adaptive online rescaling (FlashAttention 4 page,
 *       section "よりスマートなオンラインソフトマックス再スケーリング"): the running
 *       max of a row is replaced -- and the accumulated output and sum rescaled
 *       -- only when a tile's max exceeds it by more than this many powers of
 *       two.  0 reproduces the classic always-rescale rule.  Range [0, 64].
 *       attn_fwd uses 8.
 *   exp_mode : where exp2 runs (same page, section "CUDAコアによるソフトウェアの
 *       指数演算"): 0 = hardware MUFU only, 1 = the library's default split
 *       between MUFU and a cubic polynomial on the FMA pipe, 2 = polynomial only.
 *   rescale_count : optional device pointer (may be NULL) to one unsigned
 *       64-bit counter; the kernel atomically adds the number of (row, tile)
 *       events at which the output accumulator was rescaled.
 */
int attn_fwd_config(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                    int H, int Nq, int Nk, int d, float scale, int causal,
                    float rescale_threshold, int exp_mode, unsigned long long *rescale_count,
                    cudaStream_t stream);

/*
 * Backward pass: the gradients dQ, dK, dV of the forward above (causal or not,
 * grouped key/value heads allowed) for the output cotangent dO.  The pages name
 * the backward pass as what FlashAttention 4 lacks (FlashAttention 4 page,
 * ja.linux-konsole.com, sections "重要ポイント" and "互換性と現状";
 * "FlashAttention-4：非対称ハードウェアスケーリング…" (sns.style), section 二) and give no formula; this
 * library computes the chain rule through the definition above:
 *
 *     P_ij  = exp(scale * <q_i, k_j> - LSE_i)      (j visible to i, else 0)
 *     dS_ij = P_ij * (<dO_i, v_j> - <dO_i, O_i>)
 *     dV_j  = sum_i P_ij dO_i
 *     dK_j  = scale * sum_i dS_ij q_i,   dQ_i = scale * sum_j dS_ij k_j
 *
 * summed over the query heads that share a key/value head.
 *   q, o, dout : BF16 [B, H, Nq, d]      k, v : BF16 [B, Hkv, Nk, d]
 *   lse        : FP32 [B, H, Nq], the forward's log-sum-exp (natural log)
 *   dq         : BF16 [B, H, Nq, d] written;  dk, dv : BF16 [B, Hkv, Nk, d] written
 *   workspace  : DEVICE scratch of at least attn_bwd_workspace_size(B, H, Nq, d)
 *                bytes, 256-byte aligned, owned by the caller, not overlapping
 *                any other argument; its contents are overwritten (the row sums
 *                <dO_i, O_i> and dQ's fp32 accumulator)
 *   B, H, Hkv, Nq, Nk, d, scale, causal : as attn_fwd_gqa
 * All pointers 16-byte aligned (lse 4).  Outputs may not overlap inputs or each
 * other.  Nk == 0 gives dQ = 0; Nq == 0 gives dK = dV = 0.  Asynchronous on
 * `stream` like attn_fwd; argument errors are returned before anything is
 * enqueued, device-side failures through attn_status_sync().
 */
int attn_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
             const float *lse, void *dq, void *dk, void *dv, void *workspace,
             size_t workspace_bytes, int B, int H, int Hkv, int Nq, int Nk, int d, float scale,
             int causal, cudaStream_t stream);

/*
 * attn_bwd for the key band of attn_fwd_window: key j is visible to query i
 * when i - window_left <= j <= i + window_right (-1: no bound on that side;
 * (-1, 0) is causal, (-1, -1) unmasked), positions counted from 0 for queries
 * and keys alike, so Nq != Nk is allowed.  Keys no query sees get dK = dV = 0.
 * window_left, window_right below -1 return ATTN_ERR_INVALID_ARG; everything
 * else is as attn_bwd (lse must come from attn_fwd_window with the same band).
 */
int attn_bwd_window(const void *q, const void *k, const void *v, const void *o, const void *dout,
                    const float *lse, void *dq, void *dk, void *dv, void *workspace,
                    size_t workspace_bytes, int B, int H, int Hkv, int Nq, int Nk, int d,
                    float scale, int window_left, int window_right, cudaStream_t stream);

/*
 * Backward of attn_fwd_varlen: a packed variable-length batch (sequences back
 * to back, no padding; FlashAttention 4 page, ja.linux-konsole.com, section
 * "互換性と現状", names variable-length batches and the backward pass among
 * what FA4 lacks), the same chain rule as attn_bwd within each sequence.
 *   q, o, dout, dq : BF16 [total_q, H, d]    k, v, dk, dv : BF16 [total_k, Hkv, d]
 *   lse  : FP32 [H, total_q], attn_fwd_varlen's log-sum-exp
 *   cu_seqlens_q, cu_seqlens_k, num_seqs : as attn_fwd_varlen (DEVICE int32)
 *   max_seqlen_k : an upper bound on every sequence's key length (sizes the
 *       grid), 1 <= max_seqlen_k <= total_k when total_k > 0
 *   workspace : DEVICE scratch of at least attn_bwd_workspace_size(1, H, total_q, d)
 *       bytes, 256-byte aligned, owned by the caller, overwritten
 *   H, Hkv, d, scale, window_left, window_right : as attn_fwd_varlen
 * Query rows that belong to no sequence get dQ = 0; key rows that belong to no
 * sequence are not written.  Offsets that break attn_fwd_varlen's rules, or a
 * key length beyond max_seqlen_k rounded up to 128, make the kernel skip that
 * sequence and record the fact, which the next attn_status_sync() returns as
 * ATTN_ERR_INVALID_ARG.  Other errors as attn_bwd.
 */
/*
 * Backward of attn_fwd_colmask (column intervals; see that call for the mask):
 * the chain rule of attn_bwd over the visible (query, key) pairs.
 *   q, o, dout, dq : BF16 [B, H, Nq, d]    k, v, dk, dv : BF16 [B, Hkv, Nk, d]
 *   lse  : FP32 [B, H, Nq] from attn_fwd_colmask
 *   mask, Hm, causal : as attn_fwd_colmask
 *   workspace : DEVICE, 256-byte aligned; give it
 *       attn_bwd_colmask_workspace_size(B, H, Nq, d, Hm, Nk) bytes: attn_bwd's
 *       workspace followed by the mask's block summaries (together the
 *       minimum accepted), then room for an order of the CTAs (one int per
 *       head and 128-key block); overwritten
 * Each CTA owns a 128-key block; the query tiles that every key of the block
 * hides form at most two ranges per query head, which are skipped outright.
 * When the workspace has room (and the problem has at most 8192 CTAs), a
 * one-CTA kernel orders the CTAs by the query tiles they visit, longest first
 * within groups of key/value heads (the order changes no result).
 * Errors as attn_bwd, plus ATTN_ERR_INVALID_ARG for a NULL or misaligned mask,
 * Hm not in {1, H}, or a mask overlapping an output or the workspace.
 */
size_t attn_bwd_colmask_workspace_size(int B, int H, int Nq, int d, int Hm, int Nk);
int attn_bwd_colmask(const void *q, const void *k, const void *v, const void *o, const void *dout,
                     const float *lse, void *dq, void *dk, void *dv, void *workspace,
                     size_t workspace_bytes, int B, int H, int Hkv, int Nq, int Nk, int d, float scale,
                     int causal, const int *mask, int Hm, cudaStream_t stream);

int attn_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const void *dout,
                    const float *lse, void *dq, void *dk, void *dv, void *workspace,
                    size_t workspace_bytes, const int *cu_seqlens_q, const int *cu_seqlens_k,
                    int num_seqs, int max_seqlen_k, int total_q, int total_k, int H, int Hkv, int d,
                    float scale, int window_left, int window_right, cudaStream_t stream);

/* Workspace bytes attn_bwd needs (0 for d not in {64, 128} or negative sizes). */
size_t attn_bwd_workspace_size(int B, int H, int Nq, int d);

/*
 * attn_bwd without a workspace argument: the workspace is a file-scope device
 * array of 96 MiB (100663296 bytes) per device inside the library, so the call
 * allocates no memory (no cudaMalloc / cudaFree).  Problems whose
 * attn_bwd_workspace_size exceeds 96 MiB return ATTN_ERR_UNSUPPORTED before
 * anything else is done.  Every call on a device uses the same array: calls
 * must be ordered (one stream, or synchronised between streams).  Arguments
 * and results are otherwise those of attn_bwd.
 *
 * The array lives in the same device module as every backward kernel, so the
 * 96 MiB are resident on a device as soon as any backward entry point
 * (attn_bwd, attn_bwd_window, attn_bwd_varlen, attn_bwd_colmask or this one)
 * has run there -- from context creation under CUDA_MODULE_LOADING=EAGER --
 * whether or not attn_bwd_noalloc is ever called.  The array's device address
 * is looked up once per device and context (again after cudaDeviceReset or
 * when another context becomes current), on the first call there; make that
 * first call before any stream capture.
 */
int attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const void *dout,
                     const float *lse, void *dq, void *dk, void *dv, int B, int H, int Hkv, int Nq,
                     int Nk, int d, float scale, int causal, cudaStream_t stream);

/*
 * Synchronise `stream`, then read and clear the current device's status word.
 * Returns ATTN_OK, ATTN_ERR_TIMEOUT (a kernel gave up on a pipeline wait since
 * the last call; its outputs are not valid), ATTN_ERR_INVALID_ARG (an
 * attn_fwd_varlen call met bad sequence offsets on the device; the outputs of
 * those sequences were not written) or ATTN_ERR_CUDA.
 */
int attn_status_sync(cudaStream_t stream);

/* Static English text for a return code. */
const char *attn_status_string(int code);

/* Text of the last ATTN_ERR_CUDA raised on the calling thread ("" if none). */
const char *attn_last_error(void);

/*
 * Diagnostic: launch one block that waits on a pipeline barrier nothing will
 * ever signal, with the library's bounded wait limited to `timeout_us`
 * microseconds (1..10,000,000).  The wait runs out, the block records
 * ATTN_ERR_TIMEOUT in the status word and exits normally, leaving the CUDA
 * context usable.  Lets a caller check its failure handling without a fault.
 */
int attn_selftest_timeout(unsigned int timeout_us, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_152_B200_ATTN_H */
