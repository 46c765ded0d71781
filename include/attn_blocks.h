/*
 * libattn_blocks -- building-block checks for the sm_100a attention kernel.
 *
 * Each entry point runs ONE of the hardware steps the attention kernel is built
 * from, in isolation and with the same layouts and descriptors, so that a test
 * can compare it against a plain host computation:
 *   - a TMA load of a 128-byte-swizzled tile and one tcgen05 MMA with both
 *     operands K-major in shared memory (the S = Q K^T step),
 *   - one tcgen05 MMA with A (BF16 pairs) in Tensor Memory and B MN-major in
 *     shared memory (the O += P V step),
 *   - the swizzled shared-memory addressing used by the epilogue, round-tripped
 *     through a TMA load and a 32-row-box TMA store,
 *   - the MUFU and the FMA-pipe polynomial exp2.
 * The steps are those of the tiled method: Q/K/V tiles staged on chip and the
 * products formed by the tensor cores (FlashAttention 4 page, ja.linux-konsole.com,
 * section "FlashAttention 4の新機能"); exp2 partly in software on the CUDA cores
 * (same page, section "CUDAコアによるソフトウェアの指数演算").
 *
 * All pointers are caller-owned DEVICE pointers; shapes are fixed per entry
 * point as documented.  Calls enqueue on `stream` and return at once; errors in
 * arguments return BLOCKS_ERR_INVALID_ARG without launching.  A device wait
 * that times out sets this library's status word (blocks_status_sync).
 */
#ifndef EXACT_ATTENTION_152_B200_ATTN_BLOCKS_H
#define EXACT_ATTENTION_152_B200_ATTN_BLOCKS_H

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *cudaStream_t;

enum {
  BLOCKS_OK = 0,
  BLOCKS_ERR_INVALID_ARG = 1, /* null/misaligned pointer, d not in {64,128}, n < 0 */
  BLOCKS_ERR_CUDA = 3,
  BLOCKS_ERR_TIMEOUT = 4
};

/* c[128][128] (FP32) = a[128][d] * b[128][d]^T; a, b BF16 row-major. */
int blocks_mma_ss(const void *a, const void *b, float *c, int d, cudaStream_t stream);

/* c[128][d] (FP32) = p[128][128] * v[128][d]; p, v BF16 row-major.  p is
 * written to Tensor Memory by the threads, v loaded by TMA. */
int blocks_mma_ts(const void *p, const void *v, float *c, int d, cudaStream_t stream);

/* x: BF16 [128][d].  TMA-loads x into shared memory (128-byte swizzle), reads
 * it back with the swizzle address formula into y_plain, and writes it again
 * through the swizzle formula + 32-row TMA stores into y_tma.  Both outputs
 * must equal x bit for bit. */
int blocks_swizzle_roundtrip(const void *x, void *y_tma, void *y_plain, int d,
                             cudaStream_t stream);

/* y_mufu[i] = hardware ex2.approx(x[i]); y_poly[i] = polynomial exp2(x[i]). */
int blocks_exp2(const float *x, float *y_mufu, float *y_poly, int n, cudaStream_t stream);

/* E4M3 (kind::f8f6f4) tile, both operands K-major: c[128][128] (fp32) =
 * a[128][128] * b[128][128]^T, a and b row-major E4M3 bytes. */
int blocks_mma_e4m3_ss(const void *a, const void *b, float *c, cudaStream_t stream);

/* E4M3 tile with A from Tensor Memory: c[128][128] = P[128][128] * v[128][128],
 * p = 128 rows x 32 words, four E4M3 per word (key 4i in the low byte of word i),
 * v row-major E4M3 [keys][d], read MN-major. */
int blocks_mma_e4m3_ts(const void *p, const void *v, float *c, cudaStream_t stream);

/* y[i] = the four E4M3 codes of x[4i..4i+3] (x[4i] in the low byte), round to
 * nearest even, saturating at +-448; n4 words. */
int blocks_pack_e4m3(const float *x, void *y, int n4, cudaStream_t stream);

/* Synchronise `stream`, read and clear this library's status word. */
int blocks_status_sync(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_152_B200_ATTN_BLOCKS_H */
