// Building-block checks for the attention kernel (see include/attn_blocks.h).
// Each kernel exercises one hardware step with exactly the layouts, swizzle
// and descriptors attn_fwd.cu uses, on a single 128-row tile.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>

#include "attn_blocks.h"
#include "exp2.cuh"
#include "sm100.cuh"
#include "tmap.h"

namespace eab_blocks {
using namespace eab;

constexpr uint64_t kTimeoutNs = 1000000000ull;  // 1 s
constexpr int kBox = 128 * 128;                  // 128 rows x 128 bytes

__device__ unsigned int g_blk_status;

__device__ __forceinline__ uint8_t* align1024(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return raw + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, kTimeoutNs));
}

// c[128][128] = a[128][D] * b[128][D]^T, both operands K-major, 128B swizzle.
template <int D>
__global__ void __launch_bounds__(128, 1)
mma_ss_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, float* c) {
  extern __shared__ uint8_t raw[];
  uint8_t* base = align1024(raw);
  constexpr int kBoxes = D / 64;
  const uint32_t sA = smem_u32(base), sB = sA + kBoxes * kBox;
  const uint32_t full = sB + kBoxes * kBox, done = full + 8;
  uint32_t* slot = reinterpret_cast<uint32_t*>(base + 2 * kBoxes * kBox + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  bool ok = true;
  if (tid == 0) {
    mbar_arrive_expect_tx(full, 2 * kBoxes * kBox);
    for (int b = 0; b < kBoxes; ++b) {
      tma_load_3d(sA + b * kBox, &ta, b * 64, 0, 0, full);
      tma_load_3d(sB + b * kBox, &tb, b * 64, 0, 0, full);
    }
    ok = mbar_wait(full, 0, kTimeoutNs);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
        mma_ss(tmem, sdesc_sw128(sA + off, 16, 1024), sdesc_sw128(sB + off, 16, 1024), idesc,
               kk > 0 ? 1u : 0u);
      }
    } else {
      mbar_wait(full, 0, kTimeoutNs);  // give an in-flight copy one more chance to land
    }
    tc_commit(done);
  }
  __syncwarp();
  const bool ok2 = warp_wait(done, 0);
  if (ok2) {
    tc_fence_after();
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int row = warp * 32 + lane;
    for (int q = 0; q < 4; ++q) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + q * 32, r);
      tmem_ld_wait();
      reg_fence32(r);
      for (int i = 0; i < 32; ++i) c[row * 128 + q * 32 + i] = __uint_as_float(r[i]);
    }
  }
  if (!ok || !ok2) atomicOr(&g_blk_status, 1u);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// c[128][D] = p[128][128] * v[128][D]; P written to TMEM by the threads (BF16
// pairs, element 2i in the low half of column i), V MN-major via TMA.
template <int D>
__global__ void __launch_bounds__(128, 1)
mma_ts_kernel(const uint32_t* p, const __grid_constant__ CUtensorMap tv, float* c) {
  extern __shared__ uint8_t raw[];
  uint8_t* base = align1024(raw);
  constexpr int kBoxes = D / 64;
  const uint32_t sV = smem_u32(base);
  const uint32_t full = sV + kBoxes * kBox, done = full + 8;
  uint32_t* slot = reinterpret_cast<uint32_t*>(base + kBoxes * kBox + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const int row = warp * 32 + lane;
  {
    uint32_t pr0[32], pr1[32];
    for (int i = 0; i < 32; ++i) {
      pr0[i] = p[row * 64 + i];
      pr1[i] = p[row * 64 + 32 + i];
    }
    tmem_st32(tmem + lane_off, pr0);
    tmem_st32(tmem + lane_off + 32, pr1);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  if (tid == 0) {
    tc_fence_after();
    mbar_arrive_expect_tx(full, kBoxes * kBox);
    for (int b = 0; b < kBoxes; ++b) tma_load_3d(sV + b * kBox, &tv, b * 64, 0, 0, full);
    ok = mbar_wait(full, 0, kTimeoutNs);
    if (ok) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tmem + 256, tmem + kk * 8, sdesc_sw128(sV + kk * 2048, kBox, 1024), idesc,
               kk > 0 ? 1u : 0u);
    } else {
      mbar_wait(full, 0, kTimeoutNs);
    }
    tc_commit(done);
  }
  __syncwarp();
  const bool ok2 = warp_wait(done, 0);
  if (ok2) {
    tc_fence_after();
    for (int q = 0; q < D / 32; ++q) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + 256 + q * 32, r);
      tmem_ld_wait();
      reg_fence32(r);
      for (int i = 0; i < 32; ++i) c[row * D + q * 32 + i] = __uint_as_float(r[i]);
    }
  }
  if (!ok || !ok2) atomicOr(&g_blk_status, 1u);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// TMA load (128-row box) -> swizzle-formula reads -> plain global copy, and
// swizzle-formula writes -> 32-row-box TMA stores (the epilogue's path).
template <int D>
__global__ void __launch_bounds__(128, 1)
swizzle_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap ty32,
               uint16_t* y_plain) {
  extern __shared__ uint8_t raw[];
  uint8_t* base = align1024(raw);
  constexpr int kBoxes = D / 64;
  uint8_t* gX = base;
  uint8_t* gY = base + kBoxes * kBox;
  const uint32_t sX = smem_u32(gX), sY = smem_u32(gY);
  const uint32_t full = sY + kBoxes * kBox;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(full, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(full, kBoxes * kBox);
    for (int b = 0; b < kBoxes; ++b) tma_load_3d(sX + b * kBox, &tx, b * 64, 0, 0, full);
  }
  __syncwarp();
  const bool ok = warp_wait(full, 0);
  if (ok) {
    const int r = tid;
    for (int k = 0; k < D / 8; ++k) {
      const int box = k >> 3, kc = k & 7;
      const int off = box * kBox + r * 128 + ((kc ^ (r & 7)) * 16);
      const uint4 v = *reinterpret_cast<const uint4*>(gX + off);
      *reinterpret_cast<uint4*>(y_plain + r * D + k * 8) = v;
      *reinterpret_cast<uint4*>(gY + off) = v;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      for (int b = 0; b < kBoxes; ++b)
        tma_store_3d(&ty32, sY + b * kBox + warp * 32 * 128, b * 64, warp * 32, 0);
      bulk_commit_group();
      bulk_wait_group0();
    }
  } else {
    atomicOr(&g_blk_status, 1u);
  }
  __syncthreads();
}

// 8-bit operands (kind::f8f6f4, E4M3).  SS: c[128][128] = a[128][128] *
// b[128][128]^T, both K-major (one 128-byte box per row, K steps of 32 bytes).
// TS: c[128][128] = p[128][128 keys] * v[128 keys][128]; P written to TMEM by
// the threads, four E4M3 per column (key 4i in the low byte of column i), V
// MN-major (rows of 128 bytes along d, 32 key rows = 4096 bytes per K step).
template <bool TS>
__global__ void __launch_bounds__(128, 1)
mma_e4m3_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                const uint32_t* p, float* c) {
  extern __shared__ uint8_t raw[];
  uint8_t* base = align1024(raw);
  const uint32_t sA = smem_u32(base), sB = sA + kBox;
  const uint32_t full = sB + kBox, done = full + 8;
  uint32_t* slot = reinterpret_cast<uint32_t*>(base + 2 * kBox + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const int row = warp * 32 + lane;
  if (TS) {
    uint32_t pr[32];
    for (int i = 0; i < 32; ++i) pr[i] = p[row * 32 + i];
    tmem_st32(tmem + lane_off + 128, pr);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  if (tid == 0) {
    tc_fence_after();
    mbar_arrive_expect_tx(full, TS ? kBox : 2 * kBox);
    if (!TS) tma_load_3d(sA, &ta, 0, 0, 0, full);
    tma_load_3d(sB, &tb, 0, 0, 0, full);
    ok = mbar_wait(full, 0, kTimeoutNs);
    if (ok) {
      if (TS) {
        constexpr uint32_t idesc = idesc_e4m3_f32(128, 128, false, true);
        const uint64_t bd = sdesc_sw128(sB, kBox, 1024);
        const uint32_t b_lo = static_cast<uint32_t>(bd), b_hi = static_cast<uint32_t>(bd >> 32);
        mma_ts_imm_f8<0, 0>(tmem, tmem + 128, b_lo, b_hi, idesc, 0u);
        mma_ts_imm_f8<8, (4096 >> 4)>(tmem, tmem + 128, b_lo, b_hi, idesc, 1u);
        mma_ts_imm_f8<16, (8192 >> 4)>(tmem, tmem + 128, b_lo, b_hi, idesc, 1u);
        mma_ts_imm_f8<24, (12288 >> 4)>(tmem, tmem + 128, b_lo, b_hi, idesc, 1u);
      } else {
        constexpr uint32_t idesc = idesc_e4m3_f32(128, 128, false, false);
        const uint64_t ad = sdesc_sw128(sA, 16, 1024), bd = sdesc_sw128(sB, 16, 1024);
        const uint32_t a_lo = static_cast<uint32_t>(ad), a_hi = static_cast<uint32_t>(ad >> 32);
        const uint32_t b_lo = static_cast<uint32_t>(bd), b_hi = static_cast<uint32_t>(bd >> 32);
        mma_ss_imm_f8<0, 0, 0u>(tmem, a_lo, a_hi, b_lo, b_hi, idesc);
        mma_ss_imm_f8<2, 2, 1u>(tmem, a_lo, a_hi, b_lo, b_hi, idesc);
        mma_ss_imm_f8<4, 4, 1u>(tmem, a_lo, a_hi, b_lo, b_hi, idesc);
        mma_ss_imm_f8<6, 6, 1u>(tmem, a_lo, a_hi, b_lo, b_hi, idesc);
      }
    } else {
      mbar_wait(full, 0, kTimeoutNs);
    }
    tc_commit(done);
  }
  __syncwarp();
  const bool ok2 = warp_wait(done, 0);
  if (ok2) {
    tc_fence_after();
    for (int q = 0; q < 4; ++q) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + q * 32, r);
      tmem_ld_wait();
      reg_fence32(r);
      for (int i = 0; i < 32; ++i) c[row * 128 + q * 32 + i] = __uint_as_float(r[i]);
    }
  }
  if (!ok || !ok2) atomicOr(&g_blk_status, 1u);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void pack_e4m3_kernel(const float* x, uint32_t* y, int n4) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n4) y[i] = pack_e4m3x4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}

__global__ void exp2_kernel(const float* x, float* y_mufu, float* y_poly, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    y_mufu[i] = ex2_mufu(x[i]);
    y_poly[i] = ex2_poly(x[i]);
  }
}

thread_local std::string t_err;

int fail(cudaError_t e, const char* what) {
  t_err = std::string(what) + ": " + cudaGetErrorString(e);
  return BLOCKS_ERR_CUDA;
}

bool bad_ptr(const void* p) { return !p || (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

int set_smem(const void* fn, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "cudaFuncSetAttribute");
}

}  // namespace eab_blocks

using namespace eab_blocks;

extern "C" {

int blocks_mma_ss(const void* a, const void* b, float* c, int d, cudaStream_t stream) {
  if (bad_ptr(a) || bad_ptr(b) || bad_ptr(c) || (d != 64 && d != 128)) return BLOCKS_ERR_INVALID_ARG;
  CUtensorMap ta, tb;
  if (!eab::make_tmap_bf16_3d(&ta, a, 1, 128, d, 128, &t_err) ||
      !eab::make_tmap_bf16_3d(&tb, b, 1, 128, d, 128, &t_err))
    return BLOCKS_ERR_CUDA;
  const int smem = 2 * (d / 64) * kBox + 1024 + 64;
  int rc;
  if (d == 128) {
    if ((rc = set_smem((const void*)mma_ss_kernel<128>, smem)) != BLOCKS_OK) return rc;
    mma_ss_kernel<128><<<1, 128, smem, stream>>>(ta, tb, c);
  } else {
    if ((rc = set_smem((const void*)mma_ss_kernel<64>, smem)) != BLOCKS_OK) return rc;
    mma_ss_kernel<64><<<1, 128, smem, stream>>>(ta, tb, c);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "mma_ss_kernel launch");
}

int blocks_mma_ts(const void* p, const void* v, float* c, int d, cudaStream_t stream) {
  if (bad_ptr(p) || bad_ptr(v) || bad_ptr(c) || (d != 64 && d != 128)) return BLOCKS_ERR_INVALID_ARG;
  CUtensorMap tv;
  if (!eab::make_tmap_bf16_3d(&tv, v, 1, 128, d, 128, &t_err)) return BLOCKS_ERR_CUDA;
  const int smem = (d / 64) * kBox + 1024 + 64;
  int rc;
  const uint32_t* pu = static_cast<const uint32_t*>(p);
  if (d == 128) {
    if ((rc = set_smem((const void*)mma_ts_kernel<128>, smem)) != BLOCKS_OK) return rc;
    mma_ts_kernel<128><<<1, 128, smem, stream>>>(pu, tv, c);
  } else {
    if ((rc = set_smem((const void*)mma_ts_kernel<64>, smem)) != BLOCKS_OK) return rc;
    mma_ts_kernel<64><<<1, 128, smem, stream>>>(pu, tv, c);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "mma_ts_kernel launch");
}

int blocks_swizzle_roundtrip(const void* x, void* y_tma, void* y_plain, int d, cudaStream_t stream) {
  if (bad_ptr(x) || bad_ptr(y_tma) || bad_ptr(y_plain) || (d != 64 && d != 128))
    return BLOCKS_ERR_INVALID_ARG;
  CUtensorMap tx, ty;
  if (!eab::make_tmap_bf16_3d(&tx, x, 1, 128, d, 128, &t_err) ||
      !eab::make_tmap_bf16_3d(&ty, y_tma, 1, 128, d, 32, &t_err))
    return BLOCKS_ERR_CUDA;
  const int smem = 2 * (d / 64) * kBox + 1024 + 64;
  int rc;
  uint16_t* yp = static_cast<uint16_t*>(y_plain);
  if (d == 128) {
    if ((rc = set_smem((const void*)swizzle_kernel<128>, smem)) != BLOCKS_OK) return rc;
    swizzle_kernel<128><<<1, 128, smem, stream>>>(tx, ty, yp);
  } else {
    if ((rc = set_smem((const void*)swizzle_kernel<64>, smem)) != BLOCKS_OK) return rc;
    swizzle_kernel<64><<<1, 128, smem, stream>>>(tx, ty, yp);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "swizzle_kernel launch");
}

int blocks_exp2(const float* x, float* y_mufu, float* y_poly, int n, cudaStream_t stream) {
  if (n < 0) return BLOCKS_ERR_INVALID_ARG;
  if (n == 0) return BLOCKS_OK;
  if (!x || !y_mufu || !y_poly) return BLOCKS_ERR_INVALID_ARG;
  exp2_kernel<<<(n + 255) / 256, 256, 0, stream>>>(x, y_mufu, y_poly, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "exp2_kernel launch");
}

int blocks_mma_e4m3_ss(const void* a, const void* b, float* c, cudaStream_t stream) {
  if (bad_ptr(a) || bad_ptr(b) || bad_ptr(c)) return BLOCKS_ERR_INVALID_ARG;
  CUtensorMap ta, tb;
  if (!eab::make_tmap_u8_3d(&ta, a, 1, 128, 128, 128, &t_err) ||
      !eab::make_tmap_u8_3d(&tb, b, 1, 128, 128, 128, &t_err))
    return BLOCKS_ERR_CUDA;
  const int smem = 2 * kBox + 1024 + 64;
  int rc;
  if ((rc = set_smem((const void*)mma_e4m3_kernel<false>, smem)) != BLOCKS_OK) return rc;
  mma_e4m3_kernel<false><<<1, 128, smem, stream>>>(ta, tb, nullptr, c);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "mma_e4m3_kernel launch");
}

int blocks_mma_e4m3_ts(const void* p, const void* v, float* c, cudaStream_t stream) {
  if (bad_ptr(p) || bad_ptr(v) || bad_ptr(c)) return BLOCKS_ERR_INVALID_ARG;
  CUtensorMap tv;
  if (!eab::make_tmap_u8_3d(&tv, v, 1, 128, 128, 128, &t_err)) return BLOCKS_ERR_CUDA;
  const int smem = 2 * kBox + 1024 + 64;
  int rc;
  if ((rc = set_smem((const void*)mma_e4m3_kernel<true>, smem)) != BLOCKS_OK) return rc;
  mma_e4m3_kernel<true><<<1, 128, smem, stream>>>(tv, tv, static_cast<const uint32_t*>(p), c);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "mma_e4m3_kernel launch");
}

int blocks_pack_e4m3(const float* x, void* y, int n4, cudaStream_t stream) {
  if (n4 < 0) return BLOCKS_ERR_INVALID_ARG;
  if (n4 == 0) return BLOCKS_OK;
  if (!x || !y) return BLOCKS_ERR_INVALID_ARG;
  pack_e4m3_kernel<<<(n4 + 255) / 256, 256, 0, stream>>>(x, static_cast<uint32_t*>(y), n4);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BLOCKS_OK : fail(e, "pack_e4m3_kernel launch");
}

int blocks_status_sync(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(e, "cudaStreamSynchronize");
  unsigned int st = 0, zero = 0;
  e = cudaMemcpyFromSymbolAsync(&st, g_blk_status, 4, 0, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return fail(e, "read status");
  e = cudaMemcpyToSymbolAsync(g_blk_status, &zero, 4, 0, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return fail(e, "clear status");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(e, "cudaStreamSynchronize");
  return st ? BLOCKS_ERR_TIMEOUT : BLOCKS_OK;
}

}  // extern "C"
