// debug.cu -- single-tile self-tests of the sm_100a primitives (fa_debug.h):
//   * one 128 x n x k tcgen05.mma tile with operands written to shared memory in the
//     128-byte-swizzled layouts the attention kernels use (K-major and MN-major), or with A
//     staged in tensor memory as packed bf16 pairs;
//   * one TMA box load through the kernels' tensor-map encoding, read back unswizzled;
//   * a tensor-memory store / load round trip;
//   * a bounded mbarrier wait that is made to run out, to exercise the timeout path.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"
#include "ptx.cuh"

namespace fa {
namespace dbg {

// Writes a [rows][cols] bf16 row-major global matrix into shared memory as 64-column
// chunks of [rows][128 B], 128-byte swizzled (the layout TMA produces with SWIZZLE_128B).
__device__ void stage_sw128(uint8_t* dst, const __nv_bfloat16* src, int rows, int cols) {
  const int chunks16 = cols / 8;  // 16-byte pieces per row
  for (int idx = threadIdx.x; idx < rows * chunks16; idx += blockDim.x) {
    const int r = idx / chunks16, c16 = idx % chunks16;
    const int blk = c16 / 8, cin = c16 % 8;
    const uint4 val = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * cols + c16 * 8);
    *reinterpret_cast<uint4*>(dst + blk * rows * 128 + sw128_offset(r, cin)) = val;
  }
}

__global__ void __launch_bounds__(128, 1)
    umma_tile_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ Bm,
                     float* __restrict__ Cm, int n, int k, int mode, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                 // 128 x k bf16   (<= 32 KB)
  uint8_t* sB = smem + 32768;         // n x k or k x n (<= 32 KB)
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 65536);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + 65536 + 64);
  Abort* ab = reinterpret_cast<Abort*>(smem + 65536 + 128);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    ab->flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  // Operands into shared memory (A also into TMEM for mode 1).
  stage_sw128(sA, A, 128, k);
  if (mode == 0)
    stage_sw128(sB, Bm, n, k);  // [n][k], K contiguous
  else
    stage_sw128(sB, Bm, k, n);  // [k][n], N contiguous
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t lane_base = tbase + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t colA = 128;  // A (mode 1) at columns [128, 128 + k/2)

  if (mode == 1) {
    const int r = threadIdx.x;
    for (int c0 = 0; c0 < k / 2; c0 += 16) {
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int e = 2 * (c0 + i);
        pk[i] = pack_bf16x2(__bfloat162float(A[r * k + e]), __bfloat162float(A[r * k + e + 1]));
      }
      tmem_st16(lane_base + colA + c0, pk);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (threadIdx.x == 0) {
    const uint32_t aA = smem_u32(sA), aB = smem_u32(sB);
    const uint32_t idesc = idesc_bf16_f32(128, n, 0, mode == 0 ? 0 : 1);
    for (int kk = 0; kk < k / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;  // K-major A
      const uint32_t acc = kk > 0 ? 1u : 0u;
      if (mode == 0) {
        const uint32_t boff = (kk >> 2) * (n * 128) + (kk & 3) * 32;
        umma_ss(tbase, sdesc_sw128(aA + koff, 16, 1024), sdesc_sw128(aB + boff, 16, 1024), idesc,
                acc);
      } else {
        // MN-major B: K index = row of 128 B; 64-wide N blocks are k*128 bytes apart.
        const uint64_t bdesc = sdesc_sw128(aB + kk * 2048, k * 128, 1024);
        if (mode == 1)
          umma_ts(tbase, tbase + colA + kk * 8, bdesc, idesc, acc);
        else
          umma_ss(tbase, sdesc_sw128(aA + koff, 16, 1024), bdesc, idesc, acc);
      }
    }
    umma_commit(bar);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, ab, status, kDefaultWaitTimeoutNs));
  tc_fence_after();
  if (ok) {
    const int r = threadIdx.x;
    for (int c0 = 0; c0 < n; c0 += 32) {
      uint32_t u[32];
      tmem_ld32(lane_base + c0, u);
#pragma unroll
      for (int i = 0; i < 32; ++i) Cm[r * n + c0 + i] = __uint_as_float(u[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(tbase, 256);
  }
}

// One 128-row x 64-element bf16 box of a [B][N][H][d] tensor through TMA (128-byte swizzle,
// the attention kernels' encoding), copied out row-major (unswizzled) into y[128][64].
__global__ void __launch_bounds__(128, 1)
    tma_tile_kernel(const __grid_constant__ CUtensorMap tm, __nv_bfloat16* __restrict__ y, int b,
                    int h, int row0, int chunk, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tile = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(tile + 16384);
  Abort* ab = reinterpret_cast<Abort*>(tile + 16384 + 64);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    ab->flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, 16384);
    tma_load_4d(tile, &tm, bar, chunk * 64, h, row0, b, policy_evict_first());
  }
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, ab, status, kDefaultWaitTimeoutNs));
  if (ok) {
    const int r = threadIdx.x;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      reinterpret_cast<uint4*>(y + r * 64)[c] =
          *reinterpret_cast<const uint4*>(tile + sw128_offset(r, c));
  }
}

// Lane r writes in[r][0..ncols) into tensor-memory columns [0, ncols) with tcgen05.st and
// reads them back with tcgen05.ld into out[r][0..ncols).
__global__ void __launch_bounds__(128, 1)
    tmem_roundtrip_kernel(const uint32_t* __restrict__ in, uint32_t* __restrict__ out, int ncols) {
  __shared__ uint32_t tslot;
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    tmem_alloc(&tslot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t lane_base = tslot + (static_cast<uint32_t>(warp * 32) << 16);
  const int r = threadIdx.x;
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = in[r * ncols + c0 + i];
    tmem_st32(lane_base + c0, v);
  }
  tmem_st_wait();
  for (int c0 = 0; c0 < ncols; c0 += 64) {
    if (c0 + 64 <= ncols) {
      uint32_t v[64];
      tmem_ld64(lane_base + c0, v);
#pragma unroll
      for (int i = 0; i < 64; ++i) out[r * ncols + c0 + i] = v[i];
    } else {
      uint32_t v[32];
      tmem_ld32(lane_base + c0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) out[r * ncols + c0 + i] = v[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(tslot, 256);
  }
}

__global__ void wait_timeout_kernel(uint64_t timeout_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ Abort ab;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    ab.flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must give up on its own.
  mbar_wait(&bar, 0, &ab, status, timeout_ns);
}

// y_poly[i] = software exp2 (exp2_poly2), y_hw[i] = hardware ex2.approx, of x[i].
__global__ void exp2_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                            float* __restrict__ y_hw, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  float p0, p1;
  f2_unpack(exp2_poly2(f2_pack(a, b)), p0, p1);
  y_poly[i] = p0;
  y_hw[i] = ex2_approx(a);
  if (i + 1 < n) {
    y_poly[i + 1] = p1;
    y_hw[i + 1] = ex2_approx(b);
  }
}

}  // namespace dbg

cudaError_t launch_debug_exp2(const float* x, float* y_poly, float* y_hw, int n, cudaStream_t s) {
  const int pairs = (n + 1) / 2;
  dbg::exp2_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(x, y_poly, y_hw, n);
  return cudaGetLastError();
}

cudaError_t launch_debug_umma(const void* a, const void* b, float* c, int n, int k, int mode,
                              int* status, cudaStream_t s) {
  const int smem = 65536 + 256 + 1024;
  cudaError_t e = cudaFuncSetAttribute(dbg::umma_tile_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dbg::umma_tile_kernel<<<1, 128, smem, s>>>(static_cast<const __nv_bfloat16*>(a),
                                             static_cast<const __nv_bfloat16*>(b), c, n, k, mode,
                                             status);
  return cudaGetLastError();
}

cudaError_t launch_debug_tma_tile(const CUtensorMap& tm, void* y, int b, int h, int row0,
                                  int chunk, int* status, cudaStream_t s) {
  const int smem = 16384 + 256 + 1024;
  cudaError_t e = cudaFuncSetAttribute(dbg::tma_tile_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dbg::tma_tile_kernel<<<1, 128, smem, s>>>(tm, static_cast<__nv_bfloat16*>(y), b, h, row0,
                                            chunk, status);
  return cudaGetLastError();
}

cudaError_t launch_debug_tmem_roundtrip(const uint32_t* in, uint32_t* out, int ncols,
                                        cudaStream_t s) {
  dbg::tmem_roundtrip_kernel<<<1, 128, 0, s>>>(in, out, ncols);
  return cudaGetLastError();
}

cudaError_t launch_debug_wait_timeout(uint64_t timeout_ns, int* status, cudaStream_t s) {
  dbg::wait_timeout_kernel<<<1, 32, 0, s>>>(timeout_ns, status);
  return cudaGetLastError();
}

}  // namespace fa
