// fwd_f32.cu -- attention forward in full fp32 on the CUDA cores (FFMA only: no tensor
// cores, no TF32), for fp32 inputs where the tensor-core path's bf16 rounding of P would be
// too coarse.  Correctness path for small fp32 problems; it is not tuned for speed.
//
// Same tiled, online-softmax evaluation as the tensor-core kernel ("FlashAttention-2を読む",
// section タイル分割でも全体の正規化を保つ): K/V tiles of 32 rows are staged in shared
// memory; each warp owns one query row and keeps its running max m, running sum l and
// partial output in registers, rescaling them whenever the max grows.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "launch.h"

namespace fa {
namespace f32 {

constexpr int kRowsPerCta = 8;  // one warp per query row
constexpr int kTileKeys = 32;   // keys per shared-memory tile: one per lane
constexpr int kMaxD = 128;

__global__ void __launch_bounds__(kRowsPerCta * 32)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                   const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse,
                   int B, int H, int N, int d, int causal, float scale) {
  __shared__ float sK[kTileKeys][kMaxD + 1];
  __shared__ float sV[kTileKeys][kMaxD];
  __shared__ float sQ[kRowsPerCta][kMaxD];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int row0 = blockIdx.x * kRowsPerCta;
  const int row = row0 + warp;
  const bool valid = row < N;
  const size_t rstride = static_cast<size_t>(H) * d;
  const size_t base = (static_cast<size_t>(b) * N) * rstride + static_cast<size_t>(h) * d;

  for (int c = lane; c < kMaxD; c += 32)
    sQ[warp][c] = (valid && c < d) ? q[base + row * rstride + c] : 0.f;

  const int last_row = min(N - 1, row0 + kRowsPerCta - 1);
  const int key_end = causal ? last_row + 1 : N;  // keys any row of this CTA can see

  float m = -INFINITY, l = 0.f;
  float acc[kMaxD / 32];
#pragma unroll
  for (int t = 0; t < kMaxD / 32; ++t) acc[t] = 0.f;

  for (int k0 = 0; k0 < key_end; k0 += kTileKeys) {
    __syncthreads();  // previous tile fully consumed (and sQ written on the first pass)
    for (int idx = threadIdx.x; idx < kTileKeys * kMaxD; idx += blockDim.x) {
      const int r = idx / kMaxD, c = idx % kMaxD;
      const int kr = k0 + r;
      const bool in = (kr < N) && (c < d);
      sK[r][c] = in ? k[base + kr * rstride + c] : 0.f;
      sV[r][c] = in ? v[base + kr * rstride + c] : 0.f;
    }
    __syncthreads();

    // Score of the key this lane owns in the tile.
    const int key = k0 + lane;
    float dot = 0.f;
    for (int c = 0; c < d; ++c) dot = fmaf(sQ[warp][c], sK[lane][c], dot);
    const bool visible = key < N && (!causal || key <= row);
    const float s = visible ? dot * scale : -INFINITY;
    float mt = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
    if (mt == -INFINITY) continue;  // nothing visible to this row in this tile
    const float m_new = fmaxf(m, mt);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float p = expf(s - m_new);
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * alpha + ps;
    m = m_new;
#pragma unroll
    for (int t = 0; t < kMaxD / 32; ++t) acc[t] *= alpha;
    for (int r = 0; r < kTileKeys; ++r) {
      const float pr = __shfl_sync(0xffffffffu, p, r);
#pragma unroll
      for (int t = 0; t < kMaxD / 32; ++t) acc[t] = fmaf(pr, sV[r][lane + 32 * t], acc[t]);
    }
  }

  if (valid) {
    const float inv_l = 1.f / l;
#pragma unroll
    for (int t = 0; t < kMaxD / 32; ++t) {
      const int c = lane + 32 * t;
      if (c < d) o[base + row * rstride + c] = acc[t] * inv_l;
    }
    if (lane == 0) lse[(static_cast<size_t>(b) * H + h) * N + row] = m + logf(l);
  }
}

}  // namespace f32

cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int B, int H, int N, int d, int causal, float scale, cudaStream_t s) {
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid((N + f32::kRowsPerCta - 1) / f32::kRowsPerCta, static_cast<unsigned>(bh));
  f32::fwd_f32_kernel<<<grid, f32::kRowsPerCta * 32, 0, s>>>(q, k, v, o, lse, B, H, N, d, causal,
                                                             scale);
  return cudaGetLastError();
}

}  // namespace fa
