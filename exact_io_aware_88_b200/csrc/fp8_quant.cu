// fp8_quant.cu -- operand preparation for the FP8 forward pass: incoherent processing of
// Q and K (a random-sign Hadamard transform), one power-of-two scale per head and tensor,
// and E4M3 quantisation; V is quantised without the transform and stored transposed
// ([B][H][d][Npad], keys contiguous) so that it is K-major for the second product.
//
// The transform is the one of "FlashAttention-3 — FlashAttention-3" (section
// FlashAttention-3の技術的革新, item 3): rows of Q and K are multiplied by an orthogonal
// matrix, here M = diag(s) H_d / sqrt(d) with H_d the Sylvester Hadamard matrix, so that
// (Q M)(K M)^T = Q K^T and rare large entries are spread over all coordinates before the
// 8-bit rounding.  It is applied as a fast Walsh-Hadamard transform: one warp per row,
// d/32 elements per lane, log2(d/32) butterfly stages inside a lane and 5 across lanes.
//
// Two passes, both HBM-bound: (1) the transformed rows' max |x| per (batch, head, tensor)
// into a workspace (atomicMax on the float bits, valid for non-negative floats); (2) the
// scale 2^e, smallest with 448 * 2^e >= amax, and the E4M3 codes of x / 2^e (the division
// is exact), rounded to nearest even with saturation by cvt.rn.satfinite.e4m3x2.f32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "launch.h"
#include "ptx.cuh"

namespace fa {
namespace fp8q {

constexpr int kThreads = 256;

// The two bf16 values of a 32-bit word (low half first), widened exactly.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int E>  // elements per lane (d / 32)
__device__ __forceinline__ void load_row(const __nv_bfloat16* __restrict__ row, int lane,
                                         float (&x)[E]) {
  if constexpr (E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + lane * 4);
    x[0] = bf16_lo(u.x);
    x[1] = bf16_hi(u.x);
    x[2] = bf16_lo(u.y);
    x[3] = bf16_hi(u.y);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(row + lane * 2);
    x[0] = bf16_lo(u);
    x[1] = bf16_hi(u);
  }
}

// x <- (x * signs) H_d / sqrt(d) for the row spread over the warp (element lane*E + e).
template <int E>
__device__ __forceinline__ void hadamard_row(float (&x)[E], const float* __restrict__ signs,
                                             int lane, float inv_sqrt_d) {
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] *= signs[lane * E + e];
  // Index bits inside the lane.
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (e & h) continue;
      const float a = x[e], b = x[e + h];
      x[e] = a + b;
      x[e + h] = a - b;
    }
  }
  // Index bits across lanes: the element whose bit is 0 keeps a + b, the other a - b.
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = upper ? (o - x[e]) : (x[e] + o);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] *= inv_sqrt_d;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// Exponent e of the scale 2^e: the smallest e with 448 * 2^e >= amax (448 = 1.75 * 2^8),
// clamped to the normal fp32 range; 0 for amax = 0.
__device__ __forceinline__ int scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  const uint32_t bits = __float_as_uint(amax);
  const int E = static_cast<int>((bits >> 23) & 0xFF) - 127;
  const uint32_t mant = bits & 0x7FFFFFu;
  int e = (E == -127) ? -126 - 8 : (mant <= 0x600000u ? E - 8 : E - 7);
  return max(-126, min(127, e));
}
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

struct Args {
  const __nv_bfloat16 *src_q, *src_k, *src_v;
  uint8_t *dst_q, *dst_k;
  uint8_t* vt;
  const float* signs;  // nullptr: no transform
  float* scales;       // [3][B*H]
  uint32_t* amax;      // [3][B*H] float bits, zeroed before pass 1
  int B, H, N, npad;
  float inv_sqrt_d;
};

// Pass 1: one warp per (tensor, b, n, h) row.
template <int D>
__global__ void __launch_bounds__(kThreads) amax_kernel(Args a) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.B) * a.N * a.H;
  const long long warps = static_cast<long long>(gridDim.x) * (kThreads / 32);
  for (long long w = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); w < 3 * rows; w += warps) {
    const int t = static_cast<int>(w / rows);
    const long long r = w % rows;  // (b, n, h) row-major
    const int h = static_cast<int>(r % a.H);
    const int b = static_cast<int>(r / (static_cast<long long>(a.N) * a.H));
    float x[E];
    load_row<E>((t == 0 ? a.src_q : t == 1 ? a.src_k : a.src_v) + r * D, lane, x);
    if (t < 2 && a.signs) hadamard_row<E>(x, a.signs, lane, a.inv_sqrt_d);
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(x[e]));
    m = warp_max(m);
    if (lane == 0) atomicMax(a.amax + t * a.B * a.H + b * a.H + h, __float_as_uint(m));
  }
}

// Pass 2a: Q and K codes, one warp per row; the first 3*B*H threads also publish the scales.
template <int D>
__global__ void __launch_bounds__(kThreads) quant_qk_kernel(Args a) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long gtid = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x;
  if (gtid < 3LL * a.B * a.H)
    a.scales[gtid] = exp2i(scale_exp(__uint_as_float(a.amax[gtid])));
  const long long rows = static_cast<long long>(a.B) * a.N * a.H;
  const long long warps = static_cast<long long>(gridDim.x) * (kThreads / 32);
  for (long long w = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); w < 2 * rows; w += warps) {
    const int t = static_cast<int>(w / rows);
    const long long r = w % rows;
    const int h = static_cast<int>(r % a.H);
    const int b = static_cast<int>(r / (static_cast<long long>(a.N) * a.H));
    float x[E];
    load_row<E>((t == 0 ? a.src_q : a.src_k) + r * D, lane, x);
    if (a.signs) hadamard_row<E>(x, a.signs, lane, a.inv_sqrt_d);
    const float inv = exp2i(-scale_exp(__uint_as_float(a.amax[t * a.B * a.H + b * a.H + h])));
    uint8_t* out = (t == 0 ? a.dst_q : a.dst_k) + r * D + lane * E;
    if constexpr (E == 4) {
      const uint32_t lo = pack_e4m3x2(x[0] * inv, x[1] * inv), hi = pack_e4m3x2(x[2] * inv, x[3] * inv);
      *reinterpret_cast<uint32_t*>(out) = lo | (hi << 16);
    } else {
      *reinterpret_cast<uint16_t*>(out) = pack_e4m3x2(x[0] * inv, x[1] * inv);
    }
  }
}

// Pass 2b: V codes, transposed.  CTA = (b, h, 128-key block): 128 x D codes through shared
// memory, written as D rows of up to 128 contiguous keys.  Keys in [N, Npad) are zero.
template <int D>
__global__ void __launch_bounds__(kThreads) quant_vt_kernel(Args a) {
  __shared__ uint8_t tile[D][128 + 4];
  const int nblk = (a.npad + 127) / 128;
  const int blk = blockIdx.x % nblk;
  const int bh = blockIdx.x / nblk;
  const int b = bh / a.H, h = bh % a.H;
  const int n0 = blk * 128;
  const float inv = exp2i(-scale_exp(__uint_as_float(a.amax[2 * a.B * a.H + bh])));
  // Load: thread handles (key, 8-element group); D/8 groups per key.
  for (int i = threadIdx.x; i < 128 * (D / 8); i += kThreads) {
    const int key = i / (D / 8), g = i % (D / 8);
    const int n = n0 + key;
    uint32_t c[4] = {0u, 0u, 0u, 0u};
    if (n < a.N) {
      const uint4 u = *reinterpret_cast<const uint4*>(
          a.src_v + ((static_cast<size_t>(b) * a.N + n) * a.H + h) * D + g * 8);
      c[0] = pack_e4m3x2(bf16_lo(u.x) * inv, bf16_hi(u.x) * inv);
      c[1] = pack_e4m3x2(bf16_lo(u.y) * inv, bf16_hi(u.y) * inv);
      c[2] = pack_e4m3x2(bf16_lo(u.z) * inv, bf16_hi(u.z) * inv);
      c[3] = pack_e4m3x2(bf16_lo(u.w) * inv, bf16_hi(u.w) * inv);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      tile[g * 8 + 2 * j][key] = static_cast<uint8_t>(c[j] & 0xFF);
      tile[g * 8 + 2 * j + 1][key] = static_cast<uint8_t>(c[j] >> 8);
    }
  }
  __syncthreads();
  // Store: D rows x 128 keys, 4 bytes per thread.
  const int nkeys = min(128, a.npad - n0);  // a multiple of 16
  for (int i = threadIdx.x; i < D * 32; i += kThreads) {
    const int row = i / 32, q4 = i % 32;
    if (q4 * 4 >= nkeys) continue;
    const uint32_t v = tile[row][q4 * 4] | (tile[row][q4 * 4 + 1] << 8) |
                       (tile[row][q4 * 4 + 2] << 16) | (static_cast<uint32_t>(tile[row][q4 * 4 + 3]) << 24);
    *reinterpret_cast<uint32_t*>(a.vt + ((static_cast<size_t>(b) * a.H + h) * D + row) * a.npad +
                                 n0 + q4 * 4) = v;
  }
}

template <int D>
static cudaError_t launch_t(const Fp8QuantArgs& p, cudaStream_t st) {
  Args a;
  a.src_q = static_cast<const __nv_bfloat16*>(p.q);
  a.src_k = static_cast<const __nv_bfloat16*>(p.k);
  a.src_v = static_cast<const __nv_bfloat16*>(p.v);
  a.dst_q = static_cast<uint8_t*>(p.q8);
  a.dst_k = static_cast<uint8_t*>(p.k8);
  a.vt = static_cast<uint8_t*>(p.vt8);
  a.signs = p.signs;
  a.scales = p.scales;
  a.amax = p.amax;
  a.B = p.B;
  a.H = p.H;
  a.N = p.N;
  a.npad = (p.N + 15) / 16 * 16;
  a.inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
  cudaError_t e = cudaMemsetAsync(p.amax, 0, 3 * sizeof(uint32_t) * p.B * p.H, st);
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(p.B) * p.N * p.H;
  const int grid_rows = static_cast<int>(std::min<long long>((3 * rows + 7) / 8, 148LL * 16));
  amax_kernel<D><<<grid_rows, kThreads, 0, st>>>(a);
  const long long need_scale_blocks = (3LL * p.B * p.H + kThreads - 1) / kThreads;
  const int grid_q = static_cast<int>(
      std::max<long long>(need_scale_blocks, std::min<long long>((2 * rows + 7) / 8, 148LL * 16)));
  quant_qk_kernel<D><<<grid_q, kThreads, 0, st>>>(a);
  const long long grid_v = static_cast<long long>(p.B) * p.H * ((a.npad + 127) / 128);
  if (grid_v > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  quant_vt_kernel<D><<<static_cast<int>(grid_v), kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace fp8q

cudaError_t launch_fp8_quantize(const Fp8QuantArgs& p, cudaStream_t s) {
  return p.d == 64 ? fp8q::launch_t<64>(p, s) : fp8q::launch_t<128>(p, s);
}

}  // namespace fa
