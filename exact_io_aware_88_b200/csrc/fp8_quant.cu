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

// Work split of passes 1 and 2a: CTA = (tensor, b, h, slice of kRowsPerCta tokens); its 8
// warps take kUnroll rows at a time so that several row loads are in flight per warp.
constexpr int kRowsPerCta = 512;
constexpr int kUnroll = 4;

struct Slice {
  int t, b, h, n0, n1;
};
__device__ __forceinline__ Slice slice_of(const Args& a, int block) {
  const int per_head = (a.N + kRowsPerCta - 1) / kRowsPerCta;
  Slice s;
  const int hs = block / per_head;  // (t, b, h) flattened
  s.n0 = (block % per_head) * kRowsPerCta;
  s.n1 = min(a.N, s.n0 + kRowsPerCta);
  s.t = hs / (a.B * a.H);
  s.b = (hs / a.H) % a.B;
  s.h = hs % a.H;
  return s;
}
__device__ __forceinline__ const __nv_bfloat16* src_of(const Args& a, int t) {
  return t == 0 ? a.src_q : t == 1 ? a.src_k : a.src_v;
}

// Pass 1: per-head max |x| of the transformed Q, K and of V.
template <int D>
__global__ void __launch_bounds__(kThreads) amax_kernel(Args a) {
  constexpr int E = D / 32;
  __shared__ float red[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const Slice s = slice_of(a, blockIdx.x);
  const __nv_bfloat16* base = src_of(a, s.t) + (static_cast<size_t>(s.b) * a.N * a.H + s.h) * D;
  const size_t row_stride = static_cast<size_t>(a.H) * D;
  const bool xf = s.t < 2 && a.signs;
  float m = 0.f;
  for (int n = s.n0 + warp * kUnroll; n < s.n1; n += (kThreads / 32) * kUnroll) {
    float x[kUnroll][E];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (n + u < s.n1) load_row<E>(base + (n + u) * row_stride, lane, x[u]);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (n + u >= s.n1) break;
      if (xf) hadamard_row<E>(x[u], a.signs, lane, a.inv_sqrt_d);
#pragma unroll
      for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(x[u][e]));
    }
  }
  m = warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < kThreads / 32 ? red[lane] : 0.f;
    m = warp_max(m);
    if (lane == 0)
      atomicMax(a.amax + s.t * a.B * a.H + s.b * a.H + s.h, __float_as_uint(m));
  }
}

// Pass 2a: Q and K codes (CTAs as in pass 1, tensors 0 and 1); CTA 0 also publishes the
// scales of all three tensors.
template <int D>
__global__ void __launch_bounds__(kThreads) quant_qk_kernel(Args a) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < 3 * a.B * a.H; i += kThreads)
      a.scales[i] = exp2i(scale_exp(__uint_as_float(a.amax[i])));
  const Slice s = slice_of(a, blockIdx.x);
  const size_t head_off = (static_cast<size_t>(s.b) * a.N * a.H + s.h) * D;
  const __nv_bfloat16* base = src_of(a, s.t) + head_off;
  uint8_t* obase = (s.t == 0 ? a.dst_q : a.dst_k) + head_off + lane * E;
  const size_t row_stride = static_cast<size_t>(a.H) * D;
  const float inv = exp2i(-scale_exp(__uint_as_float(a.amax[s.t * a.B * a.H + s.b * a.H + s.h])));
  for (int n = s.n0 + warp * kUnroll; n < s.n1; n += (kThreads / 32) * kUnroll) {
    float x[kUnroll][E];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (n + u < s.n1) load_row<E>(base + (n + u) * row_stride, lane, x[u]);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (n + u >= s.n1) break;
      if (a.signs) hadamard_row<E>(x[u], a.signs, lane, a.inv_sqrt_d);
      uint8_t* out = obase + (n + u) * row_stride;
      if constexpr (E == 4) {
        const uint32_t lo = pack_e4m3x2(x[u][0] * inv, x[u][1] * inv);
        const uint32_t hi = pack_e4m3x2(x[u][2] * inv, x[u][3] * inv);
        *reinterpret_cast<uint32_t*>(out) = lo | (hi << 16);
      } else {
        *reinterpret_cast<uint16_t*>(out) = static_cast<uint16_t>(pack_e4m3x2(x[u][0] * inv, x[u][1] * inv));
      }
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
  const long long per_head = (p.N + kRowsPerCta - 1) / kRowsPerCta;
  const long long heads = static_cast<long long>(p.B) * p.H;
  if (3 * heads * per_head > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  amax_kernel<D><<<static_cast<int>(3 * heads * per_head), kThreads, 0, st>>>(a);
  quant_qk_kernel<D><<<static_cast<int>(2 * heads * per_head), kThreads, 0, st>>>(a);
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
