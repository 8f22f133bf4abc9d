// fp8_quant.cu -- operand preparation for the FP8 forward pass: incoherent processing of
// Q and K (a random-sign Hadamard transform), one power-of-two scale per head and tensor,
// and E4M3 quantisation; V is quantised without the transform and stored transposed
// ([B][H][d][Npad], keys contiguous) so that it is K-major for the second product.
//
// The transform is the one of "FlashAttention-3 — FlashAttention-3" (section
// FlashAttention-3の技術的革新, item 3): rows of Q and K are multiplied by an orthogonal
// matrix, here M = diag(s) H_d / sqrt(d) with H_d the Sylvester Hadamard matrix, so that
// (Q M)(K M)^T = Q K^T and rare large entries are spread over all coordinates before the
// 8-bit rounding.  It is applied as a fast Walsh-Hadamard transform: four lanes per row, d/4
// elements per lane, log2(d/4) butterfly stages inside a lane and 2 across lanes.
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
// Resident blocks per SM the two row passes are compiled for (register cap 128 at d=128, 64
// at d=64, where the rows fit without spills): fewer blocks leave too few loads in flight per
// SM to cover DRAM latency (d=64 with three blocks: 0.147 vs 0.140 ms at B=1, N=16k, H=32).
template <int D>
constexpr int kMinBlocks = D == 128 ? 2 : 4;

// The two bf16 values of a 32-bit word (low half first), widened exactly.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Row layout of passes 1 and 2a: four lanes per row, eight rows per warp (lane = 4 rl + l).
// Lane l holds the row's 16-byte pieces p = 4c + l (c < D/32), i.e. elements 32c + 8l + k
// (k < 8), kept at local index e = 8c + k.  The four lanes of a row then load and store
// contiguous 64-byte runs, and of the transform's log2(d) butterfly stages only the two over
// index bits 3 and 4 (which lane) need shuffles; the other stages are in-lane adds.
template <int D>
struct Quad {
  static constexpr int E = D / 4;  // elements per lane
  static constexpr int P = E / 8;  // 16-byte pieces per lane
};

// The lane's pieces of one row as raw bf16 words (loads only), and their widening to fp32.
// Split so that a warp can have the next rows' loads in flight while it transforms these.
template <int D>
__device__ __forceinline__ void fetch_quad(const __nv_bfloat16* __restrict__ row, int l,
                                           uint4 (&r)[Quad<D>::P]) {
#pragma unroll
  for (int c = 0; c < Quad<D>::P; ++c) r[c] = *reinterpret_cast<const uint4*>(row + 8 * (4 * c + l));
}
template <int D>
__device__ __forceinline__ void widen_quad(const uint4 (&r)[Quad<D>::P], float (&x)[Quad<D>::E]) {
#pragma unroll
  for (int c = 0; c < Quad<D>::P; ++c) {
    x[8 * c + 0] = bf16_lo(r[c].x);
    x[8 * c + 1] = bf16_hi(r[c].x);
    x[8 * c + 2] = bf16_lo(r[c].y);
    x[8 * c + 3] = bf16_hi(r[c].y);
    x[8 * c + 4] = bf16_lo(r[c].z);
    x[8 * c + 5] = bf16_hi(r[c].z);
    x[8 * c + 6] = bf16_lo(r[c].w);
    x[8 * c + 7] = bf16_hi(r[c].w);
  }
}

// Bit e set iff the sign applied to local element e of quarter l is negative.
template <int D>
__device__ __forceinline__ uint32_t quad_sign_mask(const float* __restrict__ signs, int l) {
  uint32_t m = 0u;
#pragma unroll
  for (int c = 0; c < Quad<D>::P; ++c)
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (signs[32 * c + 8 * l + k] < 0.f) m |= 1u << (8 * c + k);
  return m;
}

// x <- (x * signs) H_d / sqrt(d) for the row held by the lane's quad.  Local index bits 0-2
// are global bits 0-2 and local bits 3-4 are global bits 5-6 (in-lane butterflies); global
// bits 3-4 are the quarter l (shuffles with lanes l ^ 1 and l ^ 2).  The stages commute, so
// their order does not change the transform.  Arithmetic is done two elements at a time on
// packed pairs wherever the pairing allows (every element still gets one IEEE operation per
// stage, rounded as the scalar one would be): the butterflies 2 or more apart as one packed
// add and one packed subtract per two butterflies, the cross-lane stages as
// fma(x, +-1, partner) (x + partner in the lower lane, partner - x in the upper one), and the
// final multiply by 1/sqrt(d).  Measured: 0.138 vs 0.144 ms for a d=128 call at B=4, N=4k,
// H=16, but 0.162 vs 0.148 ms at d=64 (16 elements per lane), which keeps the scalar stages.
template <int D>
__device__ __forceinline__ void hadamard_quad(float (&x)[Quad<D>::E], uint32_t smask, int lane,
                                              float inv_sqrt_d) {
  constexpr int E = Quad<D>::E;
#pragma unroll
  for (int e = 0; e < E; ++e)
    x[e] = __uint_as_float(__float_as_uint(x[e]) ^ (((smask >> e) & 1u) << 31));
  if constexpr (D != 128) {
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
#pragma unroll
    for (int m = 1; m < 4; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float o = __shfl_xor_sync(0xffffffffu, x[e], m);
        x[e] = upper ? (o - x[e]) : (x[e] + o);
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] *= inv_sqrt_d;
    return;
  }
#pragma unroll
  for (int e = 0; e < E; e += 2) {  // butterflies 1 apart: inside a pair
    const float a = x[e], b = x[e + 1];
    x[e] = a + b;
    x[e + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      if (e & h) continue;
      const uint64_t p = f2_pack(x[e], x[e + 1]), q = f2_pack(x[e + h], x[e + h + 1]);
      f2_unpack(f2_add(p, q), x[e], x[e + 1]);
      f2_unpack(f2_sub(p, q), x[e + h], x[e + h + 1]);
    }
  }
#pragma unroll
  for (int m = 1; m < 4; m <<= 1) {
    const float sg = (lane & m) ? -1.f : 1.f;
    const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float o0 = __shfl_xor_sync(0xffffffffu, x[e], m);
      const float o1 = __shfl_xor_sync(0xffffffffu, x[e + 1], m);
      f2_unpack(f2_fma(f2_pack(x[e], x[e + 1]), sg2, f2_pack(o0, o1)), x[e], x[e + 1]);
    }
  }
  const uint64_t s2 = f2_pack(inv_sqrt_d, inv_sqrt_d);
#pragma unroll
  for (int e = 0; e < E; e += 2) f2_unpack(f2_mul(f2_pack(x[e], x[e + 1]), s2), x[e], x[e + 1]);
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
// warps take kUnroll groups of 8 rows at a time, and the loads of a warp's next groups are
// issued before it transforms the current ones, so that DRAM reads never stop while the
// warp computes.
constexpr int kRowsPerCta = 512;
constexpr int kUnroll = 1;  // groups of 8 rows per step of a warp (two: 171 registers at d=128)
constexpr int kRowStep = (kThreads / 32) * 8 * kUnroll;  // rows a CTA takes per step

// The raw words of a warp's kUnroll groups starting at row n (rows past n1 read as zeros).
template <int D>
__device__ __forceinline__ void fetch_groups(const __nv_bfloat16* __restrict__ base,
                                             size_t row_stride, int n, int n1, int rl, int l,
                                             uint4 (&r)[kUnroll][Quad<D>::P]) {
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int row = n + 8 * u + rl;
    if (row < n1) {
      fetch_quad<D>(base + row * row_stride, l, r[u]);
    } else {
#pragma unroll
      for (int c = 0; c < Quad<D>::P; ++c) r[u][c] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

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
__global__ void __launch_bounds__(kThreads, kMinBlocks<D>) amax_kernel(Args a) {
  constexpr int E = Quad<D>::E;
  __shared__ float red[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rl = lane >> 2, l = lane & 3;
  const Slice s = slice_of(a, blockIdx.x);
  const __nv_bfloat16* base = src_of(a, s.t) + (static_cast<size_t>(s.b) * a.N * a.H + s.h) * D;
  const size_t row_stride = static_cast<size_t>(a.H) * D;
  const bool xf = s.t < 2 && a.signs;
  const uint32_t smask = xf ? quad_sign_mask<D>(a.signs, l) : 0u;
  float m = 0.f;
  uint4 raw[kUnroll][Quad<D>::P];
  int n = s.n0 + warp * 8 * kUnroll;
  if (n < s.n1) fetch_groups<D>(base, row_stride, n, s.n1, rl, l, raw);
  for (; n < s.n1; n += kRowStep) {
    float x[kUnroll][E];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) widen_quad<D>(raw[u], x[u]);
    if (n + kRowStep < s.n1) fetch_groups<D>(base, row_stride, n + kRowStep, s.n1, rl, l, raw);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (xf) hadamard_quad<D>(x[u], smask, lane, a.inv_sqrt_d);
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
__global__ void __launch_bounds__(kThreads, kMinBlocks<D>) quant_qk_kernel(Args a) {
  constexpr int E = Quad<D>::E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rl = lane >> 2, l = lane & 3;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < 3 * a.B * a.H; i += kThreads)
      a.scales[i] = exp2i(scale_exp(__uint_as_float(a.amax[i])));
  const Slice s = slice_of(a, blockIdx.x);
  const size_t head_off = (static_cast<size_t>(s.b) * a.N * a.H + s.h) * D;
  const __nv_bfloat16* base = src_of(a, s.t) + head_off;
  uint8_t* obase = (s.t == 0 ? a.dst_q : a.dst_k) + head_off;
  const size_t row_stride = static_cast<size_t>(a.H) * D;
  const float inv = exp2i(-scale_exp(__uint_as_float(a.amax[s.t * a.B * a.H + s.b * a.H + s.h])));
  const uint32_t smask = a.signs ? quad_sign_mask<D>(a.signs, l) : 0u;
  uint4 raw[kUnroll][Quad<D>::P];
  int n = s.n0 + warp * 8 * kUnroll;
  if (n < s.n1) fetch_groups<D>(base, row_stride, n, s.n1, rl, l, raw);
  for (; n < s.n1; n += kRowStep) {
    float x[kUnroll][E];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) widen_quad<D>(raw[u], x[u]);
    if (n + kRowStep < s.n1) fetch_groups<D>(base, row_stride, n + kRowStep, s.n1, rl, l, raw);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (a.signs) hadamard_quad<D>(x[u], smask, lane, a.inv_sqrt_d);
      const int row = n + 8 * u + rl;
      if (row >= s.n1) continue;
      uint8_t* out = obase + row * row_stride;
#pragma unroll
      for (int c = 0; c < Quad<D>::P; ++c) {
        const float* v = &x[u][8 * c];
        const uint32_t w0 = pack_e4m3x2(v[0] * inv, v[1] * inv) | (pack_e4m3x2(v[2] * inv, v[3] * inv) << 16);
        const uint32_t w1 = pack_e4m3x2(v[4] * inv, v[5] * inv) | (pack_e4m3x2(v[6] * inv, v[7] * inv) << 16);
        *reinterpret_cast<uint2*>(out + 8 * (4 * c + l)) = make_uint2(w0, w1);
      }
    }
  }
}

// Pass 2b: V codes, transposed.  CTA = (b, h, 128-key block): 128 x D codes through shared
// memory, written as D rows of up to 128 contiguous keys.  Keys in [N, Npad) are zero.
// A work item is (4 consecutive keys, 8 consecutive head-dim elements): four 16-byte loads
// (the lanes of a warp cover whole key rows, so the loads are coalesced), and per element one
// 32-bit word holding its four keys' codes.  The tile holds words: row = head-dim element,
// 32 words = 128 keys, and word w of row r sits at column w ^ (g * 32 / G) for element group
// g = r / 8 (G groups per key), so that a warp's column writes (16 or 8 element groups x 2 or
// 4 key quads) and its row reads both touch 32 different banks.
template <int D>
__global__ void __launch_bounds__(kThreads) quant_vt_kernel(Args a) {
  constexpr int G = D / 8;                       // 8-element groups per key
  constexpr int kItems = 32 * G / kThreads;      // work items per thread: 2 (d=128) or 1
  constexpr int kSwz = 32 / G;                   // column XOR step per element group
  __shared__ uint32_t tile[D][32];
  const int nblk = (a.npad + 127) / 128;
  const int blk = blockIdx.x % nblk;
  const int bh = blockIdx.x / nblk;
  const int b = bh / a.H, h = bh % a.H;
  const int n0 = blk * 128;
  const float inv = exp2i(-scale_exp(__uint_as_float(a.amax[2 * a.B * a.H + bh])));
  const __nv_bfloat16* src = a.src_v + (static_cast<size_t>(b) * a.N * a.H + h) * D;
  const size_t row_stride = static_cast<size_t>(a.H) * D;
  uint4 u[kItems][4];
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int i = threadIdx.x + it * kThreads;
    const int g = i % G, kq = i / G;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int n = n0 + 4 * kq + kk;
      u[it][kk] = n < a.N ? *reinterpret_cast<const uint4*>(src + n * row_stride + 8 * g)
                          : make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int i = threadIdx.x + it * kThreads;
    const int g = i % G, kq = i / G;
    const int col = kq ^ (g * kSwz);
#pragma unroll
    for (int m = 0; m < 4; ++m) {  // elements 8g + 2m, 8g + 2m + 1
      uint32_t c[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t w = m == 0 ? u[it][kk].x : m == 1 ? u[it][kk].y : m == 2 ? u[it][kk].z : u[it][kk].w;
        c[kk] = pack_e4m3x2(bf16_lo(w) * inv, bf16_hi(w) * inv);  // (element 2m, 2m + 1)
      }
      const uint32_t x = c[0] | (c[1] << 16), y = c[2] | (c[3] << 16);
      tile[8 * g + 2 * m][col] = __byte_perm(x, y, 0x6420);      // keys 0..3, element 2m
      tile[8 * g + 2 * m + 1][col] = __byte_perm(x, y, 0x7531);  // keys 0..3, element 2m + 1
    }
  }
  __syncthreads();
  // Store: D rows x 128 keys, one word (4 keys) per thread and row.
  const int nkeys = min(128, a.npad - n0);  // a multiple of 16
  uint8_t* dst = a.vt + static_cast<size_t>(bh) * D * a.npad + n0;
#pragma unroll
  for (int i = threadIdx.x; i < D * 32; i += kThreads) {
    const int row = i / 32, w = i % 32;
    if (4 * w >= nkeys) continue;
    *reinterpret_cast<uint32_t*>(dst + static_cast<size_t>(row) * a.npad + 4 * w) =
        tile[row][w ^ ((row / 8) * kSwz)];
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
