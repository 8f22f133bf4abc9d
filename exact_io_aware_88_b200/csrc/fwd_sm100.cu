// fwd_sm100.cu -- attention forward on sm_100a: persistent, warp-specialised, two query
// tiles per CTA in ping-pong, TMA K/V ring, tcgen05.mma into TMEM, online softmax in base 2.
//
// The algorithm is the tiled, fused evaluation of softmax(scale*QK^T)V described in
// "Flash Attention 2で打破するローカルLLMの「メモリの壁」" (section タイリング（Tiling）と
// 再計算（Recomputation）の仕組み): query tiles stay on chip while 128-row K/V tiles stream
// past them; S and P live only in tensor memory.  The running max / sum rescaling that
// keeps the softmax globally normalised is the one of "FlashAttention-2を読む" (section
// タイル分割でも全体の正規化を保つ).  Non-matmul work is trimmed as in its first trick
// (section GPUの稼働率を高める三つの工夫): the scale is folded into one FFMA before exp2,
// masks are applied on diagonal / tail tiles only, 1/l is applied once at the end and the
// output is rescaled only when a row's running max grows by more than 2^8 (exact: the final
// normalisation uses the same, possibly stale, max).  Work is split along the sequence as
// in its second trick: the persistent grid walks (batch*head, query-tile pair) units.
//
// CTA = 12 warps (3 warpgroups):
//   warps 0-3   softmax for query tile 0 of the pair (thread t owns row t = TMEM lane t)
//   warps 4-7   softmax for query tile 1
//   warp  8     TMA producer (one lane);  warp 9: TMEM allocator + tcgen05.mma issuer
//   warps 10-11 idle
// TMEM (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 [256,384), O1 [384,512); P_t
// (bf16 pairs) overwrites the first half of S_t, O_t uses the first D columns of its slot.
//
// Tensor-core issue order per K/V tile j (after S0(0), S1(0)):
//   PV0(j), S0(j+1), PV1(j), S1(j+1)
// so each tile's softmax runs while the tensor core works on the other tile, and by the
// time softmax t sees S_t(j+1) the product PV_t(j) has completed (tcgen05 operations of
// one thread complete in order), so O_t may be rescaled in place without another wait.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "launch.h"
#include "ptx.cuh"

namespace fa {
namespace fwd {

constexpr int BM = 128;  // query rows per tile (two tiles per unit)
constexpr int BN = 128;  // key rows per tile
constexpr int kThreads = 384;
// Launch gives 65536 / 384 -> 168 registers per thread; the softmax warpgroups take
// registers from the producer / MMA warpgroup: 200 + 200 + 104 = 504 = 3 x 168 (8-bit path,
// whose softmax publishes P in two halves: 208 + 208 + 88).
constexpr uint32_t kRegsLaunch = 168;
template <bool F8>
constexpr uint32_t kRegsSoftmax = F8 ? 208 : 200;
template <bool F8>
constexpr uint32_t kRegsOther = F8 ? 88 : 104;
static_assert(2 * kRegsSoftmax<false> + kRegsOther<false> <= 3 * kRegsLaunch &&
                  2 * kRegsSoftmax<true> + kRegsOther<true> <= 3 * kRegsLaunch,
              "register split too large");
// P published in two halves of 64 keys, so that PV starts while the softmax computes the
// second half: measured +7 % on the 8-bit path, -3 to -5 % on the bf16 paths (kept off).
template <bool F8>
constexpr bool kSplitP = F8;
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Pairs out of every 8 whose exp2 runs on the FMA pipe (exp2_poly2) instead of the MUFU
// unit, on unmasked tiles.  Measured on B200: with head dim 64 (half the tensor work per
// tile) moving 2 of 8 pairs is best (+4 %; 4 of 8 is slower); head dim 128 gains nothing.
// The 8-bit path has the same tensor time per tile as head dim 64 in bf16.
template <int D, bool F8>
constexpr int kEmuPairsPer8 = (D == 64 || F8) ? 2 : 0;

// F8: Q, K and V^T are E4M3 (one byte per element); otherwise bf16.
template <int D, bool F8 = false>
struct Cfg {
  static constexpr int kElem = F8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElem;         // one head-dim row of Q or K
  static constexpr int kChunks = kRowBytes / 128;     // 128-byte column chunks
  static constexpr int kChunkElems = 128 / kElem;
  static constexpr int kChunkBytes = BM * 128;        // one TMA box: 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (kChunks == 2) ? 2 : 4;  // K/V ring depth
  static constexpr int kOffQ = 0;                     // Q0, Q1
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kBarBytes = 512;              // Bars (size checked below)
  // Block-sparse bitmasks: loader, (unused), softmax warpgroups 0 and 1 (one copy per warp).
  static constexpr int kOffMask = kOffBar + kBarBytes;
  static constexpr int kMaskBytes = (2 + 2 + 8) * 32 * 4;  // + one copy per softmax warp
  // O epilogue: one staging box per softmax warp (32 rows x 128 bytes, 128-byte swizzled),
  // written out by TMA stores.
  static constexpr int kOffStage = kOffMask + kMaskBytes;
  static constexpr int kStageBytes = 32 * 128;
  static constexpr int kSmemBytes = kOffStage + 8 * kStageBytes;  // base is 1024-aligned (checked)
  static constexpr uint32_t kColO = 256;  // O_t at kColO + 128 t
  static_assert(kOffStage % 1024 == 0, "staging boxes need 1024-byte alignment (128-byte swizzle)");
  static_assert(kSmemBytes <= 232448, "more shared memory than a CTA can have");
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[5], k_empty[5], v_full[4], v_empty[4];  // block-sparse: one more K stage
  uint64_t s_full[2], p_full[2], o_done[2], o_free[2];
  uint64_t p_half[2];  // P_t of the first 64 keys is in TMEM (and O_t rescaled)
  // Block-sparse: softmax warpgroup 1 has published its row maximum and sum (merge_ready);
  // warpgroup 0 has read them (merge_free).
  uint64_t merge_ready, merge_free;
  // End-of-CTA protocol check: [0] K/V tiles loaded, [1] units loaded, [2] K/V tiles
  // consumed by the MMA lane, [3] its units, [4 + t] softmax t's steps, [6 + t] S products
  // issued for tile t, [8 + t] softmax t's units.
  int count[10];
  uint64_t drain;
  uint32_t tmem_base;
  Abort abort;
};
static_assert(sizeof(Bars) <= Cfg<64>::kBarBytes && sizeof(Bars) <= Cfg<128>::kBarBytes,
              "barrier block larger than its shared-memory region");

// Unit schedule shared by every role.  Round r hands CTA c the unit r*G + c (even r) or
// r*G + G-1-c (odd r): a snake over the persistent grid.  Under the causal mask units are
// sorted longest first (pair index descending), so each round is a band of similar cost
// and the snake evens the per-CTA sums.
struct Unit {
  int bh, pair;
};
__device__ __forceinline__ int unit_of_round(int r, int G) {
  const int c = static_cast<int>(blockIdx.x);
  return r * G + ((r & 1) ? (G - 1 - c) : c);
}
template <bool CAUSAL>
__device__ __forceinline__ Unit decode_unit(int u, int BH, int num_pairs) {
  Unit x;
  if (CAUSAL) {
    x.pair = num_pairs - 1 - u / BH;
    x.bh = u % BH;
  } else {
    x.bh = u / num_pairs;
    x.pair = u % num_pairs;
  }
  return x;
}

// K/V tiles visible to query tile t (0 or 1) of pair p.
template <bool CAUSAL>
__device__ __forceinline__ int kv_tiles(int pair, int t, int kv_total) {
  return CAUSAL ? min(kv_total, 2 * pair + t + 1) : kv_total;
}

// Block-sparse activity of the pair's two query tiles as bitmasks in shared memory: bit j of
// tile t is set iff key tile j is visible to it (kv_tiles) and the byte mask marks block
// (query tile, j) active.  A query tile past the last one (odd tile count) has no bits.
// Each role keeps its own copy (the roles work on different units at a time): the producer
// and the MMA issuer one per tile, every softmax warp one of its own tile.
constexpr int kMaskWords = 32;  // up to 1024 key tiles (N <= 131072)
// Walks the set bits of one tile's bitmask in order, one word cached in a register.
struct BitIter {
  const uint32_t* w;
  int wi;
  uint32_t bits;
  __device__ __forceinline__ void init(const uint32_t* words) {
    w = words;
    wi = 0;
    bits = words[0];
  }
  // Returns the next set bit (consuming it), or -1 when none is left.
  __device__ __forceinline__ int pop() {
    while (bits == 0u) {
      if (++wi >= kMaskWords) return -1;
      bits = w[wi];
    }
    const int b = __ffs(bits) - 1;
    bits &= bits - 1u;
    return 32 * wi + b;
  }
};

struct PairMask {
  const uint32_t* w0;  // kMaskWords words per tile
  const uint32_t* w1;
};
// Packs the byte mask into kMaskWords bitmask words per query tile (run once per call, before
// the attention kernel): bit j of tile qt is set iff key tile j is visible to qt and
// mask[qt][j] != 0.  One thread per word.
template <bool CAUSAL>
__global__ void pack_mask_kernel(const uint8_t* __restrict__ mask, uint32_t* __restrict__ words,
                                 int nq_tiles, int kv_total) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nq_tiles * kMaskWords) return;
  const int qt = i / kMaskWords, wi = i % kMaskWords;
  const int nkv = CAUSAL ? min(kv_total, qt + 1) : kv_total;
  const uint8_t* row = mask + static_cast<size_t>(qt) * kv_total;
  uint32_t bits = 0u;
#pragma unroll 4
  for (int b = 0; b < 32; ++b) {
    const int j = 32 * wi + b;
    if (j < nkv && row[j] != 0) bits |= 1u << b;
  }
  words[i] = bits;
}

// Copies query tile qt's words into this role's shared-memory copy (128 bytes, 16 at a time).
__device__ __forceinline__ void copy_tile_words(uint32_t* dst, const uint32_t* __restrict__ words,
                                                int qt) {
  const uint4* src = reinterpret_cast<const uint4*>(words + static_cast<size_t>(qt) * kMaskWords);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < kMaskWords / 4; ++i) d4[i] = __ldg(src + i);
}

// Number of active key tiles of query tile qt (set bits of its words).
__device__ __forceinline__ int count_tile_words(const uint32_t* __restrict__ words, int qt) {
  const uint4* src = reinterpret_cast<const uint4*>(words + static_cast<size_t>(qt) * kMaskWords);
  int n = 0;
#pragma unroll
  for (int i = 0; i < kMaskWords / 4; ++i) {
    const uint4 v = __ldg(src + i);
    n += __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
  }
  return n;
}

// Maximum of n values as a tree of 3-input max operations (depth log3 n).
template <int n>
__device__ __forceinline__ float tree_max(const float* v) {
  if constexpr (n == 1) {
    return v[0];
  } else if constexpr (n == 2) {
    return fmaxf(v[0], v[1]);
  } else {
    constexpr int m = (n + 2) / 3;
    float w[m];
#pragma unroll
    for (int i = 0; i < n / 3; ++i) w[i] = max3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    if constexpr (n % 3 == 1) w[m - 1] = v[n - 1];
    if constexpr (n % 3 == 2) w[m - 1] = fmaxf(v[n - 2], v[n - 1]);
    return tree_max<m>(w);
  }
}

// F8: tm_q / tm_k map E4M3 [B][N][H][d], tm_v maps E4M3 V^T [B][H][d][Npad] (keys
// contiguous), and scales[3][B*H] holds the per-head dequantisation scales of Q, K, V.
// SPARSE: mask_words (pack_mask_kernel's output, kMaskWords words per query tile) selects the
// 128 x 128 blocks worked on (block-sparse attention).  A unit is then one query tile, not a
// pair: Q is loaded once, the loader streams the tile's active key tiles in order, and they
// go to the two ping-pong slots in turn (slot t takes the active key tiles k = t, t+2, ...),
// each slot keeping its own running max, sum and O.  So both slots stay busy whatever the
// mask, and at the end softmax warpgroup 0 merges the two partial results exactly, as the
// split-KV merge does: O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) + l_1 2^(m_1-m)),
// m = max(m_0, m_1).  A query tile with no active block gets O = 0, LSE = -inf.
template <int D, bool CAUSAL, bool F8, bool SPARSE = false>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               float* __restrict__ lse, const float* __restrict__ scales,
               const uint32_t* __restrict__ mask_words, int B, int H, int N, float scale_log2,
               int num_pairs, int* status, uint64_t timeout_ns) {
  using C = Cfg<D, F8>;
  constexpr int kKSt = SPARSE ? C::kStages + 1 : C::kStages;  // K ring depth
  constexpr int kVSt = C::kStages;                            // V ring depth
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // 128-byte-swizzled tiles need a 1024-aligned base
    if (threadIdx.x == 0) atomicCAS(status, FA_OK, FA_ERR_UNSUPPORTED);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BH = B * H;
  const int num_units = BH * num_pairs;
  const int G = gridDim.x;
  const int kv_total = (N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kKSt; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVSt; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], BM);
      mbar_init(&bars->p_half[t], BM);
      mbar_init(&bars->o_done[t], 1);
      mbar_init(&bars->o_free[t], BM);
    }
    mbar_init(&bars->merge_ready, BM);
    mbar_init(&bars->merge_free, BM);
    mbar_init(&bars->drain, 1);
    bars->abort.flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;
  Abort* ab = &bars->abort;
  uint8_t* sQ = smem + C::kOffQ;
  // Block-sparse units hold one query tile, so Q1's slot becomes one more K stage (it sits
  // right before the K ring): K runs kStages + 1 deep, V kStages.
  uint8_t* sK = SPARSE ? smem + C::kOffQ + C::kTileBytes : smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  const int wg = warp >> 2;

  // Role dispatch by warpgroup: each warpgroup reallocates its registers once, up front.
  if (wg < 2) {
    regs_set<kRegsLaunch, kRegsSoftmax<F8>>();
    // ------------------------------------------------------------------ softmax warps
    const int t = wg;                      // query tile of the pair (block-sparse: slot)
    const int r = (warp & 3) * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_base = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t colS = BN * t;
    const uint32_t colO = C::kColO + 128 * t;
    int ns = 0;     // s_full phases consumed
    int units = 0;  // units finished
    bool ok = true;
    for (int rr = 0; ok; ++rr) {
      const int u = unit_of_round(rr, G);
      if (u >= num_units) break;
      const Unit x = decode_unit<CAUSAL>(u, BH, num_pairs);
      const int b = x.bh / H, h = x.bh % H;
      const int q0 = (SPARSE ? x.pair : 2 * x.pair + t) * BM;
      const int row = q0 + r;
      const int nkv = kv_tiles<CAUSAL>(x.pair, t, kv_total);
      // Logit scale in log2 units (8-bit path: times the Q and K dequantisation scales) and
      // the output's extra factor (8-bit path: V's scale).
      float sl2 = scale_log2, out_mul = 1.f;
      if constexpr (F8) {
        sl2 *= scales[x.bh] * scales[BH + x.bh];
        out_mul = scales[2 * BH + x.bh];
      }
      float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale by < 2^8)
      float l = 0.f;
      PairMask pm;
      if constexpr (SPARSE) {
        uint32_t* words = reinterpret_cast<uint32_t*>(smem + C::kOffMask) + (4 + warp) * kMaskWords;
        __syncwarp();  // every lane is done with the previous unit's words
        words[lane] = __ldg(mask_words + static_cast<size_t>(x.pair) * kMaskWords + lane);
        __syncwarp();
        pm.w0 = pm.w1 = words;
      }
      // Block-sparse: this slot takes every other active key tile (slot 1 skips the first).
      BitIter it;
      if constexpr (SPARSE) {
        it.init(pm.w0);
        if (t == 1) it.pop();
      }
      auto next_j = [&]() -> int {
        const int jj = it.pop();
        it.pop();  // the other slot's
        return jj;
      };
      for (int j = SPARSE ? next_j() : 0; SPARSE ? j >= 0 : j < nkv; j = SPARSE ? next_j() : j + 1) {
        // Decisions guarding warp-collective tcgen05.ld/st are made warp-uniform.
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], ns & 1, ab, status, timeout_ns));
        if (!ok) break;
        ++ns;
        tc_fence_after();
        float sv[BN];
        {
          uint32_t u0[64];
          tmem_ld64(lane_base + colS, u0);
#pragma unroll
          for (int i = 0; i < 64; ++i) sv[i] = __uint_as_float(u0[i]);
        }
        {
          uint32_t u1[64];
          tmem_ld64(lane_base + colS + 64, u1);
#pragma unroll
          for (int i = 0; i < 64; ++i) sv[64 + i] = __uint_as_float(u1[i]);
        }
        const int k0 = j * BN;
        const bool masked = (CAUSAL && k0 + BN - 1 > q0) || k0 + BN > N;  // diagonal / tail
        if (masked) {
          const int lim = min(CAUSAL ? row : N - 1, N - 1) - k0;  // last visible column
#pragma unroll
          for (int i = 0; i < BN; ++i)
            if (i > lim) sv[i] = -INFINITY;
        }
        const float mx = tree_max<BN>(sv);
        const float m_tile = mx * sl2;
        float alpha = 1.f;
        bool need = false;
        if (m == -INFINITY) {
          m = m_tile;
        } else if (m_tile - m > kRescaleThreshold) {
          alpha = ex2_approx(m - m_tile);
          m = m_tile;
          need = true;
        }
        if constexpr (kSplitP<F8>) {
          // O_t holds sum_{j'<j} P V, and PV_t(j-1) has completed: it precedes S_t(j).  With P
          // published in two halves it is rescaled before the exponentials (the first PV half
          // follows the first half of P).
          auto rescale_o = [&]() {
            if (__any_sync(0xffffffffu, need)) {
  #pragma unroll
              for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_base + colO + c * 32, o);
  #pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                tmem_st32(lane_base + colO + c * 32, o);
              }
            }
          };
          rescale_o();
          // p = exp2(s * scale*log2(e) - m), two elements per packed FFMA.  On unmasked tiles
          // a fixed share of the pairs uses the FMA-pipe exp2 so that the MUFU unit and the
          // FMA pipe share the exponentials; masked tiles use the hardware exp2 only, which
          // maps the masked -inf logits to exact zeros.  P goes to the first columns of this
          // tile's S region (bf16 pairs: 64 columns, E4M3 quads: 32) in two halves of 64 keys;
          // the first is published (p_half) before the second is computed, so the tensor core
          // starts on PV while the softmax is still busy.
          const uint64_t c2 = f2_pack(sl2, sl2);
          const uint64_t nm2 = f2_pack(-m, -m);
          uint64_t acc2[2] = {0ull, 0ull};
          uint32_t pk[BN / 2];
          auto softmax_pairs = [&](auto emulate, auto half) {
            constexpr int h = decltype(half)::value;
  #pragma unroll
            for (int i = h * BN / 4; i < (h + 1) * BN / 4; ++i) {
              const uint64_t xs = f2_fma(f2_pack(sv[2 * i], sv[2 * i + 1]), c2, nm2);
              uint64_t p2;
              if (decltype(emulate)::value && (i % 8) < kEmuPairsPer8<D, F8>) {
                p2 = exp2_poly2(xs);
              } else {
                float x0, x1;
                f2_unpack(xs, x0, x1);
                p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
              }
              acc2[i & 1] = f2_add(acc2[i & 1], p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              pk[i] = F8 ? pack_e4m3x2(p0, p1) : pack_bf16x2(p0, p1);
            }
            {  // publish this half
  #pragma unroll
              for (int hh = h; hh <= h; ++hh) {
                if constexpr (F8) {
                  uint32_t w[BN / 8];
  #pragma unroll
                  for (int i = 0; i < BN / 8; ++i)
                    w[i] = pk[hh * BN / 4 + 2 * i] | (pk[hh * BN / 4 + 2 * i + 1] << 16);
                  tmem_st16(lane_base + colS + 16 * hh, w);
                } else {
                  tmem_st32(lane_base + colS + 32 * hh,
                            *reinterpret_cast<uint32_t(*)[32]>(&pk[hh * BN / 4]));
                }
              }
              tmem_st_wait();
              tc_fence_before();
              mbar_arrive(h == 0 ? &bars->p_half[t] : &bars->p_full[t]);
            }
          };
          if (masked) {
            softmax_pairs(std::false_type{}, std::integral_constant<int, 0>{});
            softmax_pairs(std::false_type{}, std::integral_constant<int, 1>{});
          } else {
            softmax_pairs(std::true_type{}, std::integral_constant<int, 0>{});
            softmax_pairs(std::true_type{}, std::integral_constant<int, 1>{});
          }
          {
            float s0, s1, s2, s3;
            f2_unpack(acc2[0], s0, s1);
            f2_unpack(acc2[1], s2, s3);
            l = l * alpha + ((s0 + s1) + (s2 + s3));
          }
        } else {
          // p = exp2(s * scale*log2(e) - m), two elements per packed FFMA.  On unmasked tiles
          // a fixed share of the pairs uses the FMA-pipe exp2 so that the MUFU unit and the
          // FMA pipe share the exponentials; masked tiles use the hardware exp2 only, which
          // maps the masked -inf logits to exact zeros.
          const uint64_t c2 = f2_pack(sl2, sl2);
          const uint64_t nm2 = f2_pack(-m, -m);
          uint64_t acc2[2] = {0ull, 0ull};
          uint32_t pk[BN / 2];
          auto softmax_pairs = [&](auto emulate) {
  #pragma unroll
            for (int i = 0; i < BN / 2; ++i) {
              const uint64_t xs = f2_fma(f2_pack(sv[2 * i], sv[2 * i + 1]), c2, nm2);
              uint64_t p2;
              if (decltype(emulate)::value && (i % 8) < kEmuPairsPer8<D, F8>) {
                p2 = exp2_poly2(xs);
              } else {
                float x0, x1;
                f2_unpack(xs, x0, x1);
                p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
              }
              acc2[i & 1] = f2_add(acc2[i & 1], p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              pk[i] = F8 ? pack_e4m3x2(p0, p1) : pack_bf16x2(p0, p1);
            }
          };
          if (masked) {
            softmax_pairs(std::false_type{});
          } else {
            softmax_pairs(std::true_type{});
          }
          {
            float s0, s1, s2, s3;
            f2_unpack(acc2[0], s0, s1);
            f2_unpack(acc2[1], s2, s3);
            l = l * alpha + ((s0 + s1) + (s2 + s3));
          }
          // P into the first columns of this tile's S region: bf16 pairs (64 columns) or
          // E4M3 quads (32 columns).
          if constexpr (F8) {
            uint32_t w[BN / 4];
  #pragma unroll
            for (int i = 0; i < BN / 4; ++i) w[i] = pk[2 * i] | (pk[2 * i + 1] << 16);
            tmem_st32(lane_base + colS, w);
          } else {
            tmem_st32(lane_base + colS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(lane_base + colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
          }
          if (__any_sync(0xffffffffu, need)) {
            // O_t holds sum_{j'<j} P V, and PV_t(j-1) has completed: it precedes S_t(j).
  #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(lane_base + colO + c * 32, o);
  #pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(lane_base + colO + c * 32, o);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&bars->p_full[t]);
        }
      }
      if (!ok) break;
      // -------------------------------------------------------------- epilogue
      // O = O / l in bf16, written as whole 128-byte lines: each warp stages its 32 rows in
      // boxes of 64 head-dim elements (128-byte swizzle: conflict-free 16-byte shared stores)
      // and lane 0 hands each box to a TMA store, which clips the rows past N.  Before a box
      // is refilled, the store that read it must be done reading.
      const int r0 = q0 + (warp & 3) * 32;
      uint8_t* stage = smem + C::kOffStage + warp * C::kStageBytes;
      if constexpr (SPARSE) {
        // The two slots' partial results of the one query tile.  Warpgroup 1 publishes its
        // row maximum and sum in shared memory (its own staging boxes, which this mode does
        // not use otherwise); warpgroup 0 merges both slots' O straight out of TMEM (the same
        // lanes), writes O and the LSE, and then hands both O regions back.
        float* mg = reinterpret_cast<float*>(smem + C::kOffStage + 4 * C::kStageBytes);
        if (t == 1) {
          if (units > 0) {  // warpgroup 0 has read the previous unit's values
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars->merge_free, (units - 1) & 1, ab, status, timeout_ns));
            if (!ok) break;
          }
          mg[r] = m;
          mg[BM + r] = l;
          mbar_arrive(&bars->merge_ready);
          ++units;
          continue;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[0], units & 1, ab, status, timeout_ns) &&
                                         mbar_wait(&bars->o_done[1], units & 1, ab, status, timeout_ns) &&
                                         mbar_wait(&bars->merge_ready, units & 1, ab, status, timeout_ns));
        if (!ok) break;
        tc_fence_after();
        const float m1 = mg[r], l1 = mg[BM + r];
        mbar_arrive(&bars->merge_free);
        // A slot that saw no key tile has l = 0 (and m = -inf): it contributes nothing.
        const float mm = fmaxf(m, m1);
        const float f0 = l > 0.f ? ex2_approx(m - mm) : 0.f;
        const float f1 = l1 > 0.f ? ex2_approx(m1 - mm) : 0.f;
        const float lt = l * f0 + l1 * f1;
        const bool empty = !(lt > 0.f);
        const float a0 = empty ? 0.f : f0 / lt, a1 = empty ? 0.f : f1 / lt;
        if (row < N)
          lse[static_cast<size_t>(x.bh) * N + row] =
              empty ? -INFINITY : (mm + __log2f(lt)) * 0.69314718055994531f;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o0[64], o1[64];
          tmem_ld64(lane_base + C::kColO + 64 * c, o0);
          tmem_ld64(lane_base + C::kColO + 128 + 64 * c, o1);
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              v[i] = __uint_as_float(o0[8 * p + i]) * a0 + __uint_as_float(o1[8 * p + i]) * a1;
            *reinterpret_cast<uint4*>(stage + sw128_offset(lane, p)) =
                make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                           pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && r0 < N) {
            tma_store_4d(&tm_o, stage, 64 * c, h, r0, b);
            bulk_commit();
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->o_free[0]);  // the next unit's first PVs may overwrite O_0, O_1
        mbar_arrive(&bars->o_free[1]);
        ++units;
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[t], units & 1, ab, status, timeout_ns));
        if (!ok) break;
        tc_fence_after();
        uint32_t o[D];
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tmem_ld64(lane_base + colO + 64 * c, *reinterpret_cast<uint32_t(*)[64]>(&o[64 * c]));
        tc_fence_before();
        mbar_arrive(&bars->o_free[t]);  // the next unit's first PV may overwrite O_t now
        ++units;
        if (row < N)
          lse[static_cast<size_t>(x.bh) * N + row] = (m + __log2f(l)) * 0.69314718055994531f;
        const float inv_l = out_mul / l;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const uint32_t* e = &o[64 * c + 8 * p];
            *reinterpret_cast<uint4*>(stage + sw128_offset(lane, p)) = make_uint4(
                pack_bf16x2(__uint_as_float(e[0]) * inv_l, __uint_as_float(e[1]) * inv_l),
                pack_bf16x2(__uint_as_float(e[2]) * inv_l, __uint_as_float(e[3]) * inv_l),
                pack_bf16x2(__uint_as_float(e[4]) * inv_l, __uint_as_float(e[5]) * inv_l),
                pack_bf16x2(__uint_as_float(e[6]) * inv_l, __uint_as_float(e[7]) * inv_l));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && r0 < N) {
            tma_store_4d(&tm_o, stage, 64 * c, h, r0, b);
            bulk_commit();
          }
        }
      }
    }
    // Every O store has completed before the CTA's shared memory goes away.
    if (lane == 0) bulk_wait_all();
    if ((warp & 3) == 0 && lane == 0) {
      bars->count[4 + t] = ns;
      bars->count[8 + t] = units;
    }
  } else {
    regs_set<kRegsLaunch, kRegsOther<F8>>();
    if (warp == kWarpLoad) {
      // ---------------------------------------------------------------- TMA producer
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        const uint64_t pol_q = policy_evict_first();
        const uint64_t pol_kv = policy_evict_last();
        int g = 0;      // K/V tiles issued so far (ring position)
        int units = 0;  // units started
        bool ok = true;
        for (int r = 0; ok; ++r) {
          const int u = unit_of_round(r, G);
          if (u >= num_units) break;
          const Unit x = decode_unit<CAUSAL>(u, BH, num_pairs);
          const int b = x.bh / H, h = x.bh % H;
          if (units > 0 &&
              !(ok = mbar_wait(&bars->q_empty, (units - 1) & 1, ab, status, timeout_ns)))
            break;
          // Dense: the pair's two query tiles.  Block-sparse: the unit's one query tile (both
          // slots read it).
          constexpr int kQTiles = SPARSE ? 1 : 2;
          mbar_arrive_expect_tx(&bars->q_full, kQTiles * C::kTileBytes);
          for (int t = 0; t < kQTiles; ++t)
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_4d(sQ + t * C::kTileBytes + c * C::kChunkBytes, &tm_q, &bars->q_full,
                          c * C::kChunkElems, h, (SPARSE ? x.pair : 2 * x.pair + t) * BM, b, pol_q);
          ++units;
          const int nkv = kv_tiles<CAUSAL>(x.pair, 1, kv_total);
          // Block-sparse: the query tile's active key tiles, in order.
          BitIter it0;
          if constexpr (SPARSE) {
            uint32_t* words = reinterpret_cast<uint32_t*>(smem + C::kOffMask);
            copy_tile_words(words, mask_words, x.pair);
            it0.init(words);
          }
          for (int j = SPARSE ? it0.pop() : 0; SPARSE ? j >= 0 : j < nkv;
               j = SPARSE ? it0.pop() : j + 1, ++g) {
            const int s = g % kKSt, sv = g % kVSt;
            if (g >= kKSt &&
                !(ok = mbar_wait(&bars->k_empty[s], ((g / kKSt) - 1) & 1, ab, status, timeout_ns)))
              break;
            mbar_arrive_expect_tx(&bars->k_full[s], C::kTileBytes);
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_4d(sK + s * C::kTileBytes + c * C::kChunkBytes, &tm_k, &bars->k_full[s],
                          c * C::kChunkElems, h, j * BN, b, pol_kv);
            if (g >= kVSt &&
                !(ok = mbar_wait(&bars->v_empty[sv], ((g / kVSt) - 1) & 1, ab, status, timeout_ns))) {
              ++g;  // K of this tile is in flight: count it for the drain below
              break;
            }
            mbar_arrive_expect_tx(&bars->v_full[sv], C::kTileBytes);
            if constexpr (F8) {  // V^T box: 128 keys x 128 head-dim rows
              tma_load_4d(sV + sv * C::kTileBytes, &tm_v, &bars->v_full[sv], j * BN, 0, h, b,
                          pol_kv);
            } else {
              for (int c = 0; c < C::kChunks; ++c)
                tma_load_4d(sV + sv * C::kTileBytes + c * C::kChunkBytes, &tm_v, &bars->v_full[sv],
                            c * 64, h, j * BN, b, pol_kv);
            }
          }
        }
        // Drain: no copy into shared memory may still be in flight when the CTA exits.
        // Only the last Q tiles, the last kKSt K tiles and the last kVSt V tiles can be
        // outstanding.  (On the abort path the last V copy may not have been issued; its wait
        // then runs out harmlessly.)
        bars->count[0] = g;
        bars->count[1] = units;
        Abort local{0};
        if (units > 0) mbar_wait(&bars->q_full, (units - 1) & 1, &local, status, timeout_ns);
        for (int gg = max(0, g - kKSt); gg < g; ++gg)
          mbar_wait(&bars->k_full[gg % kKSt], (gg / kKSt) & 1, &local, status, timeout_ns);
        for (int gg = max(0, g - kVSt); gg < g; ++gg)
          if (ok || gg < g - 1)
            mbar_wait(&bars->v_full[gg % kVSt], (gg / kVSt) & 1, &local, status, timeout_ns);
      }
    } else if (warp == kWarpMma) {
      // ---------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc_s = F8 ? idesc_e4m3_f32(BM, BN, 0, 0) : idesc_bf16_f32(BM, BN, 0, 0);
        // PV: bf16 V is [keys][d] (MN-major B); the 8-bit V^T is [d][keys] (K-major B).
        constexpr uint32_t idesc_o = F8 ? idesc_e4m3_f32(BM, D, 0, 0) : idesc_bf16_f32(BM, D, 0, 1);
        // Descriptors of the first Q, K and V tiles; the others are offsets from them.
        const uint64_t dQ0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
        const uint64_t dV0 = sdesc_sw128(smem_u32(sV), F8 ? 16 : C::kChunkBytes, 1024);
        int g = 0;            // K/V tiles consumed so far (ring position)
        int units = 0;        // units finished
        int np[2] = {0, 0};   // p_full phases consumed per tile
        bool ok = true;
        int s_issued0 = 0, s_issued1 = 0;  // S products issued per tile (protocol check)
        auto issue_s = [&](int t, int s) {  // S_t = Q_t K^T (both K-major over the head dim)
          (t ? s_issued1 : s_issued0) += 1;
          const uint64_t kd = sdesc_advance(dK0, s * C::kTileBytes);
          const uint64_t qd = sdesc_advance(dQ0, SPARSE ? 0 : t * C::kTileBytes);  // sparse: one Q
          // One MMA per 32 bytes of the head dim (16 bf16 or 32 E4M3 elements).
#pragma unroll
          for (int kk = 0; kk < C::kRowBytes / 32; ++kk) {
            const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
            if constexpr (F8)
              umma_ss_f8(tbase + BN * t, sdesc_advance(qd, off), sdesc_advance(kd, off), idesc_s,
                         kk > 0);
            else
              umma_ss(tbase + BN * t, sdesc_advance(qd, off), sdesc_advance(kd, off), idesc_s,
                      kk > 0);
          }
          umma_commit(&bars->s_full[t]);
        };
        // O_t += P_t V over keys [64 h, 64 h + 64) of the tile (P from TMEM).
        auto issue_pv_half = [&](int t, int s, bool first, int h) {
          const uint64_t vd = sdesc_advance(dV0, s * C::kTileBytes);
          if constexpr (F8) {  // 32 keys per MMA: 8 TMEM columns of P, 32 bytes of V^T rows
#pragma unroll
            for (int k2 = 0; k2 < BN / 64; ++k2) {
              const int kk = h * (BN / 64) + k2;
              umma_ts_f8(tbase + C::kColO + 128 * t, tbase + BN * t + kk * 8,
                         sdesc_advance(vd, kk * 32), idesc_o, (!first || kk > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int k2 = 0; k2 < BN / 32; ++k2) {
              const int kk = h * (BN / 32) + k2;
              umma_ts(tbase + C::kColO + 128 * t, tbase + BN * t + kk * 8,
                      sdesc_advance(vd, kk * 2048), idesc_o,
                      (!first || kk > 0) ? 1u : 0u);
            }
          }
        };
        // Both halves of PV_t: each after its half of P is published (unsplit: both after all
        // of P).  Returns false on abort.
        auto issue_pv = [&](int t, int s, bool first, int& npt) -> bool {
          if constexpr (kSplitP<F8>) {
            if (!mbar_wait(&bars->p_half[t], npt & 1, ab, status, timeout_ns)) return false;
            tc_fence_after();
            issue_pv_half(t, s, first, 0);
          } else {
            if (!mbar_wait(&bars->p_full[t], npt & 1, ab, status, timeout_ns)) return false;
            tc_fence_after();
            issue_pv_half(t, s, first, 0);
            issue_pv_half(t, s, first, 1);
            ++npt;
            return true;
          }
          if (!mbar_wait(&bars->p_full[t], npt & 1, ab, status, timeout_ns)) return false;
          tc_fence_after();
          issue_pv_half(t, s, first, 1);
          ++npt;
          return true;
        };
        if constexpr (SPARSE) {
          // Block-sparse issue order.  The unit's cnt active key tiles sit at ring positions
          // g .. g+cnt-1 in order; the k-th goes to slot k % 2.  After S_0(k=0) and S_1(k=1),
          // for k = 0, 1, 2, ...: PV_{k%2}(k), then that slot's next S (k+2) at once, so the
          // order is the dense one, PV_0, S_0, PV_1, S_1, with the two slots on different key
          // tiles.  Each K stage is read by one S and each V stage by one PV, so each is
          // released right after it.
          for (int r = 0; ok; ++r) {
            const int u = unit_of_round(r, G);
            if (u >= num_units) break;
            const Unit x = decode_unit<CAUSAL>(u, BH, num_pairs);
            const int cnt = count_tile_words(mask_words, x.pair);
            if (!(ok = mbar_wait(&bars->q_full, units & 1, ab, status, timeout_ns))) break;
            // A slot with no key tile has nothing to accumulate: its O is signalled done at
            // once, but only after warpgroup 0 has read the previous unit's O (without that
            // wait o_done could complete twice before it is polled, and a wait on a phase's
            // parity cannot tell two completions from none).
            for (int t = 0; t < 2 && ok; ++t) {
              if (cnt > t) continue;
              if (units > 0 &&
                  !(ok = mbar_wait(&bars->o_free[t], (units - 1) & 1, ab, status, timeout_ns)))
                break;
              umma_commit(&bars->o_done[t]);
            }
            if (!ok) break;
            if (cnt == 0) umma_commit(&bars->q_empty);
            auto issue_s_at = [&](int k) -> bool {  // S_{k%2} on ring position g + k
              const int pos = g + k, s = pos % kKSt;
              if (!mbar_wait(&bars->k_full[s], (pos / kKSt) & 1, ab, status, timeout_ns))
                return false;
              tc_fence_after();
              issue_s(k & 1, s);
              umma_commit(&bars->k_empty[s]);
              if (k == cnt - 1) umma_commit(&bars->q_empty);  // the unit's last S product
              return true;
            };
            if (cnt >= 1 && !(ok = issue_s_at(0))) break;
            if (cnt >= 2 && !(ok = issue_s_at(1))) break;
            for (int k = 0; ok && k < cnt; ++k) {
              const int t = k & 1, pos = g + k, s = pos % kVSt;
              if (!(ok = mbar_wait(&bars->v_full[s], (pos / kVSt) & 1, ab, status,
                                   timeout_ns)))
                break;
              if (k < 2 && units > 0 &&
                  !(ok = mbar_wait(&bars->o_free[t], (units - 1) & 1, ab, status, timeout_ns)))
                break;
              if (!(ok = issue_pv(t, s, k < 2, np[t]))) break;
              umma_commit(&bars->v_empty[s]);
              if (k + 2 < cnt) {
                if (!(ok = issue_s_at(k + 2))) break;
              } else {
                umma_commit(&bars->o_done[t]);  // slot t's last PV of the unit
              }
            }
            g += cnt;
            ++units;
          }
        } else {
          for (int r = 0; ok; ++r) {
            const int u = unit_of_round(r, G);
            if (u >= num_units) break;
            const Unit x = decode_unit<CAUSAL>(u, BH, num_pairs);
            const int nkv0 = kv_tiles<CAUSAL>(x.pair, 0, kv_total);
            const int nkv1 = kv_tiles<CAUSAL>(x.pair, 1, kv_total);
            if (!(ok = mbar_wait(&bars->q_full, units & 1, ab, status, timeout_ns))) break;
            {  // prologue: S0(0), S1(0)
              const int s = g % C::kStages;
              if (!(ok = mbar_wait(&bars->k_full[s], (g / C::kStages) & 1, ab, status, timeout_ns)))
                break;
              tc_fence_after();
              issue_s(0, s);
              issue_s(1, s);
              umma_commit(&bars->k_empty[s]);
              if (nkv1 == 1) umma_commit(&bars->q_empty);  // last S products of this unit
            }
            for (int j = 0; ok && j < nkv1; ++j) {
              const int s = (g + j) % C::kStages;
              const int s1 = (g + j + 1) % C::kStages;
              const bool more = j + 1 < nkv1;
              if (!(ok = mbar_wait(&bars->v_full[s], ((g + j) / C::kStages) & 1, ab, status,
                                   timeout_ns)))
                break;
              if (more && !(ok = mbar_wait(&bars->k_full[s1], ((g + j + 1) / C::kStages) & 1, ab,
                                           status, timeout_ns)))
                break;
              if (j < nkv0) {  // tile 0: PV0(j), S0(j+1)
                if (j == 0 && units > 0 &&
                    !(ok = mbar_wait(&bars->o_free[0], (units - 1) & 1, ab, status, timeout_ns)))
                  break;
                if (!(ok = issue_pv(0, s, j == 0, np[0]))) break;
                if (j + 1 < nkv0) {
                  issue_s(0, s1);
                } else {
                  umma_commit(&bars->o_done[0]);
                }
              }
              // tile 1: PV1(j), S1(j+1)
              if (j == 0 && units > 0 &&
                  !(ok = mbar_wait(&bars->o_free[1], (units - 1) & 1, ab, status, timeout_ns)))
                break;
              if (!(ok = issue_pv(1, s, j == 0, np[1]))) break;
              umma_commit(&bars->v_empty[s]);
              if (more) {
                issue_s(1, s1);
                umma_commit(&bars->k_empty[s1]);
                if (j + 2 == nkv1) umma_commit(&bars->q_empty);  // last S products of this unit
              } else {
                umma_commit(&bars->o_done[1]);
              }
            }
            g += nkv1;
            ++units;
          }
        }
        bars->count[2] = g;
        bars->count[3] = units;
        bars->count[6] = s_issued0;
        bars->count[7] = s_issued1;
        // Drain every MMA this thread issued before TMEM is released.
        umma_commit(&bars->drain);
        Abort local{0};
        mbar_wait(&bars->drain, 0, &local, status, timeout_ns);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The roles must agree on what they did (skipped after a timed-out wait, when they may
  // not): every K/V tile loaded was consumed, every unit was seen by all four roles, and
  // each softmax warpgroup took exactly one step per S product of its tile.
  if (threadIdx.x == 0 && !*reinterpret_cast<volatile int*>(&ab->flag)) {
    const int* c = bars->count;
    const bool agree = c[0] == c[2] && c[1] == c[3] && c[3] == c[8] && c[3] == c[9] &&
                       c[4] == c[6] && c[5] == c[7];
    if (!agree) atomicCAS(status, FA_OK, FA_ERR_INTERNAL);
  }
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Self-test: CTA c of a `grid`-CTA launch writes, round by round, the units the forward's
// persistent schedule hands it (bh * num_pairs + pair), then -1.
template <bool CAUSAL>
__global__ void schedule_kernel(int BH, int num_pairs, int* __restrict__ out, int max_rounds) {
  if (threadIdx.x != 0) return;
  const int G = gridDim.x;
  const int num_units = BH * num_pairs;
  for (int r = 0; r < max_rounds; ++r) {
    const int u = unit_of_round(r, G);
    if (u >= num_units) {
      out[blockIdx.x * max_rounds + r] = -1;
      return;
    }
    const Unit x = decode_unit<CAUSAL>(u, BH, num_pairs);
    out[blockIdx.x * max_rounds + r] = x.bh * num_pairs + x.pair;
  }
}

template <int D, bool CAUSAL, bool F8 = false, bool SPARSE = false>
static cudaError_t launch_t(const FwdArgs& a, cudaStream_t st) {
  using C = Cfg<D, F8>;
  auto kern = fwd_kernel<D, CAUSAL, F8, SPARSE>;
  // The setmaxnreg split assumes the kernel launches with exactly kRegsLaunch registers per
  // thread; with fewer, the softmax warpgroups' increase could never be satisfied.
  cudaFuncAttributes fa_attr;
  cudaError_t e = cudaFuncGetAttributes(&fa_attr, kern);
  if (e != cudaSuccess) return e;
  if (fa_attr.numRegs != static_cast<int>(kRegsLaunch)) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // Units per (batch, head): pairs of query tiles (dense), single query tiles (block-sparse).
  const int num_pairs = SPARSE ? (a.N + BM - 1) / BM : (a.N + 2 * BM - 1) / (2 * BM);
  const long long units = static_cast<long long>(a.B) * a.H * num_pairs;
  if (units > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int grid = static_cast<int>(std::min<long long>(units, a.num_sms));
  const float scale_log2 = a.scale * 1.4426950408889634f;
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_o, a.lse, a.scales,
                                              a.mask_words, a.B, a.H, a.N, scale_log2, num_pairs,
                                              a.status, kDefaultWaitTimeoutNs);
  return cudaGetLastError();
}

}  // namespace fwd

cudaError_t launch_fwd_sm100(const FwdArgs& a, cudaStream_t s) {
  if (a.d == 64) return a.causal ? fwd::launch_t<64, true>(a, s) : fwd::launch_t<64, false>(a, s);
  return a.causal ? fwd::launch_t<128, true>(a, s) : fwd::launch_t<128, false>(a, s);
}

cudaError_t launch_fwd_block_sparse(const FwdArgs& a, cudaStream_t s) {
  const int nq = (a.N + fwd::BM - 1) / fwd::BM, nk = (a.N + fwd::BN - 1) / fwd::BN;
  const int n = nq * fwd::kMaskWords;
  if (a.causal)
    fwd::pack_mask_kernel<true><<<(n + 255) / 256, 256, 0, s>>>(a.block_mask, a.mask_words, nq, nk);
  else
    fwd::pack_mask_kernel<false><<<(n + 255) / 256, 256, 0, s>>>(a.block_mask, a.mask_words, nq, nk);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.d == 64)
    return a.causal ? fwd::launch_t<64, true, false, true>(a, s)
                    : fwd::launch_t<64, false, false, true>(a, s);
  return a.causal ? fwd::launch_t<128, true, false, true>(a, s)
                  : fwd::launch_t<128, false, false, true>(a, s);
}

cudaError_t launch_debug_schedule(int B, int H, int N, int causal, int grid, int* out,
                                  int max_rounds, cudaStream_t s) {
  const int num_pairs = (N + 2 * fwd::BM - 1) / (2 * fwd::BM);
  if (causal)
    fwd::schedule_kernel<true><<<grid, 32, 0, s>>>(B * H, num_pairs, out, max_rounds);
  else
    fwd::schedule_kernel<false><<<grid, 32, 0, s>>>(B * H, num_pairs, out, max_rounds);
  return cudaGetLastError();
}

cudaError_t launch_fwd_fp8(const FwdArgs& a, cudaStream_t s) {
  if (a.d != 128) return cudaErrorNotSupported;
  return a.causal ? fwd::launch_t<128, true, true>(a, s) : fwd::launch_t<128, false, true>(a, s);
}

}  // namespace fa
