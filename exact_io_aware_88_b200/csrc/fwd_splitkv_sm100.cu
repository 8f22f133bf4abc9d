// fwd_splitkv_sm100.cu -- attention forward for few queries against many keys (decoding),
// with the key sequence split across CTAs, on sm_100a; bf16 or fp16 inputs.
//
// Prefill and decode stress different limits and are measured separately ("FlashAttention-2
// を読む", section 実装上の差を検証可能な形で残す).  With few queries per (batch, head) the
// forward kernel's units are too few to fill the GPU, so here the sequence dimension is
// split further: each CTA takes one 128-row query tile and a contiguous slice of the key
// tiles (the sequence-dimension parallelism of the second trick, section
// GPUの稼働率を高める三つの工夫), runs the same online softmax, and writes a partial result
// normalised over its slice together with the slice's logsumexp.  A second kernel merges the
// slices exactly: with L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s.
//
// Causal mask with Nq <= Nk: the last query is aligned with the last key, query i sees keys
// j <= i + (Nk - Nq).  fp16 inputs use kind::f16 with f16 operands and an f16 P; fp16 is
// FA-2's other input type ("Flash Attention 2で打破するローカルLLMの「メモリの壁」",
// section Hugging Face Transformersでの有効化設定).
//
// CTA = 6 warps: 0-3 softmax (thread t owns query row t = TMEM lane t), 4 TMA producer,
// 5 TMEM allocator + MMA issuer.  TMEM: S/P double buffer [0,128), [128,256), O [256,256+D).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "launch.h"
#include "ptx.cuh"

namespace fa {
namespace splitkv {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kChunkBytes = BM * 128;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 256;  // base is 1024-aligned (checked)
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[4], v_full[4], kv_empty[4];
  uint64_t s_full[2], p_full[2], pv_done, o_done, drain;
  uint32_t tmem_base;
  Abort abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block larger than its shared-memory region");

template <bool F16>
__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
  if constexpr (F16) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    return pack_bf16x2(lo, hi);
  }
}

// Instruction descriptor, kind::f16 with fp32 D: operand format 0 = f16, 1 = bf16.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn, bool f16) {
  return f16 ? (idesc_bf16_f32(M, N, a_mn, b_mn) & ~((7u << 7) | (7u << 10)))
             : idesc_bf16_f32(M, N, a_mn, b_mn);
}

template <int D, bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    splitkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, float* __restrict__ part_o,
                   float* __restrict__ part_lse, void* __restrict__ out, float* __restrict__ lse,
                   int H, int Nq, int Nk, int n_split,
                   int tiles_per_split, int num_qtiles, int BH, float scale_log2, int* status,
                   uint64_t timeout_ns) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, FA_OK, FA_ERR_UNSUPPORTED);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Unit (b*h, query tile, key slice).
  const int split = blockIdx.x % n_split;
  const int qt = (blockIdx.x / n_split) % num_qtiles;
  const int bh = blockIdx.x / (n_split * num_qtiles);
  const int b = bh / H, h = bh % H;
  const int q0 = qt * BM;
  const int off = Nk - Nq;  // causal alignment of the last query with the last key
  const int last_key = CAUSAL ? min(Nk - 1, q0 + BM - 1 + off) : Nk - 1;
  const int nvis = last_key / BN + 1;  // key tiles any row of this query tile can see
  const int j_begin = split * tiles_per_split;
  const int j_end = min(nvis, j_begin + tiles_per_split);
  const int nkv = max(0, j_end - j_begin);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], BM);
    }
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort.flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;
  Abort* ab = &bars->abort;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nkv > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t pol_q = policy_evict_last();
      const uint64_t pol_kv = policy_evict_first();  // each key tile is read by few CTAs
      mbar_arrive_expect_tx(&bars->q_full, C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(sQ + c * C::kChunkBytes, &tm_q, &bars->q_full, c * 64, h, q0, b, pol_q);
      int issued = 0;
      for (int n = 0; n < nkv; ++n) {
        const int j = j_begin + n;
        const int s = n % C::kStages;
        if (n >= C::kStages &&
            !mbar_wait(&bars->kv_empty[s], ((n / C::kStages) - 1) & 1, ab, status, timeout_ns))
          break;
        mbar_arrive_expect_tx(&bars->k_full[s], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sK + s * C::kTileBytes + c * C::kChunkBytes, &tm_k, &bars->k_full[s], c * 64,
                      h, j * BN, b, pol_kv);
        mbar_arrive_expect_tx(&bars->v_full[s], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sV + s * C::kTileBytes + c * C::kChunkBytes, &tm_v, &bars->v_full[s], c * 64,
                      h, j * BN, b, pol_kv);
        issued = n + 1;
      }
      Abort local{0};
      mbar_wait(&bars->q_full, 0, &local, status, timeout_ns);
      for (int n = max(0, issued - C::kStages); n < issued; ++n) {
        mbar_wait(&bars->k_full[n % C::kStages], (n / C::kStages) & 1, &local, status, timeout_ns);
        mbar_wait(&bars->v_full[n % C::kStages], (n / C::kStages) & 1, &local, status, timeout_ns);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && nkv > 0) {
      constexpr uint32_t idesc_s = idesc_f16(BM, BN, 0, 0, F16);
      constexpr uint32_t idesc_o = idesc_f16(BM, D, 0, 1, F16);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = mbar_wait(&bars->q_full, 0, ab, status, timeout_ns);
      tc_fence_after();
      auto issue_s = [&](int n) -> bool {
        const int s = n % C::kStages;
        if (!mbar_wait(&bars->k_full[s], (n / C::kStages) & 1, ab, status, timeout_ns)) return false;
        tc_fence_after();
        const uint32_t kb = aK + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          umma_ss(tbase + (n & 1) * BN, sdesc_sw128(aQ + koff, 16, 1024),
                  sdesc_sw128(kb + koff, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&bars->s_full[n & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int n = 0; ok && n < nkv; ++n) {
        if (n + 1 < nkv && !(ok = issue_s(n + 1))) break;
        const int s = n % C::kStages;
        if (!(ok = mbar_wait(&bars->p_full[n & 1], (n >> 1) & 1, ab, status, timeout_ns))) break;
        if (!(ok = mbar_wait(&bars->v_full[s], (n / C::kStages) & 1, ab, status, timeout_ns))) break;
        tc_fence_after();
        const uint32_t vb = aV + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(tbase + kColO, tbase + (n & 1) * BN + kk * 8,
                  sdesc_sw128(vb + kk * 2048, C::kChunkBytes, 1024), idesc_o, (n > 0 || kk > 0));
        umma_commit(&bars->kv_empty[s]);
        umma_commit(&bars->pv_done);
      }
      umma_commit(&bars->o_done);
      umma_commit(&bars->drain);
      Abort local{0};
      mbar_wait(&bars->drain, 0, &local, status, timeout_ns);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int r = threadIdx.x;
    const int row = q0 + r;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // Warps whose 32 rows all lie past Nq (few decoded queries) only keep the pipeline
    // moving: they hand back P without computing it.
    const bool warp_live = (q0 + warp * 32) < Nq;
    for (int n = 0; n < nkv; ++n) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[n & 1], (n >> 1) & 1, ab, status,
                                             timeout_ns));
      if (!ok) break;
      tc_fence_after();
      if (warp_live) {
        const uint32_t s_addr = lane_base + (n & 1) * BN;
        float sv[BN];
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) {
          uint32_t u[64];
          tmem_ld64(s_addr + 64 * c, u);
#pragma unroll
          for (int i = 0; i < 64; ++i) sv[64 * c + i] = __uint_as_float(u[i]);
        }
        const int k0 = (j_begin + n) * BN;
        const int lim = min(CAUSAL ? row + off : Nk - 1, Nk - 1) - k0;  // last visible column
        if (__any_sync(0xffffffffu, lim < BN - 1)) {
#pragma unroll
          for (int i = 0; i < BN; ++i)
            if (i > lim) sv[i] = -INFINITY;
        }
        float mx = sv[0];
#pragma unroll
        for (int i = 1; i < BN; ++i) mx = fmaxf(mx, sv[i]);
        const float m_tile = mx * scale_log2;
        float alpha = 1.f;
        bool need = false;
        if (m == -INFINITY) {
          m = m_tile;
        } else if (m_tile - m > kRescaleThreshold) {
          alpha = ex2_approx(m - m_tile);
          m = m_tile;
          need = true;
        }
        float sum = 0.f;
        uint32_t pk[BN / 2];
        if (m == -INFINITY) {  // row sees no key of this tile yet (only past-the-end rows)
#pragma unroll
          for (int i = 0; i < BN / 2; ++i) pk[i] = 0u;
        } else {
#pragma unroll
          for (int i = 0; i < BN / 2; ++i) {
            const float p0 = ex2_approx(fmaf(sv[2 * i], scale_log2, -m));
            const float p1 = ex2_approx(fmaf(sv[2 * i + 1], scale_log2, -m));
            sum += p0 + p1;
            pk[i] = pack_p<F16>(p0, p1);
          }
        }
        l = l * alpha + sum;
        tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        if (n > 0 && __any_sync(0xffffffffu, need)) {
          // O holds sum_{n'<n} P V; the product of step n-1 must have landed before the
          // rescale (S(n) was issued before PV(n-1), so it is not implied by s_full).
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bars->pv_done, (n - 1) & 1, ab, status, timeout_ns));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + 32 * c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(lane_base + kColO + 32 * c, o);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[n & 1]);
    }
    // ---------------------------------------------------------------- epilogue
    // Partial result of this key slice: O_s = (sum P V) / l and L_s = ln(l) + max (natural
    // log); a row that sees no key of the slice gives O_s = 0, L_s = -inf (weight 0 in the
    // merge).  With a single slice the partial result is the result: it goes straight to the
    // caller's O (bf16 / fp16, [B][Nq][H][D]) and LSE, and no merge runs.
    const size_t prow = (static_cast<size_t>(split) * BH + bh) * Nq + row;
    if (nkv > 0 && ok)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, 0, ab, status, timeout_ns));
    if (ok && warp_live) {
      const bool have = nkv > 0 && l > 0.f;
      const float inv_l = have ? 1.f / l : 0.f;
      if (nkv > 0) tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (nkv > 0) {
          tmem_ld32(lane_base + kColO + 32 * c, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (row < Nq && n_split == 1) {
          uint4* dst = reinterpret_cast<uint4*>(
              static_cast<uint16_t*>(out) + ((static_cast<size_t>(b) * Nq + row) * H + h) * D + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(o[8 * v + 2 * e]) * inv_l;
              const float x1 = __uint_as_float(o[8 * v + 2 * e + 1]) * inv_l;
              if constexpr (F16) {
                const __half2 hv = __floats2half2_rn(x0, x1);
                w[e] = *reinterpret_cast<const uint32_t*>(&hv);
              } else {
                w[e] = pack_bf16x2(x0, x1);
              }
            }
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else if (row < Nq) {
          float4* dst = reinterpret_cast<float4*>(part_o + prow * D + 32 * c);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                 __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
        }
      }
      if (row < Nq) {
        const float L = have ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (n_split == 1)
          lse[static_cast<size_t>(bh) * Nq + row] = L;
        else
          part_lse[prow] = L;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Merge of the key slices: L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s, written in
// the caller's layout ([B][Nq][H][D] in T, lse [B][H][Nq]).  D/4 threads per query row.
template <int D, typename T>
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                   T* __restrict__ out, float* __restrict__ lse, int H, int Nq, int BH, int n_split) {
  constexpr int kTPR = D / 4;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rowid = gid / kTPR;  // (bh, q) row
  const int part = static_cast<int>(gid % kTPR);
  if (rowid >= static_cast<long long>(BH) * Nq) return;
  const int bh = static_cast<int>(rowid / Nq), q = static_cast<int>(rowid % Nq);
  const size_t stride = static_cast<size_t>(BH) * Nq;
  float mx = -INFINITY;
  for (int s = 0; s < n_split; ++s) mx = fmaxf(mx, part_lse[s * stride + rowid]);
  float wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < n_split; ++s) {
    const float ls = part_lse[s * stride + rowid];
    const float w = (ls == -INFINITY) ? 0.f : expf(ls - mx);
    wsum += w;
    const float4 o = reinterpret_cast<const float4*>(part_o + (s * stride + rowid) * D)[part];
    acc.x = fmaf(w, o.x, acc.x);
    acc.y = fmaf(w, o.y, acc.y);
    acc.z = fmaf(w, o.z, acc.z);
    acc.w = fmaf(w, o.w, acc.w);
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;  // a row that sees no key: O = 0
  const int b = bh / H, h = bh % H;
  T* dst = out + ((static_cast<size_t>(b) * Nq + q) * H + h) * D + 4 * part;
  if constexpr (sizeof(T) == 2 && std::is_same<T, __half>::value) {
    reinterpret_cast<__half2*>(dst)[0] = __floats2half2_rn(acc.x * inv, acc.y * inv);
    reinterpret_cast<__half2*>(dst)[1] = __floats2half2_rn(acc.z * inv, acc.w * inv);
  } else {
    reinterpret_cast<__nv_bfloat162*>(dst)[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    reinterpret_cast<__nv_bfloat162*>(dst)[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  }
  if (part == 0) lse[rowid] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

template <int D, bool CAUSAL, bool F16>
static cudaError_t launch_t(const SplitKvArgs& a, cudaStream_t st) {
  using C = Cfg<D>;
  auto kern = splitkv_kernel<D, CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int num_qtiles = (a.Nq + BM - 1) / BM;
  const int BH = a.B * a.H;
  const long long grid = static_cast<long long>(BH) * num_qtiles * a.n_split;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, st>>>(
      a.tm_q, a.tm_k, a.tm_v, a.part_o, a.part_lse, a.o, a.lse, a.H, a.Nq, a.Nk, a.n_split,
      a.tiles_per_split, num_qtiles, BH, a.scale * 1.4426950408889634f, a.status,
      kDefaultWaitTimeoutNs);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.n_split == 1) return cudaSuccess;  // the split kernel wrote O and the LSE itself
  const long long threads = static_cast<long long>(BH) * a.Nq * (D / 4);
  const long long cgrid = (threads + 255) / 256;
  if (F16)
    combine_kernel<D, __half><<<static_cast<unsigned>(cgrid), 256, 0, st>>>(
        a.part_o, a.part_lse, static_cast<__half*>(a.o), a.lse, a.H, a.Nq, BH, a.n_split);
  else
    combine_kernel<D, __nv_bfloat16><<<static_cast<unsigned>(cgrid), 256, 0, st>>>(
        a.part_o, a.part_lse, static_cast<__nv_bfloat16*>(a.o), a.lse, a.H, a.Nq, BH, a.n_split);
  return cudaGetLastError();
}

}  // namespace splitkv

cudaError_t launch_fwd_splitkv(const SplitKvArgs& a, cudaStream_t s) {
  if (a.d == 64) {
    if (a.f16) return a.causal ? splitkv::launch_t<64, true, true>(a, s) : splitkv::launch_t<64, false, true>(a, s);
    return a.causal ? splitkv::launch_t<64, true, false>(a, s) : splitkv::launch_t<64, false, false>(a, s);
  }
  if (a.f16) return a.causal ? splitkv::launch_t<128, true, true>(a, s) : splitkv::launch_t<128, false, true>(a, s);
  return a.causal ? splitkv::launch_t<128, true, false>(a, s) : splitkv::launch_t<128, false, false>(a, s);
}

}  // namespace fa
