// fwd_sm100.cu -- attention forward on sm_100a: TMA K/V ring, tcgen05.mma into TMEM,
// warp-specialised load / MMA / softmax warps, online softmax in base 2.
//
// The algorithm is the tiled, fused evaluation of softmax(scale*QK^T)V described in
// "Flash Attention 2で打破するローカルLLMの「メモリの壁」" (section タイリング（Tiling）と
// 再計算（Recomputation）の仕組み): a 128-row Q tile stays on chip while 128-row K/V tiles
// stream past it; S and P live only in tensor memory.  The running max / sum rescaling that
// keeps the softmax globally normalised is the one of "FlashAttention-2を読む" (section
// タイル分割でも全体の正規化を保つ).  Non-matmul work is trimmed as in its first trick
// (section GPUの稼働率を高める三つの工夫): the scale is folded into one FFMA before exp2,
// masks are applied on diagonal / tail tiles only, 1/l is applied once at the end and the
// output is rescaled only when a row's running max grows by more than 2^8 (exact: the final
// normalisation uses the same, possibly stale, max).
//
// CTA = 6 warps:
//   warps 0-3  softmax: thread t owns query row t of the tile (= TMEM lane t)
//   warp  4    TMA producer (one lane)
//   warp  5    TMEM allocator + tcgen05.mma issuer (one lane)
// TMEM (512 columns): S/P double buffer at columns [0,128) and [128,256); O at [256,256+D).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"
#include "ptx.cuh"

namespace fa {
namespace fwd {

constexpr int BM = 128;               // query rows per tile
constexpr int BN = 128;               // key rows per tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;              // 64-element (128-byte) column chunks
  static constexpr int kChunkBytes = BM * 128;        // one TMA box: 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[4];
  uint64_t v_full[4];
  uint64_t kv_empty[4];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  Abort abort;
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
               float* __restrict__ lse, int B, int H, int N, float scale_log2, int num_qtiles,
               int* status, uint64_t timeout_ns) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (b, h) major so that concurrently running CTAs share K/V in L2; within a
  // head, causal tiles run longest first.
  const int bh = blockIdx.x / num_qtiles;
  int qt = blockIdx.x % num_qtiles;
  if (CAUSAL) qt = num_qtiles - 1 - qt;
  const int b = bh / H, h = bh % H;
  const int q0 = qt * BM;
  const int kv_tiles_total = (N + BN - 1) / BN;
  const int nkv = CAUSAL ? min(kv_tiles_total, qt + 1) : kv_tiles_total;

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
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();
      mbar_arrive_expect_tx(&bars->q_full, C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(sQ + c * C::kChunkBytes, &tm_q, &bars->q_full, c * 64, h, q0, b, pol_q);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % C::kStages;
        if (j >= C::kStages &&
            !mbar_wait(&bars->kv_empty[s], ((j / C::kStages) - 1) & 1, ab, status, timeout_ns))
          break;
        uint8_t* dk = sK + s * C::kTileBytes;
        uint8_t* dv = sV + s * C::kTileBytes;
        mbar_arrive_expect_tx(&bars->k_full[s], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(dk + c * C::kChunkBytes, &tm_k, &bars->k_full[s], c * 64, h, j * BN, b,
                      pol_kv);
        mbar_arrive_expect_tx(&bars->v_full[s], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(dv + c * C::kChunkBytes, &tm_v, &bars->v_full[s], c * 64, h, j * BN, b,
                      pol_kv);
        issued = j + 1;
      }
      // Drain: make sure no copy into this CTA's shared memory is still in flight.
      uint32_t drained = 1;
      Abort local{0};
      drained &= mbar_wait(&bars->q_full, 0, &local, status, timeout_ns);
      for (int j = (issued > C::kStages ? issued - C::kStages : 0); j < issued; ++j) {
        const int s = j % C::kStages;
        drained &= mbar_wait(&bars->k_full[s], (j / C::kStages) & 1, &local, status, timeout_ns);
        drained &= mbar_wait(&bars->v_full[s], (j / C::kStages) & 1, &local, status, timeout_ns);
      }
      (void)drained;
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = mbar_wait(&bars->q_full, 0, ab, status, timeout_ns);
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::kStages;
        if (!mbar_wait(&bars->k_full[s], (j / C::kStages) & 1, ab, status, timeout_ns))
          return false;
        tc_fence_after();
        const uint32_t d_tmem = tbase + (j & 1) * BN;
        const uint32_t kbase = aK + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          umma_ss(d_tmem, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024),
                  idesc_s, kk > 0);
        }
        umma_commit(&bars->s_full[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) break;
        const int s = j % C::kStages;
        if (!mbar_wait(&bars->p_full[j & 1], (j >> 1) & 1, ab, status, timeout_ns)) break;
        if (!mbar_wait(&bars->v_full[s], (j / C::kStages) & 1, ab, status, timeout_ns)) break;
        tc_fence_after();
        const uint32_t vbase = aV + s * C::kTileBytes;
        const uint32_t p_tmem = tbase + (j & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          umma_ts(tbase + kColO, p_tmem + kk * 8, sdesc_sw128(vbase + kk * 2048, C::kChunkBytes, 1024),
                  idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->kv_empty[s]);
        umma_commit(&bars->o_done);
      }
      // Drain every MMA this thread issued before TMEM is released.
      umma_commit(&bars->drain);
      Abort local{0};
      mbar_wait(&bars->drain, 0, &local, status, timeout_ns);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int r = threadIdx.x;  // row within the tile == TMEM lane
    const int row = q0 + r;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale by < 2^8)
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      // Every decision that guards a warp-collective tcgen05.ld/st is made warp-uniform.
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, ab, status,
                                             timeout_ns));
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_addr = lane_base + (j & 1) * BN;
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(s_addr + c * 32, u);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(u[i]);
      }
      const int k0 = j * BN;
      const bool diag = CAUSAL && (k0 + BN - 1 > q0);
      const bool tail = (k0 + BN > N);
      if (diag || tail) {
        const int lim = min(CAUSAL ? row : N - 1, N - 1) - k0;  // last visible column
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
#pragma unroll
      for (int i = 0; i < BN / 2; ++i) {
        const float p0 = ex2_approx(fmaf(sv[2 * i], scale_log2, -m));
        const float p1 = ex2_approx(fmaf(sv[2 * i + 1], scale_log2, -m));
        sum += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + sum;
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
        tmem_st32(s_addr, lo);
        tmem_st32(s_addr + 32, hi);
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds sum_{j'<j} P V; make sure the last PV landed before rescaling it.
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars->o_done, (j - 1) & 1, ab, status, timeout_ns));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld32(lane_base + kColO + c * 32, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          tmem_st32(lane_base + kColO + c * 32, u);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[j & 1]);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars->o_done, (nkv - 1) & 1, ab, status, timeout_ns));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = out + ((static_cast<size_t>(b) * N + row) * H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(lane_base + kColO + c * 32, u);
        uint32_t pkd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pkd[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
        if (row < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
        }
      }
      if (row < N)
        lse[(static_cast<size_t>(b) * H + h) * N + row] = (m + __log2f(l)) * 0.69314718055994531f;
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

template <int D, bool CAUSAL>
static cudaError_t launch_t(const FwdArgs& a, cudaStream_t st) {
  using C = Cfg<D>;
  auto kern = fwd_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int num_qtiles = (a.N + BM - 1) / BM;
  const long long grid = static_cast<long long>(a.B) * a.H * num_qtiles;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  kern<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, st>>>(
      a.tm_q, a.tm_k, a.tm_v, static_cast<__nv_bfloat16*>(a.o), a.lse, a.B, a.H, a.N, scale_log2,
      num_qtiles, a.status, kDefaultWaitTimeoutNs);
  return cudaGetLastError();
}

}  // namespace fwd

cudaError_t launch_fwd_sm100(const FwdArgs& a, cudaStream_t s) {
  if (a.d == 64) return a.causal ? fwd::launch_t<64, true>(a, s) : fwd::launch_t<64, false>(a, s);
  return a.causal ? fwd::launch_t<128, true>(a, s) : fwd::launch_t<128, false>(a, s);
}

}  // namespace fa
