// bwd_dq_sm100.cu -- deterministic dQ for the backward pass on sm_100a.
//
// The main backward kernel accumulates dQ with fp32 reductions from many key/value tiles,
// whose arrival order (and so the rounding of the sum) varies from run to run.  This kernel
// produces dQ in a fixed order instead, so that the whole backward pass is bitwise
// repeatable, in keeping with the "exact and deterministic" claim of "FlashAttention-2 —
// FlashAttention-2" (section パフォーマンス).  Like the main kernel it never reads a stored P:
// it rebuilds S and P from the logsumexp ("Flash Attention 2で打破するローカルLLMの「メモリの
// 壁」", section タイリング（Tiling）と再計算（Recomputation）の仕組み).
//
// One CTA per (batch*head, 128-row query tile i); it walks the key/value tiles j that query
// tile i can see, in increasing j:
//   S    = Q_i K_j^T            (tcgen05, TMEM)
//   dP   = dO_i V_j^T           (tcgen05, TMEM)
//   dS   = P o (dP - D_i),  P = exp2(S*scale*log2e - lse2_i)   (thread = query row)
//   dQ_i += dS K_j              (tcgen05, A = dS packed bf16 in TMEM, fp32 accumulator)
// and writes dQ_i = scale * dQ_i in bf16.  Cost: the S and dP products are computed a second
// time (the main kernel computes them too), 1.4x the tensor work of the atomic variant.
//
// S has two TMEM buffers, used by key tiles in turn, so the S product of tile j+2 is issued
// as soon as dQ of tile j (which reads dS_j from the same columns) is: per key tile, in issue
// order, [ds_ready j] dP(j+1), dQ(j), S(j+2).  The compute warps then wait on one product
// (dP) between tiles instead of three, and the tensor core runs S ahead of them.  K is read
// by S(j) and, two issue steps later, dQ(j), so it has a three-stage ring; V, read by dP(j)
// only, two stages.
//
// CTA = 6 warps: 0-3 compute (thread t owns query row t = TMEM lane t), 4 TMA producer,
// 5 TMEM allocator + MMA issuer.  TMEM: S / dS buffer 0 [0,128), dP [128,256),
// dQ [256,256+D), S / dS buffer 1 [384,512).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"
#include "ptx.cuh"

namespace fa {
namespace bwd_dq {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // key rows per step
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColS1 = 384;
// TMEM column of S / dS buffer b (key tile j uses buffer j % 2).
__host__ __device__ constexpr uint32_t col_s(int b) { return b ? kColS1 : kColS; }

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kChunkBytes = 128 * 128;  // one TMA box: 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kKStages = 3;             // K ring (read two issue steps apart)
  static constexpr int kVStages = 2;             // V ring
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kOffQ + kTileBytes;
  static constexpr int kOffK = kOffDO + kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 256;  // base is 1024-aligned (checked)
  static_assert(kSmemBytes <= 232448, "more shared memory than a CTA can have");
};

struct Bars {
  uint64_t qd_full;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2];  // per S buffer: one phase per use, so it never runs ahead of its waiter
  uint64_t dp_full, ds_ready, dq_done, drain;
  uint32_t tmem_base;
  Abort abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block larger than its shared-memory region");

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const float* __restrict__ lse2, const float* __restrict__ delta,
                  __nv_bfloat16* __restrict__ dq, int B, int H, int N, int n_pad, float scale,
                  float scale_log2, int num_qtiles, int* status, uint64_t timeout_ns) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, FA_OK, FA_ERR_UNSUPPORTED);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Unit (b, h, query tile i); heads major; under the causal mask longest (largest i) first.
  const int bh = blockIdx.x / num_qtiles;
  int i = blockIdx.x % num_qtiles;
  if (CAUSAL) i = num_qtiles - 1 - i;
  const int b = bh / H, h = bh % H;
  const int q0 = i * BM;
  const int kv_total = (N + BN - 1) / BN;
  const int nkv = CAUSAL ? min(kv_total, i + 1) : kv_total;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qd_full, 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->ds_ready, BM);
    mbar_init(&bars->dq_done, 1);
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
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();
      mbar_arrive_expect_tx(&bars->qd_full, 2 * C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c) {
        tma_load_4d(sQ + c * C::kChunkBytes, &tm_q, &bars->qd_full, c * 64, h, q0, b, pol_q);
        tma_load_4d(sDO + c * C::kChunkBytes, &tm_do, &bars->qd_full, c * 64, h, q0, b, pol_q);
      }
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int sk = j % C::kKStages, sv = j % C::kVStages;
        if (j >= C::kKStages &&
            !mbar_wait(&bars->k_empty[sk], ((j / C::kKStages) - 1) & 1, ab, status, timeout_ns))
          break;
        mbar_arrive_expect_tx(&bars->k_full[sk], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sK + sk * C::kTileBytes + c * C::kChunkBytes, &tm_k, &bars->k_full[sk], c * 64,
                      h, j * BN, b, pol_kv);
        k_issued = j + 1;
        if (j >= C::kVStages &&
            !mbar_wait(&bars->v_empty[sv], ((j / C::kVStages) - 1) & 1, ab, status, timeout_ns))
          break;
        mbar_arrive_expect_tx(&bars->v_full[sv], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sV + sv * C::kTileBytes + c * C::kChunkBytes, &tm_v, &bars->v_full[sv], c * 64,
                      h, j * BN, b, pol_kv);
        v_issued = j + 1;
      }
      // Drain every copy into shared memory before the CTA may exit.
      Abort local{0};
      mbar_wait(&bars->qd_full, 0, &local, status, timeout_ns);
      for (int j = max(0, k_issued - C::kKStages); j < k_issued; ++j)
        mbar_wait(&bars->k_full[j % C::kKStages], (j / C::kKStages) & 1, &local, status, timeout_ns);
      for (int j = max(0, v_issued - C::kVStages); j < v_issued; ++j)
        mbar_wait(&bars->v_full[j % C::kVStages], (j / C::kVStages) & 1, &local, status, timeout_ns);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    // Prologue S(0), dP(0), S(1); then per key tile j: [ds_ready j] dP(j+1), dQ(j) += dS_j K_j,
    // S(j+2).  S(j+2) overwrites buffer j % 2 after dQ(j) has read dS_j from it, and dP(j+1)
    // overwrites dP_j after the compute warps have read it (ds_ready j): tcgen05 operations of
    // one thread run in order.
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(BM, BN, 0, 0);   // Q K^T, dO V^T (K-major)
      constexpr uint32_t id_dq = idesc_bf16_f32(BM, D, 0, 1);   // dS K (B MN-major)
      // Low descriptor words of the operand tiles read K-major; the K and V stages are offsets
      // from the first.  kdesc / mdesc: K-major / MN-major (LBO = one 64-column chunk).
      constexpr uint32_t kHi = sdesc_sw128_hi(1024);
      constexpr uint32_t kToMn = ((C::kChunkBytes >> 4) - 1u) << 16;
      const uint32_t xQ = sdesc_sw128_lo(smem_u32(sQ), 16), xDO = sdesc_sw128_lo(smem_u32(sDO), 16);
      const uint32_t xK0 = sdesc_sw128_lo(smem_u32(sK), 16), xV0 = sdesc_sw128_lo(smem_u32(sV), 16);
      auto kdesc = [](uint32_t x, uint32_t off) { return sdesc_join(x + (off >> 4), kHi); };
      auto mdesc = [](uint32_t x, uint32_t off) { return sdesc_join(x + (off >> 4) + kToMn, kHi); };
      auto issue_s = [&](int j) -> bool {
        const int sk = j % C::kKStages;
        if (!mbar_wait(&bars->k_full[sk], (j / C::kKStages) & 1, ab, status, timeout_ns)) return false;
        tc_fence_after();
        const uint32_t xk = xK0 + ((sk * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          umma_ss(tbase + col_s(j & 1), kdesc(xQ, off), kdesc(xk, off), id_s, kk > 0);
        }
        umma_commit(&bars->s_full[j & 1]);
        return true;
      };
      auto issue_dp = [&](int j) -> bool {
        const int sv = j % C::kVStages;
        if (!mbar_wait(&bars->v_full[sv], (j / C::kVStages) & 1, ab, status, timeout_ns)) return false;
        tc_fence_after();
        const uint32_t xv = xV0 + ((sv * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          umma_ss(tbase + kColDP, kdesc(xDO, off), kdesc(xv, off), id_s, kk > 0);
        }
        umma_commit(&bars->dp_full);
        umma_commit(&bars->v_empty[sv]);  // dP is V's only reader
        return true;
      };
      bool ok = mbar_wait(&bars->qd_full, 0, ab, status, timeout_ns) && issue_s(0) && issue_dp(0) &&
                (nkv < 2 || issue_s(1));
      for (int j = 0; ok && j < nkv; ++j) {
        if (!(ok = mbar_wait(&bars->ds_ready, j & 1, ab, status, timeout_ns))) break;
        tc_fence_after();
        if (j + 1 < nkv && !(ok = issue_dp(j + 1))) break;
        const int sk = j % C::kKStages;
        const uint32_t xk = xK0 + ((sk * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(tbase + kColDQ, tbase + col_s(j & 1) + kk * 8, mdesc(xk, kk * 2048), id_dq,
                  (j > 0 || kk > 0));
        umma_commit(&bars->k_empty[sk]);  // dQ(j) is K_j's last reader
        if (j + 2 < nkv && !(ok = issue_s(j + 2))) break;
      }
      umma_commit(&bars->dq_done);
      umma_commit(&bars->drain);
      Abort local{0};
      mbar_wait(&bars->drain, 0, &local, status, timeout_ns);
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const int t = threadIdx.x;  // query row within the tile == TMEM lane
    const int row = q0 + t;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    const size_t vec = static_cast<size_t>(bh) * n_pad + q0 + t;  // rows past N hold zeros
    const float l2 = lse2[vec];
    const float dd = delta[vec];
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, ab, status, timeout_ns));
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, j & 1, ab, status, timeout_ns));
      if (!ok) break;
      tc_fence_after();
      const int k0 = j * BN;
      const uint32_t colS = col_s(j & 1);
      const int lim = min(CAUSAL ? row : N - 1, N - 1) - k0;  // last visible key column
      const bool need_mask = lim < BN - 1;
      const bool masked = __any_sync(0xffffffffu, need_mask);
#pragma unroll
      for (int c32 = 0; c32 < BN / 32; ++c32) {
        uint32_t su[32], du[32];
        tmem_ld32(lane_base + colS + 32 * c32, su);
        tmem_ld32(lane_base + kColDP + 32 * c32, du);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p0 = ex2_approx(fmaf(__uint_as_float(su[e]), scale_log2, -l2));
          float p1 = ex2_approx(fmaf(__uint_as_float(su[e + 1]), scale_log2, -l2));
          if (masked) {
            if (32 * c32 + e > lim) p0 = 0.f;
            if (32 * c32 + e + 1 > lim) p1 = 0.f;
          }
          pk[e / 2] = pack_bf16x2(p0 * (__uint_as_float(du[e]) - dd),
                                  p1 * (__uint_as_float(du[e + 1]) - dd));
        }
        // dS (bf16 pairs) into columns [16 c32, 16 c32 + 16) of this tile's S buffer: inside
        // the S columns already read (this chunk or an earlier one).
        tmem_st16(lane_base + colS + 16 * c32, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->dq_done, 0, ab, status, timeout_ns));
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dst = dq + ((static_cast<size_t>(b) * N + row) * H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(lane_base + kColDQ + 32 * c, u);
        if (row < N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(
                pack_bf16x2(__uint_as_float(u[8 * v + 0]) * scale, __uint_as_float(u[8 * v + 1]) * scale),
                pack_bf16x2(__uint_as_float(u[8 * v + 2]) * scale, __uint_as_float(u[8 * v + 3]) * scale),
                pack_bf16x2(__uint_as_float(u[8 * v + 4]) * scale, __uint_as_float(u[8 * v + 5]) * scale),
                pack_bf16x2(__uint_as_float(u[8 * v + 6]) * scale, __uint_as_float(u[8 * v + 7]) * scale));
        }
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

template <int D, bool CAUSAL>
static cudaError_t launch_t(const BwdArgs& a, cudaStream_t st) {
  using C = Cfg<D>;
  auto kern = bwd_dq_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int n_pad = (a.N + 127) / 128 * 128;
  const int num_qtiles = (a.N + BM - 1) / BM;
  const long long grid = static_cast<long long>(a.B) * a.H * num_qtiles;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, st>>>(
      a.tm_q, a.tm_k, a.tm_v, a.tm_do, a.lse2, a.delta, static_cast<__nv_bfloat16*>(a.dq), a.B,
      a.H, a.N, n_pad, a.scale, a.scale * 1.4426950408889634f, num_qtiles, a.status,
      kDefaultWaitTimeoutNs);
  return cudaGetLastError();
}

}  // namespace bwd_dq

cudaError_t launch_bwd_dq(const BwdArgs& a, cudaStream_t s) {
  if (a.d == 64) return a.causal ? bwd_dq::launch_t<64, true>(a, s) : bwd_dq::launch_t<64, false>(a, s);
  return a.causal ? bwd_dq::launch_t<128, true>(a, s) : bwd_dq::launch_t<128, false>(a, s);
}

}  // namespace fa
