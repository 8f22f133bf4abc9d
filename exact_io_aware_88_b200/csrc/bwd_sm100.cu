// bwd_sm100.cu -- attention backward on sm_100a.
//
// The backward pass does not read a stored P: it rebuilds S and P tile by tile from the
// saved logsumexp, trading recomputation for memory traffic ("Flash Attention 2で打破する
// ローカルLLMの「メモリの壁」", section タイリング（Tiling）と再計算（Recomputation）の仕組み).
// Work is split along the key sequence (the second trick of "FlashAttention-2を読む",
// section GPUの稼働率を高める三つの工夫): one CTA owns a 128-row K/V tile and walks the
// query tiles that can see it.
//
// Three kernels, all on the caller's stream:
//  1. bwd_pre    D = rowsum(dO o O) (fp32) and lse2 = LSE*log2(e), both stored padded to a
//                multiple of 128 rows; clears the fp32 dQ accumulator.          (HBM-bound)
//  2. bwd_main   per (b, h, kv tile j), for each visible query tile i:
//                  S^T  = K_j Q_i^T          (tcgen05, TMEM)
//                  dP^T = V_j dO_i^T         (tcgen05, TMEM)
//                  P^T  = exp2(S^T*scale*log2e - lse2_i)       (compute warps; bf16 -> TMEM)
//                  dS^T = P^T o (dP^T - D_i)                  (compute warps; bf16 -> smem)
//                  dV_j += P^T dO_i,  dK_j += dS^T Q_i          (tcgen05, TMEM accumulators)
//                  dQ_i  = dS K_j  -> fp32 vector atomics into the accumulator (dQ warps)
//                epilogue: dK_j*scale, dV_j -> bf16.
//  3. dq_convert dq = bf16(scale * dQacc).                                     (HBM-bound)
//
// bwd_main CTA = 16 warps (4 warpgroups): 0-7 compute (two warpgroups, each owning half of
// the 128 query columns of a step; thread t of a warpgroup owns key row t = TMEM lane t),
// 8-11 dQ drain (thread owns query row = TMEM lane), 12 TMA producer, 13 TMEM allocator +
// MMA issuer, 14-15 idle.  setmaxnreg moves registers from the last warpgroup to the rest.
// TMEM (512 columns): dK [0,D), dV [D,2D), S^T/P^T [2D,2D+128), dP^T and then dQ
// [2D+128,2D+256).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "launch.h"
#include "ptx.cuh"

namespace fa {
namespace bwd {

constexpr int BM = 128;  // key rows per CTA tile (MMA M)
constexpr int BN = 128;  // query rows per step
constexpr int kThreads = 512;
// 16 warps = 4 warpgroups; sub-partition k runs warps k, k+4, k+8, k+12, one from each
// warpgroup.  Launch gives 128 registers to every thread (65536); after setmaxnreg each
// sub-partition holds 144 + 144 + 136 + 88 = 512 registers per lane (= 512 launched).
constexpr uint32_t kRegsLaunch = 65536 / kThreads;  // 128 (ptxas allocates this at launch)
constexpr uint32_t kRegsCompute = 144;
constexpr uint32_t kRegsDrain = 136;
constexpr uint32_t kRegsOther = 88;
static_assert(2 * kRegsCompute + kRegsDrain + kRegsOther <= 4 * kRegsLaunch,
              "register split exceeds what the block is launched with");
constexpr int kWarpLoad = 12;
constexpr int kWarpMma = 13;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kChunkBytes = 128 * 128;  // one TMA box: 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kQStages = 2;
  static constexpr int kDOStages = 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;
  static constexpr int kOffDO = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffDS = kOffDO + kDOStages * kTileBytes;  // dS^T: 2 chunks x 16 KB
  static constexpr int kOffVec = kOffDS + 2 * kChunkBytes;         // lse2 / D per q stage
  static constexpr int kVecBytes = kQStages * 2 * BN * 4;
  static constexpr int kOffBar = kOffVec + kVecBytes;
  // No alignment slack: the dynamic shared window starts 1024-byte aligned (checked at
  // run time; a misaligned base makes the kernel report FA_ERR_UNSUPPORTED and return).
  static constexpr int kSmemBytes = kOffBar + 256;
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = D;
  static constexpr uint32_t kColS = 2 * D;
  static constexpr uint32_t kColDP = 2 * D + 128;
};

struct Bars {
  uint64_t kv_full;
  uint64_t q_full[2], q_empty[2];
  uint64_t do_full[2], do_empty[2];
  uint64_t s_full, dp_full, p_ready, ds_ready, dq_full, dq_empty, dkdv_done, drain;
  uint32_t tmem_base;
  Abort abort;
  // End-of-CTA protocol check, each must equal the CTA's query-tile count: [0] Q tiles and
  // [1] dO tiles loaded, [2] MMA steps, [3 + h] compute warpgroup h's steps, [5] dQ drains.
  int count[6];
};
static_assert(sizeof(Bars) <= 256, "barrier block larger than its shared-memory region");

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// With head dim 128 the dQ tile is produced transposed (M = head dim), so that a warp's
// fp32 reductions into the accumulator cover 128 contiguous bytes of one query row: one
// L2 request per warp instruction instead of 32 scattered 16-byte pieces.  Head dim 64
// keeps M = 128 query rows (an M = 64 accumulator has a different TMEM layout).
template <int D>
constexpr bool kDqTransposed = (D == 128);

// TMEM column of the A operand (packed P^T) for K step kk of the dV product: compute
// warpgroup h stores its 64 query columns as 32 packed columns at [64h, 64h+32) of the
// S^T region, i.e. inside the S^T columns it has already read.
__device__ __forceinline__ uint32_t p_col(int kk) { return 64u * (kk >> 2) + 8u * (kk & 3); }

// WITH_DQ = false drops the dQ product and its drain (dQ then comes from the separate,
// deterministic per-query-tile kernel in bwd_dq_sm100.cu).
template <int D, bool CAUSAL, bool WITH_DQ>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const float* __restrict__ lse2, const float* __restrict__ delta,
                    float* __restrict__ dq_acc, int B, int H, int N, int n_pad,
                    float scale, float scale_log2, int num_kvtiles, int* status,
                    uint64_t timeout_ns) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // 128-byte-swizzled tiles need a 1024-aligned base
    if (threadIdx.x == 0) atomicCAS(status, FA_OK, FA_ERR_UNSUPPORTED);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit (b, h, kv tile j); heads major for L2 reuse of Q/dO; under the causal mask
  // low j (the most query tiles) first.
  const int bh = blockIdx.x / num_kvtiles;
  const int j = blockIdx.x % num_kvtiles;
  const int b = bh / H, h = bh % H;
  const int k0 = j * BM;
  const int nq_total = (N + BN - 1) / BN;
  const int i_begin = CAUSAL ? j : 0;
  const int nq = nq_total - i_begin;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->do_full[s], 1);
      mbar_init(&bars->do_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_ready, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_empty, 128);
    mbar_init(&bars->dkdv_done, 1);
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

  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sDS = smem + C::kOffDS;
  float* sVec = reinterpret_cast<float*>(smem + C::kOffVec);  // [stage][lse2 | D][128]
  const size_t vec_base = static_cast<size_t>(bh) * n_pad;
  const int wg = warp >> 2;

  // Role dispatch by warpgroup, so that each warpgroup executes its register
  // reallocation once, at one place, before its role's code.
  if (wg < 2) {
    regs_set<kRegsLaunch, kRegsCompute>();
    // ------------------------------------------------------------------ compute warps
    // Warpgroup `half` handles query columns [64*half, 64*half+64) of every step for key
    // row t (= TMEM lane t).
    const int half = wg;
    const int t = (warp & 3) * 32 + lane;
    const int key = k0 + t;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t colS = C::kColS + 64 * half;
    const uint32_t colDP = C::kColDP + 64 * half;
    bool ok = true;
    int steps_done = 0;
    for (int n = 0; n < nq; ++n) {
      const int i = i_begin + n;
      const int q0 = i * BN;
      const int sq = n % C::kQStages;
      const float4* gL = reinterpret_cast<const float4*>(sVec + sq * 2 * BN + 64 * half);
      const float4* gD = reinterpret_cast<const float4*>(sVec + sq * 2 * BN + BN + 64 * half);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, n & 1, ab, status, timeout_ns));
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->q_full[sq], (n / C::kQStages) & 1, ab, status,
                                             timeout_ns));
      if (!ok) break;
      tc_fence_after();
      // Phase 1: P^T = exp2(S^T * scale*log2e - lse2) -> packed bf16 into TMEM.
      // Column c (query q0 + c) is masked when it precedes the key (causal, diagonal
      // tiles) or lies past N; key rows past N are masked whole.
      const bool row_dead = key >= N;
      const int first_vis = (CAUSAL ? key - q0 : 0) - 64 * half;  // in this half's columns
      const int last_vis = N - 1 - q0 - 64 * half;
      float p[64];
      {
        uint32_t su[64];
        tmem_ld64(lane_base + colS, su);
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 l4 = gL[c / 4];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
            p[c + u] = ex2_approx(fmaf(__uint_as_float(su[c + u]), scale_log2, -lv[u]));
        }
        // Masks only where the tile needs them (diagonal or tail tiles; decided per warp so
        // the common, unmasked tiles pay nothing).
        const bool need_mask = row_dead || first_vis > 0 || last_vis < 63;
        if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (row_dead || c < first_vis || c > last_vis) p[c] = 0.f;
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
        tmem_st32(lane_base + colS, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_ready);
      // Phase 2: dS^T = P^T o (dP^T - D) -> bf16 into shared memory (swizzled rows).
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, n & 1, ab, status, timeout_ns));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c32 = 0; c32 < 2; ++c32) {
        uint32_t du[32];
        tmem_ld32(lane_base + colDP + 32 * c32, du);
        uint32_t dpk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int c = 32 * c32 + e;
          const float4 d4 = gD[c / 4];
          dpk[e / 2] = pack_bf16x2(p[c] * (__uint_as_float(du[e]) - d4.x),
                                   p[c + 1] * (__uint_as_float(du[e + 1]) - d4.y));
          dpk[e / 2 + 1] = pack_bf16x2(p[c + 2] * (__uint_as_float(du[e + 2]) - d4.z),
                                       p[c + 3] * (__uint_as_float(du[e + 3]) - d4.w));
        }
        // dS^T row t, query columns [64*half + 32*c32, +32): chunk `half`, 16-byte pieces
        // 4*c32 .. 4*c32+3.
        uint8_t* chunk = sDS + half * C::kChunkBytes;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc)
          *reinterpret_cast<uint4*>(chunk + sw128_offset(t, 4 * c32 + pc)) =
              make_uint4(dpk[4 * pc], dpk[4 * pc + 1], dpk[4 * pc + 2], dpk[4 * pc + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready);
      ++steps_done;
    }
    if ((warp & 3) == 0 && lane == 0) bars->count[3 + half] = steps_done;
    // ---------------------------------------------------------------- dK / dV epilogue
    // Warpgroup 0 writes dK (times scale), warpgroup 1 writes dV, as whole 128-byte lines:
    // each warp stages its 32 key rows in 128-byte-swizzled boxes of 64 head-dim elements in
    // the Q stages (free once dkdv_done has fired: every product has completed) and lane 0
    // hands them to TMA stores, which clip the rows past N.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->dkdv_done, 0, ab, status, timeout_ns));
    if (ok) {
      tc_fence_after();
      const uint32_t col = half == 0 ? C::kColDK : C::kColDV;
      const float mul = half == 0 ? scale : 1.f;
      uint8_t* stage = sQ + warp * (C::kChunks * 4096);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(lane_base + col + c * 32, u);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          *reinterpret_cast<uint4*>(stage + (c >> 1) * 4096 + sw128_offset(lane, (c & 1) * 4 + v4)) =
              make_uint4(
                  pack_bf16x2(__uint_as_float(u[8 * v4 + 0]) * mul, __uint_as_float(u[8 * v4 + 1]) * mul),
                  pack_bf16x2(__uint_as_float(u[8 * v4 + 2]) * mul, __uint_as_float(u[8 * v4 + 3]) * mul),
                  pack_bf16x2(__uint_as_float(u[8 * v4 + 4]) * mul, __uint_as_float(u[8 * v4 + 5]) * mul),
                  pack_bf16x2(__uint_as_float(u[8 * v4 + 6]) * mul, __uint_as_float(u[8 * v4 + 7]) * mul));
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int r0 = k0 + (warp & 3) * 32;
      if (lane == 0 && r0 < N) {
#pragma unroll
        for (int ch = 0; ch < C::kChunks; ++ch)
          tma_store_4d(half == 0 ? &tm_dk : &tm_dv, stage + ch * 4096, 64 * ch, h, r0, b);
        bulk_commit();
        bulk_wait_all();  // the stores have completed before the CTA's shared memory goes away
      }
    }
  } else if (wg == 2) {
    regs_set<kRegsLaunch, kRegsDrain>();
    // ------------------------------------------------------------------ dQ drain warps
    // Copy the dQ_i tile out of TMEM, hand the columns back, then reduce into the fp32
    // accumulator while the next tile's MMAs run.
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;  // query row within the tile
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    int drains = WITH_DQ ? 0 : nq;
    for (int n = 0; WITH_DQ && n < nq; ++n, ++drains) {
      const int q = (i_begin + n) * BN + r;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->dq_full, n & 1, ab, status, timeout_ns));
      if (!ok) break;
      tc_fence_after();
      if constexpr (kDqTransposed<D>) {
        // Thread = head-dim index dd; 32 query columns at a time.  Lanes of a warp hold 32
        // consecutive dd of one query row: each reduction is one 128-byte line.
        // The whole tile row is loaded first so the TMEM columns go back before any
        // reduction is issued.
        const int dd = r;
        const int q0 = (i_begin + n) * BN;
        float* dst = dq_acc + (static_cast<size_t>(bh) * N + q0) * D + dd;
        uint32_t u[BN];
#pragma unroll
        for (int c64 = 0; c64 < BN / 64; ++c64)
          tmem_ld64(lane_base + C::kColDP + 64 * c64, *reinterpret_cast<uint32_t(*)[64]>(&u[64 * c64]));
        tc_fence_before();
        mbar_arrive(&bars->dq_empty);
        const int cmax = min(BN, N - q0);  // query rows past N are dropped
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e < cmax) red_add_f32(dst + static_cast<size_t>(e) * D, __uint_as_float(u[e]));
      } else {
        // Thread = query row; 64 columns at a time; the TMEM columns are handed back after
        // the last load, before the last batch of reductions.
        float* dst = dq_acc + (static_cast<size_t>(bh) * N + q) * D;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t u[64];
          tmem_ld64(lane_base + C::kColDP + 64 * c, u);
          if (c == D / 64 - 1) {
            tc_fence_before();
            mbar_arrive(&bars->dq_empty);
          }
          if (q < N) {
#pragma unroll
            for (int v = 0; v < 16; ++v)
              red_add_v4(dst + 64 * c + 4 * v, __uint_as_float(u[4 * v]), __uint_as_float(u[4 * v + 1]),
                         __uint_as_float(u[4 * v + 2]), __uint_as_float(u[4 * v + 3]));
          }
        }
      }
    }
    if (warp == 8 && lane == 0) bars->count[5] = drains;
  } else {
    regs_set<kRegsLaunch, kRegsOther>();
    if (warp == kWarpLoad) {
      // ---------------------------------------------------------------- TMA producer
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_q = policy_evict_last();
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_4d(sK + c * C::kChunkBytes, &tm_k, &bars->kv_full, c * 64, h, k0, b, pol_kv);
          tma_load_4d(sV + c * C::kChunkBytes, &tm_v, &bars->kv_full, c * 64, h, k0, b, pol_kv);
        }
        int issued_q = 0, issued_do = 0;
        for (int n = 0; n < nq; ++n) {
          const int i = i_begin + n;
          const int sq = n % C::kQStages;
          if (n >= C::kQStages &&
              !mbar_wait(&bars->q_empty[sq], ((n / C::kQStages) - 1) & 1, ab, status, timeout_ns))
            break;
          mbar_arrive_expect_tx(&bars->q_full[sq], C::kTileBytes + 2 * BN * 4);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sQ + sq * C::kTileBytes + c * C::kChunkBytes, &tm_q, &bars->q_full[sq],
                        c * 64, h, i * BN, b, pol_q);
          bulk_load(sVec + sq * 2 * BN, lse2 + vec_base + i * BN, BN * 4, &bars->q_full[sq]);
          bulk_load(sVec + sq * 2 * BN + BN, delta + vec_base + i * BN, BN * 4, &bars->q_full[sq]);
          issued_q = n + 1;
          const int sd = n % C::kDOStages;
          if (n >= C::kDOStages &&
              !mbar_wait(&bars->do_empty[sd], ((n / C::kDOStages) - 1) & 1, ab, status, timeout_ns))
            break;
          mbar_arrive_expect_tx(&bars->do_full[sd], C::kTileBytes);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sDO + sd * C::kTileBytes + c * C::kChunkBytes, &tm_do, &bars->do_full[sd],
                        c * 64, h, i * BN, b, pol_q);
          issued_do = n + 1;
        }
        bars->count[0] = issued_q;
        bars->count[1] = issued_do;
        // Drain every copy into shared memory before the CTA may exit.
        Abort local{0};
        mbar_wait(&bars->kv_full, 0, &local, status, timeout_ns);
        for (int n = max(0, issued_q - C::kQStages); n < issued_q; ++n)
          mbar_wait(&bars->q_full[n % C::kQStages], (n / C::kQStages) & 1, &local, status,
                    timeout_ns);
        for (int n = max(0, issued_do - C::kDOStages); n < issued_do; ++n)
          mbar_wait(&bars->do_full[n % C::kDOStages], (n / C::kDOStages) & 1, &local, status,
                    timeout_ns);
      }
    } else if (warp == kWarpMma) {
      // ---------------------------------------------------------------- MMA issuer
      // Per query tile n (rows i = i_begin + n), in issue order:
      //   [p_ready n]  dV += P^T_n dO_n                 -> releases dO_n
      //                S^T_{n+1} = K Q_{n+1}^T (R1)      (P^T_n already consumed, in order)
      //   [ds_ready n] dQ_n = dS_n K (R2) ; dK += dS^T_n Q_n -> releases Q_n
      //   [dq_empty n] dP^T_{n+1} = V dO_{n+1}^T (R2)
      // so the next S^T and dV overlap the dS computation, and the dQ drain only gates dP.
      // (Splitting dK in halves around dP^T_{n+1}, so that the compute warps get dP^T sooner,
      // measured 10 % slower at N = 16k: the tensor pipe then idles while the drain warps
      // empty the dQ columns, which all of dK used to cover.)
      if (lane == 0) {
        constexpr uint32_t id_sdp = idesc_bf16_f32(BM, BN, 0, 0);  // K_j Q_i^T, V_j dO_i^T
        constexpr uint32_t id_dkdv = idesc_bf16_f32(BM, D, 0, 1);  // P^T dO_i, dS^T Q_i
        constexpr uint32_t id_dq = kDqTransposed<D>
                                       ? idesc_bf16_f32(D, BN, 1, 1)   // K_j^T dS^T
                                       : idesc_bf16_f32(BN, D, 1, 1);  // dS K_j
        // Low descriptor words of the operand tiles read K-major (rows of the head dim, or of
        // the query index for dS^T: LBO unused); the Q and dO stages are offsets from the
        // first.  kdesc(x, off) / mdesc(x, off) describe the operand `off` bytes into tile x
        // read K-major / MN-major (LBO = one 64-column chunk).
        constexpr uint32_t kHi = sdesc_sw128_hi(1024);
        constexpr uint32_t kToMn = ((C::kChunkBytes >> 4) - 1u) << 16;  // LBO 16 -> chunk
        const uint32_t xK = sdesc_sw128_lo(smem_u32(sK), 16);
        const uint32_t xV = sdesc_sw128_lo(smem_u32(sV), 16);
        const uint32_t xQ0 = sdesc_sw128_lo(smem_u32(sQ), 16);
        const uint32_t xDO0 = sdesc_sw128_lo(smem_u32(sDO), 16);
        const uint32_t xDS = sdesc_sw128_lo(smem_u32(sDS), 16);
        auto kdesc = [](uint32_t x, uint32_t off) { return sdesc_join(x + (off >> 4), kHi); };
        auto mdesc = [](uint32_t x, uint32_t off) { return sdesc_join(x + (off >> 4) + kToMn, kHi); };
        auto issue_s = [&](int n) -> bool {  // S^T_n = K_j Q_n^T (K-major over the head dim)
          const int sq = n % C::kQStages;
          if (!mbar_wait(&bars->q_full[sq], (n / C::kQStages) & 1, ab, status, timeout_ns))
            return false;
          tc_fence_after();
          const uint32_t qd = xQ0 + ((sq * C::kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
            umma_ss(tbase + C::kColS, kdesc(xK, off), kdesc(qd, off), id_sdp, kk > 0);
          }
          umma_commit(&bars->s_full);
          return true;
        };
        auto issue_dp = [&](int n) -> bool {  // dP^T_n = V_j dO_n^T
          const int sd = n % C::kDOStages;
          if (!mbar_wait(&bars->do_full[sd], (n / C::kDOStages) & 1, ab, status, timeout_ns))
            return false;
          if (WITH_DQ && n > 0 && !mbar_wait(&bars->dq_empty, (n - 1) & 1, ab, status, timeout_ns))
            return false;
          tc_fence_after();
          const uint32_t dod = xDO0 + ((sd * C::kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
            umma_ss(tbase + C::kColDP, kdesc(xV, off), kdesc(dod, off), id_sdp, kk > 0);
          }
          umma_commit(&bars->dp_full);
          return true;
        };
        bool ok = mbar_wait(&bars->kv_full, 0, ab, status, timeout_ns) && issue_s(0) && issue_dp(0);
        int mma_steps = 0;
        for (int n = 0; ok && n < nq; ++n) {
          const int sq = n % C::kQStages, sd = n % C::kDOStages;
          const uint32_t xq = xQ0 + ((sq * C::kTileBytes) >> 4);
          const uint32_t xdo = xDO0 + ((sd * C::kTileBytes) >> 4);
          if (!mbar_wait(&bars->p_ready, n & 1, ab, status, timeout_ns)) break;
          tc_fence_after();
          // dV_j += P^T dO_i   (A = P^T from TMEM, B = dO_i MN-major over the query index)
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_ts(tbase + C::kColDV, tbase + C::kColS + p_col(kk),
                    mdesc(xdo, kk * 2048), id_dkdv, (n > 0 || kk > 0));
          umma_commit(&bars->do_empty[sd]);
          if (n + 1 < nq && !issue_s(n + 1)) break;
          if (!mbar_wait(&bars->ds_ready, n & 1, ab, status, timeout_ns)) break;
          tc_fence_after();
          // dQ first: only its drain gates the next dP^T, so dK runs on the tensor pipe
          // while the drain warps empty the dQ columns.
          if constexpr (!WITH_DQ) {
          } else if constexpr (kDqTransposed<D>) {
            // dQ_i^T = K_j^T dS^T   (A = K_j read MN-major over the head dim, B = dS^T
            // MN-major over the query index): TMEM lane = head-dim index, column = query.
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ss(tbase + C::kColDP, mdesc(xK, kk * 2048), mdesc(xDS, kk * 2048), id_dq, kk > 0);
          } else {
            // dQ_i = dS K_j   (A = dS: the dS^T tile read MN-major; B = K_j MN-major)
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ss(tbase + C::kColDP, mdesc(xDS, kk * 2048), mdesc(xK, kk * 2048), id_dq, kk > 0);
          }
          if constexpr (WITH_DQ) umma_commit(&bars->dq_full);
          // dK_j += dS^T Q_i   (A = dS^T K-major over the query index, B = Q_i MN-major)
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
            umma_ss(tbase + C::kColDK, kdesc(xDS, aoff), mdesc(xq, kk * 2048), id_dkdv,
                    (n > 0 || kk > 0));
          }
          umma_commit(&bars->q_empty[sq]);
          ++mma_steps;
          if (n + 1 < nq && !issue_dp(n + 1)) break;
        }
        bars->count[2] = mma_steps;
        umma_commit(&bars->dkdv_done);
        umma_commit(&bars->drain);
        Abort local{0};
        mbar_wait(&bars->drain, 0, &local, status, timeout_ns);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Every role must have done one step per query tile (skipped after a timed-out wait).
  if (threadIdx.x == 0 && !*reinterpret_cast<volatile int*>(&ab->flag)) {
    bool agree = true;
#pragma unroll
    for (int i = 0; i < 6; ++i) agree = agree && bars->count[i] == nq;
    if (!agree) atomicCAS(status, FA_OK, FA_ERR_INTERNAL);
  }
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// D[bh][n] = sum_c dO[b,n,h,c] * O[b,n,h,c];  lse2[bh][n] = lse[bh][n] * log2(e);  zero rows
// n in [N, n_pad); dQacc = 0.  Threads per row: D/8 (one 16-byte vector each).
template <int D>
__global__ void __launch_bounds__(256)
    bwd_pre_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                   const float* __restrict__ lse, float* __restrict__ delta,
                   float* __restrict__ lse2, float* __restrict__ dq_acc, int B, int H, int N,
                   int n_pad, long long acc_vec4, int row_blocks, int* clear_status) {
  constexpr int kTPR = D / 8;           // threads per row
  constexpr int kRowsPerBlock = 256 / kTPR;
  // The call's own status word (in its workspace) starts out clear; the kernels after this
  // one in the stream record their failures into it.
  if (clear_status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *clear_status = FA_OK;
  if (static_cast<int>(blockIdx.x) < row_blocks) {
    const long long rows = static_cast<long long>(B) * N * H;  // rows in memory order (b, n, h)
    const long long row = static_cast<long long>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kTPR;
    const int part = threadIdx.x % kTPR;
    float acc = 0.f;
    if (row < rows) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
      const uint4 g = *reinterpret_cast<const uint4*>(dO + row * D + part * 8);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(a2[e]);
        const float2 fg = __bfloat1622float2(g2[e]);
        acc = fmaf(fa.x, fg.x, acc);
        acc = fmaf(fa.y, fg.y, acc);
      }
    }
#pragma unroll
    for (int off = kTPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (row < rows && part == 0) {
      const int h = static_cast<int>(row % H);
      const long long bn = row / H;
      const int n = static_cast<int>(bn % N);
      const int b = static_cast<int>(bn / N);
      const size_t bhn = (static_cast<size_t>(b) * H + h);
      delta[bhn * n_pad + n] = acc;
      lse2[bhn * n_pad + n] = lse[bhn * N + n] * kLog2e;
    }
    // Padding rows [N, n_pad) of every (b, h): written by the first blocks.
    const long long pad_rows = static_cast<long long>(B) * H * (n_pad - N);
    for (long long p = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; p < pad_rows;
         p += static_cast<long long>(row_blocks) * 256) {
      const long long bhi = p / (n_pad - N);
      const int n = N + static_cast<int>(p % (n_pad - N));
      delta[bhi * n_pad + n] = 0.f;
      lse2[bhi * n_pad + n] = 0.f;
    }
  } else {
    // Zero the dQ accumulator.
    const long long nblk = static_cast<long long>(gridDim.x) - row_blocks;
    float4* acc4 = reinterpret_cast<float4*>(dq_acc);
    for (long long p = (static_cast<long long>(blockIdx.x) - row_blocks) * 256 + threadIdx.x;
         p < acc_vec4; p += nblk * 256)
      acc4[p] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dq[b][n][h][:] = bf16(scale * dQacc[b][h][n][:]).  One thread per 8 output elements.
template <int D>
__global__ void __launch_bounds__(256)
    dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, int B,
                      int H, int N, float scale) {
  constexpr int kTPR = D / 8;
  const long long rows = static_cast<long long>(B) * N * H;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gid / kTPR;
  const int part = static_cast<int>(gid % kTPR);
  if (row >= rows) return;
  const int h = static_cast<int>(row % H);
  const long long bn = row / H;
  const int n = static_cast<int>(bn % N);
  const long long b = bn / N;
  const float4* src = reinterpret_cast<const float4*>(
      dq_acc + ((static_cast<size_t>(b) * H + h) * N + n) * D + part * 8);
  const float4 x = src[0], y = src[1];
  *reinterpret_cast<uint4*>(dq + row * D + part * 8) =
      make_uint4(pack_bf16x2(x.x * scale, x.y * scale), pack_bf16x2(x.z * scale, x.w * scale),
                 pack_bf16x2(y.x * scale, y.y * scale), pack_bf16x2(y.z * scale, y.w * scale));
}

template <int D>
static cudaError_t launch_pre_t(const BwdArgs& a, cudaStream_t st) {
  const int n_pad = (a.N + 127) / 128 * 128;
  const size_t rows = static_cast<size_t>(a.B) * a.H * a.N;
  constexpr int kRowsPerBlock = 256 / (D / 8);
  const long long row_blocks = (static_cast<long long>(rows) + kRowsPerBlock - 1) / kRowsPerBlock;
  const long long acc_vec4 = static_cast<long long>(rows) * D / 4;
  const long long zero_blocks = std::min<long long>((acc_vec4 + 255) / 256, 8LL * a.num_sms);
  const long long grid = row_blocks + zero_blocks;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  bwd_pre_kernel<D><<<static_cast<unsigned>(grid), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dO), a.lse,
      a.delta, a.lse2, a.dq_acc, a.B, a.H, a.N, n_pad, acc_vec4, static_cast<int>(row_blocks),
      a.clear_status ? a.status : nullptr);
  return cudaGetLastError();
}

template <int D, bool CAUSAL, bool WITH_DQ>
static cudaError_t launch_main_t(const BwdArgs& a, cudaStream_t st) {
  using C = Cfg<D>;
  const int n_pad = (a.N + 127) / 128 * 128;
  auto kern = bwd_main_kernel<D, CAUSAL, WITH_DQ>;
  // The setmaxnreg split assumes the kernel launches with exactly kRegsLaunch registers per
  // thread; with fewer, the increasing warpgroups could never be satisfied.
  cudaFuncAttributes fa_attr;
  cudaError_t e = cudaFuncGetAttributes(&fa_attr, kern);
  if (e != cudaSuccess) return e;
  if (fa_attr.numRegs != static_cast<int>(kRegsLaunch)) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int num_kvtiles = (a.N + BM - 1) / BM;
  const long long grid = static_cast<long long>(a.B) * a.H * num_kvtiles;
  kern<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, st>>>(
      a.tm_q, a.tm_k, a.tm_v, a.tm_do, a.tm_dk, a.tm_dv, a.lse2, a.delta, a.dq_acc, a.B, a.H, a.N, n_pad,
      a.scale, a.scale * kLog2e, num_kvtiles, a.status, kDefaultWaitTimeoutNs);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_convert_t(const BwdArgs& a, cudaStream_t st) {
  const size_t rows = static_cast<size_t>(a.B) * a.H * a.N;
  const long long threads = static_cast<long long>(rows) * (D / 8);
  const long long grid = (threads + 255) / 256;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dq_convert_kernel<D><<<static_cast<unsigned>(grid), 256, 0, st>>>(
      a.dq_acc, static_cast<__nv_bfloat16*>(a.dq), a.B, a.H, a.N, a.scale);
  return cudaGetLastError();
}

}  // namespace bwd

cudaError_t launch_bwd_pre(const BwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? bwd::launch_pre_t<64>(a, s) : bwd::launch_pre_t<128>(a, s);
}

cudaError_t launch_bwd_main(const BwdArgs& a, cudaStream_t s, bool with_dq) {
  if (with_dq) {
    if (a.d == 64)
      return a.causal ? bwd::launch_main_t<64, true, true>(a, s)
                      : bwd::launch_main_t<64, false, true>(a, s);
    return a.causal ? bwd::launch_main_t<128, true, true>(a, s)
                    : bwd::launch_main_t<128, false, true>(a, s);
  }
  if (a.d == 64)
    return a.causal ? bwd::launch_main_t<64, true, false>(a, s)
                    : bwd::launch_main_t<64, false, false>(a, s);
  return a.causal ? bwd::launch_main_t<128, true, false>(a, s)
                  : bwd::launch_main_t<128, false, false>(a, s);
}

cudaError_t launch_bwd_convert(const BwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? bwd::launch_convert_t<64>(a, s) : bwd::launch_convert_t<128>(a, s);
}

}  // namespace fa
