// launch.h -- internal interface between the C ABI layer (api.cu) and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Default upper bound on any single in-kernel wait (nanoseconds).  A healthy kernel
// never waits anywhere near this long; hitting it means a pipeline stalled.
constexpr uint64_t kDefaultWaitTimeoutNs = 4000000000ull;

struct FwdArgs {
  CUtensorMap tm_q, tm_k, tm_v;  // 4-D maps over [B][N][H][d] bf16, box {64,1,128,1}
                                 // (8-bit path: E4M3 box {128,1,128,1}; tm_v over V^T
                                 // [B][H][d][Npad], box {128,128,1,1})
  CUtensorMap tm_o;               // 4-D map over the bf16 output [B][N][H][d], box {64,1,32,1}
  float* lse;
  const float* scales = nullptr;  // 8-bit path: [3][B*H] dequantisation scales
  const uint8_t* block_mask = nullptr;  // block-sparse: [ceil(N/128)][ceil(N/128)] bytes
  uint32_t* mask_words = nullptr;       // block-sparse: packed bitmasks (workspace)
  int B, H, N, d, causal;
  float scale;
  int* status;
  int num_sms;
};

struct BwdArgs {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // 4-D maps, box {64,1,128,1}
  CUtensorMap tm_dk, tm_dv;             // outputs, box {64,1,32,1} (one warp's rows)
  const void* o;
  const void* dO;
  const float* lse;
  void *dq, *dk, *dv;
  float* dq_acc;  // [B][H][N][d] fp32 workspace
  float* delta;   // [B][H][n_pad] fp32 workspace, n_pad = N rounded up to 128
  float* lse2;    // [B][H][n_pad] fp32 workspace: lse * log2(e)
  int B, H, N, d, causal;
  float scale;
  int* status;               // the call's word (workspace) or the library-owned one
  bool clear_status = false;  // the preprocess kernel clears *status (a workspace word)
  int num_sms;
};

struct SplitKvArgs {
  CUtensorMap tm_q, tm_k, tm_v;  // q over [B][Nq][H][d]; k, v over [B][Nk][H][d]
  void* o;                       // [B][Nq][H][d] bf16 or fp16
  float* lse;                    // [B][H][Nq]
  float* part_o;                 // [n_split][B*H][Nq][d] fp32 workspace
  float* part_lse;               // [n_split][B*H][Nq] fp32 workspace
  int B, H, Nq, Nk, d, causal, f16;
  int n_split, tiles_per_split;
  float scale;
  int* status;
};

cudaError_t launch_fwd_sm100(const FwdArgs& a, cudaStream_t s);
cudaError_t launch_fwd_fp8(const FwdArgs& a, cudaStream_t s);
cudaError_t launch_fwd_block_sparse(const FwdArgs& a, cudaStream_t s);

struct Fp8QuantArgs {
  const void *q, *k, *v;  // [B][N][H][d] bf16
  const float* signs;     // [d] +-1, or null (no transform)
  void *q8, *k8;          // [B][N][H][d] E4M3
  void* vt8;              // [B][H][d][Npad] E4M3, Npad = N rounded up to 16
  float* scales;          // [3][B*H]
  uint32_t* amax;         // [3][B*H] workspace
  int B, H, N, d;
};
cudaError_t launch_fp8_quantize(const Fp8QuantArgs& a, cudaStream_t s);
cudaError_t launch_fwd_splitkv(const SplitKvArgs& a, cudaStream_t s);
cudaError_t launch_bwd_pre(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_main(const BwdArgs& a, cudaStream_t s, bool with_dq);
cudaError_t launch_bwd_dq(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_convert(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int B, int H, int N, int d, int causal, float scale, cudaStream_t s);

// Debug / self-test kernels (fa_debug.h).
cudaError_t launch_debug_umma(const void* a, const void* b, float* c, int n, int k, int mode,
                              int* status, cudaStream_t s);
cudaError_t launch_debug_wait_timeout(uint64_t timeout_ns, int* status, cudaStream_t s);
cudaError_t launch_debug_tma_tile(const CUtensorMap& tm, void* y, int b, int h, int row0,
                                  int chunk, int* status, cudaStream_t s);
cudaError_t launch_debug_tmem_roundtrip(const uint32_t* in, uint32_t* out, int ncols,
                                        cudaStream_t s);
cudaError_t launch_debug_schedule(int B, int H, int N, int causal, int grid, int* out,
                                  int max_rounds, cudaStream_t s);
cudaError_t launch_debug_exp2(const float* x, float* y_poly, float* y_hw, int n, cudaStream_t s);

}  // namespace fa
