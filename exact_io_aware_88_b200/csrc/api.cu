// api.cu -- the C ABI (include/fa.h, include/fa_debug.h): argument validation, TMA
// descriptor encoding, device status word, and dispatch to the kernels.  No entry point
// allocates device memory, synchronises (except fa_read_device_status) or throws.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "fa.h"
#include "fa_debug.h"
#include "launch.h"

namespace {

// Library-owned device status word (FA_OK / FA_ERR_TIMEOUT / FA_ERR_INTERNAL); one per
// device context.
__device__ int g_fa_status = 0;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool sm100 = false;
  int num_sms = 0;
  int* status = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Looks up (once per device) the SM count, whether it is an sm_100 part and the device
// address of the status word; also resolves cuTensorMapEncodeTiled through the runtime so
// that the library needs no link-time dependency on libcuda.
int device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_status) != cudaSuccess) return FA_ERR_CUDA;
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FA_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.sm100 = (major == 10 && minor == 0);
    d.num_sms = sms;
    d.status = static_cast<int*>(p);
    d.ready = true;
  }
  *out = d;
  return d.sm100 ? FA_OK : FA_ERR_UNSUPPORTED;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by the bf16 entry points.  Returns FA_OK or an error code.
int check_shape(int B, int H, int N, int d, float scale) {
  if (B < 1 || H < 1 || N < 1 || !(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
  const long double elems = static_cast<long double>(B) * N * H * d;
  if (elems > 9.0e15L) return FA_ERR_INVALID_ARG;
  const long long tiles = static_cast<long long>(B) * H * ((N + 127) / 128);
  if (tiles > 0x7fffffffLL || N > 0x7fffff80) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// 4-D view [B][N][H][d] (innermost first: d, H, N, B) of a bf16 tensor, tiled in boxes of
// 64 d-elements (128 bytes, the 128-byte swizzle span) x 1 head x 128 rows x 1 batch.
// 8-bit tensors (E4M3 codes as UINT8) use boxes of 128 d-elements, again 128 bytes.
// `box_rows` rows per box (128; the forward's output map uses 32, one warp's rows).
int encode_bnhd(CUtensorMap* m, const void* ptr, int B, int N, int H, int d,
                CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, int box_rows = 128) {
  const cuuint64_t es = (dt == CU_TENSOR_MAP_DATA_TYPE_UINT8) ? 1 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * es,
                                 static_cast<cuuint64_t>(H) * d * es,
                                 static_cast<cuuint64_t>(N) * H * d * es};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / es), 1,
                             static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, dt, 4, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// 4-D view of an 8-bit V^T [B][H][d][npad] (innermost first: keys, d, H, B), boxes of 128
// keys (128 bytes) x 128 head-dim rows.
int encode_vt8(CUtensorMap* m, const void* ptr, int B, int H, int d, int npad) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(npad), static_cast<cuuint64_t>(d),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(npad),
                                 static_cast<cuuint64_t>(d) * npad,
                                 static_cast<cuuint64_t>(H) * d * npad};
  const cuuint32_t box[4] = {128, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return FA_OK;
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return FA_ERR_CUDA;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// A backward workspace starts with the call's status word, in a slot that keeps the parts
// after it 256-byte aligned.
constexpr size_t kBwdStatusSlot = 256;

// Split-KV plan.  The split kernel runs one CTA per SM (it holds all of TMEM and most of
// shared memory), and each unit (query tile, key slice) pays a fixed cost (launch, Q load,
// pipeline fill, partial write) of roughly five key tiles' worth of streaming.  So the plan
// picks the number of slices n (at most 64, never more than the key tiles) that minimises
//   rounds(n) * (tiles per slice + 5),  rounds = ceil(units / 148),
// the time of the busiest SM; ties go to fewer slices (less merging).  Planned for the 148
// SMs of a B200 whatever the device, so the workspace size depends on the problem only.
constexpr long long kSplitSlots = 148;
constexpr long long kSplitUnitCost = 5;  // fixed cost of a unit, in key tiles
void splitkv_plan(int B, int H, int Nq, int Nk, int* n_split, int* tiles_per_split) {
  const long long kv_tiles = (Nk + 127) / 128;
  const long long base = static_cast<long long>(B) * H * ((Nq + 127) / 128);
  long long best_cost = -1, best_tps = kv_tiles;
  for (long long n = 1; n <= std::min(kv_tiles, 64LL); ++n) {
    const long long tps = (kv_tiles + n - 1) / n;
    const long long ns = (kv_tiles + tps - 1) / tps;  // slices actually used
    const long long rounds = (base * ns + kSplitSlots - 1) / kSplitSlots;
    const long long cost = rounds * (tps + kSplitUnitCost);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_tps = tps;
    }
  }
  *tiles_per_split = static_cast<int>(best_tps);
  *n_split = static_cast<int>((kv_tiles + best_tps - 1) / best_tps);
}

int check_splitkv(int B, int H, int Nq, int Nk, int d, int causal, float scale) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || !(scale > 0.f) || !isfinite(scale))
    return FA_ERR_INVALID_ARG;
  if (causal && Nq > Nk) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long double>(B) * std::max(Nq, Nk) * H * d > 9.0e15L) return FA_ERR_INVALID_ARG;
  const long long units = static_cast<long long>(B) * H * ((Nq + 127) / 128) * 64;
  if (units > 0x7fffffffLL || Nk > 0x7fffff80) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

}  // namespace

extern "C" {

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported (head dim or device)";
    case FA_ERR_MISALIGNED: return "misaligned pointer";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device-side wait timed out";
    case FA_ERR_INTERNAL: return "internal consistency check failed (library defect)";
    default: return "unknown status";
  }
}

int fa_version(void) { return 100; }

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int rc = check_shape(B, H, N, d, scale);
  if (rc) return rc;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4))
    return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  fa::FwdArgs a;
  if ((rc = encode_bnhd(&a.tm_q, q, B, N, H, d)) || (rc = encode_bnhd(&a.tm_k, k, B, N, H, d)) ||
      (rc = encode_bnhd(&a.tm_v, v, B, N, H, d)) ||
      (rc = encode_bnhd(&a.tm_o, o, B, N, H, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32)))
    return rc;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.status = di.status;
  a.num_sms = di.num_sms;
  return from_cuda(fa::launch_fwd_sm100(a, static_cast<cudaStream_t>(stream)));
}

size_t fa_fp8_quantize_workspace_bytes(int B, int H) {
  if (B < 1 || H < 1 || static_cast<long long>(B) * H > 0x7fffffffLL / 3) return 0;
  return round_up(3 * sizeof(uint32_t) * static_cast<size_t>(B) * H, 256);
}

int fa_fp8_quantize(const void* q, const void* k, const void* v, const float* signs, void* q8,
                    void* k8, void* vt8, float* scales, int B, int H, int N, int d,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !q8 || !k8 || !vt8 || !scales) return FA_ERR_INVALID_ARG;
  int rc = check_shape(B, H, N, d, 1.0f);
  if (rc) return rc;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q8, 16) ||
      !aligned(k8, 16) || !aligned(vt8, 16) || !aligned(scales, 4) ||
      (signs && !aligned(signs, 4)))
    return FA_ERR_MISALIGNED;
  const size_t need = fa_fp8_quantize_workspace_bytes(B, H);
  if (!workspace || need == 0 || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 4)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  fa::Fp8QuantArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.signs = signs;
  a.q8 = q8;
  a.k8 = k8;
  a.vt8 = vt8;
  a.scales = scales;
  a.amax = static_cast<uint32_t*>(workspace);
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  return from_cuda(fa::launch_fp8_quantize(a, static_cast<cudaStream_t>(stream)));
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* scales, void* o,
               float* lse, int B, int H, int N, int d, int causal, float scale, void* stream) {
  if (!q8 || !k8 || !vt8 || !scales || !o || !lse) return FA_ERR_INVALID_ARG;
  int rc = check_shape(B, H, N, d, scale);
  if (rc) return rc;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(vt8, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(scales, 4))
    return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  fa::FwdArgs a;
  const int npad = (N + 15) / 16 * 16;
  if ((rc = encode_bnhd(&a.tm_q, q8, B, N, H, d, CU_TENSOR_MAP_DATA_TYPE_UINT8)) ||
      (rc = encode_bnhd(&a.tm_k, k8, B, N, H, d, CU_TENSOR_MAP_DATA_TYPE_UINT8)) ||
      (rc = encode_vt8(&a.tm_v, vt8, B, H, d, npad)) ||
      (rc = encode_bnhd(&a.tm_o, o, B, N, H, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32)))
    return rc;
  a.lse = lse;
  a.scales = scales;
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.status = di.status;
  a.num_sms = di.num_sms;
  return from_cuda(fa::launch_fwd_fp8(a, static_cast<cudaStream_t>(stream)));
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 1.0f) != FA_OK || d < 1) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  const size_t padded = static_cast<size_t>(B) * H * ((static_cast<size_t>(N) + 127) / 128 * 128);
  return kBwdStatusSlot + round_up(rows * d * sizeof(float), 256) +
         2 * round_up(padded * sizeof(float), 256);
}

}  // extern "C"

namespace {

enum BwdStage { kStagePre = 1, kStageMain = 2, kStageConvert = 4 };

// Validates the arguments the requested stages use and fills `a`.  Pointers a stage does
// not use may be null.  With `own_status` the kernels record failures in the workspace's
// status word (cleared by the preprocess kernel), else in the library-owned word.
int bwd_prepare(int stages, const void* q, const void* k, const void* v, const void* o,
                const float* lse, const void* dO, void* dq, void* dk, void* dv, int B, int H,
                int N, int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                fa::BwdArgs* a, bool own_status = true) {
  const bool pre = stages & kStagePre, mid = stages & kStageMain, cvt = stages & kStageConvert;
  if ((pre && (!o || !lse || !dO)) || (mid && (!q || !k || !v || !dO || !dk || !dv)) ||
      (cvt && !dq))
    return FA_ERR_INVALID_ARG;
  int rc = check_shape(B, H, N, d, scale);
  if (rc) return rc;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if ((pre && (!aligned(o, 16) || !aligned(dO, 16) || !aligned(lse, 16))) ||
      (mid && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dO, 16) ||
               !aligned(dk, 16) || !aligned(dv, 16))) ||
      (cvt && !aligned(dq, 16)))
    return FA_ERR_MISALIGNED;
  const size_t need = fa_bwd_workspace_bytes(B, H, N, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  if (mid && ((rc = encode_bnhd(&a->tm_q, q, B, N, H, d)) ||
              (rc = encode_bnhd(&a->tm_k, k, B, N, H, d)) ||
              (rc = encode_bnhd(&a->tm_v, v, B, N, H, d)) ||
              (rc = encode_bnhd(&a->tm_do, dO, B, N, H, d)) ||
              (rc = encode_bnhd(&a->tm_dk, dk, B, N, H, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32)) ||
              (rc = encode_bnhd(&a->tm_dv, dv, B, N, H, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32))))
    return rc;
  const size_t rows = static_cast<size_t>(B) * H * N;
  const size_t padded = static_cast<size_t>(B) * H * ((static_cast<size_t>(N) + 127) / 128 * 128);
  char* const ws0 = static_cast<char*>(workspace);
  char* ws = ws0 + kBwdStatusSlot;
  a->o = o;
  a->dO = dO;
  a->lse = lse;
  a->dq = dq;
  a->dk = dk;
  a->dv = dv;
  a->dq_acc = reinterpret_cast<float*>(ws);
  a->delta = reinterpret_cast<float*>(ws + round_up(rows * d * sizeof(float), 256));
  a->lse2 = reinterpret_cast<float*>(ws + round_up(rows * d * sizeof(float), 256) +
                                     round_up(padded * sizeof(float), 256));
  a->B = B;
  a->H = H;
  a->N = N;
  a->d = d;
  a->causal = causal ? 1 : 0;
  a->scale = scale;
  a->status = own_status ? reinterpret_cast<int*>(ws0) : di.status;
  a->clear_status = own_status;
  a->num_sms = di.num_sms;
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal,
           float scale, void* workspace, size_t workspace_bytes, void* stream) {
  fa::BwdArgs a;
  int rc = bwd_prepare(kStagePre | kStageMain | kStageConvert, q, k, v, o, lse, dO, dq, dk, dv, B,
                       H, N, d, causal, scale, workspace, workspace_bytes, &a);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = from_cuda(fa::launch_bwd_pre(a, st)))) return rc;
  if ((rc = from_cuda(fa::launch_bwd_main(a, st, true)))) return rc;
  return from_cuda(fa::launch_bwd_convert(a, st));
}

int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, int causal, float scale, void* workspace,
                         size_t workspace_bytes, void* stream) {
  fa::BwdArgs a;
  int rc = bwd_prepare(kStagePre | kStageMain | kStageConvert, q, k, v, o, lse, dO, dq, dk, dv, B,
                       H, N, d, causal, scale, workspace, workspace_bytes, &a);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = from_cuda(fa::launch_bwd_pre(a, st)))) return rc;
  if ((rc = from_cuda(fa::launch_bwd_main(a, st, false)))) return rc;
  return from_cuda(fa::launch_bwd_dq(a, st));
}

int fa_bwd_preprocess(const void* o, const float* lse, const void* dO, int B, int H, int N, int d,
                      void* workspace, size_t workspace_bytes, void* stream) {
  fa::BwdArgs a;
  int rc = bwd_prepare(kStagePre, nullptr, nullptr, nullptr, o, lse, dO, nullptr, nullptr, nullptr,
                       B, H, N, d, 0, 1.0f, workspace, workspace_bytes, &a);
  if (rc) return rc;
  return from_cuda(fa::launch_bwd_pre(a, static_cast<cudaStream_t>(stream)));
}

int fa_bwd_kv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
              int B, int H, int N, int d, int causal, float scale, void* workspace,
              size_t workspace_bytes, void* stream) {
  fa::BwdArgs a;
  int rc = bwd_prepare(kStageMain, q, k, v, nullptr, nullptr, dO, nullptr, dk, dv, B, H, N, d,
                       causal, scale, workspace, workspace_bytes, &a);
  if (rc) return rc;
  return from_cuda(fa::launch_bwd_main(a, static_cast<cudaStream_t>(stream), true));
}

int fa_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, void* workspace,
                      size_t workspace_bytes, void* stream) {
  fa::BwdArgs a;
  int rc = bwd_prepare(kStageConvert, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dq,
                       nullptr, nullptr, B, H, N, d, 0, scale, workspace, workspace_bytes, &a);
  if (rc) return rc;
  return from_cuda(fa::launch_bwd_convert(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Workspace of fa_bwd_noalloc: a fixed device array, one per GPU that loads the library.
// Host code cannot use the symbol as a device address; its address is looked up once
// per device (below) and handed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_workspace[FA_NOALLOC_WORKSPACE_BYTES];
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_workspace on the current device (set-up on first use).
int noalloc_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess || p == nullptr)
      return FA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   int causal, float scale, void* stream) {
  // Reject bad or oversized problems before touching the device.
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int rc = check_shape(B, H, N, d, scale);
  if (rc) return rc;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (fa_bwd_workspace_bytes(B, H, N, d) > FA_NOALLOC_WORKSPACE_BYTES) return FA_ERR_WORKSPACE;
  void* ws = nullptr;
  if ((rc = noalloc_workspace(&ws))) return rc;
  fa::BwdArgs a;
  rc = bwd_prepare(kStagePre | kStageMain | kStageConvert, q, k, v, o, lse, dO, dq, dk, dv, B, H,
                   N, d, causal, scale, ws, FA_NOALLOC_WORKSPACE_BYTES, &a,
                   /*own_status=*/false);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = from_cuda(fa::launch_bwd_pre(a, st)))) return rc;
  if ((rc = from_cuda(fa::launch_bwd_main(a, st, true)))) return rc;
  return from_cuda(fa::launch_bwd_convert(a, st));
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d) {
  if (check_splitkv(B, H, Nq, Nk, d, 0, 1.0f) != FA_OK) return 0;
  int n_split = 1, tps = 1;
  splitkv_plan(B, H, Nq, Nk, &n_split, &tps);
  const size_t rows = static_cast<size_t>(n_split) * B * H * Nq;
  return round_up(rows * d * sizeof(float), 256) + round_up(rows * sizeof(float), 256);
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int Nq, int Nk, int d, int causal, float scale, int dtype, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int rc = check_splitkv(B, H, Nq, Nk, d, causal, scale);
  if (rc) return rc;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_MISALIGNED;
  const size_t need = fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  fa::SplitKvArgs a;
  const CUtensorMapDataType dt =
      dtype == FA_DTYPE_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if ((rc = encode_bnhd(&a.tm_q, q, B, Nq, H, d, dt)) ||
      (rc = encode_bnhd(&a.tm_k, k, B, Nk, H, d, dt)) ||
      (rc = encode_bnhd(&a.tm_v, v, B, Nk, H, d, dt)))
    return rc;
  splitkv_plan(B, H, Nq, Nk, &a.n_split, &a.tiles_per_split);
  const size_t rows = static_cast<size_t>(a.n_split) * B * H * Nq;
  char* ws = static_cast<char*>(workspace);
  a.part_o = reinterpret_cast<float*>(ws);
  a.part_lse = reinterpret_cast<float*>(ws + round_up(rows * d * sizeof(float), 256));
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.Nq = Nq;
  a.Nk = Nk;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.f16 = dtype == FA_DTYPE_FP16 ? 1 : 0;
  a.scale = scale;
  a.status = di.status;
  return from_cuda(fa::launch_fwd_splitkv(a, static_cast<cudaStream_t>(stream)));
}

size_t fa_fwd_block_sparse_workspace_bytes(int B, int H, int N, int d) {
  (void)B;
  (void)H;
  (void)d;
  if (N < 1) return 0;
  return round_up(static_cast<size_t>((N + 127) / 128) * 32 * sizeof(uint32_t), 256);
}

int fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int N, int d, int causal, float scale, const uint8_t* block_mask,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID_ARG;
  int rc = check_shape(B, H, N, d, scale);
  if (rc) return rc;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if ((N + 127) / 128 > 1024) return FA_ERR_UNSUPPORTED;  // the kernel's per-tile bitmask limit
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < fa_fwd_block_sparse_workspace_bytes(B, H, N, d))
    return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  fa::FwdArgs a;
  if ((rc = encode_bnhd(&a.tm_q, q, B, N, H, d)) || (rc = encode_bnhd(&a.tm_k, k, B, N, H, d)) ||
      (rc = encode_bnhd(&a.tm_v, v, B, N, H, d)) ||
      (rc = encode_bnhd(&a.tm_o, o, B, N, H, d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32)))
    return rc;
  a.lse = lse;
  a.block_mask = block_mask;
  a.mask_words = static_cast<uint32_t*>(workspace);
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.status = di.status;
  a.num_sms = di.num_sms;
  return from_cuda(fa::launch_fwd_block_sparse(a, static_cast<cudaStream_t>(stream)));
}

int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H,
               int N, int d, int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || !(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d < 1 || d > 128 || (d % 4) != 0) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535 || static_cast<long double>(B) * N * H * d > 9.0e15L)
    return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4))
    return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  return from_cuda(fa::launch_fwd_f32(q, k, v, o, lse, B, H, N, d, causal ? 1 : 0, scale,
                                      static_cast<cudaStream_t>(stream)));
}

int fa_read_device_status(const void* status_word_or_null, void* stream) {
  if (status_word_or_null && !aligned(status_word_or_null, 4)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  int* word_ptr = status_word_or_null ? static_cast<int*>(const_cast<void*>(status_word_or_null))
                                      : di.status;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int word = 0;
  const int zero = 0;
  if (cudaMemcpy(&word, word_ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(word_ptr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return FA_ERR_CUDA;
  return word;
}

int fa_debug_umma_tile(const void* a, const void* b, float* c, int n, int k, int mode,
                       void* stream) {
  if (!a || !b || !c) return FA_ERR_INVALID_ARG;
  if ((n != 64 && n != 128) || (k != 64 && k != 128) || mode < 0 || mode > 2)
    return FA_ERR_UNSUPPORTED;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(c, 16)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  return from_cuda(
      fa::launch_debug_umma(a, b, c, n, k, mode, di.status, static_cast<cudaStream_t>(stream)));
}

int fa_debug_exp2(const float* x, float* y_poly, float* y_hw, int n, void* stream) {
  if (!x || !y_poly || !y_hw || n < 1 || n > (1 << 28)) return FA_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(y_poly, 4) || !aligned(y_hw, 4)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  return from_cuda(fa::launch_debug_exp2(x, y_poly, y_hw, n, static_cast<cudaStream_t>(stream)));
}

int fa_debug_tma_tile(const void* x, void* y, int B, int N, int H, int d, int b, int h, int row0,
                      int chunk, void* stream) {
  if (!x || !y) return FA_ERR_INVALID_ARG;
  int rc = check_shape(B, H, N, d, 1.0f);
  if (rc) return rc;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (b < 0 || b >= B || h < 0 || h >= H || row0 < 0 || row0 >= N || chunk < 0 ||
      chunk >= d / 64)
    return FA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  CUtensorMap tm;
  if ((rc = encode_bnhd(&tm, x, B, N, H, d))) return rc;
  return from_cuda(fa::launch_debug_tma_tile(tm, y, b, h, row0, chunk, di.status,
                                             static_cast<cudaStream_t>(stream)));
}

int fa_debug_tmem_roundtrip(const uint32_t* in, uint32_t* out, int ncols, void* stream) {
  if (!in || !out) return FA_ERR_INVALID_ARG;
  if (ncols != 32 && ncols != 64 && ncols != 128 && ncols != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned(in, 4) || !aligned(out, 4)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  return from_cuda(fa::launch_debug_tmem_roundtrip(in, out, ncols, static_cast<cudaStream_t>(stream)));
}

int fa_debug_fwd_schedule(int B, int H, int N, int causal, int grid, int* units, int max_rounds,
                          void* stream) {
  if (!units || B < 1 || H < 1 || N < 1 || grid < 1 || grid > 65535 || max_rounds < 1)
    return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(grid) * max_rounds > (1LL << 28)) return FA_ERR_INVALID_ARG;
  if (!aligned(units, 4)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  return from_cuda(fa::launch_debug_schedule(B, H, N, causal ? 1 : 0, grid, units, max_rounds,
                                             static_cast<cudaStream_t>(stream)));
}

int fa_debug_wait_timeout(long long timeout_ns, void* status_word_or_null, void* stream) {
  if (timeout_ns < 1000 || timeout_ns > 10000000000LL) return FA_ERR_INVALID_ARG;
  if (status_word_or_null && !aligned(status_word_or_null, 4)) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  int* word = status_word_or_null ? static_cast<int*>(status_word_or_null) : di.status;
  return from_cuda(fa::launch_debug_wait_timeout(static_cast<uint64_t>(timeout_ns), word,
                                                 static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
