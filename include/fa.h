/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa.so).
 *
 * What is computed.  Exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 * as written in "Flash Attention 2で打破するローカルLLMの「メモリの壁」" (section
 * 標準的なAttention機構のメモリ挙動, the Attention(Q,K,V) formula), evaluated the IO-aware
 * way the same page describes (section タイリング（Tiling）と再計算（Recomputation）の仕組み):
 * Q, K and V move through on-chip memory in tiles, a running max / sum per row keeps the
 * softmax globally normalised ("FlashAttention-2を読む", section タイル分割でも全体の
 * 正規化を保つ), and only O and the per-row logsumexp reach device memory.  The backward
 * pass recomputes S and P from the logsumexp instead of storing them.
 *
 * Conventions shared by every entry point:
 *  - Tensor layout: q, k, v, o, dO, dq, dk, dv are contiguous [B][N][H][d] arrays (the
 *    (batch, seq, heads, head_dim) order of flash_attn_func on the same page, section
 *    カスタムモデルへの組み込み).  lse is a contiguous [B][H][N] fp32 array.
 *  - lse[b][h][i] = ln sum_j exp(scale * q_i . k_j) over the keys visible to query i
 *    (natural log, scale included).
 *  - Causal mask: key j is visible to query i iff j <= i.  Q and K have the same length N
 *    (except fa_fwd_splitkv, whose causal rule aligns the last query with the last key).
 *  - scale is passed explicitly (1/sqrt(d) gives the textbook softmax); it must be a
 *    positive finite number (the kernels take each row maximum before scaling).
 *  - All tensor pointers are DEVICE pointers owned by the caller.  No entry point
 *    allocates, frees or synchronises (except fa_read_device_status); work is enqueued on
 *    `stream` (a cudaStream_t passed as void*, NULL = legacy default stream).
 *  - Alignment: every bf16 / fp32 tensor pointer must be 16-byte aligned (the TMA and
 *    vector-store rule) except fa_fwd / fa_fwd_f32's lse (4 bytes); else FA_ERR_MISALIGNED.
 *  - Return value: FA_OK (0) on success, else an fa_status code.  On any non-zero return
 *    nothing was launched and no output was touched.  No C++ exception crosses the ABI.
 *  - Device-side failures (a bounded wait inside a kernel that ran out) do not trap the
 *    GPU: the kernel records FA_ERR_TIMEOUT in a device status word, tears its CTA down
 *    cleanly and returns; read the word with fa_read_device_status().  At the end of every
 *    CTA the main forward kernel (fa_fwd, fa_fwd_block_sparse, fa_fwd_fp8) and the
 *    backward's key-tile kernel (fa_bwd, fa_bwd_kv) also check that their warp roles agree
 *    on the work done (tiles loaded = consumed, steps per role) and record FA_ERR_INTERNAL
 *    if not.
 *  - Which status word.  The backward entry points that take a workspace (fa_bwd,
 *    fa_bwd_deterministic and the staged fa_bwd_preprocess / fa_bwd_kv / fa_bwd_dq_convert)
 *    record into a word of their own: the first 4 bytes of that workspace, cleared when the
 *    call's first kernel starts.  Every other entry point (the forward family, fa_bwd_noalloc,
 *    the self-tests) records into one library-owned word per device.  Calls on several
 *    streams at once therefore each get their own backward word (one workspace per
 *    concurrent call, as the dQ accumulator already requires), while the library word is
 *    shared: it holds the first failure of any of those calls, whichever stream it came
 *    from, and reading it clears it for every caller.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* B, H or N < 1, a null pointer, scale not > 0 and finite, size overflow */
  FA_ERR_UNSUPPORTED = 2, /* head dim not supported by this entry point / no sm_100 device */
  FA_ERR_MISALIGNED = 3,  /* a pointer not 16-byte aligned                                */
  FA_ERR_WORKSPACE = 4,   /* workspace null or smaller than fa_bwd_workspace_bytes()      */
  FA_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed (launch, attribute, ...) */
  FA_ERR_TIMEOUT = 6,     /* a device-side bounded wait expired (read via status word)    */
  FA_ERR_INTERNAL = 7     /* a kernel's end-of-CTA protocol check failed: a library defect
                             (read via status word; the results of that call are not valid) */
} fa_status;

/* Forward pass, bf16 in / bf16 out, fp32 accumulation and statistics.
 *   q, k, v : [B][N][H][d] bf16 (read)        o   : [B][N][H][d] bf16 (written)
 *   lse     : [B][H][N] fp32 (written), 4-byte aligned
 *   d must be 64 or 128 (else FA_ERR_UNSUPPORTED).
 * Kernel: persistent, warp-specialised tcgen05 (TMEM accumulators, TMA K/V ring). */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, int causal, float scale, void* stream);

/* Bytes of device workspace fa_bwd needs for this problem: the call's status word (an int
 * at offset 0, in a 256-byte slot), an fp32 dQ accumulator (B*H*N*d floats), then the fp32
 * row statistic D and the base-2 logsumexp, each B*H*Np floats with Np = N rounded up to a
 * multiple of 128; every part starts on a 256-byte boundary.  Returns 0 if the arguments
 * are invalid. */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/* Backward pass.  Inputs are the forward's q, k, v, its outputs o and lse, and the
 * upstream gradient dO (all [B][N][H][d] bf16 except lse, which must be 16-byte
 * aligned here).  Writes dq, dk, dv
 * ([B][N][H][d] bf16).  `workspace` is caller-owned device memory of at least
 * fa_bwd_workspace_bytes(B, H, N, d) bytes, 256-byte aligned; its contents on entry are
 * ignored and on return are unspecified except for its first int, the call's status word
 * (read it with fa_read_device_status(workspace, stream)).  d must be 64 or 128.
 * Steps: D = rowsum(dO o O) with dQ-accumulator clearing; per key/value tile, recompute
 * S^T and P^T from lse, dP^T = V dO^T, dS^T = P^T o (dP^T - D); dV += P^T dO and
 * dK += dS^T Q accumulate in TMEM; dQ += dS K is reduced in fp32 into the workspace
 * and converted to bf16 (times scale) by a final pass. */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv,
           int B, int H, int N, int d, int causal, float scale,
           void* workspace, size_t workspace_bytes, void* stream);

/* Bitwise-repeatable backward pass: same arguments, workspace and results as fa_bwd (within
 * the same tolerance of the exact gradients), but every output is accumulated in a fixed
 * order, so repeated calls on the same inputs give identical bits.  dQ comes from a separate
 * per-query-tile kernel that recomputes S and dP (1.4x the tensor work of fa_bwd) instead of
 * fp32 reductions whose arrival order varies.  The pages call the method "exact and
 * deterministic" ("FlashAttention-2 — FlashAttention-2", section パフォーマンス). */
int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dO, void* dq, void* dk, void* dv,
                         int B, int H, int N, int d, int causal, float scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/* The three stages fa_bwd runs, exposed so a caller can time or schedule them apart.
 * Calling them in this order on one stream with the same workspace is exactly fa_bwd.
 *  fa_bwd_preprocess: D = rowsum(dO o O) and lse*log2(e) into the workspace; clears the
 *                     workspace's fp32 dQ accumulator and its status word.  Reads o, lse,
 *                     dO.
 *  fa_bwd_kv:         the recompute kernel: per key/value tile, rebuilds S^T and P^T from
 *                     the workspace statistics, writes dk, dv and adds dS K into the dQ
 *                     accumulator.  Reads q, k, v, dO; needs fa_bwd_preprocess first.
 *  fa_bwd_dq_convert: dq = bf16(scale * accumulator). */
int fa_bwd_preprocess(const void* o, const float* lse, const void* dO, int B, int H, int N,
                      int d, void* workspace, size_t workspace_bytes, void* stream);
int fa_bwd_kv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
              int B, int H, int N, int d, int causal, float scale, void* workspace,
              size_t workspace_bytes, void* stream);
int fa_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Backward pass for callers that cannot allocate device memory.
 *
 * Who needs it: code that may not call cudaMalloc -- for example a plugin hosted by a
 * framework that owns all device memory through its own allocator and forbids direct
 * driver allocations, or a latency-critical loop that cannot afford cudaMalloc's implicit
 * device-wide synchronisation -- and so cannot provide fa_bwd's workspace.  This entry
 * point has no counterpart in the source pages; it is fa_bwd with the workspace taken from
 * a fixed array inside the library instead of from the caller.
 *
 * Same arguments and results as fa_bwd minus the workspace.  The caller still owns and
 * passes every input and output.  The library holds FA_NOALLOC_WORKSPACE_BYTES of device
 * memory per GPU that loads it, for the life of the process; problems whose
 * fa_bwd_workspace_bytes() exceeds that are rejected with FA_ERR_WORKSPACE before anything
 * is launched.  Nothing here allocates or frees memory.
 *  - The first call on a device looks up the array's device address (set-up, once per
 *    device, with that device current); make that first call before any stream capture.
 *  - Every call on a device shares the one array.  Calls whose work overlaps on the GPU
 *    (e.g. on two streams without ordering between them) race on it and give wrong
 *    results; serialise them.  Each call re-initialises what it needs (the dQ accumulator
 *    is cleared), so leftovers of a previous call do not matter.
 *  - The device address found at set-up is cached per device for the life of the process.
 *    It stays valid as long as that device's primary context does: a caller that destroys
 *    the context (cudaDeviceReset) must not call this entry point on that device again.
 *  - A failure inside a kernel is recorded in the library-owned status word (read it with
 *    fa_read_device_status(NULL, stream)). */
#define FA_NOALLOC_WORKSPACE_BYTES (64u * 1024u * 1024u)
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, int causal, float scale, void* stream);

/* Element types of fa_fwd_splitkv. */
enum { FA_DTYPE_BF16 = 0, FA_DTYPE_FP16 = 1 };

/* Forward pass for few queries against many keys (decoding), with the key sequence split
 * across CTAs and the slices merged exactly through their logsumexps.  Prefill and decode
 * are measured separately ("FlashAttention-2を読む", section 実装上の差を検証可能な形で残す);
 * fp16 is FA-2's other input type ("Flash Attention 2で打破するローカルLLMの「メモリの壁」",
 * section Hugging Face Transformersでの有効化設定).
 *   q : [B][Nq][H][d]; k, v : [B][Nk][H][d]; o : [B][Nq][H][d]  (all bf16 or all fp16,
 *   `dtype` = FA_DTYPE_BF16 / FA_DTYPE_FP16);  lse : [B][H][Nq] fp32.
 *   Causal: the last query is aligned with the last key -- query i sees keys
 *   j <= i + Nk - Nq; requires Nq <= Nk.  Non-causal: any Nq, Nk >= 1.  d in {64, 128}.
 *   workspace: caller-owned device memory, >= fa_fwd_splitkv_workspace_bytes(...), 256-byte
 *   aligned (fp32 partial outputs and logsumexps of every slice). */
size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d);
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int Nq, int Nk, int d, int causal, float scale, int dtype,
                   void* workspace, size_t workspace_bytes, void* stream);

/* Block-sparse forward pass, the extension described with the original method
 * ("FlashAttention――GPUメモリの読み書きを減らし、注意機構を正確なまま高速・省メモリに",
 * section 手法): key j is visible to query i iff block_mask[i/128][j/128] != 0 (and, if
 * causal, j <= i); masked 128x128 blocks are neither loaded nor computed.
 *   q, k, v, o : [B][N][H][d] bf16; lse : [B][H][N] fp32; d in {64, 128}; N <= 131072
 *   (larger: FA_ERR_UNSUPPORTED).
 *   block_mask : DEVICE pointer, [ceil(N/128)][ceil(N/128)] bytes, shared by all batches and
 *                heads.
 *   A query that sees no key at all gets O = 0 and lse = -inf.
 *   Runs on the forward kernel of fa_fwd: per query tile, its active key tiles are dealt to
 *   the kernel's two ping-pong slots in turn and the slots' partial results merged exactly.
 *   workspace : >= fa_fwd_block_sparse_workspace_bytes(B, H, N, d) bytes (the mask packed
 *   into 128 bytes of bits per query tile), 16-byte aligned, caller-owned. */
size_t fa_fwd_block_sparse_workspace_bytes(int B, int H, int N, int d);
int fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int N, int d, int causal, float scale,
                        const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                        void* stream);

/* FP8 forward with incoherent processing ("FlashAttention-3 — FlashAttention-3", section
 * FlashAttention-3の技術的革新, item 3: Q and K are multiplied by a random orthogonal
 * matrix -- a Hadamard matrix -- before the 8-bit rounding; the matrix cancels in Q K^T).
 * Two calls: fa_fp8_quantize prepares the operands once, fa_fwd_fp8 runs attention on them
 * with both products on the tensor core in E4M3 (kind::f8f6f4).
 *
 * fa_fp8_quantize:
 *   q, k, v : [B][N][H][d] bf16 (d in {64, 128}).
 *   signs   : DEVICE [d] fp32 of +-1 (the random diagonal s), or NULL for no transform.
 *             Q and K rows are mapped x -> x diag(s) H_d / sqrt(d), H_d the Sylvester
 *             Hadamard matrix of order d.
 *   q8, k8  : [B][N][H][d] E4M3 codes (1 byte each); vt8 : [B][H][d][Npad] E4M3 codes of V
 *             transposed (keys contiguous), Npad = N rounded up to a multiple of 16, keys
 *             in [N, Npad) zero.  No transform on V.
 *   scales  : [3][B*H] fp32, the dequantisation scales of Q, K, V per (batch, head): the
 *             smallest power of two 2^e with 448 * 2^e >= max |x| over the (transformed)
 *             head (1 for an all-zero head); codes are round-to-nearest-even, saturating
 *             E4M3 of x / 2^e.
 *   workspace : >= fa_fp8_quantize_workspace_bytes(B, H) bytes, 4-byte aligned (per-head
 *             maxima; cleared by the call).
 * fa_fwd_fp8:
 *   q8, k8, vt8, scales : as produced above, d = 128 only (others: FA_ERR_UNSUPPORTED).
 *   o : [B][N][H][d] bf16, lse : [B][H][N] fp32, for
 *       O = softmax(scale * (s_q Q8)(s_k K8)^T) (s_v V8) with P rounded to E4M3 before the
 *       second product; lse is that softmax's natural-log normaliser.
 *   Errors as fa_fwd; all pointers DEVICE, 16-byte aligned (scales, lse: 4). */
size_t fa_fp8_quantize_workspace_bytes(int B, int H);
int fa_fp8_quantize(const void* q, const void* k, const void* v, const float* signs,
                    void* q8, void* k8, void* vt8, float* scales, int B, int H, int N, int d,
                    void* workspace, size_t workspace_bytes, void* stream);
int fa_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* scales, void* o,
               float* lse, int B, int H, int N, int d, int causal, float scale, void* stream);

/* Forward pass in fp32 on the CUDA cores (no tensor cores, no TF32), for fp32 inputs.
 *   q, k, v, o : [B][N][H][d] fp32; lse : [B][H][N] fp32.  1 <= d <= 128, d % 4 == 0. */
int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
               int B, int H, int N, int d, int causal, float scale, void* stream);

/* Synchronises `stream`, then returns and clears a device status word: FA_OK, or the
 * first failure recorded there (FA_ERR_TIMEOUT, FA_ERR_INTERNAL, FA_ERR_UNSUPPORTED).
 *   status_word_or_null : NULL for the library-owned word of the current device, or the
 *       DEVICE pointer of a backward call's own word, which is the start of the workspace
 *       that call was given (4-byte aligned, else FA_ERR_MISALIGNED).
 * `stream` must be the stream (or a stream ordered after the one) the calls of
 * interest ran on.  Returns FA_ERR_CUDA if the synchronisation or the copy failed (no
 * kernel ever records that code, so it cannot be confused with a word's value). */
int fa_read_device_status(const void* status_word_or_null, void* stream);

/* Static, human-readable name of a status code. */
const char* fa_status_string(int status);

/* Library ABI version (major*100 + minor). */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
