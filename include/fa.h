/*
 * fa.h — C ABI of the B200 (sm_100a) exact attention library, libfa.so.
 *
 * The library computes exact scaled dot-product attention
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 * as one fused, tiled forward kernel that never writes the Sq x Sk score or
 * probability matrix to device memory, and a backward that rebuilds the
 * probabilities from the saved per-row logsumexp instead of storing them.
 *
 * Sources (page title, section):
 *   [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练", section
 *        "性能引擎：FlashAttention 如何重塑注意力计算？" (the formula; fusion of
 *        QK^T, softmax and PV into one kernel; recomputation in the backward),
 *        section "实战集成" (fp16/bf16 inputs; no mask or causal mask only).
 *   [P2] "使用FlashAttention优化PyTorch模型注意力计算", section
 *        "FlashAttention 是如何做到又快又省内存的？" items 1-3 (fusion, tiling
 *        with an online softmax, recomputation).
 *        Section "工程实践中的关键考量" (head_dim <= 128).
 *   [P4] the FlashAttention-2 walkthrough titled "企业官网建设流程全解析",
 *        §3.1 (unscaled output, one final rescale, only the logsumexp saved),
 *        §3.2 (parallelism over batch x heads x sequence blocks), §3.3 (five
 *        matrix products in the backward), §4 (flash_attn_func on
 *        (batch, seq_len, num_heads, head_dim), causal flag), §5 (fp32 inputs
 *        are rejected).
 *   [P5] the FlashAttention "IO感知" overview (0539edu.com/news/165270),
 *        sections "H100的FP8加速能力" and "未来展望" (an FP8 data type in
 *        FlashAttention-3): fa_fwd_fp8.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout. q, o, dO and dq are [B, Sq, H, D]; k, v, dk and dv are [B, Sk, H, D]
 *   (the (batch, seq_len, num_heads, head_dim) layout of [P4] §5). The
 *   head_dim axis is contiguous. fa_fwd/fa_bwd take densely packed tensors;
 *   the *_ex forms take per-tensor element strides for batch, sequence and
 *   head (e.g. views into a packed qkv tensor [B, S, 3, H, D], [P1]
 *   "实战集成").
 * lse. fp32 [B, H, Sq], dense: LSE_i = ln sum_j exp(scale * q_i . k_j) over
 *   the keys row i may attend to (natural log of the scaled scores; [P4] §3.1
 *   names only "logsumexp"). A row with no allowed key gets -inf and O = 0.
 * Causal mask. Bottom-right aligned: query i may attend to key j iff
 *   j <= i + (Sk - Sq). With Sq == Sk this is the lower triangle.
 * dtype. FA_FP16 or FA_BF16 for every tensor of a call except lse and the
 *   workspace (fp32). Anything else is FA_ERR_UNSUPPORTED ([P4] §5).
 * head_dim. D a multiple of 8 in [8, 128] ([P2] "工程实践中的关键考量": head_dim
 *   <= 128); other values are FA_ERR_UNSUPPORTED. D <= 64 runs the 64-column
 *   kernels and 64 < D <= 128 the 128-column ones, with the columns past D
 *   read as zeros (extra tensor-core work, exact results).
 * scale. Finite and > 0 (1/sqrt(D) in the usual use); else FA_ERR_INVALID_ARG.
 * Sizes. B, H, Sq, Sk >= 1; B*H*Sq and B*H*Sk below 2^31.
 * Alignment. Every tensor base address 16-byte aligned and every stride a
 *   multiple of 8 elements (16 bytes): the kernels read tiles with the Tensor
 *   Memory Accelerator. Violations are FA_ERR_MISALIGNED.
 * Ownership. The caller allocates every tensor and the workspace, in device
 *   memory of the current device, and owns the stream. The library keeps no
 *   per-call allocations: it holds one device status word per device.
 * Asynchrony. Calls enqueue work on `stream` and return without waiting.
 *   Argument errors are detected on the host before anything is launched and
 *   return a negative fa_status with no work enqueued. A failed launch
 *   returns FA_ERR_CUDA. Errors detected inside a running kernel (a pipeline
 *   wait that exceeded its time limit) are recorded in the device status word
 *   and reported by fa_last_device_status().
 * Streams. `stream` is a cudaStream_t (0 = the legacy default stream).
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* fa_stream_t; /* identical to cudaStream_t */

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1,     /* null pointer, size < 1, bad scale or causal flag */
  FA_ERR_UNSUPPORTED = -2,     /* dtype or head_dim outside what the kernels handle */
  FA_ERR_MISALIGNED = -3,      /* base address or stride breaks the 16-byte rule */
  FA_ERR_CUDA = -4,            /* a CUDA runtime/driver call failed */
  FA_ERR_TIMEOUT = -5,         /* a device-side pipeline wait ran out (fa_last_device_status) */
  FA_ERR_NOT_IMPLEMENTED = -6, /* reserved */
  FA_ERR_WORKSPACE = -7,       /* workspace pointer null or smaller than fa_bwd_workspace_size */
  FA_ERR_SCRATCH_LIMIT = -8,   /* fa_bwd_noalloc: problem needs more than FA_NOALLOC_SCRATCH_BYTES */
  FA_ERR_BOUNDS = -9           /* check build (libfa_check.so) only: a device-side index or bounds
                                  check failed; the access was skipped (fa_last_device_status) */
} fa_status;

/* Size of the built-in device scratch buffer of fa_bwd_noalloc (64 MiB per
   device that loads the library). */
#define FA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* A strided [B, S, H, D] view: element strides for batch, sequence and head;
   the head_dim axis has stride 1. */
typedef struct {
  void* ptr;
  int64_t stride_b, stride_s, stride_h;
} fa_tensor;

typedef struct {
  fa_tensor q, k, v; /* read */
  fa_tensor o;       /* written */
  float* lse;        /* written, dense fp32 [B, H, Sq] */
  int B, H, Sq, Sk, D;
  float scale;
  int causal; /* 0 or 1 */
  int dtype;  /* fa_dtype */
  /* Optional key-range split (all three zero: off). With a workspace of at
     least fa_fwd_workspace_size_ex(B, H, Sq, Sk, D, causal, split_ranks, NULL)
     bytes (256-byte aligned, used by no other call at the same time, need not
     be initialised) the heaviest 256-row query blocks may each run as two
     CTAs, one per half of the key blocks, whose partial results are merged
     exactly (the online-softmax rescaling of [P4] §3.1 applied between the
     two halves); this shortens the longest CTA and fills the SMs when
     B * H * ceil(Sq / 256) is small ([P4] §3.2: too few blocks for the SMs).
     O and lse stay the exact attention; the rounding order differs from the
     unsplit CTAs in the last bits. split_ranks: 0 = the library chooses
     (a list-scheduling estimate of the CTAs over the current device's SMs,
     kept if it predicts a grid more than 8% shorter; never splits at four
     waves or more), k > 0 = split the first min(k,
     ceil(Sq / 256)) query-block ranks (ranks count 256-row blocks from the
     last one when causal, the heaviest first; from the first otherwise),
     -1 = never. Splits apply only when ceil(Sq / 256) <= 64. The CTAs then
     start longest first (whole ranks and halves sorted by their estimated
     length). A NULL workspace runs unsplit; a non-NULL workspace that is
     too small for the split chosen is FA_ERR_WORKSPACE, a misaligned one
     FA_ERR_MISALIGNED. */
  void* workspace;
  size_t workspace_bytes;
  int split_ranks;
} fa_fwd_params;

typedef struct {
  fa_tensor q, k, v, o, dO; /* read; o and lse are the forward's outputs */
  const float* lse;         /* read, dense fp32 [B, H, Sq] */
  fa_tensor dq, dk, dv;     /* written */
  int B, H, Sq, Sk, D;
  float scale;
  int causal;
  int dtype;
  void* workspace; /* device scratch, >= fa_bwd_workspace_size_ex(B, H, Sq, Sk, D,
                      deterministic) bytes, 256-byte aligned */
  size_t workspace_bytes;
  int deterministic; /* 0: dq summed with fp32 atomics (fast; last bits may vary
                        between runs). 1: every (query block, key block) dQ block
                        is stored in its own workspace slot and the slots are
                        added in key-block order by a last kernel, so dq, like
                        dk and dv, is bit-identical from run to run. Anything
                        else is FA_ERR_INVALID_ARG. */
} fa_bwd_params;

/* Forward ([P1] "性能引擎"; [P2] items 1-2; [P4] §3.1, §3.2).
   Reads q [B,Sq,H,D], k and v [B,Sk,H,D]; writes o [B,Sq,H,D] (rounded once,
   to nearest even, to `dtype`) and lse [B,H,Sq] fp32. Dense tensors; no
   workspace, so no key-range split (fa_fwd_ex has it). */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int Sq, int Sk, int D, float scale, int causal,
           int dtype, fa_stream_t stream);

/* Forward on strided views (packed qkv and the like), with the optional
   key-range split. Same semantics. */
int fa_fwd_ex(const fa_fwd_params* p, fa_stream_t stream);

/* Workspace bytes fa_fwd_ex needs for the split that `split_ranks` selects
   (see fa_fwd_params) on the current device; 0 when that is no split or the
   arguments are invalid. If n_split is not NULL it receives the number of
   split query-block ranks (0: none). Host only; launches nothing. */
size_t fa_fwd_workspace_size_ex(int B, int H, int Sq, int Sk, int D, int causal, int split_ranks, int* n_split);

/* fa_fwd_workspace_size_ex with split_ranks = 0 (the library's choice). */
size_t fa_fwd_workspace_size(int B, int H, int Sq, int Sk, int D, int causal);

/* The key-range split plan, for inspection (host only; launches nothing).
   Plans for `sms` SMs (0: the current device's count). *n_split receives
   the number of split query-block ranks. If it is 0 the grid is rank-major
   (head-major without a mask) and 0 is returned. Otherwise `order`
   receives the grid's units, longest first, one byte each: rank * 3 + kind
   (kind 0 = the whole rank, 1 = its first key half, 2 = its second). Ranks
   count 256-row query blocks from the last one when causal, from the first
   otherwise. Each unit is B * H CTAs. The return value is the number of
   units (ceil(Sq / 256) + n_split). Errors: as fa_fwd for the sizes;
   FA_ERR_INVALID_ARG if sms < 0 or `order_capacity` is too small;
   FA_ERR_CUDA if sms is 0 and no device can be queried. */
int fa_fwd_split_plan(int B, int H, int Sq, int Sk, int D, int causal, int split_ranks, int sms, int* n_split,
                      unsigned char* order, int order_capacity);

/* e4m3 forward: the parameters of fa_fwd_fp8_ex. */
typedef struct {
  fa_tensor q, k, v; /* read, E4M3 bytes; strides in elements (= bytes) */
  fa_tensor o;       /* written, o_dtype */
  float* lse;        /* written, dense fp32 [B, H, Sq] */
  int B, H, Sq, Sk, D;
  float scale;
  float q_descale, k_descale, v_descale; /* real value = stored E4M3 value * descale */
  int causal;
  int o_dtype; /* FA_FP16 or FA_BF16 */
} fa_fwd_fp8_params;

/* Forward from 8-bit floating-point inputs ([P5] sections "H100的FP8加速能力"
   and "未来展望：FlashAttention-3带来的新可能": FlashAttention-3 adds an FP8
   data type; the pages give no more than that, so the form below is this
   library's reading).
   q, k, v hold OCP E4M3 bytes (1 sign bit, 4 exponent bits with bias 7, 3
   mantissa bits, largest finite value 448, no infinities) in the [B, S, H, D]
   layout. The values attended over are q * q_descale, k * k_descale and
   v * v_descale: one finite, positive factor per tensor. The result is the
   same exact attention as fa_fwd on those values, computed as follows:
   Q K^T is formed by the tensor cores with fp32 accumulation (products of two
   E4M3 values are exact in fp32); the softmax runs in fp32 as in fa_fwd; the
   probabilities P (relative to the running row maximum, at most 2^8) are
   rounded to E4M3, round to nearest even, for the P V product; the row sum l
   is taken over the unrounded P. So lse is as exact as fa_fwd's, and the
   rounding of P moves each element of O by at most
       sum_j max(2^-4 P_ij, 2^-10) |v_jd| / l_i
   with P_ij = exp(scale q_i.k_j - max_j') relative to the row maximum and
   l_i = sum_j P_ij. O is written as o_dtype, lse as in fa_fwd.
   head_dim: D a multiple of 16 in [16, 128] (every tile is 128 bytes wide;
   columns past D read as zeros). Alignment: base addresses 16-byte aligned,
   strides of q, k and v multiples of 16 elements, of o multiples of 8.
   Descale factors that are not finite and > 0 are FA_ERR_INVALID_ARG; an
   o_dtype other than FA_FP16 or FA_BF16 is FA_ERR_UNSUPPORTED. Ownership,
   asynchrony and error reporting as for fa_fwd. */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
               int B, int H, int Sq, int Sk, int D, float scale,
               float q_descale, float k_descale, float v_descale, int causal,
               int o_dtype, fa_stream_t stream);

/* e4m3 forward on strided views. Same semantics. */
int fa_fwd_fp8_ex(const fa_fwd_fp8_params* p, fa_stream_t stream);

/* Backward ([P1] "性能引擎" recomputation; [P2] item 3; [P4] §3.1 logsumexp,
   §3.3 five matrix products). Given the forward's inputs, its outputs o and
   lse, and dO = dL/dO, writes dq, dk, dv = dL/dq, dL/dk, dL/dv (each rounded
   once to `dtype`). P is rebuilt from lse, never read from memory. dq is
   accumulated in fp32 in `workspace` and converted at the end; the
   accumulation order across key blocks is not fixed, so dq may differ in the
   last bits from run to run. The workspace contents on entry do not matter;
   the call overwrites them. */
int fa_bwd(const void* q, const void* k, const void* v, const void* o,
           const float* lse, const void* dO, void* dq, void* dk, void* dv,
           int B, int H, int Sq, int Sk, int D, float scale, int causal,
           int dtype, void* workspace, size_t workspace_bytes,
           fa_stream_t stream);

/* Backward on strided views. Same semantics, plus the deterministic mode
   (fa_bwd_params.deterministic; the pages are silent on it). */
int fa_bwd_ex(const fa_bwd_params* p, fa_stream_t stream);

/* Backward that allocates nothing and takes no workspace. Not a method step:
   the pages have no counterpart; it exists for callers that cannot allocate
   device memory themselves, such as code running inside a host application
   that reserves all device memory up front and hands out only input and
   output buffers, plug-in interfaces with no way to ask for a workspace, or
   latency-critical code that must not call cudaMalloc (which may synchronise
   the device).
   Same arguments, semantics and results as fa_bwd, except that the scratch
   (the fp32 dq accumulator, Dvec and the base-2 logsumexp) lives in one
   static device array of FA_NOALLOC_SCRATCH_BYTES inside the library,
   reserved on every device that loads it until the process exits. Problems
   whose fa_bwd_workspace_size() exceeds that size return
   FA_ERR_SCRATCH_LIMIT (about B*H*Sq*(D+2)*4 bytes; B*H = 8, Sq = 8192,
   D = 128 needs 34 MB). No cudaMalloc, cudaFree or other allocating call is
   made.
   Set-up: the first call on a device (the current device) looks up the
   array's device address with cudaGetSymbolAddress and caches it; make that
   first call before any stream capture on that device. Later calls only
   launch kernels.
   Sharing: every call on a device uses the same array. Each call rewrites all
   of the scratch it reads (the accumulator is zeroed by the call's first
   kernel), so leftovers of earlier calls do not matter, but two calls that
   run at the same time on one device (different streams, or host threads
   without ordering between them) race on the array and give wrong results:
   order them on one stream or with events. */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                   const float* lse, const void* dO, void* dq, void* dk,
                   void* dv, int B, int H, int Sq, int Sk, int D, float scale,
                   int causal, int dtype, fa_stream_t stream);

/* Bytes of device workspace fa_bwd needs: an fp32 dq accumulator
   [B, H, Sq_pad, Dk], the fp32 row terms Dvec_i = sum_d dO_id O_id
   [B, H, Sq_pad] and the fp32 logsumexp in base 2 [B, H, Sq_pad], where
   Sq_pad is Sq rounded up to a multiple of 128 and Dk is the kernel width
   (64 for D <= 64, else 128). Returns 0 for sizes < 1 or on overflow. */
size_t fa_bwd_workspace_size(int B, int H, int Sq, int D);

/* Workspace of fa_bwd_ex for either mode. deterministic = 0 gives
   fa_bwd_workspace_size(B, H, Sq, D). deterministic = 1 adds, after that
   (rounded up to 256 bytes), one fp32 [128][Dk] slot per (b, h, query block,
   key block): B*H*ceil(Sq/128)*ceil(Sk/128)*128*Dk*4 bytes (2.15 GB for
   B*H = 8, Sq = Sk = 8192, D = 128). Returns 0 for sizes < 1, a flag other
   than 0 or 1, or on overflow. */
size_t fa_bwd_workspace_size_ex(int B, int H, int Sq, int Sk, int D, int deterministic);

/* Synchronises the current device, returns the status word recorded by
   kernels since the last call (FA_OK, FA_ERR_TIMEOUT or, in the check
   build, FA_ERR_BOUNDS) and clears it. FA_ERR_CUDA if the device cannot be
   queried. If `detail` is non-null it receives 4 ints: code, linear block
   index, role (1 = loader, 2 = MMA issuer, 3 = softmax/epilogue, 4 =
   self-test, 5 = bounds check) and the block-loop iteration (for a bounds
   check: the number of the check site, see fa_common.cuh).
   There is one status word per device, shared by every stream and thread
   that uses the library on it: the first kernel to record a failure keeps
   it until this call, which waits for all work on the device (not only one
   stream) so that no kernel still running can record after the read.

   The check build. libfa_check.so is the same library compiled with
   FA_CHECK=1: the kernels test their own index arithmetic at the places
   where it addresses memory (tile coordinates, TMEM columns, shared-memory
   offsets, output and workspace indices against the sizes of the call). A
   failed check records FA_ERR_BOUNDS and skips that access; nothing traps.
   Results are the same as the normal build's; it runs slower. */
int fa_last_device_status(int* detail);

/* Self-test of failure detection (not a method step). Launches one block on
   `stream` whose pipeline wait never completes: after limit_us microseconds
   (1 .. 4,000,000) the wait gives up, records FA_ERR_TIMEOUT in the device
   status word with role 4 (self-test) and block 0, and the block winds down
   through the same abort path the attention kernels use. Nothing faults or
   hangs and the context stays usable; read the result with
   fa_last_device_status(). FA_ERR_INVALID_ARG for a limit out of range. */
int fa_selftest_wait_timeout(unsigned int limit_us, fa_stream_t stream);

/* Static, human-readable text for a status code. Never null. */
const char* fa_strerror(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
