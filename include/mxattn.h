/*
 * mxattn.h -- C ABI of the MXFP4 attention library for NVIDIA B200 (sm_100a).
 *
 * What it computes
 * ----------------
 * MXFP4 (OCP Microscaling) block quantization and MXFP4 attention forward as the MXAttention
 * paper defines it ("MXAttention: Data-Free Optimal Scaling and Pre-Normalization
 * Quantization for MXFP4 Attention", abstract):
 *   - 32-element blocks of E2M1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; "Quantization
 *     Error" page, section "Where the error comes from") sharing one E8M0 power-of-two scale;
 *     values are rounded to nearest-even on the grid and saturate at 6.
 *   - Scale exponent of a block with max magnitude amax:
 *       MXATTN_SCALE_OCP: e = floor(log2 amax) - 2        (the OCP MX v1.0 rule)
 *       MXATTN_SCALE_UOS: smallest e with amax / 2^e <= 7.25 (Universal Optimal Scaling)
 *     An all-zero block gets scale byte 0 and all-zero codes.
 *       MXATTN_SCALE_NVFP4: the NVFP4 comparison format for Q, K, V and P~ instead (blocks of
 *       16 with an E4M3 scale RNE(amax / 6); see mxattn_quantize_nvfp4); mxattn_forward and its
 *       prepare / attend / debug forms only.
 *   - Attention: Q, K quantized along the head dimension, V along keys; S = Q K^T as a
 *     block-scaled FP4 contraction; FlashAttention online softmax over key tiles of
 *     MXATTN_KV_TILE keys in increasing key order (running max, history rescale, fp32
 *     accumulation, final normalisation; "EFQ-Softmax" abstract).
 *     With pnq = 1 (Pre-Normalization Quantization)
 *     the unnormalised exponentials P~ = exp(S/sqrt(d) - m) are quantized to MXFP4 along keys
 *     before the row sum, and that same dequantized operand feeds both P~V and the row sum.
 *     With pnq = 0 the row sum uses the unquantized fp32 P~ (exp-then-quantize baseline).
 *     With pnq = 2 the P~ operand is made without exponentials, after the EFQ-Softmax abstract:
 *     per 32-key block the scale exponent e is the block's MXFP4 exponent (OCP or UOS) of its
 *     largest P~, and each key gets the code k = clamp(round_half_even(2 r + 2), 0, 7) of its
 *     residual r = log2(P~) - e; that operand feeds both P~V and the row sum, as under PNQ.
 *     (The abstract gives the structure -- exponent-only scale from the block max, residual
 *     domain, one affine rule -- but no constants; 2 r + 2 is the reading that lands on the
 *     grid values 1, 2 and 4 at r = 0, 1, 2.) MXFP4 scale modes only.
 *     Softmax scale is fixed at 1/sqrt(d).
 *
 * Conventions
 * -----------
 *   - Every pointer argument named as device memory must be a CUDA device pointer on the
 *     current device. The caller owns every buffer it passes, and no entry point calls
 *     cudaMalloc. Two exceptions hold library-owned resources: every device that loads the
 *     library reserves a fixed MXATTN_NOALLOC_MAX_WORKSPACE-byte static array (the workspace of
 *     mxattn_forward_noalloc) when the library's device module is loaded, and
 *     mxattn_forward_host creates its own streams and events on first use.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are asynchronous on it.
 *   - Argument errors are detected on the host and returned before anything is launched.
 *     Launch errors return MXATTN_ERR_CUDA. A device-side pipeline timeout (every wait inside
 *     the kernels is bounded) is recorded in the workspace and reported by
 *     mxattn_check_status().
 *   - Inputs must be finite; NaN / Inf inputs give unspecified codes.
 *   - Packed E2M1 layout: two codes per byte, element 2i in bits 0..3, element 2i+1 in bits
 *     4..7; code = sign << 3 | magnitude index. E8M0 byte = e + 127 (never 0xFF).
 */
#ifndef MXATTN_H_
#define MXATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MXATTN_SCALE_OCP = 0, MXATTN_SCALE_UOS = 1, MXATTN_SCALE_NVFP4 = 2 } mxattn_scale_mode;

/* Keys per tile of the online softmax. P~ is quantized with the running max in force at each
 * tile, so the tile width is part of the result (a CPU reference must use the same width). */
#define MXATTN_KV_TILE 128

/* Values of the `pnq` argument of the attention entry points: the rule that makes the P~ operand
 * and its row sum (see "What it computes" above). */
#define MXATTN_P_CONVENTIONAL 0   /* exp-then-quantize, row sum of the unquantized P~ */
#define MXATTN_P_PNQ 1            /* exp-then-quantize, row sum of the same quantized operand */
#define MXATTN_P_EFQ 2            /* exp-free codes, row sum of the same operand (MXFP4 only) */

typedef enum { MXATTN_OUT_F32 = 0, MXATTN_OUT_BF16 = 1 } mxattn_out_dtype;

typedef enum {
  MXATTN_OK = 0,
  MXATTN_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, negative or inconsistent size   */
  MXATTN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d not in {64, 128})        */
  MXATTN_ERR_WORKSPACE = 3,    /* workspace smaller than mxattn_forward_workspace_size()      */
  MXATTN_ERR_CUDA = 4,         /* a CUDA runtime / driver call or a kernel launch failed      */
  MXATTN_ERR_TIMEOUT = 5       /* a kernel gave up on a bounded wait (reported by check_status)*/
} mxattn_status;

/*
 * mxattn_quantize -- MXFP4-quantize `batch` bf16 matrices of shape [rows, cols] (row-major,
 * contiguous, device memory; `x` 2-byte aligned, 16-byte alignment enables vector loads).
 * (Method: "Quantization Error" page, "Where the error comes from"; MXAttention abstract, UOS.)
 *
 *   transpose = 0: blocks of 32 along cols.  codes  [batch][rows][ceil(cols/32) * 16] (uint8)
 *                                            scales [batch][rows][ceil(cols/32)]      (uint8)
 *   transpose = 1: blocks of 32 along rows (e.g. V along keys), written transposed:
 *                                            codes  [batch][cols][ceil(rows/32) * 16]
 *                                            scales [batch][cols][ceil(rows/32)]
 * A partial last block is zero-padded (padding never raises amax and encodes as +0).
 * `codes` must be 16-byte aligned. Sizes must satisfy batch*rows*ceil(cols/32) < 2^31 and,
 * for transpose = 1, batch <= 65535. Empty inputs (any size 0) are a no-op returning MXATTN_OK.
 */
mxattn_status mxattn_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols, int transpose,
                              int scale_mode, uint8_t* codes, uint8_t* scales, void* stream);

/*
 * Bytes of device workspace mxattn_forward needs: quantized Q, K, V^T in the tensor-core
 * layouts plus a 256-byte status area. 0 for invalid shapes.
 */
size_t mxattn_forward_workspace_size(int B, int Hq, int Hkv, int N, int d);

/*
 * mxattn_forward -- MXFP4 attention forward (MXAttention abstract: UOS + PNQ; OCP baseline).
 *   q   : bf16 [B, Hq,  N, d] contiguous, device, 16-byte aligned
 *   k, v: bf16 [B, Hkv, N, d] contiguous, device, 16-byte aligned
 *   out : [B, Hq, N, d] fp32 (out_dtype = MXATTN_OUT_F32) or bf16, device, 16-byte aligned
 *   Query head h reads KV head h / (Hq / Hkv) (contiguous GQA groups); Hq % Hkv == 0.
 *   causal = 1 masks keys after the query position. scale_mode applies to Q, K, V and P~.
 *   pnq: MXATTN_P_CONVENTIONAL, MXATTN_P_PNQ or MXATTN_P_EFQ (any other value ->
 *   MXATTN_ERR_INVALID_ARG; MXATTN_P_EFQ with MXATTN_SCALE_NVFP4 -> MXATTN_ERR_UNSUPPORTED).
 *   Supported: d in {64, 128}, 1 <= N, B*Hq*ceil(N/128) < 2^31.
 *   workspace: device memory of at least mxattn_forward_workspace_size(...) bytes, 256-byte
 *   aligned; its contents on entry are ignored; it must not be used concurrently by another
 *   call. The call runs one quantizer launch (Q, K and V^T) and then the fused kernel.
 */
mxattn_status mxattn_forward(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv,
                             int N, int d, int causal, int scale_mode, int pnq, int out_dtype,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * mxattn_forward_quantized -- the attention kernel alone, on Q, K and V already in MXFP4 (MXAttention
 * abstract: MXFP4 operands for Q K^T and P~ V; P~ is quantized inside by the rule `pnq` names).
 * The operands are in the canonical layout that mxattn_quantize writes:
 *   qc  : codes  [B, Hq,  N, d/2]   (mxattn_quantize of q, transpose = 0), 16-byte aligned
 *   qs  : scales [B, Hq,  N, d/32]  E8M0 bytes
 *   kc  : codes  [B, Hkv, N, d/2],  ks: scales [B, Hkv, N, d/32]
 *   vtc : codes  [B, Hkv, d, ceil(N/32)*16]  (mxattn_quantize of v with transpose = 1: blocks of
 *         32 keys, keys past N encoded as zero), 16-byte aligned
 *   vts : scales [B, Hkv, d, ceil(N/32)]
 *   p_scale_mode: the scale rule for P~ (the caller chose the rule of Q, K, V when quantizing);
 *   MXATTN_SCALE_OCP or MXATTN_SCALE_UOS (MXATTN_SCALE_NVFP4 -> MXATTN_ERR_UNSUPPORTED).
 * All other arguments as mxattn_forward; the workspace (mxattn_forward_workspace_size bytes)
 * receives the scales in the tensor-core layout and the status word; the codes are read in place
 * and must stay unchanged until the call has completed on the stream. Errors: null or misaligned
 * pointers -> MXATTN_ERR_INVALID_ARG; shapes as mxattn_forward.
 */
mxattn_status mxattn_forward_quantized(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                                       const uint8_t* vtc, const uint8_t* vts, void* out, int B, int Hq, int Hkv,
                                       int N, int d, int causal, int p_scale_mode, int pnq, int out_dtype,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * mxattn_gemm -- block-scaled MXFP4 matrix product C[M, N] = dq(A)[M, K] dq(B)[N, K]^T (both
 * operands K-major, as W4A4 layers and the attention's Q K^T use them). The MX format is the
 * "Quantization Error" page's (section "Where the error comes from"): E2M1 codes, one exact
 * power-of-two scale per 32 elements; no counterpart of the attention's P~ step.
 *   a_codes : [M, K/2] bytes, a_scales: [M, K/32] E8M0 bytes (mxattn_quantize of A, transpose = 0)
 *   b_codes : [N, K/2] bytes, b_scales: [N, K/32]
 *   c       : [M, N] fp32 (out_dtype = MXATTN_OUT_F32) or bf16, row-major, device
 *   Codes and c 16-byte aligned; workspace 256-byte aligned, >= mxattn_gemm_workspace_size bytes
 *   (it receives the scales in the tensor-core layout and the status word read by
 *   mxattn_check_status). Supported: K % 32 == 0, N % 8 == 0, M, N, K < 2^31, M <= 65535 * 128.
 *   Errors: null / misaligned pointers or bad dtype -> MXATTN_ERR_INVALID_ARG; other shapes ->
 *   MXATTN_ERR_UNSUPPORTED; small workspace -> MXATTN_ERR_WORKSPACE. Asynchronous on stream.
 */
size_t mxattn_gemm_workspace_size(int64_t M, int64_t N, int64_t K);
mxattn_status mxattn_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                          const uint8_t* b_scales, void* c, int64_t M, int64_t N, int64_t K, int out_dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * mxattn_selftest_wait_timeout -- exercises the failure detection every pipeline kernel uses; no
 * counterpart in the pages. Launches one CTA whose mbarrier phase never completes: its first warp
 * gives up after the library's wait bound (2 s of device time), writes 0x701 into the status word
 * and raises the CTA's abort flag; its second warp, waiting on the same phase, leaves through the
 * flag. Word 1 of the workspace then holds 3 (bit 0: the bounded wait returned, bit 1: the flag
 * was seen). workspace: >= 256 bytes of device memory, 256-byte aligned; its first 256 bytes are
 * overwritten. mxattn_check_status afterwards returns MXATTN_ERR_TIMEOUT with detail 0x701.
 * The kernel neither faults nor traps, and the context stays usable.
 */
mxattn_status mxattn_selftest_wait_timeout(void* workspace, void* stream);

/*
 * NVFP4 comparison path (MXAttention abstract: MXFP4 attention is compared with NVFP4-based
 * baselines; the pages give no NVFP4 recipe). Reading taken: blocks of 16 E2M1 elements along the
 * contiguous axis, one unsigned FP8 E4M3 scale per block, s = E4M3(amax / 6) rounded to nearest-
 * even and saturated at 448, elements x / s rounded to nearest-even on the E2M1 grid (saturating
 * at 6), no tensor-level scale; both quotients are correctly rounded fp32 divisions.
 *
 * mxattn_quantize_nvfp4: x bf16 device [rows, cols] -> codes [rows, ceil(cols/16)*8] bytes
 *   (element 2i in the low nibble; 8-byte aligned), scales [rows, ceil(cols/16)] E4M3 bytes.
 *   Empty inputs are a no-op; null or misaligned pointers -> MXATTN_ERR_INVALID_ARG.
 * mxattn_gemm_nvfp4: as mxattn_gemm with NVFP4 operands (scales [M, K/16] and [N, K/16]);
 *   workspace from mxattn_gemm_nvfp4_workspace_size; same shape rules and errors.
 */
mxattn_status mxattn_quantize_nvfp4(const void* x, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales,
                                    void* stream);
size_t mxattn_gemm_nvfp4_workspace_size(int64_t M, int64_t N, int64_t K);
mxattn_status mxattn_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                                const uint8_t* b_scales, void* c, int64_t M, int64_t N, int64_t K, int out_dtype,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * mxattn_forward_host -- mxattn_forward on HOST buffers (same arguments; q, k, v, out are host
 * pointers, best page-locked so the copies run asynchronously). The work is split into groups of
 * consecutive KV heads (with their query heads, about 512 attention CTAs per group) that rotate
 * through three device slots. Inputs are copied in on a library-owned stream; each group is
 * quantized and attended on `stream` or on a library-owned second compute stream, alternately;
 * outputs are copied out on a third library-owned stream. A slot's input buffers are refilled as
 * soon as its quantizers have read them, so copies run in both directions at once and overlap
 * the kernels. Heads are independent: the output is bit-identical to mxattn_forward's. The call
 * is asynchronous on `stream`: it starts after the work already queued there, and the output is
 * in `out` once `stream` has reached this point. Concurrent calls on one device (each with its
 * own workspace) share the library's streams: their copies and kernels interleave on them, and
 * each stays correct, since every wait is on an event recorded before it. Device workspace:
 * mxattn_forward_host_workspace_size(..., out_dtype) bytes, 256-byte aligned; its first word is
 * the status word read by mxattn_check_status.
 * Errors: as mxattn_forward (MXATTN_ERR_WORKSPACE against the host workspace size).
 */
size_t mxattn_forward_host_workspace_size(int B, int Hq, int Hkv, int N, int d, int out_dtype);
mxattn_status mxattn_forward_host(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv,
                                  int N, int d, int causal, int scale_mode, int pnq, int out_dtype, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * The two halves of mxattn_forward, for callers that time or reuse them separately:
 *   mxattn_forward_prepare quantizes q, k, v into the workspace;
 *   mxattn_forward_attend runs the fused attention kernel on a prepared workspace (same
 *   shapes and scale_mode as the prepare call).
 */
mxattn_status mxattn_forward_prepare(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                                     int N, int d, int scale_mode, void* workspace, size_t workspace_bytes,
                                     void* stream);
mxattn_status mxattn_forward_attend(void* out, int B, int Hq, int Hkv, int N, int d, int causal,
                                    int scale_mode, int pnq, int out_dtype, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * mxattn_forward_debug -- mxattn_forward that also dumps the quantized P~ operand of query
 * rows [r0, r1) of head dbg_bh (= b * Hq + h): p_codes [r1-r0][Npad/2] packed codes and
 * p_scales [r1-r0][Npad/32] scale bytes in absolute key order (Npad/16 for MXATTN_SCALE_NVFP4),
 * Npad = ceil(N/128)*128
 * (device memory). Meant for parity tests on small shapes.
 */
mxattn_status mxattn_forward_debug(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                                   int Hkv, int N, int d, int causal, int scale_mode, int pnq, int out_dtype,
                                   void* workspace, size_t workspace_bytes, void* stream, int dbg_bh,
                                   int dbg_r0, int dbg_r1, uint8_t* p_codes, uint8_t* p_scales);

/*
 * mxattn_forward_noalloc -- mxattn_forward for callers that cannot allocate device memory.
 * The paper has no counterpart to this entry point; it exists for deployment. Some callers
 * cannot call cudaMalloc: code whose device memory is owned by a host process or framework
 * (an inference server or plugin host with a fixed arena, an allocator that must account for
 * every byte), or a latency-critical loop where an allocation call, which may synchronise the
 * device or fail when a memory pool holds the free memory, is not allowed. They still pass
 * q, k, v and out exactly as for mxattn_forward; the workspace instead comes from a static
 * device array of MXATTN_NOALLOC_MAX_WORKSPACE bytes that every GPU loading the library holds
 * until the process exits.
 *   - Every argument is checked exactly as mxattn_forward checks it when handed a workspace of
 *     MXATTN_NOALLOC_MAX_WORKSPACE bytes: shapes with mxattn_forward_workspace_size(...) larger
 *     than that get MXATTN_ERR_WORKSPACE, every other rejected call the code mxattn_forward
 *     returns, all before anything is launched. No call allocates.
 *   - Each call looks up the array's device address in the current context (so it stays valid
 *     after cudaDeviceReset or in a non-primary context). The first call in a context may load
 *     the library's device module: make it before any stream capture.
 *   - All calls on a device share the array: calls whose kernels overlap on the GPU race, so
 *     serialise them (one stream, or explicit ordering). The status word is cleared at the
 *     start of each call. A device-side wait timeout is recorded only in the shared array,
 *     which no caller can read directly: the call has already returned MXATTN_OK and `out` is
 *     then unspecified. mxattn_check_status_noalloc reads (and clears) that word.
 */
#define MXATTN_NOALLOC_MAX_WORKSPACE ((size_t)16 << 20)
mxattn_status mxattn_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                                     int Hkv, int N, int d, int causal, int scale_mode, int pnq, int out_dtype,
                                     void* stream);

/*
 * mxattn_check_status -- synchronises `stream`, reads and clears the workspace status word.
 * Returns MXATTN_ERR_TIMEOUT if a kernel gave up on a bounded wait since the last check (the
 * raw code goes to *detail when detail != NULL), MXATTN_ERR_CUDA on a CUDA error, else MXATTN_OK.
 */
mxattn_status mxattn_check_status(void* workspace, void* stream, unsigned int* detail);

/*
 * mxattn_check_status_noalloc -- mxattn_check_status on the static array that
 * mxattn_forward_noalloc uses as its workspace, in the current context: synchronises `stream`,
 * reads and clears the status word the last mxattn_forward_noalloc calls wrote. Same returns as
 * mxattn_check_status. Like the forward call, it allocates nothing.
 */
mxattn_status mxattn_check_status_noalloc(void* stream, unsigned int* detail);

/* Static string for a status code. */
const char* mxattn_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int mxattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MXATTN_H_ */
