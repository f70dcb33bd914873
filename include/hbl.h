/*
 * hbl.h -- C ABI of libhbl.so: the H-BitLinear forward of BitNet v2 on B200 (sm_100a).
 *
 * The operation is the one defined in "BitNet v2: Native 4-bit Activations
 * with Hadamard Transformation for 1-bit LLMs" (architecture walkthrough,
 * section 3.4):
 *
 *   Y = Q_w(W) . Q_INT8/4(X_r),   X_r = Hadamard(X)                (Eq. 9)
 *   Q_w(W)    = alpha * RoundClip(W / (alpha + eps), -1, 1),
 *               alpha = mean|W| over the whole tensor                (Eq. 1-2)
 *   Hadamard(x) = H_m x, Sylvester H_m scaled by 2^(-m/2), n = 2^m    (Eq. 3-6)
 *   Q_INT8(x) = gamma/127 * RoundClip(127/(gamma+eps) x, -128, 127),
 *               gamma = max|x| per token                              (Eq. 7)
 *   Q_INT4(x) = beta/sqrt7 * RoundClip(sqrt7/(beta+eps) x, -8, 7),
 *               beta = mean|x| per token                              (Eq. 8)
 *
 * with eps = 1e-5 and round-half-to-even. The LN of Eq. 9 is not applied here:
 * the layer input X is taken as already normalised.
 *
 * Shapes: X is M x K (tokens x in-features), W is N x K (out x in), Y is M x N;
 * all row-major and contiguous. bf16 tensors are passed as their 16-bit
 * patterns (hbl_bf16).
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE memory owned by the caller unless stated otherwise.
 *     The library never frees caller memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Nothing throws, aborts or prints. Arguments are checked before
 *     any launch; a rejected call launches nothing and returns the status.
 *   - Return value: an hbl_status (HBL_OK = 0).
 *   - M == 0 is an empty batch: the call returns HBL_OK and launches nothing.
 *   - Y must not overlap X; Wpk and wscale are read-only during a forward.
 *   - Input values are expected to be finite.
 *   - Every tensor pointer must be 16-byte aligned (HBL_ERR_INVALID_ARG otherwise).
 */
#ifndef HBL_H_
#define HBL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t hbl_bf16;              /* bit pattern of a bfloat16 value */
typedef struct CUstream_st* hbl_stream; /* same type as cudaStream_t       */

typedef enum {
  HBL_OK = 0,
  HBL_ERR_INVALID_ARG = 1, /* null pointer, act_bits not in {4,8}, bad flag          */
  HBL_ERR_SHAPE = 2,       /* a size outside the supported set (see each call)      */
  HBL_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed                  */
  HBL_ERR_ALLOC = 4,       /* the library's own device allocation failed            */
  HBL_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out                    */
  HBL_ERR_UNSUPPORTED = 6, /* the current device is not sm_100                      */
  HBL_ERR_WORKSPACE = 7    /* caller workspace missing or smaller than required     */
} hbl_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* hbl_status_string(int status);

/* Library ABI version, currently 1. */
int hbl_version(void);

/* ------------------------------------------------------------------------
 * Weights: ternarise and pack (offline, once per weight matrix).
 * ------------------------------------------------------------------------ */

/* Bytes of the packed weight buffer for an N x K matrix: N*K/4 (2 bits per weight). */
size_t hbl_packed_bytes(int N, int K);

/*
 * hbl_pack_weights -- Eq. 1-2 (section 3.4, "Weight Quantization").
 *   W      : device fp32, N x K row-major, the latent full-precision weights.
 *   Wpk    : device, hbl_packed_bytes(N, K) bytes, written with the ternary codes.
 *   wscale : device, one fp32, written with alpha.
 * alpha is the exact mean of |W| (exact sum rounded once to fp64, divided by
 * N*K in fp64, rounded to fp32), so it does not depend on the order of
 * summation. Codes are RoundClip(W / (alpha + eps), -1, 1) with the division
 * in fp32.
 * Wpk is OPAQUE: its layout is chosen for the forward kernels. Use
 * hbl_unpack_weights for the canonical N x K view of the codes.
 * Shapes: N >= 1, N % 16 == 0, K >= 256, K % 256 == 0, N*K < 2^31.
 * Uses a small internal device scratch (allocated on the first call per
 * device); calls on different streams of one device must not overlap.
 */
int hbl_pack_weights(const float* W, int N, int K, uint8_t* Wpk, float* wscale,
                     hbl_stream stream);

/*
 * hbl_unpack_weights -- canonical view of packed weights: the ternary codes
 * RoundClip(W / (alpha + eps), -1, 1) of Eq. 1-2 (section 3.4, "Weight
 * Quantization") that hbl_pack_weights stored.
 *   Wpk : device, from hbl_pack_weights for an N x K matrix (same N, K).
 *   T   : device int8, N x K row-major, written with codes in {-1, 0, +1}.
 * Shapes as hbl_pack_weights. Asynchronous on `stream`; no allocation.
 */
int hbl_unpack_weights(const uint8_t* Wpk, int N, int K, int8_t* T, hbl_stream stream);

/* ------------------------------------------------------------------------
 * Forward.
 * ------------------------------------------------------------------------ */

/* Bytes of caller workspace needed by hbl_forward_ws for these sizes. */
size_t hbl_workspace_bytes(int M, int K, int N);

/*
 * hbl_forward_ws -- H-BitLinear forward, Eq. 9 without the LN.
 *   X            : device bf16, M x K.
 *   Wpk, wscale  : from hbl_pack_weights for an N x K matrix.
 *   act_bits     : 4 (Eq. 8, absmean, codes in [-8, 7]) or 8 (Eq. 7, absmax, codes in [-127, 127]).
 *   use_hadamard : 1 = apply the Hadamard transform along K first (K must be a
 *                  power of two, 256 <= K <= 32768); 0 = plain BitLinear
 *                  (K % 256 == 0, K <= 65536).
 *   Y            : device bf16, M x N, written with bf16_rne(acc * s[m] * alpha),
 *                  acc the exact integer product of the codes, s[m] the token scale.
 *   ws, ws_bytes : device workspace of at least hbl_workspace_bytes(M, K, N)
 *                  bytes, 256-byte aligned; clobbered.
 * Shapes: M >= 0, N % 16 == 0, N >= 16. Launches only kernels; makes no
 * allocation and no synchronisation, so it may be captured in a CUDA graph.
 */
int hbl_forward_ws(const hbl_bf16* X, int M, int K, int N, const uint8_t* Wpk,
                   const float* wscale, int act_bits, int use_hadamard, hbl_bf16* Y,
                   void* ws, size_t ws_bytes, hbl_stream stream);

/*
 * hbl_forward -- same as hbl_forward_ws with a library-owned workspace.
 * The workspace is per device and grows on demand (a cudaMalloc while the
 * stream may be busy), so this call is not for stream capture, and calls on
 * different streams of one device must not overlap.
 */
int hbl_forward(const hbl_bf16* X, int M, int K, int N, const uint8_t* Wpk,
                const float* wscale, int act_bits, int use_hadamard, hbl_bf16* Y,
                hbl_stream stream);

/*
 * hbl_forward_noalloc -- the same forward as hbl_forward_ws, for callers that
 * cannot allocate device memory: for example a serving process whose memory
 * pool has already reserved nearly all of HBM (a cudaMalloc would fail), code
 * that must not pay the device-wide synchronisation a cudaMalloc/cudaFree can
 * imply, or a host framework that forbids its plugins from allocating.
 * The paper has no counterpart; this is a deployment convenience.
 *
 * The workspace is a fixed 8 MiB device array inside the library image,
 * reserved on every GPU that loads the library until the process exits. The
 * call makes no cudaMalloc/cudaFree and no other allocation.
 *   - Sizes whose workspace, hbl_workspace_bytes(M, K, N), exceeds 8 MiB are
 *     rejected with HBL_ERR_WORKSPACE before any launch (use hbl_forward_ws
 *     with your own buffer for those, e.g. large prefill batches).
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; whatever must start at zero is cleared by the call itself.
 *     Calls whose execution overlaps on the GPU (different streams, or
 *     different host threads) race on the array: serialise them.
 * Arguments, shapes and results are those of hbl_forward_ws.
 */
int hbl_forward_noalloc(const hbl_bf16* X, int M, int K, int N, const uint8_t* Wpk,
                        const float* wscale, int act_bits, int use_hadamard, hbl_bf16* Y,
                        hbl_stream stream);

/* ------------------------------------------------------------------------
 * Stage-wise entry points (the steps of the forward, for checking each one).
 * ------------------------------------------------------------------------ */

/*
 * hbl_hadamard_f32 -- X_r = Hadamard(X) per token in fp32 (Eq. 3-5).
 *   X  : device bf16 M x K.   Xr : device fp32 M x K.
 * K must be a power of two, 256 <= K <= 32768.
 */
int hbl_hadamard_f32(const hbl_bf16* X, int M, int K, float* Xr, hbl_stream stream);

/*
 * hbl_quantize -- optional Hadamard (Eq. 3-5), then the per-token quantiser
 * (section 3.4, "Activation Quantization", Eq. 7 / Eq. 8).
 *   codes  : device int8 M x K.
 *   scales : device fp32 M: gamma/127 (act_bits 8) or beta/sqrt7 (act_bits 4).
 *   csum   : device int32 M or NULL: sum of the codes of each token. Not part
 *            of the method: the GEMM kernels multiply the codes by t + 1 (an
 *            unsigned weight code) and subtract this sum, which is exact; it is
 *            exposed so the stages can be checked one by one.
 * Shapes as hbl_forward_ws (K a power of two in [256, 32768] with the
 * Hadamard, else K % 256 == 0).
 */
int hbl_quantize(const hbl_bf16* X, int M, int K, int act_bits, int use_hadamard,
                 int8_t* codes, float* scales, int32_t* csum, hbl_stream stream);

/*
 * hbl_gemm_codes -- the integer product inside Eq. 9 (section 3.4,
 * "H-BitLinear: The Composite Layer"), before any dequantisation:
 * acc[m, n] = sum_k codes[m, k] * T[n, k], exactly, in int32, with T the
 * ternary codes of Eq. 1-2 held in Wpk.
 *   codes : device int8 M x K (any values in [-128, 127]).
 *   Wpk   : device, from hbl_pack_weights for an N x K matrix.
 *   acc   : device int32 M x N.
 * Same shape rules as hbl_forward_ws (K % 256 == 0). The per-token code
 * sums go to a small library-owned scratch that grows on demand (a
 * cudaMalloc), shared with hbl_forward: make a first call of each size
 * before any stream capture, and do not overlap calls on different streams.
 */
int hbl_gemm_codes(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk,
                   int32_t* acc, hbl_stream stream);

/* ------------------------------------------------------------------------
 * Beyond the LN-free forward: the LN of Eq. 9, the rotated-weight variant,
 * the Hadamard backward (Eq. 10) and the post-RoPE QKV quantiser.
 * ------------------------------------------------------------------------ */

/*
 * hbl_forward_ln_ws -- the full H-BitLinear of Eq. 9 (section 3.4, "H-BitLinear:
 * The Composite Layer"): X_r = Hadamard(LN(X)) with LN the RMSNorm
 *   LN(x) = x * gain / sqrt(mean(x^2) + 1e-5)
 * (the epsilon is a reading: the pages give none). gain: device fp32 K, or
 * NULL for no gain. Everything else as hbl_forward_ws (same workspace size).
 * The normalisation is fused into the Hadamard/quantise kernel: the gain is
 * applied on load and the per-token factor is folded into the transform's
 * final scaling.
 */
int hbl_forward_ln_ws(const hbl_bf16* X, int M, int K, int N, const float* gain, const uint8_t* Wpk,
                      const float* wscale, int act_bits, int use_hadamard, hbl_bf16* Y, void* ws,
                      size_t ws_bytes, hbl_stream stream);

/* hbl_quantize_ln -- hbl_quantize with the RMSNorm above applied first. */
int hbl_quantize_ln(const hbl_bf16* X, int M, int K, const float* gain, int act_bits,
                    int use_hadamard, int8_t* codes, float* scales, int32_t* csum, hbl_stream stream);

/*
 * hbl_pack_weights_rotated -- the weight-and-activation rotation variant of the
 * ablation in section 3.4 (Table 5): packs Q_w(W H^T), i.e. every weight row w
 * is replaced by H w (fp32) before the ternary quantiser of Eq. 1-2. Used with
 * use_hadamard = 1 in the forward, the product is Q_w(W H^T) . Q(H x).
 *   Wrot : device fp32 N x K caller scratch; receives W H^T.
 * K must be a power of two, 256 <= K <= 32768; otherwise as hbl_pack_weights.
 */
int hbl_pack_weights_rotated(const float* W, int N, int K, uint8_t* Wpk, float* wscale,
                             float* Wrot, hbl_stream stream);

/*
 * hbl_hadamard_backward_f32 -- Eq. 10 (section 3.4, "Gradient Handling Through
 * the Hadamard Transformation"): dL/dX = H^T dL/dX_r per token, which for the
 * symmetric Sylvester H is the same fast transform. fp32 in, fp32 out, M x K.
 * K must be a power of two, 256 <= K <= 32768.
 */
int hbl_hadamard_backward_f32(const float* dXr, int M, int K, float* dX, hbl_stream stream);

/*
 * hbl_quantize_qkv -- post-RoPE QKV quantiser (section 3.4, "QKV Attention
 * Quantization"): each head vector of d values is quantised to unsigned
 * b-bit integers from its absmax gamma. Reading of "unsigned absmax":
 *   u = RoundClip((2^b - 1)/2 * (x / (gamma + 1e-5) + 1), 0, 2^b - 1),
 *   dequantised value (2u / (2^b - 1) - 1) * gamma.
 * The heads of token `bos_token` (the BOS token; -1 for none) use 8 bits.
 *   X     : device bf16, T x H x d (token, head, channel).
 *   codes : device uint8, T x H x d, one code per byte.
 *   gamma : device fp32, T x H.
 * d in {64, 128, 256}; 2 <= bits <= 8.
 */
int hbl_quantize_qkv(const hbl_bf16* X, int T, int H, int d, int bits, int bos_token,
                     uint8_t* codes, float* gamma, hbl_stream stream);

/*
 * hbl_get_device_error -- synchronises `stream`, then reads and clears the
 * device error word that bounded waits inside the kernels set when they give
 * up. Returns HBL_OK, HBL_ERR_TIMEOUT, or HBL_ERR_CUDA if the stream reports an
 * error.
 */
int hbl_get_device_error(hbl_stream stream);

/*
 * hbl_set_gemm_path -- which kernels the forward and hbl_gemm_codes use:
 * 0 = by size (default). The forward of 1..16 tokens with K in {2048, 4096}
 * (or K = 8192 with at most 8 tokens) and N % 16 == 0 runs as ONE fused kernel
 * (transform, quantiser, GEMM and dequant; codes exchanged between the CTAs
 * of a thread-block cluster). Otherwise the quantiser kernel runs first and
 * the GEMM is chosen by size: 1..16 tokens stream the weights (the
 * weight-streaming kernel when K % 2048 == 0, else the decode kernel split
 * over K across a cluster for 9..16 tokens, or with one CTA per 16 rows);
 * up to 32 tokens, and with N < 8192 up to 255 tokens (N <= 2048: up to
 * 1023), the warp-level split-K kernel; with K >= 8192 and at least 256
 * tiles of 128 x 128, the tcgen05 kernel with one 128 x 256 tile per CTA;
 * otherwise the persistent tcgen05 kernel (128 x 128 tiles).
 * 1 = always the warp-level split-K kernel, 2 = always the persistent tcgen05
 * kernel, 3 = as 0 but never the fused, cluster or streaming decode kernels,
 * 4 = always the one-tile tcgen05 kernel, 5 = as 0 but never the fused
 * forward, 6 = as 0.
 * All give results within the parity bounds of the oracle (the fused forward
 * and the quantiser kernel share their summation order, so the paths give the
 * same bits); the knob exists to check and time each one. Process-wide; each
 * forward or hbl_gemm_codes call reads it once when it starts, so a change
 * made while calls run on other threads applies from their next call on.
 * Returns HBL_ERR_INVALID_ARG for a value outside 0..6.
 */
int hbl_set_gemm_path(int path);

/*
 * hbl_selftest_wait_timeout -- failure-detection check of the bounded waits.
 * Launches one CTA whose mbarrier wait can never complete (the barrier
 * expects two arrivals and gets one). The wait is the same bounded try_wait
 * loop the pipelined kernels use, here limited to timeout_us microseconds
 * (1 .. 10^7). On expiry the kernel records HBL_ERR_TIMEOUT in the device
 * error word, writes 1 to *gave_up (device int, may be NULL) and exits
 * normally: no trap, no hang, the context stays usable. The next
 * hbl_get_device_error returns HBL_ERR_TIMEOUT.
 */
int hbl_selftest_wait_timeout(int timeout_us, int* gave_up, hbl_stream stream);

/* ------------------------------------------------------------------------
 * Per-kernel timing of the library's own launches.
 * While enabled, every kernel the library launches is bracketed by two CUDA
 * events recorded on its launch stream; durations accumulate per kernel name.
 * Meant for measurement runs, not for stream capture.
 * ------------------------------------------------------------------------ */

/* Enable (1) or disable (0) timing on the current device; enabling clears the totals. */
int hbl_profile_enable(int enable);

/* Number of distinct kernel names recorded so far (synchronises pending events). */
int hbl_profile_count(void);

/*
 * Totals of entry i (0 <= i < hbl_profile_count()): the kernel name (copied
 * into name, at most name_len bytes including the terminator), the number of
 * launches and their summed device time in milliseconds.
 */
int hbl_profile_get(int i, char* name, int name_len, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* HBL_H_ */
