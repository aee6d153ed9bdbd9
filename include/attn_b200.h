/*
 * attn_b200.h - C ABI of a fused scaled-dot-product attention forward (and
 * its backward pass) for NVIDIA B200 (sm_100a).
 *
 * The operation ("Self-Attention, CUDA kernels and FlashAttention", section 1,
 * eq. Scores and eq. Attention; section 3, tiling / online-softmax / recompute
 * bullets), computed independently for every (batch b, head h):
 *
 *     S   = scale * Q K^T                        (N x N, never stored)
 *     P   = row-softmax(S), causal: S_ij = -inf for key j > query i
 *     O   = P V                                  (N x d)
 *     LSE_i = ln sum_j exp(S_ij)                 (natural log, scale included)
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, contiguous, row-major [B, H, N, d] with d innermost;
 *     LSE is [B, H, N]; per-tile FP8 scales are [B, H, ceil(N/128)]; MXFP8
 *     scale bytes are [B, H, N, d/32].
 *   - Every pointer argument is a DEVICE pointer owned by the caller, 16-byte
 *     aligned. The library never frees or retains caller memory.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t passed as
 *     void*, NULL = the legacy default stream). The host never synchronises.
 *   - Causal masking is square and top-left aligned: query i sees keys j <= i.
 *   - scale == 0 selects the default 1/sqrt(d) (eq. Scores); a negative or
 *     non-finite scale is an argument error.
 *   - Argument errors are detected on the host before anything is launched and
 *     returned immediately (INVALID_ARG, UNSUPPORTED, MISALIGNED). A failed
 *     launch returns ATTN_ERR_CUDA. A device-side pipeline wait that exceeds its
 *     time limit makes the kernel stop early and record ATTN_ERR_TIMEOUT in a
 *     device status word, read by attn_get_device_status().
 *   - A returned ATTN_OK means the launch was queued. The outputs are valid
 *     only once attn_get_device_status() has returned ATTN_OK after the launch
 *     completed: a launch that timed out leaves them undefined.
 *   - The status word is ONE word per device for the whole library, shared by
 *     every stream, thread and entry point: a timeout recorded by a launch on
 *     stream A is reported (and cleared) by whichever attn_get_device_status()
 *     call reads it first, whatever stream that call names.
 *   - N >= 1, B >= 1, H >= 1, and B*H*N < 2^31.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad flag        */
  ATTN_ERR_UNSUPPORTED = 2,  /* head width or dtype this build has no kernel for */
  ATTN_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned                 */
  ATTN_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed              */
  ATTN_ERR_TIMEOUT = 5,      /* a device pipeline wait ran out (see below)       */
  ATTN_ERR_BOUNDS = 6        /* debug builds: a device-side index check failed   */
} attn_status;

/* Element type of attn_fwd's q, k, v and o (passed as an int-sized enum). */
typedef enum {
  ATTN_BF16 = 0              /* bf16 inputs and output, fp32 accumulation        */
} attn_dtype;

/*
 * attn_fwd - BF16 attention forward.
 *   q, k, v : [B, H, N, d] bf16 inputs.
 *   o       : [B, H, N, d] bf16 output O = softmax(scale Q K^T) V.
 *   lse     : [B, H, N] fp32 output LSE, or NULL to skip it.
 *   d       : 64 or 128 (else ATTN_ERR_UNSUPPORTED).
 *   causal  : 0 or 1.   dtype: ATTN_BF16.
 * Cites: "Self-Attention, CUDA kernels and FlashAttention", section 1 eq. Attention
 * (what is computed) and section 3 (tiled, fused, online softmax, only O and the
 * row statistics written); "FlashAttention scaling, multi-GPU training and weight
 * quantization", section 1 (FlashAttention-2 loop order and deferred rescaling,
 * FlashAttention-3 asynchronous copies and warp specialisation).
 */
ATTN_API attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int N, int d, float scale, int causal, attn_dtype dtype,
                     void* stream);

/*
 * attn_quantize_fp8 - FP8 preparation of one tensor (incoherent processing and
 * block quantisation, "FlashAttention scaling, multi-GPU training and weight
 * quantization", section 1, FlashAttention-3 FP8 bullet).
 *   x      : [B, H, N, d] bf16 input.
 *   rot    : [d, d] bf16 orthogonal matrix (row-major), or NULL for no rotation
 *            (V is quantised without rotation).
 *   x8     : [B, H, N, d] output E4M3 codes (one byte each).
 *   scales : [B, H, ceil(N/128)] fp32 output, one per tile of 128 tokens x d.
 *   d      : 128 (else ATTN_ERR_UNSUPPORTED).
 * Definition: y = x rot accumulated in fp32 in increasing k order;
 * scale = max|y| over the tile / 448 (1 for an all-zero tile);
 * code = E4M3 round-to-nearest-even, saturating, of y / scale.
 */
ATTN_API attn_status attn_quantize_fp8(const void* x, const void* rot, void* x8, float* scales,
                              int B, int H, int N, int d, void* stream);

/*
 * attn_fwd_fp8 - attention forward on block-quantised E4M3 inputs
 * ("FlashAttention scaling, multi-GPU training and weight quantization",
 * section 1, FlashAttention-3 FP8 bullet: FP8 tensor-core inputs with one scale
 * per small tile, Q and K made incoherent by a random orthogonal matrix; what
 * is computed is the attention of "Self-Attention, CUDA kernels and
 * FlashAttention", section 1, eq. Attention, on the dequantised values).
 *   q8, k8, v8 : [B, H, N, d] E4M3 codes (q8, k8 rotated by the same orthogonal
 *                matrix, which leaves Q K^T unchanged).
 *   q_scale, k_scale, v_scale : [B, H, ceil(N/128)] fp32 tile scales; the
 *                value of a code is decode(code) * scale of its 128-token tile.
 *                Every scale must be finite and >= 0 (attn_quantize_fp8 writes
 *                only positive ones); a tile whose scale is 0 dequantises to
 *                zeros. The library cannot check device arrays on the host:
 *                a negative, infinite or NaN scale gives an undefined result.
 *   o   : [B, H, N, d] bf16 output.  lse: [B, H, N] fp32 or NULL.
 *   d   : 128 (else ATTN_ERR_UNSUPPORTED).
 * S = Q K^T runs on the E4M3 tensor-core MMA; for P V the E4M3 V tile is
 * widened on chip to f16 (exactly) and P is written as f16, with fp32
 * accumulation; the error this adds is within the FP8 tolerance of the tests.
 */
ATTN_API attn_status attn_fwd_fp8(const void* q8, const void* k8, const void* v8,
                         const float* q_scale, const float* k_scale, const float* v_scale,
                         void* o, float* lse, int B, int H, int N, int d, float scale,
                         int causal, void* stream);

/*
 * attn_quantize_mxfp8 - MXFP8 quantisation of one tensor ("Efficient MoE
 * training for biological foundation models", the low-precision paragraph:
 * MXFP8, 8-bit values sharing one power-of-two scale per block of 32, the input
 * format of Blackwell's block-scaled tensor-core products; the arithmetic below
 * is the OCP Microscaling definition).
 *   x     : [B, H, N, d] bf16 input, finite values.
 *   codes : [B, H, N, d] output E4M3 codes (one byte each).
 *   sf    : [B, H, N, d/32] output E8M0 scale bytes, one per 32 consecutive
 *           values of a row (value 2^(byte - 127)).
 *   d     : a multiple of 32, at most 4096 (else ATTN_ERR_UNSUPPORTED).
 * Definition, per block: E = floor(log2(max |v|)) - 8 clamped to [-127, 127]
 * (E = 0 for an all-zero block); byte = E + 127; code = E4M3 round-to-nearest-
 * even, saturating to +-448, of v * 2^-E. Bit-exact with that definition.
 */
ATTN_API attn_status attn_quantize_mxfp8(const void* x, void* codes, void* sf, int B, int H, int N, int d,
                                void* stream);

/*
 * attn_fwd_mxfp8 - attention forward on MXFP8 inputs (same page and paragraph as
 * attn_quantize_mxfp8; what is computed is the attention of "Self-Attention,
 * CUDA kernels and FlashAttention", section 1, eq. Attention, on the
 * dequantised values decode(code) * 2^(byte - 127)).
 *   q8, k8, v8       : [B, H, N, d] E4M3 codes.
 *   q_sf, k_sf, v_sf : [B, H, N, d/32] E8M0 scale bytes (as attn_quantize_mxfp8
 *                      writes them), 16-byte aligned.
 *   o   : [B, H, N, d] bf16 output.  lse: [B, H, N] fp32 or NULL.
 *   d   : 128 (else ATTN_ERR_UNSUPPORTED).
 * S = Q K^T runs on the block-scaled MMA (tcgen05 kind::mxf8f6f4.block_scale:
 * the scales are applied inside the tensor cores). V's blocks run along d, not
 * along the keys P V contracts over, so V is widened on chip to f16 with its
 * scales applied relative to the largest scale of its 32-column block over the
 * keys a 128-row query tile sees: exact for every block within 22 binades of
 * that largest scale (smaller blocks, below 2^-22 of the column's largest
 * values, round in f16's subnormal range or flush to zero). P is written as
 * f16; accumulation in fp32.
 */
ATTN_API attn_status attn_fwd_mxfp8(const void* q8, const void* k8, const void* v8, const void* q_sf,
                           const void* k_sf, const void* v_sf, void* o, float* lse, int B, int H, int N,
                           int d, float scale, int causal, void* stream);

/*
 * attn_bwd - backward pass of attn_fwd (BF16) from the saved statistic LSE
 * ("Self-Attention, CUDA kernels and FlashAttention", section 3, recompute
 * bullet: the forward keeps only the per-row normalisation statistics, and the
 * backward recomputes the attention weights tile by tile in on-chip memory
 * instead of reading a stored N x N matrix). For dL/dO = dout it computes
 *     P  = exp(scale Q K^T - LSE)   (causal: 0 for key j > query i)
 *     dV = P^T dO,   dP = dO V^T,   D_i = sum_c dO_ic O_ic,
 *     dS = P * (dP - D),   dQ = scale dS K,   dK = scale dS^T Q.
 *   q, k, v    : [B, H, N, d] bf16, the forward's inputs.
 *   o, lse     : the forward's outputs for those inputs ([B, H, N, d] bf16 and
 *                [B, H, N] fp32, natural log), as attn_fwd wrote them.
 *   dout       : [B, H, N, d] bf16 gradient of the loss with respect to O.
 *   dq, dk, dv : [B, H, N, d] bf16 outputs (must not alias the inputs).
 *   workspace  : device scratch of at least attn_bwd_workspace_bytes(B, H, N, d)
 *                bytes, 16-byte aligned, owned by the caller; it holds D_i and
 *                is overwritten. Calls that overlap on the GPU need separate
 *                workspaces.
 *   scale, causal: the values the forward used (scale == 0: 1/sqrt(d)).
 *   d          : 64 or 128 (else ATTN_ERR_UNSUPPORTED).
 * LSE is taken as the saved statistic, not a differentiated output: no gradient
 * flows into it. Three kernels run on `stream` in order (D_i, then dK and dV,
 * then dQ); nothing is allocated. Errors as for attn_fwd, plus
 * ATTN_ERR_INVALID_ARG for a null workspace or one smaller than required.
 */
ATTN_API attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, void* workspace,
                     size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                     void* stream);

/* attn_bwd_workspace_bytes - workspace attn_bwd needs for this shape (0 for an
 * invalid or unsupported shape). Host only; launches nothing. */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * attn_bwd_noalloc - attn_bwd for callers that cannot allocate device memory.
 * (No counterpart in the paper: this is a deployment variant, not part of the
 * method.) Some callers of this library cannot call cudaMalloc on the path that
 * runs the backward pass: an operator plugin inside a framework that owns the
 * whole device memory pool and hands its plugins no scratch buffer, or a
 * latency-critical service that must not allocate there because cudaMalloc can
 * synchronise the device and stall every other stream. For them this entry
 * point takes the same arguments as attn_bwd minus the workspace and keeps its
 * scratch (D_i, 4 bytes per row) in a fixed array inside the library instead.
 *   - Limit: B * H * N <= ATTN_BWD_NOALLOC_MAX_ROWS (2^21 rows, an 8 MiB array
 *     that every GPU which loads the library holds until the process exits);
 *     larger shapes return ATTN_ERR_UNSUPPORTED without launching anything.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current) and caches it; if that lookup
 *     fails the call returns ATTN_ERR_CUDA. Make that first call before any
 *     stream capture.
 *   - Every call shares the one array, which keeps the last call's contents
 *     (each call rewrites every row it reads before reading it, so nothing has
 *     to start at zero). Calls that overlap on the GPU (other streams, other
 *     threads) race on it: serialise them.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * Other arguments, results and errors as for attn_bwd.
 */
#define ATTN_BWD_NOALLOC_MAX_ROWS (1 << 21)
ATTN_API attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * attn_get_device_status - synchronises `stream`, then reads and clears the
 * device status word that kernels set when a pipeline wait timed out (or, in
 * a debug build, when an index check failed).
 * Returns ATTN_OK, ATTN_ERR_BOUNDS (debug builds: some check failed since the
 * last read; it takes precedence over a timeout recorded in the same word),
 * ATTN_ERR_TIMEOUT, or ATTN_ERR_CUDA if the read failed.
 */
ATTN_API attn_status attn_get_device_status(void* stream);

/*
 * Debug build (libattn_b200_debug.so, compiled with -DATTN_DEBUG; the pages
 * define no counterpart: this is the library's own checking aid). Every kernel
 * then checks, before the access, the row index of each global store of O,
 * LSE, dQ, dK, dV, FP8 tile scales, MXFP8 codes and scale bytes and W4A16
 * output columns against the extent the call's sizes give, the row of each
 * MXFP8 scale-byte load and backward LSE / D_i load, and each TMA coordinate
 * (x a multiple of 16 elements, stores at non-negative coordinates, work units
 * inside the launch). A failing check skips the access (nothing traps) and
 * records ATTN_ERR_BOUNDS in the status word, plus its site and index; a
 * skipped TMA load leaves its pipeline barrier incomplete, so the launch also
 * ends through the bounded-wait timeout. Results of a debug build are
 * bit-identical to the release build's when no check fails.
 *
 * attn_debug_build - 1 in a debug build, 0 otherwise.
 *
 * attn_debug_last_failure - synchronises `stream`, then reads and clears the
 * site and index of the first check that failed since the last call (site 0:
 * none). Sites: 1 O / LSE row (two-Q-tile forward), 2 O / LSE row (one-Q-tile
 * forward), 3 MXFP8 scale-byte row load, 4 dK / dV row, 5 LSE / D_i load (dK dV
 * kernel), 6 dQ row and its LSE / D_i load, 7 FP8 tile scale, 8 MXFP8 block,
 * 9 W4A16 output column, 10 TMA coordinate or work unit, 11 split-K W4A16
 * partial slot (index: the slot). `site` and `index`
 * are host pointers. Returns ATTN_OK, ATTN_ERR_INVALID_ARG for a null pointer,
 * or ATTN_ERR_CUDA. In a release build the site is always 0.
 */
ATTN_API int attn_debug_build(void);
ATTN_API attn_status attn_debug_last_failure(int* site, long long* index, void* stream);

/* attn_status_string - static, human-readable name of a status code. */
ATTN_API const char* attn_status_string(int status);

/* attn_abi_version - version of this ABI (incremented on incompatible change). */
ATTN_API int attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
