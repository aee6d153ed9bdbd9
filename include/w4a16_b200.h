/*
 * w4a16_b200.h - C ABI of the W4A16 GEMM (4-bit weights dequantised on the fly,
 * 16-bit activations) of the same library (libattn_b200.so), for NVIDIA B200.
 *
 * "FlashAttention scaling, multi-GPU training and weight quantization",
 * section 3, the W4A16 kernels paragraph: packed 4-bit weights, eight to a
 * 32-bit word, are read from HBM, unpacked in registers with shifts and masks,
 * made 16-bit floats with the stored scale and zero point, and fed to the
 * tensor cores with the 16-bit activations; expanded weights are never written
 * back to memory.
 *
 *     Y[M, N] = X[M, K] W[K, N]
 *     W[k, n] = fp16((q[k, n] - zeros[k / 128, n]) * scales[k / 128, n])
 *
 * Layouts (row-major, device memory owned by the caller, 16-byte aligned):
 *   x       : fp16 [M, K] activations.
 *   qweight : int32 [K / 8, N]; word (w, n) holds the codes q (0..15) of the
 *             weights k = 8w .. 8w+7 of column n, weight 8w + PERM[i] in bits
 *             4i .. 4i+3, PERM = {0, 2, 4, 6, 1, 3, 5, 7} (adjacent weights
 *             2j, 2j+1 sit 16 bits apart, so one mask extracts the pair).
 *   scales  : fp16 [K / 128, N], one per group of 128 k and column.
 *   zeros   : uint8 [K / 128, N], zero points 0..15.
 *   y       : fp16 [M, N] output, fp32 accumulation, rounded once.
 * Sizes: 1 <= M <= 128 (decode-sized token counts), N a multiple of 128, K a
 * multiple of 128 (else ATTN_ERR_UNSUPPORTED); non-positive sizes or a null
 * pointer: ATTN_ERR_INVALID_ARG; unaligned pointers: ATTN_ERR_MISALIGNED.
 * Asynchronous on `stream`; nothing is allocated; a pipeline wait that runs
 * out is reported through attn_get_device_status() like the attention calls.
 * w4a16_gemm launches one CTA per 128 output columns; w4a16_gemm_splitk below
 * balances the work over all SMs and is the faster call when N / 128 is not a
 * multiple of twice the SM count.
 */
#ifndef W4A16_B200_H
#define W4A16_B200_H

#include "attn_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

ATTN_API attn_status w4a16_gemm(const void* x, const void* qweight, const void* scales, const void* zeros,
                                void* y, int M, int N, int K, void* stream);

/*
 * w4a16_gemm_splitk - the same product with the K slices balanced over every
 * SM (split-K). w4a16_gemm gives each CTA one 128-column tile and all of its
 * K; when the tile count N / 128 is not a multiple of the CTAs the GPU holds at
 * once (two per SM), some SMs run two tiles while others run one, and the
 * launch takes as long as the busiest SM. Here the (tile, 128-deep slice) units
 * are cut into equal runs, one per CTA, and a tile whose slices fall into
 * several runs is summed from fp32 partials. Each run's partial covers its
 * share of the tile's K, and the last CTA to finish a tile adds the partials
 * in a fixed order (by run), so repeated calls give bit-identical Y. The
 * summation order differs from w4a16_gemm's (one accumulator along all of K),
 * so the two entry points agree to fp32 rounding, not bit for bit.
 *   workspace       : device memory of at least
 *                     w4a16_gemm_splitk_workspace_bytes(M, N, K) bytes, 16-byte
 *                     aligned, owned by the caller. Zero it once after
 *                     allocating it: its first 16 * N / 128 bytes are tickets
 *                     that every call finds zero and leaves zero. After a call
 *                     whose device status is not ATTN_OK (a pipeline timeout),
 *                     zero it again before its next use. Calls that overlap on
 *                     the GPU need separate workspaces.
 *   workspace_bytes : its size in bytes.
 * Other arguments, layouts and errors as for w4a16_gemm, plus
 * ATTN_ERR_INVALID_ARG for a null workspace or one smaller than required.
 * One launch on `stream`; nothing is allocated.
 */
ATTN_API attn_status w4a16_gemm_splitk(const void* x, const void* qweight, const void* scales, const void* zeros,
                                       void* y, void* workspace, size_t workspace_bytes, int M, int N, int K,
                                       void* stream);

/* w4a16_gemm_splitk_workspace_bytes - workspace w4a16_gemm_splitk needs for
 * this shape: the tickets (16 bytes per 128 columns, rounded up to 256 bytes)
 * and two fp32 partial slots of M (rounded up to 16) x 128 values per CTA, for
 * at most 296 CTAs (two per SM of a B200). 0 for an invalid or unsupported
 * shape. Host only; launches nothing. */
ATTN_API size_t w4a16_gemm_splitk_workspace_bytes(int M, int N, int K);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_B200_H */
