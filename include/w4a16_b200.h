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
 */
#ifndef W4A16_B200_H
#define W4A16_B200_H

#include "attn_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

ATTN_API attn_status w4a16_gemm(const void* x, const void* qweight, const void* scales, const void* zeros,
                                void* y, int M, int N, int K, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_B200_H */
