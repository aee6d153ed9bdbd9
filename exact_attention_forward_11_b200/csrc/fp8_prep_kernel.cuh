// fp8_prep_kernel.cuh - incoherent rotation and block quantisation to E4M3.
//
// "FlashAttention scaling, multi-GPU training and weight quantization", section 1,
// FlashAttention-3 FP8 bullet: Q and K are multiplied by a random orthogonal
// matrix before quantisation so that outliers are spread over all channels, and
// each small tile gets its own scale. Here a tile is 128 tokens x 128 channels of
// one (batch, head), which is also the attention kernel's Q/K/V tile, so one scale
// applies to a whole MMA operand tile.
//
// Definition (fixed so the result is unique and checkable bit for bit):
//   y[i][c] = sum_k x[i][k] * R[k][c], accumulated in fp32 in increasing k order
//             (x and R are bf16, so every product is exact in fp32 and an FMA
//             rounds exactly once per step);
//   scale   = max |y| over the tile / 448 (IEEE fp32 division), 1 for all zeros;
//   code    = cvt.rn.satfinite E4M3 of y / scale (IEEE fp32 division).
// One CTA per tile; 256 threads, each owning an 8 x 8 block of outputs. Rows past
// N read as zero and are not written.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace attn {

constexpr int kPrepThreads = 256;
constexpr int kPrepTile = 128;
constexpr int kPrepPad = 4;  // floats of padding per shared-memory row
constexpr int kPrepSmemBytes = 2 * kPrepTile * (kPrepTile + kPrepPad) * 4 + 64;

__global__ void __launch_bounds__(kPrepThreads)
    fp8_rotate_quantize(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ rot,
                        uint8_t* __restrict__ x8, float* __restrict__ scales, int N) {
  extern __shared__ float prep_smem[];
  constexpr int LD = kPrepTile + kPrepPad;
  float* xt = prep_smem;                        // x transposed: xt[k][row]
  float* rs = prep_smem + kPrepTile * LD;       // R: rs[k][col]
  float* red = rs + kPrepTile * LD;             // 8 warp maxima

  const int T = (N + kPrepTile - 1) / kPrepTile;
  const int bh = blockIdx.x / T;
  const int tile = blockIdx.x % T;
  const int row0 = tile * kPrepTile;
  const int rows = min(kPrepTile, N - row0);
  const __nv_bfloat16* xb = x + (static_cast<size_t>(bh) * N + row0) * kPrepTile;
  const int tid = threadIdx.x;

  // stage x (transposed) and R as fp32; 8 bf16 per 16-byte load
  for (int i = tid; i < kPrepTile * kPrepTile / 8; i += kPrepThreads) {
    const int r = i / (kPrepTile / 8), c8 = (i % (kPrepTile / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows) v = *reinterpret_cast<const uint4*>(xb + static_cast<size_t>(r) * kPrepTile + c8);
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
    for (int e = 0; e < 8; ++e) xt[(c8 + e) * LD + r] = __bfloat162float(h[e]);
  }
  if (rot != nullptr) {
    for (int i = tid; i < kPrepTile * kPrepTile / 8; i += kPrepThreads) {
      const int r = i / (kPrepTile / 8), c8 = (i % (kPrepTile / 8)) * 8;
      const uint4 v = *reinterpret_cast<const uint4*>(rot + static_cast<size_t>(r) * kPrepTile + c8);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int e = 0; e < 8; ++e) rs[r * LD + c8 + e] = __bfloat162float(h[e]);
    }
  }
  __syncthreads();

  const int ty = tid / 16, tx = tid % 16;   // rows ty*8.., cols tx*8..
  float acc[8][8];
  if (rot != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < kPrepTile; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(xt + k * LD + ty * 8);
      const float4 a1 = *reinterpret_cast<const float4*>(xt + k * LD + ty * 8 + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(rs + k * LD + tx * 8);
      const float4 b1 = *reinterpret_cast<const float4*>(rs + k * LD + tx * 8 + 4);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = xt[(tx * 8 + j) * LD + ty * 8 + i];
  }

  // tile amax (max is exact in any order)
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(acc[i][j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kPrepThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (tid == 0) scales[static_cast<size_t>(bh) * T + tile] = sc;

  uint8_t* ob = x8 + (static_cast<size_t>(bh) * N + row0) * kPrepTile;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = ty * 8 + i;
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      w[h] = b200::pack_e4m3x4(__fdiv_rn(acc[i][4 * h], sc), __fdiv_rn(acc[i][4 * h + 1], sc),
                               __fdiv_rn(acc[i][4 * h + 2], sc), __fdiv_rn(acc[i][4 * h + 3], sc));
    if (r < rows) *reinterpret_cast<uint2*>(ob + static_cast<size_t>(r) * kPrepTile + tx * 8) = make_uint2(w[0], w[1]);
  }
}

}  // namespace attn
