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
//
// Persistent CTAs (one per SM) of 256 threads walk the tiles; R is staged once
// per CTA as fp32. Thread (ty, tx) = (tid % 16, tid / 16) owns the outputs of
// rows ty + 16 i (i < 8) and columns 8 tx .. 8 tx + 7: interleaved rows make the
// float4 reads of x from shared memory conflict-free, and the k loop runs four
// steps per round of loads while every output still accumulates in k order
// (two columns per packed fma.rn.f32x2).
// Rows past N read as zero and are not written.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace attn {

constexpr int kPrepThreads = 256;
constexpr int kPrepTile = 128;
constexpr int kPrepLd = kPrepTile + 4;  // floats per shared-memory row
constexpr int kPrepSmemBytes = 2 * kPrepTile * kPrepLd * 4 + 8 * 4 + 16;

__global__ void __launch_bounds__(kPrepThreads, 1)
    fp8_rotate_quantize(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ rot,
                        uint8_t* __restrict__ x8, float* __restrict__ scales, int N, int num_tiles) {
  extern __shared__ __align__(16) float prep_smem[];
  float* xs = prep_smem;                         // x tile, row-major [128][kPrepLd]
  float* rs = prep_smem + kPrepTile * kPrepLd;   // R, row-major [128][kPrepLd]
  float* red = rs + kPrepTile * kPrepLd;         // 8 warp maxima
  const int tid = threadIdx.x;
  const int ty = tid % 16, tx = tid / 16;
  const int T = (N + kPrepTile - 1) / kPrepTile;
  const bool rotate = rot != nullptr;

  if (rotate) {
    for (int i = tid; i < kPrepTile * kPrepTile / 8; i += kPrepThreads) {
      const int r = i / (kPrepTile / 8), c8 = (i % (kPrepTile / 8)) * 8;
      const uint4 v = *reinterpret_cast<const uint4*>(rot + static_cast<size_t>(r) * kPrepTile + c8);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
      float4 lo = make_float4(__bfloat162float(h[0]), __bfloat162float(h[1]), __bfloat162float(h[2]),
                              __bfloat162float(h[3]));
      float4 hi = make_float4(__bfloat162float(h[4]), __bfloat162float(h[5]), __bfloat162float(h[6]),
                              __bfloat162float(h[7]));
      *reinterpret_cast<float4*>(rs + r * kPrepLd + c8) = lo;
      *reinterpret_cast<float4*>(rs + r * kPrepLd + c8 + 4) = hi;
    }
  }

  for (int tile_id = blockIdx.x; tile_id < num_tiles; tile_id += gridDim.x) {
    const int bh = tile_id / T;
    const int tile = tile_id % T;
    const int row0 = tile * kPrepTile;
    const int rows = min(kPrepTile, N - row0);
    const __nv_bfloat16* xb = x + (static_cast<size_t>(bh) * N + row0) * kPrepTile;

    __syncthreads();   // previous tile's readers of xs / red are done (and R is staged)
    for (int i = tid; i < kPrepTile * kPrepTile / 8; i += kPrepThreads) {
      const int r = i / (kPrepTile / 8), c8 = (i % (kPrepTile / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < rows) v = *reinterpret_cast<const uint4*>(xb + static_cast<size_t>(r) * kPrepTile + c8);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
      float4 lo = make_float4(__bfloat162float(h[0]), __bfloat162float(h[1]), __bfloat162float(h[2]),
                              __bfloat162float(h[3]));
      float4 hi = make_float4(__bfloat162float(h[4]), __bfloat162float(h[5]), __bfloat162float(h[6]),
                              __bfloat162float(h[7]));
      *reinterpret_cast<float4*>(xs + r * kPrepLd + c8) = lo;
      *reinterpret_cast<float4*>(xs + r * kPrepLd + c8 + 4) = hi;
    }
    __syncthreads();

    float acc[8][8];
    if (rotate) {
      // packed FMAs on column pairs: fma.rn.f32x2 rounds each lane exactly like a
      // scalar fma.rn, so every output still accumulates in k order, once-rounded
      // per step (bit-identical), at half the instruction count
      uint64_t acc2[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc2[i][j] = 0ull;
#pragma unroll 1
      for (int k0 = 0; k0 < kPrepTile; k0 += 4) {
        float4 xa[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) xa[i] = *reinterpret_cast<const float4*>(xs + (ty + 16 * i) * kPrepLd + k0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const float4 r0 = *reinterpret_cast<const float4*>(rs + (k0 + kk) * kPrepLd + tx * 8);
          const float4 r1 = *reinterpret_cast<const float4*>(rs + (k0 + kk) * kPrepLd + tx * 8 + 4);
          const uint64_t b2[4] = {b200::f2_pack(r0.x, r0.y), b200::f2_pack(r0.z, r0.w), b200::f2_pack(r1.x, r1.y),
                                  b200::f2_pack(r1.z, r1.w)};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = kk == 0 ? xa[i].x : kk == 1 ? xa[i].y : kk == 2 ? xa[i].z : xa[i].w;
            const uint64_t a2 = b200::f2_pack(a, a);
#pragma unroll
            for (int j = 0; j < 4; ++j) acc2[i][j] = b200::f2_fma(a2, b2[j], acc2[i][j]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) b200::f2_unpack(acc2[i][j], acc[i][2 * j], acc[i][2 * j + 1]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 v0 = *reinterpret_cast<const float4*>(xs + (ty + 16 * i) * kPrepLd + tx * 8);
        const float4 v1 = *reinterpret_cast<const float4*>(xs + (ty + 16 * i) * kPrepLd + tx * 8 + 4);
        acc[i][0] = v0.x; acc[i][1] = v0.y; acc[i][2] = v0.z; acc[i][3] = v0.w;
        acc[i][4] = v1.x; acc[i][5] = v1.y; acc[i][6] = v1.z; acc[i][7] = v1.w;
      }
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
      const int r = ty + 16 * i;
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        w[h] = b200::pack_e4m3x4(__fdiv_rn(acc[i][4 * h], sc), __fdiv_rn(acc[i][4 * h + 1], sc),
                                 __fdiv_rn(acc[i][4 * h + 2], sc), __fdiv_rn(acc[i][4 * h + 3], sc));
      if (r < rows) *reinterpret_cast<uint2*>(ob + static_cast<size_t>(r) * kPrepTile + tx * 8) = make_uint2(w[0], w[1]);
    }
  }
}

}  // namespace attn
