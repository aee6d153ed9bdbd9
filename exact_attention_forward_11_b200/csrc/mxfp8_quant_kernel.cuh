// mxfp8_quant_kernel.cuh - bf16 -> MXFP8 (E4M3 codes, one E8M0 scale per 32
// consecutive values).
//
// Format ("Efficient MoE training for biological foundation models", the
// low-precision paragraph: MXFP8 with one shared power-of-two scale per block of
// 32 values; the arithmetic is the OCP Microscaling definition): for each block,
// E = floor(log2(max |v|)) - 8 clamped to [-127, 127] (E = 0 for an all-zero
// block), scale byte E + 127, codes = E4M3 round-to-nearest-even, saturating to
// +-448, of v * 2^-E.
//
// Exactness: the block maximum of bf16 values is exact in fp32, and its binade is
// read from the fp32 exponent field (an fp32-subnormal maximum, below 2^-126,
// always gives the clamped E = -127). v * 2^-E is an exact fp32 product whenever
// it is at least 2^-126; smaller products lie far below E4M3's smallest half-step
// (2^-10) and round to a signed zero either way. The conversion is the
// hardware's cvt.rn.satfinite.e4m3x2.f32.
//
// Layout: the input is a flat sequence of 32-value blocks (any [rows, d] array
// with d a multiple of 32, row-major), four lanes per block, eight values per
// lane (one 16-byte load, one 8-byte store), so a warp reads 512 contiguous bytes.
// Inputs must be finite.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "status.cuh"

namespace attn {

constexpr int kMxQuantThreads = 256;
constexpr int kMxQuantUnroll = 4;

__device__ __forceinline__ int mx_block_exponent(float amax) {
  const int ef = static_cast<int>(__float_as_uint(amax) >> 23);   // amax >= 0
  if (amax == 0.f) return 0;
  if (ef == 0) return -127;
  const int e = ef - 127 - 8;
  return e < -127 ? -127 : e;
}

__global__ void __launch_bounds__(kMxQuantThreads)
    mxfp8_quantize_sm100(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ codes,
                         uint8_t* __restrict__ sf, long long nblk) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nthr = static_cast<long long>(gridDim.x) * blockDim.x;
  const int sub = threadIdx.x & 3;                 // eighth of the block this lane holds
  const int gq = (threadIdx.x & 31) >> 2;          // block of this lane within the warp's eight
  const long long per_iter = nthr >> 2;            // blocks per pass of the grid
  // the loop runs on the warp's first block, so all 32 lanes take the shuffles
  for (long long w0 = (tid >> 2) - gq; w0 < nblk; w0 += per_iter * kMxQuantUnroll) {
    const long long b0 = w0 + gq;
    uint4 raw[kMxQuantUnroll];
#pragma unroll
    for (int k = 0; k < kMxQuantUnroll; ++k) {
      const long long b = b0 + k * per_iter;
      raw[k] = b < nblk ? *reinterpret_cast<const uint4*>(x + b * 32 + sub * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kMxQuantUnroll; ++k) {
      const long long b = b0 + k * per_iter;   // the same for the four lanes of a block
      float v[8];
      const uint32_t w[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const int e = mx_block_exponent(amax);
      const float inv = __int_as_float((127 - e) << 23);   // 2^-E, E in [-127, 119]: a normal fp32
      if (b < nblk && dbg_ok(b >= 0, kSiteMxBlock, static_cast<unsigned long long>(b))) {
        const uint32_t lo = b200::pack_e4m3x4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
        const uint32_t hi = b200::pack_e4m3x4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
        *reinterpret_cast<uint2*>(codes + b * 32 + sub * 8) = make_uint2(lo, hi);
        if (sub == 0) sf[b] = static_cast<uint8_t>(e + 127);
      }
    }
  }
}

}  // namespace attn
