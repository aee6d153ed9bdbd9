// w4a16_kernel.cuh - GEMM with 4-bit weights dequantised on the fly (W4A16).
//
// "FlashAttention scaling, multi-GPU training and weight quantization", section 3,
// the W4A16 kernels paragraph: the packed 4-bit weights (eight to a 32-bit word)
// are read from HBM, unpacked in registers with shifts and masks, turned into
// 16-bit floats with the stored scale and zero point, and fed to the tensor cores
// with the 16-bit activations; the expanded weights never go back to memory.
//
//   Y[M, N] = X[M, K] W[K, N],  W[k, n] = fp16((q[k, n] - z[g, n]) * s[g, n]),
//   g = k / 128, q from qweight[k / 8, n] (weight 8w + PERM[i] in bits 4i..4i+3,
//   PERM = 0 2 4 6 1 3 5 7), fp32 accumulation, Y rounded to fp16.
//
// Decode-sized M (1..128 tokens) makes the GEMM HBM-bound on the weights (half a
// byte per weight), so the layout is chosen for a stream: one CTA per 128 output
// columns walks K in 128-deep slices. The MMA is issued with the operands swapped
// (D[128 columns n][M tokens] = W^T X^T) so that M = 128 is the weight side and
// the token count only sets the MMA's N (padded to a multiple of 16). The
// dequantised weights go straight from registers into tensor memory (one thread
// per output column = one TMEM lane, tcgen05.st) and are the MMA's A operand
// from TMEM; only the small X slice is read from shared memory by the MMA.
//
// CTA: 12 warps. warp 0 TMA producer (weight words, scales, zero points and the X
// slice of each K slice into a ring of up to 8 stages), warp 1 MMA issuer (owns
// TMEM), warps 2-3 idle, warps 4-11 dequantise (thread t of quarter q: column
// n0 + 32 q + t; warps 4-7 take the first 8 words of a slice, 8-11 the last 8)
// and warps 4-7 write Y. Two CTAs fit on an SM (85 registers per thread).
// TMEM: three (two for M > 64) 64-column A buffers (a 128-deep slice of fp16
// pairs each) and the MPAD-column fp32 accumulator. Every wait is bounded (Waiter).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "sm100.cuh"
#include "status.cuh"

namespace attn {

struct W4Cfg {
  // dequantisation warpgroups: with two, the two warps of a TMEM lane quarter
  // each unpack half of a slice's words (64 of its 128 k), so one warp's TMEM
  // store and wait overlap the other's unpacking
#ifndef ATTN_W4_SPLIT
#define ATTN_W4_SPLIT 2
#endif
  static constexpr int SPLIT = ATTN_W4_SPLIT;
  static constexpr int WORDS = 16 / SPLIT;     // packed words per thread per slice
  static constexpr int THREADS = 128 + 128 * SPLIT;
  static constexpr int MAX_NST = 8;            // ring stages: as many as ~110 KB of shared memory holds
  static constexpr int GROUP = 128;            // k per scale / zero point = k per slice
  static constexpr int BN = 128;               // output columns per CTA
  static constexpr int WQ_BYTES = 16 * BN * 4; // 16 words (128 k) x 128 columns
  static constexpr int S_BYTES = BN * 2;
  static constexpr int Z_BYTES = BN;
  static constexpr int MAX_M = 128;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t T_A = 0;           // A buffers: 64 columns each from column 0
  static constexpr int MAX_NA = 3;
  // A buffers in flight: three when the accumulator (MPAD columns after them)
  // leaves room in the 256 columns, else two
  __host__ __device__ static constexpr int na(int mpad) { return mpad <= 64 ? 3 : 2; }
  __host__ __device__ static constexpr uint32_t t_d(int mpad) { return 64u * na(mpad); }
  // stage layout (offsets inside a stage; X first so its chunks stay 1024-aligned)
  __host__ __device__ static constexpr int x_chunk(int mpad) { return mpad * 128; }
  __host__ __device__ static constexpr int stage_bytes(int mpad) {
    return ((2 * x_chunk(mpad) + WQ_BYTES + S_BYTES + Z_BYTES) + 1023) / 1024 * 1024;
  }
  // stages in flight: 8 for small M (two CTAs per SM then keep ~200 KB of weights in
  // flight per SM), fewer as the X slice grows
  __host__ __device__ static constexpr int nst(int mpad) {
    return (110 * 1024) / stage_bytes(mpad) < 2 ? 2
           : ((110 * 1024) / stage_bytes(mpad) > MAX_NST ? MAX_NST : (110 * 1024) / stage_bytes(mpad));
  }
  __host__ __device__ static constexpr int bar_offset(int mpad) { return nst(mpad) * stage_bytes(mpad); }
  __host__ __device__ static constexpr int smem_bytes(int mpad) {
    return bar_offset(mpad) + (2 * MAX_NST + 2 * MAX_NA + 2) * 8 + 16 + 1024;
  }
  // the largest smem_bytes over every M (the kernel attribute must cover all)
  __host__ static constexpr int max_smem_bytes() {
    int m = 0;
    for (int mp = 16; mp <= MAX_M; mp += 16) m = smem_bytes(mp) > m ? smem_bytes(mp) : m;
    return m;
  }
};

struct W4Params {
  int M, N, K;
  int mpad;                  // M rounded up to a multiple of 16
  __half* y;                 // [M, N]
  uint64_t timeout_cycles;
};

__global__ void __launch_bounds__(W4Cfg::THREADS, 2)
    w4a16_gemm_sm100(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_z,
                     const W4Params p) {
  using namespace b200;
  using C = W4Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int mpad = p.mpad;
  const int SB = C::stage_bytes(mpad);
  const int XC = C::x_chunk(mpad);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::bar_offset(mpad));
  const int NST = C::nst(mpad);
  uint64_t* full = bars;                     // NST: TMA bytes
  uint64_t* empty = full + C::MAX_NST;       // NST: MMA commit (X read) + 4 dequant warps (words read)
  const int NA = C::na(mpad);
  const uint32_t T_D = C::t_d(mpad);
  uint64_t* a_full = empty + C::MAX_NST;     // NA: 4 dequant warps
  uint64_t* a_empty = a_full + C::MAX_NA;    // NA: MMA commit
  uint64_t* done = a_empty + C::MAX_NA;      // 1
  uint64_t* drain_bar = done + 1;            // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::MAX_NST + 2 * C::MAX_NA + 2);
  uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::BN;
  const int G = p.K / C::GROUP;              // slices

  auto x_at = [&](int s) { return smem + s * SB; };
  auto w_at = [&](int s) { return reinterpret_cast<const uint32_t*>(smem + s * SB + 2 * XC); };
  auto s_at = [&](int s) { return reinterpret_cast<const __half*>(smem + s * SB + 2 * XC + C::WQ_BYTES); };
  auto z_at = [&](int s) { return smem + s * SB + 2 * XC + C::WQ_BYTES + C::S_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1 + 4 * C::SPLIT);
    }
    for (int b = 0; b < NA; ++b) {
      mbar_init(a_full + b, 4 * C::SPLIT);
      mbar_init(a_empty + b, 1);
    }
    mbar_init(done, 1);
    mbar_init(drain_bar, 1);
    *abort_word = 0u;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Waiter waiter{abort_word, p.timeout_cycles};
  auto wait_all = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, waiter.wait(bar, parity)); };
  bool ok = true;

  if (warp == 0) {
    // ======================= producer =======================
    if (elect_one()) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_w);
      tma_prefetch_desc(&tm_s);
      tma_prefetch_desc(&tm_z);
    }
    __syncwarp();
    const uint64_t pol_w = l2_policy_evict_first();   // weights are read once
    const uint64_t pol_x = l2_policy_evict_last();    // X is read by every CTA
    const uint32_t bytes = static_cast<uint32_t>(2 * XC + C::WQ_BYTES + C::S_BYTES + C::Z_BYTES);
    int g = 0;
    for (; g < G; ++g) {
      const int s = g % NST;
      if (g >= NST && !(ok = wait_all(empty + s, ((g / NST) - 1) & 1))) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(full + s, bytes);
        tma_load_3d(x_at(s), &tm_x, full + s, g * C::GROUP, 0, 0, pol_x);
        tma_load_3d(x_at(s) + XC, &tm_x, full + s, g * C::GROUP + 64, 0, 0, pol_x);
        tma_load_3d(const_cast<uint32_t*>(w_at(s)), &tm_w, full + s, n0, g * 16, 0, pol_w);
        tma_load_3d(const_cast<__half*>(s_at(s)), &tm_s, full + s, n0, g, 0, pol_w);
        tma_load_3d(z_at(s), &tm_z, full + s, n0, g, 0, pol_w);
      }
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) record_timeout();
      const uint64_t t0 = sm_clock();
      for (int j = (g > NST ? g - NST : 0); j < g; ++j)
        while (!mbar_try_wait(full + (j % NST), (j / NST) & 1) && sm_clock() - t0 < p.timeout_cycles) {
        }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    const uint32_t leader = elect_one() ? 1u : 0u;
    const uint32_t idesc = instr_desc(0u /* f16 */, 128, static_cast<uint32_t>(mpad), 0, 0);
    constexpr uint32_t hi = smem_desc_hi(1024);
    const uint32_t x_lo = smem_desc_lo(smem_addr(smem), 16);
    for (int g = 0; g < G; ++g) {
      const int s = g % NST, b = g % NA;
      if (!(ok = wait_all(full + s, (g / NST) & 1))) break;
      if (!(ok = wait_all(a_full + b, (g / NA) & 1))) break;
      tc_fence_after();
      const uint32_t xa = x_lo + ((s * SB) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = ((kk >> 2) * XC + (kk & 3) * 32) >> 4;
        mma_f16_ts(tmem_base + T_D, tmem_base + C::T_A + 64 * b + 8 * kk, smem_desc(xa + off, hi), idesc,
                   (g > 0 || kk > 0) ? 1u : 0u, leader);
      }
      mma_commit(empty + s, leader);
      mma_commit(a_empty + b, leader);
    }
    if (ok) mma_commit(done, leader);
    if (!ok && lane == 0) record_timeout();
    mma_commit(drain_bar, leader);
    const uint64_t t0 = sm_clock();
    while (!mbar_try_wait(drain_bar, 0) && sm_clock() - t0 < p.timeout_cycles) {
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ======================= dequantise, then Y =======================
    const int wq = warp & 3;                         // TMEM lane quarter
    const int h = (warp - 4) >> 2;                   // which words of the slice (SPLIT 2)
    const int t = wq * 32 + lane;                    // output column n0 + t, TMEM lane t
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    for (int g = 0; g < G; ++g) {
      const int s = g % NST, b = g % NA;
      if (!(ok = wait_all(full + s, (g / NST) & 1))) break;
      if (g >= NA && !(ok = wait_all(a_empty + b, ((g / NA) - 1) & 1))) break;
      const __half2 ss = __half2half2(s_at(s)[t]);
      // 1024 + z as fp16: the unpacked words below hold 1024 + q (exponent bits
      // 0x6400 with q in the low mantissa bits), so one subtraction gives q - z exactly
      const __half zh = __ushort_as_half(static_cast<unsigned short>(0x6400u | z_at(s)[t]));
      const __half2 zz = __half2half2(zh);
      const uint32_t* wrow = w_at(s);
      uint32_t pk[4 * C::WORDS];
#pragma unroll
      for (int i = 0; i < C::WORDS; ++i) {
        const uint32_t word = wrow[(C::WORDS * h + i) * C::BN + t];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // bits 4j..4j+3 (weight 8i+2j) into the low half, bits 16+4j.. (8i+2j+1) into the high half
          const uint32_t v = ((word >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
          const __half2 h = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&v), zz), ss);
          pk[4 * i + j] = *reinterpret_cast<const uint32_t*>(&h);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);         // this warp's words, scale and zero are read
#pragma unroll
      for (int q = 0; q < C::WORDS / 8; ++q)
        tmem_st32(tmem_base + lane_off + C::T_A + 64 * b + 4 * C::WORDS * h + 32 * q, pk + 32 * q);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(a_full + b);
    }
    // Y: the first warpgroup reads the accumulator and writes the tile
    if (ok && h == 0) ok = wait_all(done, 0);
    if (!ok) {
      if (lane == 0) record_timeout();
    } else if (h == 0) {
      tc_fence_after();
      __half* ycol = p.y + n0 + t;
      const bool col_ok = dbg_ok(n0 + t < p.N, kSiteW4Out, static_cast<unsigned>(n0 + t));
      for (int c0 = 0; c0 < mpad; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_base + lane_off + T_D + c0, v);
        tmem_ld_wait<16>(v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = c0 + i;
          if (m < p.M && col_ok) ycol[static_cast<size_t>(m) * p.N] = __float2half_rn(__uint_as_float(v[i]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace attn
