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
// byte per weight), so the layout is chosen for a stream: a CTA walks K in
// 128-deep slices of 128 output columns. The work is the list of (column tile,
// slice) units, tile-major; CTA c of C takes units [c U / C, (c+1) U / C). With
// C = the number of tiles every CTA owns one whole tile. With C = two per SM
// (balanced split-K) a CTA's run may start or end inside a tile: the part of a
// tile it covers is a segment, written as an fp32 partial to a caller workspace
// slot (2c for the run's first tile, 2c+1 for its last); the warp that takes the
// last ticket of its tile's 32-column quarter adds the tile's partials in CTA
// order (so the sum does not depend on which CTA finishes last), writes Y and
// resets the ticket. The MMA is issued with the operands swapped
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
// and warps 4-7 write each segment's Y or partial. Two CTAs fit on an SM.
// TMEM: three (two for M > 64) 64-column A buffers (a 128-deep slice of fp16
// pairs each) and the MPAD-column fp32 accumulator, which the MMA reuses for the
// next segment once warps 4-7 have read it. Every wait is bounded (Waiter); the
// tickets are atomics, never waited on.
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
    return bar_offset(mpad) + (2 * MAX_NST + 2 * MAX_NA + 3) * 8 + 32 + 1024;
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
  int ctas;                  // C: CTAs of the launch (the grid)
  long long units;           // U = (N / 128) * (K / 128)
  __half* y;                 // [M, N]
  float* part;               // [2 C][mpad][128] fp32 segment partials (split-K only)
  uint32_t* tickets;         // [4 N / 128] per tile quarter, zero between launches (split-K only)
  uint64_t timeout_cycles;
};

// First unit of CTA c, and the CTA whose run holds unit u.
__host__ __device__ __forceinline__ long long w4_unit0(int c, long long U, int C) {
  return static_cast<long long>(c) * U / C;
}
__host__ __device__ __forceinline__ int w4_cta_of(long long u, long long U, int C) {
  return static_cast<int>(((u + 1) * C - 1) / U);
}

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
  uint64_t* seg_done = a_empty + C::MAX_NA;  // 1: MMA commit at each segment's end
  uint64_t* d_free = seg_done + 1;           // 1: warps 4-7 have read the accumulator
  uint64_t* drain_bar = d_free + 1;          // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::MAX_NST + 2 * C::MAX_NA + 3);
  uint32_t* abort_word = tmem_slot + 1;
  int* run_info = reinterpret_cast<int*>(tmem_slot + 2);   // [units in the run, first tile, first slice]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.K / C::GROUP;              // slices per tile
  const long long U = p.units;

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
    mbar_init(seg_done, 1);
    mbar_init(d_free, 4);
    mbar_init(drain_bar, 1);
    *abort_word = 0u;
    // the run, computed once here (64-bit divisions) and read back from shared memory
    const long long u0 = w4_unit0(blockIdx.x, U, p.ctas);
    run_info[0] = static_cast<int>(w4_unit0(blockIdx.x + 1, U, p.ctas) - u0);
    run_info[1] = static_cast<int>(u0 / G);
    run_info[2] = static_cast<int>(u0 - static_cast<long long>(run_info[1]) * G);
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
  // this CTA's run: n_units units from slice g0 of tile tile0
  const int n_units = run_info[0], tile0 = run_info[1], g0 = run_info[2];
  const Waiter waiter{abort_word, p.timeout_cycles};
  auto wait_all = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, waiter.wait(bar, parity)); };
  bool ok = true;

  // Every role walks the run as segments (outer loop: one tile each) of slices
  // [gs, ge) (inner loop); i counts units across the run for the ring phases.
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
    int i = 0, s = 0, r = 0;                 // unit, its ring stage, and the ring round
    for (int tile = tile0, gs = g0; ok && i < n_units; ++tile, gs = 0) {
      const int ge = min(G, gs + (n_units - i));
      const int n0 = tile * C::BN;
      for (int g = gs; g < ge; ++g, ++i, s = (s == NST - 1 ? 0 : s + 1), r += (s == 0)) {
        if (r > 0 && !(ok = wait_all(empty + s, (r - 1) & 1))) break;
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
    }
    if (!ok) {
      if (lane == 0) record_timeout();
      const uint64_t t0 = sm_clock();
      for (int j = (i > NST ? i - NST : 0); j < i; ++j)
        while (!mbar_try_wait(full + (j % NST), (j / NST) & 1) && sm_clock() - t0 < p.timeout_cycles) {
        }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    const uint32_t leader = elect_one() ? 1u : 0u;
    const uint32_t idesc = instr_desc(0u /* f16 */, 128, static_cast<uint32_t>(mpad), 0, 0);
    constexpr uint32_t hi = smem_desc_hi(1024);
    const uint32_t x_lo = smem_desc_lo(smem_addr(smem), 16);
    int i = 0, s = 0, r = 0, b = 0, ra = 0;  // unit; ring stage and round; A buffer and its round
    for (int seg = 0, gs = g0; ok && i < n_units; ++seg, gs = 0) {
      const int ge = min(G, gs + (n_units - i));
      // the accumulator is reused: the previous segment must have been read
      if (seg > 0 && !(ok = wait_all(d_free, (seg - 1) & 1))) break;
      for (int g = gs; g < ge; ++g, ++i, s = (s == NST - 1 ? 0 : s + 1), r += (s == 0),
               b = (b == NA - 1 ? 0 : b + 1), ra += (b == 0)) {
        if (!(ok = wait_all(full + s, r & 1))) break;
        if (!(ok = wait_all(a_full + b, ra & 1))) break;
        tc_fence_after();
        const uint32_t xa = x_lo + ((s * SB) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * XC + (kk & 3) * 32) >> 4;
          mma_f16_ts(tmem_base + T_D, tmem_base + C::T_A + 64 * b + 8 * kk, smem_desc(xa + off, hi), idesc,
                     (g > gs || kk > 0) ? 1u : 0u, leader);
        }
        mma_commit(empty + s, leader);
        mma_commit(a_empty + b, leader);
      }
      if (ok) mma_commit(seg_done, leader);
    }
    if (!ok && lane == 0) record_timeout();
    mma_commit(drain_bar, leader);
    const uint64_t t0 = sm_clock();
    while (!mbar_try_wait(drain_bar, 0) && sm_clock() - t0 < p.timeout_cycles) {
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ======================= dequantise; Y or partial at each segment's end =======================
    const int wq = warp & 3;                         // TMEM lane quarter
    const int h = (warp - 4) >> 2;                   // which words of the slice (SPLIT 2)
    const int t = wq * 32 + lane;                    // output column n0 + t, TMEM lane t
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    int i = 0, s = 0, r = 0, b = 0, ra = 0;  // unit; ring stage and round; A buffer and its round
    for (int seg = 0, tile = tile0, gs = g0; ok && i < n_units; ++seg, ++tile, gs = 0) {
      const int ge = min(G, gs + (n_units - i));
      for (int g = gs; g < ge; ++g, ++i, s = (s == NST - 1 ? 0 : s + 1), r += (s == 0),
               b = (b == NA - 1 ? 0 : b + 1), ra += (b == 0)) {
        if (!(ok = wait_all(full + s, r & 1))) break;
        if (ra > 0 && !(ok = wait_all(a_empty + b, (ra - 1) & 1))) break;
        const __half sh = s_at(s)[t];
        const uint32_t zb = z_at(s)[t];
        const __half2 ss = __half2half2(sh);
        // 1024 + z as fp16: the unpacked words below hold 1024 + q (exponent bits
        // 0x6400 with q in the low mantissa bits), so one subtraction gives q - z exactly
        const __half2 zz = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6400u | zb)));
        // Nibbles masked in place one position higher (bits 4..7 of a half) read as
        // 1024 + 16 q: less 1024 + 16 z that is 16 (q - z), exact, and times s / 16 it is
        // the same real product (q - z) s, rounded once: the same fp16 value, one shift
        // fewer per nibble pair. Taken when s / 16 is exact (s * 2^-4 times 16 gives s
        // back) for every lane of the warp; otherwise every pair goes the shifting way.
        const __half s16 = __hmul(sh, __ushort_as_half(static_cast<unsigned short>(0x2C00u)));   // 2^-4
        const bool exact16 = __heq(__hmul(s16, __ushort_as_half(static_cast<unsigned short>(0x4C00u))), sh);
        const uint32_t* wrow = w_at(s);
        uint32_t pk[4 * C::WORDS];
        if (__all_sync(0xffffffffu, exact16)) {
          const __half2 ss16 = __half2half2(s16);
          const __half2 zz16 = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6400u | (zb << 4))));
#pragma unroll
          for (int k = 0; k < C::WORDS; ++k) {
            const uint32_t word = wrow[(C::WORDS * h + k) * C::BN + t];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // pairs 2j, 2j+1: bits 4j..4j+3 and 16+4j..; odd j stays 4 bits up
              const uint32_t src = j < 2 ? word : word >> 8;
              const uint32_t v = (src & ((j & 1) ? 0x00F000F0u : 0x000F000Fu)) | 0x64006400u;
              const __half2 hv = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&v), (j & 1) ? zz16 : zz),
                                         (j & 1) ? ss16 : ss);
              pk[4 * k + j] = *reinterpret_cast<const uint32_t*>(&hv);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < C::WORDS; ++k) {
            const uint32_t word = wrow[(C::WORDS * h + k) * C::BN + t];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // bits 4j..4j+3 (weight 8k+2j) into the low half, bits 16+4j.. (8k+2j+1) into the high half
              const uint32_t v = ((word >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
              const __half2 hv = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&v), zz), ss);
              pk[4 * k + j] = *reinterpret_cast<const uint32_t*>(&hv);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);       // this warp's words, scale and zero are read
#pragma unroll
        for (int q = 0; q < C::WORDS / 8; ++q)
          tmem_st32(tmem_base + lane_off + C::T_A + 64 * b + 4 * C::WORDS * h + 32 * q, pk + 32 * q);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full + b);
      }
      if (!ok) break;
      if (h != 0) continue;
      // ---- segment end (warps 4-7): read the accumulator, then Y or a partial ----
      if (!(ok = wait_all(seg_done, seg & 1))) break;
      tc_fence_after();
      const long long tu0 = static_cast<long long>(tile) * G;
      const int c_lo = w4_cta_of(tu0, U, p.ctas), c_hi = w4_cta_of(tu0 + G - 1, U, p.ctas);
      const int n0 = tile * C::BN;
      const bool whole = c_lo == c_hi;
      const bool col_ok = dbg_ok(n0 + t < p.N, kSiteW4Out, static_cast<unsigned>(n0 + t));
      const int slot = 2 * static_cast<int>(blockIdx.x) + (tile == tile0 ? 0 : 1);
      const bool part_ok = whole || dbg_ok(slot < 2 * p.ctas && tile < p.N / C::BN, kSiteW4Split,
                                           static_cast<unsigned long long>(slot));
      float* mine = whole ? nullptr : p.part + static_cast<size_t>(slot) * mpad * C::BN;
      for (int c0 = 0; c0 < mpad; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_base + lane_off + T_D + c0, v);
        tmem_ld_wait<16>(v);
        if (c0 + 16 >= mpad) {                       // the accumulator is free for the next segment
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(d_free);
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int m = c0 + k;
          if (whole) {
            if (m < p.M && col_ok) p.y[static_cast<size_t>(m) * p.N + n0 + t] = __float2half_rn(__uint_as_float(v[k]));
          } else if (part_ok) {
            __stcg(mine + static_cast<size_t>(m) * C::BN + t, __uint_as_float(v[k]));
          }
        }
      }
      if (whole || !part_ok) continue;
      // publish this segment's quarter; the last of the tile's segments sums them in CTA order
      __threadfence();
      __syncwarp();
      uint32_t prev = 0;
      uint32_t* ticket = p.tickets + 4 * tile + wq;
      if (lane == 0) prev = atomicAdd(ticket, 1u);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != static_cast<uint32_t>(c_hi - c_lo)) continue;
      __threadfence();
      for (int c0 = 0; c0 < p.M; c0 += 8) {          // 8 rows at a time, partials added in CTA order
        float acc[8];
        for (int c = c_lo; c <= c_hi; ++c) {
          const int ht = static_cast<int>(w4_unit0(c, U, p.ctas) / G);
          const float* src = p.part + (static_cast<size_t>(2 * c + (ht == tile ? 0 : 1)) * mpad + c0) * C::BN + t;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float val = __ldcg(src + k * C::BN);
            acc[k] = c == c_lo ? val : acc[k] + val;
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (c0 + k < p.M && col_ok) p.y[static_cast<size_t>(c0 + k) * p.N + n0 + t] = __float2half_rn(acc[k]);
      }
      __syncwarp();
      if (lane == 0) *ticket = 0u;                   // ready for the next launch
    }
    if (!ok && lane == 0) record_timeout();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace attn
