// attn_bwd_kernel.cuh - backward pass of the fused attention for sm_100a (BF16).
//
// The forward keeps only O and the per-row statistic LSE; the backward recomputes
// the attention weights tile by tile from Q, K and LSE instead of reading an
// N x N matrix ("Self-Attention, CUDA kernels and FlashAttention", section 3,
// recompute bullet). For dL/dO = dO it computes, per (batch, head):
//
//   P   = exp(scale Q K^T - LSE)  (row-wise, causal: 0 for key > query)
//   dV  = P^T dO                  dP = dO V^T
//   D_i = sum_c dO_ic O_ic        dS = P * (dP - D)
//   dQ  = scale dS K              dK = scale dS^T Q
//
// Three launches, all dense contractions on tcgen05 with fp32 accumulation in
// tensor memory and bf16 operands:
//   attn_bwd_rowdot   D_i = dO_i . O_i into the caller's workspace (HBM-bound
//                     stream, one 16-byte load per lane);
//   attn_bwd_dkdv     one CTA per (128-key block, head): K and V stay in shared
//                     memory, the Q / dO tiles of every visible query block stream
//                     through a two-stage TMA ring; per query block
//                       S^T = K Q^T and dP^T = V dO^T into TMEM,
//                       P^T (bf16) over S^T, dV += P^T dO,
//                       dS^T (bf16) over dP^T, dK += dS^T Q;
//                     the MMA thread issues the next block's S^T before waiting
//                     for this block's dS^T, so the exponentials of block i+1 run
//                     under the dK / dP^T MMAs of block i;
//   attn_bwd_dq       one CTA per (128-query block, head): Q and dO stay, K / V
//                     tiles stream; S = Q K^T (two TMEM buffers), dP = dO V^T,
//                     dS (bf16) over S, dQ += dS K.
// dQ is accumulated on chip by its own kernel instead of with atomics, so the
// result is deterministic and the only scratch memory is D (4 bytes per row).
//
// CTA: 8 warps. warp 0 TMA producer, warp 1 MMA issuer (owns TMEM), warps 2-3
// idle, warps 4-7 compute (one thread per TMEM lane = one row of the block).
// Every wait is bounded (Waiter); a wait that runs out records ATTN_ERR_TIMEOUT
// in the device status word, the CTA drains its copies and MMAs and exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "status.cuh"

namespace attn {

template <int D_>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr int CHUNK_BYTES = 128 * 128;              // 64 bf16 columns x 128 rows
  static constexpr int CHUNKS = D / 64;
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;    // one 128-row tile of Q, K, V or dO
  static constexpr int NST = 2;                              // ring stages
  // compute warpgroups: with two, the two warps of a TMEM lane quarter split the
  // 128 columns of each row (64 each), so each thread has half the exponentials
  // and the latencies of one warp hide under the other's work
#ifndef ATTN_BWD_SPLIT
#define ATTN_BWD_SPLIT 2
#endif
  static constexpr int SPLIT = ATTN_BWD_SPLIT;
  static constexpr int NCOL = 128 / SPLIT;                   // columns per compute thread
  static constexpr int THREADS = 128 + 128 * SPLIT;
  static constexpr int COMPUTE_WARP0 = 4;
  static constexpr uint32_t TMEM_COLS = 512;
  // dkdv shared memory: K, V, then per stage {Q, dO, LSE[128], D[128]}
  static constexpr int DKDV_K = 0;
  static constexpr int DKDV_V = TILE_BYTES;
  static constexpr int DKDV_STAGE = 2 * TILE_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES + 2 * 128 * 4;
  static constexpr int DKDV_BAR = DKDV_STAGE + NST * STAGE_BYTES;
  // dq shared memory: Q, dO, then per stage {K, V}
  static constexpr int DQ_Q = 0;
  static constexpr int DQ_DO = TILE_BYTES;
  static constexpr int DQ_STAGE = 2 * TILE_BYTES;
  static constexpr int DQ_BAR = DQ_STAGE + NST * 2 * TILE_BYTES;
  static constexpr int NUM_BARS = 16;
  static constexpr int DKDV_SMEM = DKDV_BAR + NUM_BARS * 8 + 16 + 1024;
  static constexpr int DQ_SMEM = DQ_BAR + NUM_BARS * 8 + 16 + 1024;
  // TMEM columns
  static constexpr uint32_t T_S = 0;          // dkdv: S^T (P^T over it); dq: S buffers 0 and 1
  static constexpr uint32_t T_DP = 128;       // dkdv: dP^T (dS^T over it)
  static constexpr uint32_t T_DV = 256;       // dkdv: dV accumulator
  static constexpr uint32_t T_DK = 256 + D;   // dkdv: dK accumulator
  static constexpr uint32_t T_DPQ = 256;      // dq: dP
  static constexpr uint32_t T_DQ = 384;       // dq: dQ accumulator
  static_assert(T_DK + D <= TMEM_COLS && T_DQ + D <= TMEM_COLS, "TMEM");
};

struct BwdParams {
  int N;
  int BH;
  int causal;
  float scale;            // multiplier of Q K^T (dQ and dK carry it once more)
  float scale_log2;       // scale * log2(e)
  const float* lse;       // [BH, N] natural log
  const float* dd;        // [BH, N] D_i (workspace)
  __nv_bfloat16* dq;      // [BH, N, D]
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  uint64_t timeout_cycles;
};

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- D_i = dO_i . O_i
// One row per D/8 lanes (16-byte loads of both tensors), fp32 products summed in
// a fixed order (lane-local, then a butterfly over the row's lanes).
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_rowdot(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout, float* __restrict__ dd,
                                                       long long rows) {
  constexpr int LANES = D / 8;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = t / LANES;
  const int part = static_cast<int>(t % LANES);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
    const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(ha[e]), fb = __bfloat1622float2(hb[e]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
  }
#pragma unroll
  for (int off = LANES / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && part == 0) dd[row] = acc;
}

// ---------------------------------------------------------------- MMA helpers
// D[tmem] (+)= A B^T over D/16 K-steps with both operands K-major in shared
// memory (128-byte swizzle, 64-element chunks of CHUNK_BYTES).
template <class C>
__device__ __forceinline__ void mma_ss_kmajor(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t leader) {
  constexpr uint32_t idesc = b200::instr_desc(1u, 128, 128, 0, 0);
  constexpr uint32_t hi = b200::smem_desc_hi(1024);
#pragma unroll
  for (int kk = 0; kk < C::D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4;
    b200::mma_f16_ss(d_tmem, b200::smem_desc(a_lo + off, hi), b200::smem_desc(b_lo + off, hi), idesc, kk > 0,
                     leader);
  }
}
// D[tmem, N = D] (+)= A[tmem, 128 x 128 bf16] B[128 x D], B MN-major in shared
// memory (rows = the K dimension).
template <class C>
__device__ __forceinline__ void mma_ts_mnmajor(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, bool acc,
                                               uint32_t leader) {
  constexpr uint32_t idesc = b200::instr_desc(1u, 128, C::D, 0, 1);
  constexpr uint32_t hi = b200::smem_desc_hi(1024);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    b200::mma_f16_ts(d_tmem, a_tmem + kk * 8, b200::smem_desc(b_lo + ((kk * 16 * 128) >> 4), hi), idesc,
                     (acc || kk > 0) ? 1u : 0u, leader);
}

__device__ __forceinline__ void wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const uint64_t t0 = b200::sm_clock();
  while (!b200::mbar_try_wait(bar, parity) && b200::sm_clock() - t0 < limit) {
  }
}

// Stores one row of an fp32 TMEM accumulator (D columns at `taddr`) as bf16,
// multiplied by `mul`, to `dst` (skipped when !in_range; the TMEM loads are
// warp-collective and always run).
template <int D>
__device__ __forceinline__ void store_row_bf16(uint32_t taddr, float mul, __nv_bfloat16* dst, bool in_range) {
#pragma unroll
  for (int cb = 0; cb < D; cb += 32) {
    uint32_t v[32];
    b200::tmem_ld32(taddr + cb, v);
    b200::tmem_ld_wait<32>(v);
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      packed[i] = b200::pack_bf16x2(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
    if (in_range) {
      uint4* o = reinterpret_cast<uint4*>(dst + cb);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    }
  }
}

// ---------------------------------------------------------------- dK, dV
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd_dkdv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using namespace b200;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DKDV_BAR);
  uint64_t* kv_full = bars;                 // 1
  uint64_t* q_full = bars + 1;              // NST (TMA bytes + 32 producer lanes)
  uint64_t* q_empty = q_full + C::NST;      // NST
  uint64_t* s_full = q_empty + C::NST;      // 1
  uint64_t* dp_full = s_full + 1;           // 1
  uint64_t* p_ready = dp_full + 1;          // 1 (4 compute warps)
  uint64_t* ds_ready = p_ready + 1;         // 1 (4 compute warps)
  uint64_t* done = ds_ready + 1;            // 1
  uint64_t* drain_bar = done + 1;           // 1
  uint64_t* s_read = drain_bar + 1;         // 1 (SPLIT 2: the first column half has read S^T)
  uint64_t* dp_read = s_read + 1;           // 1 (SPLIT 2: the first column half has read dP^T)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int QB = (p.N + 127) / 128;
  // CTA -> (key block, head). Head-major order keeps the CTAs that run together
  // on a few heads, whose Q / dO tiles they all stream, so those come from L2;
  // inside a head the heaviest causal key blocks go first.
#ifndef ATTN_BWD_HEAD_MAJOR
#define ATTN_BWD_HEAD_MAJOR 1
#endif
  const int jb = ATTN_BWD_HEAD_MAJOR ? static_cast<int>(blockIdx.x) % QB : static_cast<int>(blockIdx.x) / p.BH;
  const int bh = ATTN_BWD_HEAD_MAJOR ? static_cast<int>(blockIdx.x) / QB : static_cast<int>(blockIdx.x) % p.BH;
  const int i0 = p.causal ? jb : 0;                 // first visible query block
  const int n = QB - i0;                            // query blocks visited

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(q_full + s, 33);
      mbar_init(q_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 4 * C::SPLIT);
    mbar_init(ds_ready, 4 * C::SPLIT);
    mbar_init(done, 1);
    mbar_init(drain_bar, 1);
    mbar_init(s_read, 4);
    mbar_init(dp_read, 4);
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
  auto stage_q = [&](int s) { return smem + C::DKDV_STAGE + s * C::STAGE_BYTES; };
  auto stage_do = [&](int s) { return smem + C::DKDV_STAGE + s * C::STAGE_BYTES + C::TILE_BYTES; };
  auto stage_lse = [&](int s) {
    return reinterpret_cast<float*>(smem + C::DKDV_STAGE + s * C::STAGE_BYTES + 2 * C::TILE_BYTES);
  };
  auto stage_dd = [&](int s) { return stage_lse(s) + 128; };

  if (warp == 0) {
    // ======================= producer =======================
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint64_t pol = l2_policy_evict_first();
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c) {
        tma_load_3d(smem + C::DKDV_K + c * C::CHUNK_BYTES, &tm_k, kv_full, c * 64, jb * 128, bh, pol);
        tma_load_3d(smem + C::DKDV_V + c * C::CHUNK_BYTES, &tm_v, kv_full, c * 64, jb * 128, bh, pol);
      }
    }
    __syncwarp();
    const uint64_t pol_q = l2_policy_evict_last();   // Q / dO tiles are shared by the key blocks of a head
    int it = 0;
    for (; it < n; ++it) {
      const int s = it % C::NST, i = i0 + it;
      if (it >= C::NST && !(ok = wait_all(q_empty + s, ((it / C::NST) - 1) & 1))) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full + s, 2 * C::TILE_BYTES);
        for (int c = 0; c < C::CHUNKS; ++c) {
          tma_load_3d(stage_q(s) + c * C::CHUNK_BYTES, &tm_q, q_full + s, c * 64, i * 128, bh, pol_q);
          tma_load_3d(stage_do(s) + c * C::CHUNK_BYTES, &tm_do, q_full + s, c * 64, i * 128, bh, pol_q);
        }
      }
      // the block's row statistics LSE and D, copied asynchronously (zeros past N;
      // the compute threads mask those queries): each lane's copies arrive on the
      // stage's barrier when they land, so the producer never waits for them
      for (int t = lane; t < 128; t += 32) {
        const int q = i * 128 + t;
        const size_t gq = static_cast<size_t>(bh) * p.N + q;
        const bool in = q < p.N && dbg_ok(gq < static_cast<size_t>(p.BH) * p.N, kSiteBwdStats, gq);
        const size_t g = in ? gq : static_cast<size_t>(0);
        cp_async_4(stage_lse(s) + t, p.lse + g, in);
        cp_async_4(stage_dd(s) + t, p.dd + g, in);
      }
      cp_async_arrive_noinc(q_full + s);
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) record_timeout();
      for (int j = (it > C::NST ? it - C::NST : 0); j < it; ++j)
        wait_bounded(q_full + (j % C::NST), (j / C::NST) & 1, p.timeout_cycles);
    }
    wait_bounded(kv_full, 0, p.timeout_cycles);
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    const uint32_t leader = elect_one() ? 1u : 0u;
    const uint32_t k_lo = smem_desc_lo(smem_addr(smem + C::DKDV_K), 16);
    const uint32_t v_lo = smem_desc_lo(smem_addr(smem + C::DKDV_V), 16);
    auto q_lo = [&](int s) { return smem_desc_lo(smem_addr(stage_q(s)), 16); };
    auto do_lo = [&](int s) { return smem_desc_lo(smem_addr(stage_do(s)), 16); };
    auto q_mn = [&](int s) { return smem_desc_lo(smem_addr(stage_q(s)), C::CHUNK_BYTES); };
    auto do_mn = [&](int s) { return smem_desc_lo(smem_addr(stage_do(s)), C::CHUNK_BYTES); };
    do {
      if (!(ok = wait_all(kv_full, 0))) break;
      if (!(ok = wait_all(q_full + 0, 0))) break;
      tc_fence_after();
      mma_ss_kmajor<C>(tmem_base + C::T_S, k_lo, q_lo(0), leader);      // S^T(0) = K Q^T
      mma_commit(s_full, leader);
      mma_ss_kmajor<C>(tmem_base + C::T_DP, v_lo, do_lo(0), leader);    // dP^T(0) = V dO^T
      mma_commit(dp_full, leader);
      for (int it = 0; it < n; ++it) {
        const int s = it % C::NST;
        if (!(ok = wait_all(p_ready, it & 1))) break;
        tc_fence_after();
        mma_ts_mnmajor<C>(tmem_base + C::T_DV, tmem_base + C::T_S, do_mn(s), it > 0, leader);   // dV += P^T dO
        if (it + 1 < n) {
          const int s1 = (it + 1) % C::NST;
          if (!(ok = wait_all(q_full + s1, ((it + 1) / C::NST) & 1))) break;
          tc_fence_after();
          mma_ss_kmajor<C>(tmem_base + C::T_S, k_lo, q_lo(s1), leader);   // S^T(it+1)
          mma_commit(s_full, leader);
        }
        if (!(ok = wait_all(ds_ready, it & 1))) break;
        tc_fence_after();
        mma_ts_mnmajor<C>(tmem_base + C::T_DK, tmem_base + C::T_DP, q_mn(s), it > 0, leader);   // dK += dS^T Q
        mma_commit(q_empty + s, leader);
        if (it + 1 < n) {
          mma_ss_kmajor<C>(tmem_base + C::T_DP, v_lo, do_lo((it + 1) % C::NST), leader);   // dP^T(it+1)
          mma_commit(dp_full, leader);
        }
      }
      if (ok) mma_commit(done, leader);
    } while (false);
    if (!ok && lane == 0) record_timeout();
    mma_commit(drain_bar, leader);
    wait_bounded(drain_bar, 0, p.timeout_cycles);
    __syncwarp();
  } else if (warp >= C::COMPUTE_WARP0) {
    // ======================= compute: one thread per key =======================
    // Thread (key r, column half h) owns the queries [NCOL h, NCOL h + NCOL) of its
    // row. Packed bf16 P^T / dS^T of half h goes to the columns [NCOL h / 2, ...)
    // of S^T / dP^T, which for h = 1 overlap columns half 0 reads: half 1 stores
    // only after half 0 has read (s_read, dp_read).
    constexpr int NCOL = C::NCOL;
    const int cw = warp - C::COMPUTE_WARP0;
    const int wq = warp & 3;                            // TMEM lane quarter of this warp
    const int h = cw >> 2;                              // column half
    const int col0 = NCOL * h;
    const int r = wq * 32 + lane;                       // key inside the block
    const int key = jb * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + C::T_S;
    const uint32_t t_dp = tmem_base + lane_off + C::T_DP;
    const float c = p.scale_log2;
    for (int it = 0; it < n; ++it) {
      const int s = it % C::NST, i = i0 + it;
      if (!(ok = wait_all(q_full + s, (it / C::NST) & 1))) break;
      if (!(ok = wait_all(s_full, it & 1))) break;
      tc_fence_after();
      // the block's statistics are the same for every thread: 16-byte broadcast loads
      const float4* lse2 = reinterpret_cast<const float4*>(stage_lse(s) + col0);
      const float4* dd = reinterpret_cast<const float4*>(stage_dd(s) + col0);
      float pr[NCOL];
      {
        uint32_t sr[NCOL];
#pragma unroll
        for (int q = 0; q < NCOL / 32; ++q) tmem_ld32(t_s + col0 + 32 * q, sr + 32 * q);
        tmem_ld_wait<NCOL>(sr);
        if (C::SPLIT > 1 && h == 0) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_read);
        }
        // visible: key < N, query < N, and for the diagonal block of a causal
        // launch, key <= query
        const int first_visible = (key >= p.N) ? 128 : ((p.causal && i == jb) ? r : 0);
        const int end_visible = p.N - i * 128;            // queries past N read LSE = D = 0
#pragma unroll
        for (int j4 = 0; j4 < NCOL / 4; ++j4) {
          const float4 l4 = lse2[j4];
          const float lv[4] = {l4.x * kLog2e, l4.y * kLog2e, l4.z * kLog2e, l4.w * kLog2e};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * j4 + e;
            const float x = ex2_approx(fmaf(__uint_as_float(sr[j]), c, -lv[e]));
            pr[j] = (col0 + j >= first_visible && col0 + j < end_visible) ? x : 0.f;
          }
        }
        uint32_t pk[NCOL / 2];
#pragma unroll
        for (int j = 0; j < NCOL / 2; ++j) pk[j] = pack_bf16x2(pr[2 * j], pr[2 * j + 1]);
        if (C::SPLIT > 1 && h > 0) {
          if (!(ok = wait_all(s_read, it & 1))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int q = 0; q < NCOL / 64; ++q) tmem_st32(t_s + col0 / 2 + 32 * q, pk + 32 * q);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready);
      if (!(ok = wait_all(dp_full, it & 1))) break;
      tc_fence_after();
      bool first_store = true;
#pragma unroll
      for (int ch = 0; ch < NCOL / 32; ++ch) {
        uint32_t dp[32];
        tmem_ld32(t_dp + col0 + 32 * ch, dp);
        tmem_ld_wait<32>(dp);
        if (C::SPLIT > 1 && h == 0 && ch == NCOL / 32 - 1) {   // half 0 has read all its dP^T
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dp_read);
        }
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const int q0 = 32 * ch + 2 * j;
          const float4 d4 = dd[q0 >> 2];
          pk[j] = pack_bf16x2(pr[q0] * (__uint_as_float(dp[2 * j]) - d4.x),
                              pr[q0 + 1] * (__uint_as_float(dp[2 * j + 1]) - d4.y));
          pk[j + 1] = pack_bf16x2(pr[q0 + 2] * (__uint_as_float(dp[2 * j + 2]) - d4.z),
                                  pr[q0 + 3] * (__uint_as_float(dp[2 * j + 3]) - d4.w));
        }
        if (C::SPLIT > 1 && h > 0 && first_store) {
          if (!(ok = wait_all(dp_read, it & 1))) break;
          tc_fence_after();
        }
        first_store = false;
        tmem_st16(t_dp + col0 / 2 + 16 * ch, pk);   // dS^T over dP^T columns already read
      }
      if (!ok) break;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_ready);
    }
    if (ok) ok = wait_all(done, 0);
    if (ok) {
      tc_fence_after();
      const size_t krow = static_cast<size_t>(bh) * p.N + key;
      const bool in_range = key < p.N && dbg_ok(krow < static_cast<size_t>(p.BH) * p.N, kSiteBwdDkDv, krow);
      const size_t row = in_range ? krow : static_cast<size_t>(0);
      if (C::SPLIT == 1 || h == 0)
        store_row_bf16<C::D>(tmem_base + lane_off + C::T_DV, 1.f, p.dv + row * C::D, in_range);
      if (C::SPLIT == 1 || h == 1)
        store_row_bf16<C::D>(tmem_base + lane_off + C::T_DK, p.scale, p.dk + row * C::D, in_range);
    } else if (lane == 0) {
      record_timeout();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------- dQ
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd_dq(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const BwdParams p) {
  using namespace b200;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DQ_BAR);
  uint64_t* q_full = bars;                  // 1
  uint64_t* kv_full = bars + 1;             // NST
  uint64_t* kv_empty = kv_full + C::NST;    // NST
  uint64_t* s_full = kv_empty + C::NST;     // 2 (S buffers)
  uint64_t* dp_full = s_full + 2;           // 1
  uint64_t* ds_ready = dp_full + 1;         // 1 (all compute warps)
  uint64_t* done = ds_ready + 1;            // 1
  uint64_t* drain_bar = done + 1;           // 1
  uint64_t* s_read = drain_bar + 1;         // 1 (SPLIT 2: the first column half has read S)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int QB = (p.N + 127) / 128;
  // CTA -> (query block, head): head-major (the K / V tiles of the CTAs running
  // together come from L2), heaviest causal query blocks first inside a head
  const int ib = QB - 1 - (ATTN_BWD_HEAD_MAJOR ? static_cast<int>(blockIdx.x) % QB
                                               : static_cast<int>(blockIdx.x) / p.BH);
  const int bh = ATTN_BWD_HEAD_MAJOR ? static_cast<int>(blockIdx.x) / QB : static_cast<int>(blockIdx.x) % p.BH;
  const int n = p.causal ? ib + 1 : QB;                          // key blocks visited

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full + 0, 1);
    mbar_init(s_full + 1, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_ready, 4 * C::SPLIT);
    mbar_init(done, 1);
    mbar_init(drain_bar, 1);
    mbar_init(s_read, 4);
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
  auto stage_k = [&](int s) { return smem + C::DQ_STAGE + s * 2 * C::TILE_BYTES; };
  auto stage_v = [&](int s) { return smem + C::DQ_STAGE + s * 2 * C::TILE_BYTES + C::TILE_BYTES; };

  if (warp == 0) {
    // ======================= producer =======================
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint64_t pol = l2_policy_evict_first();
      mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c) {
        tma_load_3d(smem + C::DQ_Q + c * C::CHUNK_BYTES, &tm_q, q_full, c * 64, ib * 128, bh, pol);
        tma_load_3d(smem + C::DQ_DO + c * C::CHUNK_BYTES, &tm_do, q_full, c * 64, ib * 128, bh, pol);
      }
    }
    __syncwarp();
    const uint64_t pol_kv = l2_policy_evict_last();
    int j = 0;
    for (; j < n; ++j) {
      const int s = j % C::NST;
      if (j >= C::NST && !(ok = wait_all(kv_empty + s, ((j / C::NST) - 1) & 1))) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(kv_full + s, 2 * C::TILE_BYTES);
        for (int c = 0; c < C::CHUNKS; ++c) {
          tma_load_3d(stage_k(s) + c * C::CHUNK_BYTES, &tm_k, kv_full + s, c * 64, j * 128, bh, pol_kv);
          tma_load_3d(stage_v(s) + c * C::CHUNK_BYTES, &tm_v, kv_full + s, c * 64, j * 128, bh, pol_kv);
        }
      }
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) record_timeout();
      for (int t = (j > C::NST ? j - C::NST : 0); t < j; ++t)
        wait_bounded(kv_full + (t % C::NST), (t / C::NST) & 1, p.timeout_cycles);
    }
    wait_bounded(q_full, 0, p.timeout_cycles);
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    const uint32_t leader = elect_one() ? 1u : 0u;
    const uint32_t q_lo = smem_desc_lo(smem_addr(smem + C::DQ_Q), 16);
    const uint32_t do_lo = smem_desc_lo(smem_addr(smem + C::DQ_DO), 16);
    auto k_lo = [&](int s) { return smem_desc_lo(smem_addr(stage_k(s)), 16); };
    auto v_lo = [&](int s) { return smem_desc_lo(smem_addr(stage_v(s)), 16); };
    auto k_mn = [&](int s) { return smem_desc_lo(smem_addr(stage_k(s)), C::CHUNK_BYTES); };
    do {
      if (!(ok = wait_all(q_full, 0))) break;
      if (!(ok = wait_all(kv_full + 0, 0))) break;
      tc_fence_after();
      mma_ss_kmajor<C>(tmem_base + C::T_S, q_lo, k_lo(0), leader);        // S(0) = Q K^T
      mma_commit(s_full + 0, leader);
      mma_ss_kmajor<C>(tmem_base + C::T_DPQ, do_lo, v_lo(0), leader);     // dP(0) = dO V^T
      mma_commit(dp_full, leader);
      if (n > 1) {
        if (!(ok = wait_all(kv_full + 1 % C::NST, (1 / C::NST) & 1))) break;
        tc_fence_after();
        mma_ss_kmajor<C>(tmem_base + C::T_S + 128, q_lo, k_lo(1 % C::NST), leader);
        mma_commit(s_full + 1, leader);
      }
      for (int j = 0; j < n; ++j) {
        const int s = j % C::NST;
        if (!(ok = wait_all(ds_ready, j & 1))) break;
        tc_fence_after();
        mma_ts_mnmajor<C>(tmem_base + C::T_DQ, tmem_base + C::T_S + 128 * (j & 1), k_mn(s), j > 0, leader);
        mma_commit(kv_empty + s, leader);
        if (j + 1 < n) {
          mma_ss_kmajor<C>(tmem_base + C::T_DPQ, do_lo, v_lo((j + 1) % C::NST), leader);   // dP(j+1)
          mma_commit(dp_full, leader);
        }
        if (j + 2 < n) {
          const int s2 = (j + 2) % C::NST;
          if (!(ok = wait_all(kv_full + s2, ((j + 2) / C::NST) & 1))) break;
          tc_fence_after();
          mma_ss_kmajor<C>(tmem_base + C::T_S + 128 * (j & 1), q_lo, k_lo(s2), leader);   // S(j+2)
          mma_commit(s_full + (j & 1), leader);
        }
      }
      if (ok) mma_commit(done, leader);
    } while (false);
    if (!ok && lane == 0) record_timeout();
    mma_commit(drain_bar, leader);
    wait_bounded(drain_bar, 0, p.timeout_cycles);
    __syncwarp();
  } else if (warp >= C::COMPUTE_WARP0) {
    // ======================= compute: one thread per query =======================
    // Thread (query r, column half h) owns the keys [NCOL h, NCOL h + NCOL) of its
    // row; its packed bf16 dS goes to S columns [NCOL h / 2, ...), which for h = 1
    // overlap columns half 0 reads: half 1 stores only after half 0 has read (s_read).
    constexpr int NCOL = C::NCOL;
    const int cw = warp - C::COMPUTE_WARP0;
    const int wq = warp & 3;
    const int h = cw >> 2;
    const int col0 = NCOL * h;
    const int r = wq * 32 + lane;
    const int qrow = ib * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float c = p.scale_log2;
    const size_t gq = static_cast<size_t>(bh) * p.N + qrow;
    const bool q_in = qrow < p.N && dbg_ok(gq < static_cast<size_t>(p.BH) * p.N, kSiteBwdDq, gq);
    const size_t g = q_in ? gq : static_cast<size_t>(0);
    const float l2 = q_in ? p.lse[g] * kLog2e : __int_as_float(0x7f800000);
    const float dd = q_in ? p.dd[g] : 0.f;
    for (int j = 0; j < n; ++j) {
      const uint32_t t_s = tmem_base + lane_off + C::T_S + 128 * (j & 1);
      if (!(ok = wait_all(s_full + (j & 1), (j >> 1) & 1))) break;
      tc_fence_after();
      float pr[NCOL];
      {
        uint32_t sr[NCOL];
#pragma unroll
        for (int q = 0; q < NCOL / 32; ++q) tmem_ld32(t_s + col0 + 32 * q, sr + 32 * q);
        tmem_ld_wait<NCOL>(sr);
        if (C::SPLIT > 1 && h == 0) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_read);
        }
        // visible keys: j*128 + col < N and, on a causal diagonal block, col <= r
        int last = p.N - 1 - j * 128;
        if (p.causal && j == ib) last = min(last, r);
#pragma unroll
        for (int k = 0; k < NCOL; ++k) {
          const float x = ex2_approx(fmaf(__uint_as_float(sr[k]), c, -l2));
          pr[k] = (col0 + k <= last) ? x : 0.f;
        }
      }
      if (!(ok = wait_all(dp_full, j & 1))) break;
      tc_fence_after();
      const uint32_t t_dp = tmem_base + lane_off + C::T_DPQ + col0;
#pragma unroll
      for (int ch = 0; ch < NCOL / 32; ++ch) {
        uint32_t dp[32];
        tmem_ld32(t_dp + 32 * ch, dp);
        tmem_ld_wait<32>(dp);
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int k0 = 32 * ch + 2 * k;
          pk[k] = pack_bf16x2(pr[k0] * (__uint_as_float(dp[2 * k]) - dd), pr[k0 + 1] * (__uint_as_float(dp[2 * k + 1]) - dd));
        }
        if (C::SPLIT > 1 && h > 0 && ch == 0) {
          if (!(ok = wait_all(s_read, j & 1))) break;
          tc_fence_after();
        }
        tmem_st16(t_s + col0 / 2 + 16 * ch, pk);   // dS over the S columns already read
      }
      if (!ok) break;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_ready);
    }
    if (ok) ok = wait_all(done, 0);
    if (ok) {
      tc_fence_after();
      const bool in_range = q_in;
      // the two column halves of a row store the two halves of its dQ
      constexpr int DC = C::D / C::SPLIT;
      store_row_bf16<DC>(tmem_base + lane_off + C::T_DQ + DC * h, p.scale, p.dq + g * C::D + DC * h, in_range);
    } else if (lane == 0) {
      record_timeout();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace attn
