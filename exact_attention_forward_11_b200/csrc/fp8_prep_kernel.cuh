// fp8_prep_kernel.cuh - incoherent rotation and block quantisation to E4M3.
//
// "FlashAttention scaling, multi-GPU training and weight quantization", section 1,
// FlashAttention-3 FP8 bullet: Q and K are multiplied by a random orthogonal
// matrix before quantisation so that outliers are spread over all channels, and
// each small tile gets its own scale. Here a tile is 128 tokens x 128 channels of
// one (batch, head), which is also the attention kernel's Q/K/V tile, so one scale
// applies to a whole MMA operand tile.
//
// Definition:
//   y     = x R, the plain matrix product (bf16 operands, fp32 accumulation on
//           the tensor cores), or y = x without rotation;
//   scale = max |y| over the tile / 448 (IEEE fp32 division), 1 for all zeros;
//   code  = E4M3 (round to nearest even, saturating) of fp32(y * r) with
//           r = 1 / scale (one IEEE fp32 division per tile).
//
// The rotation is a dense contraction (128 multiply-adds per element), so it runs
// as tcgen05 MMAs: per tile D[128 x 128] = X[128 x 128] R[128 x 128], X K-major
// and R MN-major in shared memory, D in tensor memory. The kernel as a whole is
// bound by HBM (2 bytes read and 1 written per element), so its structure is a
// stream: persistent CTAs (one per SM) walk the tiles; a producer warp keeps a
// ring of X tiles in flight with TMA; an MMA warp turns each X tile into y in one
// of two TMEM accumulators; an epilogue warpgroup (one thread per row) reads y,
// reduces the tile amax through shared memory, quantises its row into a
// shared-memory staging tile with the same 128-byte swizzle the TMA store uses,
// and one of its threads stores the tile with TMA (rows past N are not written).
// Without rotation the epilogue reads X straight from the shared-memory slot.
//
// CTA: 8 warps. warp 0 TMA producer, warp 1 MMA issuer (owns TMEM), warps 2-3
// idle, warps 4-7 epilogue (warp w reads TMEM lanes 32 (w % 4) .. + 31).
// Every wait is bounded (Waiter): a wait that runs out records ATTN_ERR_TIMEOUT
// in the device status word, in-flight copies and MMAs are drained, TMEM is
// released and the CTA exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "status.cuh"

namespace attn {

constexpr int kPrepTile = 128;

struct PrepCfg {
  static constexpr int THREADS = 256;
  static constexpr int NSLOT = 4;                  // X tiles in flight per CTA
  static constexpr int CHUNK_BYTES = 128 * 128;    // 64 bf16 columns x 128 rows
  static constexpr int TILE_BYTES = 2 * CHUNK_BYTES;
  static constexpr int OUT_BYTES = 128 * 128;      // one tile of E4M3 codes
  static constexpr int NOUT = 2;                   // staging tiles for the TMA store
  static constexpr int EPI_WARP0 = 4;
  static constexpr uint32_t TMEM_COLS = 256;       // two 128-column fp32 accumulators
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int SMEM_R = 0;
  static constexpr int SMEM_X = SMEM_R + TILE_BYTES;
  static constexpr int SMEM_OUT = SMEM_X + NSLOT * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_OUT + NOUT * OUT_BYTES;
  // r_full, x_full[NSLOT], x_empty[NSLOT], acc_full[2], acc_empty[2],
  // red_full[2], out_full[NOUT], out_free[NOUT], drain
  static constexpr int NUM_BARS = 1 + 2 * NSLOT + 2 + 2 + 2 + 2 * NOUT + 1;
  static constexpr int SMEM_RED = SMEM_BAR + NUM_BARS * 8;        // 2 x 4 warp maxima
  static constexpr int SMEM_MISC = SMEM_RED + 2 * 4 * 4;          // tmem slot, abort word
  static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;
};

template <bool ROTATE>
__global__ void __launch_bounds__(PrepCfg::THREADS, 1)
    fp8_prep_sm100(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                   const __grid_constant__ CUtensorMap tm_out, float* __restrict__ scales, int T, int num_tiles,
                   uint64_t timeout_cycles) {
  using namespace b200;
  using C = PrepCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint64_t* r_full = bars;
  uint64_t* x_full = r_full + 1;
  uint64_t* x_empty = x_full + C::NSLOT;
  uint64_t* acc_full = x_empty + C::NSLOT;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* red_full = acc_empty + 2;
  uint64_t* out_full = red_full + 2;
  uint64_t* out_free = out_full + C::NOUT;
  uint64_t* drain_bar = out_free + C::NOUT;
  float* red = reinterpret_cast<float*>(smem + C::SMEM_RED);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(r_full, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(x_full + i, 1);
      mbar_init(x_empty + i, ROTATE ? 1 : 4);   // MMA commit, or one arrival per epilogue warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);
      mbar_init(red_full + i, 4);
    }
    for (int i = 0; i < C::NOUT; ++i) {
      mbar_init(out_full + i, 128);
      mbar_init(out_free + i, 1);
    }
    mbar_init(drain_bar, 1);
    *abort_word = 0u;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (ROTATE && warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ROTATE ? *tmem_slot : 0u;
  const Waiter waiter{abort_word, timeout_cycles};
  auto wait_all = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, waiter.wait(bar, parity)); };
  bool ok = true;

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (elect_one()) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_out);
      if (ROTATE) {
        tma_prefetch_desc(&tm_r);
        mbar_arrive_expect_tx(r_full, C::TILE_BYTES);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + C::SMEM_R + c * C::CHUNK_BYTES, &tm_r, r_full, c * 64, 0, 0, l2_policy_evict_last());
      }
    }
    __syncwarp();
    const uint64_t pol = l2_policy_evict_first();
    uint32_t i = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
      const uint32_t slot = i % C::NSLOT;
      if (i >= C::NSLOT && !(ok = wait_all(x_empty + slot, ((i / C::NSLOT) - 1) & 1))) break;
      const int bh = tile / T, row0 = (tile % T) * kPrepTile;
      if (elect_one()) {
        mbar_arrive_expect_tx(x_full + slot, C::TILE_BYTES);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + C::SMEM_X + slot * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_x, x_full + slot, c * 64,
                      row0, bh, pol);
      }
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) record_timeout();
      // let the copies still in flight land before shared memory is released
      const uint64_t t0 = sm_clock();
      for (uint32_t j = (i > C::NSLOT ? i - C::NSLOT : 0); j < i; ++j)
        while (!mbar_try_wait(x_full + (j % C::NSLOT), (j / C::NSLOT) & 1) && sm_clock() - t0 < timeout_cycles) {
        }
      if (ROTATE)
        while (!mbar_try_wait(r_full, 0) && sm_clock() - t0 < timeout_cycles) {
        }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer (rotation only) =======================
    if (ROTATE) {
      const uint32_t leader = elect_one() ? 1u : 0u;
      constexpr uint32_t idesc = instr_desc(1u, 128, 128, 0, 1);   // bf16 x bf16 -> f32, B MN-major
      constexpr uint32_t hi = smem_desc_hi(1024);
      const uint32_t x_lo = smem_desc_lo(smem_addr(smem + C::SMEM_X), 16);
      const uint32_t r_lo = smem_desc_lo(smem_addr(smem + C::SMEM_R), C::CHUNK_BYTES);
      ok = wait_all(r_full, 0);
      uint32_t i = 0;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++i) {
        const uint32_t slot = i % C::NSLOT, a = i & 1;
        if (!(ok = wait_all(x_full + slot, (i / C::NSLOT) & 1))) break;
        if (i >= 2 && !(ok = wait_all(acc_empty + a, ((i >> 1) - 1) & 1))) break;
        tc_fence_after();
        const uint32_t xa = x_lo + ((slot * C::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A: K-major X, 16 k per step (4 steps per 128-byte chunk); B: R rows k, MN-major
          const uint32_t aoff = ((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4;
          const uint32_t boff = (kk * 16 * 128) >> 4;
          mma_f16_ss(tmem_base + a * 128, smem_desc(xa + aoff, hi), smem_desc(r_lo + boff, hi), idesc, kk > 0,
                     leader);
        }
        mma_commit(x_empty + slot, leader);
        mma_commit(acc_full + a, leader);
      }
      if (!ok && lane == 0) record_timeout();
      // every MMA this warp issued completes before TMEM is released
      mma_commit(drain_bar, leader);
      const uint64_t t0 = sm_clock();
      while (!mbar_try_wait(drain_bar, 0) && sm_clock() - t0 < timeout_cycles) {
      }
      __syncwarp();
    }
  } else if (warp >= C::EPI_WARP0) {
    // ======================= epilogue warpgroup =======================
    const int wq = warp - C::EPI_WARP0;          // lane quarter of TMEM
    const int r = wq * 32 + lane;                // row of the tile
    const bool store_leader = (wq == 0 && lane == 0);
    uint32_t i = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
      const uint32_t slot = i % C::NSLOT, a = i & 1, ob = i % C::NOUT;
      float y[128];
      if (ROTATE) {
        if (!(ok = wait_all(acc_full + a, (i >> 1) & 1))) break;
        tc_fence_after();
        uint32_t v[128];
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + a * 128;
        tmem_ld32(taddr + 0, v + 0);
        tmem_ld32(taddr + 32, v + 32);
        tmem_ld32(taddr + 64, v + 64);
        tmem_ld32(taddr + 96, v + 96);
        tmem_ld_wait<128>(v);
#pragma unroll
        for (int j = 0; j < 128; ++j) y[j] = __uint_as_float(v[j]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + a);   // this warp's rows are out of TMEM
      } else {
        if (!(ok = wait_all(x_full + slot, (i / C::NSLOT) & 1))) break;
        const uint8_t* xs = smem + C::SMEM_X + slot * C::TILE_BYTES + r * 128;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(xs + c * C::CHUNK_BYTES + ((u ^ (r & 7)) << 4));
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h[e]);
              y[c * 64 + u * 8 + 2 * e] = f.x;
              y[c * 64 + u * 8 + 2 * e + 1] = f.y;
            }
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(x_empty + slot);   // this warp's rows are read
      }
      // tile amax: row, warp, then the four warps through shared memory
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 128; ++j) m = fmaxf(m, fabsf(y[j]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float* red_i = red + (i & 1) * 4;
      if (lane == 0) {
        red_i[wq] = m;
        mbar_arrive(red_full + (i & 1));
      }
      // the staging tile of this store buffer must have been read by its last store
      if (i >= C::NOUT && !(ok = wait_all(out_free + ob, ((i / C::NOUT) - 1) & 1))) break;
      if (!(ok = wait_all(red_full + (i & 1), (i >> 1) & 1))) break;
      const float amax = fmaxf(fmaxf(red_i[0], red_i[1]), fmaxf(red_i[2], red_i[3]));
      const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      const float inv = __fdiv_rn(1.0f, sc);
      uint8_t* orow = smem + C::SMEM_OUT + ob * C::OUT_BYTES + r * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = u * 16 + 4 * e;
          w[e] = pack_e4m3x4(__fmul_rn(y[j], inv), __fmul_rn(y[j + 1], inv), __fmul_rn(y[j + 2], inv),
                             __fmul_rn(y[j + 3], inv));
        }
        *reinterpret_cast<uint4*>(orow + ((u ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_shared();   // the TMA store (async proxy) reads what this thread wrote
      mbar_arrive(out_full + ob);
      if (store_leader) {
        if (!waiter.wait(out_full + ob, (i / C::NOUT) & 1)) {
          ok = false;
        } else {
          const int bh = tile / T, t = tile % T;
          tma_store_3d(&tm_out, smem + C::SMEM_OUT + ob * C::OUT_BYTES, 0, t * kPrepTile, bh);
          bulk_commit_group();
          if (dbg_ok(tile < num_tiles, kSiteFp8Scale, static_cast<unsigned>(tile)))
            scales[static_cast<size_t>(bh) * T + t] = sc;
          // the previous store has read its staging tile: free it
          if (i >= 1) {
            bulk_wait_group_read<1>();
            mbar_arrive(out_free + ((i - 1) % C::NOUT));
          }
        }
      }
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
    }
    if (store_leader) bulk_wait_group_all();   // stores complete before the CTA exits
    if (!ok && lane == 0) record_timeout();
  }

  // ---- teardown: every TMEM access and MMA of this CTA is complete here
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ROTATE && warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace attn
