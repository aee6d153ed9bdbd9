// attn_fwd_kernel.cuh - fused attention forward for sm_100a (BF16 and FP8 E4M3).
//
// What it computes: O = softmax(scale * Q K^T) V and LSE = ln sum_j exp(scale q.k_j)
// per (batch, head) ("Self-Attention, CUDA kernels and FlashAttention", section 1,
// eq. Scores and eq. Attention), without ever writing the N x N scores: Q, K and V
// are cut into 128-row tiles that live on chip, and the softmax is computed online
// with a running row maximum and normaliser (same page, section 3, tiling and
// online-softmax bullets). The division by the normaliser happens once at the end
// (FlashAttention-2 bullet on non-matmul work, "FlashAttention scaling, multi-GPU
// training and weight quantization", section 1); the outer loop runs over Q tiles
// spread across CTAs and the inner loop over K/V tiles (FlashAttention-2 bullet on
// sequence parallelism and loop order). Copies are asynchronous (TMA) and the
// warps are specialised into a load role, a tensor-core role and softmax roles
// (FlashAttention-3 TMA and warp-specialisation bullets), re-designed for
// Blackwell: accumulators live in tensor memory (TMEM), the MMAs are tcgen05
// issued by one thread, and P goes back into TMEM as the A operand of P V.
//
// CTA layout (Q_TILES = 2): 10 warps.
//   warps 0-3  softmax group for Q tile 0 (one thread per query row)
//   warps 4-7  softmax group for Q tile 1
//   warp  8    TMA producer (one elected lane)
//   warp  9    MMA issuer (one elected lane); owns the TMEM allocation
// TMEM (512 columns x 128 lanes of 32 bit):
//   S_t  columns [128 t, 128 t + 128)   fp32 scores of tile t; P_t (bf16 pairs or
//                                        E4M3 quads) is written over its first
//                                        columns once S_t has been read
//   O_t  columns [256 + D t, 256 + D t + D)   fp32 output accumulator of tile t
// Shared memory: Q tiles (resident for the CTA) + a ring of NSLOT tile slots
// that the producer fills in the order K_0, V_0, K_1, V_1, ...
//
// Per KV block j the MMA thread issues, for t = 0, 1:
//   O_t (+)= P_t(j-1) V_{j-1}   then   S_t = Q_t K_j^T
// so S_t(j) is issued after the MMA that reads P_t(j-1) from the same columns
// (tcgen05 MMAs of one thread execute in issue order), and the commit that
// signals "S_t(j) ready" also guarantees that O_t holds every earlier P V: the
// softmax group may rescale O_t without a further wait.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace attn {

constexpr int kBlockM = 128;  // query rows per Q tile
constexpr int kBlockN = 128;  // keys per K/V block
constexpr uint32_t kStatusTimeout = 1u;

// Device status word (global memory of this module). A kernel whose bounded
// wait ran out ORs kStatusTimeout into it; attn_get_device_status reads and
// clears it.
__device__ uint32_t g_status;

template <int D_, bool FP8_>
struct FwdCfg {
  static constexpr int D = D_;
  static constexpr bool FP8 = FP8_;
  static constexpr int Q_TILES = 2;
  static constexpr int ELEM = FP8 ? 1 : 2;                      // bytes per element
  static constexpr int SW_COLS = 128 / ELEM;                    // elements per 128-byte row
  static constexpr int CHUNKS = D / SW_COLS;                    // 128-byte column chunks per row
  static constexpr int CHUNK_BYTES = 128 * 128;                 // one chunk of a 128-row tile
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;       // one 128-row tile of Q, K or V
  static constexpr int NSLOT = (TILE_BYTES == 32768) ? 4 : 8;   // K/V ring slots
  static constexpr int UMMA_K = FP8 ? 32 : 16;                  // K elements per MMA
  static constexpr int S_KSTEPS = D / UMMA_K;
  static constexpr int PV_KSTEPS = kBlockN / UMMA_K;
  // P in TMEM: bf16 pairs (64 columns), or for FP8 two E4M3 terms hi + lo of
  // each value (32 + 32 columns), so the P V product sees ~7 significant bits
  // of P instead of E4M3's 4; P V then runs over K = 256 (hi | lo) x (V ; V).
  static constexpr int P_COLS = 64;
  static constexpr int PV_KSTEPS_TOTAL = FP8 ? 2 * PV_KSTEPS : PV_KSTEPS;
  static constexpr int NUM_SOFTMAX_THREADS = 128 * Q_TILES;
  static constexpr int PRODUCER_WARP = NUM_SOFTMAX_THREADS / 32;
  static constexpr int MMA_WARP = PRODUCER_WARP + 1;
  static constexpr int THREADS = NUM_SOFTMAX_THREADS + 64;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL0 = 256;
  // Lazy rescaling: the running maximum is only moved when a new block raises it
  // by more than this (log2 units). Exact for any value; 8 keeps bf16 P <= 256.
  // FP8 P must stay below 448 after a 2^8 pre-scale, so it moves every time.
  static constexpr float RESCALE_THRESHOLD = FP8 ? 0.0f : 8.0f;
  static constexpr float P_PRESCALE_LOG2 = 8.0f;  // FP8 only

  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = SMEM_Q + Q_TILES * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_KV + NSLOT * TILE_BYTES;
  static constexpr int NUM_BARS = 1 + 2 * NSLOT + 3 * Q_TILES + 1;
  static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;  // + alignment slack
};

struct FwdParams {
  int N;          // sequence length
  int BH;         // batch * heads
  int num_units;  // work units = BH * ceil(ceil(N/128) / Q_TILES)
  int causal;
  float scale_log2;       // scale * log2(e)
  __nv_bfloat16* o;       // [BH, N, D]
  float* lse;             // [BH, N] or nullptr
  const float* q_scale;   // FP8: [BH, ceil(N/128)]
  const float* k_scale;
  const float* v_scale;
  uint64_t timeout_ns;
};

// Bounded wait that ignores the abort word (used only while draining after an
// abort, so that in-flight copies and MMAs land before the CTA exits).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = b200::global_timer_ns();
  while (!b200::mbar_try_wait(bar, parity)) {
    if (b200::global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ void record_timeout() { atomicOr(&g_status, kStatusTimeout); }

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using namespace b200;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint64_t* q_full = bars;                       // 1
  uint64_t* kv_full = bars + 1;                  // NSLOT
  uint64_t* kv_empty = kv_full + C::NSLOT;       // NSLOT
  uint64_t* s_full = kv_empty + C::NSLOT;        // Q_TILES
  uint64_t* p_full = s_full + C::Q_TILES;        // Q_TILES
  uint64_t* o_done = p_full + C::Q_TILES;        // Q_TILES
  uint64_t* drain_bar = o_done + C::Q_TILES;     // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: (head bh, pair of Q tiles); heavy causal units first
  const int QB = (p.N + kBlockM - 1) / kBlockM;
  const int NPAIR = (QB + C::Q_TILES - 1) / C::Q_TILES;
  const int unit = blockIdx.x;
  const int qpair = NPAIR - 1 - unit / p.BH;
  const int bh = unit % p.BH;
  int nkv[C::Q_TILES];
  int nkv_max = 0;
#pragma unroll
  for (int t = 0; t < C::Q_TILES; ++t) {
    const int qb = qpair * C::Q_TILES + t;
    nkv[t] = (qb >= QB) ? 0 : (p.causal ? qb + 1 : QB);
    nkv_max = max(nkv_max, nkv[t]);
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int t = 0; t < C::Q_TILES; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + t, 128);
      mbar_init(o_done + t, 1);
    }
    mbar_init(drain_bar, 1);
    *abort_word = 0u;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Waiter waiter{abort_word, p.timeout_ns};

  if (warp == C::PRODUCER_WARP) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      mbar_arrive_expect_tx(q_full, C::Q_TILES * C::TILE_BYTES);
#pragma unroll
      for (int t = 0; t < C::Q_TILES; ++t)
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(smem + C::SMEM_Q + t * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_q, q_full, c * C::SW_COLS,
                      (qpair * C::Q_TILES + t) * kBlockM, bh, pol_q);
      const int nloads = 2 * nkv_max;
      int issued = 0;
      for (int i = 0; i < nloads; ++i) {
        const int slot = i % C::NSLOT;
        if (i >= C::NSLOT) {
          if (!waiter.wait(kv_empty + slot, ((i / C::NSLOT) - 1) & 1)) {
            record_timeout();
            break;
          }
        }
        const CUtensorMap* tm = (i & 1) ? &tm_v : &tm_k;
        uint8_t* dst = smem + C::SMEM_KV + slot * C::TILE_BYTES;
        mbar_arrive_expect_tx(kv_full + slot, C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(dst + c * C::CHUNK_BYTES, tm, kv_full + slot, c * C::SW_COLS, (i >> 1) * kBlockN, bh, pol_kv);
        issued = i + 1;
      }
      if (waiter.aborted()) {
        // let every copy still in flight land before shared memory is released
        drain_wait(q_full, 0, p.timeout_ns);
        for (int i = max(0, issued - C::NSLOT); i < issued; ++i)
          drain_wait(kv_full + (i % C::NSLOT), (i / C::NSLOT) & 1, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t fmt = C::FP8 ? 0u : 1u;
      constexpr uint32_t idesc_s = instr_desc(fmt, 128, kBlockN, 0, 0);
      constexpr uint32_t idesc_o = instr_desc(fmt, 128, C::D, 0, 1);
      const uint32_t q_base = smem_addr(smem + C::SMEM_Q);
      const uint32_t kv_base = smem_addr(smem + C::SMEM_KV);
      bool ok = waiter.wait(q_full, 0);
      // S_t = Q_t K_j^T over D in UMMA_K steps (K-major operands, 128B swizzle)
      auto issue_s = [&](int t, uint32_t k_addr) {
        const uint32_t qa = q_base + t * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
          const uint32_t off = (kk / (C::SW_COLS / C::UMMA_K)) * C::CHUNK_BYTES + (kk % (C::SW_COLS / C::UMMA_K)) * 32;
          const uint64_t da = smem_desc(qa + off, 16, 1024);
          const uint64_t db = smem_desc(k_addr + off, 16, 1024);
          if constexpr (C::FP8)
            mma_f8_ss(tmem_base + t * 128, da, db, idesc_s, kk > 0);
          else
            mma_f16_ss(tmem_base + t * 128, da, db, idesc_s, kk > 0);
        }
      };
      // O_t (+)= P_t V_j: P from TMEM (over S_t), V MN-major in shared memory
      auto issue_pv = [&](int t, uint32_t v_addr, bool acc) {
#pragma unroll
        for (int kk = 0; kk < C::PV_KSTEPS_TOTAL; ++kk) {
          const uint64_t db = smem_desc(v_addr + (kk % C::PV_KSTEPS) * C::UMMA_K * 128, C::CHUNK_BYTES, 1024);
          const uint32_t a_tmem = tmem_base + t * 128 + kk * 8;
          if constexpr (C::FP8)
            mma_f8_ts(tmem_base + C::O_COL0 + t * C::D, a_tmem, db, idesc_o, (acc || kk > 0) ? 1u : 0u);
          else
            mma_f16_ts(tmem_base + C::O_COL0 + t * C::D, a_tmem, db, idesc_o, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // K_0: S_t(0) for every tile
      if (ok && nkv_max > 0) {
        ok = waiter.wait(kv_full + 0, 0);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < C::Q_TILES; ++t)
            if (nkv[t] > 0) {
              issue_s(t, kv_base);
              mma_commit(s_full + t);
            }
          mma_commit(kv_empty + 0);
        }
      }
      for (int j = 0; ok && j < nkv_max; ++j) {
        const int vi = 2 * j + 1, ki = 2 * j + 2;
        const int vslot = vi % C::NSLOT, kslot = ki % C::NSLOT;
        bool v_ready = false, k_ready = false, any_s = false;
#pragma unroll
        for (int t = 0; t < C::Q_TILES; ++t) {
          if (j >= nkv[t]) continue;
          if (!(ok = waiter.wait(p_full + t, j & 1))) break;
          if (!v_ready) {
            if (!(ok = waiter.wait(kv_full + vslot, (vi / C::NSLOT) & 1))) break;
            v_ready = true;
          }
          tc_fence_after();
          issue_pv(t, kv_base + vslot * C::TILE_BYTES, j > 0);
          if (j + 1 < nkv[t]) {
            if (!k_ready) {
              if (!(ok = waiter.wait(kv_full + kslot, (ki / C::NSLOT) & 1))) break;
              k_ready = true;
              tc_fence_after();
            }
            issue_s(t, kv_base + kslot * C::TILE_BYTES);
            mma_commit(s_full + t);
            any_s = true;
          } else {
            mma_commit(o_done + t);
          }
        }
        if (!ok) break;
        mma_commit(kv_empty + vslot);
        if (any_s) mma_commit(kv_empty + kslot);
      }
      if (!ok) record_timeout();
      // every MMA this thread issued completes before TMEM can be released
      mma_commit(drain_bar);
      drain_wait(drain_bar, 0, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ======================= softmax groups =======================
    const int t = warp >> 2;                 // Q tile of this group
    const int wq = warp & 3;                 // lane quarter of TMEM this warp may access
    const int r = wq * 32 + lane;            // row inside the tile
    const int qb = qpair * C::Q_TILES + t;
    const int row = qb * kBlockM + r;        // query row inside the head
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_tm = tmem_base + lane_off + t * 128;
    const uint32_t o_tm = tmem_base + lane_off + C::O_COL0 + t * C::D;
    const int T = (p.N + kBlockN - 1) / kBlockN;   // tiles per head (FP8 scales)

    float m_run = __int_as_float(0xff800000u);   // running max of scale*log2(e)*s, log2 units
    float l_run = 0.f;         // running normaliser, relative to 2^m_run
    float q_sc = 1.f, v_max = 1.f;
    if constexpr (C::FP8) {
      if (nkv[t] > 0) {
        q_sc = p.q_scale[bh * T + qb];
        float vm = 0.f;
        for (int i = 0; i < T; ++i) vm = fmaxf(vm, p.v_scale[bh * T + i]);
        v_max = vm > 0.f ? vm : 1.f;
      }
    }
    bool ok = true;
    for (int j = 0; j < nkv[t]; ++j) {
      // TMEM loads/stores below are warp-collective: the whole warp goes on or stops
      ok = __all_sync(0xffffffffu, waiter.wait(s_full + t, j & 1));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(s_tm + 0, sr + 0);
      tmem_ld32(s_tm + 32, sr + 32);
      tmem_ld32(s_tm + 64, sr + 64);
      tmem_ld32(s_tm + 96, sr + 96);
      tmem_ld_wait<128>(sr);

      float c = p.scale_log2;
      float v_log2_ratio = 0.f;
      if constexpr (C::FP8) {
        c *= q_sc * p.k_scale[bh * T + j];
        v_log2_ratio = __log2f(p.v_scale[bh * T + j] / v_max);
      }
      // masking: causal diagonal block and the ragged last key block
      if (j == nkv[t] - 1 && (p.causal || (p.N % kBlockN) != 0)) {
        const int limit = (p.causal ? min(row, p.N - 1) : p.N - 1) - j * kBlockN;  // last visible column
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > limit) sr[i] = 0xff800000u;  // -inf
      }
      float mx = __int_as_float(0xff800000u);
#pragma unroll
      for (int i = 0; i < 128; ++i) mx = fmaxf(mx, __uint_as_float(sr[i]));
      const float m_blk = mx * c;
      float m_use = m_run;
      if (m_blk - m_run > C::RESCALE_THRESHOLD) m_use = m_blk;
      const float alpha = ex2_approx(m_run - m_use);     // 0 on the first block
      // exponent offset: FP8 folds the V tile scale ratio and a 2^8 pre-scale in
      const float m_exp = C::FP8 ? (m_use - v_log2_ratio - C::P_PRESCALE_LOG2) : m_use;
      float sum = 0.f;
      uint32_t pk[C::P_COLS];
      if constexpr (!C::FP8) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * i]), c, -m_exp));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), c, -m_exp));
          sum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
      } else {
        // P = hi + lo, both E4M3: hi = e4m3(p), lo = e4m3(p - hi) (residual in f16)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[4 * i]), c, -m_exp));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[4 * i + 1]), c, -m_exp));
          const float p2 = ex2_approx(fmaf(__uint_as_float(sr[4 * i + 2]), c, -m_exp));
          const float p3 = ex2_approx(fmaf(__uint_as_float(sr[4 * i + 3]), c, -m_exp));
          sum += (p0 + p1) + (p2 + p3);
          const uint32_t h01 = pack_f16x2(p0, p1), h23 = pack_f16x2(p2, p3);
          const uint16_t hi01 = e4m3x2_from_f16x2(h01), hi23 = e4m3x2_from_f16x2(h23);
          const uint16_t lo01 = e4m3x2_from_f16x2(hsub2_u32(h01, f16x2_from_e4m3x2(hi01)));
          const uint16_t lo23 = e4m3x2_from_f16x2(hsub2_u32(h23, f16x2_from_e4m3x2(hi23)));
          pk[i] = static_cast<uint32_t>(hi01) | (static_cast<uint32_t>(hi23) << 16);
          pk[32 + i] = static_cast<uint32_t>(lo01) | (static_cast<uint32_t>(lo23) << 16);
        }
        // back to the units of 2^m_use
        sum *= ex2_approx(-v_log2_ratio - C::P_PRESCALE_LOG2);
      }
      // O_t rescale when this warp moved its maximum (O_t already holds every
      // earlier P V: the commit behind s_full covers them)
      if (j > 0 && __any_sync(0xffffffffu, m_use != m_run)) {
#pragma unroll
        for (int cb = 0; cb < C::D; cb += 32) {
          uint32_t ov[32];
          tmem_ld32(o_tm + cb, ov);
          tmem_ld_wait<32>(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(o_tm + cb, ov);
        }
      }
      // P_t over the first columns of S_t
      tmem_st32(s_tm + 0, pk);
      tmem_st32(s_tm + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full + t);
      l_run = l_run * alpha + sum;
      m_run = m_use;
    }
    if (!ok) record_timeout();
    // ---- epilogue: O = O_acc / l, LSE = (m + log2 l) ln 2
    if (ok && nkv[t] > 0) {
      if (__all_sync(0xffffffffu, waiter.wait(o_done + t, 0))) {
        tc_fence_after();
        float inv_l = 1.f / l_run;
        if constexpr (C::FP8) inv_l *= v_max * 0.00390625f;  // undo the V ratio and 2^8 pre-scale
        const bool in_range = row < p.N;
        __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + (in_range ? row : 0)) * C::D;
#pragma unroll
        for (int cb = 0; cb < C::D; cb += 32) {
          uint32_t ov[32];
          tmem_ld32(o_tm + cb, ov);
          tmem_ld_wait<32>(ov);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
          if (in_range) {
            uint4* dst = reinterpret_cast<uint4*>(orow + cb);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
        if (p.lse != nullptr && in_range)
          p.lse[static_cast<size_t>(bh) * p.N + row] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      } else {
        record_timeout();
      }
    }
  }

  // ---- teardown: every TMEM access and MMA of this CTA is complete here
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace attn
