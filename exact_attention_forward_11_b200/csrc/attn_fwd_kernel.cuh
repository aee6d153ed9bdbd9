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
// CTA layout (Q_TILES = 2): 12 warps = 3 warpgroups.
//   warps 0-3  softmax group for Q tile 0 (one thread per query row)
//   warps 4-7  softmax group for Q tile 1
//   warp  8    TMA producer (one elected lane)
//   warp  9    MMA issuer (one elected lane); owns the TMEM allocation
//   warps 10-11 FP8 (f16 P V): convert each E4M3 V tile to f16 in shared memory;
//              otherwise idle (they complete the control warpgroup, whose
//              registers are handed to the softmax warpgroups)
// TMEM (512 columns x 128 lanes of 32 bit):
//   S_t  columns [128 t, 128 t + 128)   fp32 scores of tile t; P_t (bf16 pairs, or
//                                        f16 pairs for FP8) is written over its first
//                                        columns once S_t has been read
//   O_t  columns [256 + D t, 256 + D t + D)   fp32 output accumulator of tile t
// Shared memory: the Q tiles of the current work unit (reloaded for the next unit
// once its last S MMAs have completed) + a ring of NSLOT tile slots that the
// producer fills in the order K_0, V_0, K_1, V_1, ... CTAs are persistent (one
// per SM) and walk the work units of the launch (see unit_of_round).
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
#include "status.cuh"

namespace attn {

constexpr int kBlockM = 128;  // query rows per Q tile
constexpr int kBlockN = 128;  // keys per K/V block

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
  // FP8 P V in 16 bits: the two otherwise idle control warps convert each E4M3 V
  // tile to an f16 tile in shared memory (exact: every E4M3 value is an f16
  // value) and P is written as f16 pairs, so P V is one kind::f16 MMA over the
  // block's keys. (Measured against P as two E4M3 terms hi + lo over K = 256 with
  // V kept in E4M3: 15 % faster at the same accuracy.)
  static constexpr bool PV_F16 = FP8;
  static constexpr int NSLOT = (TILE_BYTES == 32768) ? 4 : (PV_F16 ? 6 : 8);   // K/V ring slots
  static constexpr int UMMA_K = FP8 ? 32 : 16;                  // K elements per S MMA
  static constexpr int S_KSTEPS = D / UMMA_K;
  static constexpr int PV_UMMA_K = 16;                          // K elements (keys) per P V MMA
  static constexpr int PV_KSTEPS = kBlockN / PV_UMMA_K;
  // P in TMEM: 16-bit pairs (bf16, or f16 for FP8) over the first 64 columns of S
  static constexpr int P_COLS = 64;
  static constexpr int VCONV_BYTES = PV_F16 ? 2 * 128 * 128 : 0;   // one f16 V tile (2 chunks)
  static constexpr int VCONV_BUFS = PV_F16 ? 2 : 0;
  // P is handed to the MMA in P_CHUNKS chunks of 64 keys, each with its own
  // barrier, so P V of a tile starts under the tile's remaining exponentials.
#ifndef ATTN_P_CHUNKS
#define ATTN_P_CHUNKS 2
#endif
  static constexpr int P_CHUNKS = ATTN_P_CHUNKS;
  static constexpr int KEYS_PER_CHUNK = kBlockN / P_CHUNKS;
  static constexpr int NUM_SOFTMAX_THREADS = 128 * Q_TILES;
  static constexpr int PRODUCER_WARP = NUM_SOFTMAX_THREADS / 32;
  static constexpr int MMA_WARP = PRODUCER_WARP + 1;
  static constexpr int THREADS = NUM_SOFTMAX_THREADS + 128;   // + one control warpgroup
  // Register split (launch: 65536 / 384 -> 168 per thread = 64512 in total):
  // softmax warpgroups 216, control warpgroup 64: 2*128*216 + 128*64 = 63488.
  static constexpr uint32_t REGS_SOFTMAX = 216;
  static constexpr uint32_t REGS_CONTROL = 64;
  static_assert(Q_TILES * 128 * REGS_SOFTMAX + 128 * REGS_CONTROL <= 168 * THREADS, "register split");
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL0 = 256;
  // Lazy rescaling: the running maximum is only moved when a new block raises it
  // by more than this (log2 units). Exact for any value; 8 keeps P <= 256, which
  // bf16 and f16 both hold.
  static constexpr float RESCALE_THRESHOLD = 8.0f;
  // Pairs of P values (by index mod 8) whose exp2 runs as a polynomial on the
  // FMA pipe instead of the MUFU unit, in blocks that need no masking. MUFU
  // throughput alone (16/clk/SM) matches the tensor cores at d = 128, so part
  // of the exponentials moves to the otherwise idler FMA pipe.
#ifndef ATTN_POLY_MASK_BF16
#define ATTN_POLY_MASK_BF16 0x00u
#endif
#ifndef ATTN_POLY_MASK_FP8
#define ATTN_POLY_MASK_FP8 0x00u
#endif
  static constexpr uint32_t POLY_MASK = FP8 ? ATTN_POLY_MASK_FP8 : ATTN_POLY_MASK_BF16;

  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = SMEM_Q + Q_TILES * TILE_BYTES;
  static constexpr int SMEM_VCONV = SMEM_KV + NSLOT * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_VCONV + VCONV_BUFS * VCONV_BYTES;
  static constexpr int NUM_BARS = 2 + 2 * NSLOT + (2 + P_CHUNKS) * Q_TILES + 1 + 2 * VCONV_BUFS;
  static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;  // + alignment slack
};

struct FwdParams {
  int N;          // sequence length
  int BH;         // batch * heads
  int num_units;  // work units = BH * ceil(ceil(N/128) / Q_TILES)
  int heads_per_group;  // units walk groups of this many heads (K/V of a group fit in L2)
  int causal;
  float scale_log2;       // scale * log2(e)
  __nv_bfloat16* o;       // [BH, N, D]
  float* lse;             // [BH, N] or nullptr
  const float* q_scale;   // FP8: [BH, ceil(N/128)]
  const float* k_scale;
  const float* v_scale;
  uint64_t timeout_cycles;  // per pipeline wait, in SM cycles
  int fault_unit;           // testing only: the producer withholds this unit's first K tile (-1: none)
  uint32_t out_rows;        // rows of O and LSE the kernel may write (BH * N); checked in debug builds
};

// Bounded wait that ignores the abort word (used only while draining after an
// abort, so that in-flight copies and MMAs land before the CTA exits).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_cycles) {
  const uint64_t t0 = b200::sm_clock();
  while (!b200::mbar_try_wait(bar, parity)) {
    if (b200::sm_clock() - t0 > limit_cycles) return false;
  }
  return true;
}

// 2^x for a pair of fp32 arguments on the FMA/ALU pipes. Cody-Waite style
// reduction x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in the low
// mantissa bits), f in [-1/2, 1/2]; 2^f from a degree-3 polynomial minimising the
// relative error (Remez exchange, fit_exp2_poly.py: max relative error 7.5e-5);
// 2^n is applied by adding n to the exponent field. Arguments are clamped at
// -125 so the result stays normal; 2^-125 stands in for 0, far below any P value
// that survives bf16 / f16 rounding next to the row maximum (P <= 2^8).
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ void exp2_poly_x2(float x0, float x1, float& p0, float& p1) {
  using namespace b200;
  const uint64_t xc = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t tt = f2_add(xc, f2_pack(kRoundMagic, kRoundMagic));   // n in the low mantissa bits
  const uint64_t n = f2_add(tt, f2_pack(-kRoundMagic, -kRoundMagic));  // round(x), exact
  float f0, f1, t0, t1;
  f2_unpack(f2_sub(xc, n), f0, f1);                                    // f = x - n in [-1/2, 1/2]
  f2_unpack(tt, t0, t1);
  // Horner with scalar FMAs (the packed FMA would compete with MUFU for issue)
  float q0 = fmaf(f0, kExp2C3, kExp2C2), q1 = fmaf(f1, kExp2C3, kExp2C2);
  q0 = fmaf(q0, f0, kExp2C1);
  q1 = fmaf(q1, f1, kExp2C1);
  q0 = fmaf(q0, f0, kExp2C0);
  q1 = fmaf(q1, f1, kExp2C0);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

template <uint32_t POLY_MASK>
__device__ __forceinline__ void exp2_pair(float x0, float x1, int i, float& p0, float& p1) {
  if ((POLY_MASK >> (i & 7)) & 1u) {
    exp2_poly_x2(x0, x1, p0, p1);
  } else {
    p0 = b200::ex2_approx(x0);
    p1 = b200::ex2_approx(x1);
  }
}

// Maximum of NCOL (64 or 128) values with 3-input max in eight independent chains.
template <int NCOL = 128>
__device__ __forceinline__ float row_max(const uint32_t* sr) {
  using b200::max3f;
  constexpr int L = NCOL / 8;   // values per chain
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float m = max3f(__uint_as_float(sr[L * k]), __uint_as_float(sr[L * k + 1]), __uint_as_float(sr[L * k + 2]));
#pragma unroll
    for (int j = 3; j < L - 1; j += 2)
      m = max3f(m, __uint_as_float(sr[L * k + j]), __uint_as_float(sr[L * k + j + 1]));
    a[k] = fmaxf(m, __uint_as_float(sr[L * k + L - 1]));
  }
  return max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}
__device__ __forceinline__ float row_max128(const uint32_t (&sr)[128]) { return row_max<128>(sr); }

// P = 2^(s c - m) for keys [32 ch, 32 ch + 32) of one row, as 16 bf16 pairs in
// pk; adds the fp32 values to the packed accumulators. The scale-and-subtract
// is a scalar FMA per element (a packed FMA would compete with MUFU for issue);
// the sums use packed adds, which do not.
template <uint32_t POLY_MASK, int PAIRS = 16, bool F16 = false>
__device__ __forceinline__ void p_chunk_bf16(const uint32_t* sr, int ch, float c, float m,
                                             uint64_t (&acc)[4], uint32_t (&pk)[PAIRS]) {
  using namespace b200;
#pragma unroll
  for (int i = 0; i < PAIRS; ++i) {
    const int k = 2 * PAIRS * ch + 2 * i;
    float p0, p1;
    exp2_pair<POLY_MASK>(fmaf(__uint_as_float(sr[k]), c, -m), fmaf(__uint_as_float(sr[k + 1]), c, -m), i, p0, p1);
    acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
    pk[i] = F16 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
  }
}

// Hands a P chunk to the MMA thread: each thread waits for its own TMEM stores
// and arrives (the barrier counts the 128 threads of the group).
__device__ __forceinline__ void release_chunk(uint64_t* bar) {
  b200::tmem_st_wait();
  b200::tc_fence_before();
  b200::mbar_arrive(bar);
}

// Writes P chunk by chunk into TMEM (over the first columns of S_t) and
// releases each chunk to the MMA thread; returns the fp32 row sum. Software
// pipelined: chunk c is stored, chunk c+1 is computed, and only then does the
// thread wait for chunk c's store and release it, so the store latency hides
// under the next chunk's exponentials.
template <class C, uint32_t POLY_MASK>
__device__ __forceinline__ float p_row_to_tmem(const uint32_t (&sr)[128], float c, float m, uint32_t s_tm,
                                               uint64_t* p_full_t) {
  using namespace b200;
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  constexpr int COLS = 64 / C::P_CHUNKS;   // TMEM columns of P per chunk (bf16 pairs / hi+lo quads)
#pragma unroll
  for (int ch = 0; ch < C::P_CHUNKS; ++ch) {
    uint32_t pk[COLS];
    p_chunk_bf16<POLY_MASK, COLS, C::PV_F16>(sr, ch, c, m, acc, pk);
    if (ch > 0) {
      release_chunk(p_full_t + ch - 1);
    }
    if constexpr (COLS == 16) tmem_st16(s_tm + COLS * ch, pk);
    else if constexpr (COLS == 32) tmem_st32(s_tm + COLS * ch, pk);
    else { tmem_st32(s_tm, pk); tmem_st32(s_tm + 32, pk + 32); }
  }
  release_chunk(p_full_t + C::P_CHUNKS - 1);
  float a, b;
  f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a, b);
  return a + b;
}

// Work unit u of a launch: the pair of Q tiles `qpair` of head `bh`. Units are
// numbered heaviest causal pairs first (pairs count down; heads vary fastest).
// Non-causal launches walk the heads in groups whose K and V fit in L2 together,
// so the CTAs running at the same time share K/V tiles through L2 (causal
// launches use one group: their balance needs the global heavy-first order). A
// persistent CTA b takes one unit per round k in snake order: unit
// k*G + b on even rounds and k*G + G-1-b on odd rounds (G = gridDim.x), so a CTA
// that got one of the heavier units of a round gets one of the lighter ones in
// the next: the causal work per CTA balances without a shared work counter.
__device__ __forceinline__ int unit_of_round(int k) {
  const int base = k * static_cast<int>(gridDim.x);
  return (k & 1) ? base + static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                 : base + static_cast<int>(blockIdx.x);
}

template <class C>
struct UnitInfo {
  int qpair, bh, nkv_max;
  int nkv[C::Q_TILES];
  __device__ __forceinline__ UnitInfo(const FwdParams& p, int u, int QB, int NPAIR) {
    // heads are taken in groups of heads_per_group (the last group may be
    // smaller); inside a group, pairs count down and heads vary fastest
    const int per_group = p.heads_per_group * NPAIR;
    const int grp = u / per_group;
    const int h0 = grp * p.heads_per_group;
    const int hg = min(p.heads_per_group, p.BH - h0);
    const int v = u - grp * per_group;
    qpair = NPAIR - 1 - v / hg;
    bh = h0 + v % hg;
    nkv_max = 0;
#pragma unroll
    for (int t = 0; t < C::Q_TILES; ++t) {
      const int qb = qpair * C::Q_TILES + t;
      nkv[t] = (qb >= QB) ? 0 : (p.causal ? qb + 1 : QB);
      nkv_max = max(nkv_max, nkv[t]);
    }
  }
};

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
  uint64_t* p_full = s_full + C::Q_TILES;        // Q_TILES x P_CHUNKS
  uint64_t* o_done = p_full + C::Q_TILES * C::P_CHUNKS;  // Q_TILES
  uint64_t* drain_bar = o_done + C::Q_TILES;     // 1
  uint64_t* q_empty = drain_bar + 1;             // 1
  uint64_t* vconv_full = q_empty + 1;            // VCONV_BUFS (f16 V tile written: 2 converter warps)
  uint64_t* vconv_empty = vconv_full + C::VCONV_BUFS;  // VCONV_BUFS (its P V MMAs done: MMA commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int QB = (p.N + kBlockM - 1) / kBlockM;
  const int NPAIR = (QB + C::Q_TILES - 1) / C::Q_TILES;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(kv_full + i, 1);
      // slots alternate K, V (NSLOT is even); with the f16 V conversion the two
      // converter warps, not the MMA, are the last readers of a V slot
      mbar_init(kv_empty + i, (C::PV_F16 && (i & 1)) ? 2 : 1);
    }
    for (int b = 0; b < C::VCONV_BUFS; ++b) {
      mbar_init(vconv_full + b, 2);
      mbar_init(vconv_empty + b, 1);
    }
    for (int t = 0; t < C::Q_TILES; ++t) {
      mbar_init(s_full + t, 1);
      for (int c = 0; c < C::P_CHUNKS; ++c) mbar_init(p_full + t * C::P_CHUNKS + c, 128);
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
  const Waiter waiter{abort_word, p.timeout_cycles};

  // Every barrier phase below is a running count over all units this CTA
  // processes (the pipeline is not reset between units). Each role re-sizes
  // its registers inside its own branch, so the compiler can give every branch
  // the budget it was granted.
  if (warp == C::PRODUCER_WARP) {
    // ======================= TMA producer =======================
    // The control warps run their loops with all 32 lanes, so loop state and
    // addresses stay warp-uniform; one elected lane issues each asynchronous
    // operation. (A single divergent lane issuing work is starved of issue
    // slots by the softmax warps that share its scheduler.)
    regs_decrease<C::REGS_CONTROL>();
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, waiter.wait(bar, parity));
    };
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    uint32_t g = 0;        // K/V tile loads issued so far (slot g % NSLOT, phase g / NSLOT)
    int q_loads = 0;       // Q loads issued so far (phase of q_full)
    bool ok = true;
    for (int k = 0; ok && k * static_cast<int>(gridDim.x) < p.num_units; ++k) {
      const int u = unit_of_round(k);
      if (u >= p.num_units) continue;
      const UnitInfo<C> w(p, u, QB, NPAIR);
      // Q is reused by the previous unit's S MMAs until they complete
      if (q_loads > 0 && !(ok = wait_all(q_empty, (q_loads - 1) & 1))) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full, C::Q_TILES * C::TILE_BYTES);
        // (debug) a unit outside the launch's heads or Q tiles loads nothing
        const bool unit_ok = dbg_ok(w.bh < p.BH && w.qpair * C::Q_TILES * kBlockM < p.N, kSiteTmaCoord,
                                    static_cast<unsigned>(u));
#pragma unroll
        for (int t = 0; t < C::Q_TILES && unit_ok; ++t)
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d(smem + C::SMEM_Q + t * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_q, q_full, c * C::SW_COLS,
                        (w.qpair * C::Q_TILES + t) * kBlockM, w.bh, pol_q);
      }
      __syncwarp();
      ++q_loads;
      for (int i = 0; i < 2 * w.nkv_max; ++i, ++g) {
        // testing hook: a tile that is never loaded leaves its full barrier
        // incomplete, so the MMA warp's bounded wait runs out
        if (i == 0 && u == p.fault_unit) continue;
        const uint32_t slot = g % C::NSLOT;
        if (g >= C::NSLOT && !(ok = wait_all(kv_empty + slot, ((g / C::NSLOT) - 1) & 1))) break;
        const CUtensorMap* tm = (i & 1) ? &tm_v : &tm_k;
        uint8_t* dst = smem + C::SMEM_KV + slot * C::TILE_BYTES;
        if (elect_one()) {
          mbar_arrive_expect_tx(kv_full + slot, C::TILE_BYTES);
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d(dst + c * C::CHUNK_BYTES, tm, kv_full + slot, c * C::SW_COLS, (i >> 1) * kBlockN, w.bh,
                        pol_kv);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      if (lane == 0) record_timeout();
      // let every copy still in flight land before shared memory is released
      if (q_loads > 0) drain_wait(q_full, (q_loads - 1) & 1, p.timeout_cycles);
      for (uint32_t i = (g > C::NSLOT ? g - C::NSLOT : 0); i < g; ++i)
        drain_wait(kv_full + (i % C::NSLOT), (i / C::NSLOT) & 1, p.timeout_cycles);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ======================= MMA issuer =======================
    // Warp-uniform loop. One lane, elected once, issues every tcgen05.mma and
    // commit (a commit tracks the MMAs of its own thread only); the instructions
    // are predicated on it, so the warp never diverges. The issue rate of this
    // warp, not the tensor pipe, bounds the MMA segments: under the softmax
    // load on its SM sub-partition one MMA takes ~65-80 cycles to issue.
    regs_decrease<C::REGS_CONTROL>();
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, waiter.wait(bar, parity));
    };
    const uint32_t leader = elect_one() ? 1u : 0u;
    auto commit = [&](uint64_t* bar) { mma_commit(bar, leader); };
    constexpr uint32_t fmt = C::FP8 ? 0u : 1u;                 // e4m3 (kind::f8f6f4) / bf16
    constexpr uint32_t fmt_o = C::PV_F16 ? 0u : fmt;           // f16 P V: kind::f16 with f16 operands
    constexpr uint32_t idesc_s = instr_desc(fmt, 128, kBlockN, 0, 0);
    constexpr uint32_t idesc_o = instr_desc(fmt_o, 128, C::D, 0, 1);
    // Descriptor words, computed once: per k-step and per slot only the low
    // word moves (by a compile-time or per-slot constant).
    constexpr uint32_t hi_kmaj = smem_desc_hi(1024);   // 8 rows x 128 B per swizzle atom
    constexpr uint32_t hi_mnmaj = smem_desc_hi(1024);
    const uint32_t q_lo = smem_desc_lo(smem_addr(smem + C::SMEM_Q), 16);
    const uint32_t k_lo = smem_desc_lo(smem_addr(smem + C::SMEM_KV), 16);
    const uint32_t v_lo = C::PV_F16 ? smem_desc_lo(smem_addr(smem + C::SMEM_VCONV), 128 * 128)
                                    : smem_desc_lo(smem_addr(smem + C::SMEM_KV), C::CHUNK_BYTES);
    // S_t = Q_t K_j^T over D in UMMA_K steps (K-major operands, 128B swizzle)
    auto issue_s = [&](int t, uint32_t slot) {
      const uint32_t qa = q_lo + ((t * C::TILE_BYTES) >> 4);
      const uint32_t ka = k_lo + ((slot * C::TILE_BYTES) >> 4);
      const uint32_t d_tmem = tmem_base + t * 128;
#pragma unroll
      for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
        constexpr int per_chunk = C::SW_COLS / C::UMMA_K;
        const uint32_t off = ((kk / per_chunk) * C::CHUNK_BYTES + (kk % per_chunk) * 32) >> 4;
        const uint64_t da = smem_desc(qa + off, hi_kmaj);
        const uint64_t db = smem_desc(ka + off, hi_kmaj);
        if constexpr (C::FP8)
          mma_f8_ss(d_tmem, da, db, idesc_s, kk > 0, leader);
        else
          mma_f16_ss(d_tmem, da, db, idesc_s, kk > 0, leader);
      }
    };
    // O_t (+)= P_t V_j for the keys of P chunk c: P from TMEM (over S_t), V
    // MN-major in shared memory, K = 16 keys per step: the bf16 V slot, or for
    // FP8 the converted f16 V buffer `slot`.
    auto issue_pv_chunk = [&](int t, uint32_t slot, int c, bool acc) {
      const uint32_t va = v_lo + ((slot * (C::PV_F16 ? C::VCONV_BYTES : C::TILE_BYTES)) >> 4);
      const uint32_t o_tmem = tmem_base + C::O_COL0 + t * C::D;
      const uint32_t p_tmem = tmem_base + t * 128;
      constexpr int STEPS = C::PV_KSTEPS / C::P_CHUNKS;   // K steps per chunk per term
#pragma unroll
      for (int i = 0; i < STEPS; ++i) {
        const int kv = c * STEPS + i;                       // K step within V
        const uint64_t db = smem_desc(va + ((kv * C::PV_UMMA_K * 128) >> 4), hi_mnmaj);
        mma_f16_ts(o_tmem, p_tmem + kv * 8, db, idesc_o, (acc || i > 0) ? 1u : 0u, leader);
      }
    };
    uint32_t g = 0;                       // K/V tiles consumed so far (same count as the producer's)
    uint32_t vb = 0;                      // f16 V buffers consumed so far (vconv phases)
    uint32_t pc[C::Q_TILES];              // blocks of P consumed per tile (p_full phases)
#pragma unroll
    for (int t = 0; t < C::Q_TILES; ++t) pc[t] = 0;
    int units = 0;
    bool ok = true;
    for (int k = 0; ok && k * static_cast<int>(gridDim.x) < p.num_units; ++k) {
      const int u = unit_of_round(k);
      if (u >= p.num_units) continue;
      const UnitInfo<C> w(p, u, QB, NPAIR);
      if (!(ok = wait_all(q_full, units & 1))) break;
      // K_0: S_t(0) for every tile (issued after the previous unit's last P V on
      // this thread, so it overwrites that P only after it has been read)
      if (!(ok = wait_all(kv_full + (g % C::NSLOT), (g / C::NSLOT) & 1))) break;
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < C::Q_TILES; ++t)
        if (w.nkv[t] > 0) {
          issue_s(t, g % C::NSLOT);
          commit(s_full + t);
        }
      commit(kv_empty + (g % C::NSLOT));
      if (w.nkv_max == 1) commit(q_empty);   // the unit's last S MMAs are issued
      for (int j = 0; ok && j < w.nkv_max; ++j) {
        const uint32_t vg = g + 2 * j + 1, kg = g + 2 * j + 2;
        const uint32_t vslot = vg % C::NSLOT, kslot = kg % C::NSLOT;
        bool v_ready = false, k_ready = false, any_s = false;
#pragma unroll
        for (int t = 0; t < C::Q_TILES; ++t) {
          if (j >= w.nkv[t]) continue;
          if (!v_ready) {
            if constexpr (C::PV_F16)
              ok = wait_all(vconv_full + (vb & 1), (vb >> 1) & 1);
            else
              ok = wait_all(kv_full + vslot, (vg / C::NSLOT) & 1);
            if (!ok) break;
            v_ready = true;
          }
#pragma unroll
          for (int c = 0; c < C::P_CHUNKS; ++c) {
            if (!(ok = wait_all(p_full + t * C::P_CHUNKS + c, pc[t] & 1))) break;
            tc_fence_after();
            issue_pv_chunk(t, C::PV_F16 ? (vb & 1) : vslot, c, j > 0 || c > 0);
          }
          if (!ok) break;
          ++pc[t];
          if (j + 1 < w.nkv[t]) {
            if (!k_ready) {
              if (!(ok = wait_all(kv_full + kslot, (kg / C::NSLOT) & 1))) break;
              k_ready = true;
              tc_fence_after();
            }
            issue_s(t, kslot);
            commit(s_full + t);
            any_s = true;
          } else {
            commit(o_done + t);
          }
        }
        if (!ok) break;
        if constexpr (C::PV_F16) {
          commit(vconv_empty + (vb & 1));   // the converted tile's P V MMAs are issued
          ++vb;
        } else {
          commit(kv_empty + vslot);
        }
        if (any_s) commit(kv_empty + kslot);
        if (any_s && j + 2 == w.nkv_max) commit(q_empty);   // the unit's last S MMAs are issued
      }
      g += 2 * w.nkv_max;
      ++units;
    }
    if (!ok && lane == 0) record_timeout();
    // every MMA this warp issued completes before TMEM can be released
    commit(drain_bar);
    drain_wait(drain_bar, 0, p.timeout_cycles);
    __syncwarp();
  } else if (warp > C::MMA_WARP) {
    regs_decrease<C::REGS_CONTROL>();
    if constexpr (C::PV_F16) {
      // ======================= E4M3 -> f16 V conversion =======================
      // The two remaining control warps turn each E4M3 V tile (128 keys x 128
      // bytes, 128-byte swizzle) into an f16 tile of two 64-column chunks with
      // the same swizzle, the MN-major B operand of the f16 P V MMA. Every E4M3
      // value is exactly an f16 value. Thread ct handles (row, 16-byte unit)
      // pairs ct, ct + 64, ...: eight threads read one 128-byte row.
      auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, waiter.wait(bar, parity));
      };
      const int ct = (warp - C::MMA_WARP - 1) * 32 + lane;
      uint32_t g = 0, vb = 0;
      bool ok = true;
      for (int k = 0; ok && k * static_cast<int>(gridDim.x) < p.num_units; ++k) {
        const int u = unit_of_round(k);
        if (u >= p.num_units) continue;
        const UnitInfo<C> w(p, u, QB, NPAIR);
        for (int j = 0; j < w.nkv_max; ++j, ++vb) {
          const uint32_t vg = g + 2 * j + 1, vslot = vg % C::NSLOT, b = vb & 1;
          if (!(ok = wait_all(kv_full + vslot, (vg / C::NSLOT) & 1))) break;
          if (vb >= 2 && !(ok = wait_all(vconv_empty + b, ((vb >> 1) - 1) & 1))) break;
          const uint8_t* src = smem + C::SMEM_KV + vslot * C::TILE_BYTES;
          uint8_t* dst = smem + C::SMEM_VCONV + b * C::VCONV_BYTES;
#pragma unroll 2
          for (int i = 0; i < 16; ++i) {
            const int pr = ct + 64 * i, r = pr >> 3, un = pr & 7;        // key row, 16-code unit (d = 16 un ..)
            const uint4 c16 = *reinterpret_cast<const uint4*>(src + r * 128 + ((un ^ (r & 7)) << 4));
            const uint32_t wds[4] = {c16.x, c16.y, c16.z, c16.w};
            uint32_t h[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              h[2 * q] = f16x2_from_e4m3x2(static_cast<uint16_t>(wds[q] & 0xFFFFu));
              h[2 * q + 1] = f16x2_from_e4m3x2(static_cast<uint16_t>(wds[q] >> 16));
            }
            // f16 d = 16 un + e sits in chunk un / 4, 16-byte unit 2 (un % 4) + (e / 8)
            uint8_t* drow = dst + (un >> 2) * (128 * 128) + r * 128;
            const int u0 = 2 * (un & 3);
            *reinterpret_cast<uint4*>(drow + ((u0 ^ (r & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(drow + (((u0 + 1) ^ (r & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
          }
          fence_proxy_async_shared();   // the MMA (async proxy) reads what these threads wrote
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(vconv_full + b);
            mbar_arrive(kv_empty + vslot);   // the E4M3 V slot is read
          }
        }
        g += 2 * w.nkv_max;
      }
      if (!ok && lane == 0) record_timeout();
    }
  } else {
    // ======================= softmax groups =======================
    regs_increase<C::REGS_SOFTMAX>();
    const int t = warp >> 2;                 // Q tile of this group
    const int wq = warp & 3;                 // lane quarter of TMEM this warp may access
    const int r = wq * 32 + lane;            // row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_tm = tmem_base + lane_off + t * 128;
    const uint32_t o_tm = tmem_base + lane_off + C::O_COL0 + t * C::D;
    const int T = (p.N + kBlockN - 1) / kBlockN;   // tiles per head (FP8 scales)
    uint32_t sc = 0;                               // S_t completions consumed (s_full phases)
    uint32_t oc = 0;                               // O_t completions consumed (o_done phases)
    bool ok = true;
    for (int k = 0; ok && k * static_cast<int>(gridDim.x) < p.num_units; ++k) {
      const int u = unit_of_round(k);
      if (u >= p.num_units) continue;
      const UnitInfo<C> w(p, u, QB, NPAIR);
      int nkv_t = w.nkv[0];                        // (no dynamic indexing: keeps nkv in registers)
#pragma unroll
      for (int i = 1; i < C::Q_TILES; ++i)
        if (t == i) nkv_t = w.nkv[i];
      if (nkv_t == 0) continue;
      const int bh = w.bh;
      const int qb = w.qpair * C::Q_TILES + t;
      const int row = qb * kBlockM + r;            // query row inside the head
      float m_run = __int_as_float(0xff800000u);   // running max of scale*log2(e)*s, log2 units
      float l_run = 0.f;                           // running normaliser, relative to 2^m_run
      float q_sc = 1.f, v_max = 1.f;
      float ks_next = 1.f, vs_next = 1.f;          // FP8: block j's K and V tile scales, loaded one block ahead
      if constexpr (C::FP8) {
        ks_next = p.k_scale[bh * T];
        vs_next = p.v_scale[bh * T];
        q_sc = p.q_scale[bh * T + qb];
        float vm = 0.f;
        for (int i = 0; i < T; ++i) vm = fmaxf(vm, p.v_scale[bh * T + i]);
        v_max = vm > 0.f ? vm : 1.f;
      }
      for (int j = 0; j < nkv_t; ++j) {
        const float ks = ks_next, vs = vs_next;
        if (C::FP8 && j + 1 < nkv_t) {   // issued before the S wait, used one block later
          ks_next = p.k_scale[bh * T + j + 1];
          vs_next = p.v_scale[bh * T + j + 1];
        }
        // TMEM loads/stores below are warp-collective: the whole warp goes on or stops
        ok = __all_sync(0xffffffffu, waiter.wait(s_full + t, sc & 1));
        if (!ok) break;
        ++sc;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(s_tm + 0, sr + 0);
        tmem_ld32(s_tm + 32, sr + 32);
        tmem_ld32(s_tm + 64, sr + 64);
        tmem_ld32(s_tm + 96, sr + 96);
        tmem_ld_wait<128>(sr);
        float c = p.scale_log2, v_log2_ratio = 0.f;
        if constexpr (C::FP8) {
          // A tile scale of 0 (a tile that dequantises to zeros) must not turn
          // the row into NaN: the score factor is kept positive (the scores
          // of such a tile are then ~0, as they should be) and the V ratio at
          // or above 2^-64 (its P rounds to zero in E4M3; the fp32 row sum
          // keeps its exact share of the normaliser).
          c = fmaxf(c * (q_sc * ks), 1e-30f);
          v_log2_ratio = __log2f(fmaxf(vs / v_max, 5.421010862427522e-20f));
        }
        // masking: causal diagonal block and the ragged last key block
        const bool masked = (j == nkv_t - 1) && (p.causal || (p.N % kBlockN) != 0);
        if (masked) {
          const int limit = (p.causal ? min(row, p.N - 1) : p.N - 1) - j * kBlockN;  // last visible column
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > limit) sr[i] = 0xff800000u;  // -inf
        }
        const float m_blk = row_max128(sr) * c;
        float m_use = m_run;
        if (m_blk - m_run > C::RESCALE_THRESHOLD) m_use = m_blk;
        // exponent offset: FP8 folds the V tile scale ratio in
        const float m_exp = C::FP8 ? (m_use - v_log2_ratio) : m_use;
        const bool moved = m_use != m_run;
        // 2^(m_run - m_use); 0 on the first block
        const float alpha = moved ? ex2_approx(m_run - m_use) : 1.f;
        // O_t rescale when this warp moved its maximum (O_t already holds every
        // earlier P V: the commit behind s_full covers them); it must land
        // before the first P chunk of this block is released to the MMA.
        if (j > 0 && __any_sync(0xffffffffu, moved)) {
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
        // P_t over the first columns of S_t, chunk by chunk; masked blocks keep
        // every exponential on MUFU (exact zeros for -inf)
        uint64_t* pf = p_full + t * C::P_CHUNKS;
        float sum = masked ? p_row_to_tmem<C, 0u>(sr, c, m_exp, s_tm, pf)
                           : p_row_to_tmem<C, C::POLY_MASK>(sr, c, m_exp, s_tm, pf);
        if constexpr (C::FP8) sum *= ex2_approx(-v_log2_ratio);  // units of 2^m_use
        l_run = l_run * alpha + sum;
        m_run = m_use;
      }
      if (!ok) break;
      // ---- epilogue: O = O_acc / l, LSE = (m + log2 l) ln 2. The next unit's
      // first P V (which overwrites O_t) waits for this group's P, which comes
      // after these TMEM loads.
      ok = __all_sync(0xffffffffu, waiter.wait(o_done + t, oc & 1));
      if (!ok) break;
      ++oc;
      tc_fence_after();
      float inv_l = 1.f / l_run;
      if constexpr (C::FP8) inv_l *= v_max;   // undo the V ratio folded into P
      const size_t grow = static_cast<size_t>(bh) * p.N + row;   // row over all heads
      const bool in_range = row < p.N && dbg_ok(grow < p.out_rows, kSiteFwdOut, grow);
      __nv_bfloat16* orow = p.o + (in_range ? grow : 0) * C::D;
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
      if (p.lse != nullptr && in_range) p.lse[grow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
    if (!ok) record_timeout();
  }

  // ---- teardown: every TMEM access and MMA of this CTA is complete here
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace attn
