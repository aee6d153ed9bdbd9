// attn_fwd1_kernel.cuh - fused attention forward with one Q tile per CTA and
// double-buffered scores in tensor memory (BF16, and MXFP8 with hardware block
// scales).
//
// Same operation as attn_fwd_kernel.cuh ("Self-Attention, CUDA kernels and
// FlashAttention", section 1, eq. Scores and eq. Attention, section 3 tiling and
// online softmax; "FlashAttention scaling, multi-GPU training and weight
// quantization", section 1, FlashAttention-2/-3 bullets) on a different on-chip
// schedule: a persistent CTA works on one 128-row Q tile at a time and keeps two
// S buffers in tensor memory, so the MMA thread computes S(j+2) while the softmax
// warps turn S(j+1) into P, and every SM sub-partition hosts exactly one softmax
// warp.
//
// MXFP8 ("Efficient MoE training for biological foundation models", the
// low-precision paragraph: one power-of-two scale per block of 32 values, the
// products on the tensor cores' block-scaled instructions): Q, K and V are E4M3
// codes with an E8M0 scale byte per 32 consecutive values of a row (d = 128: four
// bytes per row).
//  * S = Q K^T is tcgen05.mma.kind::mxf8f6f4.block_scale (K = 32 per
//    instruction: one scale of each operand per row and instruction, read from
//    tensor memory), so S leaves the tensor cores already dequantised.
//  * V's blocks run along d, not along the keys that P V contracts over, so the
//    tensor cores cannot apply them. The two otherwise idle control warps turn
//    each V tile into f16 with its scales applied, relative to the largest V
//    scale byte sv_b of that 32-column block over the keys the Q tile sees:
//    V16 = code * 2^(e - sv_b + 7), exact in f16 for every block whose scale lies
//    within 22 binades of sv_b (smaller ones round in f16's subnormal range or
//    flush to zero: below 2^-22 of the column block's largest values). P V is an
//    f16 MMA (P as f16 pairs); the epilogue multiplies column block b by
//    2^(sv_b - 127 - 7). Each softmax warp finds the same sv_b on its own (a
//    running byte-wise maximum of the V scale words of every key row it passes),
//    so no value passes between the groups.
//
// CTA: warps 0-3 softmax (one thread per query row; warp w reads TMEM lanes
// 32 w .. 32 w + 31), warp 4 TMA producer, warp 5 MMA issuer (owns TMEM); BF16:
// 8 warps (6-7 idle); MXFP8: 12 warps, 6-9 the V conversion (one per SM
// sub-partition), 10-11 idle, registers re-split per warpgroup.
// TMEM (512 columns): S buffers [0, 128) and [128, 256) (P over their first 64
// columns), O [256, 256 + D). MXFP8 scale factors: Q [384, 388), K of S buffer b
// [388 + 4 b, 392 + 4 b), in the layout the block-scaled MMA reads for M = N =
// 128: lane 32 q + r of every lane quarter q holds, in column base + h, the four
// block scales (bytes 0..3 = 32-value blocks 0..3) of row 32 h + r.
// Every barrier phase is a running count over the CTA's units (a global block
// counter B for the per-block barriers); every wait is bounded (Waiter) and a
// wait that runs out records ATTN_ERR_TIMEOUT.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_fwd_kernel.cuh"
#include "sm100.cuh"
#include "status.cuh"

namespace attn {

#ifndef ATTN_FWD1_POLY_MASK
#define ATTN_FWD1_POLY_MASK 0x00u
#endif
#ifndef ATTN_FWD1_NSLOT_BF16
#define ATTN_FWD1_NSLOT_BF16 5
#endif

template <int D_, bool MX_>
struct Fwd1Cfg {
  static constexpr int D = D_;
  static constexpr bool MX = MX_;
  static_assert(!MX || D == 128, "MXFP8 rows hold 4 blocks of 32 codes");
  static constexpr bool PV_F16 = MX;             // P as f16 pairs for the f16 P V
  static constexpr int Q_TILES = 1;
  static constexpr int ELEM = MX ? 1 : 2;
  static constexpr int SW_COLS = 128 / ELEM;     // elements per 128-byte row chunk
  static constexpr int CHUNKS = D / SW_COLS;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;
  static constexpr int NSLOT = MX ? 8 : (TILE_BYTES == 32768 ? ATTN_FWD1_NSLOT_BF16 : 8);
  static_assert(!MX || NSLOT % 2 == 0, "K and V alternate over the ring slots");
  static constexpr int UMMA_K = MX ? 32 : 16;    // K per S instruction
  static constexpr int S_KSTEPS = D / UMMA_K;
  static constexpr int PV_KSTEPS = kBlockN / 16;
  static constexpr int P_CHUNKS = ATTN_P_CHUNKS;
  static constexpr float RESCALE_THRESHOLD = 8.0f;
  static constexpr uint32_t POLY_MASK = ATTN_FWD1_POLY_MASK;
  // MXFP8: 16 warps. The softmax of the Q tile runs on two warpgroups (warps 0-3
  // and 12-15), warpgroup h taking keys [64 h, 64 h + 64) of every row: one warp
  // on an SM sub-partition cannot issue exponentials at the MUFU unit's rate,
  // two warps sharing it can. The two warps of a lane quarter trade their row
  // maxima (every block) and row sums (every unit) through shared memory and a
  // bounded mbarrier. The V conversion runs on warps 6-9, one per sub-partition;
  // warps 10-11 are idle. Register split (launch: 65536 / 512 -> 128 per
  // thread): softmax warpgroups 176, the other two 80: 2 * 128 * (176 + 80).
  // BF16: 8 warps, one softmax warpgroup (keys of a row on one thread).
  static constexpr int SPLIT = MX ? 2 : 1;
  static constexpr int SOFTMAX_WARP1 = 12;       // first warp of the second softmax warpgroup (SPLIT == 2)
  static constexpr int THREADS = MX ? 512 : 256;
  static constexpr int PRODUCER_WARP = 4;
  static constexpr int MMA_WARP = 5;
  static constexpr int CONV_WARPS = MX ? 4 : 0;
  static constexpr int CONV_ITERS = MX ? 128 * 8 / (32 * CONV_WARPS) : 1;   // (row, 16-code unit) pairs per thread
  static constexpr uint32_t REGS_SOFTMAX = 176;
  static constexpr uint32_t REGS_OTHER = 80;
  static_assert(!MX || 2 * 128 * (REGS_SOFTMAX + REGS_OTHER) <= 65536, "register split");
  static_assert(SPLIT == 1 || ATTN_P_CHUNKS == 2, "one P chunk per softmax warpgroup");
  // TMEM column of P chunk c inside its S buffer: P chunk c (keys 64 c ..) lies over
  // the S columns of the warpgroup that writes it
  static constexpr uint32_t P_COL_STEP = SPLIT == 2 ? 64 : 32;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL0 = 256;
  static constexpr uint32_t SFA_COL = 384;
  static constexpr uint32_t SFB_COL = 388;       // + 4 b
  static constexpr int VCONV_BYTES = MX ? 2 * 128 * 128 : 0;   // one f16 V tile (two 64-column chunks)
  static constexpr int VCONV_BUFS = MX ? 2 : 0;
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = SMEM_Q + TILE_BYTES;
  static constexpr int SMEM_VCONV = SMEM_KV + NSLOT * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_VCONV + VCONV_BUFS * VCONV_BYTES;
  // q_full, q_empty, kv_full[NSLOT], kv_empty[NSLOT], s_full[2], p_full[2][P_CHUNKS],
  // pv_done[2], sfb_ready[2], vconv_full[2], vconv_empty[2], drain, xch[4], sv_ready[4]
  static constexpr int NUM_BARS = 2 + 2 * NSLOT + 2 + 2 * P_CHUNKS + 2 + 2 + 2 + 2 + 1 + 4 + 4;
  static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;    // TMEM address, abort word, sv words [4]
  static constexpr int SMEM_XCH = SMEM_MISC + 32;              // [2 slots][2 warpgroups][128 rows] fp32
  static constexpr int SMEM_BYTES = SMEM_XCH + (SPLIT > 1 ? 2 * 2 * 128 * 4 : 0) + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

struct Fwd1Params {
  int N, BH, num_units, heads_per_group, causal;
  float scale_log2;          // scale * log2(e)
  __nv_bfloat16* o;          // [BH, N, D]
  float* lse;                // [BH, N] or nullptr
  const uint8_t* q_sf;       // MXFP8: [BH, N, 4] E8M0 bytes (16-byte aligned)
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  uint64_t timeout_cycles;   // per pipeline wait, in SM cycles
  int fault_unit;            // testing only: the producer withholds this unit's first K tile (-1: none)
  uint32_t out_rows;         // rows of O and LSE the kernel may write (BH * N); checked in debug builds
};

// (debug builds) a scale-byte row index inside the [BH * N] arrays
__device__ __forceinline__ bool sf_row_ok(const Fwd1Params& p, size_t r) {
  return dbg_ok(r < static_cast<size_t>(p.BH) * p.N, kSiteFwd1ScaleLoad, r);
}

// Instruction descriptor of the block-scaled E4M3 x E4M3 MMA with fp32
// accumulation and UE8M0 scales, both operands K-major; sf_id picks the scale
// byte (32-value block) that this K = 32 step uses.
__device__ __forceinline__ uint32_t mx_instr_desc(uint32_t M, uint32_t N, uint32_t sf_id) {
  return (sf_id << 4) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24) | (sf_id << 29);
}

// D[tmem] (+)= (A * 2^sfa) (B * 2^sfb)^T over one K = 32 step (predicated on `leader`)
__device__ __forceinline__ void mma_mx_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate,
                                          uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %7, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "r"(leader)
      : "memory");
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&w)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3])
               : "memory");
}

// Read-only global loads issued exactly where they stand (volatile: the compiler
// may neither sink them to their use nor reload them there), so that a load
// issued a pipeline stage ahead keeps its latency hidden.
__device__ __forceinline__ uint32_t ld_nc_u8(const uint8_t* ptr) {
  uint32_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=r"(v) : "l"(ptr));
  return v;
}
__device__ __forceinline__ uint32_t ld_nc_u32(const uint32_t* ptr) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(ptr));
  return v;
}

// Byte-wise maximum of two words of four scale bytes.
__device__ __forceinline__ uint32_t max_u8x4(uint32_t a, uint32_t b) { return __vmaxu4(a, b); }

// f16 bits of 2^x for x <= 15 (0 below f16's smallest subnormal 2^-24), with
// selects only (no branch: the lanes of a warp hold different x).
__device__ __forceinline__ uint32_t f16_pow2_bits(int x) {
  const uint32_t normal = static_cast<uint32_t>(max(x + 15, 0)) << 10;
  const uint32_t sub = 1u << min(max(x + 24, 0), 31);
  return x >= -14 ? normal : (x >= -24 ? sub : 0u);
}

// fp32 2^x for integer x in [-149, 127].
__device__ __forceinline__ float f32_pow2(int x) {
  return x >= -126 ? __int_as_float((x + 127) << 23) : __int_as_float(1 << (x + 149));
}

// Byte-wise maximum of the scale words of key rows [0, kend) of one head (all
// 32 lanes of the calling warp take part; every lane returns the result). A
// row's word is 4 bytes; 16-byte loads where the head's rows are 16-byte aligned.
__device__ __forceinline__ uint32_t head_sf_max(const uint8_t* sf, size_t head_row0, int kend, int lane) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(sf) + head_row0;
  const int a0 = min(static_cast<int>((4u - static_cast<uint32_t>(head_row0 & 3u)) & 3u), kend);
  const int nq = (kend - a0) >> 2;
  const int tail0 = a0 + 4 * nq;
  uint32_t m = 0u;
  if (lane < a0) m = w[lane];
  if (tail0 + lane < kend) m = max_u8x4(m, w[tail0 + lane]);
  const uint4* w4 = reinterpret_cast<const uint4*>(w + a0);
  int i = lane;
  for (; i + 96 < nq; i += 128) {   // four 16-byte loads in flight per lane
    const uint4 x0 = w4[i], x1 = w4[i + 32], x2 = w4[i + 64], x3 = w4[i + 96];
    m = max_u8x4(m, max_u8x4(max_u8x4(x0.x, x0.y), max_u8x4(x0.z, x0.w)));
    m = max_u8x4(m, max_u8x4(max_u8x4(x1.x, x1.y), max_u8x4(x1.z, x1.w)));
    m = max_u8x4(m, max_u8x4(max_u8x4(x2.x, x2.y), max_u8x4(x2.z, x2.w)));
    m = max_u8x4(m, max_u8x4(max_u8x4(x3.x, x3.y), max_u8x4(x3.z, x3.w)));
  }
  for (; i < nq; i += 32) {
    const uint4 x = w4[i];
    m = max_u8x4(m, max_u8x4(max_u8x4(x.x, x.y), max_u8x4(x.z, x.w)));
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) m = max_u8x4(m, __shfl_xor_sync(0xffffffffu, m, s));
  return m;
}

// One softmax warpgroup's share of a row (64 keys, SPLIT == 2): P = 2^(s c - m)
// as 16-bit pairs into TMEM at p_tm, released to the MMA thread on `bar`;
// returns the fp32 sum of the share.
template <class C>
__device__ __forceinline__ float p_share_to_tmem(const uint32_t (&sr)[64], float c, float m, uint32_t p_tm,
                                                 uint64_t* bar) {
  using namespace b200;
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  uint32_t pk[32];
  p_chunk_bf16<0u, 32, C::PV_F16>(sr, 0, c, m, acc, pk);
  tmem_st32(p_tm, pk);
  release_chunk(bar);
  float a, b;
  f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a, b);
  return a + b;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd1_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Fwd1Params p) {
  using namespace b200;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 1;
  uint64_t* kv_full = q_empty + 1;                   // NSLOT
  uint64_t* kv_empty = kv_full + C::NSLOT;           // NSLOT
  uint64_t* s_full = kv_empty + C::NSLOT;            // 2: S of a buffer complete (MMA commit)
  uint64_t* p_full = s_full + 2;                     // 2 x P_CHUNKS: P chunk in TMEM (128 softmax threads)
  uint64_t* pv_done = p_full + 2 * C::P_CHUNKS;      // 2: P V of the buffer's block complete (MMA commit)
  uint64_t* sfb_ready = pv_done + 2;                 // 2: MX scale factors for the buffer's S (4 softmax warps)
  uint64_t* vconv_full = sfb_ready + 2;              // 2: MX f16 V tile written (2 converter warps)
  uint64_t* vconv_empty = vconv_full + 2;            // 2: its P V done (MMA commit)
  uint64_t* drain_bar = vconv_empty + 2;
  uint64_t* xch = drain_bar + 1;                     // 4: the two softmax warps of a lane quarter traded values
  uint64_t* sv_ready = xch + 4;                      // 4: MX, a unit's V scale maxima written (converter warp)
  float* xbuf = reinterpret_cast<float*>(smem + C::SMEM_XCH);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  uint32_t* abort_word = tmem_slot + 1;
  uint32_t* sv_word = tmem_slot + 4;                 // 4 slots (unit index mod 4)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int QB = (p.N + kBlockM - 1) / kBlockM;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, (C::MX && (i & 1)) ? C::CONV_WARPS : 1);   // MX V slots: the converter warps read them last
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      for (int c = 0; c < C::P_CHUNKS; ++c) mbar_init(p_full + b * C::P_CHUNKS + c, 128);
      mbar_init(pv_done + b, 1);
      mbar_init(sfb_ready + b, 4);
      mbar_init(vconv_full + b, C::CONV_WARPS > 0 ? C::CONV_WARPS : 1);
      mbar_init(vconv_empty + b, 1);
    }
    mbar_init(drain_bar, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(xch + q, 2);
      mbar_init(sv_ready + q, 1);
    }
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
  auto wait_all = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, waiter.wait(bar, parity)); };
  FwdParams up{};   // the fields the unit decoder reads
  up.N = p.N;
  up.BH = p.BH;
  up.num_units = p.num_units;
  up.heads_per_group = p.heads_per_group;
  up.causal = p.causal;
  // first valid unit at or after round k0 (its round in kk), or -1
  auto find_unit = [&](int k0, int& kk) -> int {
    for (kk = k0; kk * static_cast<int>(gridDim.x) < p.num_units; ++kk) {
      const int u = unit_of_round(kk);
      if (u < p.num_units) return u;
    }
    return -1;
  };
  bool ok = true;

  if (warp == C::PRODUCER_WARP) {
    // ======================= TMA producer =======================
    if constexpr (C::MX) regs_decrease<C::REGS_OTHER>();
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    uint32_t g = 0;   // K/V tiles loaded (slot g % NSLOT, phase g / NSLOT)
    int units = 0;
    int kc;
    for (int u = find_unit(0, kc); ok && u >= 0; u = find_unit(kc + 1, kc)) {
      const UnitInfo<C> w(up, u, QB, QB);
      // Q is read by the previous unit's S MMAs until they complete
      if (units > 0 && !(ok = wait_all(q_empty, (units - 1) & 1))) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
        // (debug) a unit outside the launch's heads or Q tiles loads nothing
        const bool unit_ok = dbg_ok(w.bh < p.BH && w.qpair * kBlockM < p.N, kSiteTmaCoord, static_cast<unsigned>(u));
        for (int c = 0; c < C::CHUNKS && unit_ok; ++c)
          tma_load_3d(smem + C::SMEM_Q + c * C::CHUNK_BYTES, &tm_q, q_full, c * C::SW_COLS, w.qpair * kBlockM, w.bh,
                      pol_q);
      }
      __syncwarp();
      ++units;
      for (int i = 0; i < 2 * w.nkv[0]; ++i, ++g) {
        // testing hook: a tile that is never loaded leaves its full barrier
        // incomplete, so the MMA warp's bounded wait runs out
        if (i == 0 && u == p.fault_unit) continue;
        const uint32_t slot = g % C::NSLOT;
        if (g >= C::NSLOT && !(ok = wait_all(kv_empty + slot, ((g / C::NSLOT) - 1) & 1))) break;
        const CUtensorMap* tm = (i & 1) ? &tm_v : &tm_k;
        if (elect_one()) {
          mbar_arrive_expect_tx(kv_full + slot, C::TILE_BYTES);
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d(smem + C::SMEM_KV + slot * C::TILE_BYTES + c * C::CHUNK_BYTES, tm, kv_full + slot,
                        c * C::SW_COLS, (i >> 1) * kBlockN, w.bh, pol_kv);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      if (lane == 0) record_timeout();
      // every copy still in flight lands before shared memory is released
      if (units > 0) drain_wait(q_full, (units - 1) & 1, p.timeout_cycles);
      for (uint32_t i = (g > C::NSLOT ? g - C::NSLOT : 0); i < g; ++i)
        drain_wait(kv_full + (i % C::NSLOT), (i / C::NSLOT) & 1, p.timeout_cycles);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ======================= MMA issuer =======================
    if constexpr (C::MX) regs_decrease<C::REGS_OTHER>();
    // Per unit: S(0), S(1), then for each block j: P V(j) (chunk by chunk as P
    // arrives), then S(j + 2) into the buffer P(j) occupied. The tensor pipe runs
    // one thread's MMAs in issue order, so S(j + 2) overwrites P(j) only after
    // P V(j) has read it.
    const uint32_t leader = elect_one() ? 1u : 0u;
    auto commit = [&](uint64_t* bar) { mma_commit(bar, leader); };
    constexpr uint32_t idesc_s = instr_desc(1u, 128, kBlockN, 0, 0);                 // bf16 S
    constexpr uint32_t idesc_o = instr_desc(C::MX ? 0u : 1u, 128, C::D, 0, 1);       // f16 / bf16 P V
    constexpr uint32_t hi = smem_desc_hi(1024);
    const uint32_t q_lo = smem_desc_lo(smem_addr(smem + C::SMEM_Q), 16);
    const uint32_t k_lo = smem_desc_lo(smem_addr(smem + C::SMEM_KV), 16);
    const uint32_t v_lo = C::MX ? smem_desc_lo(smem_addr(smem + C::SMEM_VCONV), 128 * 128)
                                : smem_desc_lo(smem_addr(smem + C::SMEM_KV), C::CHUNK_BYTES);
    // S(buffer b) = Q K(slot)^T over D in UMMA_K steps (K-major, 128-byte swizzle)
    auto issue_s = [&](uint32_t b, uint32_t slot) {
      const uint32_t ka = k_lo + ((slot * C::TILE_BYTES) >> 4);
      const uint32_t d_tmem = tmem_base + b * 128;
#pragma unroll
      for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
        constexpr int per_chunk = C::SW_COLS / C::UMMA_K;
        const uint32_t off = ((kk / per_chunk) * C::CHUNK_BYTES + (kk % per_chunk) * 32) >> 4;
        const uint64_t da = smem_desc(q_lo + off, hi), db = smem_desc(ka + off, hi);
        if constexpr (C::MX)
          mma_mx_ss(d_tmem, da, db, mx_instr_desc(128, kBlockN, static_cast<uint32_t>(kk)),
                    tmem_base + C::SFA_COL, tmem_base + C::SFB_COL + 4 * b, kk > 0, leader);
        else
          mma_f16_ss(d_tmem, da, db, idesc_s, kk > 0, leader);
      }
    };
    // O (+)= P(buffer b) V for the keys of P chunk c; V MN-major: the bf16 ring
    // slot, or for MXFP8 the f16 buffer `src`
    auto issue_pv_chunk = [&](uint32_t b, uint32_t src, int c, bool acc) {
      const uint32_t va = v_lo + ((src * (C::MX ? C::VCONV_BYTES : C::TILE_BYTES)) >> 4);
      constexpr int STEPS = C::PV_KSTEPS / C::P_CHUNKS;
#pragma unroll
      for (int i = 0; i < STEPS; ++i) {
        const int kv = c * STEPS + i;
        mma_f16_ts(tmem_base + C::O_COL0, tmem_base + b * 128 + c * C::P_COL_STEP + i * 8,
                   smem_desc(va + ((kv * 16 * 128) >> 4), hi), idesc_o, (acc || i > 0) ? 1u : 0u, leader);
      }
    };
    uint32_t g = 0, blk = 0, vb = 0;
    int units = 0;
    int kc;
    for (int u = find_unit(0, kc); ok && u >= 0; u = find_unit(kc + 1, kc)) {
      const UnitInfo<C> w(up, u, QB, QB);
      const int nkv = w.nkv[0];
      if (!(ok = wait_all(q_full, units & 1))) break;
      // K tile jj of the unit is ring tile g + 2 jj, V tile jj is g + 2 jj + 1
      auto s_for = [&](int jj) -> bool {
        const uint32_t kg = g + 2 * jj, B = blk + jj, b = B & 1;
        if (!wait_all(kv_full + (kg % C::NSLOT), (kg / C::NSLOT) & 1)) return false;
        if constexpr (C::MX)
          if (!wait_all(sfb_ready + b, (B >> 1) & 1)) return false;
        tc_fence_after();
        issue_s(b, kg % C::NSLOT);
        commit(s_full + b);
        commit(kv_empty + (kg % C::NSLOT));
        if (jj == nkv - 1) commit(q_empty);   // the unit's last S MMAs are issued
        return true;
      };
      if (!(ok = s_for(0))) break;
      if (nkv > 1 && !(ok = s_for(1))) break;
      for (int j = 0; ok && j < nkv; ++j) {
        const uint32_t B = blk + j, bj = B & 1, ph = (B >> 1) & 1;
        const uint32_t vg = g + 2 * j + 1, vslot = vg % C::NSLOT;
        if constexpr (C::MX)
          ok = wait_all(vconv_full + (vb & 1), (vb >> 1) & 1);
        else
          ok = wait_all(kv_full + vslot, (vg / C::NSLOT) & 1);
        if (!ok) break;
#pragma unroll
        for (int c = 0; c < C::P_CHUNKS; ++c) {
          if (!(ok = wait_all(p_full + bj * C::P_CHUNKS + c, ph))) break;
          tc_fence_after();
          issue_pv_chunk(bj, C::MX ? (vb & 1) : vslot, c, j > 0 || c > 0);
        }
        if (!ok) break;
        commit(pv_done + bj);
        if constexpr (C::MX) {
          commit(vconv_empty + (vb & 1));
          ++vb;
        } else {
          commit(kv_empty + vslot);
        }
        if (j + 2 < nkv && !(ok = s_for(j + 2))) break;
      }
      g += 2 * nkv;
      blk += nkv;
      ++units;
    }
    if (!ok && lane == 0) record_timeout();
    // every MMA this warp issued completes before TMEM can be released
    commit(drain_bar);
    drain_wait(drain_bar, 0, p.timeout_cycles);
    __syncwarp();
  } else if (warp > C::MMA_WARP && (C::SPLIT == 1 || warp < C::SOFTMAX_WARP1)) {
    if constexpr (C::MX) {
      regs_decrease<C::REGS_OTHER>();
    }
    if (C::MX && warp <= C::MMA_WARP + C::CONV_WARPS) {
      // ======================= MXFP8 V -> f16 with its block scales =======================
      // Thread ct (0 .. 32 CONV_WARPS - 1) handles (key row, 16-code unit) pairs
      // ct, ct + 32 CONV_WARPS, ...: key rows ct / 8 + (4 CONV_WARPS) i, unit
      // un = ct % 8 (d = 16 un .. 16 un + 15, block un / 2).
      constexpr int ITERS = C::CONV_ITERS;
      constexpr int ROW_STEP = 4 * C::CONV_WARPS;
      const int ct = (warp - C::MMA_WARP - 1) * 32 + lane;
      const int un = ct & 7, blk_d = un >> 1;
      uint32_t g = 0, vb = 0, cu = 0;
      int kc;
      for (int u = find_unit(0, kc); ok && u >= 0; u = find_unit(kc + 1, kc)) {
        const UnitInfo<C> w(up, u, QB, QB);
        const int nkv = w.nkv[0];
        const size_t head_row0 = static_cast<size_t>(w.bh) * p.N;
        const int kend = min(nkv * kBlockN, p.N);
        // scale bytes of this thread's 16 key rows, loaded one tile ahead (keys past
        // N: marked 0xFFFF, their codes are zero-filled and their factor is 0)
        auto load_e = [&](int jt, uint32_t (&e)[ITERS]) {
#pragma unroll
          for (int i = 0; i < ITERS; ++i) {
            const int key = jt * kBlockN + (ct >> 3) + ROW_STEP * i;
            e[i] = key < p.N && sf_row_ok(p, head_row0 + key) ? ld_nc_u8(p.v_sf + (head_row0 + key) * 4 + blk_d)
                                                              : 0xFFFFu;
          }
        };
        uint32_t e_next[ITERS];
        load_e(0, e_next);
        const uint32_t vmax = sf_row_ok(p, head_row0 + kend - 1) ? head_sf_max(p.v_sf, head_row0, kend, lane) : 0u;
        const int sv = static_cast<int>((vmax >> (8 * blk_d)) & 0xFFu);
        // the softmax scales O column block b by 2^(sv_b - 134) in the unit's
        // epilogue: the first converter warp hands the word over (slot = unit
        // index mod 4; the converters run at most two units ahead of the softmax)
        if (warp == C::MMA_WARP + 1 && lane == 0) {
          sv_word[cu & 3] = vmax;
          mbar_arrive(sv_ready + (cu & 3));
        }
        ++cu;
        for (int j = 0; j < nkv; ++j, ++vb) {
          const uint32_t vg = g + 2 * j + 1, vslot = vg % C::NSLOT, b = vb & 1;
          uint32_t e_cur[ITERS];
#pragma unroll
          for (int i = 0; i < ITERS; ++i) e_cur[i] = e_next[i];
          if (j + 1 < nkv) load_e(j + 1, e_next);
          if (!(ok = wait_all(kv_full + vslot, (vg / C::NSLOT) & 1))) break;
          if (vb >= 2 && !(ok = wait_all(vconv_empty + b, ((vb >> 1) - 1) & 1))) break;
          const uint8_t* src = smem + C::SMEM_KV + vslot * C::TILE_BYTES;
          uint8_t* dst = smem + C::SMEM_VCONV + b * C::VCONV_BYTES;
#pragma unroll
          for (int i = 0; i < ITERS; ++i) {
            const int r = (ct >> 3) + ROW_STEP * i;
            // f16 factor 2^(e - sv + 7)
            const uint32_t sb = e_cur[i] != 0xFFFFu ? f16_pow2_bits(static_cast<int>(e_cur[i]) - sv + 7) : 0u;
            const uint32_t s2u = sb * 0x10001u;
            const __half2 s2 = *reinterpret_cast<const __half2*>(&s2u);
            const uint4 c16 = *reinterpret_cast<const uint4*>(src + r * 128 + ((un ^ (r & 7)) << 4));
            const uint32_t wds[4] = {c16.x, c16.y, c16.z, c16.w};
            uint32_t hh[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t lo = f16x2_from_e4m3x2(static_cast<uint16_t>(wds[q] & 0xFFFFu));
              uint32_t hi2 = f16x2_from_e4m3x2(static_cast<uint16_t>(wds[q] >> 16));
              const __half2 a = __hmul2(*reinterpret_cast<const __half2*>(&lo), s2);
              const __half2 bb = __hmul2(*reinterpret_cast<const __half2*>(&hi2), s2);
              hh[2 * q] = *reinterpret_cast<const uint32_t*>(&a);
              hh[2 * q + 1] = *reinterpret_cast<const uint32_t*>(&bb);
            }
            // f16 d = 16 un + e sits in chunk un / 4, 16-byte unit 2 (un % 4) + e / 8
            uint8_t* drow = dst + (un >> 2) * (128 * 128) + r * 128;
            const int u0 = 2 * (un & 3);
            *reinterpret_cast<uint4*>(drow + ((u0 ^ (r & 7)) << 4)) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
            *reinterpret_cast<uint4*>(drow + (((u0 + 1) ^ (r & 7)) << 4)) = make_uint4(hh[4], hh[5], hh[6], hh[7]);
          }
          fence_proxy_async_shared();   // the MMA (async proxy) reads what these threads wrote
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(vconv_full + b);
            mbar_arrive(kv_empty + vslot);   // the E4M3 V slot is read
          }
        }
        g += 2 * nkv;
      }
      if (!ok && lane == 0) record_timeout();
    }
  } else {
    // ======================= softmax: one thread per (query row, key share) =======================
    // Warpgroup h (SPLIT of them) takes keys [NCOL h, NCOL h + NCOL) of row
    // 32 (warp % 4) + lane and writes P chunk h over its own S columns. The first
    // warpgroup (lead) also keeps the MX scale factors in TMEM, rescales O and
    // writes LSE; each warpgroup writes its share of the O columns.
    if constexpr (C::MX) regs_increase<C::REGS_SOFTMAX>();
    constexpr int NCOL = 128 / C::SPLIT;           // keys of a block per thread
    constexpr int OCOL = C::D / C::SPLIT;          // output columns per thread
    const int h = (C::SPLIT > 1 && warp >= C::SOFTMAX_WARP1) ? 1 : 0;
    const bool lead = h == 0;
    const int wq = warp & 3;                       // lane quarter of TMEM this warp may access
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t o_tm = tmem_base + lane_off + C::O_COL0;
    // (SPLIT == 2) value of this row from the other warpgroup: both warps of the
    // lane quarter write theirs, arrive, and wait with the bounded waiter; the two
    // slots alternate, so a slot is rewritten only after the partner has passed
    // the exchange that followed its read. Sets ok = false when the wait gives up.
    uint32_t xc = 0;
    auto exchange = [&](float v) -> float {
      float* xb = xbuf + (xc & 1u) * 256;
      xb[h * 128 + r] = v;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(xch + wq);
      ok = wait_all(xch + wq, xc & 1u);
      tc_fence_after();
      ++xc;
      return xb[(h ^ 1) * 128 + r];
    };
    // MX scale factors into TMEM: this warp's lane quarter gets, in column col + q,
    // the scale word of row row0 + 32 q + lane (rows past N: 0x7F bytes, scale 1).
    // The loads are issued ahead of the waits they would otherwise stall.
    auto sf_load = [&](const uint8_t* sf, size_t hrow0, int row0, uint32_t (&wv)[4]) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int rr = row0 + 32 * q + lane;
        wv[q] = rr < p.N && sf_row_ok(p, hrow0 + rr) ? ld_nc_u32(reinterpret_cast<const uint32_t*>(sf) + hrow0 + rr)
                                                      : 0x7F7F7F7Fu;
      }
    };
    auto sf_store = [&](const uint8_t* sf, size_t hrow0, int row0, uint32_t col) {
      uint32_t wv[4];
      sf_load(sf, hrow0, row0, wv);
      tmem_st4(tmem_base + lane_off + col, wv);
    };
    // the stores are complete and ordered before the MMA thread's reads
    auto sf_publish = [&](uint32_t b0, bool second) {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sfb_ready + b0);
        if (second) mbar_arrive(sfb_ready + (b0 ^ 1u));
      }
    };
    uint32_t blk = 0;
    uint32_t su = 0;   // units so far (MX: slot and phase of sv_ready)
    int kc;
    int u = find_unit(0, kc);
    if constexpr (C::MX) {
      if (u >= 0 && lead) {
        const UnitInfo<C> w(up, u, QB, QB);
        const size_t hrow0 = static_cast<size_t>(w.bh) * p.N;
        sf_store(p.q_sf, hrow0, w.qpair * kBlockM, C::SFA_COL);
        sf_store(p.k_sf, hrow0, 0, C::SFB_COL);
        if (w.nkv[0] > 1) sf_store(p.k_sf, hrow0, kBlockN, C::SFB_COL + 4);
        sf_publish(0u, w.nkv[0] > 1);
      }
    }
    while (ok && u >= 0) {
      const UnitInfo<C> w(up, u, QB, QB);
      const int nkv = w.nkv[0];
      const int row = w.qpair * kBlockM + r;
      const size_t head_row0 = static_cast<size_t>(w.bh) * p.N;
      int kn = kc;
      const int un = find_unit(kc + 1, kn);
      int nkv_next = 0, bh_next = 0, qb_next = 0;
      if (un >= 0) {
        const UnitInfo<C> wn(up, un, QB, QB);
        nkv_next = wn.nkv[0];
        bh_next = wn.bh;
        qb_next = wn.qpair;
      }
      const size_t next_row0 = static_cast<size_t>(bh_next) * p.N;
      const uint32_t L = blk + nkv - 1;   // the unit's last global block
      float m_run = __int_as_float(0xff800000u);
      float l_run = 0.f;                  // this thread's share of the row sum
      for (int j = 0; j < nkv; ++j) {
        const uint32_t B = blk + j, bj = B & 1, ph = (B >> 1) & 1;
        const uint32_t s_tm = tmem_base + lane_off + bj * 128;
        // MX: the K scale words this iteration stores (block j + 2, or the next
        // unit's block 0), loaded before the S wait so that their latency hides
        // behind it
        uint32_t wa[4];
        if constexpr (C::MX) {
          if (lead) {
            if (j + 2 < nkv)
              sf_load(p.k_sf, head_row0, (j + 2) * kBlockN, wa);
            else if (un >= 0 && (B + 1 == L || (B == L && nkv == 1)))
              sf_load(p.k_sf, next_row0, 0, wa);
          }
        }
        ok = wait_all(s_full + bj, ph);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[NCOL];
#pragma unroll
        for (int q = 0; q < NCOL / 32; ++q) tmem_ld32(s_tm + NCOL * h + 32 * q, sr + 32 * q);
        tmem_ld_wait<NCOL>(sr);
        if constexpr (C::MX) {
          // Every S MMA up to block B is complete: the K scale columns of buffer
          // bj (read by S(B)) take the scales of block B + 2; once S of the unit's
          // last block is read, the Q columns take the next unit's.
          if (lead) {
            if (j + 2 < nkv) {
              tmem_st4(tmem_base + lane_off + C::SFB_COL + 4 * bj, wa);
              sf_publish(bj, false);
            } else if (un >= 0) {
              if (B + 1 == L) tmem_st4(tmem_base + lane_off + C::SFB_COL + 4 * bj, wa);   // next unit's block 0
              if (B == L) {   // once per unit: these loads are not prefetched
                sf_store(p.q_sf, next_row0, qb_next * kBlockM, C::SFA_COL);
                if (nkv == 1) tmem_st4(tmem_base + lane_off + C::SFB_COL + 4 * (bj ^ 1u), wa);
                if (nkv_next > 1) sf_store(p.k_sf, next_row0, kBlockN, C::SFB_COL + 4 * bj);
                sf_publish(bj ^ 1u, nkv_next > 1);
              }
            }
          }
        }
        const float c = p.scale_log2;
        const bool masked = (j == nkv - 1) && (p.causal || (p.N % kBlockN) != 0);
        if (masked) {
          // last visible key of this thread's share
          const int limit = (p.causal ? min(row, p.N - 1) : p.N - 1) - j * kBlockN - NCOL * h;
#pragma unroll
          for (int i = 0; i < NCOL; ++i)
            if (i > limit) sr[i] = 0xff800000u;
        }
        float m_blk = row_max<NCOL>(sr) * c;
        if constexpr (C::SPLIT > 1) {
          const float m_other = exchange(m_blk);
          if (!ok) break;
          m_blk = fmaxf(m_blk, m_other);
        }
        float m_use = m_run;
        if (m_blk - m_run > C::RESCALE_THRESHOLD) m_use = m_blk;
        const bool moved = m_use != m_run;
        const float alpha = moved ? ex2_approx(m_run - m_use) : 1.f;
        // Both warpgroups see the same maximum, so they move together. The lead
        // rescales every column of O before it releases P chunk 0, and the MMA
        // issues chunk 0 before chunk 1: all of this block's P V follows it.
        if (lead && j > 0 && __any_sync(0xffffffffu, moved)) {
          // O holds P V up to block B - 1 once that P V has completed
          if (!(ok = wait_all(pv_done + (bj ^ 1u), ((B - 1) >> 1) & 1))) break;
          tc_fence_after();
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
        uint64_t* pf = p_full + bj * C::P_CHUNKS;
        float sum;
        if constexpr (C::SPLIT == 1) {
          sum = masked ? p_row_to_tmem<C, 0u>(sr, c, m_use, s_tm, pf)
                       : p_row_to_tmem<C, C::POLY_MASK>(sr, c, m_use, s_tm, pf);
        } else {
          sum = p_share_to_tmem<C>(sr, c, m_use, s_tm + C::P_COL_STEP * h, pf + h);
        }
        l_run = l_run * alpha + sum;
        m_run = m_use;
      }
      if (!ok) break;
      // ---- epilogue: the unit's last P V complete, then O / l and LSE. The next
      // unit's first P V (which overwrites O) waits for the lead's P, which comes
      // after its own TMEM loads and (through the first exchange of the next
      // unit) after the other warpgroup's.
      if (!(ok = wait_all(pv_done + (L & 1), (L >> 1) & 1))) break;
      tc_fence_after();
      float l_row = l_run;
      if constexpr (C::SPLIT > 1) {
        const float l_other = exchange(l_run);
        if (!ok) break;
        l_row += l_other;
      }
      const float inv_l = 1.f / l_row;
      float f_blk[4] = {inv_l, inv_l, inv_l, inv_l};
      if constexpr (C::MX) {
        // sv_b, the maximum V scale byte of column block b over the unit's key
        // rows, as the converter warps reduced it for the V widening
        if (!(ok = wait_all(sv_ready + (su & 3), (su >> 2) & 1))) break;
        const uint32_t v_sfmax = sv_word[su & 3];
#pragma unroll
        for (int b = 0; b < 4; ++b) f_blk[b] = inv_l * f32_pow2(static_cast<int>((v_sfmax >> (8 * b)) & 0xFFu) - 134);
      }
      ++su;
      const size_t grow = head_row0 + row;   // row over all heads
      const bool in_range = row < p.N && dbg_ok(grow < p.out_rows, kSiteFwd1Out, grow);
      __nv_bfloat16* orow = p.o + (in_range ? grow : 0) * C::D + OCOL * h;
#pragma unroll
      for (int cb = 0; cb < OCOL; cb += 32) {
        const float f = f_blk[((OCOL * h + cb) / 32) & 3];
        uint32_t ov[32];
        tmem_ld32(o_tm + OCOL * h + cb, ov);
        tmem_ld_wait<32>(ov);
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * f, __uint_as_float(ov[2 * i + 1]) * f);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cb);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
      if (lead && p.lse != nullptr && in_range) p.lse[grow] = (m_run + __log2f(l_row)) * 0.69314718055994531f;
      blk += nkv;
      u = un;
      kc = kn;
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
