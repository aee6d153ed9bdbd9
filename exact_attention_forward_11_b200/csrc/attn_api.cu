// attn_api.cu - host side of the C ABI declared in include/attn_b200.h.
//
// Validates arguments (before anything touches the GPU), encodes TMA tensor maps
// for the [B*H, N, d] operands, and launches the kernels on the caller's stream.
// Nothing is allocated per call; the library owns one device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn_b200.h"
#include "attn_b200_testing.h"
#include "w4a16_b200.h"
#include "attn_bwd_kernel.cuh"
#include "attn_fwd1_kernel.cuh"
#include "attn_fwd_kernel.cuh"
#include "fp8_prep_kernel.cuh"
#include "mxfp8_quant_kernel.cuh"
#include "w4a16_kernel.cuh"

// Scratch of attn_bwd_noalloc (D_i, 4 bytes per row) for at most
// ATTN_BWD_NOALLOC_MAX_ROWS rows: an 8 MiB array that every GPU which loads this
// library holds until the process exits. In host code its name is only a
// stand-in: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) float g_bwd_noalloc_scratch[ATTN_BWD_NOALLOC_MAX_ROWS];

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Each pipeline wait gives up after 2^31 SM cycles: about 1.1 s at the 1965 MHz
// maximum clock, longer at lower clocks.
constexpr uint64_t kWaitLimitCycles = 1ull << 31;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Encoded maps are kept in a small cache keyed by everything the encoding
// depends on (a map is a pure function of base address, type and shape), so a
// caller that repeats a call on the same buffers skips the host-side encoding.
struct MapKey {
  const void* base;
  int fp8, d, N, BH, rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && fp8 == o.fp8 && d == o.d && N == o.N && BH == o.BH && rows == o.rows;
  }
};
constexpr int kMapCacheSize = 32;
struct MapCache {
  std::mutex mu;
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  int used = 0, next = 0;
};
MapCache& map_cache() {
  static MapCache c;
  return c;
}

bool encode_qkv_map_uncached(CUtensorMap* map, const void* base, bool fp8, int d, int N, int BH, int rows);

// 3-D map over a contiguous [BH, N, d] tensor: dims {d, N, BH}, box {128 bytes of
// d, `rows` rows, 1}, 128-byte swizzle (the layout the MMA descriptors expect).
// Rows past N read as zero.
bool encode_qkv_map(CUtensorMap* map, const void* base, bool fp8, int d, int N, int BH, int rows) {
  const MapKey k{base, fp8 ? 1 : 0, d, N, BH, rows};
  MapCache& c = map_cache();
  {
    std::lock_guard<std::mutex> lock(c.mu);
    for (int i = 0; i < c.used; ++i)
      if (c.key[i] == k) {
        *map = c.map[i];
        return true;
      }
  }
  if (!encode_qkv_map_uncached(map, base, fp8, d, N, BH, rows)) return false;
  std::lock_guard<std::mutex> lock(c.mu);
  const int slot = c.used < kMapCacheSize ? c.used++ : (c.next++ % kMapCacheSize);
  c.key[slot] = k;
  c.map[slot] = *map;
  return true;
}

bool encode_qkv_map_uncached(CUtensorMap* map, const void* base, bool fp8, int d, int N, int BH, int rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  const int elem = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem, static_cast<cuuint64_t>(N) * d * elem};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Map over a row-major matrix [outer, inner] viewed as {inner, outer, 1}, box
// {box_inner, box_outer, 1}: elements past the matrix read as zero.
bool encode_matrix_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem, long long inner,
                       long long outer, int box_inner, int box_outer, bool swizzle128) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer), 1};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * elem, static_cast<cuuint64_t>(inner) * elem * outer};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Number of SMs of the current device (cached per device ordinal).
int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < 64) cache[dev] = n;
  return n;
}

// Raises a kernel's dynamic shared-memory limit once per device (the attribute
// belongs to the function on the current device; later calls skip the driver
// call). `tag` identifies the kernel. A failed launch forgets the flag, so a
// context that was reset gets the attribute again on the next call.
std::atomic<uint32_t> g_smem_done[64][16];

void forget_smem(int tag) {
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 && tag < 16)
    g_smem_done[dev][tag].store(0u, std::memory_order_release);
}

bool set_smem_once(const void* func, int bytes, int tag) {
  auto& done = g_smem_done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  if (dev < 64 && tag < 16 && done[dev][tag].load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (dev < 64 && tag < 16) done[dev][tag].store(1u, std::memory_order_release);
  return true;
}

template <int D, bool FP8>
constexpr int fwd_tag() { return FP8 ? 2 : (D == 128 ? 0 : 1); }

// scale == 0 selects 1/sqrt(d); negative or non-finite scales are rejected
// (the kernels take the row maximum of scale * Q K^T through the maximum of
// Q K^T, which only holds for a positive scale).
attn_status resolve_scale(float& scale, int d) {
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (scale == 0.f) scale = 1.0f / std::sqrt(static_cast<float>(d));
  return ATTN_OK;
}

attn_status check_shape(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// Non-causal: heads per group such that the group's K and V (2 N d elements per
// head) take about 48 MB of the 126 MB L2. Causal: all heads unless
// ATTN_CAUSAL_GROUP_MB gives a budget for causal groups too.
#ifndef ATTN_CAUSAL_GROUP_MB
#define ATTN_CAUSAL_GROUP_MB 0
#endif
int heads_per_group(int BH, int N, int D, int elem, int causal) {
  const long long kv_bytes = 2ll * N * D * elem;
  const long long budget = causal ? (static_cast<long long>(ATTN_CAUSAL_GROUP_MB) << 20) : (48ll << 20);
  long long hg = budget == 0 ? BH : budget / (kv_bytes > 0 ? kv_bytes : 1);
  if (hg < 1) hg = 1;
  if (hg > BH) hg = BH;
  return static_cast<int>(hg);
}

template <int D, bool FP8>
attn_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const float* qs,
                       const float* ks, const float* vs, int BH, int N, float scale, int causal,
                       cudaStream_t stream, int fault_unit = -1, uint64_t wait_limit = kWaitLimitCycles,
                       long long out_rows = -1) {
  using C = attn::FwdCfg<D, FP8>;
  auto kern = attn::attn_fwd_sm100<C>;
  CUtensorMap tq, tk, tv;
  if (!encode_qkv_map(&tq, q, FP8, D, N, BH, attn::kBlockM) ||
      !encode_qkv_map(&tk, k, FP8, D, N, BH, attn::kBlockN) || !encode_qkv_map(&tv, v, FP8, D, N, BH, attn::kBlockN))
    return ATTN_ERR_CUDA;
  if (!set_smem_once(reinterpret_cast<const void*>(kern), C::SMEM_BYTES, fwd_tag<D, FP8>())) return ATTN_ERR_CUDA;
  const int QB = (N + attn::kBlockM - 1) / attn::kBlockM;
  const int npair = (QB + C::Q_TILES - 1) / C::Q_TILES;
  attn::FwdParams p;
  p.N = N;
  p.BH = BH;
  p.num_units = BH * npair;
  p.heads_per_group = heads_per_group(BH, N, C::D, C::FP8 ? 1 : 2, causal);
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.q_scale = qs;
  p.k_scale = ks;
  p.v_scale = vs;
  p.timeout_cycles = wait_limit;
  p.fault_unit = fault_unit;
  p.out_rows = static_cast<uint32_t>(out_rows < 0 ? static_cast<long long>(BH) * N : out_rows);
  // persistent grid: one CTA per SM (shared memory and TMEM allow one), each
  // walking the units blockIdx.x, blockIdx.x + gridDim.x, ...
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const int grid = p.num_units < sms ? p.num_units : sms;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) {
    forget_smem(fwd_tag<D, FP8>());
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// The one-Q-tile forward (attn_fwd1_kernel.cuh): BF16 (MX = false) or MXFP8
// codes with their scale-byte arrays (MX = true).
template <int D, bool MX>
attn_status launch_fwd1(const void* q, const void* k, const void* v, void* o, float* lse, const void* q_sf,
                        const void* k_sf, const void* v_sf, int BH, int N, float scale, int causal,
                        cudaStream_t stream, int fault_unit = -1, uint64_t wait_limit = kWaitLimitCycles,
                        long long out_rows = -1) {
  using C = attn::Fwd1Cfg<D, MX>;
  auto kern = attn::attn_fwd1_sm100<C>;
  const int tag = MX ? 12 : (D == 128 ? 10 : 11);
  CUtensorMap tq, tk, tv;
  if (!encode_qkv_map(&tq, q, MX, D, N, BH, attn::kBlockM) || !encode_qkv_map(&tk, k, MX, D, N, BH, attn::kBlockN) ||
      !encode_qkv_map(&tv, v, MX, D, N, BH, attn::kBlockN))
    return ATTN_ERR_CUDA;
  if (!set_smem_once(reinterpret_cast<const void*>(kern), C::SMEM_BYTES, tag)) return ATTN_ERR_CUDA;
  attn::Fwd1Params p;
  p.N = N;
  p.BH = BH;
  p.num_units = BH * ((N + attn::kBlockM - 1) / attn::kBlockM);
  p.heads_per_group = heads_per_group(BH, N, D, MX ? 1 : 2, causal);
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.q_sf = static_cast<const uint8_t*>(q_sf);
  p.k_sf = static_cast<const uint8_t*>(k_sf);
  p.v_sf = static_cast<const uint8_t*>(v_sf);
  p.timeout_cycles = wait_limit;
  p.fault_unit = fault_unit;
  p.out_rows = static_cast<uint32_t>(out_rows < 0 ? static_cast<long long>(BH) * N : out_rows);
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const int grid = p.num_units < sms ? p.num_units : sms;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) {
    forget_smem(tag);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

template <int D>
attn_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, float* dd, int BH, int N, float scale,
                       int causal, cudaStream_t stream) {
  using C = attn::BwdCfg<D>;
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_qkv_map(&tq, q, false, D, N, BH, 128) || !encode_qkv_map(&tk, k, false, D, N, BH, 128) ||
      !encode_qkv_map(&tv, v, false, D, N, BH, 128) || !encode_qkv_map(&tdo, dout, false, D, N, BH, 128))
    return ATTN_ERR_CUDA;
  auto kdkdv = attn::attn_bwd_dkdv<C>;
  auto kdq = attn::attn_bwd_dq<C>;
  const int tag = D == 128 ? 5 : 6;
  if (!set_smem_once(reinterpret_cast<const void*>(kdkdv), C::DKDV_SMEM, tag) ||
      !set_smem_once(reinterpret_cast<const void*>(kdq), C::DQ_SMEM, tag + 2))
    return ATTN_ERR_CUDA;
  // D_i = dO_i . O_i (D/8 lanes per row)
  const long long rows = static_cast<long long>(BH) * N;
  const long long threads = rows * (D / 8);
  attn::attn_bwd_rowdot<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), dd, rows);
  attn::BwdParams p;
  p.N = N;
  p.BH = BH;
  p.causal = causal;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lse = lse;
  p.dd = dd;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.timeout_cycles = kWaitLimitCycles;
  const int QB = (N + 127) / 128;
  kdkdv<<<QB * BH, C::THREADS, C::DKDV_SMEM, stream>>>(tq, tk, tv, tdo, p);
  kdq<<<QB * BH, C::THREADS, C::DQ_SMEM, stream>>>(tq, tk, tv, tdo, p);
  if (cudaGetLastError() != cudaSuccess) {
    forget_smem(tag);
    forget_smem(tag + 2);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// Bytes of workspace attn_bwd needs: D_i for every row, fp32, rounded to 256.
size_t bwd_workspace_bytes(long long BH, long long N) { return static_cast<size_t>((BH * N * 4 + 255) / 256 * 256); }

// ---- attn_bwd_noalloc: the backward with its scratch in a fixed device array
// Device address of g_bwd_noalloc_scratch on the current device. The name is a
// host-side stand-in in host code, so the address is asked of the runtime once
// per device (with that device current) and cached; nullptr if that fails.
float* noalloc_scratch_on_current_device() {
  static std::atomic<float*> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  float* ptr = cache[dev].load(std::memory_order_acquire);
  if (ptr != nullptr) return ptr;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_bwd_noalloc_scratch) != cudaSuccess || addr == nullptr) return nullptr;
  ptr = static_cast<float*>(addr);
  cache[dev].store(ptr, std::memory_order_release);
  return ptr;
}

}  // namespace

extern "C" {

int attn_abi_version(void) { return 1; }

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_MISALIGNED: return "ATTN_ERR_MISALIGNED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_BOUNDS: return "ATTN_ERR_BOUNDS";
    default: return "ATTN_UNKNOWN_STATUS";
  }
}

}  // extern "C"

namespace {

// attn_fwd with the rows of O / LSE the kernels may write (-1: all B*H*N;
// fewer only through the debug-build hook).
attn_status fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                     float scale, int causal, attn_dtype dtype, void* stream, long long out_rows) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = resolve_scale(scale, d); s != ATTN_OK) return s;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
#ifndef ATTN_FWD_ONE_TILE
#define ATTN_FWD_ONE_TILE 0
#endif
  // Launches with fewer two-Q-tile units than SMs (a few short heads, e.g. one
  // ViT image) leave most SMs idle under the two-tile schedule: the one-tile
  // kernel gives them twice the CTAs, each with half the chain (measured on the
  // 12-head, N = 196 case: 9.3 against 11.1 us). Everything larger runs two-tile.
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const long long pair_units = static_cast<long long>(BH) * ((N + 2 * attn::kBlockM - 1) / (2 * attn::kBlockM));
  const uint64_t wl = kWaitLimitCycles;
  if (ATTN_FWD_ONE_TILE || pair_units < sms) {
    if (d == 128)
      return launch_fwd1<128, false>(q, k, v, o, lse, nullptr, nullptr, nullptr, BH, N, scale, causal, st, -1, wl,
                                     out_rows);
    return launch_fwd1<64, false>(q, k, v, o, lse, nullptr, nullptr, nullptr, BH, N, scale, causal, st, -1, wl,
                                  out_rows);
  }
  if (d == 128)
    return launch_fwd<128, false>(q, k, v, o, lse, nullptr, nullptr, nullptr, BH, N, scale, causal, st, -1, wl,
                                  out_rows);
  return launch_fwd<64, false>(q, k, v, o, lse, nullptr, nullptr, nullptr, BH, N, scale, causal, st, -1, wl,
                               out_rows);
}

}  // namespace

extern "C" {

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                     float scale, int causal, attn_dtype dtype, void* stream) {
  return fwd_bf16(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, stream, -1);
}

attn_status attn_fwd_debug_row_limit(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                     int N, int d, float scale, int causal, long long row_limit, void* stream) {
  if (!attn::kDebugChecks) return ATTN_ERR_UNSUPPORTED;
  if (B < 1 || H < 1 || N < 1 || row_limit < 0 || row_limit > static_cast<long long>(B) * H * N)
    return ATTN_ERR_INVALID_ARG;
  return fwd_bf16(q, k, v, o, lse, B, H, N, d, scale, causal, ATTN_BF16, stream, row_limit);
}

int attn_debug_build(void) { return attn::kDebugChecks ? 1 : 0; }

attn_status attn_debug_last_failure(int* site, long long* index, void* stream) {
  if (site == nullptr || index == nullptr) return ATTN_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  uint32_t s = 0;
  unsigned long long i = 0;
  if (cudaMemcpyFromSymbol(&s, attn::g_debug_site, sizeof(s)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&i, attn::g_debug_index, sizeof(i)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  *site = static_cast<int>(s);
  *index = static_cast<long long>(i);
  const uint32_t zs = 0;
  const unsigned long long zi = 0;
  if (cudaMemcpyToSymbol(attn::g_debug_site, &zs, sizeof(zs)) != cudaSuccess ||
      cudaMemcpyToSymbol(attn::g_debug_index, &zi, sizeof(zi)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

attn_status attn_fwd_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                    int N, int d, float scale, int causal, int fault_unit,
                                    unsigned long long wait_limit_cycles, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = resolve_scale(scale, d); s != ATTN_OK) return s;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (fault_unit < 0 || wait_limit_cycles < 1024) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  return launch_fwd<128, false>(q, k, v, o, lse, nullptr, nullptr, nullptr, B * H, N, scale, causal,
                                static_cast<cudaStream_t>(stream), fault_unit, wait_limit_cycles);
}

attn_status attn_fwd_one_tile_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse,
                                             int B, int H, int N, int d, float scale, int causal, int fault_unit,
                                             unsigned long long wait_limit_cycles, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = resolve_scale(scale, d); s != ATTN_OK) return s;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (fault_unit < 0 || wait_limit_cycles < 1024) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  return launch_fwd1<128, false>(q, k, v, o, lse, nullptr, nullptr, nullptr, B * H, N, scale, causal,
                                 static_cast<cudaStream_t>(stream), fault_unit, wait_limit_cycles);
}

attn_status attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
                         const float* v_scale, void* o, float* lse, int B, int H, int N, int d, float scale,
                         int causal, void* stream) {
  if (q8 == nullptr || k8 == nullptr || v8 == nullptr || o == nullptr || q_scale == nullptr ||
      k_scale == nullptr || v_scale == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = resolve_scale(scale, d); s != ATTN_OK) return s;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  return launch_fwd<128, true>(q8, k8, v8, o, lse, q_scale, k_scale, v_scale, B * H, N, scale, causal,
                               static_cast<cudaStream_t>(stream));
}

attn_status attn_quantize_mxfp8(const void* x, void* codes, void* sf, int B, int H, int N, int d, void* stream) {
  if (x == nullptr || codes == nullptr || sf == nullptr) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d < 32 || d % 32 != 0 || d > 4096) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf)) return ATTN_ERR_MISALIGNED;
  const long long nblk = static_cast<long long>(B) * H * N * (d / 32);
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  // 2048 threads per SM (8 CTAs of 256), fewer for small tensors: four lanes per block
  const long long need = (nblk * 4 + attn::kMxQuantThreads - 1) / attn::kMxQuantThreads;
  const long long cap = 8ll * sms;
  const int grid = static_cast<int>(need < cap ? need : cap);
  attn::mxfp8_quantize_sm100<<<grid, attn::kMxQuantThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(codes), static_cast<uint8_t*>(sf), nblk);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

}  // extern "C"

namespace {

// attn_fwd_mxfp8's argument checks and launch; fault_unit / wait_limit are the
// testing hook's (-1 / the normal limit otherwise).
attn_status fwd_mxfp8(const void* q8, const void* k8, const void* v8, const void* q_sf, const void* k_sf,
                      const void* v_sf, void* o, float* lse, int B, int H, int N, int d, float scale, int causal,
                      void* stream, int fault_unit, uint64_t wait_limit) {
  if (q8 == nullptr || k8 == nullptr || v8 == nullptr || o == nullptr || q_sf == nullptr || k_sf == nullptr ||
      v_sf == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = resolve_scale(scale, d); s != ATTN_OK) return s;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(q_sf) || !aligned16(k_sf) ||
      !aligned16(v_sf) || !aligned16(o) || (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  return launch_fwd1<128, true>(q8, k8, v8, o, lse, q_sf, k_sf, v_sf, B * H, N, scale, causal,
                                static_cast<cudaStream_t>(stream), fault_unit, wait_limit);
}

}  // namespace

extern "C" {

attn_status attn_fwd_mxfp8(const void* q8, const void* k8, const void* v8, const void* q_sf, const void* k_sf,
                           const void* v_sf, void* o, float* lse, int B, int H, int N, int d, float scale,
                           int causal, void* stream) {
  return fwd_mxfp8(q8, k8, v8, q_sf, k_sf, v_sf, o, lse, B, H, N, d, scale, causal, stream, -1, kWaitLimitCycles);
}

attn_status attn_fwd_mxfp8_inject_timeout(const void* q8, const void* k8, const void* v8, const void* q_sf,
                                          const void* k_sf, const void* v_sf, void* o, float* lse, int B, int H,
                                          int N, int d, float scale, int causal, int fault_unit,
                                          unsigned long long wait_limit_cycles, void* stream) {
  if (fault_unit < 0 || wait_limit_cycles < 1024) return ATTN_ERR_INVALID_ARG;
  return fwd_mxfp8(q8, k8, v8, q_sf, k_sf, v_sf, o, lse, B, H, N, d, scale, causal, stream, fault_unit,
                   wait_limit_cycles);
}

attn_status attn_quantize_fp8(const void* x, const void* rot, void* x8, float* scales, int B, int H, int N, int d,
                              void* stream) {
  if (x == nullptr || x8 == nullptr || scales == nullptr) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d != attn::kPrepTile) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x8) || (rot != nullptr && !aligned16(rot))) return ATTN_ERR_MISALIGNED;
  const int BH = B * H;
  const int T = (N + attn::kPrepTile - 1) / attn::kPrepTile;
  // X tiles {128 rows of bf16 in two 64-column chunks}, R as one such tile, the
  // codes as {128 rows x 128 bytes}; all with the 128-byte swizzle
  CUtensorMap tx, tr, to;
  if (!encode_qkv_map(&tx, x, false, d, N, BH, attn::kPrepTile) ||
      !encode_qkv_map(&to, x8, true, d, N, BH, attn::kPrepTile) ||
      !encode_qkv_map(&tr, rot != nullptr ? rot : x, false, d, rot != nullptr ? d : N, rot != nullptr ? 1 : BH,
                      attn::kPrepTile))
    return ATTN_ERR_CUDA;
  const bool rotate = rot != nullptr;
  const void* kern = rotate ? reinterpret_cast<const void*>(attn::fp8_prep_sm100<true>)
                            : reinterpret_cast<const void*>(attn::fp8_prep_sm100<false>);
  const int tag = rotate ? 3 : 4;
  if (!set_smem_once(kern, attn::PrepCfg::SMEM_BYTES, tag)) return ATTN_ERR_CUDA;
  const int num_tiles = BH * T;
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const int grid = num_tiles < sms ? num_tiles : sms;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (rotate)
    attn::fp8_prep_sm100<true><<<grid, attn::PrepCfg::THREADS, attn::PrepCfg::SMEM_BYTES, st>>>(
        tx, tr, to, scales, T, num_tiles, kWaitLimitCycles);
  else
    attn::fp8_prep_sm100<false><<<grid, attn::PrepCfg::THREADS, attn::PrepCfg::SMEM_BYTES, st>>>(
        tx, tr, to, scales, T, num_tiles, kWaitLimitCycles);
  if (cudaGetLastError() != cudaSuccess) {
    forget_smem(tag);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

size_t attn_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  return bwd_workspace_bytes(static_cast<long long>(B) * H, N);
}

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N,
                     int d, float scale, int causal, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr || dout == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr || workspace == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = resolve_scale(scale, d); s != ATTN_OK) return s;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (workspace_bytes < bwd_workspace_bytes(static_cast<long long>(B) * H, N)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return ATTN_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* dd = static_cast<float*>(workspace);
  if (d == 128) return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, dd, B * H, N, scale, causal, st);
  return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, dd, B * H, N, scale, causal, st);
}

namespace {

constexpr int kW4MaxCtas = 296;      // two per SM of a B200: the most a split-K launch uses
constexpr int kW4MinSlices = 8;      // a split-K run covers at least this many 128-deep slices

// Split-K CTA cap for U units, before the device's SM count is applied.
int w4_cta_cap(long long units) {
  const long long c = units / kW4MinSlices;
  return static_cast<int>(c < 1 ? 1 : (c > kW4MaxCtas ? kW4MaxCtas : c));
}

size_t w4_tickets_bytes(int N) { return static_cast<size_t>((16ll * (N / 128) + 255) / 256 * 256); }

attn_status w4_check(const void* x, const void* qweight, const void* scales, const void* zeros, const void* y, int M,
                     int N, int K) {
  using C = attn::W4Cfg;
  if (x == nullptr || qweight == nullptr || scales == nullptr || zeros == nullptr || y == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1) return ATTN_ERR_INVALID_ARG;
  if (M > C::MAX_M || N % C::BN != 0 || K % C::GROUP != 0) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(y))
    return ATTN_ERR_MISALIGNED;
  if (static_cast<long long>(K) * N >= (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// One launch of w4a16_gemm_sm100 over `ctas` CTAs (ctas = N / 128: a tile each).
attn_status launch_w4(const void* x, const void* qweight, const void* scales, const void* zeros, void* y, void* ws,
                      int M, int N, int K, int ctas, cudaStream_t stream) {
  using C = attn::W4Cfg;
  const int mpad = (M + 15) / 16 * 16;
  CUtensorMap tx, tw, ts, tz;
  if (!encode_matrix_map(&tx, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K, M, 64, mpad, true) ||
      !encode_matrix_map(&tw, qweight, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, N, K / 8, C::BN, 16, false) ||
      !encode_matrix_map(&ts, scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, K / C::GROUP, C::BN, 1, false) ||
      !encode_matrix_map(&tz, zeros, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / C::GROUP, C::BN, 1, false))
    return ATTN_ERR_CUDA;
  const int smem = C::smem_bytes(mpad);
  if (!set_smem_once(reinterpret_cast<const void*>(attn::w4a16_gemm_sm100), C::max_smem_bytes(), 9))
    return ATTN_ERR_CUDA;
  attn::W4Params p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.mpad = mpad;
  p.ctas = ctas;
  p.units = static_cast<long long>(N / C::BN) * (K / C::GROUP);
  p.y = static_cast<__half*>(y);
  p.tickets = ws == nullptr ? nullptr : static_cast<uint32_t*>(ws);
  p.part = ws == nullptr ? nullptr
                         : reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w4_tickets_bytes(N));
  p.timeout_cycles = kWaitLimitCycles;
  attn::w4a16_gemm_sm100<<<ctas, C::THREADS, smem, stream>>>(tx, tw, ts, tz, p);
  if (cudaGetLastError() != cudaSuccess) {
    forget_smem(9);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace

attn_status w4a16_gemm(const void* x, const void* qweight, const void* scales, const void* zeros, void* y, int M,
                       int N, int K, void* stream) {
  if (attn_status s = w4_check(x, qweight, scales, zeros, y, M, N, K); s != ATTN_OK) return s;
  return launch_w4(x, qweight, scales, zeros, y, nullptr, M, N, K, N / attn::W4Cfg::BN,
                   static_cast<cudaStream_t>(stream));
}

size_t w4a16_gemm_splitk_workspace_bytes(int M, int N, int K) {
  using C = attn::W4Cfg;
  if (M < 1 || N < 1 || K < 1 || M > C::MAX_M || N % C::BN != 0 || K % C::GROUP != 0) return 0;
  if (static_cast<long long>(K) * N >= (1ll << 40)) return 0;
  const long long mpad = (M + 15) / 16 * 16;
  const int cap = w4_cta_cap(static_cast<long long>(N / C::BN) * (K / C::GROUP));
  return w4_tickets_bytes(N) + static_cast<size_t>(2ll * cap * mpad * C::BN * 4);
}

attn_status w4a16_gemm_splitk(const void* x, const void* qweight, const void* scales, const void* zeros, void* y,
                              void* workspace, size_t workspace_bytes, int M, int N, int K, void* stream) {
  using C = attn::W4Cfg;
  if (attn_status s = w4_check(x, qweight, scales, zeros, y, M, N, K); s != ATTN_OK) return s;
  if (workspace == nullptr || workspace_bytes < w4a16_gemm_splitk_workspace_bytes(M, N, K))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const long long units = static_cast<long long>(N / C::BN) * (K / C::GROUP);
  const int cap = w4_cta_cap(units);
  const int ctas = 2 * sms < cap ? 2 * sms : cap;
  return launch_w4(x, qweight, scales, zeros, y, workspace, M, N, K, ctas, static_cast<cudaStream_t>(stream));
}

attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                             float scale, int causal, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr || dout == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (attn_status s = resolve_scale(scale, d); s != ATTN_OK) return s;
  if (attn_status s = check_shape(B, H, N); s != ATTN_OK) return s;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N > ATTN_BWD_NOALLOC_MAX_ROWS) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return ATTN_ERR_MISALIGNED;
  float* dd = noalloc_scratch_on_current_device();
  if (dd == nullptr) return ATTN_ERR_CUDA;
  // every row of D that the kernels read is written by the first launch of
  // this call: nothing in the array has to start at zero
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128) return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, dd, B * H, N, scale, causal, st);
  return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, dd, B * H, N, scale, causal, st);
}

attn_status attn_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, attn::g_status, sizeof(v)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (v == 0) return ATTN_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(attn::g_status, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  return (v & attn::kStatusBounds) ? ATTN_ERR_BOUNDS : ATTN_ERR_TIMEOUT;
}

}  // extern "C"
