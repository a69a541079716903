// libi8q: the C ABI declared in include/i8q.h.  Host-side argument checks, launch
// configuration, TMA tensor-map encoding; all arithmetic of the method runs in the kernels
// included below.  Built as a single translation unit so that the device error word is one
// symbol per device.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <climits>
#include <mutex>

#include "../../include/i8q.h"
#include "common.cuh"
#include "gemm_w8a16.cuh"
#include "gemm_w8a8.cuh"
#include "gemm_w8a8_small.cuh"
#include "quant.cuh"

namespace i8q {

// ------------------------------------------------------------------ error text --------------
static thread_local char t_last_error[256] = "";

static i8q_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
  return I8Q_ERR_CUDA;
}

#define I8Q_CUDA(call)                                   \
  do {                                                   \
    cudaError_t e_ = (call);                             \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);  \
  } while (0)

#define I8Q_LAUNCHED(what)                                    \
  do {                                                        \
    cudaError_t e_ = cudaGetLastError();                      \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);        \
  } while (0)

// ------------------------------------------------------------------ device info -------------
struct DeviceInfo {
  int ok = -1;   // -1 unknown, 0 unsupported, 1 supported
  int sms = 0;
};
static constexpr int kMaxDevices = 64;
static DeviceInfo g_dev[kMaxDevices];
static std::mutex g_dev_mu;

static i8q_status current_device(int* sms) {
  int dev = 0;
  I8Q_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return I8Q_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.ok < 0) {
    int major = 0, minor = 0, n = 0;
    I8Q_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    I8Q_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    I8Q_CUDA(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev));
    d.ok = (major == 10 && minor == 0) ? 1 : 0;
    d.sms = n;
    if (!d.ok)
      snprintf(t_last_error, sizeof(t_last_error), "device %d is sm_%d%d; libi8q is built for sm_100a", dev, major,
               minor);
  }
  if (!d.ok) return I8Q_ERR_UNSUPPORTED;
  *sms = d.sms;
  return I8Q_OK;
}

// ------------------------------------------------------------------ TMA tensor maps ---------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

// 2-D row-major tensor [rows][cols] of `elem` bytes, box = box_rows x box_cols, given swizzle.
// Encoded maps are cached: a map is a pure function of these arguments, so a cache hit is valid
// even when the memory behind `base` was freed and reallocated in between.
struct TmapKey {
  const void* base;
  uint64_t rows, cols, ld;
  uint32_t box_rows, box_cols;
  int dtype, elem, swz;
  bool operator==(const TmapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && ld == o.ld && box_rows == o.box_rows &&
           box_cols == o.box_cols && dtype == o.dtype && elem == o.elem && swz == o.swz;
  }
};
struct TmapEntry {
  TmapKey key;
  CUtensorMap map;
  bool valid = false;
};
static constexpr int kTmapCache = 256;
static TmapEntry g_tmap_cache[kTmapCache];
static std::mutex g_tmap_mu;

static i8q_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem,
                               uint64_t rows, uint64_t cols, uint64_t ld_elems, uint32_t box_rows,
                               uint32_t box_cols, CUtensorMapSwizzle swz) {
  const TmapKey key{base, rows, cols, ld_elems, box_rows, box_cols, (int)dtype, elem, (int)swz};
  const size_t h = (reinterpret_cast<uintptr_t>(base) >> 8) ^ (rows * 131) ^ (cols * 7919) ^ (box_rows * 31) ^ box_cols;
  TmapEntry& e = g_tmap_cache[h % kTmapCache];
  {
    std::lock_guard<std::mutex> lk(g_tmap_mu);
    if (e.valid && e.key == key) {
      *map = e.map;
      return I8Q_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled is unavailable");
    return I8Q_ERR_CUDA;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld_elems * (uint64_t)elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return I8Q_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_tmap_mu);
  e.key = key;
  e.map = *map;
  e.valid = true;
  return I8Q_OK;
}

// ------------------------------------------------------------------ argument checks ---------
static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define I8Q_REQUIRE(cond, code)  \
  do {                           \
    if (!(cond)) return (code);  \
  } while (0)

static inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Dynamic shared memory above 48 KB must be opted into per kernel, and the attribute belongs to
// the current device: it is set once per (kernel, device).
static std::mutex g_smem_mu;
static const void* g_smem_kern[256];
static int g_smem_dev[256];
static int g_smem_n = 0;

template <typename Kern>
static i8q_status ensure_smem(Kern k, int bytes) {
  int dev = 0;
  I8Q_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_smem_mu);
  for (int i = 0; i < g_smem_n; ++i)
    if (g_smem_kern[i] == (const void*)k && g_smem_dev[i] == dev) return I8Q_OK;
  I8Q_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (g_smem_n < 256) {
    g_smem_kern[g_smem_n] = (const void*)k;
    g_smem_dev[g_smem_n] = dev;
    ++g_smem_n;
  }
  return I8Q_OK;
}

static constexpr int64_t kMaxDim = (int64_t)1 << 30;
static constexpr int64_t kFusedQuantMaxM = 16;   // decode batches (see i8q_gemm_w8a8_block_fused_quant)

// Resident CTAs per SM of a kernel at a block size (queried once per kernel and block size).
template <typename Kern>
static int64_t resident_grid(Kern k, int threads, int sms) {
  static std::mutex mu;
  static const void* keys[64];
  static int vals[64];
  static int n = 0;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n; ++i)
    if (keys[i] == (const void*)k) return (int64_t)vals[i] * sms;
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
  if (n < 64) { keys[n] = (const void*)k; vals[n] = per_sm; ++n; }
  return (int64_t)per_sm * sms;
}

// Launch with programmatic stream serialization (the kernel calls grid_dependency_wait() before
// its first global-memory access).
template <typename... KArgs, typename... Args>
static i8q_status launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  I8Q_CUDA(cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...));
  return I8Q_OK;
}
// The same with dynamic shared memory.
template <typename... KArgs, typename... Args>
static i8q_status launch_pdl_smem(void (*kern)(KArgs...), unsigned grid, unsigned block, int smem, cudaStream_t s,
                                  Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  I8Q_CUDA(cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...));
  return I8Q_OK;
}

// ------------------------------------------------------------------ W8A16 launch ------------
// Split-K factor of the W8A16 GEMM: the largest cluster size s in 1..8 (and <= K / 128) whose
// tiles x s CTAs stay within one wave of co-resident CTAs (about 95% of the SMs' CTA slots: cluster
// placement within GPCs leaves a few SMs unused).  Filling both CTA slots of an SM matters: one CTA
// streams weights well below an SM's share of HBM bandwidth (measured: N = 4096, K = 12288, 16
// tokens takes 24 us at s = 4 and 16.5 us at s = 8), while an extra wave would pay the per-CTA
// start-up and pipeline-fill latency again.
static int decode_splits(int64_t tiles, int64_t KB, int sms, int per_sm) {
  const int64_t slots = (int64_t)(sms * 95 / 100) * per_sm;
  int s = 1;
  while (s < 8 && s < KB && tiles * (s + 1) <= slots) ++s;
  return s;
}

// Split-K factor of the decode-size W8A8 GEMM: the largest cluster size s in 1..4 (and <= K / 128)
// whose tiles x s CTAs are all co-resident (CPS per SM), so that as many CTAs as fit stream weights
// at once, in one wave.  Clusters stay at 4 CTAs or fewer: larger ones did not all find room while
// the quantizer that precedes the GEMM still held some SMs (dependent launch), leaving a tail.
static int w8a8_small_splits(int64_t tiles, int64_t KB, int sms, int cps) {
  int s = 1;
  while (s < 4 && s < KB && tiles * (s + 1) <= (int64_t)sms * cps) ++s;
  return s;
}

template <int MP, bool BF16>
static i8q_status launch_w8a16_mp(const uint16_t* x, const int8_t* wq, const uint16_t* s, int M, int N, int K,
                                  uint16_t* y, int sms, cudaStream_t stream) {
  using C = W8A16Cfg<MP>;
  auto kern = k_gemm_w8a16<MP, BF16>;
  const i8q_status attr = ensure_smem(kern, C::SMEM_BYTES);
  if (attr) return attr;
  CUtensorMap tw, tx;
  i8q_status st = make_tmap_2d(&tw, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, W8A16_BN, 128,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  st = make_tmap_2d(&tx, x, BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, M, K, K,
                    MP, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  const int64_t tiles = cdiv(N, W8A16_BN);
  const int64_t mtiles = cdiv(M, MP);           // token tiles (one for decode batches)
  const int splits = decode_splits(tiles * mtiles, K / 128, sms, C::CTAS_PER_SM);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles, (unsigned)splits, (unsigned)mtiles);
  cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = (unsigned)splits;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait()
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  W8A16Args a{s, M, N, K, y};
  I8Q_CUDA(cudaLaunchKernelEx(&cfg, kern, tw, tx, a));
  return I8Q_OK;
}

template <bool BF16>
static i8q_status launch_w8a16(const uint16_t* x, const int8_t* wq, const uint16_t* s, int M, int N, int K,
                               uint16_t* y, int sms, cudaStream_t stream) {
  if (M <= 16) return launch_w8a16_mp<16, BF16>(x, wq, s, M, N, K, y, sms, stream);
  if (M <= 32) return launch_w8a16_mp<32, BF16>(x, wq, s, M, N, K, y, sms, stream);
  if (M <= 64) return launch_w8a16_mp<64, BF16>(x, wq, s, M, N, K, y, sms, stream);
  return launch_w8a16_mp<128, BF16>(x, wq, s, M, N, K, y, sms, stream);   // prefill: 128-token tiles
}

// ------------------------------------------------------------------ W8A8 launch -------------
static i8q_status gemm_w8a8_common_checks(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                          int64_t M, int64_t N, int64_t K, const void* y, const void* dbg) {
  I8Q_REQUIRE(M >= 0 && N >= 0 && K >= 0 && M < kMaxDim && N < kMaxDim && K < kMaxDim, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(K % 128 == 0, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(127LL * 127LL * K < (1LL << 31), I8Q_ERR_SHAPE);
  if (M == 0 || N == 0) return I8Q_OK;
  I8Q_REQUIRE(y, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(y) && aligned16(dbg), I8Q_ERR_ALIGN);
  if (K == 0) return I8Q_OK;
  I8Q_REQUIRE(xq && sx && wq && sw, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(xq) && aligned16(sx) && aligned16(wq) && aligned16(sw), I8Q_ERR_ALIGN);
  return I8Q_OK;
}

template <int BN, bool BLOCKWISE, bool F32, bool DBG, bool ALIGNED = true>
static i8q_status launch_w8a8(const int8_t* xq, const int8_t* wq, const W8A8Args& a, int sms, cudaStream_t s) {
  constexpr bool TS = BLOCKWISE && !F32 && ALIGNED;   // the kernel's TMA-store epilogue
  using C = W8A8Cfg<BN, TS ? 1 : 0>;
  auto kern = k_gemm_w8a8<BN, BLOCKWISE, F32, DBG, false, ALIGNED>;
  const i8q_status attr = ensure_smem(kern, C::SMEM_BYTES);
  if (attr) return attr;
  CUtensorMap ta, tb, ty;
  i8q_status st = make_tmap_2d(&ta, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.K, a.K, 128, GEMM_BK,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  st = make_tmap_2d(&tb, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, a.K, a.K, BN / 2, GEMM_BK,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  if constexpr (TS) {
    // bf16 output tiles of 32 rows x 64 columns (128 bytes: the 128-byte swizzle span); N % 8 == 0
    st = make_tmap_2d(&ty, a.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.N, a.N, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st) return st;
  } else {
    ty = ta;   // unused
  }
  const int64_t tiles = cdiv(a.M, GEMM_BM) * cdiv(a.N, BN);
  const int64_t pairs = tiles < sms / 2 ? tiles : sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait()
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  I8Q_CUDA(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, a));
  return I8Q_OK;
}

// Grouped (MoE) problems: the pair-tile kernel with the expert map.  The number of m-tiles is
// known only on the device (the offsets are device data), so the grid covers the worst case:
// every expert may add one partial m-tile, ceil(M / 256) + E m-tiles in all.
template <bool BLOCKWISE, bool F32, bool DBG, bool ALIGNED>
static i8q_status launch_w8a8_grouped_k(const int8_t* xq, const int8_t* wq, const W8A8Args& a, int sms,
                                        cudaStream_t s) {
  constexpr int BN = 256;
  constexpr bool TS = BLOCKWISE && !F32 && ALIGNED;   // the kernel's TMA-store epilogue
  using C = W8A8Cfg<BN, TS ? 2 : 0>;
  auto kern = k_gemm_w8a8<BN, BLOCKWISE, F32, DBG, true, ALIGNED>;
  const i8q_status attr = ensure_smem(kern, C::SMEM_BYTES_GROUPED);
  if (attr) return attr;
  CUtensorMap ta, tb, ty;
  i8q_status st = make_tmap_2d(&ta, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.K, a.K, 128, GEMM_BK,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  st = make_tmap_2d(&tb, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.E * a.N, a.K, a.K, BN / 2, GEMM_BK,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  if constexpr (TS) {
    st = make_tmap_2d(&ty, a.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.N, a.N, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st) return st;
  } else {
    ty = ta;   // unused
  }
  const int64_t tiles = (cdiv(a.M, GEMM_BM) + a.E) * cdiv(a.N, BN);
  const int64_t pairs = tiles < sms / 2 ? tiles : sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES_GROUPED;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait()
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  I8Q_CUDA(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, a));
  return I8Q_OK;
}

template <bool BLOCKWISE, bool F32, bool DBG>
static i8q_status launch_w8a8_grouped(const int8_t* xq, const int8_t* wq, const W8A8Args& a, int sms,
                                      cudaStream_t s) {
  if (a.N % 8 == 0) return launch_w8a8_grouped_k<BLOCKWISE, F32, DBG, true>(xq, wq, a, sms, s);
  return launch_w8a8_grouped_k<BLOCKWISE, F32, DBG, false>(xq, wq, a, sms, s);
}

static i8q_status grouped_checks(const int32_t* off, int64_t E, int64_t M, int64_t N, int64_t K) {
  I8Q_REQUIRE(E >= 1 && E <= kMaxExperts, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(E * N < ((int64_t)1 << 31), I8Q_ERR_SHAPE);   // row coordinates of the stacked weights
  (void)M;
  (void)K;
  I8Q_REQUIRE(off, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(off), I8Q_ERR_ALIGN);
  return I8Q_OK;
}

// Decode-size batches (M <= 64): weight rows on the MMA's M side, tokens padded to 16/32/64 on its
// N side, K split over a thread-block cluster.
template <int MP, bool BLOCKWISE, bool F32, bool DBG>
static i8q_status launch_w8a8_small_mp(const int8_t* xq, const int8_t* wq, const W8A8Args& a, int sms,
                                       cudaStream_t s) {
  constexpr int CPS = MP <= 64 ? 2 : 1;   // 128 tokens: one CTA per SM (TMEM and registers)
  using C = W8A8SmallCfg<MP, BLOCKWISE, CPS>;
  auto kern = k_gemm_w8a8_small<MP, BLOCKWISE, CPS, F32, DBG>;
  const i8q_status attr = ensure_smem(kern, C::SMEM_BYTES);
  if (attr) return attr;
  CUtensorMap tw, tx;
  i8q_status st = make_tmap_2d(&tw, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, a.K, a.K, 128, 128,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  st = make_tmap_2d(&tx, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.K, a.K, MP, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  const int64_t tiles = cdiv(a.N, 128);
  const int splits = w8a8_small_splits(tiles, a.K / 128, sms, CPS);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles, (unsigned)splits, 1);
  cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = (unsigned)splits;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait()
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  I8Q_CUDA(cudaLaunchKernelEx(&cfg, kern, tw, tx, a));
  return I8Q_OK;
}

// Block-wise GEMM with the activation quantization fused in (decode batches, M <= 16): the decode
// kernel with quantizer warps; X arrives as bf16 through its own TMA map.
template <int MP, bool F32>
static i8q_status launch_w8a8_fused_mp(const uint16_t* x, int64_t ldx, const int8_t* wq, const W8A8Args& a, int sms,
                                       cudaStream_t s) {
  constexpr int CPS = 2;
  using C = W8A8SmallCfg<MP, true, CPS, true>;
  auto kern = k_gemm_w8a8_small<MP, true, CPS, F32, false, true>;
  const i8q_status attr = ensure_smem(kern, C::SMEM_BYTES);
  if (attr) return attr;
  CUtensorMap tw, tx;
  i8q_status st = make_tmap_2d(&tw, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, a.K, a.K, 128, 128,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  st = make_tmap_2d(&tx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.K, ldx, MP, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st) return st;
  const int64_t tiles = cdiv(a.N, 128);
  const int splits = w8a8_small_splits(tiles, a.K / 128, sms, CPS);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles, (unsigned)splits, 1);
  cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = (unsigned)splits;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait()
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  I8Q_CUDA(cudaLaunchKernelEx(&cfg, kern, tw, tx, a));
  return I8Q_OK;
}

template <bool F32>
static i8q_status launch_w8a8_fused(const uint16_t* x, int64_t ldx, const int8_t* wq, const W8A8Args& a, int sms,
                                    cudaStream_t s) {
  return launch_w8a8_fused_mp<16, F32>(x, ldx, wq, a, sms, s);
}

// Tile width of the channel-wise pair tiles (256 x BN): the persistent pairs run ceil(tiles / pairs)
// rounds of work proportional to BN, plus a cost per tile that grows as tiles narrow (each tile
// re-reads its 256 token rows from L2; measured: at M = 16384, N = 7168 tiles of 256 beat 224 by
// 7% although 224 fills the rounds better), so a narrower tile wins only when it fills the last
// round much better.
static int channel_tile_n(int64_t M, int64_t N, int sms) {
  const int64_t pairs = sms / 2;
  const int cands[3] = {256, 224, 192};
  int best = 256;
  int64_t best_cost = INT64_MAX;
  for (int bn : cands) {
    const int64_t tiles = cdiv(M, GEMM_BM) * cdiv(N, bn);
    const int64_t cost = cdiv(tiles, pairs) * (bn + 64);
    if (cost < best_cost) { best_cost = cost; best = bn; }
  }
  return best;
}

template <bool BLOCKWISE, bool F32, bool DBG>
static i8q_status launch_w8a8_any(const int8_t* xq, const int8_t* wq, const W8A8Args& a, int sms, cudaStream_t s) {
  if (a.M <= 16) return launch_w8a8_small_mp<16, BLOCKWISE, F32, DBG>(xq, wq, a, sms, s);
  if (a.M <= 32) return launch_w8a8_small_mp<32, BLOCKWISE, F32, DBG>(xq, wq, a, sms, s);
  if (a.M <= 64) return launch_w8a8_small_mp<64, BLOCKWISE, F32, DBG>(xq, wq, a, sms, s);
  if (a.M <= W8A8_SMALL_MAX_M) return launch_w8a8_small_mp<128, BLOCKWISE, F32, DBG>(xq, wq, a, sms, s);
  // output rows that are not 16-byte aligned take the element-wise epilogue (its own instantiation)
  if (a.N % 8 != 0) return launch_w8a8<256, BLOCKWISE, F32, DBG, false>(xq, wq, a, sms, s);
  if constexpr (!BLOCKWISE) {
    switch (channel_tile_n(a.M, a.N, sms)) {
      case 224: return launch_w8a8<224, false, F32, DBG>(xq, wq, a, sms, s);
      case 192: return launch_w8a8<192, false, F32, DBG>(xq, wq, a, sms, s);
      default: break;
    }
  }
  return launch_w8a8<256, BLOCKWISE, F32, DBG>(xq, wq, a, sms, s);
}


}  // namespace i8q

using namespace i8q;

// ================================================================== entry points =============
extern "C" {

int i8q_version(void) { return 100; }

const char* i8q_status_string(i8q_status s) {
  switch (s) {
    case I8Q_OK: return "I8Q_OK";
    case I8Q_ERR_NULL: return "I8Q_ERR_NULL";
    case I8Q_ERR_SHAPE: return "I8Q_ERR_SHAPE";
    case I8Q_ERR_ALIGN: return "I8Q_ERR_ALIGN";
    case I8Q_ERR_DTYPE: return "I8Q_ERR_DTYPE";
    case I8Q_ERR_CUDA: return "I8Q_ERR_CUDA";
    case I8Q_ERR_TIMEOUT: return "I8Q_ERR_TIMEOUT";
    case I8Q_ERR_UNSUPPORTED: return "I8Q_ERR_UNSUPPORTED";
  }
  return "I8Q_ERR_UNKNOWN";
}

const char* i8q_last_error_string(void) { return t_last_error; }

i8q_status i8q_status_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word = 0, zero = 0;
  I8Q_CUDA(cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)));
  if (word != 0) {
    I8Q_CUDA(cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)));
    snprintf(t_last_error, sizeof(t_last_error), "bounded device wait expired (site %u)", (word >> 8) & 0xFFu);
    return I8Q_ERR_TIMEOUT;
  }
  return I8Q_OK;
}

// ---------------------------------------------------------------- test aids ------------------
i8q_status i8q_test_set_wait_limit_ns(uint64_t ns) {
  unsigned long long v = ns ? (unsigned long long)ns : kWaitTimeoutNs;
  I8Q_CUDA(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
  return I8Q_OK;
}

i8q_status i8q_test_skip_accumulator_signal(int armed) {
  unsigned int v = armed ? 1u : 0u;
  I8Q_CUDA(cudaMemcpyToSymbol(g_test_skip_acc_signal, &v, sizeof(v)));
  return I8Q_OK;
}

// ---------------------------------------------------------------- a1 -------------------------
i8q_status i8q_quant_act_token_group(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int8_t* xq, float* sx,
                                     int64_t ld_sx, void* stream) {
  I8Q_REQUIRE(M >= 0 && K >= 0 && M < kMaxDim && K < kMaxDim, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(K % 128 == 0, I8Q_ERR_SHAPE);
  if (M == 0 || K == 0) return I8Q_OK;
  I8Q_REQUIRE(x && xq && sx, I8Q_ERR_NULL);
  I8Q_REQUIRE(ldx >= K && ldx % 8 == 0 && ld_sx >= M && ld_sx % 4 == 0, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(aligned16(x) && aligned16(xq) && aligned16(sx), I8Q_ERR_ALIGN);
  int sms;
  i8q_status st = current_device(&sms);
  if (st) return st;
  const int64_t KB = K / 128;
  constexpr int U = 1;   // one warp step per item: 63 registers, four CTAs per SM (U = 2: 99, two)
  const int64_t items = M * cdiv(cdiv(KB, 8), U);
  I8Q_REQUIRE(items < ((int64_t)1 << 31), I8Q_ERR_SHAPE);
  int64_t blocks = cdiv(items, 8);
  const int64_t cap = resident_grid(k_quant_act_token_group<U>, 256, sms);
  if (blocks > cap) blocks = cap;
  st = launch_pdl(k_quant_act_token_group<U>, (unsigned)blocks, 256, S(stream), x, (int)M, (int)KB, ldx, xq, sx, ld_sx);
  if (st) return st;
  I8Q_LAUNCHED("k_quant_act_token_group");
  return I8Q_OK;
}

// ---------------------------------------------------------------- a2 -------------------------
i8q_status i8q_quant_act_token(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int8_t* xq, float* sx,
                               void* stream) {
  I8Q_REQUIRE(M >= 0 && K >= 0 && M < kMaxDim && K < kMaxDim, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(K % 8 == 0, I8Q_ERR_SHAPE);   // rows move as 16-byte bf16 / 8-byte int8 vectors
  if (M == 0) return I8Q_OK;
  I8Q_REQUIRE(x && xq && sx, I8Q_ERR_NULL);
  I8Q_REQUIRE(ldx >= K && ldx % 8 == 0, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(aligned16(x) && aligned16(xq) && aligned16(sx), I8Q_ERR_ALIGN);
  int sms;
  i8q_status st = current_device(&sms);
  if (st) return st;
  const int64_t nv = K / 8;
  if (nv <= 32 * 8) {   // warp per row, row in registers
    const int64_t warps = M;
    const int64_t cap1 = resident_grid(k_quant_act_token_warp<8, false>, 256, sms);
    if (cdiv(warps, 8) <= cap1) {          // every row in flight at once: no prefetch needed
      const unsigned grid = (unsigned)cdiv(warps, 8);
      if (nv <= 32 * 2)
        st = launch_pdl(k_quant_act_token_warp<2, false>, grid, 256, S(stream), x, (int)M, (int)K, ldx, xq, sx);
      else if (nv <= 32 * 4)
        st = launch_pdl(k_quant_act_token_warp<4, false>, grid, 256, S(stream), x, (int)M, (int)K, ldx, xq, sx);
      else
        st = launch_pdl(k_quant_act_token_warp<8, false>, grid, 256, S(stream), x, (int)M, (int)K, ldx, xq, sx);
    } else {                                 // warps own several rows: prefetch the next
      int64_t grid = cdiv(M, 8);
      const int64_t cap = resident_grid(k_quant_act_token_warp<8, true>, 256, sms);
      if (grid > cap) grid = cap;
      st = launch_pdl(k_quant_act_token_warp<8, true>, (unsigned)grid, 256, S(stream), x, (int)M, (int)K, ldx, xq, sx);
    }
  } else {              // CTA per row
    st = launch_pdl(k_quant_act_token_cta, (unsigned)M, 256, S(stream), x, (int)K, ldx, xq, sx);
  }
  if (st) return st;
  I8Q_LAUNCHED("k_quant_act_token");
  return I8Q_OK;
}

// ---------------------------------------------------------------- a3', a3 --------------------
i8q_status i8q_quant_weight_block(const uint16_t* w, int64_t N, int64_t K, int8_t* wq, float* sw, void* stream) {
  I8Q_REQUIRE(N >= 0 && K >= 0 && N < kMaxDim && K < kMaxDim && K % 128 == 0, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(cdiv(N, 128) * (K / 128) < kMaxDim, I8Q_ERR_SHAPE);   // block indices are 32-bit
  if (N == 0 || K == 0) return I8Q_OK;
  I8Q_REQUIRE(w && wq && sw, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(w) && aligned16(wq) && aligned16(sw), I8Q_ERR_ALIGN);
  int sms;
  i8q_status st = current_device(&sms);
  if (st) return st;
  int64_t blocks = cdiv(N, 128) * (K / 128);
  const int64_t cap = resident_grid(k_quant_weight_block, 256, sms);
  if (blocks > cap) blocks = cap;
  k_quant_weight_block<<<(unsigned)blocks, 256, 0, S(stream)>>>(w, (int)N, (int)K, wq, sw);
  I8Q_LAUNCHED("k_quant_weight_block");
  return I8Q_OK;
}

// stages (= warp pairs) per CTA of the FP8 block requantization: 12 x 16 KB per SM, 24 warps
constexpr int REQUANT_NP = 12;

i8q_status i8q_requant_fp8_to_int8_block(const uint8_t* w, const float* sf, int64_t N, int64_t K, int8_t* wq,
                                         float* sw, void* stream) {
  I8Q_REQUIRE(N >= 0 && K >= 0 && N < kMaxDim && K < kMaxDim && K % 128 == 0, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(cdiv(N, 128) * (K / 128) < kMaxDim, I8Q_ERR_SHAPE);   // block indices are 32-bit
  if (N == 0 || K == 0) return I8Q_OK;
  I8Q_REQUIRE(w && sf && wq && sw, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(w) && aligned16(sf) && aligned16(wq) && aligned16(sw), I8Q_ERR_ALIGN);
  int sms;
  i8q_status st = current_device(&sms);
  if (st) return st;
  // one CTA per SM of REQUANT_NP warp pairs, each streaming its blocks through one TMA stage
  using C = RequantCfg<REQUANT_NP>;
  auto kern = k_requant_fp8_block<REQUANT_NP>;
  const i8q_status attr = ensure_smem(kern, C::SMEM_BYTES);
  if (attr) return attr;
  CUtensorMap tw;
  st = make_tmap_2d(&tw, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st) return st;
  const int64_t nblocks = cdiv(N, 128) * (K / 128);
  int64_t ctas = cdiv(nblocks, REQUANT_NP);
  if (ctas > sms) ctas = sms;
  st = launch_pdl_smem(kern, (unsigned)ctas, C::NUM_THREADS, C::SMEM_BYTES, S(stream), tw, sf, (int)N, (int)K, wq, sw);
  if (st) return st;
  I8Q_LAUNCHED("k_requant_fp8_block");
  return I8Q_OK;
}

i8q_status i8q_requant_fp8_to_int8_channel(const uint8_t* w, const float* sf, int64_t N, int64_t K, int8_t* wq,
                                           float* sw, void* stream) {
  I8Q_REQUIRE(N >= 0 && K >= 0 && N < kMaxDim && K < kMaxDim && K % 128 == 0, I8Q_ERR_SHAPE);
  if (N == 0) return I8Q_OK;
  I8Q_REQUIRE(w && sf && wq && sw, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(w) && aligned16(sf) && aligned16(wq) && aligned16(sw), I8Q_ERR_ALIGN);
  int sms;
  i8q_status st = current_device(&sms);
  if (st) return st;
  k_requant_fp8_channel<<<(unsigned)N, 256, 0, S(stream)>>>(w, sf, (int)K, wq, sw);
  I8Q_LAUNCHED("k_requant_fp8_channel");
  return I8Q_OK;
}

// ---------------------------------------------------------------- a4, a5 ---------------------
i8q_status i8q_gemm_w8a8_channel(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                                 int64_t N, int64_t K, uint16_t* y, int32_t* dbg, void* stream) {
  i8q_status st = gemm_w8a8_common_checks(xq, sx, wq, sw, M, N, K, y, dbg);
  if (st || M == 0 || N == 0) return st;
  int sms;
  st = current_device(&sms);
  if (st) return st;
  if (K == 0) {
    I8Q_CUDA(cudaMemsetAsync(y, 0, (size_t)M * N * 2, S(stream)));
    if (dbg) I8Q_CUDA(cudaMemsetAsync(dbg, 0, (size_t)M * N * 4, S(stream)));
    return I8Q_OK;
  }
  W8A8Args a{sx, 0, sw, (int)M, (int)N, (int)K, y, dbg, nullptr, 1};
  if (dbg) return launch_w8a8_any<false, false, true>(xq, wq, a, sms, S(stream));
  return launch_w8a8_any<false, false, false>(xq, wq, a, sms, S(stream));
}

i8q_status i8q_gemm_w8a8_block(const int8_t* xq, const float* sx, int64_t ld_sx, const int8_t* wq, const float* sw,
                               int64_t M, int64_t N, int64_t K, void* y, i8q_out_dtype out, int32_t* dbg,
                               void* stream) {
  I8Q_REQUIRE(out == I8Q_OUT_BF16 || out == I8Q_OUT_FP32, I8Q_ERR_DTYPE);
  i8q_status st = gemm_w8a8_common_checks(xq, sx, wq, sw, M, N, K, y, dbg);
  if (st || M == 0 || N == 0) return st;
  if (K > 0) I8Q_REQUIRE(ld_sx >= M && ld_sx % 4 == 0, I8Q_ERR_SHAPE);
  int sms;
  st = current_device(&sms);
  if (st) return st;
  const size_t osz = out == I8Q_OUT_FP32 ? 4 : 2;
  if (K == 0) {
    I8Q_CUDA(cudaMemsetAsync(y, 0, (size_t)M * N * osz, S(stream)));
    return I8Q_OK;
  }
  W8A8Args a{sx, ld_sx, sw, (int)M, (int)N, (int)K, y, dbg, nullptr, 1};
  const bool f32 = out == I8Q_OUT_FP32;
  if (dbg) {
    if (f32) return launch_w8a8_any<true, true, true>(xq, wq, a, sms, S(stream));
    return launch_w8a8_any<true, false, true>(xq, wq, a, sms, S(stream));
  }
  if (f32) return launch_w8a8_any<true, true, false>(xq, wq, a, sms, S(stream));
  return launch_w8a8_any<true, false, false>(xq, wq, a, sms, S(stream));
}

// ---------------------------------------------------------------- a1 fused into a4 ----------
i8q_status i8q_gemm_w8a8_block_fused_quant(const uint16_t* x, int64_t ldx, const int8_t* wq, const float* sw,
                                           int64_t M, int64_t N, int64_t K, void* y, i8q_out_dtype out,
                                           int8_t* xq_out, float* sx_out, int64_t ld_sx, void* stream) {
  I8Q_REQUIRE(out == I8Q_OUT_BF16 || out == I8Q_OUT_FP32, I8Q_ERR_DTYPE);
  I8Q_REQUIRE(M >= 0 && N >= 0 && K >= 0 && N < kMaxDim && K < kMaxDim, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(M <= kFusedQuantMaxM && K % 128 == 0, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(127LL * 127LL * K < (1LL << 31), I8Q_ERR_SHAPE);
  if (M == 0 || N == 0) return I8Q_OK;
  I8Q_REQUIRE(y, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(y) && aligned16(xq_out) && aligned16(sx_out), I8Q_ERR_ALIGN);
  if (sx_out) I8Q_REQUIRE(ld_sx >= M && ld_sx % 4 == 0, I8Q_ERR_SHAPE);
  if (K > 0) {
    I8Q_REQUIRE(x && wq && sw, I8Q_ERR_NULL);
    I8Q_REQUIRE(ldx >= K && ldx % 8 == 0, I8Q_ERR_SHAPE);
    I8Q_REQUIRE(aligned16(x) && aligned16(wq) && aligned16(sw), I8Q_ERR_ALIGN);
  }
  int sms;
  i8q_status st = current_device(&sms);
  if (st) return st;
  const size_t osz = out == I8Q_OUT_FP32 ? 4 : 2;
  if (K == 0) {
    I8Q_CUDA(cudaMemsetAsync(y, 0, (size_t)M * N * osz, S(stream)));
    return I8Q_OK;
  }
  W8A8Args a{nullptr, ld_sx, sw, (int)M, (int)N, (int)K, y, nullptr, nullptr, 1, xq_out, sx_out};
  if (out == I8Q_OUT_FP32) return launch_w8a8_fused<true>(x, ldx, wq, a, sms, S(stream));
  return launch_w8a8_fused<false>(x, ldx, wq, a, sms, S(stream));
}

// ---------------------------------------------------------------- grouped (MoE) a5, a4 ------
i8q_status i8q_gemm_w8a8_channel_grouped(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                         const int32_t* expert_offsets, int64_t E, int64_t M, int64_t N, int64_t K,
                                         uint16_t* y, int32_t* dbg, void* stream) {
  i8q_status st = gemm_w8a8_common_checks(xq, sx, wq, sw, M, N, K, y, dbg);
  if (st || M == 0 || N == 0) return st;
  st = grouped_checks(expert_offsets, E, M, N, K);
  if (st) return st;
  int sms;
  st = current_device(&sms);
  if (st) return st;
  if (K == 0) {
    I8Q_CUDA(cudaMemsetAsync(y, 0, (size_t)M * N * 2, S(stream)));
    if (dbg) I8Q_CUDA(cudaMemsetAsync(dbg, 0, (size_t)M * N * 4, S(stream)));
    return I8Q_OK;
  }
  W8A8Args a{sx, 0, sw, (int)M, (int)N, (int)K, y, dbg, expert_offsets, (int)E};
  if (dbg) return launch_w8a8_grouped<false, false, true>(xq, wq, a, sms, S(stream));
  return launch_w8a8_grouped<false, false, false>(xq, wq, a, sms, S(stream));
}

i8q_status i8q_gemm_w8a8_block_grouped(const int8_t* xq, const float* sx, int64_t ld_sx, const int8_t* wq,
                                       const float* sw, const int32_t* expert_offsets, int64_t E, int64_t M,
                                       int64_t N, int64_t K, void* y, i8q_out_dtype out, int32_t* dbg, void* stream) {
  I8Q_REQUIRE(out == I8Q_OUT_BF16 || out == I8Q_OUT_FP32, I8Q_ERR_DTYPE);
  i8q_status st = gemm_w8a8_common_checks(xq, sx, wq, sw, M, N, K, y, dbg);
  if (st || M == 0 || N == 0) return st;
  if (K > 0) I8Q_REQUIRE(ld_sx >= M && ld_sx % 4 == 0, I8Q_ERR_SHAPE);
  st = grouped_checks(expert_offsets, E, M, N, K);
  if (st) return st;
  int sms;
  st = current_device(&sms);
  if (st) return st;
  const size_t osz = out == I8Q_OUT_FP32 ? 4 : 2;
  if (K == 0) {
    I8Q_CUDA(cudaMemsetAsync(y, 0, (size_t)M * N * osz, S(stream)));
    return I8Q_OK;
  }
  W8A8Args a{sx, ld_sx, sw, (int)M, (int)N, (int)K, y, dbg, expert_offsets, (int)E};
  const bool f32 = out == I8Q_OUT_FP32;
  if (dbg) {
    if (f32) return launch_w8a8_grouped<true, true, true>(xq, wq, a, sms, S(stream));
    return launch_w8a8_grouped<true, false, true>(xq, wq, a, sms, S(stream));
  }
  if (f32) return launch_w8a8_grouped<true, true, false>(xq, wq, a, sms, S(stream));
  return launch_w8a8_grouped<true, false, false>(xq, wq, a, sms, S(stream));
}

// ---------------------------------------------------------------- a6 -------------------------
static i8q_status gemm_w8a16_any(const uint16_t* x, const int8_t* wq, const uint16_t* s, int64_t M, int64_t N,
                                 int64_t K, uint16_t* y, bool bf16, void* stream) {
  I8Q_REQUIRE(M >= 0 && N >= 0 && K >= 0 && M < kMaxDim && N < kMaxDim && K < kMaxDim, I8Q_ERR_SHAPE);
  I8Q_REQUIRE(cdiv(M, 128) < 65536 && K % 128 == 0, I8Q_ERR_SHAPE);   // token tiles: the grid's z dimension
  if (M == 0 || N == 0) return I8Q_OK;
  I8Q_REQUIRE(y, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(y), I8Q_ERR_ALIGN);
  int sms;
  i8q_status st = current_device(&sms);
  if (st) return st;
  if (K == 0) {
    I8Q_CUDA(cudaMemsetAsync(y, 0, (size_t)M * N * 2, S(stream)));
    return I8Q_OK;
  }
  I8Q_REQUIRE(x && wq && s, I8Q_ERR_NULL);
  I8Q_REQUIRE(aligned16(x) && aligned16(wq) && aligned16(s), I8Q_ERR_ALIGN);
  if (bf16) return launch_w8a16<true>(x, wq, s, (int)M, (int)N, (int)K, y, sms, S(stream));
  return launch_w8a16<false>(x, wq, s, (int)M, (int)N, (int)K, y, sms, S(stream));
}

i8q_status i8q_gemm_w8a16_group(const uint16_t* x, const int8_t* wq, const uint16_t* s, int64_t M, int64_t N,
                                int64_t K, uint16_t* y, void* stream) {
  return gemm_w8a16_any(x, wq, s, M, N, K, y, false, stream);
}

i8q_status i8q_gemm_w8a16_group_bf16(const uint16_t* x, const int8_t* wq, const uint16_t* s, int64_t M, int64_t N,
                                     int64_t K, uint16_t* y, void* stream) {
  return gemm_w8a16_any(x, wq, s, M, N, K, y, true, stream);
}

}  // extern "C"
