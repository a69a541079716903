// W8A8 GEMMs on the 5th-generation tensor cores (tcgen05.mma kind::i8, int32 accumulators in
// TMEM), for both schemes of "DeepSeek R1 INT8 quantization practice on SGLang", section 2.3:
//
//  * channel-wise (Fig. 3 right): the whole K reduction accumulates in TMEM; the epilogue applies
//    the per-token x per-output-channel scale once and writes bf16.
//  * block-wise (Fig. 3 left): every 128-wide K slab gets a fresh TMEM accumulator; the epilogue
//    warps read each slab's exact int32 partial sum and fold it into an fp32 running sum with the
//    slab's activation-group x weight-block scale (the "several dequantizations inside the INT8
//    matmul, on the CUDA cores").  Two TMEM accumulator buffers let the tensor core run the next
//    slab while the CUDA cores dequantize the previous one.
//
// Kernel structure: persistent, one CTA pair (thread-block cluster of 2) per 2 SMs, each pair
// computes 256 x BN output tiles with the pair-wide MMA (tcgen05 cta_group::2, M = 256):
// CTA r of the pair stages token rows [128 r, 128 r + 128) of the tile's activations and weight
// rows [BN/2 r, BN/2 (r + 1)) of its weights, so each SM streams 128 + BN/2 rows per K slab for
// 128 x BN outputs.  12 warps per CTA:
//   warp 0       TMA producer (both CTAs): per slab, own activation + weight halves into a
//                STAGES-deep ring of 128B-swizzled buffers; completion is counted on the leader
//                CTA's barrier (the leader expects both CTAs' bytes).
//   warp 1       TMEM allocation (both CTAs, pair-wide) and, in the leader CTA, MMA issue:
//                4 x tcgen05.mma (K = 32) per slab; tcgen05.commit multicasts stage release and
//                accumulator-ready signals to both CTAs.
//   warps 4..11  epilogue: warp w reads TMEM lane quarter (w % 4) (tile rows) and column half
//                (w - 4) / 4; one row per thread.  Both CTAs' epilogue warps release an
//                accumulator buffer by arriving on the leader's barrier.  Block-wise bf16 tiles
//                leave through TMA stores from per-warp shared-memory boxes (see W8A8Cfg).
// Register split: warpgroup 0 drops to 24 registers per thread, the epilogue warpgroups rise to
// 240 (block-wise keeps a 128-column fp32 running sum per thread).
// Tiles are visited in bands of 16 pair-rows (4096 tokens): the band's activations stay resident
// in L2 while the weights stream through it once per band.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace i8q {

constexpr int GEMM_BM = 256;       // tokens per pair tile (MMA M, cta_group::2)
constexpr int GEMM_BK = 128;       // K per slab (bytes of int8 = one 128B swizzle row)
constexpr int GEMM_GROUP_M = 16;   // pair-tile rows per raster band
constexpr int kMaxExperts = 1024;  // grouped (MoE) GEMMs: experts per call

// OUT_MODE 1 and 2 (block-wise bf16 output): the epilogue hands each finished tile to TMA stores
// from a 64 KB output buffer instead of storing it itself, so that the MMAs of the next tile do not
// wait for the tile-end write burst (every SM finishes its tile at about the same time).  1 (dense):
// one stage of the ring gives way for the buffer.  2 (grouped): a store box must not cross into the
// next expert's rows, so warps whose 32 rows straddle an expert boundary keep the direct stores
// (and their staging slab); two stages give way.  0: direct stores.
template <int BN, int OUT_MODE = 0>
struct W8A8Cfg {
  static constexpr int A_BYTES = 128 * GEMM_BK;          // this CTA's 128 token rows
  static constexpr int B_BYTES = (BN / 2) * GEMM_BK;     // this CTA's BN/2 weight rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr bool TS = OUT_MODE != 0;
  static constexpr int STAGES = OUT_MODE == 0 ? 6 : (OUT_MODE == 1 ? 5 : 4);
  static constexpr int TMEM_COLS = 512;                  // two accumulator buffers of BN columns
  static constexpr int NUM_THREADS = 384;
  static constexpr int EPI_WARPS = 8;
  static constexpr int BAR_BYTES = 256;
  static constexpr int OUT_WARP_BYTES = 32 * (BN / 2) * 2;          // TS: a warp's 32 rows x BN/2 bf16
  static constexpr int OUT_BYTES = TS ? EPI_WARPS * OUT_WARP_BYTES : 0;
  static constexpr int EPI_STAGE_BYTES = OUT_MODE == 1 ? 0 : EPI_WARPS * 32 * 80;   // per epilogue warp: 32 rows x 80 B
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + OUT_BYTES + BAR_BYTES + EPI_STAGE_BYTES + 1024;  // + alignment slack
  // grouped (MoE) problems: per-expert row offsets and m-tile prefix sums, kMaxExperts + 1 each
  static constexpr int GROUP_BYTES = 2 * (kMaxExperts + 1) * 4;
  static constexpr int SMEM_BYTES_GROUPED = SMEM_BYTES + GROUP_BYTES;
  static_assert(2 * BN <= TMEM_COLS, "two accumulators must fit in TMEM");
  static_assert(!TS || BN == 256, "TMA-store epilogue: two 64-column boxes per warp");
  static_assert((OUT_MODE == 1 ? SMEM_BYTES : SMEM_BYTES_GROUPED) <= 232448, "shared memory");
  static_assert(BN % 32 == 0 && BN <= 256, "MMA N (each CTA's BN / 2 weight rows: whole 8-row groups)");
};

struct W8A8Args {
  const float* sx;      // channel: [M]; block: [KB][ld_sx]
  int64_t ld_sx;
  const float* sw;      // channel: [N]; block: [ceil(N/128)][KB]  (grouped: one such array per expert)
  int M, N, K;
  void* y;              // [M][N] bf16 or fp32
  int32_t* dbg;         // channel: [M][N] accumulators; block: [M][N][KB] slab partials
  const int32_t* off;   // grouped only: [E + 1] row offsets, expert e owns rows off[e] .. off[e+1]-1
  int E;                // grouped only: number of experts (weights [E][N][K])
  int8_t* qx_out;       // fused quantization only (nullable): [M][K] int8 codes of the activations
  float* qs_out;        // fused quantization only (nullable): [K/128][ld_sx] group scales
};

// ------------------------------------------------------------------ pair-wide PTX wrappers ----
__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of the pair; the .aligned barrier needs each warp converged, so it reconverges first.
__device__ __forceinline__ void cluster_sync() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA 2-D tile load issued by either CTA of the pair; bytes are counted on the barrier at
// `bar_cluster` (the leader CTA's).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive once on the barrier at the same offset in both CTAs of the pair when all prior MMAs end
__device__ __forceinline__ void tc_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair_self(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// 32 lanes x 32 columns of 32-bit registers -> TMEM
__device__ __forceinline__ void tmem_st32_const(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(
          taddr),
      "r"(v)
      : "memory");
}

// TMA tile store shared -> global (bulk async-group of the issuing thread; parts of the box
// outside the tensor are not written), and the waits on this thread's groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------ helpers -------------------
__device__ __forceinline__ void gemm_tile_coords(int t, int Mt, int Nt, int& mb, int& nb) {
  const int band_tiles = GEMM_GROUP_M * Nt;
  const int band = t / band_tiles;
  const int first_m = band * GEMM_GROUP_M;
  const int rows = min(GEMM_GROUP_M, Mt - first_m);
  const int idx = t - band * band_tiles;
  mb = first_m + idx % rows;
  nb = idx / rows;
}

// Grouped (MoE) tables, built by one warp after the dependency wait (the offsets may have been
// written by the kernel before): s_off[e] = the offsets made non-decreasing and clamped to [0, M]
// (so that no row outside [0, M) is ever touched, whatever the caller passed), s_pre[e] = the
// number of 256-row m-tiles of experts 0 .. e-1.  Global m-tile g belongs to the largest e with
// s_pre[e] <= g (experts without tokens own no m-tile).
__device__ __forceinline__ void build_group_tables(const int32_t* __restrict__ off, int E, int M, int* s_off,
                                                   int* s_pre, int lane) {
  const int n = E + 1;
  const int chunk = (n + 31) / 32;
  const int b = min(n, lane * chunk), e_ = min(n, b + chunk);
  int mx = 0;
  for (int i = b; i < e_; ++i) {
    const int v = min(max(__ldg(off + i), 0), M);
    s_off[i] = v;
    mx = max(mx, v);
  }
  // exclusive prefix max over the lanes' chunks, then a running max inside the chunk
  int incl = mx;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl = max(incl, o);
  }
  int run = __shfl_up_sync(0xFFFFFFFFu, incl, 1);
  if (lane == 0) run = 0;
  for (int i = b; i < e_; ++i) {
    run = max(run, s_off[i]);
    s_off[i] = run;
  }
  __syncwarp();
  // m-tiles per expert, exclusive prefix sum
  int cnt = 0;
  for (int i = b; i < e_ && i < E; ++i) cnt += (s_off[i + 1] - s_off[i] + GEMM_BM - 1) / GEMM_BM;
  int inc = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, inc, d);
    if (lane >= d) inc += o;
  }
  int pre = inc - cnt;
  for (int i = b; i < e_; ++i) {
    s_pre[i] = pre;
    if (i < E) pre += (s_off[i + 1] - s_off[i] + GEMM_BM - 1) / GEMM_BM;
  }
  __syncwarp();
}

// Rows of global m-tile g: expert e, first row, one past the last row of the expert.
template <bool GROUPED>
__device__ __forceinline__ void tile_rows(int g, int M, const int* s_off, const int* s_pre, int E, int& e,
                                          int& row0, int& row_end) {
  if constexpr (!GROUPED) {
    e = 0;
    row0 = g * GEMM_BM;
    row_end = M;
  } else {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_pre[mid] <= g) lo = mid; else hi = mid;
    }
    e = lo;
    row0 = s_off[lo] + (g - s_pre[lo]) * GEMM_BM;
    row_end = s_off[lo + 1];
  }
}

// fp32 bits 0x4B400000 = 1.5 * 2^23 = 12582912.  An int32 accumulator that starts from these bits
// holds 0x4B400000 + P after the MMA adds P; for |P| < 2^22 those are exactly the bits of the
// float 12582912 + P, so subtracting 12582912 recovers P exactly.
constexpr uint32_t kAccBiasBits = 0x4B400000u;
constexpr float kAccBias = 12582912.0f;

__device__ __forceinline__ void store_row8(void* y, bool f32out, int64_t off, const float (&v)[8]) {
  if (f32out) {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + off);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 u;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
    u.x = *reinterpret_cast<uint32_t*>(&h0);
    u.y = *reinterpret_cast<uint32_t*>(&h1);
    u.z = *reinterpret_cast<uint32_t*>(&h2);
    u.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(y) + off) = u;
  }
}

// One warp's row-per-thread bf16 results -> global memory with whole-sector stores: lane l holds
// columns nc .. nc + W - 1 (W = 16 or 32) of row m_base + l as bf16 pairs.  The 32 rows go through
// a 32 x 80-byte staging slab in shared memory (80-byte rows: conflict-free for row-wise writes and
// column-wise reads), then each store instruction writes 8 rows x 64 contiguous bytes instead of
// 16 bytes of 32 different rows (half-filled sectors).  When N % 8 != 0 (ALIGNED false) the rows of
// y are not 16-byte aligned: every element is then stored on its own (lane = column), masked at N.
template <bool ALIGNED>
__device__ __forceinline__ void store_rows_bf16(uint8_t* stg, int lane, const uint32_t (&p)[16], int W, uint16_t* y,
                                                int N, int m_base, int M, int nc) {
  uint4* srow = reinterpret_cast<uint4*>(stg + lane * 80);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q * 8 < W) srow[q] = make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
  __syncwarp();
  if constexpr (ALIGNED) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = i * 8 + (lane & 7), c = lane >> 3;
      const int m = m_base + r, n = nc + c * 8;
      if (c * 8 < W && m < M && n < N)
        *reinterpret_cast<uint4*>(y + (int64_t)m * N + n) = *reinterpret_cast<const uint4*>(stg + r * 80 + c * 16);
    }
  } else {
    const int n = nc + lane;
    for (int r = 0; r < 32; ++r) {
      const int m = m_base + r;
      if (lane < W && m < M && n < N) y[(int64_t)m * N + n] = reinterpret_cast<const uint16_t*>(stg + r * 80)[lane];
    }
  }
  __syncwarp();
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN, bool BLOCKWISE, bool OUT_F32, bool DEBUG, bool GROUPED = false, bool ALIGNED = true>
__global__ void __launch_bounds__(384, 1)
    k_gemm_w8a8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, const W8A8Args args) {
  constexpr bool TS = BLOCKWISE && !OUT_F32 && ALIGNED;   // TMA-store epilogue (tmY)
  using C = W8A8Cfg<BN, TS ? (GROUPED ? 2 : 1) : 0>;
  static_assert(!BLOCKWISE || BN == 256, "block-wise pair tiles are two weight blocks wide");
  constexpr int HALF = BN / 2;                 // columns per epilogue warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* sOut = smem + C::STAGES * C::STAGE_BYTES;   // TS: output boxes (1024-byte aligned)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::OUT_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* sStage = smem + C::STAGES * C::STAGE_BYTES + C::OUT_BYTES + C::BAR_BYTES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank_in_cluster();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int M = args.M, N = args.N, K = args.K;
  const int Nt = (N + BN - 1) / BN, KB = K / GEMM_BK;
  int Mt = (M + GEMM_BM - 1) / GEMM_BM;   // grouped: set from the expert offsets below
  int num_tiles = Mt * Nt;
  // ALIGNED (N % 8 == 0, chosen by the host): rows of y, sw and the debug outputs allow vector
  // accesses.  A compile-time choice: a run-time test in the epilogue cost 10% at K = 2048.
  constexpr bool nvec = ALIGNED;
  int* s_off = reinterpret_cast<int*>(sStage + C::EPI_STAGE_BYTES);   // grouped tables
  int* s_pre = s_off + (kMaxExperts + 1);
  const int E = GROUPED ? args.E : 1;
  // per-expert stride of the weight scales: channel [E][N], block [E][ceil(N/128)][KB]
  const int64_t sw_estride = BLOCKWISE ? (int64_t)((N + 127) / 128) * KB : (int64_t)N;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * C::EPI_WARPS);   // every epilogue warp of both CTAs
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // The kernel may be launched while the preceding kernel (typically the activation quantizer) is
  // still running: until grid_dependency_wait() it touches no global memory except L2 prefetches of
  // the weight slabs of its first tile.
  if (!GROUPED && warp == 0 && lane == 0 && pair < num_tiles) {
    int mb, nb;
    gemm_tile_coords(pair, Mt, Nt, mb, nb);
    for (int kb = 0; kb < KB && kb < C::STAGES; ++kb)
      tma_prefetch_l2_2d(&tmB, kb * GEMM_BK, nb * BN + (int)rank * HALF);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();
  if constexpr (GROUPED) {
    if (warp == 2) build_group_tables(args.off, E, M, s_off, s_pre, lane);
    __syncthreads();
    Mt = s_pre[E];
    num_tiles = Mt * Nt;
  }

  if (warp < 4) {
    setmaxnreg_dec<24>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t expected = 0, exp_parity = 0;   // leader: stages whose completion it expects
      bool ok = true;
      for (int t = pair; ok && t < num_tiles; t += npairs) {
        int mb, nb, e, row0, row_end;
        gemm_tile_coords(t, Mt, Nt, mb, nb);
        tile_rows<GROUPED>(mb, M, s_off, s_pre, E, e, row0, row_end);
        const int arow = row0 + (int)rank * 128;
        const int brow = e * N + nb * BN + (int)rank * HALF;   // grouped: W is [E * N][K]
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, SITE_EMPTY, abort_flag)) { ok = false; break; }
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            expected |= 1u << stage;
            exp_parity = (exp_parity & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t bar = map_to_rank(&full[stage], 0);
          tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, bar, kb * GEMM_BK, arow);
          tma_load_2d_pair(sB + stage * C::B_BYTES, &tmB, bar, kb * GEMM_BK, brow);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok && leader) {  // let copies already in flight land before the pair can exit
        for (int s = 0; s < C::STAGES; ++s)
          if (expected & (1u << s)) mbar_wait(&full[s], (exp_parity >> s) & 1u, SITE_DRAIN, nullptr);
      }
    } else if (warp == 1 && lane == 0 && leader) {
      // ------------------------------------------------------------------ MMA issuer (leader)
      constexpr uint32_t idesc = idesc_i8(GEMM_BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_iter = 0;
      bool ok = true;
      for (int t = pair; ok && t < num_tiles; t += npairs) {
        uint32_t acc = 0;
        if (!BLOCKWISE) {
          acc = acc_iter & 1;
          if (!mbar_wait(&tempty[acc], ((acc_iter >> 1) & 1) ^ 1, SITE_TMEM_EMPTY, abort_flag)) { ok = false; break; }
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb) {
          // the stage first: it has normally landed long before, and a satisfied wait still costs
          // this thread a few hundred cycles, which it then spends while the accumulator is busy
          if (!mbar_wait(&full[stage], phase, SITE_FULL, abort_flag)) { ok = false; break; }
          if (BLOCKWISE) {
            // use u of buffer acc waits for the epilogue's u-th release (its bias initialisation)
            acc = acc_iter & 1;
            if (!mbar_wait(&tempty[acc], (acc_iter >> 1) & 1, SITE_TMEM_EMPTY, abort_flag)) { ok = false; break; }
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
          const uint32_t d = tmem + acc * BN;
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 32; ++kk) {
            const uint32_t accumulate = BLOCKWISE ? 1u : (uint32_t)(kb > 0 || kk > 0);
            mma_i8_pair(d, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc, accumulate);
          }
          tc_commit_pair_both(&empty[stage]);
          if (BLOCKWISE) {
            tc_commit_pair_both(&tfull[acc]);
            ++acc_iter;
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!BLOCKWISE && ok) {
          tc_commit_pair_both(&tfull[acc]);
          ++acc_iter;
        }
      }
      // every MMA this thread issued has finished once `done` completes
      tc_commit_pair_self(done);
      mbar_wait(done, 0, SITE_DRAIN, nullptr);
    }
  } else {
    setmaxnreg_inc<240>();
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                         // TMEM lane quarter
    const int h = (warp - 4) >> 2;                  // column half
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int row = (int)rank * 128 + q * 32 + lane;  // row within the 256-row pair tile
    uint8_t* stg = sStage + (warp - 4) * 32 * 80;     // this warp's store staging slab
    const uint32_t tempty_leader0 = map_to_rank(&tempty[0], 0), tempty_leader1 = map_to_rank(&tempty[1], 0);
    uint32_t acc_iter = 0;

    if constexpr (BLOCKWISE) {
      // pre-load both accumulator buffers with the float bias, then release them to the MMA
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int c = 0; c < HALF / 32; ++c) tmem_st32_const(tmem + lane_addr + a * BN + h * HALF + c * 32, kAccBiasBits);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(tempty_leader0);
        mbar_arrive_cluster(tempty_leader1);
      }
    }

    for (int t = pair; t < num_tiles; t += npairs) {
      int mb, nb, e, row0, row_end;
      gemm_tile_coords(t, Mt, Nt, mb, nb);
      tile_rows<GROUPED>(mb, M, s_off, s_pre, E, e, row0, row_end);
      const int m = row0 + row;
      const int n0 = nb * BN + h * HALF;           // first column of this warp's half
      const bool row_ok = m < row_end;
      const float* swp = args.sw + (GROUPED ? (int64_t)e * sw_estride : 0);
      if constexpr (!BLOCKWISE) {
        const uint32_t acc = acc_iter & 1;
        if (!warp_wait(&tfull[acc], (acc_iter >> 1) & 1, SITE_TMEM_FULL, abort_flag)) break;
        tc_fence_after();
        const float sxm = row_ok ? __ldg(args.sx + m) : 0.f;
        // scale W columns starting at column nc of the row and store them (whole-sector stores)
        auto emit = [&](const uint32_t* r, int nc, int W) {
          uint32_t pk[16];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int n = nc + g * 8;
            if (g * 8 < W) {
              float ws[8];
              if constexpr (nvec) {
                float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
                if (n < N) {
                  w0 = __ldg(reinterpret_cast<const float4*>(swp + n));
                  w1 = __ldg(reinterpret_cast<const float4*>(swp + n + 4));
                }
                ws[0] = w0.x; ws[1] = w0.y; ws[2] = w0.z; ws[3] = w0.w;
                ws[4] = w1.x; ws[5] = w1.y; ws[6] = w1.z; ws[7] = w1.w;
              } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) ws[j] = n + j < N ? __ldg(swp + n + j) : 0.f;
              }
              float v[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) v[j] = __int2float_rn((int)r[g * 8 + j]) * (sxm * ws[j]);
#pragma unroll
              for (int j = 0; j < 4; ++j) pk[g * 4 + j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
              if constexpr (DEBUG) {
                if (row_ok && n < N) {
                  if constexpr (nvec) {
                    int4* dp = reinterpret_cast<int4*>(args.dbg + (int64_t)m * N + n);
                    dp[0] = make_int4(r[g * 8 + 0], r[g * 8 + 1], r[g * 8 + 2], r[g * 8 + 3]);
                    dp[1] = make_int4(r[g * 8 + 4], r[g * 8 + 5], r[g * 8 + 6], r[g * 8 + 7]);
                  } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                      if (n + j < N) args.dbg[(int64_t)m * N + n + j] = (int32_t)r[g * 8 + j];
                  }
                }
              }
            }
          }
          store_rows_bf16<nvec>(stg, lane, pk, W, reinterpret_cast<uint16_t*>(args.y), N, m - lane, row_end, nc);
        };
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + acc * BN + h * HALF + c * 32, r);
          tmem_ld_wait();
          emit(r, n0 + c * 32, 32);
        }
        if constexpr (HALF % 32 == 16) {   // 16-column tail of a 224- or 160-column tile
          uint32_t r[32];
          tmem_ld16(tmem + lane_addr + acc * BN + h * HALF + (HALF / 32) * 32,
                    *reinterpret_cast<uint32_t(*)[16]>(r));
          tmem_ld_wait();
          emit(r, n0 + (HALF / 32) * 32, 16);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        ++acc_iter;
      } else {
        float2 sum[HALF / 2];
#pragma unroll
        for (int j = 0; j < HALF / 2; ++j) sum[j] = make_float2(0.f, 0.f);
        bool ok = true;
        const bool live = row_ok && n0 < N;              // this row and weight block exist
        const float* swrow = swp + (int64_t)(n0 / 128) * KB;
        // raw scales of the next slab are loaded one slab ahead; the product is formed when used
        float sx_next = 0.f, sw_next = 0.f;
        if (KB > 0 && live) {
          sx_next = __ldg(args.sx + m);
          sw_next = __ldg(swrow);
        }
        const float2 nbias = make_float2(-kAccBias, -kAccBias);
        for (int kb = 0; kb < KB; ++kb) {
          const float s = sx_next * sw_next;
          if (kb + 1 < KB && live) {
            sx_next = __ldg(args.sx + (int64_t)(kb + 1) * args.ld_sx + m);
            sw_next = __ldg(swrow + kb + 1);
          }
          const float2 s2 = make_float2(s, s);
          const uint32_t acc = acc_iter & 1;
          if (!warp_wait(&tfull[acc], (acc_iter >> 1) & 1, SITE_TMEM_FULL, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = tmem + lane_addr + acc * BN + h * HALF;
#pragma unroll
          for (int c = 0; c < HALF / 32; ++c) {
            uint32_t r0[32];
            tmem_ld32(base + c * 32, r0);
            tmem_ld_wait();
            // re-arm these columns with the bias for the buffer's next use while the math runs
            tmem_st32_const(base + c * 32, kAccBiasBits);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float2 p = __fadd2_rn(make_float2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1])), nbias);
              sum[c * 16 + j] = __ffma2_rn(p, s2, sum[c * 16 + j]);
            }
            if constexpr (DEBUG) {
              if (row_ok) {
                for (int j = 0; j < 32; ++j) {
                  const int na = n0 + c * 32 + j;
                  if (na < N) args.dbg[((int64_t)m * N + na) * KB + kb] = (int32_t)(r0[j] - kAccBiasBits);
                }
              }
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
          ++acc_iter;
        }
        if (!ok) break;
        if constexpr (OUT_F32) {   // 8 fp32 = 32 bytes: whole sectors already
          if (live) {
#pragma unroll
            for (int g = 0; g < HALF / 8; ++g) {
              const int n = n0 + g * 8;
              if (n < N) {
                float v[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  v[2 * j] = sum[g * 4 + j].x;
                  v[2 * j + 1] = sum[g * 4 + j].y;
                }
                if constexpr (nvec) {
                  store_row8(args.y, true, (int64_t)m * N + n, v);
                } else {
#pragma unroll
                  for (int j = 0; j < 8; ++j)
                    if (n + j < N) reinterpret_cast<float*>(args.y)[(int64_t)m * N + n + j] = v[j];
                }
              }
            }
          }
        } else if (TS && (!GROUPED || m - lane + 32 <= row_end || row_end >= M)) {
          // the warp's 32 rows x 128 columns as two 128B-swizzled boxes of 32 x 64 bf16 (row = lane:
          // 16-byte chunk c of a row at chunk c ^ (row % 8)), then two TMA stores (rows >= M and
          // columns >= N are clipped by the tensor map; grouped: only boxes inside the expert's rows).
          // The buffer is rewritten only once the previous tile's stores have read it.
          uint8_t* obuf = sOut + (warp - 4) * C::OUT_WARP_BYTES;
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int j = 32 * k + 4 * c;
              *reinterpret_cast<uint4*>(obuf + k * 4096 + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(sum[j].x, sum[j].y), pack_bf16x2(sum[j + 1].x, sum[j + 1].y),
                             pack_bf16x2(sum[j + 2].x, sum[j + 2].y), pack_bf16x2(sum[j + 3].x, sum[j + 3].y));
            }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0 && m - lane < row_end) {
            if (n0 < N) tma_store_2d(&tmY, obuf, n0, m - lane);
            if (n0 + 64 < N) tma_store_2d(&tmY, obuf + 4096, n0 + 64, m - lane);
            bulk_commit();
          }
        } else {
#pragma unroll
          for (int c = 0; c < HALF / 32; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(sum[c * 16 + j].x, sum[c * 16 + j].y);
            store_rows_bf16<nvec>(stg, lane, pk, 32, reinterpret_cast<uint16_t*>(args.y), N, m - lane, row_end,
                                  n0 + c * 32);
          }
        }
      }
    }
    // the last tiles' stores complete (and stop reading shared memory) before the CTA can exit
    if constexpr (TS) {
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // neither CTA leaves while its pair may still touch its shared memory / TMEM
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, C::TMEM_COLS);
}

}  // namespace i8q
