// The three separable forward DCT passes of TACT-KV stage 2 in one kernel, with the fp32 volume Y
// kept in L2 between the S pass and the H/W pass.
//
// A cluster of kCluster CTAs owns one (unit, 32-channel chunk).  Each CTA runs the DCT along S on
// its share of the grid cells (tiles of 8 cells, one per warp, the next tile in flight) and writes
// Y to the volume; a cluster barrier makes the chunk's Y visible to the whole cluster; each CTA
// then runs the DCT along H and W (with the per-bin energy sums) on its share of the S slabs,
// reading Y and writing X over it.  A chunk's Y (S*H*W*32 floats, 2 MB for 64 x 16 x 16) is
// written and read back by the same cluster shortly after, so it is served by L2 instead of DRAM:
// only the clusters in flight hold Y lines, and the streams that pass through once (the input and
// the finished coefficients X) are marked evict-first so that they give way to it.
//
// The common grids (16x16, 14x14, 8x8 with S = 8, 16, 32 or 64, and 24x24 with S up to 32) have a
// fused kernel; this file is compiled once per S (TACTKV_FUSED_S).  Other shapes use the separate S-axis and H/W-axis
// kernels.
#include "axis_s.cuh"
#include "axis_hw.cuh"
#include "tc.cuh"
#include "dct_limbs.inc"

#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#ifndef TACTKV_FUSED_S
#error "TACTKV_FUSED_S must be defined"
#endif

namespace tactkv {
namespace {

constexpr int kCluster = 8;             // CTAs per (unit, chunk)
constexpr int kNC = 8;                  // cells per S tile: one per warp
constexpr int kFusedThreads = STile<kNC>::kThreads;
static_assert(kFusedThreads == kMaxHwThreads, "the H/W pieces run with the same block");

// Every thread of every CTA of the cluster: global writes before it are visible to the cluster's
// reads after it (release and acquire at cluster scope; the reads are ordinary cp.async copies).
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

template <int L>
__host__ __device__ inline size_t s_tile_bytes(bool fp32_in) {
  return (size_t)L * kNC * 32 * (fp32_in ? 4 : 2);
}

// Shared memory of the forward kernel: the H/W layout, and one or two S tiles overlaid on it.
template <int L>
__host__ __device__ inline size_t fused_fwd_smem(int H, int W, bool fp32_in, int* s_bufs) {
  const size_t hw = hw_layout(H, W, kLayStats).total, st = s_tile_bytes<L>(fp32_in);
  *s_bufs = 2 * st <= hw ? 2 : 1;
  return hw > st ? hw : st;
}

// Pencil length class of an H or W length, and CTAs per SM: the 16-class grids fit 80 registers
// (three CTAs), the 24 x 24 grid's 32-class float2 pencils 128 (two CTAs).
__host__ __device__ constexpr int hw_class(int x) { return x > 16 ? 32 : 16; }
__host__ __device__ constexpr int fused_min_blocks(int hx) { return hx > 16 ? 2 : 3; }

// NX: the channel count when fixed at compile time (the common 512 and 1024), else 0.
template <int L, int HX, int WX, int NX, bool VAR>
__global__ void __launch_bounds__(kFusedThreads, fused_min_blocks(HX)) fdct3_kernel(const __grid_constant__ Geom g,
                                                                 const __grid_constant__ UnitList ul,
                                                                 float* __restrict__ Y, float* __restrict__ partial,
                                                                 int lg_cpr) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = blockIdx.x, chunk = blockIdx.y, u = g.unit0 + blockIdx.z, c0 = chunk * kChunk;
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  const int esz = fp32 ? 4 : 2;
  int nbuf = 1;
  fused_fwd_smem<L>(HX, WX, fp32, &nbuf);
  const size_t tb = s_tile_bytes<L>(fp32);
  const UnitDev& ud = ul.u[u];
  // DCT along S on tiles r, r + kCluster, ... of the chunk's cells (the next tile in flight)
  const int tiles = (HX * WX + kNC - 1) / kNC;
  int buf = 0;
  if (r < tiles) stage_input<L, kNC, true>(g, ud, r * kNC, c0, esz, lg_cpr, smem);
  for (int t = r; t < tiles; t += kCluster) {
    const bool next = t + kCluster < tiles;
    if (nbuf == 2 && next) {
      stage_input<L, kNC, true>(g, ud, (t + kCluster) * kNC, c0, esz, lg_cpr, smem + (buf ^ 1) * tb);
      cp_async_wait_one();
    } else {
      cp_async_wait_all();
    }
    __syncthreads();
    fdct_s_cells<L, kNC, HX * WX, NX, VAR>(g, u, t * kNC, c0, smem + buf * tb, fp32, Y);
    __syncthreads();   // the tile's buffer is free again
    if (nbuf == 2) buf ^= 1;
    else if (next) stage_input<L, kNC, true>(g, ud, (t + kCluster) * kNC, c0, esz, lg_cpr, smem);
  }
  cluster_barrier();   // the chunk's Y is complete
  // DCT along H and W on this CTA's range of slabs
  constexpr int spc = (L + kCluster - 1) / kCluster;
  const int ks0 = r * spc, ks1 = min(L, ks0 + spc);
  if (ks0 < ks1)
    fdct_hw_slabs<hw_class(HX), hw_class(WX), HX, WX, true, NX, VAR>(g, Y, partial, u, chunk, ks0, ks1, smem);
}

// ------------------------------------------------------------- S pass on the tensor cores ---
// The DCT along S of a tile of 4 grid cells x 32 channels is the product
//     Y[(cell, c), k] = sum_s x[(cell, c), s] * C[k, s]
// with M = 128 rows (cell, c), N = S columns k and K = S.  x is exact in bf16; C is carried as
// three bf16 limbs (hi + mid + lo, fp32 accuracy), accumulated into one fp32 TMEM accumulator.
//   A = the input tile, loaded by TMA as [cell][s][32 channels] bf16 with 64-byte swizzle: MN-major,
//       32 channels of one cell per 64-byte row, 8 rows of consecutive s per 512-byte atom;
//   B = a limb of C, [k][s] with s contiguous: K-major with 128-byte swizzle (rows padded to 64 s).
// Thread (warp w, lane l) then reads row 32 (w % 4) + l (cell w % 4, channel l) of the tile, half
// (w / 4) of its S columns, and stores them to Y[k][cell][c]: 128 contiguous bytes per warp store.
constexpr int kTcCells = 4;               // grid cells per tile (M = 128)
constexpr int kTcEpilogueWarps = 8;       // warps 0..7 drain the accumulators; warp 8 produces
constexpr int kTcThreads = 32 * (kTcEpilogueWarps + 1);

template <int L>
struct TcS {
  static_assert(L == 16 || L == 32 || L == 64, "S of the tensor-core pass");
  static constexpr int kABytes = kTcCells * L * 64;      // one input tile
  static constexpr int kBBytes = L * 128;                // one limb of C, rows padded to 128 bytes
  static constexpr int kSmem = 3 * kBBytes + 2 * kABytes + 1024;   // + alignment slack
  static constexpr int kCols = L < 32 ? 32 : L;          // TMEM columns of one accumulator (power of two >= 32)
  static constexpr int kHalf = L / 2;                    // columns read per thread
};

template <int L>
__device__ __forceinline__ const uint16_t* dct_limb_fwd() {
  if constexpr (L == 16) return &kDctLimbFwd16[0][0][0];
  else if constexpr (L == 32) return &kDctLimbFwd32[0][0][0];
  else return &kDctLimbFwd64[0][0][0];
}

// S pass of one (unit u, chunk) on this CTA's tiles t = r, r + kCluster, ... into Y, pipelined:
//   warp 8 (one lane)  TMA producer and MMA issuer: the input tiles go through two shared-memory
//                      stages, the products into two TMEM accumulators (64 columns each), so the
//                      MMAs of a tile run while the epilogue drains the previous one;
//   warps 0..7         epilogue: warp w reads lanes 32 (w % 4).. (cell w % 4 of the tile) and half
//                      w / 4 of the S columns of a finished accumulator, frees it, and stores those
//                      S values to Y.
// mbarriers: full[s] (TMA -> MMA, transaction bytes), done[a] (MMA commit -> epilogue and producer),
// freed[a] (8 epilogue warps -> MMA).  Every wait is bounded; on expiry the CTA records
// TACTKV_TIMEOUT, waits (bounded) for what is in flight, releases TMEM and returns false.  The
// caller still takes part in every barrier of the cluster.  Called by every thread of the CTA.
template <int L, int HWX>
__device__ bool fdct_s_tc(const Geom& g, int u, int chunk, int r, const CUtensorMap* tmap, float* __restrict__ Y,
                          unsigned char* smem, uint64_t* bars, uint32_t* tmem_slot, int nx, unsigned int* status) {
  using P = TcS<L>;
  constexpr int kTiles = (HWX + kTcCells - 1) / kTcCells;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = chunk * kChunk, head = c0 / g.head_dim, d0 = c0 - head * g.head_dim;
  const int uw = u - g.unit0;   // the tensor map's unit coordinate: the unit's place in the wave
  unsigned char* sB = smem;
  unsigned char* sA = smem + 3 * P::kBBytes;
  uint64_t* full = bars;          // [2]
  uint64_t* done = bars + 2;      // [2]
  uint64_t* freed = bars + 4;     // [2]
  __shared__ int s_err;
  const int mine = r < kTiles ? (kTiles - r + kCluster - 1) / kCluster : 0;

  // B: the three limbs of C, swizzled (16-byte chunk j of row k at chunk j ^ (k & 7))
  const uint16_t* tab = dct_limb_fwd<L>();
  for (int e = tid; e < 3 * L * 8; e += blockDim.x) {
    const int l = e / (L * 8), rem = e - l * (L * 8), k = rem >> 3, j = rem & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j * 8 < L) v = *reinterpret_cast<const uint4*>(tab + ((size_t)l * L + k) * L + j * 8);
    *reinterpret_cast<uint4*>(sB + l * P::kBBytes + k * 128 + ((j ^ (k & 7)) << 4)) = v;
  }
  tc::fence_proxy_async();
  if (tid == 0) {
    tc::prefetch_tmap(tmap);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&done[i], 1);
      tc::mbar_init(&freed[i], kTcEpilogueWarps);
    }
    tc::fence_mbar_init();
    s_err = 0;
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, 2 * P::kCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTcEpilogueWarps && lane == 0 && mine > 0) {
    // ---- producer and MMA issuer
    const uint64_t pol = l2_evict_first();
    auto load = [&](int j) {
      tc::mbar_expect_tx(&full[j & 1], P::kABytes);
      tc::tma_load_5d_hint(sA + (j & 1) * P::kABytes, tmap, &full[j & 1], d0, head, 0,
                           (r + kCluster * j) * kTcCells, uw, pol);
    };
    load(0);
    if (mine > 1) load(1);
    constexpr uint32_t kIdesc = tc::idesc_bf16(128, L, true);
    bool ok = true;
    for (int j = 0; j < mine && ok; ++j) {
      const int st = j & 1;
      if (j >= 2) ok = tc::mbar_wait(&freed[st], ((j - 2) >> 1) & 1);     // accumulator st drained
      if (ok) ok = tc::mbar_wait(&full[st], (j >> 1) & 1);                 // tile j landed
      if (!ok) break;
      tc::fence_after_sync();
      const uint32_t a0 = tc::smem_u32(sA + st * P::kABytes), b0 = tc::smem_u32(sB);
      const uint32_t d = tmem + st * P::kCols;
      bool acc = false;
#pragma unroll
      for (int l = 0; l < 3; ++l)
#pragma unroll
        for (int ks = 0; ks < L / 16; ++ks) {
          tc::mma_bf16(d, tc::smem_desc(a0 + ks * 1024, L * 64, 512, 4),
                       tc::smem_desc(b0 + l * P::kBBytes + ks * 32, 16, 1024, 2), kIdesc, acc);
          acc = true;
        }
      tc::mma_commit(&done[st]);
      // the stage of tile j - 1 is free once its MMAs completed: refill it with tile j + 1
      if (j >= 1 && j + 1 < mine) {
        ok = tc::mbar_wait(&done[(j - 1) & 1], ((j - 1) >> 1) & 1);
        if (ok) load(j + 1);
      }
    }
    if (!ok) {
      s_err = 1;
      // bounded waits for the copies and MMAs that may still be in flight
      for (int i = 0; i < 2; ++i) {
        tc::mbar_wait(&full[i], 0);
        tc::mbar_wait(&done[i], 0);
      }
    }
  } else if (warp < kTcEpilogueWarps && mine > 0) {
    // ---- epilogue: warp w drains TMEM lanes 32 (w % 4).. (cell w % 4 of each tile), columns of
    //      half w / 4
    const int q = warp & 3, half = warp >> 2;
    for (int j = 0; j < mine; ++j) {
      const int st = j & 1;
      // (a warp vote keeps the warp converged for the .sync.aligned TMEM loads)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&done[st], (j >> 1) & 1))) {
        s_err = 1;
        break;
      }
      tc::fence_after_sync();
      const int cell = (r + kCluster * j) * kTcCells + q;
      float* yo = Y + ((size_t)u * L * HWX + cell) * nx + c0 + lane + (size_t)half * P::kHalf * HWX * nx;
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + st * P::kCols + half * P::kHalf;
      float v[P::kHalf];
      tc::tmem_ld<P::kHalf>(taddr, v);
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&freed[st]);   // the accumulator may take the next tile
      if (cell < HWX) {
#pragma unroll
        for (int k = 0; k < P::kHalf; ++k) yo[(size_t)k * HWX * nx] = v[k];
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const bool ok = s_err == 0;
  if (!ok && tid == 0) atomicCAS(status, 0u, (unsigned int)TACTKV_TIMEOUT);
  if (warp == 0) {
    __syncwarp();
    tc::tmem_free(tmem, 2 * P::kCols);
  }
  return ok;
}

// The fused forward kernel with the S pass on the tensor cores (bf16 input described by tmap).
template <int L, int HX, int WX, int NX>
__global__ void __launch_bounds__(kTcThreads, 3) fdct3_tc_kernel(const __grid_constant__ Geom g,
                                                                    const __grid_constant__ UnitList ul,
                                                                    float* __restrict__ Y, float* __restrict__ partial,
                                                                    const __grid_constant__ CUtensorMap tmap,
                                                                    unsigned int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_bars[6];
  __shared__ uint32_t s_tmem;
  unsigned char* smem =
      smem_raw + ((1024 - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // 1024-byte aligned (swizzle atoms)
  const int r = blockIdx.x, chunk = blockIdx.y, u = g.unit0 + blockIdx.z;
  const bool ok = fdct_s_tc<L, HX * WX>(g, u, chunk, r, &tmap, Y, smem, s_bars, &s_tmem, NX ? NX : g.n, status);
  cluster_barrier();   // the chunk's Y is complete
  if (!ok) return;     // (after the cluster barrier: no CTA of the cluster waits for this one)
  constexpr int spc = (L + kCluster - 1) / kCluster;
  const int ks0 = r * spc, ks1 = min(L, ks0 + spc);
  if (ks0 < ks1) fdct_hw_slabs<16, 16, HX, WX, true, NX>(g, Y, partial, u, chunk, ks0, ks1, smem);
}

template <class K, class... Args>
cudaError_t launch_cluster(K kernel, int threads, const Geom& g, int nu, size_t smem, cudaStream_t st, Args... args) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCluster, g.nch, nu);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kCluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Tensor map of the wave's bf16 inputs for the tensor-core S pass: 5-D (d, head, s, cell, unit),
// box (32, 1, S, 4 cells, 1) with 64-byte swizzle, so that a box lands as [cell][s][32 channels].
// Needs head_dim a multiple of 32 (a chunk inside one head), 16-byte aligned pointers and
// strides, and the wave's units equally spaced in memory with equal strides (one map for all);
// false otherwise (the caller then uses the cp.async S pass).
bool make_input_map(const Geom& g, const UnitList& ul, int nu, CUtensorMap* map) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!encode || (g.flags & TACTKV_FP32_IO) || has_variant(g.flags) || g.head_dim % kChunk != 0) return false;
  const UnitDev& a = ul.u[g.unit0];
  const long long tok = a.tok_stride, hs = a.head_stride;
  if (tok * 2 % 16 || hs * 2 % 16 || reinterpret_cast<uintptr_t>(a.in) % 16) return false;
  long long ustride = 16;
  if (nu > 1) ustride = static_cast<const char*>(ul.u[g.unit0 + 1].in) - static_cast<const char*>(a.in);
  if (ustride <= 0 || ustride % 16) return false;
  for (int i = 1; i < nu; ++i) {
    const UnitDev& b = ul.u[g.unit0 + i];
    if (b.tok_stride != tok || b.head_stride != hs ||
        static_cast<const char*>(b.in) - static_cast<const char*>(a.in) != (long long)i * ustride)
      return false;
  }
  const cuuint64_t dims[5] = {(cuuint64_t)g.head_dim, (cuuint64_t)g.heads, (cuuint64_t)g.S, (cuuint64_t)g.HW,
                              (cuuint64_t)nu};
  const cuuint64_t strides[4] = {(cuuint64_t)(hs * 2), (cuuint64_t)(g.HW * tok * 2), (cuuint64_t)(tok * 2),
                                 (cuuint64_t)ustride};
  const cuuint32_t box[5] = {(cuuint32_t)kChunk, 1u, (cuuint32_t)g.S, (cuuint32_t)kTcCells, 1u};
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(a.in), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int HX, int WX>
cudaError_t launch_grid(const Geom& g, const UnitList& ul, int nu, float* buf, float* partial, unsigned int* status,
                        cudaStream_t st) {
  constexpr int L = TACTKV_FUSED_S;
  const HwLayout Ls = hw_layout(HX, WX, kLayStats);
  const size_t regions[] = {Ls.tile, Ls.sbuf, Ls.meta, Ls.lv, Ls.tile_bytes};
  for (size_t x : regions)
    if (x % 16) return cudaErrorMisalignedAddress;   // never launch a misaligned layout
#if TACTKV_FUSED_S >= 16
  if constexpr (HX <= 16) {   // (the tensor-core form covers the 16-class grids)
  CUtensorMap map;
  if (tc_s_pass_enabled() && make_input_map(g, ul, nu, &map)) {
    const size_t smem = std::max<size_t>(TcS<L>::kSmem, Ls.total + 1024);
    if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    if (g.n == 1024)
      return launch_cluster(fdct3_tc_kernel<L, HX, WX, 1024>, kTcThreads, g, nu, smem, st, g, ul, buf, partial, map, status);
    if (g.n == 512)
      return launch_cluster(fdct3_tc_kernel<L, HX, WX, 512>, kTcThreads, g, nu, smem, st, g, ul, buf, partial, map, status);
    return launch_cluster(fdct3_tc_kernel<L, HX, WX, 0>, kTcThreads, g, nu, smem, st, g, ul, buf, partial, map, status);
  }
  }
#endif
  int nbuf = 1;
  const size_t smem = fused_fwd_smem<L>(HX, WX, (g.flags & TACTKV_FP32_IO) != 0, &nbuf);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  const int lg_cpr = input_pieces_lg(g, ul, g.unit0, nu);
  if (has_variant(g.flags))
    return launch_cluster(fdct3_kernel<L, HX, WX, 0, true>, kFusedThreads, g, nu, smem, st, g, ul, buf, partial, lg_cpr);
  if (g.n == 1024)
    return launch_cluster(fdct3_kernel<L, HX, WX, 1024, false>, kFusedThreads, g, nu, smem, st, g, ul, buf, partial, lg_cpr);
  if (g.n == 512)
    return launch_cluster(fdct3_kernel<L, HX, WX, 512, false>, kFusedThreads, g, nu, smem, st, g, ul, buf, partial, lg_cpr);
  return launch_cluster(fdct3_kernel<L, HX, WX, 0, false>, kFusedThreads, g, nu, smem, st, g, ul, buf, partial, lg_cpr);
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
// Fused forward transforms of one wave for the grids above (g.S == TACTKV_FUSED_S):
// x -> X in buf, energies in partial; cudaErrorNotSupported for any other grid.
cudaError_t TACTKV_CAT(launch_fused_, TACTKV_FUSED_S)(const Geom& g, const UnitList& ul, int nu, float* buf,
                                                      float* partial, unsigned int* status, cudaStream_t st) {
  if (g.S != TACTKV_FUSED_S) return cudaErrorNotSupported;
  if (g.H == 16 && g.W == 16) return launch_grid<16, 16>(g, ul, nu, buf, partial, status, st);
  if (g.H == 14 && g.W == 14) return launch_grid<14, 14>(g, ul, nu, buf, partial, status, st);
  if (g.H == 8 && g.W == 8) return launch_grid<8, 8>(g, ul, nu, buf, partial, status, st);
#if TACTKV_FUSED_S <= 32
  if (g.H == 24 && g.W == 24) return launch_grid<24, 24>(g, ul, nu, buf, partial, status, st);
#endif
  return cudaErrorNotSupported;
}

}  // namespace tactkv
