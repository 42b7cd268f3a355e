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
// The common grids (16x16, 14x14, 8x8) with S = 8, 16, 32 or 64 have a fused kernel; this file is
// compiled once per S (TACTKV_FUSED_S).  Other shapes use the separate S-axis and H/W-axis
// kernels.
#include "axis_s.cuh"
#include "axis_hw.cuh"

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
// reads after it.
__device__ __forceinline__ void cluster_barrier() {
  __threadfence();
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

// NX: the channel count when fixed at compile time (the common 512 and 1024), else 0.
template <int L, int HX, int WX, int NX>
__global__ void __launch_bounds__(kFusedThreads, 3) fdct3_kernel(const __grid_constant__ Geom g,
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
    fdct_s_cells<L, kNC, HX * WX, NX>(g, u, t * kNC, c0, smem + buf * tb, fp32, Y);
    __syncthreads();   // the tile's buffer is free again
    if (nbuf == 2) buf ^= 1;
    else if (next) stage_input<L, kNC, true>(g, ud, (t + kCluster) * kNC, c0, esz, lg_cpr, smem);
  }
  cluster_barrier();   // the chunk's Y is complete
  // DCT along H and W on this CTA's range of slabs
  constexpr int spc = (L + kCluster - 1) / kCluster;
  const int ks0 = r * spc, ks1 = min(L, ks0 + spc);
  if (ks0 < ks1) fdct_hw_slabs<16, 16, HX, WX, true, NX>(g, Y, partial, u, chunk, ks0, ks1, smem);
}

template <class K, class... Args>
cudaError_t launch_cluster(K kernel, const Geom& g, int nu, size_t smem, cudaStream_t st, Args... args) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCluster, g.nch, nu);
  cfg.blockDim = dim3(kFusedThreads, 1, 1);
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

template <int HX, int WX>
cudaError_t launch_grid(const Geom& g, const UnitList& ul, int nu, float* buf, float* partial, cudaStream_t st) {
  constexpr int L = TACTKV_FUSED_S;
  const HwLayout Ls = hw_layout(HX, WX, kLayStats);
  const size_t regions[] = {Ls.tile, Ls.sbuf, Ls.meta, Ls.lv, Ls.tile_bytes};
  for (size_t x : regions)
    if (x % 16) return cudaErrorMisalignedAddress;   // never launch a misaligned layout
  int nbuf = 1;
  const size_t smem = fused_fwd_smem<L>(HX, WX, (g.flags & TACTKV_FP32_IO) != 0, &nbuf);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  const int lg_cpr = input_pieces_lg(g, ul, g.unit0, nu);
  if (g.n == 1024) return launch_cluster(fdct3_kernel<L, HX, WX, 1024>, g, nu, smem, st, g, ul, buf, partial, lg_cpr);
  if (g.n == 512) return launch_cluster(fdct3_kernel<L, HX, WX, 512>, g, nu, smem, st, g, ul, buf, partial, lg_cpr);
  return launch_cluster(fdct3_kernel<L, HX, WX, 0>, g, nu, smem, st, g, ul, buf, partial, lg_cpr);
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
// Fused forward transforms of one wave for the grids above (g.S == TACTKV_FUSED_S):
// x -> X in buf, energies in partial; cudaErrorNotSupported for any other grid.
cudaError_t TACTKV_CAT(launch_fused_, TACTKV_FUSED_S)(const Geom& g, const UnitList& ul, int nu, float* buf,
                                                      float* partial, cudaStream_t st) {
  if (g.S != TACTKV_FUSED_S) return cudaErrorNotSupported;
  if (g.H == 16 && g.W == 16) return launch_grid<16, 16>(g, ul, nu, buf, partial, st);
  if (g.H == 14 && g.W == 14) return launch_grid<14, 14>(g, ul, nu, buf, partial, st);
  if (g.H == 8 && g.W == 8) return launch_grid<8, 8>(g, ul, nu, buf, partial, st);
  return cudaErrorNotSupported;
}

}  // namespace tactkv
