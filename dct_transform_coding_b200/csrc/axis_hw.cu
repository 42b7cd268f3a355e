// Kernels for the DCT along the H and W axes with the per-bin energies, and for its inverse with
// unpacking and dequantization; each CTA walks one range of S slabs of one (unit, 32-channel
// chunk) with the pieces of axis_hw.cuh.
//
// Compiled once per pair of length classes (TACTKV_HCLASS, TACTKV_WCLASS: 16 or 32 each).
#include "axis_hw.cuh"

#if !defined(TACTKV_HCLASS) || !defined(TACTKV_WCLASS)
#error "TACTKV_HCLASS and TACTKV_WCLASS must be defined"
#endif

namespace tactkv {
namespace {

// Register budget: class-16 pencils fit two CTAs of 256 threads per SM; the generic class-32
// float2 pencils need more than 128 registers, the exact 24 x 24 ones fit two CTAs per SM.
constexpr int kHwMinBlocks = (TACTKV_HCLASS == 16 && TACTKV_WCLASS == 16) ? 2 : 1;
// The exact-size class-16 inverse kernels fit 64 registers without spilling: four CTAs per SM.
template <int HX>
constexpr int hw_min_blocks_inv() { return (TACTKV_HCLASS == 16 && TACTKV_WCLASS == 16) ? (HX > 0 ? 4 : 2) : (HX > 0 ? 2 : 1); }

template <int HC, int WC, int HX, int WX, bool VAR>
__global__ void __launch_bounds__(kMaxHwThreads, (HX > 0 ? 2 : kHwMinBlocks)) fdct_hw_kernel(const __grid_constant__ Geom g,
                                                                              const __grid_constant__ UnitList ul,
                                                                              float* __restrict__ Y,
                                                                              float* __restrict__ partial, int spc) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int ks0 = blockIdx.y * spc;
  fdct_hw_slabs<HC, WC, HX, WX, false, 0, VAR>(g, Y, partial, g.unit0 + blockIdx.z, blockIdx.x, ks0,
                                               min(g.S, ks0 + spc), smem);
}

// NX: the channel count when fixed at compile time (512 or 1024, the exact grids' plain decode), else 0.
template <int HC, int WC, int HX, int WX, int MODE, bool VAR, int NX = 0>
__global__ void __launch_bounds__(kMaxHwThreads, hw_min_blocks_inv<HX>()) idct_hw_kernel(const __grid_constant__ Geom g,
                                                                                         const __grid_constant__ UnitList ul,
                                                                                         float* __restrict__ V,
                                                                                         const uint32_t* __restrict__ index,
                                                                                         const uint4* __restrict__ recs,
                                                                                         int spc) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int ks0 = blockIdx.y * spc;
  idct_hw_slabs<HC, WC, HX, WX, MODE, false, VAR, NX>(g, ul, V, index, recs, g.unit0 + blockIdx.z, blockIdx.x, ks0,
                                                      min(g.S, ks0 + spc), smem);
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
#define TACTKV_HWNAME(base) TACTKV_CAT(TACTKV_CAT(TACTKV_CAT(base, TACTKV_HCLASS), _), TACTKV_WCLASS)
namespace {
template <int HX, int WX>
cudaError_t launch_hw(bool inverse, int mode, const Geom& g, const UnitList& ul, int nu, float* buf, float* partial,
                      const uint32_t* slab_off, const uint4* recs, int spc, cudaStream_t st) {
  const HwLayout L = hw_layout(g.H, g.W, inverse ? kLayDecode : kLayStats);
  const dim3 grid(g.nch, (g.S + spc - 1) / spc, nu);
  const int threads = hw_threads(g.H, g.W);
  constexpr int H = TACTKV_HCLASS, W = TACTKV_WCLASS;
  const int sm = (int)L.total;
  const size_t regions[] = {L.tile, L.sbuf, L.meta, L.sig, L.lv, L.bsl, L.tile_bytes, L.bsl_stride};
  for (size_t r : regions)
    if (r % 16) return cudaErrorMisalignedAddress;   // never launch a misaligned layout
  if (L.total > 227 * 1024) return cudaErrorInvalidConfiguration;
#define TACTKV_GO(kern, ...)                                                           \
  do {                                                                                 \
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);       \
    kern<<<grid, threads, sm, st>>>(__VA_ARGS__);                                      \
  } while (0)
  const bool var = has_variant(g.flags);
  if (inverse) {
    if (mode == kRaw) {
      if (var) TACTKV_GO((idct_hw_kernel<H, W, HX, WX, kRaw, true>), g, ul, buf, slab_off, recs, spc);
      else TACTKV_GO((idct_hw_kernel<H, W, HX, WX, kRaw, false>), g, ul, buf, slab_off, recs, spc);
    } else {
      if (var) TACTKV_GO((idct_hw_kernel<H, W, HX, WX, kQuant, true>), g, ul, buf, slab_off, recs, spc);
      else if (HX > 0 && g.n == 1024) TACTKV_GO((idct_hw_kernel<H, W, HX, WX, kQuant, false, HX ? 1024 : 0>), g, ul, buf, slab_off, recs, spc);
      else if (HX > 0 && g.n == 512) TACTKV_GO((idct_hw_kernel<H, W, HX, WX, kQuant, false, HX ? 512 : 0>), g, ul, buf, slab_off, recs, spc);
      else TACTKV_GO((idct_hw_kernel<H, W, HX, WX, kQuant, false>), g, ul, buf, slab_off, recs, spc);
    }
  } else {
    if (var) TACTKV_GO((fdct_hw_kernel<H, W, HX, WX, true>), g, ul, buf, partial, spc);
    else TACTKV_GO((fdct_hw_kernel<H, W, HX, WX, false>), g, ul, buf, partial, spc);
  }
#undef TACTKV_GO
  return cudaGetLastError();
}
}  // namespace

// The grids of the common layouts (medical volumes 16x16 and 24x24, video frames 14x14, the 8x8
// test volume) have their own exact-size kernels; every other grid of the class runs the generic one.
cudaError_t TACTKV_HWNAME(launch_axis_hw_)(bool inverse, int mode, const Geom& g, const UnitList& ul, int nu, float* buf,
                                           float* partial, const uint32_t* slab_off, const uint4* recs, int spc,
                                           cudaStream_t st) {
#if TACTKV_HCLASS == 16 && TACTKV_WCLASS == 16
  if (g.H == 16 && g.W == 16) return launch_hw<16, 16>(inverse, mode, g, ul, nu, buf, partial, slab_off, recs, spc, st);
  if (g.H == 14 && g.W == 14) return launch_hw<14, 14>(inverse, mode, g, ul, nu, buf, partial, slab_off, recs, spc, st);
  if (g.H == 8 && g.W == 8) return launch_hw<8, 8>(inverse, mode, g, ul, nu, buf, partial, slab_off, recs, spc, st);
#elif TACTKV_HCLASS == 32 && TACTKV_WCLASS == 32
  if (g.H == 24 && g.W == 24) return launch_hw<24, 24>(inverse, mode, g, ul, nu, buf, partial, slab_off, recs, spc, st);
#endif
  return launch_hw<0, 0>(inverse, mode, g, ul, nu, buf, partial, slab_off, recs, spc, st);
}

// Shared memory and threads of one CTA (host queries used to size the slab ranges).
void TACTKV_HWNAME(axis_hw_shape_)(const Geom& g, bool inverse, int mode, size_t* smem, int* threads) {
  *smem = hw_layout(g.H, g.W, inverse ? kLayDecode : kLayStats).total;
  *threads = hw_threads(g.H, g.W);
}

}  // namespace tactkv
