// DCT along the S axis (TACT-KV stage 2, first of the three separable passes, and the last pass
// of decoding).  A CTA takes 32 channels x 4 grid cells x all S; it stages that tile in shared
// memory with cp.async (every load of the tile in flight at once, no registers held), then each
// thread owns the pencil of S values of one channel at one (h, w) cell in registers for the whole
// transform.  Each warp store writes 128 contiguous bytes of the fp32 volume.  The channel group
// is the fastest grid index, so the CTAs that read the same token rows run next to each other.
//
// Kernels are instantiated per exact length S (straight-line transform, no bounds tests inside
// the pencil); this file is compiled once per length class (TACTKV_CLASS = 16, 32 or 64).
#include "axis_s.cuh"

#ifndef TACTKV_CLASS
#error "TACTKV_CLASS must be defined"
#endif

namespace tactkv {
namespace {

constexpr int kCells = 4;   // grid cells per CTA, one warp each
constexpr int kThreads = STile<kCells>::kThreads;
constexpr int kMinBlocks = 4;

// Forward: x (bf16 or fp32, strided) -> Y[u][k_s][hw][c] fp32.
template <int L, bool VAR>
__global__ void __launch_bounds__(kThreads, kMinBlocks) fdct_s_kernel(const __grid_constant__ Geom g,
                                                                      const __grid_constant__ UnitList ul,
                                                                      float* __restrict__ Y, int lg_cpr) {
  extern __shared__ __align__(16) unsigned char tile[];
  const int hw0 = blockIdx.y * kCells, c0 = blockIdx.x * 32, u = g.unit0 + blockIdx.z;
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  stage_input<L, kCells, false>(g, ul.u[u], hw0, c0, fp32 ? 4 : 2, lg_cpr, tile);
  cp_async_wait_all();
  __syncthreads();
  fdct_s_cells<L, kCells, 0, 0, VAR>(g, u, hw0, c0, tile, fp32, Y);
}

// Inverse: V[u][k_s][hw][c] fp32 -> x_hat (bf16, rounded to nearest even, or fp32), strided.
template <int L, bool VAR>
__global__ void __launch_bounds__(kThreads, kMinBlocks) idct_s_kernel(const __grid_constant__ Geom g,
                                                                      const __grid_constant__ UnitList ul,
                                                                      const float* __restrict__ V) {
  extern __shared__ __align__(16) float vtile[];   // [L][kCells][32]
  const int hw0 = blockIdx.y * kCells, c0 = blockIdx.x * 32, u = g.unit0 + blockIdx.z;
  stage_volume<L, kCells>(g, u, hw0, c0, V, vtile);
  cp_async_wait_all();
  __syncthreads();
  drop_volume<L, kCells>(g, u, hw0, c0, V);
  idct_s_cells<L, kCells, VAR>(g, ul.u[u], hw0, c0, vtile);
}

template <int L>
cudaError_t launch_len(bool inverse, const Geom& g, const UnitList& ul, int nu, float* buf, cudaStream_t st) {
  const dim3 grid(g.n / 32, (g.HW + kCells - 1) / kCells, nu);
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  const bool var = has_variant(g.flags);
  if (inverse) {
    const size_t sm = (size_t)L * kCells * 32 * 4;
    if (var) idct_s_kernel<L, true><<<grid, kThreads, sm, st>>>(g, ul, buf);
    else idct_s_kernel<L, false><<<grid, kThreads, sm, st>>>(g, ul, buf);
  } else {
    const size_t sm = (size_t)L * kCells * 32 * (fp32 ? 4 : 2);
    const int lg = input_pieces_lg(g, ul, g.unit0, nu);
    if (var) fdct_s_kernel<L, true><<<grid, kThreads, sm, st>>>(g, ul, buf, lg);
    else fdct_s_kernel<L, false><<<grid, kThreads, sm, st>>>(g, ul, buf, lg);
  }
  return cudaGetLastError();
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
#define TACTKV_LEN(n) \
  case n:             \
    return launch_len<n>(inverse, g, ul, nu, buf, st);
cudaError_t TACTKV_CAT(launch_axis_s_, TACTKV_CLASS)(bool inverse, const Geom& g, const UnitList& ul, int nu,
                                                     float* buf, cudaStream_t st) {
  switch (g.S) {
#if TACTKV_CLASS == 16
    TACTKV_LEN(1) TACTKV_LEN(2) TACTKV_LEN(3) TACTKV_LEN(4) TACTKV_LEN(5) TACTKV_LEN(6) TACTKV_LEN(7)
    TACTKV_LEN(8) TACTKV_LEN(9) TACTKV_LEN(10) TACTKV_LEN(11) TACTKV_LEN(12) TACTKV_LEN(13) TACTKV_LEN(14)
    TACTKV_LEN(15) TACTKV_LEN(16)
#elif TACTKV_CLASS == 32
    TACTKV_LEN(20) TACTKV_LEN(24) TACTKV_LEN(28) TACTKV_LEN(32)
#else
    TACTKV_LEN(40) TACTKV_LEN(48) TACTKV_LEN(56) TACTKV_LEN(64)
#endif
    default: return cudaErrorInvalidValue;
  }
}
#undef TACTKV_LEN

}  // namespace tactkv
