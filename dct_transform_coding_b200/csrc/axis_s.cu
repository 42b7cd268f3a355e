// DCT along the S axis (TACT-KV stage 2, first of the three separable passes, and the last
// pass of decoding).  One thread owns one pencil of S values of two adjacent channels at one
// (h, w) grid column and keeps it in registers for the whole transform; a warp covers
// 16 channel pairs x 2 columns, so every load or store instruction moves two full 64-byte rows.
//
// Compiled once per length class (TACTKV_CLASS = 16, 32 or 64).
#include "common.cuh"

#ifndef TACTKV_CLASS
#error "TACTKV_CLASS must be defined"
#endif

namespace tactkv {
namespace {

// Forward: x (bf16 or fp32, strided) -> Y[u][k_s][hw][c] fp32.
template <int CLASS>
__global__ void __launch_bounds__(128) fdct_s_kernel(const __grid_constant__ Geom g,
                                                     const __grid_constant__ UnitList ul, float* __restrict__ Y) {
  const int pair = threadIdx.x & 15;
  const int hw = blockIdx.x * 8 + (threadIdx.x >> 4);
  const int u = blockIdx.z;
  if (hw >= g.HW) return;
  const int c = blockIdx.y * kChunk + 2 * pair;
  const int head = c / g.head_dim, d = c - head * g.head_dim;
  const UnitDev& ud = ul.u[u];
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  const long long base = (long long)hw * ud.tok_stride + (long long)head * ud.head_stride + d;
  const long long sstep = (long long)g.HW * ud.tok_stride;
  float2 v[CLASS];
#pragma unroll
  for (int s = 0; s < CLASS; ++s)
    if (s < g.S) v[s] = load_pair(ud.in, base + s * sstep, fp32);
  dct_pencil<CLASS, false>(v, g.S);
  float2* yo = reinterpret_cast<float2*>(Y + ((size_t)u * g.S * g.HW + hw) * g.n + c);
  const size_t kstep = (size_t)g.HW * g.n / 2;
#pragma unroll
  for (int k = 0; k < CLASS; ++k)
    if (k < g.S) yo[k * kstep] = v[k];
}

// Inverse: V[u][k_s][hw][c] fp32 -> x_hat (bf16, rounded to nearest even, or fp32), strided.
template <int CLASS>
__global__ void __launch_bounds__(128) idct_s_kernel(const __grid_constant__ Geom g,
                                                     const __grid_constant__ UnitList ul, const float* __restrict__ V) {
  const int pair = threadIdx.x & 15;
  const int hw = blockIdx.x * 8 + (threadIdx.x >> 4);
  const int u = blockIdx.z;
  if (hw >= g.HW) return;
  const int c = blockIdx.y * kChunk + 2 * pair;
  const int head = c / g.head_dim, d = c - head * g.head_dim;
  const UnitDev& ud = ul.u[u];
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  const float2* vi = reinterpret_cast<const float2*>(V + ((size_t)u * g.S * g.HW + hw) * g.n + c);
  const size_t kstep = (size_t)g.HW * g.n / 2;
  float2 v[CLASS];
#pragma unroll
  for (int k = 0; k < CLASS; ++k)
    if (k < g.S) v[k] = vi[k * kstep];
  dct_pencil<CLASS, true>(v, g.S);
  const long long base = (long long)hw * ud.tok_stride + (long long)head * ud.head_stride + d;
  const long long sstep = (long long)g.HW * ud.tok_stride;
#pragma unroll
  for (int s = 0; s < CLASS; ++s)
    if (s < g.S) store_pair(ud.out, base + s * sstep, v[s], fp32);
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
cudaError_t TACTKV_CAT(launch_axis_s_, TACTKV_CLASS)(bool inverse, const Geom& g, const UnitList& ul, int nu,
                                                     float* buf, cudaStream_t st) {
  const dim3 grid((g.HW + 7) / 8, g.nch, nu);
  if (inverse) idct_s_kernel<TACTKV_CLASS><<<grid, 128, 0, st>>>(g, ul, buf);
  else fdct_s_kernel<TACTKV_CLASS><<<grid, 128, 0, st>>>(g, ul, buf);
  return cudaGetLastError();
}

}  // namespace tactkv
