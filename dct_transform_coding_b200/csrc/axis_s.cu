// DCT along the S axis (TACT-KV stage 2, first of the three separable passes, and the last
// pass of decoding).  A CTA takes 32 channels x 4 grid cells x all S; it first stages that tile
// in shared memory with cp.async (all of its loads in flight at once, no registers held), then
// each thread owns the pencil of S values of one channel at one (h, w) cell in registers for
// the whole transform (one channel per thread keeps the register count low enough for 3-4 CTAs
// per SM; the fp32 pipe rate is the same as with packed pairs).  Each warp store writes 128
// contiguous bytes of the fp32 scratch.  The channel group is the fastest grid index, so the
// CTAs that read the same token rows run next to each other.
//
// Compiled once per length class (TACTKV_CLASS = 16, 32 or 64).
#include "common.cuh"

#ifndef TACTKV_CLASS
#error "TACTKV_CLASS must be defined"
#endif

namespace tactkv {
namespace {

constexpr int kWarps = 4;   // grid cells per CTA
constexpr int kMinBlocks = TACTKV_CLASS >= 64 ? 3 : 4;

// Stage the CTA's tile [S][kWarps cells][32 channels] of a strided bf16/fp32 input in shared
// memory with cp.async: every load of the tile is in flight at once and holds no registers.
// vec16: 16-byte copies are legal (pointer, strides and head_dim multiples of 16 bytes).
__device__ __forceinline__ void stage_input(const Geom& g, const UnitDev& ud, int hw0, int c0, bool fp32, bool vec16,
                                            unsigned char* tile) {
  const int esz = fp32 ? 4 : 2;
  const int cb = vec16 ? 16 : 4;                   // bytes per copy
  const int per_row = 32 * esz / cb;               // copies per (s, cell) row of 32 channels
  const int ch_per = cb / esz;                     // channels per copy
  const int total = g.S * kWarps * per_row;
  const unsigned char* in = static_cast<const unsigned char*>(ud.in);
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int s = i / (kWarps * per_row);
    const int r = i - s * (kWarps * per_row);
    const int hwl = r / per_row, q = r - hwl * per_row;
    const int hw = hw0 + hwl;
    if (hw >= g.HW) continue;
    const int c = c0 + q * ch_per;
    const int head = c / g.head_dim, d = c - head * g.head_dim;
    const long long e = ((long long)s * g.HW + hw) * ud.tok_stride + (long long)head * ud.head_stride + d;
    unsigned char* dst = tile + ((size_t)(s * kWarps + hwl) * 32 + q * ch_per) * esz;
    if (vec16) cp_async16(dst, in + e * esz);
    else cp_async4(dst, in + e * esz);
  }
  cp_async_commit();
}

// Forward: x (bf16 or fp32, strided) -> Y[u][k_s][hw][c] fp32.
template <int CLASS>
__global__ void __launch_bounds__(32 * kWarps, kMinBlocks) fdct_s_kernel(const __grid_constant__ Geom g,
                                                                         const __grid_constant__ UnitList ul,
                                                                         float* __restrict__ Y, bool vec16) {
  extern __shared__ __align__(16) unsigned char tile[];
  const int lane = threadIdx.x & 31, hwl = threadIdx.x >> 5;
  const int hw0 = blockIdx.y * kWarps, hw = hw0 + hwl;
  const int c0 = blockIdx.x * 32, c = c0 + lane;
  const int u = blockIdx.z;
  const UnitDev& ud = ul.u[u];
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  stage_input(g, ud, hw0, c0, fp32, vec16, tile);
  cp_async_wait_all();
  __syncthreads();
  if (hw >= g.HW) return;
  float v[CLASS];
  if (fp32) {
    const float* t = reinterpret_cast<const float*>(tile) + hwl * 32 + lane;
#pragma unroll
    for (int s = 0; s < CLASS; ++s)
      if (s < g.S) v[s] = t[s * kWarps * 32];
  } else {
    const __nv_bfloat16* t = reinterpret_cast<const __nv_bfloat16*>(tile) + hwl * 32 + lane;
#pragma unroll
    for (int s = 0; s < CLASS; ++s)
      if (s < g.S) v[s] = __bfloat162float(t[s * kWarps * 32]);
  }
  dct_pencil<CLASS, false>(v, g.S);
  float* yo = Y + ((size_t)u * g.S * g.HW + hw) * g.n + c;
  const size_t kstep = (size_t)g.HW * g.n;
#pragma unroll
  for (int k = 0; k < CLASS; ++k)
    if (k < g.S) yo[k * kstep] = v[k];
}

// Inverse: V[u][k_s][hw][c] fp32 -> x_hat (bf16, rounded to nearest even, or fp32), strided.
template <int CLASS>
__global__ void __launch_bounds__(32 * kWarps, kMinBlocks) idct_s_kernel(const __grid_constant__ Geom g,
                                                                         const __grid_constant__ UnitList ul,
                                                                         const float* __restrict__ V) {
  extern __shared__ __align__(16) unsigned char tile[];
  const int lane = threadIdx.x & 31, hwl = threadIdx.x >> 5;
  const int hw0 = blockIdx.y * kWarps, hw = hw0 + hwl;
  const int c0 = blockIdx.x * 32, c = c0 + lane;
  const int u = blockIdx.z;
  const UnitDev& ud = ul.u[u];
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  {  // tile [S][kWarps][32] fp32 of V: 128-byte rows, 8 copies of 16 bytes each
    float* t = reinterpret_cast<float*>(tile);
    const int total = g.S * kWarps * 8;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
      const int s = i / (kWarps * 8);
      const int r = i - s * (kWarps * 8);
      const int h = r >> 3, q = r & 7;
      if (hw0 + h >= g.HW) continue;
      cp_async16(t + (s * kWarps + h) * 32 + q * 4,
                 V + (((size_t)u * g.S + s) * g.HW + hw0 + h) * g.n + c0 + q * 4);
    }
    cp_async_commit();
  }
  cp_async_wait_all();
  __syncthreads();
  if (hw >= g.HW) return;
  float v[CLASS];
  const float* t = reinterpret_cast<const float*>(tile) + hwl * 32 + lane;
#pragma unroll
  for (int k = 0; k < CLASS; ++k)
    if (k < g.S) v[k] = t[k * kWarps * 32];
  dct_pencil<CLASS, true>(v, g.S);
  const long long base = (long long)hw * ud.tok_stride + (long long)(c / g.head_dim) * ud.head_stride + c % g.head_dim;
  const long long sstep = (long long)g.HW * ud.tok_stride;
#pragma unroll
  for (int s = 0; s < CLASS; ++s)
    if (s < g.S) store_one(ud.out, base + s * sstep, v[s], fp32);
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
cudaError_t TACTKV_CAT(launch_axis_s_, TACTKV_CLASS)(bool inverse, const Geom& g, const UnitList& ul, int nu,
                                                     float* buf, cudaStream_t st) {
  const dim3 grid(g.n / 32, (g.HW + kWarps - 1) / kWarps, nu);
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  if (inverse) {
    const size_t sm = (size_t)g.S * kWarps * 32 * 4;
    idct_s_kernel<TACTKV_CLASS><<<grid, 32 * kWarps, sm, st>>>(g, ul, buf);
  } else {
    // 16-byte copies need every unit's pointer, strides and head_dim on 16-byte boundaries
    const int esz = fp32 ? 4 : 2, per = 16 / esz;
    bool vec16 = g.head_dim % per == 0;
    for (int i = 0; i < nu && vec16; ++i)
      vec16 = reinterpret_cast<uintptr_t>(ul.u[i].in) % 16 == 0 && ul.u[i].tok_stride % per == 0 &&
              ul.u[i].head_stride % per == 0;
    const size_t sm = (size_t)g.S * kWarps * 32 * esz;
    fdct_s_kernel<TACTKV_CLASS><<<grid, 32 * kWarps, sm, st>>>(g, ul, buf, vec16);
  }
  return cudaGetLastError();
}

}  // namespace tactkv
