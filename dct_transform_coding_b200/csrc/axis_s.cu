// DCT along the S axis (TACT-KV stage 2, first of the three separable passes, and the last pass
// of decoding).  A CTA takes 32 channels x 4 grid cells x all S; it stages that tile in shared
// memory with cp.async (every load of the tile in flight at once, no registers held), then each
// thread owns the pencil of S values of one channel at one (h, w) cell in registers for the whole
// transform.  Each warp store writes 128 contiguous bytes of the fp32 volume.  The channel group
// is the fastest grid index, so the CTAs that read the same token rows run next to each other.
//
// Kernels are instantiated per exact length S (straight-line transform, no bounds tests inside
// the pencil); this file is compiled once per length class (TACTKV_CLASS = 16, 32 or 64).
#include "common.cuh"

#ifndef TACTKV_CLASS
#error "TACTKV_CLASS must be defined"
#endif

namespace tactkv {
namespace {

constexpr int kCells = 4;   // grid cells per CTA, one warp each
constexpr int kThreads = 32 * kCells;
constexpr int kMinBlocks = 4;

// Stage the tile [S][4 cells][32 channels] of a strided bf16/fp32 input.  A row of one cell holds
// 32 channels = 2^lg_cpr copies of cb bytes; thread t copies piece (t mod 2^lg_cpr) of cell
// (t >> lg_cpr) mod 4 for s = t >> (lg_cpr + 2), then every (128 >> (lg_cpr + 2))-th s after it.
template <int L>
__device__ __forceinline__ void stage_input(const Geom& g, const UnitDev& ud, int hw0, int c0, int esz, int lg_cpr,
                                            unsigned char* tile) {
  const int cpr = 1 << lg_cpr, cb = (32 * esz) >> lg_cpr, ch_per = cb / esz;
  const int q = threadIdx.x & (cpr - 1), cl = (threadIdx.x >> lg_cpr) & (kCells - 1);
  const int s0 = threadIdx.x >> (lg_cpr + 2), ds = kThreads >> (lg_cpr + 2);
  if (hw0 + cl < g.HW && s0 < L) {
    const int c = c0 + q * ch_per;
    const int head = c / g.head_dim, d = c - head * g.head_dim;
    const unsigned char* src = static_cast<const unsigned char*>(ud.in) +
                               (((long long)s0 * g.HW + hw0 + cl) * ud.tok_stride + (long long)head * ud.head_stride + d) * esz;
    const long long sstep = (long long)ds * g.HW * ud.tok_stride * esz;
    unsigned char* dst = tile + ((s0 * kCells + cl) * 32 + q * ch_per) * esz;
    const int dstep = ds * kCells * 32 * esz;
    if (cb == 16) {
      for (int s = s0; s < L; s += ds, src += sstep, dst += dstep) cp_async16(dst, src);
    } else {
      for (int s = s0; s < L; s += ds, src += sstep, dst += dstep) cp_async4(dst, src);
    }
  }
  cp_async_commit();
}

// Forward: x (bf16 or fp32, strided) -> Y[u][k_s][hw][c] fp32.
template <int L>
__global__ void __launch_bounds__(kThreads, kMinBlocks) fdct_s_kernel(const __grid_constant__ Geom g,
                                                                      const __grid_constant__ UnitList ul,
                                                                      float* __restrict__ Y, int lg_cpr) {
  extern __shared__ __align__(16) unsigned char tile[];
  const int lane = threadIdx.x & 31, hwl = threadIdx.x >> 5;
  const int hw0 = blockIdx.y * kCells, hw = hw0 + hwl;
  const int c0 = blockIdx.x * 32;
  const int u = g.unit0 + blockIdx.z;
  const UnitDev& ud = ul.u[u];
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  stage_input<L>(g, ud, hw0, c0, fp32 ? 4 : 2, lg_cpr, tile);
  cp_async_wait_all();
  __syncthreads();
  if (hw >= g.HW) return;
  float v[L];
  if (fp32) {
    const float* t = reinterpret_cast<const float*>(tile) + hwl * 32 + lane;
#pragma unroll
    for (int s = 0; s < L; ++s) v[s] = t[s * kCells * 32];
  } else {
    const __nv_bfloat16* t = reinterpret_cast<const __nv_bfloat16*>(tile) + hwl * 32 + lane;
#pragma unroll
    for (int s = 0; s < L; ++s) v[s] = __bfloat162float(t[s * kCells * 32]);
  }
  dct_exact<L, false>(v);
  float* yo = Y + ((size_t)u * L * g.HW + hw) * g.n + c0 + lane;
  const size_t kstep = (size_t)g.HW * g.n;
#pragma unroll
  for (int k = 0; k < L; ++k) yo[k * kstep] = v[k];
}

// Inverse: V[u][k_s][hw][c] fp32 -> x_hat (bf16, rounded to nearest even, or fp32), strided.
template <int L>
__global__ void __launch_bounds__(kThreads, kMinBlocks) idct_s_kernel(const __grid_constant__ Geom g,
                                                                      const __grid_constant__ UnitList ul,
                                                                      const float* __restrict__ V) {
  extern __shared__ __align__(16) float vtile[];   // [L][kCells][32]
  const int lane = threadIdx.x & 31, hwl = threadIdx.x >> 5;
  const int hw0 = blockIdx.y * kCells, hw = hw0 + hwl;
  const int c0 = blockIdx.x * 32;
  const int u = g.unit0 + blockIdx.z;
  const UnitDev& ud = ul.u[u];
  {  // 128-byte rows of 32 channels, 8 copies of 16 bytes each; 4 values of s per pass
    const int q = threadIdx.x & 7, cl = (threadIdx.x >> 3) & 3, s0 = threadIdx.x >> 5;
    if (hw0 + cl < g.HW && s0 < L) {
      const float* src = V + (((size_t)u * L + s0) * g.HW + hw0 + cl) * g.n + c0 + 4 * q;
      const size_t sstep = (size_t)4 * g.HW * g.n;
      float* dst = vtile + (s0 * kCells + cl) * 32 + 4 * q;
      for (int s = s0; s < L; s += 4, src += sstep, dst += 4 * kCells * 32) cp_async16(dst, src);
    }
    cp_async_commit();
  }
  cp_async_wait_all();
  __syncthreads();
  {  // V is dead once staged: drop its lines from L2 without writing them back to memory
    const int q = threadIdx.x & 7, cl = (threadIdx.x >> 3) & 3, s0 = threadIdx.x >> 5;
    if (q == 0 && hw0 + cl < g.HW && s0 < L) {
      const float* src = V + (((size_t)u * L + s0) * g.HW + hw0 + cl) * g.n + c0;
      const size_t sstep = (size_t)4 * g.HW * g.n;
      for (int s = s0; s < L; s += 4, src += sstep) discard_l2_line(src);
    }
  }
  if (hw >= g.HW) return;
  float v[L];
  const float* t = vtile + hwl * 32 + lane;
#pragma unroll
  for (int k = 0; k < L; ++k) v[k] = t[k * kCells * 32];
  dct_exact<L, true>(v);
  const int c = c0 + lane, head = c / g.head_dim, d = c - head * g.head_dim;
  const long long base = (long long)hw * ud.tok_stride + (long long)head * ud.head_stride + d;
  const long long sstep = (long long)g.HW * ud.tok_stride;
  if (g.flags & TACTKV_FP32_IO) {
    float* o = static_cast<float*>(ud.out) + base;
#pragma unroll
    for (int s = 0; s < L; ++s) o[s * sstep] = v[s];
  } else {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(ud.out) + base;
#pragma unroll
    for (int s = 0; s < L; ++s) o[s * sstep] = __float2bfloat16_rn(v[s]);
  }
}

template <int L>
cudaError_t launch_len(bool inverse, const Geom& g, const UnitList& ul, int nu, float* buf, cudaStream_t st) {
  const dim3 grid(g.n / 32, (g.HW + kCells - 1) / kCells, nu);
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  if (inverse) {
    const size_t sm = (size_t)L * kCells * 32 * 4;
    idct_s_kernel<L><<<grid, kThreads, sm, st>>>(g, ul, buf);
  } else {
    // 16-byte copies need every unit's pointer, strides and head_dim on 16-byte boundaries
    const int esz = fp32 ? 4 : 2, per = 16 / esz;
    bool vec16 = g.head_dim % per == 0;
    for (int i = g.unit0; i < g.unit0 + nu && vec16; ++i)
      vec16 = reinterpret_cast<uintptr_t>(ul.u[i].in) % 16 == 0 && ul.u[i].tok_stride % per == 0 &&
              ul.u[i].head_stride % per == 0;
    // copies per 32-channel row: 64 or 128 bytes in pieces of 16 or 4 bytes
    const int lg_cpr = (fp32 ? 3 : 2) + (vec16 ? 0 : 2);
    const size_t sm = (size_t)L * kCells * 32 * esz;
    fdct_s_kernel<L><<<grid, kThreads, sm, st>>>(g, ul, buf, lg_cpr);
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
