// Pieces of the DCT along the S axis (TACT-KV stage 2, first of the three separable passes, and
// the last pass of decoding), shared by the S-axis kernels and the fused three-axis kernels.
//
// A tile is 32 channels x NC grid cells x all S values, staged in shared memory as [S][NC][32]
// with cp.async (every load of the tile in flight at once, no registers held).  Warp w then owns
// cell w of the tile: lane l holds the pencil of S values of channel l in registers for the whole
// transform, and each warp store writes 128 contiguous bytes of the fp32 volume [k_s][hw][c].
// The functions are called by NC * 32 threads.
#pragma once
#include "common.cuh"

namespace tactkv {
namespace {

template <int NC>
struct STile {
  static_assert(NC == 4 || NC == 8, "tiles of 4 or 8 cells");
  static constexpr int kThreads = 32 * NC;
  static constexpr int kLg = NC == 8 ? 3 : 2;
};

// Stage the input tile [S][NC cells][32 channels] of a strided bf16/fp32 input.  A row of one
// cell holds 32 channels = 2^lg_cpr copies of cb bytes; thread t copies piece (t mod 2^lg_cpr) of
// cell (t >> lg_cpr) mod NC for s = t >> (lg_cpr + lg NC), then every s a whole block further on.
// EF: the loads are marked evict-first in L2 (the input is read once).
template <int L, int NC, bool EF>
__device__ __forceinline__ void stage_input(const Geom& g, const UnitDev& ud, int hw0, int c0, int esz, int lg_cpr,
                                            unsigned char* tile) {
  const int cpr = 1 << lg_cpr, cb = (32 * esz) >> lg_cpr, ch_per = cb / esz;
  const int q = threadIdx.x & (cpr - 1), cl = (threadIdx.x >> lg_cpr) & (NC - 1);
  const int s0 = threadIdx.x >> (lg_cpr + STile<NC>::kLg), ds = STile<NC>::kThreads >> (lg_cpr + STile<NC>::kLg);
  if (hw0 + cl < g.HW && s0 < L) {
    const int c = c0 + q * ch_per;
    const int head = c / g.head_dim, d = c - head * g.head_dim;
    const unsigned char* src = static_cast<const unsigned char*>(ud.in) +
                               (((long long)s0 * g.HW + hw0 + cl) * ud.tok_stride + (long long)head * ud.head_stride + d) * esz;
    const long long sstep = (long long)ds * g.HW * ud.tok_stride * esz;
    unsigned char* dst = tile + ((s0 * NC + cl) * 32 + q * ch_per) * esz;
    const int dstep = ds * NC * 32 * esz;
    if constexpr (EF) {
      const uint64_t pol = l2_evict_first();
      if (cb == 16) {
        for (int s = s0; s < L; s += ds, src += sstep, dst += dstep) cp_async16_ef(dst, src, pol);
      } else {
        for (int s = s0; s < L; s += ds, src += sstep, dst += dstep) cp_async4_ef(dst, src, pol);
      }
    } else {
      if (cb == 16) {
        for (int s = s0; s < L; s += ds, src += sstep, dst += dstep) cp_async16(dst, src);
      } else {
        for (int s = s0; s < L; s += ds, src += sstep, dst += dstep) cp_async4(dst, src);
      }
    }
  }
  cp_async_commit();
}

// Forward pencils of a staged input tile: cell hw0 + warp -> Y[u][k_s][hw][c0 + lane], fp32.
// HWX, NX > 0 fix H*W and the channel count n at compile time (constant strides).
template <int L, int NC, int HWX = 0, int NX = 0, bool VAR = false>
__device__ __forceinline__ void fdct_s_cells(const Geom& g, int u, int hw0, int c0, const unsigned char* tile,
                                             bool fp32, float* __restrict__ Y) {
  const int lane = threadIdx.x & 31, hwl = threadIdx.x >> 5, hw = hw0 + hwl;
  const int HW = HWX ? HWX : g.HW, n = NX ? NX : g.n;
  if (hw >= HW) return;
  float v[L];
  if (fp32) {
    const float* t = reinterpret_cast<const float*>(tile) + hwl * 32 + lane;
#pragma unroll
    for (int s = 0; s < L; ++s) v[s] = t[s * NC * 32];
  } else {
    const __nv_bfloat16* t = reinterpret_cast<const __nv_bfloat16*>(tile) + hwl * 32 + lane;
#pragma unroll
    for (int s = 0; s < L; ++s) v[s] = __bfloat162float(t[s * NC * 32]);
  }
  if (!VAR || !(g.flags & TACTKV_SKIP_S)) dct_exact<L, false>(v);
  float* yo = Y + ((size_t)u * L * HW + hw) * n + c0 + lane;
  const size_t kstep = (size_t)HW * n;
#pragma unroll
  for (int k = 0; k < L; ++k) yo[k * kstep] = v[k];
}

// Stage the tile [L][NC cells][32 channels] of the fp32 volume V: 128-byte rows of 32 channels,
// 8 copies of 16 bytes each; 4 values of s per pass.
template <int L, int NC>
__device__ __forceinline__ void stage_volume(const Geom& g, int u, int hw0, int c0, const float* V, float* vtile) {
  const int q = threadIdx.x & 7, cl = (threadIdx.x >> 3) & (NC - 1), s0 = threadIdx.x >> (3 + STile<NC>::kLg);
  if (hw0 + cl < g.HW && s0 < L) {
    const float* src = V + (((size_t)u * L + s0) * g.HW + hw0 + cl) * g.n + c0 + 4 * q;
    const size_t sstep = (size_t)4 * g.HW * g.n;
    float* dst = vtile + (s0 * NC + cl) * 32 + 4 * q;
    for (int s = s0; s < L; s += 4, src += sstep, dst += 4 * NC * 32) cp_async16(dst, src);
  }
  cp_async_commit();
}

// Once a volume tile is staged (after the block barrier), its lines are dead: drop them from L2
// without writing them back to memory.
template <int L, int NC>
__device__ __forceinline__ void drop_volume(const Geom& g, int u, int hw0, int c0, const float* V) {
  const int q = threadIdx.x & 7, cl = (threadIdx.x >> 3) & (NC - 1), s0 = threadIdx.x >> (3 + STile<NC>::kLg);
  if (q == 0 && hw0 + cl < g.HW && s0 < L) {
    const float* src = V + (((size_t)u * L + s0) * g.HW + hw0 + cl) * g.n + c0;
    const size_t sstep = (size_t)4 * g.HW * g.n;
    for (int s = s0; s < L; s += 4, src += sstep) discard_l2_line(src);
  }
}

// Inverse pencils of a staged volume tile: cell hw0 + warp -> x_hat (bf16, rounded to nearest
// even, or fp32), strided.
template <int L, int NC, bool VAR = false>
__device__ __forceinline__ void idct_s_cells(const Geom& g, const UnitDev& ud, int hw0, int c0, const float* vtile) {
  const int lane = threadIdx.x & 31, hwl = threadIdx.x >> 5, hw = hw0 + hwl;
  if (hw >= g.HW) return;
  float v[L];
  const float* t = vtile + hwl * 32 + lane;
#pragma unroll
  for (int k = 0; k < L; ++k) v[k] = t[k * NC * 32];
  if (!VAR || !(g.flags & TACTKV_SKIP_S)) dct_exact<L, true>(v);
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

// Pieces per 32-channel input row (log2): 64 or 128 bytes in copies of 16 bytes when every unit's
// pointer, strides and head_dim allow it, else of 4 bytes.
inline int input_pieces_lg(const Geom& g, const UnitList& ul, int u0, int nu) {
  const bool fp32 = g.flags & TACTKV_FP32_IO;
  const int esz = fp32 ? 4 : 2, per = 16 / esz;
  bool vec16 = g.head_dim % per == 0;
  for (int i = u0; i < u0 + nu && vec16; ++i)
    vec16 = reinterpret_cast<uintptr_t>(ul.u[i].in) % 16 == 0 && ul.u[i].tok_stride % per == 0 &&
            ul.u[i].head_stride % per == 0;
  return (fp32 ? 3 : 2) + (vec16 ? 0 : 2);
}

}  // namespace
}  // namespace tactkv
