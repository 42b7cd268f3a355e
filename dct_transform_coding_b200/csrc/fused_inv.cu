// Decoding (the paragraph after stage 4 of "Methodology in Plain English" on the TACT-KV summary
// page: unpack, dequantize, inverse 3D DCT) in one kernel per (unit, 32-channel chunk) cluster.
//
// A cluster of kCluster CTAs owns one (unit, chunk).  Phase 1: each CTA decodes its share of the S
// slabs and runs the inverse DCT along W and H on them (axis_hw.cuh), writing the result V as bf16
// hi/lo pairs into the workspace; the chunk's V (2 MB for 64 x 16 x 16) is read back by the same
// cluster right after, so it is served by L2.  A cluster barrier makes it visible.  Phase 2: the
// inverse DCT along S of tiles of 4 grid cells x 32 channels on the tensor cores,
//     x[(cell, c), s] = sum_k V[(cell, c), k] * C[k, s],
// M = 128 rows, N = S, K = S, with V = V_hi + V_lo and C = C_hi + C_mid in bf16 limbs (products
// hi*hi + hi*mid + lo*hi, fp32 accumulation in TMEM: about 2^-16 relative), then rounded to bf16
// (or kept as fp32) and stored with the caller's strides.
//   A = a V tile, loaded by TMA as [cell pair][k][32 channels x 2 cells] bf16 with 128-byte swizzle:
//       MN-major, one 128-byte row of 64 M-elements (channel, cell of the pair) per k;
//   B = a limb of C^T, [s][k] with k contiguous: K-major with 128-byte swizzle.
// Compiled once per S (TACTKV_FUSED_S = 16, 32, 64) for the grids 16x16, 14x14 and 8x8.  Opt-in
// (TACTKV_FUSED_DECODE=1): on B200 it measured slower than the two separate inverse kernels (its V
// pairs left L2, and few CTAs of its 8-CTA clusters were resident at a time).
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

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kCells = 4;                 // grid cells per tile (M = 128: 2 cell pairs x 32 channels x 2)

template <int L>
struct TcInv {
  static_assert(L == 16 || L == 32 || L == 64, "S of the tensor-core pass");
  static constexpr int kABytes = 2 * L * 128;          // one limb of a V tile: 2 cell pairs x L rows of 128 B
  static constexpr int kBBytes = L * 128;              // one limb of C^T, rows padded to 128 bytes
  static constexpr int kSmem = 2 * kBBytes + 2 * kABytes + 1024;
  static constexpr int kCols = L < 32 ? 32 : L;
  static constexpr int kHalf = L / 2;
};

template <int L>
__device__ __forceinline__ const uint16_t* dct_limb_inv() {
  if constexpr (L == 16) return &kDctLimbInv16[0][0][0];
  else if constexpr (L == 32) return &kDctLimbInv32[0][0][0];
  else return &kDctLimbInv64[0][0][0];
}

// Every thread of every CTA of the cluster: its global writes before it (ordinary stores) are
// visible after it to the cluster's reads, the tensor-memory copies (async proxy) included.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Phase 2 of one (unit u, chunk) on this CTA's tiles t = r, r + kCluster, ...; false (and
// TACTKV_TIMEOUT recorded) if a copy or an MMA did not complete.  Called by every thread.
template <int L, int HWX>
__device__ bool idct_s_tc(const Geom& g, const UnitDev& ud, int u, int chunk, int r, const CUtensorMap* mhi,
                          const CUtensorMap* mlo, unsigned char* smem, uint64_t* bars, uint32_t* tmem_slot,
                          unsigned int* status) {
  using P = TcInv<L>;
  constexpr int kTiles = HWX / kCells;
  static_assert(HWX % kCells == 0, "whole tiles");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int uw = u - g.unit0;
  unsigned char* sB = smem;
  unsigned char* sAh = smem + 2 * P::kBBytes;
  unsigned char* sAl = sAh + P::kABytes;
  uint64_t* tma_bar = bars;
  uint64_t* mma_bar = bars + 1;
  const int mine = r < kTiles ? (kTiles - r + kCluster - 1) / kCluster : 0;

  // B: limbs hi and mid of C^T, swizzled (16-byte chunk j of row s at chunk j ^ (s & 7))
  const uint16_t* tab = dct_limb_inv<L>();
  for (int e = tid; e < 2 * L * 8; e += blockDim.x) {
    const int l = e / (L * 8), rem = e - l * (L * 8), n = rem >> 3, j = rem & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j * 8 < L) v = *reinterpret_cast<const uint4*>(tab + ((size_t)l * L + n) * L + j * 8);
    *reinterpret_cast<uint4*>(sB + l * P::kBBytes + n * 128 + ((j ^ (n & 7)) << 4)) = v;
  }
  tc::fence_proxy_async();
  if (tid == 0) {
    tc::prefetch_tmap(mhi);
    tc::prefetch_tmap(mlo);
    tc::mbar_init(tma_bar, 1);
    tc::mbar_init(mma_bar, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, P::kCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  auto load = [&](int t) {
    tc::mbar_expect_tx(tma_bar, 2 * P::kABytes);
    tc::tma_load_5d(sAh, mhi, tma_bar, chunk * 2 * kChunk, 0, t * (kCells / 2), uw, 0);
    tc::tma_load_5d(sAl, mlo, tma_bar, chunk * 2 * kChunk, 0, t * (kCells / 2), uw, 0);
  };
  if (tid == 0 && mine > 0) load(r);
  constexpr uint32_t kIdesc = tc::idesc_bf16(128, L, true);
  const bool fp32_out = g.flags & TACTKV_FP32_IO;
  // this thread's accumulator row 32 (warp % 4) + lane: cell pair (warp % 4) / 2 of the tile,
  // channel ((warp % 4) % 2) * 16 + lane / 2, cell (lane % 2) of the pair; columns of half warp / 4
  const int q = warp & 3, half = warp >> 2;
  const int c = chunk * kChunk + (q & 1) * 16 + (lane >> 1);
  const int head = c / g.head_dim, d = c - head * g.head_dim;
  bool ok = true;
  for (int j = 0; j < mine; ++j) {
    const int t = r + kCluster * j;
    bool ok_t = true;
    if (tid == 0) {
      ok_t = tc::mbar_wait(tma_bar, j & 1);
      if (ok_t) {
        tc::fence_after_sync();
        const uint32_t ah = tc::smem_u32(sAh), al = tc::smem_u32(sAl), b0 = tc::smem_u32(sB);
        bool acc = false;
#pragma unroll
        for (int ks = 0; ks < L / 16; ++ks) {
          const uint64_t dah = tc::smem_desc(ah + ks * 2048, L * 128, 1024, 2);
          const uint64_t dal = tc::smem_desc(al + ks * 2048, L * 128, 1024, 2);
          const uint64_t dbh = tc::smem_desc(b0 + ks * 32, 16, 1024, 2);
          const uint64_t dbm = tc::smem_desc(b0 + P::kBBytes + ks * 32, 16, 1024, 2);
          tc::mma_bf16(tmem, dah, dbh, kIdesc, acc);
          tc::mma_bf16(tmem, dah, dbm, kIdesc, true);
          tc::mma_bf16(tmem, dal, dbh, kIdesc, true);
          acc = true;
        }
        tc::mma_commit(mma_bar);
      }
    }
    ok_t = __syncthreads_and(ok_t) != 0;
    if (ok_t) ok_t = __syncthreads_and(tc::mbar_wait(mma_bar, j & 1)) != 0;
    if (!ok_t) {
      if (tid == 0) {   // bounded wait for what may still be in flight before its memory is released
        tc::mbar_wait(tma_bar, j & 1);
        tc::mbar_wait(mma_bar, j & 1);
      }
      __syncthreads();
      ok = false;
      break;
    }
    tc::fence_after_sync();
    if (tid == 0 && j + 1 < mine) load(t + kCluster);   // the tile's shared memory is free again
    float v[P::kHalf];
    tc::tmem_ld<P::kHalf>(tmem + ((uint32_t)(32 * q) << 16) + half * P::kHalf, v);
    tc::tmem_ld_wait();
    const int cell = t * kCells + (q >> 1) * 2 + (lane & 1);
    const long long step = (long long)HWX * ud.tok_stride;
    const long long base = ((long long)half * P::kHalf * HWX + cell) * ud.tok_stride + (long long)head * ud.head_stride + d;
    if (fp32_out) {
      float* o = static_cast<float*>(ud.out) + base;
#pragma unroll
      for (int k = 0; k < P::kHalf; ++k) o[k * step] = v[k];
    } else {
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(ud.out) + base;
#pragma unroll
      for (int k = 0; k < P::kHalf; ++k) o[k * step] = __float2bfloat16_rn(v[k]);
    }
    tc::fence_before_sync();
    __syncthreads();   // every thread has read the accumulator before the next tile's MMAs
  }
  if (!ok && tid == 0) atomicCAS(status, 0u, (unsigned int)TACTKV_TIMEOUT);
  tc::fence_after_sync();
  if (warp == 0) {
    __syncwarp();
    tc::tmem_free(tmem, P::kCols);
  }
  return ok;
}

template <int L, int HX, int WX>
__global__ void __launch_bounds__(kThreads, 3) idct3_tc_kernel(const __grid_constant__ Geom g,
                                                               const __grid_constant__ UnitList ul,
                                                               float* __restrict__ Vhi, __nv_bfloat162* __restrict__ Vlo,
                                                               const uint32_t* __restrict__ index,
                                                               const uint4* __restrict__ recs,
                                                               const __grid_constant__ CUtensorMap mhi,
                                                               const __grid_constant__ CUtensorMap mlo,
                                                               unsigned int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_bars[2];
  __shared__ uint32_t s_tmem;
  unsigned char* smem = smem_raw + ((1024 - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const int r = blockIdx.x, chunk = blockIdx.y, u = g.unit0 + blockIdx.z;
  constexpr int spc = (L + kCluster - 1) / kCluster;
  const int ks0 = r * spc, ks1 = min(L, ks0 + spc);
  if (ks0 < ks1) {
    if (has_variant_dev(g.flags))
      idct_hw_slabs<16, 16, HX, WX, kQuant, true, true>(g, ul, Vhi, index, recs, u, chunk, ks0, ks1, smem, Vlo);
    else
      idct_hw_slabs<16, 16, HX, WX, kQuant, true, false>(g, ul, Vhi, index, recs, u, chunk, ks0, ks1, smem, Vlo);
  }
  cluster_barrier();   // the chunk's V is complete
  idct_s_tc<L, HX * WX>(g, ul.u[u], u, chunk, r, &mhi, &mlo, smem, s_bars, &s_tmem, status);
}

// Tensor map of one limb of the wave's V: 5-D (element e = 2 c + cell bit, k, cell pair, unit, 1),
// box (64, S, 2, 1, 1) with 128-byte swizzle, so a box lands as [cell pair][k][64 elements].
bool make_v_map(const Geom& g, int nu, const void* base, CUtensorMap* map) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!encode || reinterpret_cast<uintptr_t>(base) % 16) return false;
  const cuuint64_t row = (cuuint64_t)g.n * 2 * 2;   // bytes of one cell pair: n channels x 2 cells x bf16
  const cuuint64_t dims[5] = {(cuuint64_t)(2 * g.n), (cuuint64_t)g.S, (cuuint64_t)(g.HW / 2), (cuuint64_t)nu, 1};
  const cuuint64_t strides[4] = {(cuuint64_t)(g.HW / 2) * row, row, (cuuint64_t)g.S * (g.HW / 2) * row,
                                 (cuuint64_t)nu * g.S * (g.HW / 2) * row};
  const cuuint32_t box[5] = {2u * kChunk, (cuuint32_t)g.S, (cuuint32_t)(kCells / 2), 1u, 1u};
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HX, int WX>
cudaError_t launch_grid(const Geom& g, const UnitList& ul, int nu, float* big, const uint32_t* index,
                        const uint4* recs, unsigned int* status, cudaStream_t st) {
  constexpr int L = TACTKV_FUSED_S;
  const HwLayout Ld = hw_layout(HX, WX, kLayDecode);
  const size_t regions[] = {Ld.tile, Ld.sbuf, Ld.meta, Ld.lv, Ld.tile_bytes};
  for (size_t x : regions)
    if (x % 16) return cudaErrorMisalignedAddress;   // never launch a misaligned layout
  // V_hi and V_lo (bf16 each) share the fp32 volume's workspace region
  const size_t half = (size_t)nu * g.T * g.n * 2;
  float* vhi = big;
  __nv_bfloat162* vlo = reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<unsigned char*>(big) + half);
  CUtensorMap mhi, mlo;
  if (!make_v_map(g, nu, vhi, &mhi) || !make_v_map(g, nu, vlo, &mlo)) return cudaErrorNotSupported;
  const size_t smem = std::max<size_t>(TcInv<L>::kSmem, Ld.total + 1024);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  auto kernel = idct3_tc_kernel<L, HX, WX>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCluster, g.nch, nu);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kCluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, g, ul, vhi, vlo, index, recs, mhi, mlo, status);
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
// Fused decode + inverse transforms of one wave of quantized payloads (g.S == TACTKV_FUSED_S):
// cudaErrorNotSupported for any other grid, for NO_QUANT payloads, or when the volume cannot be
// described by tensor maps (the caller then runs the separate inverse kernels).
cudaError_t TACTKV_CAT(launch_fused_inv_, TACTKV_FUSED_S)(const Geom& g, const UnitList& ul, int nu, float* big,
                                                          const uint32_t* index, const uint4* recs,
                                                          unsigned int* status, cudaStream_t st) {
  if (g.S != TACTKV_FUSED_S || (g.flags & (TACTKV_NO_QUANT | TACTKV_SKIP_S | TACTKV_SKIP_H | TACTKV_SKIP_W)) ||
      !fused_decode_enabled())
    return cudaErrorNotSupported;
  if (g.H == 16 && g.W == 16) return launch_grid<16, 16>(g, ul, nu, big, index, recs, status, st);
  if (g.H == 14 && g.W == 14) return launch_grid<14, 14>(g, ul, nu, big, index, recs, status, st);
  if (g.H == 8 && g.W == 8) return launch_grid<8, 8>(g, ul, nu, big, index, recs, status, st);
  return cudaErrorNotSupported;
}

}  // namespace tactkv
