// Shared device code of the TACT-KV codec kernels (internal header).
//
// The method is the one of the TACT-KV summary page ("TACT-KV: Tri-Axis Cosine Transform for
// Compressing Volumetric KV Caches in Medical VLMs"), "Methodology in Plain English"; the C ABI,
// payload format and calling rules are in include/tactkv.h.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "tactkv.h"

namespace tactkv {

constexpr uint32_t kMagic = 0x31564B54u;   // "TKV1"
constexpr int kVersion = 1;
constexpr int kMaxUnits = 256;             // units per launch (descriptors travel as kernel parameters, 12 KB)
constexpr int kHeaderBytes = 64;
constexpr int kChunk = 32;                 // channels per H/W-axis CTA
constexpr int kPairs = kChunk / 2;         // channel pairs: every pencil carries two channels (float2)
constexpr int kAllocThreads = 1024;
constexpr size_t kStatusBytes = 256;       // status word at the start of the workspace
constexpr int kMaxHW = 1024;               // H*W limit of the H/W-axis kernels
constexpr int kMaxSlabs = 64;              // S limit
constexpr int kMaxN = kMaxSlabs * kMaxHW;  // bins per unit limit
// Records per packing range (one CTA) when a lane packs four channels; 4 * kPackRecs when it packs one.
constexpr int kPackRecs = 256;

enum HwMode { kStats = 0, kQuant = 1, kRaw = 2 };

// flags recorded in the payload header (everything but the I/O type)
constexpr uint32_t kPayloadFlags = TACTKV_NO_QUANT | TACTKV_SKIP_S | TACTKV_SKIP_H | TACTKV_SKIP_W |
                                   TACTKV_UNIFORM_ALLOC | TACTKV_ROTATE | TACTKV_HEAD_GAIN;
constexpr uint32_t kAllFlags = kPayloadFlags | TACTKV_FP32_IO;
constexpr unsigned long long kRotationSeed = 0x544143544B56ull;
// Variant flags (axis skips, shared rotation, per-head gains): kernels take a compile-time VAR
// switch and carry the code for them only when it is set, so that the default kernels keep their
// register budgets.
constexpr uint32_t kVariantFlags = TACTKV_SKIP_S | TACTKV_SKIP_H | TACTKV_SKIP_W | TACTKV_ROTATE | TACTKV_HEAD_GAIN;
inline bool has_variant(int flags) { return (flags & kVariantFlags) != 0; }
__host__ __device__ inline bool has_variant_dev(int flags) { return (flags & kVariantFlags) != 0; }

// ------------------------------------------------------------------------ launch descriptors ---
struct UnitDev {
  const void* in;
  void* out;
  unsigned char* payload;
  long long tok_stride, head_stride;   // elements
  int layer, kv;
};
struct UnitList {
  UnitDev u[kMaxUnits];
};
struct Geom {
  int S, H, W, HW, T, heads, head_dim, n, nch, N, bits, flags;
  int off_sigma, off_codes;     // payload byte offsets
  long long capacity;           // payload bytes available (minimum over the launch)
  int unit0;                    // the transform kernels: unit of blockIdx.z == 0 within the wave
};

__host__ __device__ inline long long pad16(long long x) { return (x + 15) / 16 * 16; }

// Gain vectors of N floats in a payload: one per head with TACTKV_HEAD_GAIN on a quantized
// payload (sigma[head][bin]), else one (sigma[bin]).
__host__ __device__ inline bool head_gains_on(int flags) {
  return (flags & TACTKV_HEAD_GAIN) && !(flags & TACTKV_NO_QUANT);
}
__host__ __device__ inline int gain_vectors(int flags, int heads) { return head_gains_on(flags) ? heads : 1; }

// Per-unit index block in the workspace: P(k_s) for k_s = 0..S (first stream bit of each slab,
// P(S) = code_bits), the decoder's ok flag, then NZ(k_s) for k_s = 0..S (first record of each slab
// in the unit's list of bins with bits).
__host__ __device__ inline int unit_index_words(int S) { return 2 * S + 3; }

// Codebook b (1..8) has 2^b - 1 thresholds and 2^b levels, stored for b = 1, 2, ... in turn.
__host__ __device__ constexpr int lm_thr_offset(int b) { return (1 << b) - b - 1; }
__host__ __device__ constexpr int lm_lv_offset(int b) { return (1 << b) - 2; }
constexpr int kLmThrTotal = lm_thr_offset(9);   // 502
constexpr int kLmLvTotal = lm_lv_offset(9);     // 510

// Length classes: a kernel instantiated for class C holds pencils of up to C values in
// registers and dispatches only the generated lengths of that class.
inline bool supported_length(int L) {
  if (L >= 1 && L <= 16) return true;
  switch (L) {
    case 20: case 24: case 28: case 32: case 40: case 48: case 56: case 64: return true;
    default: return false;
  }
}
inline int length_class(int L) { return L <= 16 ? 16 : (L <= 32 ? 32 : 64); }
__host__ __device__ inline int length_class_dev(int L) { return L <= 16 ? 16 : (L <= 32 ? 32 : 64); }

// Opt-in tensor-core forms (both measured slower on B200 than the default CUDA-core kernels):
// TACTKV_TC_S=1 in the environment runs the S-axis DCT of the fused forward kernel on the tensor
// cores; TACTKV_FUSED_DECODE=1 decodes with the single fused kernel (inverse S on the tensor cores)
// instead of the two inverse kernels.  Both are read once per process.
bool tc_s_pass_enabled();
bool fused_decode_enabled();


// --------------------------------------------------------------------------------- launchers ---
cudaError_t launch_axis_s(int cls, bool inverse, const Geom& g, const UnitList& ul, int nu, float* buf,
                          cudaStream_t st);
cudaError_t launch_axis_hw(int hcls, int wcls, bool inverse, int mode, const Geom& g, const UnitList& ul, int nu, float* buf,
                           float* partial, const uint32_t* index, const uint4* recs, int spc, cudaStream_t st);
void axis_hw_shape(int hcls, int wcls, const Geom& g, bool inverse, int mode, size_t* smem, int* threads);
// Per-unit bit allocation: writes b, sigma and the header into the payload, P and NZ into the
// unit's index block, and the records {bin, bits, P_i, 1/sigma_i} of the bins with bits into recs
// (N per unit).
cudaError_t launch_allocate(const Geom& g, const UnitList& ul, int nu, const float* partial, double* var,
                            uint32_t* index, uint4* recs, cudaStream_t st);
// The allocation alone, on the fp64 variances var[u][bin] given in the workspace (which it
// overwrites): the same kernel and outputs as launch_allocate without the variance reduction.
cudaError_t launch_allocate_from_var(const Geom& g, const UnitList& ul, int nu, double* var, uint32_t* index,
                                     uint4* recs, cudaStream_t st);
// Quantization and packing of the finished coefficients X (workspace volume) into the payloads.
cudaError_t launch_pack(const Geom& g, const UnitList& ul, int nu, const float* X, const uint4* recs,
                        const uint32_t* index, cudaStream_t st);
// Decoding index: checks every unit's header and bit widths, writes P, the unit's ok flag and NZ
// into its index block and the records {bin, bits, first stream bit, sigma} of the bins with bits
// into recs; a bad unit sets TACTKV_CORRUPT_PAYLOAD in *status.
cudaError_t launch_decode_index(const Geom& g, const UnitList& ul, int nu, uint32_t* index, uint4* recs,
                                unsigned int* status, cudaStream_t st);

#ifdef __CUDACC__
// ------------------------------------------------------------------ float2 value operations ---
// Every pencil carries two channels; the packed f32x2 instructions issue both halves at once.
__device__ __forceinline__ float2 vadd(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 vsub(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }
__device__ __forceinline__ float2 vneg(float2 a) { return make_float2(-a.x, -a.y); }
__device__ __forceinline__ float2 vmul(float2 a, float c) { return __fmul2_rn(a, make_float2(c, c)); }
__device__ __forceinline__ float2 vfma(float2 a, float c, float2 b) { return __ffma2_rn(a, make_float2(c, c), b); }

// one-channel pencils use plain fp32 operations
__device__ __forceinline__ float vadd(float a, float b) { return a + b; }
__device__ __forceinline__ float vsub(float a, float b) { return a - b; }
__device__ __forceinline__ float vneg(float a) { return -a; }
__device__ __forceinline__ float vmul(float a, float c) { return a * c; }
__device__ __forceinline__ float vfma(float a, float c, float b) { return fmaf(a, c, b); }

// the generated pencil transforms (templates over the value type) live in this namespace too
#include "dct_gen.cuh"

// Orthonormal DCT-II (INV = false) or DCT-III (INV = true) of x[0..L) held in registers.
template <int CLASS, bool INV, class V>
__device__ __forceinline__ void dct_pencil(V* x, int L) {
#define TACTKV_CASE(n)                          \
  case n:                                       \
    if constexpr (INV) idct_##n(x);             \
    else fdct_##n(x);                           \
    break;
  if constexpr (CLASS == 16) {
    switch (L) {
      TACTKV_CASE(1) TACTKV_CASE(2) TACTKV_CASE(3) TACTKV_CASE(4) TACTKV_CASE(5) TACTKV_CASE(6)
      TACTKV_CASE(7) TACTKV_CASE(8) TACTKV_CASE(9) TACTKV_CASE(10) TACTKV_CASE(11) TACTKV_CASE(12)
      TACTKV_CASE(13) TACTKV_CASE(14) TACTKV_CASE(15) TACTKV_CASE(16)
      default: break;
    }
  } else if constexpr (CLASS == 32) {
    switch (L) {
      TACTKV_CASE(20) TACTKV_CASE(24) TACTKV_CASE(28) TACTKV_CASE(32)
      default: break;
    }
  } else {
    switch (L) {
      TACTKV_CASE(40) TACTKV_CASE(48) TACTKV_CASE(56) TACTKV_CASE(64)
      default: break;
    }
  }
#undef TACTKV_CASE
}

// Orthonormal DCT-II (INV = false) or DCT-III (INV = true) of exactly L values in registers.
template <int L, bool INV, class V>
__device__ __forceinline__ void dct_exact(V* x) {
#define TACTKV_EXACT(n)              \
  if constexpr (L == n) {            \
    if constexpr (INV) idct_##n(x);  \
    else fdct_##n(x);                \
  }
  TACTKV_EXACT(1) TACTKV_EXACT(2) TACTKV_EXACT(3) TACTKV_EXACT(4) TACTKV_EXACT(5) TACTKV_EXACT(6) TACTKV_EXACT(7)
  TACTKV_EXACT(8) TACTKV_EXACT(9) TACTKV_EXACT(10) TACTKV_EXACT(11) TACTKV_EXACT(12) TACTKV_EXACT(13)
  TACTKV_EXACT(14) TACTKV_EXACT(15) TACTKV_EXACT(16) TACTKV_EXACT(20) TACTKV_EXACT(24) TACTKV_EXACT(28)
  TACTKV_EXACT(32) TACTKV_EXACT(40) TACTKV_EXACT(48) TACTKV_EXACT(56) TACTKV_EXACT(64)
#undef TACTKV_EXACT
}

__device__ __forceinline__ void set_status(unsigned int* status, unsigned int code) { atomicCAS(status, 0u, code); }

// Sums over the 32 lanes of the warp of 32 values per lane (recursive halving: at each step a
// lane keeps half of its values and adds the partner lane's copy of that half); lane l returns the
// total of value l.
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int h = 16; h >= 1; h >>= 1) {
    const bool upper = lane & h;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h], keep = upper ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, h);
    }
  }
  return v[0];
}

// ------------------------------------------------------------------ shared shape rotation ---
// Sign of channel c in the rotation: the top bit of output c of SplitMix64 (Steele, Lea and
// Flood, OOPSLA 2014) started from kRotationSeed (state seed + (c+1) * gamma, then the variant-13
// finalizer of MurmurHash3).
__device__ __forceinline__ float rotation_sign(unsigned long long c) {
  unsigned long long z = kRotationSeed + (c + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (z >> 63) ? -1.f : 1.f;
}
// Walsh-Hadamard transform of the 32 lanes' values (Sylvester order: lane i gets
// sum_j (-1)^popcount(i & j) v_j), unnormalised; every lane of the warp calls it.
__device__ __forceinline__ float warp_wht(float v, int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const float p = __shfl_xor_sync(0xffffffffu, v, h);
    v = fmaf(v, (lane & h) ? -1.f : 1.f, p);   // lower lane: p + v; upper lane: p - v
  }
  return v;
}

// Asynchronous global -> shared copies (LDGSTS): issued now, waited for with cp_async_wait_all.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
// A table of n 16-byte vectors from global memory into shared memory, vector i by thread i (mod the
// block), one load each: copied out of constant memory instead, a warp's 32 different addresses
// would be served one after another.
__device__ __forceinline__ void copy_vec16(void* smem, const void* gmem, int n) {
  uint4* d = reinterpret_cast<uint4*>(smem);
  const uint4* s = reinterpret_cast<const uint4*>(gmem);
  for (int i = threadIdx.x; i < n; i += blockDim.x) d[i] = __ldg(s + i);
}
// Streams that pass through L2 once (the input, the finished coefficients) are marked
// evict-first in the fused forward kernel, so that they give way to the fp32 volume that is read
// back soon after.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}
__device__ __forceinline__ void cp_async16_ef(void* smem, const void* gmem, uint64_t pol) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(sa), "l"(gmem), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async4_ef(void* smem, const void* gmem, uint64_t pol) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 4, %2;\n" ::"r"(sa), "l"(gmem), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void st_ef(float* p, float v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;\n" ::"l"(p), "f"(v), "l"(pol) : "memory");
}
// Invalidate the 128-byte L2 line at p (global memory, 128-byte aligned) without writing it back,
// for scratch data that nothing reads again; its contents become undefined.
__device__ __forceinline__ void discard_l2_line(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;\n" ::"l"(__cvta_generic_to_global(p)) : "memory");
}

// In place exclusive scan of a[0..n) in shared memory; blockDim.x a multiple of 32; returns the total.
__device__ inline uint32_t block_exclusive_scan(uint32_t* a, int n, uint32_t* s_warp /* 33 entries */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, (int)threadIdx.x * per), end = min(n, beg + per);
  uint32_t sum = 0;
  for (int i = beg; i < end; ++i) sum += a[i];
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < nwarps ? s_warp[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    s_warp[lane] = wi - w;
    if (lane == 31) s_warp[32] = wi;
  }
  __syncthreads();
  uint32_t run = s_warp[warp] + incl - sum;
  for (int i = beg; i < end; ++i) {
    const uint32_t v = a[i];
    a[i] = run;
    run += v;
  }
  const uint32_t total = s_warp[32];
  __syncthreads();
  return total;
}
#endif  // __CUDACC__

}  // namespace tactkv
