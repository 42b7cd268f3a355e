// DCT along the H and W axes plus the per-bin epilogues (TACT-KV stages 2-4 and their inverse).
//
// One CTA owns one (unit, 32-channel chunk) and walks the S frequency slabs k_s in order.  Per
// slab it stages the H*W x 32 coefficients in shared memory (16 channel pairs per row), runs
// the pencil DCTs along H and then along W, and finishes with one of:
//   kStats  per-bin energy sum_c X^2 over its 32 channels -> partial[u][chunk][bin] (pass 1)
//   kQuant  u = X / sigma_i, Lloyd-Max code at b_i bits, packed into the 32 channel streams
//   kRaw    float32 coefficients into the streams (TACTKV_NO_QUANT)
// Because a CTA owns its channels' streams from the first bit to the last, each output word is
// assembled in shared memory and stored exactly once; the word that straddles two slabs is
// carried to the next slab.  Decoding (idct_hw) reads the same words, dequantizes and applies
// the inverse DCTs along W and H.
//
// Compiled once per pair of length classes (TACTKV_HCLASS, TACTKV_WCLASS: 16 or 32 each).
#include "common.cuh"
#include "lloyd_max_tables.inc"

#if !defined(TACTKV_HCLASS) || !defined(TACTKV_WCLASS)
#error "TACTKV_HCLASS and TACTKV_WCLASS must be defined"
#endif

namespace tactkv {
namespace {

struct HwSmem {
  float2* tile;       // [HW][16] channel pairs of one S slab
  float* thr;         // all Lloyd-Max thresholds
  float* lv;          // all Lloyd-Max levels
  float* gain;        // [HW] 1/sigma (encode) or sigma (decode) of the slab's bins
  uint32_t* b;        // [HW] bits of the slab's bins
  uint32_t* off;      // [HW] bit offset of each bin, relative to the word holding the slab's first bit
  uint32_t* sbuf;     // [32][words] stream words of the slab, per channel
  uint32_t* carry;    // [32]
  uint32_t* warp;     // [33] scan scratch
  int words;          // stride of sbuf rows
};

__device__ HwSmem carve(unsigned char* sm, int HW) {
  HwSmem s;
  s.words = stream_words_per_slab(HW);
  s.tile = reinterpret_cast<float2*>(sm); sm += (size_t)HW * kPairs * sizeof(float2);
  s.thr = reinterpret_cast<float*>(sm); sm += kLmThrTotal * 4;
  s.lv = reinterpret_cast<float*>(sm); sm += kLmLvTotal * 4;
  s.gain = reinterpret_cast<float*>(sm); sm += (size_t)HW * 4;
  s.b = reinterpret_cast<uint32_t*>(sm); sm += (size_t)HW * 4;
  s.off = reinterpret_cast<uint32_t*>(sm); sm += (size_t)HW * 4;
  s.sbuf = reinterpret_cast<uint32_t*>(sm); sm += (size_t)kChunk * s.words * 4;
  s.carry = reinterpret_cast<uint32_t*>(sm); sm += kChunk * 4;
  s.warp = reinterpret_cast<uint32_t*>(sm);
  return s;
}

// Lloyd-Max code: the number of thresholds t_j <= u (branch-free bisection over 2^b - 1 values).
__device__ __forceinline__ uint32_t lm_code(float u, int bits, const float* thr) {
  const float* t = thr + lm_thr_offset(bits);
  uint32_t code = 0;
  for (int step = 1 << (bits - 1); step > 0; step >>= 1)
    if (u >= t[code + step - 1]) code += step;
  return code;
}

// Pencil DCTs along one axis of the tile: along H the pencils are (w, pair) with stride W*16,
// along W they are (h, pair) with stride 16.
template <int CLASS, bool INV>
__device__ __forceinline__ void tile_pass(const Geom& g, float2* tile, bool along_h) {
  const int L = along_h ? g.H : g.W;
  const int npen = (along_h ? g.W : g.H) * kPairs;
  const int step = along_h ? g.W * kPairs : kPairs;
  for (int p = threadIdx.x; p < npen; p += blockDim.x) {
    const int q = p >> 4, pair = p & 15;
    const int base = along_h ? q * kPairs + pair : q * g.W * kPairs + pair;
    float2 x[CLASS];
#pragma unroll
    for (int t = 0; t < CLASS; ++t)
      if (t < L) x[t] = tile[base + t * step];
    dct_pencil<CLASS, INV>(x, L);
#pragma unroll
    for (int t = 0; t < CLASS; ++t)
      if (t < L) tile[base + t * step] = x[t];
  }
}

template <int HC, int WC>
__global__ void __launch_bounds__(kHwThreads) fdct_hw_kernel(const __grid_constant__ Geom g,
                                                             const __grid_constant__ UnitList ul, int mode,
                                                             const float* __restrict__ Y, float* __restrict__ partial) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  HwSmem s = carve(smem_raw, g.HW);
  const int chunk = blockIdx.x, u = blockIdx.y;
  const UnitDev& ud = ul.u[u];
  unsigned char* pay = ud.payload;
  uint32_t* words_out = reinterpret_cast<uint32_t*>(pay + g.off_codes);
  uint32_t cstride = 0, stride_words = 0;
  if (mode != kStats) {  // the header was written by the allocation kernel
    cstride = reinterpret_cast<const uint32_t*>(pay)[11];
    stride_words = cstride / 4;
  }
  if (mode == kQuant) {
    for (int i = threadIdx.x; i < kLmThrTotal; i += blockDim.x) s.thr[i] = c_lm_thresholds[i];
    if (threadIdx.x < kChunk) s.carry[threadIdx.x] = 0;
  }
  const float4* ysrc = reinterpret_cast<const float4*>(Y + (size_t)u * g.S * g.HW * g.n) + chunk * (kChunk / 4);
  const int rowq = g.n / 4;
  uint32_t P = 0;  // stream bits written so far, identical for every channel
  for (int ks = 0; ks < g.S; ++ks) {
    // stage the slab: HW rows of 32 channels
    const float4* src = ysrc + (size_t)ks * g.HW * rowq;
    float4* dst = reinterpret_cast<float4*>(s.tile);
    for (int i = threadIdx.x; i < g.HW * (kChunk / 4); i += blockDim.x) dst[i] = src[(size_t)(i >> 3) * rowq + (i & 7)];
    const uint32_t shift0 = P & 31u;
    uint32_t slab_bits = 0;
    if (mode == kQuant) {
      const int i0 = ks * g.HW;
      for (int j = threadIdx.x; j < g.HW; j += blockDim.x) {
        const uint32_t b = pay[kHeaderBytes + i0 + j];
        s.b[j] = b;
        s.off[j] = b;
        s.gain[j] = b ? 1.0f / reinterpret_cast<const float*>(pay + g.off_sigma)[i0 + j] : 0.0f;
      }
      __syncthreads();
      slab_bits = block_exclusive_scan(s.off, g.HW, s.warp);
      for (int j = threadIdx.x; j < g.HW; j += blockDim.x) s.off[j] += shift0;
      const int nw = (int)((shift0 + slab_bits + 31) >> 5) + 1;
      for (int i = threadIdx.x; i < kChunk * nw; i += blockDim.x) {
        const int ch = i / nw, w = i - ch * nw;
        s.sbuf[ch * s.words + w] = w == 0 ? s.carry[ch] : 0u;
      }
    }
    __syncthreads();
    tile_pass<HC, false>(g, s.tile, true);
    __syncthreads();
    // W pass fused with the per-bin epilogue
    for (int p = threadIdx.x; p < g.H * kPairs; p += blockDim.x) {
      const int kh = p >> 4, pair = p & 15;
      const int base = kh * g.W * kPairs + pair;
      float2 x[WC];
#pragma unroll
      for (int t = 0; t < WC; ++t)
        if (t < g.W) x[t] = s.tile[base + t * kPairs];
      dct_pencil<WC, false>(x, g.W);
      if (mode == kStats) {
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < g.W) s.tile[base + t * kPairs].x = x[t].x * x[t].x + x[t].y * x[t].y;
      } else if (mode == kRaw) {
        const int c = chunk * kChunk + 2 * pair;
        float* s0 = reinterpret_cast<float*>(pay + g.off_codes + (size_t)c * cstride) + ks * g.HW + kh * g.W;
        float* s1 = reinterpret_cast<float*>(pay + g.off_codes + (size_t)(c + 1) * cstride) + ks * g.HW + kh * g.W;
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < g.W) {
            s0[t] = x[t].x;
            s1[t] = x[t].y;
          }
      } else {
        uint32_t* r0 = s.sbuf + (2 * pair) * s.words;
        uint32_t* r1 = r0 + s.words;
#pragma unroll
        for (int t = 0; t < WC; ++t) {
          if (t < g.W) {
            const int j = kh * g.W + t;
            const int bits = (int)s.b[j];
            if (bits) {
              const float inv = s.gain[j];
              const uint32_t c0 = lm_code(x[t].x * inv, bits, s.thr);
              const uint32_t c1 = lm_code(x[t].y * inv, bits, s.thr);
              const uint32_t off = s.off[j], wi = off >> 5, sh = off & 31u;
              atomicOr(r0 + wi, c0 << sh);
              atomicOr(r1 + wi, c1 << sh);
              if (sh + bits > 32) {
                atomicOr(r0 + wi + 1, c0 >> (32 - sh));
                atomicOr(r1 + wi + 1, c1 >> (32 - sh));
              }
            }
          }
        }
      }
    }
    __syncthreads();
    if (mode == kStats) {
      float* dst = partial + ((size_t)u * g.nch + chunk) * g.N + (size_t)ks * g.HW;
      for (int j = threadIdx.x; j < g.HW; j += blockDim.x) {
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < kPairs; ++q) acc += s.tile[j * kPairs + q].x;
        dst[j] = acc;
      }
    } else if (mode == kQuant) {
      // complete words go out now; the word holding the run's last bits carries over
      const uint32_t endbit = shift0 + slab_bits;
      const int full = (int)(endbit >> 5);
      const uint32_t w0 = P >> 5;
      for (int i = threadIdx.x; i < kChunk * full; i += blockDim.x) {
        const int ch = i / full, w = i - ch * full;
        words_out[(size_t)(chunk * kChunk + ch) * stride_words + w0 + w] = s.sbuf[ch * s.words + w];
      }
      __syncthreads();
      if (threadIdx.x < kChunk) s.carry[threadIdx.x] = (endbit & 31u) ? s.sbuf[threadIdx.x * s.words + full] : 0u;
      P += slab_bits;
    }
    __syncthreads();
  }
  if (mode == kQuant) {
    // the last partial word, then zero padding up to the channel stride
    const uint32_t wlast = P >> 5;
    const int tail = (int)stride_words - (int)wlast;
    for (int i = threadIdx.x; i < kChunk * tail; i += blockDim.x) {
      const int ch = i / tail, w = i - ch * tail;
      words_out[(size_t)(chunk * kChunk + ch) * stride_words + wlast + w] = (w == 0) ? s.carry[ch] : 0u;
    }
  } else if (mode == kRaw) {
    const int pad = (int)cstride - 4 * g.N;
    for (int i = threadIdx.x; i < kChunk * pad; i += blockDim.x) {
      const int ch = i / pad, b = i - ch * pad;
      pay[g.off_codes + (size_t)(chunk * kChunk + ch) * cstride + 4 * g.N + b] = 0;
    }
  }
}

template <int HC, int WC>
__global__ void __launch_bounds__(kHwThreads) idct_hw_kernel(const __grid_constant__ Geom g,
                                                             const __grid_constant__ UnitList ul, int mode,
                                                             float* __restrict__ V, unsigned int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  HwSmem s = carve(smem_raw, g.HW);
  __shared__ int s_ok;
  __shared__ unsigned int s_bad_b;
  const int chunk = blockIdx.x, u = blockIdx.y;
  const UnitDev& ud = ul.u[u];
  const unsigned char* pay = ud.payload;
  const bool raw = mode == kRaw;
  if (threadIdx.x == 0) {
    // the header must describe exactly the unit the caller asked for
    const uint32_t* h32 = reinterpret_cast<const uint32_t*>(pay);
    const int32_t* i32 = reinterpret_cast<const int32_t*>(pay);
    const uint32_t ver_flags = h32[1], code_bits = h32[10], cstride = h32[11];
    const unsigned long long total = *reinterpret_cast<const unsigned long long*>(pay + 48);
    bool ok = h32[0] == kMagic && (ver_flags & 0xffffu) == (uint32_t)kVersion &&
              ((ver_flags >> 16) & TACTKV_NO_QUANT) == (raw ? TACTKV_NO_QUANT : 0u) && i32[2] == ud.layer &&
              i32[3] == ud.kv && i32[4] == g.S && i32[5] == g.H && i32[6] == g.W && i32[7] == g.heads &&
              i32[8] == g.head_dim && i32[9] == g.bits;
    if (ok) {
      ok = (raw ? code_bits == 32u * (uint32_t)g.N : code_bits <= (uint32_t)g.bits * (uint32_t)g.N) &&
           (long long)cstride == pad16(((long long)code_bits + 7) / 8) &&
           (long long)total == (long long)g.off_codes + (long long)g.n * cstride && (long long)total <= g.capacity;
    }
    s_ok = ok;
    s_bad_b = 0;
    if (!ok && chunk == 0) set_status(status, TACTKV_CORRUPT_PAYLOAD);
  }
  for (int i = threadIdx.x; i < kLmLvTotal; i += blockDim.x) s.lv[i] = c_lm_levels[i];
  __syncthreads();
  const bool ok = s_ok;
  const uint32_t stride_words = ok ? reinterpret_cast<const uint32_t*>(pay)[11] / 4 : 0u;
  const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes);
  float4* vdst = reinterpret_cast<float4*>(V + (size_t)u * g.S * g.HW * g.n) + chunk * (kChunk / 4);
  const int rowq = g.n / 4;
  uint32_t P = 0;
  for (int ks = 0; ks < g.S; ++ks) {
    const int i0 = ks * g.HW;
    const uint32_t shift0 = P & 31u;
    uint32_t slab_bits = 0;
    if (ok) {
      for (int j = threadIdx.x; j < g.HW; j += blockDim.x) {
        const uint32_t b = raw ? 0u : pay[kHeaderBytes + i0 + j];
        if (b > 8) s_bad_b = 1;
        s.b[j] = b > 8 ? 0u : b;
        s.off[j] = s.b[j];
        s.gain[j] = reinterpret_cast<const float*>(pay + g.off_sigma)[i0 + j];
      }
      __syncthreads();
      if (!raw) {
        slab_bits = block_exclusive_scan(s.off, g.HW, s.warp);
        for (int j = threadIdx.x; j < g.HW; j += blockDim.x) s.off[j] += shift0;
        const int nw = (int)((shift0 + slab_bits + 31) >> 5);
        const uint32_t w0 = P >> 5;
        for (int i = threadIdx.x; i < kChunk * (nw + 1); i += blockDim.x) {
          const int ch = i / (nw + 1), w = i - ch * (nw + 1);
          const uint32_t word = w0 + w;
          s.sbuf[ch * s.words + w] =
              (w < nw && word < stride_words) ? streams[(size_t)(chunk * kChunk + ch) * stride_words + word] : 0u;
        }
      }
      __syncthreads();
    }
    // inverse DCT along W from the dequantized coefficients
    for (int p = threadIdx.x; p < g.H * kPairs; p += blockDim.x) {
      const int kh = p >> 4, pair = p & 15;
      const int base = kh * g.W * kPairs + pair;
      const int c = chunk * kChunk + 2 * pair;
      float2 x[WC];
#pragma unroll
      for (int t = 0; t < WC; ++t) {
        if (t < g.W) {
          float2 v = make_float2(0.f, 0.f);
          if (ok) {
            const int j = kh * g.W + t;
            if (raw) {
              const float* st = reinterpret_cast<const float*>(streams);
              v.x = st[(size_t)c * stride_words + i0 + j];
              v.y = st[(size_t)(c + 1) * stride_words + i0 + j];
            } else {
              const int bits = (int)s.b[j];
              if (bits) {
                const uint32_t off = s.off[j], wi = off >> 5, sh = off & 31u, mask = (1u << bits) - 1u;
                const uint32_t* r0 = s.sbuf + (2 * pair) * s.words + wi;
                const uint32_t* r1 = r0 + s.words;
                const uint32_t c0 = (uint32_t)(((((unsigned long long)r0[1]) << 32) | r0[0]) >> sh) & mask;
                const uint32_t c1 = (uint32_t)(((((unsigned long long)r1[1]) << 32) | r1[0]) >> sh) & mask;
                const float* lv = s.lv + lm_lv_offset(bits);
                const float sg = s.gain[j];
                v = make_float2(sg * lv[c0], sg * lv[c1]);
              }
            }
          }
          x[t] = v;
        }
      }
      dct_pencil<WC, true>(x, g.W);
#pragma unroll
      for (int t = 0; t < WC; ++t)
        if (t < g.W) s.tile[base + t * kPairs] = x[t];
    }
    __syncthreads();
    tile_pass<HC, true>(g, s.tile, true);
    __syncthreads();
    float4* dst = vdst + (size_t)ks * g.HW * rowq;
    const float4* src = reinterpret_cast<const float4*>(s.tile);
    for (int i = threadIdx.x; i < g.HW * (kChunk / 4); i += blockDim.x) dst[(size_t)(i >> 3) * rowq + (i & 7)] = src[i];
    P += slab_bits;
    __syncthreads();
  }
  if (threadIdx.x == 0 && ok && !raw) {
    const uint32_t code_bits = reinterpret_cast<const uint32_t*>(pay)[10];
    if (P != code_bits || s_bad_b) set_status(status, TACTKV_CORRUPT_PAYLOAD);
  }
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
#define TACTKV_LAUNCHER(h, w) TACTKV_CAT(TACTKV_CAT(TACTKV_CAT(launch_axis_hw_, h), _), w)
cudaError_t TACTKV_LAUNCHER(TACTKV_HCLASS, TACTKV_WCLASS)(bool inverse, int mode, const Geom& g, const UnitList& ul,
                                                      int nu, float* buf, float* partial, unsigned int* status,
                                                      cudaStream_t st) {
  const size_t sm = hw_smem_bytes(g.HW);
  const dim3 grid(g.nch, nu);
  if (inverse) {
    cudaFuncSetAttribute(idct_hw_kernel<TACTKV_HCLASS, TACTKV_WCLASS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    idct_hw_kernel<TACTKV_HCLASS, TACTKV_WCLASS><<<grid, kHwThreads, sm, st>>>(g, ul, mode, buf, status);
  } else {
    cudaFuncSetAttribute(fdct_hw_kernel<TACTKV_HCLASS, TACTKV_WCLASS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    fdct_hw_kernel<TACTKV_HCLASS, TACTKV_WCLASS><<<grid, kHwThreads, sm, st>>>(g, ul, mode, buf, partial);
  }
  return cudaGetLastError();
}

}  // namespace tactkv
