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
// carried to the next slab.  The next slab's coefficients are fetched with cp.async into a
// second buffer while the current one is transformed (when two buffers fit in shared memory).
//
// Both directions first compute the stream offset of every (k_s, k_h) pencil from the bit
// allocation, so no per-slab scan is needed; decoding (idct_hw) prefetches the stream words of
// slab k_s+1 while slab k_s is dequantized and put through the inverse DCTs along W and H.
//
// Compiled once per pair of length classes (TACTKV_HCLASS, TACTKV_WCLASS: 16 or 32 each).
#include "common.cuh"
#include "lloyd_max_tables.inc"

#if !defined(TACTKV_HCLASS) || !defined(TACTKV_WCLASS)
#error "TACTKV_HCLASS and TACTKV_WCLASS must be defined"
#endif

namespace tactkv {
namespace {

constexpr size_t kSmemBudget = 220 * 1024;
constexpr int kEnergyStride = kPairs + 1;   // padded row of per-pair energies: conflict-free both ways
constexpr int kMaxSlabs = 64;

__host__ __device__ inline int stream_words_per_slab(int HW) { return (8 * HW + 31) / 32 + 2; }

struct HwLayout {
  size_t tile, thr, lv, pen, meta, off, uni, carry, warp, bsl, sig2, total;
  size_t bsl_stride;
  int nbuf;
  int words;
};

enum LayoutKind { kLayStats = 0, kLayQuant = 1, kLayDecode = 2 };

// Shared memory carve-up of one launch.  stats: slab tiles and padded energy rows; quant: slab
// tiles, thresholds, pencil offsets, per-bin metadata, the bit widths and sigmas of two slabs
// and the stream words of a slab; decode: one tile, levels, the same metadata and two slabs of
// stream words.  Regions a kind does not use have size 0.
__host__ __device__ inline HwLayout hw_layout(int HW, int N, int S, int H, int kind) {
  HwLayout L;
  L.words = stream_words_per_slab(HW);
  const bool st = kind == kLayStats, qu = kind == kLayQuant, de = kind == kLayDecode;
  const size_t tile1 = (size_t)HW * kPairs * 8;
  const size_t energy = st ? (size_t)HW * kEnergyStride * 4 : 0;
  const size_t words = st ? 0 : (size_t)kChunk * L.words * 4 * (de ? 2 : 1);
  const size_t thr = qu ? kLmThrTotal * 4 : 0, lv = de ? kLmLvTotal * 4 : 0;
  const size_t pen = st ? 0 : ((size_t)S * H * 4 + 15) / 16 * 16;
  const size_t meta = st ? 0 : (size_t)HW * 8, off = st ? 0 : ((size_t)HW * 4 + 15) / 16 * 16;
  // a slab's bit widths are fetched as the 16-byte aligned window around them
  L.bsl_stride = ((size_t)HW + 15) / 16 * 16 + 32;
  const size_t bsl = st ? 0 : 2 * L.bsl_stride, sig2 = st ? 0 : (size_t)HW * 8;
  const size_t fixed = thr + lv + pen + meta + off + energy + words + kChunk * 4 + 33 * 4 + bsl + sig2 + 256;
  L.nbuf = (de || 2 * tile1 + fixed > kSmemBudget) ? 1 : 2;
  size_t o = 0;
  L.tile = o; o += tile1 * L.nbuf;
  L.uni = o; o += ((energy > words ? energy : words) + 15) / 16 * 16;
  L.bsl = o; o += bsl;
  L.thr = o; o += thr;
  L.lv = o; o += lv;
  L.pen = o; o += pen;
  L.meta = o; o += meta;
  L.off = o; o += off;
  L.sig2 = o; o += sig2;
  L.carry = o; o += kChunk * 4;
  L.warp = o; o += 33 * 4;
  L.total = o;
  return L;
}

// Lloyd-Max code: the number of thresholds t_j <= u (bisection over the 2^b - 1 thresholds).
__device__ __forceinline__ uint32_t lm_code(float u, int bits, const float* thr) {
  const float* t = thr + lm_thr_offset(bits);
  uint32_t code = 0;
  for (int step = 1 << (bits - 1); step > 0; step >>= 1)
    if (u >= t[code + step - 1]) code += step;
  return code;
}

// Code for u at 1, 2 or more bits (the count of thresholds t <= u).  The 1- and 2-bit codebooks
// have thresholds {0} and {-t, 0, t}: a sign test and three compares; wider ones use bisection.
__device__ __forceinline__ uint32_t quant_code(float u, int bits, const float* thr) {
  if (bits == 1) return u >= 0.f;
  if (bits == 2) {
    const float t = thr[lm_thr_offset(2) + 2];
    return (uint32_t)(u >= -t) + (uint32_t)(u >= 0.f) + (uint32_t)(u >= t);
  }
  return lm_code(u, bits, thr);
}

// Pencil DCTs along H of the tile: pencils (w, pair), stride W*16 between elements.
template <int CLASS, bool INV>
__device__ __forceinline__ void h_pass(const Geom& g, float2* tile) {
  const int step = g.W * kPairs;
  for (int p = threadIdx.x; p < g.W * kPairs; p += blockDim.x) {
    const int base = (p >> 4) * kPairs + (p & 15);
    float2 x[CLASS];
#pragma unroll
    for (int t = 0; t < CLASS; ++t)
      if (t < g.H) x[t] = tile[base + t * step];
    dct_pencil<CLASS, INV>(x, g.H);
#pragma unroll
    for (int t = 0; t < CLASS; ++t)
      if (t < g.H) tile[base + t * step] = x[t];
  }
}

// Copy one S slab of Y (HW rows of 32 channels, 128 bytes each) into a tile, asynchronously.
__device__ __forceinline__ void issue_tile(const Geom& g, const float4* ysrc_unit, int ks, float2* tile) {
  const int rowq = g.n / 4;
  const float4* src = ysrc_unit + (size_t)ks * g.HW * rowq;
  float4* dst = reinterpret_cast<float4*>(tile);
  for (int i = threadIdx.x; i < g.HW * (kChunk / 4); i += blockDim.x)
    cp_async16(dst + i, src + (size_t)(i >> 3) * rowq + (i & 7));
}

// The unit's bit widths into shared memory (16-byte copies: the payload and its b[] array are
// 16-byte aligned and padded), used once to compute the pencil offsets.
__device__ __forceinline__ void issue_bits(const Geom& g, const unsigned char* pay_b, unsigned char* dst) {
  for (int i = threadIdx.x; i < (g.N + 15) / 16; i += blockDim.x) cp_async16(dst + 16 * i, pay_b + 16 * i);
}
// The bit widths of slab ks as the 16-byte aligned window that holds them; they start at byte
// (ks * HW) % 16 of dst.  The window ends inside the padded b[] array.
__device__ __forceinline__ void issue_slab_bits(const Geom& g, const unsigned char* pay_b, int ks, unsigned char* dst) {
  const size_t a0 = (size_t)ks * g.HW, q0 = a0 / 16, q1 = (a0 + g.HW + 15) / 16;
  for (int i = threadIdx.x; i < (int)(q1 - q0); i += blockDim.x) cp_async16(dst + 16 * i, pay_b + 16 * (q0 + i));
}
// The sigmas of slab ks (4-byte copies).
__device__ __forceinline__ void issue_sigma(const Geom& g, const float* pay_sig, int ks, float* dst) {
  for (int j = threadIdx.x; j < g.HW; j += blockDim.x) cp_async4(dst + j, pay_sig + (size_t)ks * g.HW + j);
}

// Stream bit offset of every (k_s, k_h) pencil: the bits of each row of W bins, then an exclusive
// scan in bin order.  bfull: the unit's bit widths in shared memory.  Returns the total; sets
// *bad when a width exceeds 8.
__device__ __forceinline__ uint32_t pencil_offsets(const Geom& g, const unsigned char* bfull, uint32_t* pen,
                                                   uint32_t* swarp, unsigned int* bad) {
  const int npen = g.S * g.H;
  for (int p = threadIdx.x; p < npen; p += blockDim.x) {
    const unsigned char* b = bfull + (size_t)p * g.W;
    uint32_t t = 0;
    bool over = false;
    for (int w = 0; w < g.W; ++w) {
      const uint32_t v = b[w];
      over |= v > 8;
      t += v;
    }
    if (over) *bad = 1;
    pen[p] = t;
  }
  __syncthreads();
  return block_exclusive_scan(pen, npen, swarp);
}

// Bits, gain and stream bit offset of every bin of slab ks: one warp per (k_s, k_h) row of at most
// 32 bins, the offset being the row's start (pen) plus a shuffle scan of the row's bit widths.
// gain_inv: store 1/sigma (encoding) instead of sigma (decoding).
// bsl: this slab's bit widths in shared memory; sig: its sigmas.
__device__ __forceinline__ void slab_meta(const Geom& g, int ks, const unsigned char* bsl, const float* sig,
                                          const uint32_t* pen, uint32_t wbase, bool gain_inv, uint32_t* sb_bits,
                                          float* sb_gain, uint32_t* sb_off) {
  const int lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  for (int kh = threadIdx.x >> 5; kh < g.H; kh += nwarp) {
    const int j = kh * g.W + lane;
    const uint32_t b = lane < g.W ? bsl[j] : 0u;
    uint32_t incl = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane < g.W) {
      sb_bits[j] = b;
      sb_off[j] = pen[ks * g.H + kh] - wbase + incl - b;
      const float sg = sig[j];
      sb_gain[j] = gain_inv ? (b ? __frcp_rn(sg) : 0.f) : sg;
    }
  }
}

template <int HC, int WC, int MODE>
__global__ void __launch_bounds__(kHwThreads) fdct_hw_kernel(const __grid_constant__ Geom g,
                                                             const __grid_constant__ UnitList ul,
                                                             const float* __restrict__ Y, float* __restrict__ partial) {
  extern __shared__ __align__(16) unsigned char smem[];
  const HwLayout L = hw_layout(g.HW, g.N, g.S, g.H, MODE == kStats ? kLayStats : kLayQuant);
  float2* tiles = reinterpret_cast<float2*>(smem + L.tile);
  float* thr = reinterpret_cast<float*>(smem + L.thr);
  uint32_t* pen = reinterpret_cast<uint32_t*>(smem + L.pen);   // bit offset of every (k_s, k_h) pencil
  uint32_t* sb_bits = reinterpret_cast<uint32_t*>(smem + L.meta);  // this slab: bits of every bin
  float* sb_gain = reinterpret_cast<float*>(smem + L.meta) + g.HW;   // 1/sigma of every bin
  uint32_t* sb_off = reinterpret_cast<uint32_t*>(smem + L.off);      // bit offset in the slab's words
  unsigned char* bsl = smem + L.bsl;                                   // bit widths of two slabs
  float* sig2 = reinterpret_cast<float*>(smem + L.sig2);               // sigmas of two slabs
  float* energy = reinterpret_cast<float*>(smem + L.uni);
  uint32_t* sbuf = reinterpret_cast<uint32_t*>(smem + L.uni);
  uint32_t* carry = reinterpret_cast<uint32_t*>(smem + L.carry);
  uint32_t* swarp = reinterpret_cast<uint32_t*>(smem + L.warp);
  const int words = L.words;
  const int chunk = blockIdx.x, u = blockIdx.y;
  const UnitDev& ud = ul.u[u];
  unsigned char* pay = ud.payload;
  uint32_t* words_out = reinterpret_cast<uint32_t*>(pay + g.off_codes);
  const bool quant = MODE == kQuant;
  uint32_t cstride = 0, stride_words = 0;
  if (MODE != kStats) {  // written by the allocation kernel
    cstride = reinterpret_cast<const uint32_t*>(pay)[11];
    stride_words = cstride / 4;
  }
  const float4* ysrc = reinterpret_cast<const float4*>(Y + (size_t)u * g.S * g.HW * g.n) + chunk * (kChunk / 4);
  const unsigned char* pay_b = pay + kHeaderBytes;
  const float* pay_sig = reinterpret_cast<const float*>(pay + g.off_sigma);

  // The unit's bit widths, needed once for the pencil offsets, go to the tile buffer that slab 0
  // does not use; with a single buffer they go there first and slab 0 follows.
  unsigned char* bstage = reinterpret_cast<unsigned char*>(tiles + (L.nbuf == 2 ? (size_t)g.HW * kPairs : 0));
  if (!quant || L.nbuf == 2) issue_tile(g, ysrc, 0, tiles);
  if (quant) {
    issue_bits(g, pay_b, bstage);
    issue_slab_bits(g, pay_b, 0, bsl);
    issue_sigma(g, pay_sig, 0, sig2);
  }
  cp_async_commit();
  if (quant) {
    __shared__ unsigned int s_unused;
    for (int i = threadIdx.x; i < kLmThrTotal; i += blockDim.x) thr[i] = c_lm_thresholds[i];
    if (threadIdx.x < kChunk) carry[threadIdx.x] = 0;
    cp_async_wait_all();
    __syncthreads();
    pencil_offsets(g, bstage, pen, swarp, &s_unused);   // widths come from the allocation: all <= 8
    if (L.nbuf == 1) {  // every read of bstage is done
      issue_tile(g, ysrc, 0, tiles);
      cp_async_commit();
    }
  }
  uint32_t P = 0;  // stream bits written so far, identical for every channel
  for (int ks = 0; ks < g.S; ++ks) {
    const int cur = L.nbuf == 2 ? (ks & 1) : 0;
    float2* tile = tiles + (size_t)cur * g.HW * kPairs;
    cp_async_wait_all();
    __syncthreads();  // slab ks is in place and every thread is done with slab ks - 1
    if (L.nbuf == 2 && ks + 1 < g.S) issue_tile(g, ysrc, ks + 1, tiles + (size_t)(cur ^ 1) * g.HW * kPairs);
    if (quant && ks + 1 < g.S) {
      issue_slab_bits(g, pay_b, ks + 1, bsl + ((ks + 1) & 1) * L.bsl_stride);
      issue_sigma(g, pay_sig, ks + 1, sig2 + ((ks + 1) & 1) * g.HW);
    }
    if (ks + 1 < g.S && (L.nbuf == 2 || quant)) cp_async_commit();
    const uint32_t slab_end = quant ? (ks + 1 < g.S ? pen[(ks + 1) * g.H] : (uint32_t)0) : 0u;
    const uint32_t w0 = P >> 5;                 // first stream word this slab touches
    uint32_t slab_bits = 0;
    if (quant) {
      slab_bits = (ks + 1 < g.S ? slab_end : reinterpret_cast<const uint32_t*>(pay)[10]) - P;
      const int nw = (int)(((P & 31u) + slab_bits + 31) >> 5) + 1;
      for (int i = threadIdx.x; i < kChunk * nw; i += blockDim.x) {
        const int ch = i / nw, w = i - ch * nw;
        sbuf[ch * words + w] = w == 0 ? carry[ch] : 0u;
      }
      slab_meta(g, ks, bsl + (ks & 1) * L.bsl_stride + (((size_t)ks * g.HW) & 15), sig2 + (ks & 1) * g.HW, pen,
                w0 << 5, true, sb_bits, sb_gain, sb_off);
    }
    h_pass<HC, false>(g, tile);
    __syncthreads();
    // W pass fused with the per-bin epilogue.  Rows are dealt so that warp w takes k_h = w and
    // k_h = H-1-w: the low-frequency rows, which carry most of the code bits, pair with light ones.
    for (int p = threadIdx.x; p < g.H * kPairs; p += blockDim.x) {
      const int r = p >> 4, pair = p & 15;
      const int kh = (r & 1) ? g.H - 1 - (r >> 1) : (r >> 1);
      const int base = kh * g.W * kPairs + pair;
      float2 x[WC];
#pragma unroll
      for (int t = 0; t < WC; ++t)
        if (t < g.W) x[t] = tile[base + t * kPairs];
      dct_pencil<WC, false>(x, g.W);
      if (MODE == kStats) {
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < g.W) energy[(kh * g.W + t) * kEnergyStride + pair] = x[t].x * x[t].x + x[t].y * x[t].y;
      } else if (MODE == kRaw) {
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
        // the pencil's codes are contiguous in both channel streams: pack them in 64-bit
        // registers and OR whole words into the slab's stream buffer
        const int i0 = kh * g.W;
        const uint32_t o0 = sb_off[i0];
        uint32_t* r0 = sbuf + (2 * pair) * words + (o0 >> 5);
        uint32_t* r1 = r0 + words;
        unsigned long long a0 = 0, a1 = 0;
        uint32_t apos = o0 & 31u;
#pragma unroll
        for (int t = 0; t < WC; ++t) {
          if (t < g.W) {
            const int bits = (int)sb_bits[i0 + t];
            if (bits) {
              const float inv = sb_gain[i0 + t];
              a0 |= (unsigned long long)quant_code(x[t].x * inv, bits, thr) << apos;
              a1 |= (unsigned long long)quant_code(x[t].y * inv, bits, thr) << apos;
              apos += bits;
              if (apos >= 32) {
                atomicOr(r0++, (uint32_t)a0);
                atomicOr(r1++, (uint32_t)a1);
                a0 >>= 32;
                a1 >>= 32;
                apos -= 32;
              }
            }
          }
        }
        if (a0 | a1) {
          atomicOr(r0, (uint32_t)a0);
          atomicOr(r1, (uint32_t)a1);
        }
      }
    }
    __syncthreads();
    if (MODE == kStats) {
      float* dst = partial + ((size_t)u * g.nch + chunk) * g.N + (size_t)ks * g.HW;
      for (int j = threadIdx.x; j < g.HW; j += blockDim.x) {
        const float* e = energy + j * kEnergyStride;
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < kPairs; ++q) acc += e[q];
        dst[j] = acc;
      }
    } else if (quant) {
      // complete words go out now; the word holding the run's last bits carries over
      const uint32_t endbit = (P & 31u) + slab_bits;
      const int full = (int)(endbit >> 5);
      for (int i = threadIdx.x; i < kChunk * full; i += blockDim.x) {
        const int ch = i / full, w = i - ch * full;
        words_out[(size_t)(chunk * kChunk + ch) * stride_words + w0 + w] = sbuf[ch * words + w];
      }
      if (threadIdx.x < kChunk) carry[threadIdx.x] = (endbit & 31u) ? sbuf[threadIdx.x * words + full] : 0u;
      P += slab_bits;
    }
    if (L.nbuf == 1 && ks + 1 < g.S) {
      __syncthreads();  // everyone is done with the only tile
      issue_tile(g, ysrc, ks + 1, tiles);
      cp_async_commit();
    }
  }
  cp_async_wait_all();
  if (quant) {
    __syncthreads();
    // the last partial word, then zero padding up to the channel stride
    const uint32_t wlast = P >> 5;
    const int tail = (int)stride_words - (int)wlast;
    for (int i = threadIdx.x; i < kChunk * tail; i += blockDim.x) {
      const int ch = i / tail, w = i - ch * tail;
      words_out[(size_t)(chunk * kChunk + ch) * stride_words + wlast + w] = (w == 0) ? carry[ch] : 0u;
    }
  } else if (MODE == kRaw) {
    const int pad = (int)cstride - 4 * g.N;
    for (int i = threadIdx.x; i < kChunk * pad; i += blockDim.x) {
      const int ch = i / pad, b = i - ch * pad;
      pay[g.off_codes + (size_t)(chunk * kChunk + ch) * cstride + 4 * g.N + b] = 0;
    }
  }
}

// ----------------------------------------------------------------------------------- decode ---
template <int HC, int WC, int MODE>
__global__ void __launch_bounds__(kHwThreads) idct_hw_kernel(const __grid_constant__ Geom g,
                                                             const __grid_constant__ UnitList ul,
                                                             float* __restrict__ V, unsigned int* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  const HwLayout L = hw_layout(g.HW, g.N, g.S, g.H, kLayDecode);
  float2* tile = reinterpret_cast<float2*>(smem + L.tile);
  float* lvs = reinterpret_cast<float*>(smem + L.lv);
  uint32_t* pen = reinterpret_cast<uint32_t*>(smem + L.pen);   // first stream bit of every pencil
  uint32_t* sbufs = reinterpret_cast<uint32_t*>(smem + L.uni);
  uint32_t* swarp = reinterpret_cast<uint32_t*>(smem + L.warp);
  uint32_t* sb_bits = reinterpret_cast<uint32_t*>(smem + L.meta);  // this slab: bits of every bin
  float* sb_gain = reinterpret_cast<float*>(smem + L.meta) + g.HW;   // sigma of every bin
  uint32_t* sb_off = reinterpret_cast<uint32_t*>(smem + L.off);      // bit offset in the slab's words
  unsigned char* bsl = smem + L.bsl;                                   // bit widths of two slabs
  float* sig2 = reinterpret_cast<float*>(smem + L.sig2);               // sigmas of two slabs
  __shared__ int s_ok;
  __shared__ unsigned int s_bad;
  const int words = L.words;
  const int chunk = blockIdx.x, u = blockIdx.y;
  const UnitDev& ud = ul.u[u];
  const unsigned char* pay = ud.payload;
  const bool raw = MODE == kRaw;
  uint32_t code_bits = 0;
  if (threadIdx.x == 0) {
    // the header must describe exactly the unit the caller asked for
    const uint32_t* h32 = reinterpret_cast<const uint32_t*>(pay);
    const int32_t* i32 = reinterpret_cast<const int32_t*>(pay);
    const uint32_t ver_flags = h32[1], cb = h32[10], cs = h32[11];
    const unsigned long long total = *reinterpret_cast<const unsigned long long*>(pay + 48);
    bool ok = h32[0] == kMagic && (ver_flags & 0xffffu) == (uint32_t)kVersion &&
              ((ver_flags >> 16) & TACTKV_NO_QUANT) == (raw ? TACTKV_NO_QUANT : 0u) && i32[2] == ud.layer &&
              i32[3] == ud.kv && i32[4] == g.S && i32[5] == g.H && i32[6] == g.W && i32[7] == g.heads &&
              i32[8] == g.head_dim && i32[9] == g.bits;
    if (ok) {
      ok = (raw ? cb == 32u * (uint32_t)g.N : cb <= (uint32_t)g.bits * (uint32_t)g.N) &&
           (long long)cs == pad16(((long long)cb + 7) / 8) &&
           (long long)total == (long long)g.off_codes + (long long)g.n * cs && (long long)total <= g.capacity;
    }
    s_ok = ok;
    s_bad = 0;
  }
  for (int i = threadIdx.x; i < kLmLvTotal; i += blockDim.x) lvs[i] = c_lm_levels[i];
  __syncthreads();
  const bool ok0 = s_ok;
  const uint32_t stride_words = ok0 ? reinterpret_cast<const uint32_t*>(pay)[11] / 4 : 0u;
  if (ok0) code_bits = reinterpret_cast<const uint32_t*>(pay)[10];
  const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes);
  const unsigned char* pay_b = pay + kHeaderBytes;
  const float* pay_sig = reinterpret_cast<const float*>(pay + g.off_sigma);
  // every pencil's first stream bit, from the unit's bit widths staged in the (still unused) tile
  if (ok0 && !raw) {
    unsigned char* bstage = reinterpret_cast<unsigned char*>(tile);
    issue_bits(g, pay_b, bstage);
    issue_slab_bits(g, pay_b, 0, bsl);
    issue_sigma(g, pay_sig, 0, sig2);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    const uint32_t total = pencil_offsets(g, bstage, pen, swarp, &s_bad);
    __syncthreads();
    if (threadIdx.x == 0 && (total != code_bits || s_bad)) s_ok = 0;
  }
  __syncthreads();
  const bool ok = s_ok;
  if (threadIdx.x == 0 && !ok && chunk == 0) set_status(status, TACTKV_CORRUPT_PAYLOAD);
  const int ch0 = chunk * kChunk;
  auto slab_begin = [&](int ks) -> uint32_t { return ks < g.S ? pen[ks * g.H] : code_bits; };

  auto issue_words = [&](int ks, uint32_t* sb) {  // stream words of slab ks for the 32 channels
    const uint32_t p0 = slab_begin(ks), p1 = slab_begin(ks + 1);
    const uint32_t w0 = p0 >> 5;
    const int nw = (int)(((p0 & 31u) + (p1 - p0) + 31) >> 5);
    for (int i = threadIdx.x; i < kChunk * (nw + 1); i += blockDim.x) {
      const int ch = i / (nw + 1), w = i - ch * (nw + 1);
      const uint32_t word = w0 + w;
      if (w < nw && word < stride_words) cp_async4(sb + ch * words + w, streams + (size_t)(ch0 + ch) * stride_words + word);
      else sb[ch * words + w] = 0u;
    }
  };

  if (ok && !raw) {
    issue_words(0, sbufs);
    cp_async_commit();
  }
  float4* vdst = reinterpret_cast<float4*>(V + (size_t)u * g.S * g.HW * g.n) + chunk * (kChunk / 4);
  const int rowq = g.n / 4;
  for (int ks = 0; ks < g.S; ++ks) {
    const int mc = ks & 1;
    const uint32_t* sb = sbufs + (size_t)mc * kChunk * words;
    cp_async_wait_all();
    __syncthreads();  // slab ks's stream words are in place; slab ks - 1 is done
    if (ok && !raw && ks + 1 < g.S) {
      issue_words(ks + 1, sbufs + (size_t)(mc ^ 1) * kChunk * words);
      issue_slab_bits(g, pay_b, ks + 1, bsl + (mc ^ 1) * L.bsl_stride);
      issue_sigma(g, pay_sig, ks + 1, sig2 + (mc ^ 1) * g.HW);
      cp_async_commit();
    }
    const int i0s = ks * g.HW;
    const uint32_t wbase = raw ? 0u : (slab_begin(ks) >> 5) << 5;
    if (ok && !raw) {
      slab_meta(g, ks, bsl + mc * L.bsl_stride + (((size_t)ks * g.HW) & 15), sig2 + mc * g.HW, pen, wbase, false,
                sb_bits, sb_gain, sb_off);
      __syncthreads();
    }
    // dequantize in registers, fused with the inverse DCT along W: a thread takes one pencil (a
    // k_h row of W bins, two channels), whose codes are contiguous in both streams and are read
    // through 64-bit windows; rows are dealt as in encoding (k_h = w with k_h = H-1-w)
    for (int p = threadIdx.x; p < g.H * kPairs; p += blockDim.x) {
      const int r = p >> 4, pair = p & 15;
      const int kh = (r & 1) ? g.H - 1 - (r >> 1) : (r >> 1);
      const int base = kh * g.W * kPairs + pair;
      const int i0 = kh * g.W;
      float2 x[WC];
      if (!ok) {
#pragma unroll
        for (int t = 0; t < WC; ++t) x[t] = make_float2(0.f, 0.f);
      } else if (raw) {
        const float* st = reinterpret_cast<const float*>(streams);
        const int c = ch0 + 2 * pair;
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < g.W)
            x[t] = make_float2(st[(size_t)c * stride_words + i0s + i0 + t], st[(size_t)(c + 1) * stride_words + i0s + i0 + t]);
      } else {
        const uint32_t* row0 = sb + (2 * pair) * words;
        const uint32_t* row1 = row0 + words;
        const uint32_t o0 = sb_off[i0];
        uint32_t wi = o0 >> 5, pos = o0 & 31u;
        unsigned long long w0v = (unsigned long long)row0[wi] | ((unsigned long long)row0[wi + 1] << 32);
        unsigned long long w1v = (unsigned long long)row1[wi] | ((unsigned long long)row1[wi + 1] << 32);
#pragma unroll
        for (int t = 0; t < WC; ++t) {
          if (t < g.W) {
            const int bits = (int)sb_bits[i0 + t];
            float2 v = make_float2(0.f, 0.f);
            if (bits) {
              const uint32_t mask = (1u << bits) - 1u;
              const float* lv = lvs + lm_lv_offset(bits);
              const float sg = sb_gain[i0 + t];
              v = make_float2(sg * lv[(uint32_t)(w0v >> pos) & mask], sg * lv[(uint32_t)(w1v >> pos) & mask]);
              pos += bits;
              if (pos >= 32) {
                ++wi;
                const bool in = wi + 1 < (uint32_t)words;
                w0v = (w0v >> 32) | ((unsigned long long)(in ? row0[wi + 1] : 0u) << 32);
                w1v = (w1v >> 32) | ((unsigned long long)(in ? row1[wi + 1] : 0u) << 32);
                pos -= 32;
              }
            }
            x[t] = v;
          }
        }
      }
      dct_pencil<WC, true>(x, g.W);
#pragma unroll
      for (int t = 0; t < WC; ++t)
        if (t < g.W) tile[base + t * kPairs] = x[t];
    }
    __syncthreads();
    h_pass<HC, true>(g, tile);
    __syncthreads();
    float4* dst = vdst + (size_t)ks * g.HW * rowq;
    const float4* src = reinterpret_cast<const float4*>(tile);
    for (int i = threadIdx.x; i < g.HW * (kChunk / 4); i += blockDim.x) dst[(size_t)(i >> 3) * rowq + (i & 7)] = src[i];
  }
  cp_async_wait_all();
}

}  // namespace

#define TACTKV_CAT2(a, b) a##b
#define TACTKV_CAT(a, b) TACTKV_CAT2(a, b)
#define TACTKV_LAUNCHER(h, w) TACTKV_CAT(TACTKV_CAT(TACTKV_CAT(launch_axis_hw_, h), _), w)
cudaError_t TACTKV_LAUNCHER(TACTKV_HCLASS, TACTKV_WCLASS)(bool inverse, int mode, const Geom& g, const UnitList& ul,
                                                          int nu, float* buf, float* partial, unsigned int* status,
                                                          cudaStream_t st) {
  const HwLayout L = hw_layout(g.HW, g.N, g.S, g.H, inverse ? kLayDecode : (mode == kStats ? kLayStats : kLayQuant));
  const dim3 grid(g.nch, nu);
  constexpr int H = TACTKV_HCLASS, W = TACTKV_WCLASS;
  const int sm = (int)L.total;
  if (inverse) {
    if (mode == kRaw) {
      cudaFuncSetAttribute(idct_hw_kernel<H, W, kRaw>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
      idct_hw_kernel<H, W, kRaw><<<grid, kHwThreads, sm, st>>>(g, ul, buf, status);
    } else {
      cudaFuncSetAttribute(idct_hw_kernel<H, W, kQuant>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
      idct_hw_kernel<H, W, kQuant><<<grid, kHwThreads, sm, st>>>(g, ul, buf, status);
    }
  } else if (mode == kStats) {
    cudaFuncSetAttribute(fdct_hw_kernel<H, W, kStats>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    fdct_hw_kernel<H, W, kStats><<<grid, kHwThreads, sm, st>>>(g, ul, buf, partial);
  } else if (mode == kRaw) {
    cudaFuncSetAttribute(fdct_hw_kernel<H, W, kRaw>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    fdct_hw_kernel<H, W, kRaw><<<grid, kHwThreads, sm, st>>>(g, ul, buf, partial);
  } else {
    cudaFuncSetAttribute(fdct_hw_kernel<H, W, kQuant>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    fdct_hw_kernel<H, W, kQuant><<<grid, kHwThreads, sm, st>>>(g, ul, buf, partial);
  }
  return cudaGetLastError();
}

}  // namespace tactkv
