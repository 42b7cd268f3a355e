// Pieces of the DCT along the H and W axes (TACT-KV stage 2, after the S pass) with the per-bin
// energies of stage 3, and of the inverse with unpacking and dequantization (the decoding
// paragraph), shared by the H/W-axis kernels and the fused three-axis kernels.
//
// A CTA owns one (unit, 32-channel chunk, range of S slabs) and walks its slabs in order.  Lane l
// of every warp is channel l of the chunk, and a thread's float2 holds two pencils of that
// channel: two columns (w, w+1) in the pass along H, two rows (h, h+1) in the pass along W.  All
// lanes of a warp therefore work on the same frequency bins at the same time, and everything that
// depends on a bin (its bit width, its gain, where its code sits in the stream) is uniform across
// the warp.
//
// Forward (fdct_hw), per slab k_s: the slab's H*W x 32 coefficients of the S-transformed volume
// arrive by cp.async (the next slab's meanwhile); the DCT along H runs in place (a warp reads a
// column pair and writes it back into the same bytes as row pairs); the DCT along W runs on row
// pairs, writes the finished coefficients X back over the slab in global memory and sums X^2 over
// the 32 channels into partial[u][chunk][bin].
//
// Inverse (idct_hw), per slab: the slab's stream words arrive by cp.async (the next slab's
// meanwhile where there is room for a second slot; the common grids keep one slot and run more CTAs
// per SM instead); per-bin records give each bin's bits, gain and stream position; warp j decodes
// rows 2j and 2j+1 (unpack + dequantize in registers: a row whose codes fit in two stream words is
// read once and its codes shifted out of that 64-bit window), runs the inverse DCT along W and
// writes column pairs; then runs the inverse DCT along H on column pair j and stores the result into
// the fp32 volume V.
#pragma once
#include "common.cuh"
#include "lloyd_max_tables.inc"
static_assert(TACTKV_LV0_VEC * 4 >= tactkv::kLmLvTotal + 1, "level table");

namespace tactkv {
namespace {

constexpr size_t kSmemBudget = 220 * 1024;

enum LayoutKind { kLayStats = 0, kLayDecode = 2 };

struct HwLayout {
  size_t tile, tile_bytes, sbuf, meta, bsl, bsl_stride, sig, lv, total;
  int nbuf, words;
  int nslot;   // decode: slabs of stream words and records held at once (2: the next one prefetched)
};

__host__ __device__ inline int row_pairs(int L) { return (L + 1) >> 1; }

// One warp per column pair (pass along H) and per row pair (pass along W), at most 8 warps; with
// more pairs than warps, a warp takes several in turn.
constexpr int kMaxHwThreads = 256;
__host__ __device__ inline int hw_threads(int H, int W) {
  const int HP = row_pairs(H), WP = row_pairs(W), m = 32 * (HP > WP ? HP : WP);
  return m < kMaxHwThreads ? m : kMaxHwThreads;
}

// Shared memory of one launch.  A tile buffer holds a slab as cells of 32 floats on a grid of
// 2*ceil(H/2) rows of Wp = 2*ceil(W/2) cells (the padding row and column are never read), which
// also holds its row-pair (forward) or column-pair (inverse) rearrangement.  stats: the slab tiles
// (two when they fit, so the next slab loads while this one is transformed; the energies reuse
// the rearranged tile).  decode: one tile, the stream words and the records of two slabs, levels.  words (the stride of a channel's word row) is odd, so the 32
// lanes reading 32 channels' rows hit 32 different banks.
__host__ __device__ inline HwLayout hw_layout(int H, int W, int kind) {
  HwLayout L;
  const int HP = row_pairs(H), WP = row_pairs(W), HW = H * W;
  const bool de = kind == kLayDecode;
  L.tile_bytes = (size_t)(2 * HP) * (2 * WP) * 32 * 4;
  L.words = ((8 * HW + 31) / 32 + 3) | 1;
  const size_t words1 = (size_t)32 * L.words * 4, meta1 = (size_t)HW * 16;
  // the exact-size decode kernels of the common grids run four CTAs per SM: one slot then leaves
  // room for the fourth, which hides more latency than the prefetched slot did (measured on B200)
  // likewise two CTAs per SM for the exact 24 x 24 kernels (one slot or tile buffer each)
  const bool four_per_sm = (H == 16 && W == 16) || (H == 14 && W == 14) || (H == 8 && W == 8) || (H == 24 && W == 24);
  L.nslot = (de && (four_per_sm || (size_t)(2 * HP) * (2 * WP) * 128 + 2 * (words1 + meta1) + kLmLvTotal * 4 + 256 >
                                       kSmemBudget))
                ? 1
                : 2;
  const size_t words = de ? words1 * L.nslot : 0;
  const size_t meta = de ? meta1 * L.nslot : 0;       // records
  L.bsl_stride = 0;
  const size_t bsl = 0;
  const size_t sig = 0;
  const size_t lv = de ? (size_t)TACTKV_LV0_VEC * 16 : 0;   // a zero in front of the levels
  const size_t rest = words + meta + bsl + sig + lv + 256;
  L.nbuf = (de || (H == 24 && W == 24) || 2 * L.tile_bytes + rest > kSmemBudget) ? 1 : 2;
  // every region starts on a 16-byte boundary (cp.async of 16 bytes, 16-byte record loads)
  auto p16 = [](size_t x) { return (x + 15) / 16 * 16; };
  size_t o = 0;
  L.tile = o; o += p16(L.tile_bytes * L.nbuf);
  L.sbuf = o; o += p16(words);
  L.meta = o; o += p16(meta);
  L.sig = o; o += p16(sig);
  L.lv = o; o += p16(lv);
  L.bsl = o; o += p16(bsl);
  L.total = o;
  return L;
}


// Grid sizes of a launch.  HX, WX > 0 are exact lengths fixed at compile time (the common grids
// get their own kernels: straight-line transforms, no bounds tests); 0 takes them from the Geom.
// NX > 0 fixes the channel count n as well (constant strides: immediate address offsets).
template <int HX, int WX, int NX = 0>
struct Dims {
  static constexpr int hx = HX, wx = WX;
  int H, W, HW, n;
  __device__ __forceinline__ explicit Dims(const Geom& g)
      : H(HX ? HX : g.H), W(WX ? WX : g.W), HW((HX ? HX : g.H) * (WX ? WX : g.W)), n(NX ? NX : g.n) {}
};

// Pencil transform of length L (= EXACT when EXACT > 0) from length class CLASS.
template <int CLASS, int EXACT, bool INV, class V>
__device__ __forceinline__ void pencil(V* x, int L) {
  if constexpr (EXACT > 0) dct_exact<EXACT, INV>(x);
  else dct_pencil<CLASS, INV>(x, L);
}

// Copy one S slab of Y (H*W cells of 32 channels, 128 bytes each) into a tile with rows of Wp
// cells, asynchronously.
template <class D>
__device__ __forceinline__ void issue_tile(const D& g, const float* slab_src, float* tile) {
  const int Wp = 2 * row_pairs(g.W);
  for (int r = threadIdx.x >> 3; r < g.H; r += blockDim.x >> 3)      // blockDim.x is a multiple of 32
    for (int w = 0; w < g.W; ++w)
      cp_async16(tile + (r * Wp + w) * 32 + (threadIdx.x & 7) * 4,
                 slab_src + (size_t)(r * g.W + w) * g.n + (threadIdx.x & 7) * 4);
}


// Forward rearrangement.  The tile's cells (h, w) sit at cell index h*Wp + w.  After the pass
// along H, element (row pair kp, column w, channel c) = {X[2kp][w], X[2kp+1][w]} (float2) sits at
// float2 index ((2kp + (w & 1))*Wp + (w & ~1))*16 + c: the 256 bytes of cells (2kp + d, w0) and
// (2kp + d, w0 + 1) hold row pair kp of column w0 + d.  Those are bytes that column pair w0 itself
// read, so a warp rewrites its own column pair in place with no other warp involved.
__device__ __forceinline__ int rp_index(int Wp, int kp, int w) { return ((2 * kp + (w & 1)) * Wp + (w & ~1)) * 16; }

// Column pair (w0, w0+1): read, DCT along H, written back in place as row pairs.
template <int HC, class D>
__device__ __forceinline__ void h_pass_fwd(const D& g, float* tile, int w0, int lane, bool skip) {
  const int Wp = 2 * row_pairs(g.W), HP = row_pairs(g.H);
  float2 xh[HC];
#pragma unroll
  for (int h = 0; h < HC; ++h)
    if (h < g.H) {
      const float* cell = tile + (h * Wp + w0) * kChunk + lane;
      xh[h] = make_float2(cell[0], cell[kChunk]);   // column W (odd W) is padding: read, never used
    }
  __syncwarp();   // the whole column pair is read before any lane rewrites it
  if (!skip) pencil<HC, D::hx, false>(xh, g.H);
  float2* t2 = reinterpret_cast<float2*>(tile);
#pragma unroll
  for (int kp = 0; kp < (HC + 1) / 2; ++kp)
    if (kp < HP) {
      const float2 a = xh[2 * kp];
      const float2 b = (2 * kp + 1 < g.H) ? xh[2 * kp + 1] : make_float2(0.f, 0.f);
      t2[rp_index(Wp, kp, w0) + lane] = make_float2(a.x, b.x);
      t2[rp_index(Wp, kp, w0 + 1) + lane] = make_float2(a.y, b.y);
    }
}
// Row pair kp -> DCT along W.
template <int WC, class D>
__device__ __forceinline__ void w_load_fdct(const D& g, const float2* t2, int kp, int lane, float2 (&x)[WC],
                                            bool skip) {
  const int Wp = 2 * row_pairs(g.W);
#pragma unroll
  for (int t = 0; t < WC; ++t)
    if (t < g.W) x[t] = t2[rp_index(Wp, kp, t) + lane];
  if (!skip) pencil<WC, D::wx, false>(x, g.W);
}
// Energies of row pair kp summed over the warp's 32 channels and stored to dst (the slab's bins):
// the squares of rows 2kp and 2kp+1 go through the transpose sum 16 columns at a time, so that
// lane l ends with column (l & 15) of row 2kp + (l >> 4) of that group of columns.
template <int WC, class D>
__device__ __forceinline__ void store_energy(const D& g, int kp, int lane, const float2 (&x)[WC], float* dst) {
  const int row = 2 * kp + (lane >> 4);
#pragma unroll
  for (int t0 = 0; t0 < WC; t0 += 16) {
    float v[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 e = t0 + j < g.W ? __fmul2_rn(x[t0 + j], x[t0 + j]) : make_float2(0.f, 0.f);
      v[j] = e.x;
      v[16 + j] = e.y;
    }
    const float sum = warp_transpose_sum(v, lane);
    const int t = t0 + (lane & 15);
    if (t < g.W && row < g.H) dst[row * g.W + t] = sum;
  }
}

// Pass 1 of compression: the 3D DCT is completed (H and W after the S pass) and written back over
// the S-transformed slab, and the per-bin energies are summed over the CTA's 32 channels.  The
// packing kernel then quantizes the finished coefficients without transforming anything.
// Slabs [ks0, ks1) of channel chunk `chunk` of unit u; called by every thread of the CTA.  EF: the
// stores of X are marked evict-first in L2 (X is read again only by the packing kernel).
template <int HC, int WC, int HX, int WX, bool EF, int NX = 0, bool VAR = false>
__device__ __forceinline__ void fdct_hw_slabs(const Geom& g, float* __restrict__ Y, float* __restrict__ partial, int u,
                                              int chunk, int ks0, int ks1, unsigned char* smem) {
  const Dims<HX, WX, NX> D(g);
  const HwLayout L = hw_layout(D.H, D.W, kLayStats);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int HP = row_pairs(D.H), WP = row_pairs(D.W);
  float* yunit = Y + (size_t)u * g.S * D.HW * D.n + chunk * kChunk;
  auto tile_of = [&](int ks) {
    return reinterpret_cast<float*>(smem + L.tile + (L.nbuf == 2 ? (ks & 1) : 0) * L.tile_bytes);
  };

  issue_tile(D, yunit + (size_t)ks0 * D.HW * D.n, tile_of(ks0));
  cp_async_commit();
  for (int ks = ks0; ks < ks1; ++ks) {
    float* tile = tile_of(ks);
    float* yslab = yunit + (size_t)ks * D.HW * D.n + lane;
    cp_async_wait_all();
    __syncthreads();  // slab ks is in place; every thread is done with slab ks - 1
    if (L.nbuf == 2 && ks + 1 < ks1) {
      issue_tile(D, yunit + (size_t)(ks + 1) * D.HW * D.n, tile_of(ks + 1));
      cp_async_commit();
    }
    // DCT along H, in place, one column pair at a time per warp
    for (int wp = warp; wp < WP; wp += nwarps) h_pass_fwd<HC>(D, tile, 2 * wp, lane, VAR && (g.flags & TACTKV_SKIP_H));
    __syncthreads();
    float2* t2 = reinterpret_cast<float2*>(tile);
    // DCT along W on row pair kp; the coefficients go back over the slab of Y (this CTA's own
    // bytes), their squares summed over the 32 channels to the slab's bins of partial
    float* dst = partial + ((size_t)u * (NX ? NX / kChunk : g.nch) + chunk) * g.N + (size_t)ks * D.HW;
    for (int kp = warp; kp < HP; kp += nwarps) {
      float2 x[WC];
      w_load_fdct<WC>(D, t2, kp, lane, x, VAR && (g.flags & TACTKV_SKIP_W));
      const bool second = 2 * kp + 1 < D.H;
      float* y0 = yslab + (size_t)(2 * kp * D.W) * D.n;
      if constexpr (EF) {
        const uint64_t pol = l2_evict_first();
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < D.W) {
            st_ef(y0 + (size_t)t * D.n, x[t].x, pol);
            if (second) st_ef(y0 + (size_t)(D.W + t) * D.n, x[t].y, pol);
          }
      } else {
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < D.W) {
            y0[(size_t)t * D.n] = x[t].x;
            if (second) y0[(size_t)(D.W + t) * D.n] = x[t].y;
          }
      }
      store_energy<WC>(D, kp, lane, x, dst);
    }
    if (L.nbuf == 1 && ks + 1 < ks1) {
      __syncthreads();  // everyone is done with the only tile
      issue_tile(D, yunit + (size_t)(ks + 1) * D.HW * D.n, tile_of(ks + 1));
      cp_async_commit();
    }
  }
  cp_async_wait_all();
}


// Column-pair element (h, column pair wp, channel c) = {X[h][2wp], X[h][2wp+1]} at float2 index
// (h*Wp + 2wp)*16 + c: rows 2kp and 2kp+1 of the cell grid hold row pair kp (forward
// rearrangement) and its column pairs alike, so the inverse pass along W rewrites its row pair
// in place.
__device__ __forceinline__ int cp_index(int Wp, int h, int wp) { return (h * Wp + 2 * wp) * 16; }

// Per slab: the stream words and the slab's dense records (per row pair and column: sigma and
// code offset within the slab's words of the two rows' bins) arrive by cp.async, the next slab's
// meanwhile.  Warp kp decodes rows 2kp and 2kp+1 in registers and runs the inverse DCT along W,
// writing column pairs; then the inverse DCT along H runs on column pairs, into the fp32 volume V.
// PAIRS: instead of fp32 V[u][k_s][cell][c], write the result as bf16 pairs for the tensor-core
// inverse along S: V_hi[u][k_s][cell pair][c] = (bf16(v[2p]), bf16(v[2p+1])) over V (as
// __nv_bfloat162) and the remainders V_lo = bf16(v - float(V_hi)) over Vlo (W even).  Together
// they carry v to about 2^-17 relative.
template <int HC, int WC, int HX, int WX, int MODE, bool PAIRS = false, bool VAR = false, int NX = 0>
__device__ __forceinline__ void idct_hw_slabs(const Geom& g, const UnitList& ul, float* __restrict__ V,
                                              const uint32_t* __restrict__ index, const uint4* __restrict__ recs, int u,
                                              int chunk, int ks0, int ks1, unsigned char* smem,
                                              __nv_bfloat162* __restrict__ Vlo = nullptr) {
  const Dims<HX, WX, NX> D(g);
  constexpr bool raw = MODE == kRaw;
  const HwLayout L = hw_layout(D.H, D.W, kLayDecode);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int HP = row_pairs(D.H), WP = row_pairs(D.W), Wp = 2 * WP;
  const unsigned char* pay = ul.u[u].payload;
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const bool ok = P[g.S + 1] != 0;   // the index kernel checked the header and the bit widths
  // the shared rotation's inverse (variant kernels only): sign of this lane's channel / sqrt(32)
  const bool rotate = VAR && MODE == kQuant && (g.flags & TACTKV_ROTATE);
  // per-head gains (variant kernels only): this chunk's head's sigma[bin], else the records' gains
  const float* hgain = (VAR && MODE == kQuant && head_gains_on(g.flags))
                           ? reinterpret_cast<const float*>(pay + g.off_sigma) + (size_t)(chunk * kChunk / g.head_dim) * g.N
                           : nullptr;
  const float rot_scale = rotate ? rotation_sign((unsigned long long)(chunk * kChunk + lane)) * 0.17677669529663687f : 1.f;
  const uint32_t cstride = ok ? reinterpret_cast<const uint32_t*>(pay)[11] : 0u, sw = cstride / 4;
  const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes) + (size_t)chunk * kChunk * sw;
  const uint4* urecs = recs + (size_t)u * g.N;
  float2* tile = reinterpret_cast<float2*>(smem + L.tile);
  float* lvs = reinterpret_cast<float*>(smem + L.lv);
  auto slot = [&](int ks) { return L.nslot == 2 ? (ks & 1) : 0; };
  auto sbuf_of = [&](int ks) { return reinterpret_cast<uint32_t*>(smem + L.sbuf) + slot(ks) * kChunk * L.words; };
  auto rbuf_of = [&](int ks) { return reinterpret_cast<uint4*>(smem + L.meta) + slot(ks) * D.HW; };

  // stream words of slab ks for the 32 channels from word P(ks) >> 5 on, then two zero words for
  // the look-ahead of the code reads; and the slab's records
  auto issue_slab = [&](int ks) {
    uint32_t* sb = sbuf_of(ks);
    const uint32_t p0 = P[ks], p1 = P[ks + 1];
    const uint32_t w0 = p0 >> 5;
    const int nw = (int)(((p0 & 31u) + (p1 - p0) + 31) >> 5);
    for (int c = warp; c < kChunk; c += nwarps)
      for (int w = lane; w < nw + 2; w += 32) {
        if (w < nw) cp_async4(sb + c * L.words + w, streams + (size_t)c * sw + w0 + w);
        else sb[c * L.words + w] = 0u;
      }
    const int RP = row_pairs(D.H) * D.W;   // dense records of the slab
    uint4* rb = rbuf_of(ks);
    for (int e = threadIdx.x; e < RP; e += blockDim.x) cp_async16(rb + e, urecs + (size_t)ks * RP + e);
  };
  if (!raw) {
    for (int i = threadIdx.x; i < TACTKV_LV0_VEC; i += blockDim.x) cp_async16(lvs + 4 * i, g_lm_levels0 + 4 * i);
    if (ok) issue_slab(ks0);
    cp_async_commit();
  }
  float* vunit = V + (size_t)u * g.S * D.HW * D.n + chunk * kChunk + lane;

  for (int ks = ks0; ks < ks1; ++ks) {
    cp_async_wait_all();
    __syncthreads();  // slab ks's words and records are in place; slab ks - 1 is done
    if (L.nslot == 2 && ok && !raw && ks + 1 < ks1) {
      issue_slab(ks + 1);
      cp_async_commit();
    }
    // decode rows 2kp, 2kp+1 of warp kp (dequantize in registers) and run the inverse DCT along W;
    // column pairs go to the tile
    const uint4* rs = rbuf_of(ks);
    const uint32_t* row = sbuf_of(ks) + lane * L.words;   // this lane's channel stream
    for (int kp = warp; kp < HP; kp += nwarps) {
      float2 x[WC];
      if (!ok) {
#pragma unroll
        for (int t = 0; t < WC; ++t) x[t] = make_float2(0.f, 0.f);
      } else if (raw) {
        const float* s = reinterpret_cast<const float*>(pay + g.off_codes + (size_t)(chunk * kChunk + lane) * cstride) +
                         (size_t)ks * D.HW + 2 * kp * D.W;
        const bool second = 2 * kp + 1 < D.H;
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < D.W) x[t] = make_float2(s[t], second ? s[D.W + t] : 0.f);
      } else {
        // lvs1[-1] is the zero in front of the levels: a bin without bits (mask 0) reads it, so
        // every code is read the same way, without a branch
        const float* lvs1 = lvs + 1;
        // record: sigma of each row, shift << 26 | offset << 8 | code mask of each row
        const uint4* rr = rs + kp * D.W;
        // Each row's bins are consecutive in the stream: from its first bin's offset to its last
        // bin's offset plus its bits.  When each row's bits lie in two stream words (most rows at
        // 1-3 bits per element), those words are read once and every code is shifted out of them
        // by the shift its record carries.
        const uint4 mf = rr[0], ml = rr[D.W - 1];
        const uint32_t base0 = (mf.z >> 8) & 0x3ffe0u, base1 = (mf.w >> 8) & 0x3ffe0u;
        const uint32_t end0 = ((ml.z >> 8) & 0x3ffffu) + (uint32_t)__popc(ml.z & 0xffu);
        const uint32_t end1 = ((ml.w >> 8) & 0x3ffffu) + (uint32_t)__popc(ml.w & 0xffu);
        if (end0 <= base0 + 64u && end1 <= base1 + 64u) {
          const unsigned long long win0 = ((unsigned long long)row[(base0 >> 5) + 1] << 32) | row[base0 >> 5];
          const unsigned long long win1 = ((unsigned long long)row[(base1 >> 5) + 1] << 32) | row[base1 >> 5];
#pragma unroll
          for (int t = 0; t < WC; ++t)
            if (t < D.W) {
              const uint4 m = rr[t];
              const uint32_t k0 = m.z & 0xffu, k1 = m.w & 0xffu;
              // (a bin without bits has mask 0 whatever its shift)
              const uint32_t c0 = (uint32_t)(win0 >> (m.z >> 26)) & k0;
              const uint32_t c1 = (uint32_t)(win1 >> (m.w >> 26)) & k1;
              const float l0 = lvs1[(int)(k0 + c0) - 1], l1 = lvs1[(int)(k1 + c1) - 1];
              float s0 = __uint_as_float(m.x), s1 = __uint_as_float(m.y);
              if (VAR && hgain) {   // (a row without bits keeps its gain 0; the padding row reads nothing)
                const size_t i0 = (size_t)ks * D.HW + (size_t)(2 * kp) * D.W + t;
                s0 = k0 ? __ldg(hgain + i0) : 0.f;
                s1 = k1 ? __ldg(hgain + i0 + D.W) : 0.f;
              }
              x[t] = __fmul2_rn(make_float2(l0, l1), make_float2(s0, s1));
            }
        } else {
#pragma unroll
          for (int t = 0; t < WC; ++t)
            if (t < D.W) {
              const uint4 m = rr[t];
              const uint32_t k0 = m.z & 0xffu, k1 = m.w & 0xffu;
              // offsets from the slab's first word
              const uint32_t off0 = (m.z >> 8) & 0x3ffffu, off1 = (m.w >> 8) & 0x3ffffu;
              const uint32_t* w0 = row + (off0 >> 5);
              const uint32_t* w1 = row + (off1 >> 5);
              const float l0 = lvs1[(int)(k0 + (__funnelshift_r(w0[0], w0[1], off0) & k0)) - 1];
              const float l1 = lvs1[(int)(k1 + (__funnelshift_r(w1[0], w1[1], off1) & k1)) - 1];
              float s0 = __uint_as_float(m.x), s1 = __uint_as_float(m.y);
              if (VAR && hgain) {
                const size_t i0 = (size_t)ks * D.HW + (size_t)(2 * kp) * D.W + t;
                s0 = k0 ? __ldg(hgain + i0) : 0.f;
                s1 = k1 ? __ldg(hgain + i0 + D.W) : 0.f;
              }
              x[t] = __fmul2_rn(make_float2(l0, l1), make_float2(s0, s1));
            }
        }
      }
      if (rotate) {   // R^T = diag(s) H_32 / sqrt(32) across the warp's 32 channels, both rows
#pragma unroll
        for (int t = 0; t < WC; ++t)
          if (t < D.W)
            x[t] = make_float2(warp_wht(x[t].x, lane) * rot_scale, warp_wht(x[t].y, lane) * rot_scale);
      }
      if (!VAR || !(g.flags & TACTKV_SKIP_W)) pencil<WC, WX, true>(x, D.W);
      const bool second = 2 * kp + 1 < D.H;
#pragma unroll
      for (int wp = 0; wp < (WC + 1) / 2; ++wp)
        if (wp < WP) {
          const float2 a = x[2 * wp];
          const float2 b = (2 * wp + 1 < D.W) ? x[2 * wp + 1] : make_float2(0.f, 0.f);
          tile[cp_index(Wp, 2 * kp, wp) + lane] = make_float2(a.x, b.x);
          if (second) tile[cp_index(Wp, 2 * kp + 1, wp) + lane] = make_float2(a.y, b.y);
        }
    }
    __syncthreads();
    // the words and records of slab ks are used up: with a single slot, the next slab's load
    // starts now and overlaps the pass along H and the stores
    if (L.nslot == 1 && ok && !raw && ks + 1 < ks1) {
      issue_slab(ks + 1);
      cp_async_commit();
    }
    // inverse DCT along H on column pair wp; store to V
    for (int wp = warp; wp < WP; wp += nwarps) {
      float2 xh[HC];
#pragma unroll
      for (int h = 0; h < HC; ++h)
        if (h < D.H) xh[h] = tile[cp_index(Wp, h, wp) + lane];
      if (!VAR || !(g.flags & TACTKV_SKIP_H)) pencil<HC, HX, true>(xh, D.H);
      if constexpr (PAIRS) {
        // pair (cell h*W + 2wp, cell h*W + 2wp + 1) = pair index h*(W/2) + wp
        const size_t base = ((size_t)u * g.S + ks) * (D.HW / 2) * g.n + chunk * kChunk + lane;
        __nv_bfloat162* vh = reinterpret_cast<__nv_bfloat162*>(V) + base + (size_t)wp * g.n;
        __nv_bfloat162* vl = Vlo + base + (size_t)wp * g.n;
#pragma unroll
        for (int h = 0; h < HC; ++h)
          if (h < D.H) {
            const __nv_bfloat162 hi = __floats2bfloat162_rn(xh[h].x, xh[h].y);
            const float2 back = __bfloat1622float2(hi);
            const size_t o = (size_t)h * (D.W / 2) * g.n;
            vh[o] = hi;
            vl[o] = __floats2bfloat162_rn(xh[h].x - back.x, xh[h].y - back.y);
          }
      } else {
        float* v = vunit + ((size_t)ks * D.HW + 2 * wp) * D.n;
        const bool two = 2 * wp + 1 < D.W;
#pragma unroll
        for (int h = 0; h < HC; ++h)
          if (h < D.H) {
            float* cell = v + (size_t)h * D.W * D.n;
            cell[0] = xh[h].x;
            if (two) cell[D.n] = xh[h].y;
          }
      }
    }
  }
  cp_async_wait_all();
}


}  // namespace
}  // namespace tactkv
