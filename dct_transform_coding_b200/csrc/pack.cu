// Quantization and bit packing (TACT-KV stage 4: gain-shape scalar quantization with the fixed
// Lloyd-Max codebook at each bin's bit width), on the finished 3D-DCT coefficients X.
//
// The allocation kernel lists, once per unit, every bin that received bits, in bin order, as a
// 16-byte record {bin, bits, first stream bit P_i, 1/sigma_i}; P_i = sum of the bits of every
// earlier bin, the same in every channel's stream.  A CTA owns one (unit, CPL consecutive 32-channel
// chunks, range of records); lane l of a warp packs channel l of each of its CPL chunks, so every
// decision about a record is uniform across the warp and only the coefficient values differ.  CPL
// is 4 on the default path (a record's position, width and gain are read and turned into a word and
// a shift once for four channels; ranges of kPackRecs records) and 1 for the variant kernels and for
// channel counts whose chunks do not come in fours (ranges of 4 * kPackRecs).  Bins without bits are
// never read.
//
// The CTA clears the word rows of its bit span in shared memory and puts its records there grouped
// by bit width (records are independent of each other: each carries its stream position), each
// group padded to whole blocks.  Each warp takes blocks of records of one width (quantized by code
// specialised for 1 bit, 2 bits, or 3 and more bits by table); while it quantizes one block, the
// coefficient rows (128 bytes each) of its next block are in flight.  For a record it computes
// u = X * (1/sigma) and the code, and ORs the code into the channel's word row at its stream
// position (a shared-memory reduction).  The span's words are then stored once; its first and last
// words may hold bits of the neighbouring ranges, and there the range clears its own bit field and
// ORs its codes in atomically.  The CTA with the last record also writes the zero padding of the
// channel streams.
//
// With TACTKV_ROTATE every record's 32 coefficients (one bin, the CTA's 32 channels) are first
// rotated by R = H_32 diag(s) / sqrt(32) across the warp (sign, Walsh-Hadamard, scale).  With
// TACTKV_HEAD_GAIN the scale of a record is the reciprocal of its bin's gain in the CTA's head.
//
// NO_QUANT (raw) copies X into the channel streams as float32.
#include "common.cuh"
#include "lloyd_max_tables.inc"

namespace tactkv {
namespace {

constexpr int kPackThreads = 256;
constexpr int kPackRows = 16;   // coefficient rows per warp step (blocks of 16 / CPL records)

template <int CPL>
__host__ __device__ constexpr int pack_recs() { return 4 * kPackRecs / CPL; }   // records per range
template <int CPL>
__host__ __device__ constexpr int pack_block() { return kPackRows / CPL; }      // records per block
// Words of a channel's row: a range spans at most 8 * R + 31 bits from its first word; then a word
// for the padding records' codes and one for their carry; odd, so that the 32 lanes' rows at one
// offset fall in 32 different banks.
template <int CPL>
__host__ __device__ constexpr int pack_words() { return ((8 * pack_recs<CPL>() + 31) / 32 + 3) | 1; }
template <int CPL>
__host__ __device__ constexpr int pack_pad_word() { return (8 * pack_recs<CPL>() + 31) / 32 + 1; }
static_assert(pack_pad_word<1>() + 2 <= pack_words<1>() && pack_pad_word<4>() + 2 <= pack_words<4>(), "rows");

struct PackLayout {
  size_t rec, sbuf, thr2, qcell, total;
};
// A range's records grouped by bit width, each group padded to whole blocks; then the word rows of
// the CPL * 32 channels and the codebook tables.
template <int CPL>
__host__ __device__ inline PackLayout pack_layout() {
  PackLayout L;
  auto p16 = [](size_t x) { return (x + 15) / 16 * 16; };
  size_t o = 0;
  L.rec = o; o += p16((size_t)(pack_recs<CPL>() + 8 * pack_block<CPL>()) * 16);
  L.sbuf = o; o += p16((size_t)CPL * kChunk * pack_words<CPL>() * 4);
  L.thr2 = o; o += (size_t)TACTKV_THR_PAIR_VEC * 16;
  L.qcell = o; o += (size_t)TACTKV_QCELL_VEC * 16;
  L.total = o;
  return L;
}

// Code of u at b bits: the number of thresholds t_j <= u (float32 compares, ties go up).  B is
// the width when fixed at compile time (1 or 2), 0 for a width b >= 3 known at run time.  b = 1:
// the sign test, which needs no gain (1/sigma is positive and finite, so u >= 0 exactly when
// x >= 0); b = 2: three compares against {-t, 0, t}; b >= 3: the cell of u in a uniform grid gives
// the count c of thresholds below the cell, and two compares finish it (a cell holds at most two
// thresholds; the thresholds are padded with +inf), against the pair (t_c, t_{c+1}) read in one
// load (pair 2^b - 8 + c).  The cell index saturates: the conversion to unsigned takes values
// below the grid to 0, min() those above it to the last cell.
template <int B>
__device__ __forceinline__ uint32_t quant_code_b(float x, float inv_sigma, int b, const float2* __restrict__ thr2,
                                                 const unsigned char* __restrict__ qcell) {
  if constexpr (B == 1) {
    return x >= 0.f;
  } else {
    const float u = x * inv_sigma;
    if constexpr (B == 2) {
      return (uint32_t)(u >= -TACTKV_LM_T2) + (uint32_t)(u >= 0.f) + (uint32_t)(u >= TACTKV_LM_T2);
    } else {
      const uint32_t j = min(__float2uint_rd(fmaf(u, TACTKV_Q_SCALE, TACTKV_Q_OFFSET)), TACTKV_Q_CELLS - 1u);
      const uint32_t c = qcell[(b - 3) * TACTKV_Q_CELLS + j];
      const float2 t = thr2[(1 << b) - 8 + c];
      return c + (uint32_t)(u >= t.x) + (uint32_t)(u >= t.y);
    }
  }
}

// OR into a shared-memory word without reading the old value back (a reduction, not an atomic
// with a result): nothing waits for it, so consecutive codes of a warp do not stall on each other.
__device__ __forceinline__ void red_or_shared(uint32_t* p, uint32_t v) {
  asm volatile("red.shared.or.b32 [%0], %1;\n" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(v)
               : "memory");
}

// One block of PB records, all of width b (= B when B > 0): quantize x[][] (record j, chunk k of
// the lane's CPL channels) and OR the codes into the rows (row + k * 32 rows; a code of more than
// one bit may straddle into the next word).  In three phases -- the block's records, then its
// codes, then the ORs -- so that the loads of one phase are all in flight together instead of each
// waiting behind the previous record's OR.
template <int B, int CPL, int PB>
__device__ __forceinline__ void pack_block(const uint4* __restrict__ rs, const float (&x)[PB][CPL],
                                           uint32_t* __restrict__ row, uint32_t base, int b,
                                           const float2* __restrict__ thr2, const unsigned char* __restrict__ qcell) {
  constexpr int kRowStride = kChunk * pack_words<CPL>();
  uint2 r[PB];
#pragma unroll
  for (int j = 0; j < PB; ++j) r[j] = reinterpret_cast<const uint2*>(rs + j)[1];   // {position, 1/sigma}
  uint32_t code[PB][CPL];
#pragma unroll
  for (int j = 0; j < PB; ++j)
#pragma unroll
    for (int k = 0; k < CPL; ++k) code[j][k] = quant_code_b<B>(x[j][k], __uint_as_float(r[j].y), b, thr2, qcell);
#pragma unroll
  for (int j = 0; j < PB; ++j) {
    const uint32_t off = r[j].x - base, w = off >> 5, sh = off & 31u;
    uint32_t* rw = row + w;
#pragma unroll
    for (int k = 0; k < CPL; ++k) red_or_shared(rw + k * kRowStride, code[j][k] << sh);
    if constexpr (B != 1) {
      if (sh + (uint32_t)b > 32u) {
#pragma unroll
        for (int k = 0; k < CPL; ++k) red_or_shared(rw + k * kRowStride + 1, code[j][k] >> (32u - sh));
      }
    }
  }
}

// VAR: the payload has variant flags (the shared rotation, per-head gains), a compile-time switch
// so that the default kernel keeps its register budget; the variant kernel packs one channel per
// lane (CPL = 1), since a rotation mixes the 32 channels of one chunk and a head gain is per head.
template <bool VAR, int CPL>
__global__ void __launch_bounds__(kPackThreads, 4) pack_kernel(const __grid_constant__ Geom g,
                                                            const __grid_constant__ UnitList ul,
                                                            const float* __restrict__ X, const uint4* __restrict__ recs,
                                                            const uint32_t* __restrict__ index) {
  static_assert(!VAR || CPL == 1, "variant kernels pack one channel per lane");
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int kWarps = kPackThreads / 32;
  constexpr int R = pack_recs<CPL>(), PB = pack_block<CPL>(), kWords = pack_words<CPL>();
  constexpr int kChan = CPL * kChunk;   // channels of the CTA
  __shared__ uint32_t s_cnt[9][kWarps];   // per bit width and warp: record counts, then first slots
  __shared__ uint32_t s_fill[9];          // end of each width's records
  __shared__ uint32_t s_grp[10];          // first slot of each width's group; s_grp[9]: all slots
  const PackLayout L = pack_layout<CPL>();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk0 = blockIdx.x * CPL, u = blockIdx.z;
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const uint32_t nrec = P[2 * g.S + 2], code_bits = P[g.S];      // NZ(S) and P(S)
  const uint32_t r0 = blockIdx.y * R;
  if (r0 >= nrec && !(r0 == 0 && nrec == 0)) return;             // (range 0 also pads an empty unit)
  const uint32_t r1 = min(nrec, r0 + R);
  const int m = (int)(r1 - r0);
  unsigned char* pay = ul.u[u].payload;
  const uint4* urecs = recs + (size_t)u * g.N;
  const float* xu = X + (size_t)u * g.N * g.n + chunk0 * kChunk + lane;
  uint4* rs = reinterpret_cast<uint4*>(smem + L.rec);
  uint32_t* sbuf = reinterpret_cast<uint32_t*>(smem + L.sbuf);
  float2* thr2 = reinterpret_cast<float2*>(smem + L.thr2);
  unsigned char* qcell = smem + L.qcell;
  const uint32_t cstride = reinterpret_cast<const uint32_t*>(pay)[11], sw = cstride / 4;
  uint32_t* words_out = reinterpret_cast<uint32_t*>(pay + g.off_codes) + (size_t)chunk0 * kChunk * sw;

  // Thread t holds records t, t + 256, ... of the range (empty slots past m have width 0).
  constexpr int kPer = (R + kPackThreads - 1) / kPackThreads;
  uint4 mine[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int e = q * kPackThreads + (int)threadIdx.x;
    mine[q] = e < m ? urecs[r0 + e] : make_uint4(0u, 0u, 0u, 0u);
  }
  if (VAR && head_gains_on(g.flags)) {   // 1/gain of the CTA's head (0 for a zero gain: u = 0)
    const float* hg =
        reinterpret_cast<const float*>(pay + g.off_sigma) + (size_t)(chunk0 * kChunk / g.head_dim) * g.N;
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (mine[q].y) {
        const float gh = hg[mine[q].x];
        mine[q].w = gh > 0.f ? __float_as_uint(__frcp_rn(gh)) : 0u;
      }
  }
  if (threadIdx.x < 9 * kWarps) (&s_cnt[0][0])[threadIdx.x] = 0u;
  copy_vec16(thr2, g_thr_pairs, TACTKV_THR_PAIR_VEC);
  copy_vec16(qcell, g_qcell, TACTKV_QCELL_VEC);
  // bit span [A, B) of the range; its words from word A >> 5 on are assembled in shared memory
  const uint32_t A = m > 0 ? urecs[r0].z : code_bits;
  const uint32_t B = r1 < nrec ? urecs[r1].z : code_bits;
  const uint32_t base = A & ~31u;
  const int nw = (int)((B - base + 31) >> 5);
  for (int c = warp; c < kChan; c += kWarps)
    for (int w = lane; w <= nw; w += 32) sbuf[c * kWords + w] = 0u;
  __syncthreads();

  // The records are grouped by bit width (each carries its own stream position, so their order
  // does not matter), and every block of PB records then has a single width.
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t rank[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const uint32_t b = mine[q].y;
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    rank[q] = s_cnt[b][warp] + __popc(peers & lt);
    __syncwarp();
    if ((peers & lt) == 0u) s_cnt[b][warp] += __popc(peers);   // the lowest lane of each width
    __syncwarp();
  }
  __syncthreads();
  if (warp == 0) {   // lane b - 1: width b's first slot (groups padded to whole blocks), its warps' slots
    const int b = lane + 1;
    uint32_t tot = 0;
    if (lane < 8)
      for (int w = 0; w < kWarps; ++w) tot += s_cnt[b][w];
    const uint32_t padded = (tot + PB - 1) / PB * PB;
    uint32_t incl = padded;
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane < 8) {
      uint32_t run = incl - padded;
      s_grp[b] = run;
      for (int w = 0; w < kWarps; ++w) {
        const uint32_t c = s_cnt[b][w];
        s_cnt[b][w] = run;
        run += c;
      }
      s_fill[b] = run;
    }
    if (lane == 7) s_grp[9] = incl;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < kPer; ++q)
    if (mine[q].y) rs[s_cnt[mine[q].y][warp] + rank[q]] = mine[q];
  // padding records fill each group to whole blocks: width b, coefficient row 0, gain 0, code bits
  // into a word of the rows past every range's span, which is never stored
  if (threadIdx.x < 8 * PB) {
    const int b = 1 + (int)threadIdx.x / PB;
    const uint32_t e = s_fill[b] + threadIdx.x % PB;
    if (e < s_grp[b + 1]) rs[e] = make_uint4(0u, (uint32_t)b, base + 32u * pack_pad_word<CPL>(), 0u);
  }
  __syncthreads();

  uint32_t* row = sbuf + lane * kWords;
  const bool rotate = VAR && (g.flags & TACTKV_ROTATE);
  const float rot_in = rotate ? rotation_sign((unsigned long long)(chunk0 * kChunk + lane)) : 1.f;
  // blocks of PB records per warp; the next block's coefficients are loaded while this one is
  // quantized
  const int m_pad = (int)s_grp[9];
  constexpr int stride = kWarps * PB;
  int e0 = warp * PB;
  float x[PB][CPL];
  if (e0 < m_pad) {
#pragma unroll
    for (int j = 0; j < PB; ++j) {
      const float* xr = xu + (size_t)rs[e0 + j].x * g.n;
#pragma unroll
      for (int k = 0; k < CPL; ++k) x[j][k] = __ldcs(xr + k * kChunk);
    }
  }
  for (; e0 < m_pad; e0 += stride) {
    float xn[PB][CPL];
    const int e1 = e0 + stride;
    if (e1 < m_pad) {
#pragma unroll
      for (int j = 0; j < PB; ++j) {
        const float* xr = xu + (size_t)rs[e1 + j].x * g.n;
#pragma unroll
        for (int k = 0; k < CPL; ++k) xn[j][k] = __ldcs(xr + k * kChunk);
      }
    }
    if (rotate) {
#pragma unroll
      for (int j = 0; j < PB; ++j) x[j][0] = warp_wht(x[j][0] * rot_in, lane) * 0.17677669529663687f;
    }
    const uint4* blk = rs + e0;
    const int b = (int)blk[0].y;
    if (b == 1) pack_block<1, CPL, PB>(blk, x, row, base, 1, thr2, qcell);
    else if (b == 2) pack_block<2, CPL, PB>(blk, x, row, base, 2, thr2, qcell);
    else pack_block<0, CPL, PB>(blk, x, row, base, b, thr2, qcell);
#pragma unroll
    for (int j = 0; j < PB; ++j)
#pragma unroll
      for (int k = 0; k < CPL; ++k) x[j][k] = xn[j][k];
  }
  __syncthreads();
  // The span's words.  Its first word may also hold the previous range's last bits, its last word
  // the next range's first bits: in such a word this range owns bits [lo, hi) (the last range
  // also the zero padding after the last code bit), clears them and ORs its codes in.  The two
  // ranges' fields are disjoint, so their AND and OR reductions leave the word right in any order,
  // whatever it held before.
  const uint32_t wbase = base >> 5, wlast = (B - 1) >> 5;
  const bool first_shared = (A & 31u) != 0, last_shared = (B & 31u) != 0 && r1 < nrec;
  for (int c = warp; c < kChan; c += kWarps) {
    uint32_t* out = words_out + (size_t)c * sw;
    for (int w = lane; w < nw; w += 32) {
      const uint32_t gw = wbase + w, v = sbuf[c * kWords + w];
      const bool first = gw == wbase && first_shared, last = gw == wlast && last_shared;
      if (first || last) {
        const uint32_t below_lo = first ? (1u << (A & 31u)) - 1u : 0u;
        const uint32_t below_hi = last ? (1u << (B & 31u)) - 1u : ~0u;
        atomicAnd(out + gw, ~(below_hi & ~below_lo));
        atomicOr(out + gw, v);
      } else {
        out[gw] = v;
      }
    }
  }
  if (r1 == nrec) {   // zero padding of the streams after the last code bit
    const uint32_t first = (code_bits + 31) >> 5;
    for (int c = warp; c < kChan; c += kWarps)
      for (uint32_t w = first + lane; w < sw; w += 32) words_out[(size_t)c * sw + w] = 0u;
  }
}

// NO_QUANT: the float32 coefficients of every bin into the channel streams (stream c holds X[i, c]
// at byte 4i), then the zero padding up to the channel stride.
__global__ void __launch_bounds__(kPackThreads) pack_raw_kernel(const __grid_constant__ Geom g,
                                                                const __grid_constant__ UnitList ul,
                                                                const float* __restrict__ X, int spc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int chunk = blockIdx.x, u = blockIdx.z;
  const int ks0 = blockIdx.y * spc, ks1 = min(g.S, ks0 + spc);
  unsigned char* pay = ul.u[u].payload;
  const uint32_t cstride = reinterpret_cast<const uint32_t*>(pay)[11];
  float* stream = reinterpret_cast<float*>(pay + g.off_codes + (size_t)(chunk * kChunk + lane) * cstride);
  const float* xu = X + (size_t)u * g.N * g.n + chunk * kChunk + lane;
  for (int i = ks0 * g.HW + warp; i < ks1 * g.HW; i += nwarps) stream[i] = xu[(size_t)i * g.n];
  if (ks1 == g.S) {
    const int pad = (int)cstride - 4 * g.N;
    for (int i = threadIdx.x; i < kChunk * pad; i += blockDim.x) {
      const int c = i / pad, b = i - c * pad;
      pay[g.off_codes + (size_t)(chunk * kChunk + c) * cstride + 4 * g.N + b] = 0;
    }
  }
}

}  // namespace

cudaError_t launch_pack(const Geom& g, const UnitList& ul, int nu, const float* X, const uint4* recs,
                        const uint32_t* index, cudaStream_t st) {
  if (g.flags & TACTKV_NO_QUANT) {
    const int spc = 1;
    pack_raw_kernel<<<dim3(g.nch, g.S, nu), kPackThreads, 0, st>>>(g, ul, X, spc);
  } else {
    // four channels per lane where the chunks come in fours, else one; a unit has at most N
    // records, CTAs past its last record exit (measured: a CTA looping over two ranges, to launch
    // fewer CTAs without work, was slower; so were eight channels per lane, ranges of 128 records)
    auto go = [&](auto kernel, int cpl, size_t smem, int recs_per_cta) {
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      const dim3 grid(g.nch / cpl, (g.N + recs_per_cta - 1) / recs_per_cta, nu);
      kernel<<<grid, kPackThreads, smem, st>>>(g, ul, X, recs, index);
    };
    if (has_variant(g.flags)) go(pack_kernel<true, 1>, 1, pack_layout<1>().total, pack_recs<1>());
    else if (g.nch % 4 == 0) go(pack_kernel<false, 4>, 4, pack_layout<4>().total, pack_recs<4>());
    else go(pack_kernel<false, 1>, 1, pack_layout<1>().total, pack_recs<1>());
  }
  return cudaGetLastError();
}

}  // namespace tactkv
