// Quantization and bit packing (TACT-KV stage 4: gain-shape scalar quantization with the fixed
// Lloyd-Max codebook at each bin's bit width), on the finished 3D-DCT coefficients X.
//
// The allocation kernel lists, once per unit, every bin that received bits, in bin order, as a
// 16-byte record {bin, bits, first stream bit P_i, 1/sigma_i}; P_i = sum of the bits of every
// earlier bin, the same in every channel's stream.  A CTA owns one (unit, 32-channel chunk, range
// of kPackRecs records); lane l of a warp is channel l, so every decision about a record is
// uniform across the warp and only the 32 coefficient values differ.  Bins without bits are never
// read.
//
// The CTA clears the word rows of its bit span in shared memory and puts its records there grouped
// by bit width (records are independent of each other: each carries its stream position), each
// group padded to whole blocks of 16.  Each warp takes blocks of 16 records of one width (quantized
// by code specialised for 1 bit, 2 bits, or 3 and more bits by table); while it quantizes one
// block, the 16 coefficient rows (128 bytes each) of its next block are in flight.  For a record
// it computes u = X * (1/sigma) and the code, and ORs the code into the channel's word row at its
// stream position (a shared-memory reduction).  The span's words are then stored once; its first and
// last words may hold bits of the neighbouring ranges and are ORed into the payload atomically (the allocation zeroes those
// words first).  The CTA with the last record also writes the zero padding of the channel streams.
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
constexpr int kPackBlock = 16;  // records per warp step

// Thresholds of width b padded with two +inf, stored for b = 1, 2, ... in turn.
__device__ __forceinline__ int thr_pad_offset(int b) { return (1 << b) + b - 3; }

struct PackLayout {
  size_t rec, sbuf, thr, qcell, total;
  int words;
};
// A range's records grouped by bit width, each group padded to whole blocks of kPackBlock.
constexpr int kPackRecSlots = kPackRecs + 8 * kPackBlock;
__host__ __device__ inline PackLayout pack_layout() {
  PackLayout L;
  auto p16 = [](size_t x) { return (x + 15) / 16 * 16; };
  L.words = ((8 * kPackRecs + 31) / 32 + 3) | 1;   // odd: 32 channels' rows in 32 different banks
  size_t o = 0;
  L.rec = o; o += p16((size_t)kPackRecSlots * 16);
  L.sbuf = o; o += p16((size_t)kChunk * L.words * 4);
  L.thr = o; o += (size_t)TACTKV_THR_VEC * 16;
  L.qcell = o; o += (size_t)TACTKV_QCELL_VEC * 16;
  L.total = o;
  return L;
}

// Code of u at b bits: the number of thresholds t_j <= u (float32 compares, ties go up).  B is
// the width when fixed at compile time (1 or 2), 0 for a width b >= 3 known at run time.  b = 1:
// the sign test, which needs no gain (1/sigma is positive and finite, so u >= 0 exactly when
// x >= 0); b = 2: three compares against {-t, 0, t}; b >= 3: the cell of u in a uniform grid gives
// the count c of thresholds below the cell, and two compares finish it (a cell holds at most two
// thresholds; the thresholds are padded with +inf).
template <int B>
__device__ __forceinline__ uint32_t quant_code_b(float x, float inv_sigma, int b, const float* __restrict__ thr,
                                                 const unsigned char* __restrict__ qcell) {
  if constexpr (B == 1) {
    return x >= 0.f;
  } else {
    const float u = x * inv_sigma;
    if constexpr (B == 2) {
      return (uint32_t)(u >= -TACTKV_LM_T2) + (uint32_t)(u >= 0.f) + (uint32_t)(u >= TACTKV_LM_T2);
    } else {
      int j = __float2int_rd(fmaf(u, TACTKV_Q_SCALE, TACTKV_Q_OFFSET));
      j = min(max(j, 0), TACTKV_Q_CELLS - 1);
      const uint32_t c = qcell[(b - 3) * TACTKV_Q_CELLS + j];
      const float* t = thr + thr_pad_offset(b) + c;
      return c + (uint32_t)(u >= t[0]) + (uint32_t)(u >= t[1]);
    }
  }
}

// OR into a shared-memory word without reading the old value back (a reduction, not an atomic
// with a result): nothing waits for it, so consecutive codes of a warp do not stall on each other.
__device__ __forceinline__ void red_or_shared(uint32_t* p, uint32_t v) {
  asm volatile("red.shared.or.b32 [%0], %1;\n" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(v)
               : "memory");
}

// One block of kPackBlock records, all of width b (= B when B > 0): quantize x[] and OR the codes
// into the row (a code of more than one bit may straddle into the next word).  In three phases --
// the block's records, then its codes, then the ORs -- so that the loads of one phase are all in
// flight together instead of each waiting behind the previous record's OR.
template <int B>
__device__ __forceinline__ void pack_block(const uint4* __restrict__ rs, const float (&x)[kPackBlock],
                                           uint32_t* __restrict__ row, uint32_t base, int b,
                                           const float* __restrict__ thr, const unsigned char* __restrict__ qcell) {
  uint2 r[kPackBlock];
#pragma unroll
  for (int j = 0; j < kPackBlock; ++j) r[j] = reinterpret_cast<const uint2*>(rs + j)[1];   // {position, 1/sigma}
  uint32_t code[kPackBlock];
#pragma unroll
  for (int j = 0; j < kPackBlock; ++j) code[j] = quant_code_b<B>(x[j], __uint_as_float(r[j].y), b, thr, qcell);
#pragma unroll
  for (int j = 0; j < kPackBlock; ++j) {
    const uint32_t off = r[j].x - base, w = off >> 5, sh = off & 31u;
    red_or_shared(row + w, code[j] << sh);
    if constexpr (B != 1) {
      if (sh + (uint32_t)b > 32u) red_or_shared(row + w + 1, code[j] >> (32u - sh));
    }
  }
}

// VAR: the payload has variant flags (the shared rotation), a compile-time switch so that the
// default kernel keeps its register budget.
template <bool VAR>
__global__ void __launch_bounds__(kPackThreads, 4) pack_kernel(const __grid_constant__ Geom g,
                                                            const __grid_constant__ UnitList ul,
                                                            const float* __restrict__ X, const uint4* __restrict__ recs,
                                                            const uint32_t* __restrict__ index) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int kWarps = kPackThreads / 32;
  __shared__ uint32_t s_cnt[9][kWarps];   // per bit width and warp: record counts, then first slots
  __shared__ uint32_t s_fill[9];          // end of each width's records
  __shared__ uint32_t s_grp[10];          // first slot of each width's group; s_grp[9]: all slots
  const PackLayout L = pack_layout();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = blockIdx.x, u = blockIdx.z;
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const uint32_t nrec = P[2 * g.S + 2], code_bits = P[g.S];      // NZ(S) and P(S)
  const uint32_t r0 = blockIdx.y * kPackRecs;
  if (r0 >= nrec && !(r0 == 0 && nrec == 0)) return;             // (range 0 also pads an empty unit)
  const uint32_t r1 = min(nrec, r0 + kPackRecs);
  const int m = (int)(r1 - r0);
  unsigned char* pay = ul.u[u].payload;
  const uint4* urecs = recs + (size_t)u * g.N;
  const float* xu = X + (size_t)u * g.N * g.n + chunk * kChunk + lane;
  uint4* rs = reinterpret_cast<uint4*>(smem + L.rec);
  uint32_t* sbuf = reinterpret_cast<uint32_t*>(smem + L.sbuf);
  float* thr = reinterpret_cast<float*>(smem + L.thr);
  unsigned char* qcell = smem + L.qcell;
  const uint32_t cstride = reinterpret_cast<const uint32_t*>(pay)[11], sw = cstride / 4;
  uint32_t* words_out = reinterpret_cast<uint32_t*>(pay + g.off_codes) + (size_t)chunk * kChunk * sw;

  // Thread t holds records t, t + 256, ... of the range (empty slots past m have width 0).
  constexpr int kPer = kPackRecs / kPackThreads;
  uint4 mine[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int e = q * kPackThreads + (int)threadIdx.x;
    mine[q] = e < m ? urecs[r0 + e] : make_uint4(0u, 0u, 0u, 0u);
  }
  if (VAR && head_gains_on(g.flags)) {   // 1/gain of the CTA's head (0 for a zero gain: u = 0)
    const float* hg = reinterpret_cast<const float*>(pay + g.off_sigma) + (size_t)(chunk * kChunk / g.head_dim) * g.N;
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (mine[q].y) {
        const float gh = hg[mine[q].x];
        mine[q].w = gh > 0.f ? __float_as_uint(__frcp_rn(gh)) : 0u;
      }
  }
  if (threadIdx.x < 9 * kWarps) (&s_cnt[0][0])[threadIdx.x] = 0u;
  copy_vec16(thr, g_thr_pad, TACTKV_THR_VEC);
  copy_vec16(qcell, g_qcell, TACTKV_QCELL_VEC);
  // bit span [A, B) of the range; its words from word A >> 5 on are assembled in shared memory
  const uint32_t A = m > 0 ? urecs[r0].z : code_bits;
  const uint32_t B = r1 < nrec ? urecs[r1].z : code_bits;
  const uint32_t base = A & ~31u;
  const int nw = (int)((B - base + 31) >> 5);
  for (int c = warp; c < kChunk; c += kWarps)
    for (int w = lane; w <= nw; w += 32) sbuf[c * L.words + w] = 0u;
  __syncthreads();

  // The records are grouped by bit width (each carries its own stream position, so their order
  // does not matter), and every block of kPackBlock records then has a single width.
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
  if (threadIdx.x == 0) {
    uint32_t run = 0;
    for (int b = 1; b <= 8; ++b) {
      s_grp[b] = run;
      for (int w = 0; w < kWarps; ++w) {
        const uint32_t c = s_cnt[b][w];
        s_cnt[b][w] = run;
        run += c;
      }
      s_fill[b] = run;
      run = (run + kPackBlock - 1) / kPackBlock * kPackBlock;
    }
    s_grp[9] = run;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < kPer; ++q)
    if (mine[q].y) rs[s_cnt[mine[q].y][warp] + rank[q]] = mine[q];
  // padding records fill each group to whole blocks: width b, coefficient row 0, gain 0, code bits
  // into word 257 of the row, which is past every range's span (at most 8 * kPackRecs + 31 bits =
  // 257 words) and never stored
  if (threadIdx.x < 8 * kPackBlock) {
    const int b = 1 + (int)threadIdx.x / kPackBlock;
    const uint32_t e = s_fill[b] + threadIdx.x % kPackBlock;
    if (e < s_grp[b + 1]) rs[e] = make_uint4(0u, (uint32_t)b, base + 32u * 257u, 0u);
  }
  __syncthreads();

  uint32_t* row = sbuf + lane * L.words;
  const bool rotate = VAR && (g.flags & TACTKV_ROTATE);
  const float rot_in = rotate ? rotation_sign((unsigned long long)(chunk * kChunk + lane)) : 1.f;
  // blocks of kPackBlock records per warp; the next block's coefficients are loaded while this
  // one is quantized
  const int m_pad = (int)s_grp[9];
  constexpr int stride = kWarps * kPackBlock;
  int e0 = warp * kPackBlock;
  float x[kPackBlock];
  if (e0 < m_pad) {
#pragma unroll
    for (int j = 0; j < kPackBlock; ++j) x[j] = __ldcs(xu + (size_t)rs[e0 + j].x * g.n);
  }
  for (; e0 < m_pad; e0 += stride) {
    float xn[kPackBlock];
    const int e1 = e0 + stride;
    if (e1 < m_pad) {
#pragma unroll
      for (int j = 0; j < kPackBlock; ++j) xn[j] = __ldcs(xu + (size_t)rs[e1 + j].x * g.n);
    }
    if (rotate) {
#pragma unroll
      for (int j = 0; j < kPackBlock; ++j) x[j] = warp_wht(x[j] * rot_in, lane) * 0.17677669529663687f;
    }
    const uint4* blk = rs + e0;
    const int b = (int)blk[0].y;
    if (b == 1) pack_block<1>(blk, x, row, base, 1, thr, qcell);
    else if (b == 2) pack_block<2>(blk, x, row, base, 2, thr, qcell);
    else pack_block<0>(blk, x, row, base, b, thr, qcell);
#pragma unroll
    for (int j = 0; j < kPackBlock; ++j) x[j] = xn[j];
  }
  __syncthreads();
  // the span's words; the first and the last may be shared with the neighbouring ranges
  const uint32_t wbase = base >> 5, wlast = (B - 1) >> 5;
  const bool first_shared = (A & 31u) != 0, last_shared = (B & 31u) != 0;
  for (int c = warp; c < kChunk; c += kWarps) {
    uint32_t* out = words_out + (size_t)c * sw;
    for (int w = lane; w < nw; w += 32) {
      const uint32_t gw = wbase + w, v = sbuf[c * L.words + w];
      if ((gw == wbase && first_shared) || (gw == wlast && last_shared)) atomicOr(out + gw, v);
      else out[gw] = v;
    }
  }
  if (r1 == nrec) {   // zero padding of the streams after the last code bit
    const uint32_t first = (code_bits + 31) >> 5;
    for (int c = warp; c < kChunk; c += kWarps)
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
    const PackLayout L = pack_layout();
    auto kernel = has_variant(g.flags) ? pack_kernel<true> : pack_kernel<false>;
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    // ranges of kPackRecs records; a unit has at most N records, CTAs past its last record exit
    const dim3 grid(g.nch, (g.N + kPackRecs - 1) / kPackRecs, nu);
    kernel<<<grid, kPackThreads, L.total, st>>>(g, ul, X, recs, index);
  }
  return cudaGetLastError();
}

}  // namespace tactkv
