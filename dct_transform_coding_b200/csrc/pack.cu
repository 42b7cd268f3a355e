// Quantization and bit packing (TACT-KV stage 4: gain-shape scalar quantization with the fixed
// Lloyd-Max codebook at each bin's bit width), on the finished 3D-DCT coefficients X.
//
// The allocation kernel lists, once per unit, every bin that received bits, in bin order, as a
// 16-byte record {bin, bits, first stream bit P_i, 1/sigma_i}; P_i = sum of the bits of every
// earlier bin, the same in every channel's stream.  A warp owns kRange consecutive records of one
// (unit, 32-channel chunk); lane l is channel l, so every decision about a record is uniform across
// the warp and only the 32 coefficient values differ.  Bins without bits are never read.
//
// The codes of consecutive records are consecutive bits of every channel stream, so each lane
// appends its channel's codes to a 64-bit register and emits a 32-bit word whenever one is full.
// A warp owns exactly the stream words whose first bit lies in its range [P_first, P_end): it drops
// the bits in front of its first owned word (the previous warp writes that word) and, to finish its
// last word, goes on into the next range's first records (fewer than 32 bits of them).  Every word
// is therefore written once by a plain store: no atomics and nothing to clear beforehand.  The warp
// that holds the end of the streams also writes their zero padding.
//
// NO_QUANT (raw) copies X into the channel streams as float32.
#include "common.cuh"
#include "lloyd_max_tables.inc"

namespace tactkv {
namespace {

constexpr int kPackThreads = 256;
constexpr int kPackWarps = kPackThreads / 32;
constexpr int kRange = 128;               // records per warp
constexpr int kExtra = 32;                // records staged past the range (a word is < 32 records)
constexpr int kBlock = 16;                // coefficient loads in flight per lane

// Thresholds of width b padded with two +inf, stored for b = 1, 2, ... in turn.
__device__ __forceinline__ int thr_pad_offset(int b) { return (1 << b) + b - 3; }

struct PackLayout {
  size_t rec, thr, qcell, total;
};
__host__ __device__ inline PackLayout pack_layout() {
  PackLayout L;
  auto p16 = [](size_t x) { return (x + 15) / 16 * 16; };
  size_t o = 0;
  L.rec = o; o += p16((size_t)kPackWarps * (kRange + kExtra) * 16);
  L.thr = o; o += p16((size_t)TACTKV_THR_PAD_TOTAL * 4);
  L.qcell = o; o += p16((size_t)6 * TACTKV_Q_CELLS);
  L.total = o;
  return L;
}

// Code of x at b bits (1..8): the number of thresholds t_j <= u = x * (1/sigma) (float32 compares,
// ties go up).  b = 1: the sign test, which needs no gain (1/sigma is positive and finite, so
// u >= 0 exactly when x >= 0); b = 2: three compares against {-t, 0, t}; b >= 3: the cell of u in a
// uniform grid gives the count c of thresholds below the cell, and two compares finish it (a cell
// holds at most two thresholds; the thresholds are padded with +inf).  b is warp-uniform.
__device__ __forceinline__ uint32_t quant_code(float x, float inv_sigma, int b, const float* __restrict__ thr,
                                               const unsigned char* __restrict__ qcell) {
  if (b == 1) return x >= 0.f;
  const float u = x * inv_sigma;
  if (b == 2) return (uint32_t)(u >= -TACTKV_LM_T2) + (uint32_t)(u >= 0.f) + (uint32_t)(u >= TACTKV_LM_T2);
  int j = __float2int_rd(fmaf(u, TACTKV_Q_SCALE, TACTKV_Q_OFFSET));
  j = min(max(j, 0), TACTKV_Q_CELLS - 1);
  const uint32_t c = qcell[(b - 3) * TACTKV_Q_CELLS + j];
  const float* t = thr + thr_pad_offset(b) + c;
  return c + (uint32_t)(u >= t[0]) + (uint32_t)(u >= t[1]);
}

__global__ void __launch_bounds__(kPackThreads) pack_kernel(const __grid_constant__ Geom g,
                                                            const __grid_constant__ UnitList ul,
                                                            const float* __restrict__ X, const uint4* __restrict__ recs,
                                                            const uint32_t* __restrict__ index) {
  extern __shared__ __align__(16) unsigned char smem[];
  const PackLayout L = pack_layout();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = blockIdx.x, u = blockIdx.z;
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const uint32_t nrec = P[2 * g.S + 2], code_bits = P[g.S];      // NZ(S) and P(S)
  const uint4* urecs = recs + (size_t)u * g.N;
  float* thr = reinterpret_cast<float*>(smem + L.thr);
  unsigned char* qcell = smem + L.qcell;
  uint4* rs = reinterpret_cast<uint4*>(smem + L.rec) + warp * (kRange + kExtra);
  for (int i = threadIdx.x; i < TACTKV_THR_PAD_TOTAL; i += kPackThreads) thr[i] = c_thr_pad[i];
  for (int i = threadIdx.x; i < 6 * TACTKV_Q_CELLS; i += kPackThreads) qcell[i] = c_qcell[i];
  const uint32_t r0 = (blockIdx.y * kPackWarps + warp) * kRange;
  const uint32_t r1 = min(nrec, r0 + kRange);
  const int staged = r0 < nrec ? (int)min((uint32_t)(kRange + kExtra), nrec - r0) : 0;
  for (int e = lane; e < staged; e += 32) rs[e] = urecs[r0 + e];
  __syncthreads();
  if (r0 >= nrec) return;
  __syncwarp();

  unsigned char* pay = ul.u[u].payload;
  const uint32_t cstride = reinterpret_cast<const uint32_t*>(pay)[11], sw = cstride / 4;
  uint32_t* out = reinterpret_cast<uint32_t*>(pay + g.off_codes) + (size_t)(chunk * kChunk + lane) * sw;
  const float* xu = X + (size_t)u * g.N * g.n + chunk * kChunk + lane;

  // the shared rotation R = H_32 diag(s) / sqrt(32) of each bin's 32 channels of this chunk
  const bool rotate = g.flags & TACTKV_ROTATE;
  const float rot_in = rotate ? rotation_sign((unsigned long long)(chunk * kChunk + lane)) : 1.f;

  const uint32_t A = rs[0].z;                                    // first bit of the range
  const uint32_t end_bit = r1 < nrec ? rs[r1 - r0].z : code_bits;
  const uint32_t first_word = (A + 31) >> 5;                     // words [first_word, stop_word) are ours
  const uint32_t stop_bit = min(code_bits, ((end_bit + 31) >> 5) << 5);
  // records past the range whose first bit is still below stop_bit finish our last word
  int extra = 0;
  if (r1 < nrec) {
    const uint32_t k = r1 - r0 + lane;
    const bool need = (int)k < staged && rs[k].z < stop_bit;
    extra = __popc(__ballot_sync(0xffffffffu, need));
  }
  const int m = (int)(r1 - r0) + extra;

  unsigned long long acc = 0;
  int nacc = (int)(A & 31u);          // bits of the current word below the first record's code
  uint32_t w = A >> 5;
  for (int e0 = 0; e0 < m; e0 += kBlock) {
    float x[kBlock];
#pragma unroll
    for (int j = 0; j < kBlock; ++j)
      if (e0 + j < m) x[j] = __ldcs(xu + (size_t)rs[e0 + j].x * g.n);
    if (rotate) {
#pragma unroll
      for (int j = 0; j < kBlock; ++j)
        if (e0 + j < m) x[j] = warp_wht(x[j] * rot_in, lane) * 0.17677669529663687f;
    }
#pragma unroll
    for (int j = 0; j < kBlock; ++j) {
      if (e0 + j >= m) break;
      const uint4 r = rs[e0 + j];
      const int b = (int)r.y;
      acc |= (unsigned long long)quant_code(x[j], __uint_as_float(r.w), b, thr, qcell) << nacc;
      nacc += b;
      if (nacc >= 32) {
        if (w >= first_word) out[w] = (uint32_t)acc;
        acc >>= 32;
        nacc -= 32;
        ++w;
      }
    }
  }
  if (nacc > 0 && w >= first_word && (w << 5) < stop_bit) out[w] = (uint32_t)acc;   // the streams' last word
  if (r1 == nrec) {   // zero padding of the streams after the last code bit
    for (uint32_t z = (code_bits + 31) >> 5; z < sw; ++z) out[z] = 0u;
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
    cudaFuncSetAttribute(pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    // ranges of kRange records per warp; a unit has at most N records, warps past its last record exit
    const dim3 grid(g.nch, (g.N + kPackWarps * kRange - 1) / (kPackWarps * kRange), nu);
    pack_kernel<<<grid, kPackThreads, L.total, st>>>(g, ul, X, recs, index);
  }
  return cudaGetLastError();
}

}  // namespace tactkv
