// One decode step of attention over compressed visual K/V, without reconstructing the cache (the
// paragraph after stage 4 of "Methodology in Plain English" on the TACT-KV summary page: decoding
// can be fused into the attention kernel).
//
// The 3D DCT is linear and orthonormal per channel, so with X_K, X_V the dequantized coefficients
// (bin i, channel c) and C3 the 3D DCT-II:
//   scores   s_j[t] = q_j . K[t] / sqrt(D) = idct3(z_j)[t],   z_j[i] = sum_d q_j[d] X_K[i, hD + d] / sqrt(D)
//   output   o_j    = sum_t p_j[t] V[t]    = sum_i dct3(p_j)[i] X_V[i, hD + d]
// with p_j[t] = exp(s_j[t] - m_j), m_j = max_t s_j[t], l_j = sum_t p_j[t], and out_j = o_j / l_j
// (query head j uses K/V head h = j / G).  Only bins with bits are decoded, from each slab's words
// of the payloads' channel streams staged in shared memory (read from the payload directly when a
// slab's codes span more than the rows, sized for the call's rate, hold); the volumes of T values
// per query head are transformed in shared memory.  A unit whose K or V payload fails the index
// checks contributes no tokens (out 0, m -inf, l 0).  With the shared rotation R (per 32-channel
// group), X = R^T X' for the coded X': the query is rotated (q . R^T x' = (R q) . x') and the
// output rotated back at the end.
//
// Kernels (one launch each, all units of a call share one shape):
//   decode_index   (allocate.cu) the K and V payloads' checks, slab offsets and dense records;
//   attn_scores    grid (S slabs, K/V heads, units): z for the G query heads of the head;
//   attn_softmax   grid (query heads, units): inverse 3D DCT of z, softmax, forward 3D DCT of p;
//   attn_values    grid (S slabs, K/V heads, units): per-slab sums of dct3(p)[i] X_V[i, :];
//   attn_reduce    grid (query heads, units): sum over slabs in a fixed order, rotation back, / l.
#include "common.cuh"
#include "lloyd_max_tables.inc"

namespace tactkv {
namespace {

constexpr int kAttnThreads = 256;
constexpr int kMaxG = 16;                   // query heads per K/V head
constexpr float kInvSqrt32 = 0.17677669529663687f;
constexpr int kLv0Floats = TACTKV_LV0_VEC * 4;   // the levels behind a zero, in whole 16-byte vectors
static_assert(kLv0Floats >= kLmLvTotal + 1, "level table");

// Words of a channel stream held per slab in shared memory: what a slab spans at 2 * bits + 2 bits
// per bin (at most 8), from any bit of its first word, two zero words for the look-ahead of the
// code reads, and an odd count, so that 32 lanes reading 32 channels' rows at one offset hit 32
// banks.  A slab whose codes span more (its bins hold far more than the average bits) is decoded
// from the payload in global memory instead.  Sizing the rows for the call's rate rather than for
// 8 bits per bin leaves room for more CTAs per SM.
__host__ __device__ inline int attn_cap_bits(int bits) { return 2 * bits + 2 < 8 ? 2 * bits + 2 : 8; }
__host__ __device__ inline int attn_word_stride(int HW, int bits) {
  return ((attn_cap_bits(bits) * HW + 31) / 32 + 3) | 1;
}
__host__ __device__ inline int pad32(int x) { return (x + 31) / 32 * 32; }

// Copy the words of slab ks of the D channel streams from `row0` (channel 0's stream, word P(ks)
// >> 5) into words[c][stride], asynchronously, with the two look-ahead words zeroed.  Every thread.
__device__ __forceinline__ void stage_words(const uint32_t* __restrict__ row0, uint32_t sw, int D, int nw, int stride,
                                            uint32_t* __restrict__ words) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int c = warp; c < D; c += nwarps)
    for (int w = lane; w < nw + 2; w += 32) {
      if (w < nw) cp_async4(words + c * stride + w, row0 + (size_t)c * sw + w);
      else words[c * stride + w] = 0u;
    }
  cp_async_commit();
}

// Stage the slab's dense decoding records and list the slab's bins that have bits (in bin order):
// act[a] = bin index j, actrec[a] = {sigma, offset << 8 | code mask} of that bin, for a < count;
// actrec is then zero up to the next multiple of 32 (a zero record decodes to 0).  Returns the
// count.  Called by every thread; ends with a barrier.
__device__ int stage_active(const uint4* __restrict__ srec, int HW, int W, uint2* __restrict__ actrec,
                            int* __restrict__ act, int* s_count, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (threadIdx.x == 0) *s_count = 0;
  __syncthreads();
  for (int j0 = 0; j0 < HW; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    uint2 r = make_uint2(0u, 0u);
    if (j < HW) {
      const int kh = j / W, t = j - kh * W;
      const uint4 m = srec[(kh >> 1) * W + t];
      r = (kh & 1) ? make_uint2(m.y, m.w) : make_uint2(m.x, m.z);
      r.y &= 0x03ffffffu;   // offset << 8 | mask (the decoder's window shift dropped)
    }
    const bool has = (r.y & 0xffu) != 0u;
    const unsigned bal = __ballot_sync(0xffffffffu, has);
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    if (threadIdx.x == 0) {   // exclusive prefix over the warps, in warp order (bin order kept)
      int run = *s_count;
      for (int w = 0; w < nw; ++w) {
        const int c = s_warp[w];
        s_warp[w] = run;
        run += c;
      }
      *s_count = run;
    }
    __syncthreads();
    if (has) {
      const int a = s_warp[warp] + __popc(bal & ((1u << lane) - 1u));
      act[a] = j;
      actrec[a] = r;
    }
    __syncthreads();
  }
  const int na = *s_count;
  for (int a = na + (int)threadIdx.x; a < pad32(na); a += blockDim.x) actrec[a] = make_uint2(0u, 0u);
  __syncthreads();
  return na;
}

// Codebook level of a bin's code (record word y = offset << 8 | mask) in a channel's row from the
// slab's first word on: staged in shared memory (GLOBAL false: two zero words after the slab make
// the second word always readable) or the payload's stream itself (GLOBAL true: the second word is
// read only when the code reaches into it, so nothing past the stream is touched).  A bin without
// bits (mask 0) gives the zero in front of the levels.
template <bool GLOBAL>
__device__ __forceinline__ float level_at(const uint32_t* __restrict__ row, uint32_t y, const float* lvs1) {
  const uint32_t k = y & 0xffu, off = y >> 8;
  const uint32_t* w = row + (off >> 5);
  uint32_t lo, hi;
  if constexpr (GLOBAL) {
    lo = __ldg(w);
    hi = (off & 31u) + (uint32_t)__popc(k) > 32u ? __ldg(w + 1) : 0u;   // uniform across the warp
  } else {
    lo = w[0];
    hi = w[1];
  }
  return lvs1[(int)(k + (__funnelshift_r(lo, hi, off) & k)) - 1];
}

// With per-head gains: the staged records of the active bins take head h's gains instead of the
// bins' (sigma[h][bin] in the payload).  Every thread; the caller synchronizes before use.
__device__ __forceinline__ void head_gain_records(const Geom& g, const unsigned char* pay, int h, int ks, int na,
                                                  uint2* actrec, const int* act) {
  const float* hg = reinterpret_cast<const float*>(pay + g.off_sigma) + (size_t)h * g.N + (size_t)ks * g.HW;
  for (int a = threadIdx.x; a < na; a += blockDim.x) actrec[a].x = __float_as_uint(hg[act[a]]);
}

// z_j[i] for the G query heads of K/V head h over the bins of slab ks.  The slab's words of the
// head's D channel streams are staged in shared memory when they fit (else read from the payload).
// The warps work in pairs on batches of 16 active bins (pair p takes batches p, p + 4, ...); warp
// w of the pair takes the channel groups cg = w, w + 2, ... (lane = channel within a group) and,
// for two query heads at a time, accumulates q_j[d] X_K[i, d] over them in registers (32 sums: two
// heads x 16 bins), sums over its 32 lanes (transpose sum: lane l ends with head l >> 4 and active
// bin a0 + (l & 15)), and the second warp's sums are added to the first's through shared memory.
// z of the bins without bits is 0.
constexpr int kScoreThreads = 256;
constexpr int kScorePairs = kScoreThreads / 64;
constexpr int kScoreBatch = 16;
template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

__global__ void __launch_bounds__(kScoreThreads, 4) attn_scores_kernel(const __grid_constant__ Geom g,
                                                                       const __grid_constant__ UnitList ul,
                                                                       const uint32_t* __restrict__ index,
                                                                       const uint4* __restrict__ recs,
                                                                       const float* __restrict__ q, int q_heads,
                                                                       float* __restrict__ z) {
  extern __shared__ __align__(16) float sh[];
  __shared__ int s_count, s_warp[32];
  __shared__ float s_red[kScorePairs][32];
  const int ks = blockIdx.x, h = blockIdx.y, u = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int G = q_heads / g.heads, D = g.head_dim, HW = g.HW, stride = attn_word_stride(HW, g.bits);
  float* lvs1 = sh + 1;                                        // a zero in front of the levels
  float* qs = sh + kLv0Floats;                                 // [G][D], rotated when the payload is
  float* zs = qs + G * D;                                      // [G][HW]
  uint2* actrec = reinterpret_cast<uint2*>(zs + (G * HW + 1) / 2 * 2);   // [pad32(HW)]
  int* act = reinterpret_cast<int*>(actrec + pad32(HW));                 // [HW]
  uint32_t* words = reinterpret_cast<uint32_t*>(act + pad32(HW));        // [D][stride]
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const bool ok = P[g.S + 1] != 0;
  const unsigned char* pay = ul.u[u].payload;
  const uint32_t p0 = ok ? P[ks] : 0u, p1 = ok ? P[ks + 1] : 0u;
  const uint32_t sw = ok ? reinterpret_cast<const uint32_t*>(pay)[11] / 4 : 0u;
  const int nw = (int)(((p0 & 31u) + (p1 - p0) + 31) >> 5);
  const bool staged = nw + 2 <= stride;                        // the same for the whole CTA
  const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes) + (size_t)h * D * sw + (p0 >> 5);
  if (ok && staged) stage_words(streams, sw, D, nw, stride, words);
  copy_vec16(sh, g_lm_levels0, TACTKV_LV0_VEC);
  for (int i = threadIdx.x; i < G * HW; i += blockDim.x) zs[i] = 0.f;
  const float* qu = q + ((size_t)u * q_heads + (size_t)h * G) * D;
  const bool rotate = g.flags & TACTKV_ROTATE;
  for (int gg = warp; gg < G * (D / 32); gg += nwarps) {   // (query head, channel group) per warp
    const int gq = gg / (D / 32), cg = gg - gq * (D / 32), d = cg * 32 + lane;
    float v = qu[(size_t)gq * D + d];
    if (rotate) v = warp_wht(v * rotation_sign((unsigned long long)(h * D + d)), lane) * kInvSqrt32;
    qs[gq * D + d] = v;
  }
  const uint4* srec = recs + (size_t)u * g.N + (size_t)ks * ((g.H + 1) / 2) * g.W;
  const int na = ok ? stage_active(srec, HW, g.W, actrec, act, &s_count, s_warp) : 0;
  if (head_gains_on(g.flags)) head_gain_records(g, pay, h, ks, na, actrec, act);
  cp_async_wait_all();
  __syncthreads();
  const float scale = rsqrtf((float)D);
  const int pair = warp >> 1, half = warp & 1;
  const int rounds = (na + kScorePairs * kScoreBatch - 1) / (kScorePairs * kScoreBatch);   // the same for every warp
  auto batches = [&](auto global) {
    constexpr bool kGlobal = decltype(global)::value;
    for (int it = 0; it < rounds; ++it) {
      const int a0 = (it * kScorePairs + pair) * kScoreBatch;
      for (int gp = 0; gp < G; gp += 2) {
        const bool two = gp + 1 < G;
        float s = 0.f;
        if (a0 < na) {
          float acc[2 * kScoreBatch];   // [head gp, gp + 1][bin a0 ..]
#pragma unroll
          for (int b = 0; b < 2 * kScoreBatch; ++b) acc[b] = 0.f;
          for (int d = half * 32 + lane; d < D; d += 64) {
            const uint32_t* row = kGlobal ? streams + (size_t)d * sw : words + d * stride;
            const float q0 = qs[gp * D + d], q1 = two ? qs[(gp + 1) * D + d] : 0.f;
#pragma unroll
            for (int b = 0; b < kScoreBatch; ++b) {
              const uint2 r = actrec[a0 + b];   // {sigma, offset << 8 | mask}
              const float x = __uint_as_float(r.x) * level_at<kGlobal>(row, r.y, lvs1);
              acc[b] = fmaf(x, q0, acc[b]);
              acc[kScoreBatch + b] = fmaf(x, q1, acc[kScoreBatch + b]);
            }
          }
          s = warp_transpose_sum(acc, lane);
          if (half) s_red[pair][lane] = s;
        }
        __syncthreads();
        const int a = a0 + (lane & (kScoreBatch - 1)), gq = gp + (lane >> 4);
        if (!half && a0 < na && a < na && (gq == gp || two)) zs[gq * HW + act[a]] = (s + s_red[pair][lane]) * scale;
        __syncthreads();
      }
    }
  };
  if (staged) batches(BoolTag<false>{});
  else batches(BoolTag<true>{});
  float* zu = z + ((size_t)u * q_heads + (size_t)h * G) * g.N + (size_t)ks * HW;
  for (int i = threadIdx.x; i < G * HW; i += blockDim.x) {
    const int gq = i / HW, j = i - gq * HW;
    zu[(size_t)gq * g.N + j] = zs[i];
  }
}

// In-place separable DCT-II (INV = false) or DCT-III (INV = true) of a single-channel volume
// vol[S][H][W] in shared memory, skipping the axes the payload left untransformed.  LX > 0 is the
// pencil length fixed at compile time (straight-line code), 0 dispatches on the run-time length.
template <int LX, int CLASS, bool INV>
__device__ __forceinline__ void pencils(float* vol, int L, int count, int stride, int step_outer, int inner) {
  constexpr int R = LX > 0 ? LX : CLASS;
  for (int p = threadIdx.x; p < count; p += blockDim.x) {
    const int o = p / inner, i = p - o * inner;
    float* base = vol + (size_t)o * step_outer + i;
    float x[R];
#pragma unroll
    for (int k = 0; k < R; ++k)
      if (LX > 0 || k < L) x[k] = base[(size_t)k * stride];
    if constexpr (LX > 0) dct_exact<LX, INV>(x);
    else dct_pencil<CLASS, INV>(x, L);
#pragma unroll
    for (int k = 0; k < R; ++k)
      if (LX > 0 || k < L) base[(size_t)k * stride] = x[k];
  }
}
template <int LX, bool INV>
__device__ void pencils_any(float* vol, int L, int count, int stride, int step_outer, int inner) {
  if constexpr (LX > 0) {
    pencils<LX, LX, INV>(vol, L, count, stride, step_outer, inner);
  } else {
    const int c = length_class_dev(L);
    if (c == 16) pencils<0, 16, INV>(vol, L, count, stride, step_outer, inner);
    else if (c == 32) pencils<0, 32, INV>(vol, L, count, stride, step_outer, inner);
    else pencils<0, 64, INV>(vol, L, count, stride, step_outer, inner);
  }
}
// Row length of the score volume in shared memory: W rounded up to an odd count, so that the 32
// lanes of a warp, each on its own row of the pass along W, hit 32 different banks.
__host__ __device__ inline int vol_row(int W) { return W | 1; }
__host__ __device__ inline size_t softmax_smem(const Geom& g) { return (size_t)g.S * g.H * vol_row(g.W) * 4; }

// vol[s][h][w] at (s*H + h)*Wr + w, Wr = vol_row(W).
template <bool INV, int SX, int HX, int WX>
__device__ void dct3_volume(float* vol, const Geom& g) {
  const int S = g.S, H = g.H, W = g.W, Wr = vol_row(W);
  // along W: pencils (s, h), contiguous; along H: (s, w), stride Wr; along S: (h, w), stride H*Wr
  if (!(g.flags & TACTKV_SKIP_W)) pencils_any<WX, INV>(vol, W, S * H, 1, Wr, 1);
  __syncthreads();
  if (!(g.flags & TACTKV_SKIP_H)) pencils_any<HX, INV>(vol, H, S * W, Wr, H * Wr, W);
  __syncthreads();
  if (!(g.flags & TACTKV_SKIP_S)) pencils_any<SX, INV>(vol, S, H * W, H * Wr, Wr, W);
  __syncthreads();
}

__device__ float block_reduce(float v, float* red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float p = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, p) : v + p;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < nw; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// Per query head: scores = idct3(z), p = exp(scores - max), l = sum p, then dct3(p) over z's place.
// SX, HX, WX > 0: the grid's lengths fixed at compile time (the benchmark grids), 0: any grid.
constexpr int kSoftmaxThreads = 256;
// A unit whose K or V payload failed the index checks contributes no tokens: p = 0, m = -inf, l = 0.
template <int SX, int HX, int WX>
__global__ void __launch_bounds__(kSoftmaxThreads, 2) attn_softmax_kernel(const __grid_constant__ Geom g,
                                                                    const uint32_t* __restrict__ kidx,
                                                                    const uint32_t* __restrict__ vidx,
                                                                    float* __restrict__ zp, float* __restrict__ m_out,
                                                                    float* __restrict__ l_out, int q_heads) {
  extern __shared__ __align__(16) float vol[];
  __shared__ float red[32];
  const int j = blockIdx.x, u = blockIdx.y;
  float* zg = zp + ((size_t)u * q_heads + j) * g.N;
  const size_t iw = (size_t)unit_index_words(g.S);
  if (kidx[u * iw + g.S + 1] == 0u || vidx[u * iw + g.S + 1] == 0u) {   // the same for the whole CTA
    for (int i = threadIdx.x; i < g.N; i += blockDim.x) zg[i] = 0.f;
    if (threadIdx.x == 0) {
      m_out[(size_t)u * q_heads + j] = -INFINITY;
      l_out[(size_t)u * q_heads + j] = 0.f;
    }
    return;
  }
  const int W = WX ? WX : g.W, Wr = vol_row(W);   // (a division by a constant on the exact grids)
  auto at = [&](int i) { return (i / W) * Wr + (i - (i / W) * W); };   // bin i -> its padded place
  constexpr int kBatch = 8;   // loads of z in flight per thread before their stores
  for (int i0 = threadIdx.x; i0 < g.N; i0 += kBatch * blockDim.x) {
    float t[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int i = i0 + r * (int)blockDim.x;
      t[r] = i < g.N ? zg[i] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int i = i0 + r * (int)blockDim.x;
      if (i < g.N) vol[at(i)] = t[r];
    }
  }
  __syncthreads();
  dct3_volume<true, SX, HX, WX>(vol, g);
  float mx = -INFINITY;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) mx = fmaxf(mx, vol[at(i)]);
  mx = block_reduce(mx, red, true);
  float sum = 0.f;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
    const float e = __expf(vol[at(i)] - mx);
    vol[at(i)] = e;
    sum += e;
  }
  sum = block_reduce(sum, red, false);
  __syncthreads();
  dct3_volume<false, SX, HX, WX>(vol, g);
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) zg[i] = vol[at(i)];
  if (threadIdx.x == 0) {
    m_out[(size_t)u * q_heads + j] = mx;
    l_out[(size_t)u * q_heads + j] = sum;
  }
}

// part[u][ks][j][d] = sum over the bins i of slab ks of dct3(p_j)[i] * X_V[i, hD + d] (rotated
// domain when the payload is); thread = channel, G accumulators each, no reduction across threads.
// The slab's words of the head's channel streams are staged in shared memory, and only bins with
// bits are visited; their weights dct3(p_j)[i] * sigma_i are formed once per CTA.  GM: the most
// query heads per K/V head the instance handles (4 keeps the accumulators few).
template <int GM>
__global__ void __launch_bounds__(kAttnThreads) attn_values_kernel(const __grid_constant__ Geom g,
                                                                   const __grid_constant__ UnitList ul,
                                                                   const uint32_t* __restrict__ index,
                                                                   const uint4* __restrict__ recs,
                                                                   const float* __restrict__ ptil, int q_heads,
                                                                   float* __restrict__ part) {
  extern __shared__ __align__(16) float sh[];
  __shared__ int s_count, s_warp[32];
  const int ks = blockIdx.x, h = blockIdx.y, u = blockIdx.z;
  const int G = q_heads / g.heads, D = g.head_dim, HW = g.HW, stride = attn_word_stride(HW, g.bits);
  float* lvs1 = sh + 1;
  float* wt = sh + kLv0Floats;        // [HW][G]: weight of active bin a for head g
  uint2* actrec = reinterpret_cast<uint2*>(wt + ((size_t)G * HW + 1) / 2 * 2);   // [pad32(HW)], 8-byte aligned
  int* act = reinterpret_cast<int*>(actrec + pad32(HW));                         // [HW]
  uint32_t* words = reinterpret_cast<uint32_t*>(act + pad32(HW));                // [D][stride]
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const bool ok = P[g.S + 1] != 0;
  const unsigned char* pay = ul.u[u].payload;
  const uint32_t p0 = ok ? P[ks] : 0u, p1 = ok ? P[ks + 1] : 0u;
  const uint32_t sw = ok ? reinterpret_cast<const uint32_t*>(pay)[11] / 4 : 0u;
  const int nw = (int)(((p0 & 31u) + (p1 - p0) + 31) >> 5);
  const bool staged = nw + 2 <= stride;                        // the same for the whole CTA
  const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes) + (size_t)h * D * sw + (p0 >> 5);
  if (ok && staged) stage_words(streams, sw, D, nw, stride, words);
  copy_vec16(sh, g_lm_levels0, TACTKV_LV0_VEC);
  const uint4* srec = recs + (size_t)u * g.N + (size_t)ks * ((g.H + 1) / 2) * g.W;
  const int na = ok ? stage_active(srec, HW, g.W, actrec, act, &s_count, s_warp) : 0;
  if (head_gains_on(g.flags)) {
    head_gain_records(g, pay, h, ks, na, actrec, act);
    __syncthreads();
  }
  for (int i = threadIdx.x; i < G * na; i += blockDim.x) {
    const int a = i / G, gq = i - a * G;
    wt[i] = ptil[((size_t)u * q_heads + (size_t)h * G + gq) * g.N + (size_t)ks * HW + act[a]] *
            __uint_as_float(actrec[a].x);
  }
  cp_async_wait_all();
  __syncthreads();
  auto channels = [&](auto global) {
    constexpr bool kGlobal = decltype(global)::value;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float acc[GM];
#pragma unroll
      for (int gq = 0; gq < GM; ++gq) acc[gq] = 0.f;
      const uint32_t* row = kGlobal ? streams + (size_t)d * sw : words + d * stride;
      // four bins' loads in flight at a time; the sums keep their order
#pragma unroll 4
      for (int a = 0; a < na; ++a) {
        const float lv = level_at<kGlobal>(row, actrec[a].y, lvs1);   // (sigma is in the weights)
#pragma unroll
        for (int gq = 0; gq < GM; ++gq)
          if (gq < G) acc[gq] = fmaf(wt[a * G + gq], lv, acc[gq]);
      }
#pragma unroll
      for (int gq = 0; gq < GM; ++gq)
        if (gq < G) part[(((size_t)u * g.S + ks) * q_heads + (size_t)h * G + gq) * D + d] = acc[gq];
    }
  };
  if (staged) channels(BoolTag<false>{});
  else channels(BoolTag<true>{});
}

// out[u][j][d] = (R^T) sum over slabs, in slab order, of part / l (blockDim a multiple of 32;
// channels d of one warp are 32 consecutive ones of a rotation group).
__global__ void __launch_bounds__(kAttnThreads) attn_reduce_kernel(const __grid_constant__ Geom g,
                                                                   const float* __restrict__ part,
                                                                   const float* __restrict__ l_in, int q_heads,
                                                                   float* __restrict__ out) {
  const int j = blockIdx.x, u = blockIdx.y, D = g.head_dim, G = q_heads / g.heads, h = j / G;
  const float lj = l_in[(size_t)u * q_heads + j];
  const float inv_l = lj > 0.f ? 1.f / lj : 0.f;   // l = 0: a unit without tokens (corrupt payload)
  const bool rotate = g.flags & TACTKV_ROTATE;
  const int lane = threadIdx.x & 31;
  for (int d0 = 0; d0 < D; d0 += blockDim.x) {
    const int d = d0 + threadIdx.x;
    float acc = 0.f;
    if (d < D) {   // in slab order; the loads of 16 slabs are issued before their sums
      const float* pp = part + ((size_t)u * g.S * q_heads + j) * D + d;
      const size_t st = (size_t)q_heads * D;
      int ks = 0;
      for (; ks + 16 <= g.S; ks += 16) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = pp[(size_t)(ks + i) * st];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc += v[i];
      }
      for (; ks < g.S; ++ks) acc += pp[(size_t)ks * st];
    }
    if (rotate)   // R^T y = diag(s) H y / sqrt(32); D is a multiple of 32, so whole warps take part
      acc = warp_wht(acc, lane) * kInvSqrt32 * rotation_sign((unsigned long long)(h * D + (d < D ? d : 0)));
    if (d < D) out[((size_t)u * q_heads + j) * D + d] = acc * inv_l;
  }
}

}  // namespace

size_t attention_scores_smem(const Geom& g, int q_heads) {
  const int G = q_heads / g.heads;
  return (size_t)(kLv0Floats + G * g.head_dim + (G * g.HW + 1) / 2 * 2) * 4 +
         (size_t)pad32(g.HW) * 12 + (size_t)g.head_dim * attn_word_stride(g.HW, g.bits) * 4;
}
size_t attention_softmax_smem(const Geom& g) { return softmax_smem(g); }
size_t attention_values_smem(const Geom& g, int q_heads) {
  const int G = q_heads / g.heads;
  return (size_t)(kLv0Floats + (G * g.HW + 1) / 2 * 2) * 4 + (size_t)pad32(g.HW) * 12 +
         (size_t)g.head_dim * attn_word_stride(g.HW, g.bits) * 4;
}

// One thread per channel of the head (head_dim is a multiple of 32), at most kAttnThreads.
inline int values_threads(int D) { return D < kAttnThreads ? D : kAttnThreads; }

cudaError_t launch_attention(const Geom& g, const UnitList& kl, const UnitList& vl, int nu, int q_heads,
                             const uint32_t* kidx, const uint4* krec, const uint32_t* vidx, const uint4* vrec,
                             const float* q, float* zp, float* part, float* out, float* m, float* l,
                             cudaStream_t st) {
  const size_t s1 = attention_scores_smem(g, q_heads), s3 = attention_values_smem(g, q_heads);
  const size_t s2 = softmax_smem(g);
  if (s1 > 227 * 1024 || s2 > 227 * 1024 || s3 > 227 * 1024 || q_heads / g.heads > kMaxG)
    return cudaErrorInvalidConfiguration;
  cudaFuncSetAttribute(attn_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
  // the softmax kernel for this grid: exact pencil lengths for the common ones
  auto softmax = attn_softmax_kernel<0, 0, 0>;
  if (g.S == 64 && g.H == 16 && g.W == 16) softmax = attn_softmax_kernel<64, 16, 16>;
  else if (g.S == 64 && g.H == 14 && g.W == 14) softmax = attn_softmax_kernel<64, 14, 14>;
  else if (g.S == 32 && g.H == 24 && g.W == 24) softmax = attn_softmax_kernel<32, 24, 24>;
  else if (g.S == 8 && g.H == 8 && g.W == 8) softmax = attn_softmax_kernel<8, 8, 8>;
  cudaFuncSetAttribute(softmax, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
  auto values = q_heads / g.heads <= 4 ? attn_values_kernel<4> : attn_values_kernel<kMaxG>;
  cudaFuncSetAttribute(values, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3);
  attn_scores_kernel<<<dim3(g.S, g.heads, nu), kScoreThreads, s1, st>>>(g, kl, kidx, krec, q, q_heads, zp);
  softmax<<<dim3(q_heads, nu), kSoftmaxThreads, s2, st>>>(g, kidx, vidx, zp, m, l, q_heads);
  values<<<dim3(g.S, g.heads, nu), values_threads(g.head_dim), s3, st>>>(g, vl, vidx, vrec, zp, q_heads, part);
  attn_reduce_kernel<<<dim3(q_heads, nu), kAttnThreads, 0, st>>>(g, part, l, q_heads, out);
  return cudaGetLastError();
}

}  // namespace tactkv
