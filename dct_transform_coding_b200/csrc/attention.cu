// One decode step of attention over compressed visual K/V, without reconstructing the cache (the
// paragraph after stage 4 of "Methodology in Plain English" on the TACT-KV summary page: decoding
// can be fused into the attention kernel).
//
// The 3D DCT is linear and orthonormal per channel, so with X_K, X_V the dequantized coefficients
// (bin i, channel c) and C3 the 3D DCT-II:
//   scores   s_j[t] = q_j . K[t] / sqrt(D) = idct3(z_j)[t],   z_j[i] = sum_d q_j[d] X_K[i, hD + d] / sqrt(D)
//   output   o_j    = sum_t p_j[t] V[t]    = sum_i dct3(p_j)[i] X_V[i, hD + d]
// with p_j[t] = exp(s_j[t] - m_j), m_j = max_t s_j[t], l_j = sum_t p_j[t], and out_j = o_j / l_j
// (query head j uses K/V head h = j / G).  Only bins with bits are decoded, straight from the
// payloads' channel streams; the volumes of T values per query head are transformed in shared
// memory.  With the shared rotation R (per 32-channel group), X = R^T X' for the coded X': the
// query is rotated (q . R^T x' = (R q) . x') and the output rotated back at the end.
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

// Value of bin (ks, j) of this lane's channel, from the payload's channel stream and the slab's
// dense decoding record: sigma * level[code] (0 for a bin without bits).  `row` points at the
// channel's stream word where slab ks starts (P(ks) rounded down to 32 bits).
__device__ __forceinline__ float decode_value(const uint4* __restrict__ srec, const uint32_t* __restrict__ row,
                                              const float* __restrict__ lvs1, int W, int j) {
  const int kh = j / W, t = j - kh * W;
  const uint4 m = srec[(kh >> 1) * W + t];
  const uint32_t mk = (kh & 1) ? m.w : m.z;
  const float sg = __uint_as_float((kh & 1) ? m.y : m.x);
  const uint32_t k = mk & 0xffu, off = mk >> 8;
  if (k == 0u) return 0.f;                 // no bits: nothing of this bin is in the stream
  // the code's bits lie inside the stream, so only words that hold some of them are read
  const uint32_t* w = row + (off >> 5);
  const uint32_t lo = __ldg(w), hi = (off & 31u) + (uint32_t)__popc(k) > 32u ? __ldg(w + 1) : 0u;
  const uint32_t code = __funnelshift_r(lo, hi, off) & k;
  return sg * lvs1[(int)(k + code) - 1];
}

// z_j[i] for the G query heads of K/V head h over the bins of slab ks.  Warp w handles the channel
// groups w, w + 8, ... of the head (lane = channel); each warp's per-bin sums over its 32 channels
// go to its own row of s_part and are added up in warp order (deterministic).
__global__ void __launch_bounds__(kAttnThreads) attn_scores_kernel(const __grid_constant__ Geom g,
                                                                   const __grid_constant__ UnitList ul,
                                                                   const uint32_t* __restrict__ index,
                                                                   const uint4* __restrict__ recs,
                                                                   const float* __restrict__ q, int q_heads,
                                                                   float* __restrict__ z) {
  extern __shared__ __align__(16) float sh[];
  const int ks = blockIdx.x, h = blockIdx.y, u = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int G = q_heads / g.heads, D = g.head_dim, HW = g.HW;
  float* lvs1 = sh + 1;                             // a zero in front of the levels
  float* qs = sh + (kLmLvTotal + 1 + 3) / 4 * 4;    // [G][D], rotated when the payload is
  float* s_part = qs + G * D;                       // [nwarps][G][HW]
  for (int i = threadIdx.x; i <= kLmLvTotal; i += blockDim.x) sh[i] = i ? c_lm_levels[i - 1] : 0.f;
  const float* qu = q + ((size_t)u * q_heads + (size_t)h * G) * D;
  const bool rotate = g.flags & TACTKV_ROTATE;
  for (int gg = warp; gg < G * (D / 32); gg += nwarps) {   // (query head, channel group) per warp
    const int gq = gg / (D / 32), cg = gg - gq * (D / 32), d = cg * 32 + lane;
    float v = qu[(size_t)gq * D + d];
    if (rotate) v = warp_wht(v * rotation_sign((unsigned long long)(h * D + d)), lane) * kInvSqrt32;
    qs[gq * D + d] = v;
  }
  for (int i = threadIdx.x; i < nwarps * G * HW; i += blockDim.x) s_part[i] = 0.f;
  __syncthreads();
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const bool ok = P[g.S + 1] != 0;
  const unsigned char* pay = ul.u[u].payload;
  if (ok) {
    const uint32_t sw = reinterpret_cast<const uint32_t*>(pay)[11] / 4, w0 = P[ks] >> 5;
    const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes);
    const uint4* srec = recs + (size_t)u * g.N + (size_t)ks * ((g.H + 1) / 2) * g.W;
    float* mine = s_part + (size_t)warp * G * HW;
    for (int cg = warp; cg < D / 32; cg += nwarps) {
      const int d = cg * 32 + lane;
      const uint32_t* row = streams + (size_t)(h * D + d) * sw + w0;
      for (int j0 = 0; j0 < HW; j0 += 32) {
        float val[32];
#pragma unroll
        for (int b = 0; b < 32; ++b) val[b] = j0 + b < HW ? decode_value(srec, row, lvs1, g.W, j0 + b) : 0.f;
        for (int gq = 0; gq < G; ++gq) {
          const float qd = qs[gq * D + d];
          float t[32];
#pragma unroll
          for (int b = 0; b < 32; ++b) t[b] = val[b] * qd;
          // sum over the warp's 32 channels: lane l ends with bin j0 + l
#pragma unroll
          for (int hh = 16; hh >= 1; hh >>= 1) {
            const bool upper = lane & hh;
#pragma unroll
            for (int i = 0; i < hh; ++i) {
              const float send = upper ? t[i] : t[i + hh], keep = upper ? t[i + hh] : t[i];
              t[i] = keep + __shfl_xor_sync(0xffffffffu, send, hh);
            }
          }
          if (j0 + lane < HW) mine[gq * HW + j0 + lane] += t[0];
        }
      }
    }
  }
  __syncthreads();
  const float scale = rsqrtf((float)D);
  for (int i = threadIdx.x; i < G * HW; i += blockDim.x) {
    float acc = 0.f;
    for (int w = 0; w < nwarps; ++w) acc += s_part[(size_t)w * G * HW + i];
    const int gq = i / HW, j = i - gq * HW;
    z[((size_t)u * q_heads + (size_t)h * G + gq) * g.N + (size_t)ks * HW + j] = acc * scale;
  }
}

// In-place separable DCT-II (INV = false) or DCT-III (INV = true) of a single-channel volume
// vol[S][H][W] in shared memory, skipping the axes the payload left untransformed.
template <int CLASS, bool INV>
__device__ __forceinline__ void pencils(float* vol, int L, int count, int stride, int step_outer, int inner) {
  for (int p = threadIdx.x; p < count; p += blockDim.x) {
    const int o = p / inner, i = p - o * inner;
    float* base = vol + (size_t)o * step_outer + i;
    float x[CLASS];
#pragma unroll
    for (int k = 0; k < CLASS; ++k)
      if (k < L) x[k] = base[(size_t)k * stride];
    dct_pencil<CLASS, INV>(x, L);
#pragma unroll
    for (int k = 0; k < CLASS; ++k)
      if (k < L) base[(size_t)k * stride] = x[k];
  }
}
template <bool INV>
__device__ void pencils_any(float* vol, int L, int count, int stride, int step_outer, int inner) {
  const int c = length_class_dev(L);
  if (c == 16) pencils<16, INV>(vol, L, count, stride, step_outer, inner);
  else if (c == 32) pencils<32, INV>(vol, L, count, stride, step_outer, inner);
  else pencils<64, INV>(vol, L, count, stride, step_outer, inner);
}
template <bool INV>
__device__ void dct3_volume(float* vol, const Geom& g) {
  const int S = g.S, H = g.H, W = g.W;
  // along W: pencils (s, h), contiguous; along H: (s, w), stride W; along S: (h, w), stride H*W
  if (!(g.flags & TACTKV_SKIP_W)) pencils_any<INV>(vol, W, S * H, 1, W, 1);
  __syncthreads();
  if (!(g.flags & TACTKV_SKIP_H)) pencils_any<INV>(vol, H, S * W, W, H * W, W);
  __syncthreads();
  if (!(g.flags & TACTKV_SKIP_S)) pencils_any<INV>(vol, S, H * W, H * W, 0, H * W);
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
__global__ void __launch_bounds__(kAttnThreads) attn_softmax_kernel(const __grid_constant__ Geom g,
                                                                    float* __restrict__ zp, float* __restrict__ m_out,
                                                                    float* __restrict__ l_out, int q_heads) {
  extern __shared__ __align__(16) float vol[];
  __shared__ float red[32];
  const int j = blockIdx.x, u = blockIdx.y;
  float* zg = zp + ((size_t)u * q_heads + j) * g.N;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) vol[i] = zg[i];
  __syncthreads();
  dct3_volume<true>(vol, g);
  float mx = -INFINITY;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) mx = fmaxf(mx, vol[i]);
  mx = block_reduce(mx, red, true);
  float sum = 0.f;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
    const float e = __expf(vol[i] - mx);
    vol[i] = e;
    sum += e;
  }
  sum = block_reduce(sum, red, false);
  __syncthreads();
  dct3_volume<false>(vol, g);
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) zg[i] = vol[i];
  if (threadIdx.x == 0) {
    m_out[(size_t)u * q_heads + j] = mx;
    l_out[(size_t)u * q_heads + j] = sum;
  }
}

// part[u][ks][j][d] = sum over the bins i of slab ks of dct3(p_j)[i] * X_V[i, hD + d] (rotated
// domain when the payload is); thread = channel, G accumulators each, no reduction across threads.
__global__ void __launch_bounds__(kAttnThreads) attn_values_kernel(const __grid_constant__ Geom g,
                                                                   const __grid_constant__ UnitList ul,
                                                                   const uint32_t* __restrict__ index,
                                                                   const uint4* __restrict__ recs,
                                                                   const float* __restrict__ ptil, int q_heads,
                                                                   float* __restrict__ part) {
  extern __shared__ __align__(16) float sh[];
  const int ks = blockIdx.x, h = blockIdx.y, u = blockIdx.z;
  const int G = q_heads / g.heads, D = g.head_dim, HW = g.HW;
  float* lvs1 = sh + 1;
  float* pt = sh + (kLmLvTotal + 1 + 3) / 4 * 4;    // [G][HW]
  for (int i = threadIdx.x; i <= kLmLvTotal; i += blockDim.x) sh[i] = i ? c_lm_levels[i - 1] : 0.f;
  for (int i = threadIdx.x; i < G * HW; i += blockDim.x) {
    const int gq = i / HW, jj = i - gq * HW;
    pt[i] = ptil[((size_t)u * q_heads + (size_t)h * G + gq) * g.N + (size_t)ks * HW + jj];
  }
  __syncthreads();
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const bool ok = P[g.S + 1] != 0;
  const unsigned char* pay = ul.u[u].payload;
  const uint32_t sw = ok ? reinterpret_cast<const uint32_t*>(pay)[11] / 4 : 0u, w0 = P[ks] >> 5;
  const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes);
  const uint4* srec = recs + (size_t)u * g.N + (size_t)ks * ((g.H + 1) / 2) * g.W;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc[kMaxG];
#pragma unroll
    for (int gq = 0; gq < kMaxG; ++gq) acc[gq] = 0.f;
    if (ok) {
      const uint32_t* row = streams + (size_t)(h * D + d) * sw + w0;
      for (int j = 0; j < HW; ++j) {
        const float v = decode_value(srec, row, lvs1, g.W, j);
#pragma unroll
        for (int gq = 0; gq < kMaxG; ++gq)
          if (gq < G) acc[gq] = fmaf(pt[gq * HW + j], v, acc[gq]);
      }
    }
    for (int gq = 0; gq < G; ++gq)
      part[(((size_t)u * g.S + ks) * q_heads + (size_t)h * G + gq) * D + d] = acc[gq];
  }
}

// out[u][j][d] = (R^T) sum over slabs, in slab order, of part / l (blockDim a multiple of 32;
// channels d of one warp are 32 consecutive ones of a rotation group).
__global__ void __launch_bounds__(kAttnThreads) attn_reduce_kernel(const __grid_constant__ Geom g,
                                                                   const float* __restrict__ part,
                                                                   const float* __restrict__ l_in, int q_heads,
                                                                   float* __restrict__ out) {
  const int j = blockIdx.x, u = blockIdx.y, D = g.head_dim, G = q_heads / g.heads, h = j / G;
  const float inv_l = 1.f / l_in[(size_t)u * q_heads + j];
  const bool rotate = g.flags & TACTKV_ROTATE;
  const int lane = threadIdx.x & 31;
  for (int d0 = 0; d0 < D; d0 += blockDim.x) {
    const int d = d0 + threadIdx.x;
    float acc = 0.f;
    if (d < D)
      for (int ks = 0; ks < g.S; ++ks) acc += part[(((size_t)u * g.S + ks) * q_heads + j) * D + d];
    if (rotate)   // R^T y = diag(s) H y / sqrt(32); D is a multiple of 32, so whole warps take part
      acc = warp_wht(acc, lane) * kInvSqrt32 * rotation_sign((unsigned long long)(h * D + (d < D ? d : 0)));
    if (d < D) out[((size_t)u * q_heads + j) * D + d] = acc * inv_l;
  }
}

}  // namespace

size_t attention_scores_smem(const Geom& g, int q_heads) {
  const int G = q_heads / g.heads;
  return (size_t)((kLmLvTotal + 1 + 3) / 4 * 4 + G * g.head_dim + (kAttnThreads / 32) * G * g.HW) * 4;
}
size_t attention_values_smem(const Geom& g, int q_heads) {
  const int G = q_heads / g.heads;
  return (size_t)((kLmLvTotal + 1 + 3) / 4 * 4 + G * g.HW) * 4;
}

cudaError_t launch_attention(const Geom& g, const UnitList& kl, const UnitList& vl, int nu, int q_heads,
                             const uint32_t* kidx, const uint4* krec, const uint32_t* vidx, const uint4* vrec,
                             const float* q, float* zp, float* part, float* out, float* m, float* l,
                             cudaStream_t st) {
  const size_t s1 = attention_scores_smem(g, q_heads), s3 = attention_values_smem(g, q_heads);
  const size_t s2 = (size_t)g.N * 4;
  if (s1 > 227 * 1024 || s2 > 227 * 1024 || s3 > 227 * 1024 || q_heads / g.heads > kMaxG)
    return cudaErrorInvalidConfiguration;
  cudaFuncSetAttribute(attn_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
  cudaFuncSetAttribute(attn_softmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
  cudaFuncSetAttribute(attn_values_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3);
  attn_scores_kernel<<<dim3(g.S, g.heads, nu), kAttnThreads, s1, st>>>(g, kl, kidx, krec, q, q_heads, zp);
  attn_softmax_kernel<<<dim3(q_heads, nu), kAttnThreads, s2, st>>>(g, zp, m, l, q_heads);
  attn_values_kernel<<<dim3(g.S, g.heads, nu), kAttnThreads, s3, st>>>(g, vl, vidx, vrec, zp, q_heads, part);
  attn_reduce_kernel<<<dim3(q_heads, nu), kAttnThreads, 0, st>>>(g, part, l, q_heads, out);
  return cudaGetLastError();
}

}  // namespace tactkv
