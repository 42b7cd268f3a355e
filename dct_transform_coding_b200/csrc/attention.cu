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

// Stage the slab's dense decoding records in shared memory and list the slab's bins that have
// bits (in bin order): act[a] = bin index j, actrec[a] = {sigma, offset << 8 | code mask} of that
// bin.  Returns the count.  Called by every thread; ends with a barrier.
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
  return *s_count;
}

// Code of a bin with bits (record {sigma, offset << 8 | mask}) in this lane's channel stream
// `row` (the slab's first word); only words that hold some of its bits are read.
__device__ __forceinline__ uint32_t read_code(const uint32_t* __restrict__ row, uint32_t mk) {
  const uint32_t k = mk & 0xffu, off = mk >> 8;
  const uint32_t* w = row + (off >> 5);
  const uint32_t lo = __ldg(w), hi = (off & 31u) + (uint32_t)__popc(k) > 32u ? __ldg(w + 1) : 0u;
  return __funnelshift_r(lo, hi, off) & k;
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
  __shared__ int s_count, s_warp[32];
  const int ks = blockIdx.x, h = blockIdx.y, u = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int G = q_heads / g.heads, D = g.head_dim, HW = g.HW;
  float* lvs1 = sh + 1;                             // a zero in front of the levels
  float* qs = sh + (kLmLvTotal + 1 + 3) / 4 * 4;    // [G][D], rotated when the payload is
  float* s_part = qs + G * D;                       // [nwarps][G][HW], by active-bin index
  uint2* actrec = reinterpret_cast<uint2*>(s_part + (size_t)nwarps * G * HW);   // [HW]
  int* act = reinterpret_cast<int*>(actrec + HW);                                 // [HW]
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
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const bool ok = P[g.S + 1] != 0;
  const unsigned char* pay = ul.u[u].payload;
  const uint4* srec = recs + (size_t)u * g.N + (size_t)ks * ((g.H + 1) / 2) * g.W;
  const int na = ok ? stage_active(srec, HW, g.W, actrec, act, &s_count, s_warp) : 0;
  if (!ok) __syncthreads();
  if (na > 0) {
    const uint32_t sw = reinterpret_cast<const uint32_t*>(pay)[11] / 4, w0 = P[ks] >> 5;
    const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes);
    float* mine = s_part + (size_t)warp * G * HW;
    for (int cg = warp; cg < D / 32; cg += nwarps) {
      const int d = cg * 32 + lane;
      const uint32_t* row = streams + (size_t)(h * D + d) * sw + w0;
      for (int a0 = 0; a0 < na; a0 += 32) {
        float val[32];
#pragma unroll
        for (int b = 0; b < 32; ++b) {
          val[b] = 0.f;
          if (a0 + b < na) {
            const uint2 r = actrec[a0 + b];
            const uint32_t k = r.y & 0xffu;
            val[b] = __uint_as_float(r.x) * lvs1[(int)(k + read_code(row, r.y)) - 1];
          }
        }
        for (int gq = 0; gq < G; ++gq) {
          const float qd = qs[gq * D + d];
          float t[32];
#pragma unroll
          for (int b = 0; b < 32; ++b) t[b] = val[b] * qd;
          // sum over the warp's 32 channels: lane l ends with active bin a0 + l
#pragma unroll
          for (int hh = 16; hh >= 1; hh >>= 1) {
            const bool upper = lane & hh;
#pragma unroll
            for (int i = 0; i < hh; ++i) {
              const float send = upper ? t[i] : t[i + hh], keep = upper ? t[i + hh] : t[i];
              t[i] = keep + __shfl_xor_sync(0xffffffffu, send, hh);
            }
          }
          if (a0 + lane < na) mine[gq * HW + a0 + lane] += t[0];
        }
      }
    }
  }
  __syncthreads();
  const float scale = rsqrtf((float)D);
  float* zu = z + ((size_t)u * q_heads + (size_t)h * G) * g.N + (size_t)ks * HW;
  for (int i = threadIdx.x; i < G * HW; i += blockDim.x) {   // bins without bits: z = 0
    const int gq = i / HW, j = i - gq * HW;
    zu[(size_t)gq * g.N + j] = 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * na; i += blockDim.x) {
    const int gq = i / na, a = i - gq * na;
    float acc = 0.f;
    for (int w = 0; w < nwarps; ++w) acc += s_part[((size_t)w * G + gq) * HW + a];
    zu[(size_t)gq * g.N + act[a]] = acc * scale;
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
template <bool INV, int SX, int HX, int WX>
__device__ void dct3_volume(float* vol, const Geom& g) {
  const int S = g.S, H = g.H, W = g.W;
  // along W: pencils (s, h), contiguous; along H: (s, w), stride W; along S: (h, w), stride H*W
  if (!(g.flags & TACTKV_SKIP_W)) pencils_any<WX, INV>(vol, W, S * H, 1, W, 1);
  __syncthreads();
  if (!(g.flags & TACTKV_SKIP_H)) pencils_any<HX, INV>(vol, H, S * W, W, H * W, W);
  __syncthreads();
  if (!(g.flags & TACTKV_SKIP_S)) pencils_any<SX, INV>(vol, S, H * W, H * W, 0, H * W);
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
constexpr int kSoftmaxThreads = 512;
template <int SX, int HX, int WX>
__global__ void __launch_bounds__(kSoftmaxThreads) attn_softmax_kernel(const __grid_constant__ Geom g,
                                                                    float* __restrict__ zp, float* __restrict__ m_out,
                                                                    float* __restrict__ l_out, int q_heads) {
  extern __shared__ __align__(16) float vol[];
  __shared__ float red[32];
  const int j = blockIdx.x, u = blockIdx.y;
  float* zg = zp + ((size_t)u * q_heads + j) * g.N;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) vol[i] = zg[i];
  __syncthreads();
  dct3_volume<true, SX, HX, WX>(vol, g);
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
  dct3_volume<false, SX, HX, WX>(vol, g);
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) zg[i] = vol[i];
  if (threadIdx.x == 0) {
    m_out[(size_t)u * q_heads + j] = mx;
    l_out[(size_t)u * q_heads + j] = sum;
  }
}

// part[u][ks][j][d] = sum over the bins i of slab ks of dct3(p_j)[i] * X_V[i, hD + d] (rotated
// domain when the payload is); thread = channel, G accumulators each, no reduction across threads.
// Only bins with bits are visited; their weights dct3(p_j)[i] * sigma_i are formed once per CTA.
__global__ void __launch_bounds__(kAttnThreads) attn_values_kernel(const __grid_constant__ Geom g,
                                                                   const __grid_constant__ UnitList ul,
                                                                   const uint32_t* __restrict__ index,
                                                                   const uint4* __restrict__ recs,
                                                                   const float* __restrict__ ptil, int q_heads,
                                                                   float* __restrict__ part) {
  extern __shared__ __align__(16) float sh[];
  __shared__ int s_count, s_warp[32];
  const int ks = blockIdx.x, h = blockIdx.y, u = blockIdx.z;
  const int G = q_heads / g.heads, D = g.head_dim, HW = g.HW;
  float* lvs1 = sh + 1;
  float* wt = sh + (kLmLvTotal + 1 + 3) / 4 * 4;        // [HW][G]: weight of active bin a for head g
  uint2* actrec = reinterpret_cast<uint2*>(wt + ((size_t)G * HW + 1) / 2 * 2);   // 8-byte aligned
  int* act = reinterpret_cast<int*>(actrec + HW);
  for (int i = threadIdx.x; i <= kLmLvTotal; i += blockDim.x) sh[i] = i ? c_lm_levels[i - 1] : 0.f;
  const uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  const bool ok = P[g.S + 1] != 0;
  const unsigned char* pay = ul.u[u].payload;
  const uint4* srec = recs + (size_t)u * g.N + (size_t)ks * ((g.H + 1) / 2) * g.W;
  const int na = ok ? stage_active(srec, HW, g.W, actrec, act, &s_count, s_warp) : 0;
  if (!ok) __syncthreads();
  for (int i = threadIdx.x; i < G * na; i += blockDim.x) {
    const int a = i / G, gq = i - a * G;
    wt[i] = ptil[((size_t)u * q_heads + (size_t)h * G + gq) * g.N + (size_t)ks * HW + act[a]] *
            __uint_as_float(actrec[a].x);
  }
  __syncthreads();
  const uint32_t sw = ok ? reinterpret_cast<const uint32_t*>(pay)[11] / 4 : 0u, w0 = P[ks] >> 5;
  const uint32_t* streams = reinterpret_cast<const uint32_t*>(pay + g.off_codes);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc[kMaxG];
#pragma unroll
    for (int gq = 0; gq < kMaxG; ++gq) acc[gq] = 0.f;
    const uint32_t* row = streams + (size_t)(h * D + d) * sw + w0;
    for (int a = 0; a < na; ++a) {
      const uint32_t mk = actrec[a].y;
      const float lv = lvs1[(int)((mk & 0xffu) + read_code(row, mk)) - 1];
#pragma unroll
      for (int gq = 0; gq < kMaxG; ++gq)
        if (gq < G) acc[gq] = fmaf(wt[a * G + gq], lv, acc[gq]);
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
  return (size_t)((kLmLvTotal + 1 + 3) / 4 * 4 + G * g.head_dim + (kAttnThreads / 32) * G * g.HW) * 4 +
         (size_t)g.HW * 12;
}
size_t attention_values_smem(const Geom& g, int q_heads) {
  const int G = q_heads / g.heads;
  return (size_t)((kLmLvTotal + 1 + 3) / 4 * 4 + (G * g.HW + 1) / 2 * 2) * 4 + (size_t)g.HW * 12;
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
  // the softmax kernel for this grid: exact pencil lengths for the common ones
  auto softmax = attn_softmax_kernel<0, 0, 0>;
  if (g.S == 64 && g.H == 16 && g.W == 16) softmax = attn_softmax_kernel<64, 16, 16>;
  else if (g.S == 64 && g.H == 14 && g.W == 14) softmax = attn_softmax_kernel<64, 14, 14>;
  else if (g.S == 32 && g.H == 24 && g.W == 24) softmax = attn_softmax_kernel<32, 24, 24>;
  else if (g.S == 8 && g.H == 8 && g.W == 8) softmax = attn_softmax_kernel<8, 8, 8>;
  cudaFuncSetAttribute(softmax, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
  cudaFuncSetAttribute(attn_values_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3);
  attn_scores_kernel<<<dim3(g.S, g.heads, nu), kAttnThreads, s1, st>>>(g, kl, kidx, krec, q, q_heads, zp);
  softmax<<<dim3(q_heads, nu), kSoftmaxThreads, s2, st>>>(g, zp, m, l, q_heads);
  attn_values_kernel<<<dim3(g.S, g.heads, nu), kAttnThreads, s3, st>>>(g, vl, vidx, vrec, zp, q_heads, part);
  attn_reduce_kernel<<<dim3(q_heads, nu), kAttnThreads, 0, st>>>(g, part, l, q_heads, out);
  return cudaGetLastError();
}

}  // namespace tactkv
