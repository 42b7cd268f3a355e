// Per-unit bit allocation (TACT-KV stage 3) and payload header, one CTA per unit.
//
// sigma_i^2 = (1/n) sum_c X[i, c]^2 is assembled in fp64 from the per-chunk fp32 energy sums in
// a fixed order (deterministic) by reduce_var_kernel, spread over the whole GPU.  The pages allocate by reverse water-filling,
// b_i = max(0, 1/2 log2(sigma_i^2 / theta)) with theta from bisection, rounding, a +-1 greedy
// fix to hit the budget B = bits * N exactly and a cap of 8 bits.  Rounding at theta keeps the
// keys sigma_i^2 4^-k (k = 0..7) that are >= 2 theta, and each greedy step adds the largest
// missing key or drops the smallest kept one, so the result is the set of the B largest keys
// (ties to the lower bin index).  This kernel selects that set directly and exactly:
//   * count(v) = #keys >= v is evaluated per bin from the fp64 exponent and mantissa fields
//     (sigma^2 4^-k >= v  <=>  2k <= e(sigma^2) - e(v) - 1 + [m(sigma^2) >= m(v)]);
//   * the B-th largest key is found by bisection over the 64-bit patterns of positive doubles
//     (monotone in value), ~62 steps of one block-wide count;
//   * keys equal to that value are handed out in bin order until the budget is met.
// If the active bins cannot absorb B (8 * #active <= B) every active bin gets 8 bits.
#include "common.cuh"

namespace tactkv {
namespace {

constexpr size_t kAllocSmemVar = 200 * 1024;   // variances kept in shared memory up to N = 25600 bins

// Number of keys var * 4^-k (k = 0..7) that are >= v, exactly; var > 0, v >= 0.
__device__ __forceinline__ int key_count(double var, double v) {
  const unsigned long long a = __double_as_longlong(var), b = __double_as_longlong(v);
  const int ea = (int)(a >> 52), eb = (int)(b >> 52);
  if (ea == 0 || eb == 0) {  // subnormal or zero operand: compare the keys directly (exact)
    int c = 0;
    double k = var;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c += k >= v;
      k *= 0.25;
    }
    return c;
  }
  const int g = (a & 0xFFFFFFFFFFFFFull) >= (b & 0xFFFFFFFFFFFFFull);
  const int d = ea - eb - 1 + g;  // key k qualifies iff 2k <= d
  if (d < 0) return 0;
  return min(8, d / 2 + 1);
}

template <class T>
__device__ T block_sum(T v, T* s_red /* 32 entries */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  T r = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += s_red[w];
  return r;
}

__device__ double block_max(double v, double* s_red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  double r = s_red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = fmax(r, s_red[w]);
  return r;
}

// sigma_i^2 = (1/n) sum over the channel chunks of the fp32 per-chunk energy sums, in fp64 and
// in a fixed order; one thread per bin across the whole GPU.
__global__ void __launch_bounds__(256) reduce_var_kernel(const __grid_constant__ Geom g, const float* __restrict__ partial,
                                                         double* __restrict__ var_ws) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int u = blockIdx.y;
  if (i >= g.N) return;
  const float* p = partial + (size_t)u * g.nch * g.N + i;
  double acc = 0.0;
#pragma unroll 8
  for (int q = 0; q < g.nch; ++q) acc += (double)__ldcs(p + (size_t)q * g.N);
  var_ws[(size_t)u * g.N + i] = acc / (double)g.n;
}

__global__ void __launch_bounds__(kAllocThreads) allocate_kernel(const __grid_constant__ Geom g,
                                                                 const __grid_constant__ UnitList ul,
                                                                 double* __restrict__ var_ws, bool var_in_smem) {
  __shared__ long long s_ll[32];
  __shared__ double s_d[32];
  __shared__ uint32_t s_scan[33];
  __shared__ uint32_t s_cnt[kAllocThreads];
  extern __shared__ __align__(16) unsigned char smem_var[];
  const int u = blockIdx.x;
  const UnitDev& ud = ul.u[u];
  unsigned char* pay = ud.payload;
  // the bisection reads every variance ~64 times: keep them in shared memory when they fit
  double* var = var_in_smem ? reinterpret_cast<double*>(smem_var) : var_ws + (size_t)u * g.N;
  const bool raw = g.flags & TACTKV_NO_QUANT;
  // each thread owns a contiguous range of bins, so thread order is bin order
  const int per = (g.N + blockDim.x - 1) / blockDim.x;
  const int beg = min(g.N, (int)threadIdx.x * per), end = min(g.N, beg + per);

  // 1. sigma^2 (reduced over the channel chunks by reduce_var_kernel)
  long long act = 0;
  double vmax = 0.0;
  const double* var_g = var_ws + (size_t)u * g.N;
  for (int i = beg; i < end; ++i) {
    const double v = var_g[i];
    var[i] = v;
    act += v > 0.0;
    vmax = fmax(vmax, v);
  }
  act = block_sum<long long>(act, s_ll);
  vmax = block_max(vmax, s_d);
  const long long B = (long long)g.bits * g.N;
  const bool select = !raw && 8 * act > B;

  // 2. the B-th largest key: largest pattern lo with count(lo) >= B; count(lo + 1) < B
  unsigned long long lo = 0, hi = 0;
  if (select) {
    hi = (unsigned long long)__double_as_longlong(vmax) + 1ull;   // above every key: count = 0 < B
    while (hi - lo > 1) {                                         // count(+0) = 8 * act > B
      const unsigned long long mid = lo + (hi - lo) / 2;
      const double v = __longlong_as_double((long long)mid);
      long long c = 0;
      for (int i = beg; i < end; ++i) {
        const double x = var[i];
        if (x > 0.0) c += key_count(x, v);
      }
      c = block_sum<long long>(c, s_ll);
      if (c >= B) lo = mid;
      else hi = mid;
    }
  }
  const double v_lo = __longlong_as_double((long long)lo), v_hi = __longlong_as_double((long long)hi);

  // 3. keys strictly above the threshold key are all taken; equal keys go to the lowest bins
  long long c_gt = 0;
  uint32_t my_eq = 0;
  if (select) {
    for (int i = beg; i < end; ++i) {
      const double x = var[i];
      if (x > 0.0) {
        const int above = key_count(x, v_hi);
        c_gt += above;
        my_eq += key_count(x, v_lo) - above;
      }
    }
    c_gt = block_sum<long long>(c_gt, s_ll);
  }
  const long long need = B - c_gt;
  s_cnt[threadIdx.x] = my_eq;
  __syncthreads();
  block_exclusive_scan(s_cnt, blockDim.x, s_scan);
  long long rank = s_cnt[threadIdx.x];
  long long code_bits_local = 0;
  for (int i = beg; i < end; ++i) {
    const double x = var[i];
    int b = 0;
    if (!raw && x > 0.0) {
      if (!select) {
        b = 8;
      } else {
        b = key_count(x, v_hi);
        if (key_count(x, v_lo) > b) {
          if (rank < need) b += 1;
          rank += 1;
        }
      }
    }
    pay[kHeaderBytes + i] = (unsigned char)b;
    reinterpret_cast<float*>(pay + g.off_sigma)[i] = (float)sqrt(x);
    code_bits_local += b;
  }
  // zero padding after the b[] and sigma[] arrays
  for (int i = kHeaderBytes + g.N + threadIdx.x; i < g.off_sigma; i += blockDim.x) pay[i] = 0;
  for (int i = g.off_sigma + 4 * g.N + threadIdx.x; i < g.off_codes; i += blockDim.x) pay[i] = 0;
  const long long code_bits = raw ? 32LL * g.N : block_sum<long long>(code_bits_local, s_ll);
  if (threadIdx.x == 0) {
    const long long cstride = pad16((code_bits + 7) / 8);
    uint32_t* h32 = reinterpret_cast<uint32_t*>(pay);
    int32_t* i32 = reinterpret_cast<int32_t*>(pay);
    h32[0] = kMagic;
    h32[1] = (uint32_t)kVersion | ((uint32_t)(g.flags & TACTKV_NO_QUANT) << 16);
    i32[2] = ud.layer;
    i32[3] = ud.kv;
    i32[4] = g.S;
    i32[5] = g.H;
    i32[6] = g.W;
    i32[7] = g.heads;
    i32[8] = g.head_dim;
    i32[9] = g.bits;
    h32[10] = (uint32_t)code_bits;
    h32[11] = (uint32_t)cstride;
    *reinterpret_cast<unsigned long long*>(pay + 48) =
        (unsigned long long)((long long)g.off_codes + (long long)g.n * cstride);
    h32[14] = 0;
    h32[15] = 0;
  }
}

}  // namespace

cudaError_t launch_allocate(const Geom& g, const UnitList& ul, int nu, const float* partial, double* var,
                            cudaStream_t st) {
  const size_t var_bytes = (size_t)g.N * sizeof(double);
  const bool in_smem = var_bytes <= kAllocSmemVar;
  if (in_smem) cudaFuncSetAttribute(allocate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)var_bytes);
  reduce_var_kernel<<<dim3((g.N + 255) / 256, nu), 256, 0, st>>>(g, partial, var);
  allocate_kernel<<<nu, kAllocThreads, in_smem ? var_bytes : 0, st>>>(g, ul, var, in_smem);
  return cudaGetLastError();
}

}  // namespace tactkv
