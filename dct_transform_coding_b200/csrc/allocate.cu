// Per-unit bit allocation (TACT-KV stage 3) and payload header, one CTA per unit.
//
// sigma_i^2 = (1/n) sum_c X[i, c]^2 is assembled in fp64 from the per-chunk fp32 energy sums in
// a fixed order (deterministic) by reduce_var_kernel, spread over the whole GPU.  The pages allocate by reverse water-filling,
// b_i = max(0, 1/2 log2(sigma_i^2 / theta)) with theta from bisection, rounding, a +-1 greedy
// fix to hit the budget B = bits * N exactly and a cap of 8 bits.  Rounding at theta keeps the
// keys sigma_i^2 4^-k (k = 0..7) that are >= 2 theta, and each greedy step adds the largest
// missing key or drops the smallest kept one, so the result is the set of the B largest keys
// (ties to the lower bin index).  This kernel selects that set directly and exactly:
//   * the B-th largest key K is found by radix selection on its fp64 bit pattern (patterns of
//     positive doubles order like their values): a histogram of all keys' exponents, then 11-bit
//     digits of the mantissa among the keys with K's exponent.  Every key is a normal fp64
//     number: a variance is an fp64 sum of float32 energies divided by n <= 2^16, so a positive
//     one is at least 2^-149 / 2^16 = 2^-165, and its smallest key (4^-7 of it) 2^-179 lies far
//     above the smallest normal double 2^-1022;
//   * count(v) = #keys >= v is evaluated per bin from the fp64 exponent and mantissa fields
//     (sigma^2 4^-k >= v  <=>  2k <= e(sigma^2) - e(v) - 1 + [m(sigma^2) >= m(v)]);
//   * keys above K are all taken, keys equal to K are handed out in bin order until the budget
//     is met.
// If the active bins cannot absorb B (8 * #active <= B) every active bin gets 8 bits.
//
// The kernel also writes the first stream bit P(k_s) of every S slab (the same for every
// channel) and the list of bins with bits (records {bin, bits, first stream bit, 1/sigma}, in bin
// order) into the workspace.  decode_index_kernel rebuilds P from a payload before
// decoding and checks the header and the bit widths.
#include "common.cuh"

namespace tactkv {
namespace {

constexpr size_t kAllocSmemVar = 192 * 1024;   // variances kept in shared memory up to N = 24576 bins
constexpr int kExpBuckets = 2048;                // biased exponents of fp64

// Number of keys var * 4^-k (k = 0..7) that are >= v, exactly, for positive normal var and v (every
// variance and every selection threshold here is normal, see the head of this file).
__device__ __forceinline__ int key_count(double var, double v) {
  const unsigned long long a = __double_as_longlong(var), b = __double_as_longlong(v);
  const int ea = (int)(a >> 52), eb = (int)(b >> 52);
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

// sigma_i^2 = (1/n) sum over the channel chunks of the fp32 per-chunk energy sums, in fp64 and
// in a fixed order; one thread per bin across the whole GPU.  With per-head gains the same sums,
// restarted at every head's first chunk, give the gains float32(sqrt(sum / head_dim)) of bin i in
// every head, written straight into the payload's sigma[head][bin].
__global__ void __launch_bounds__(256) reduce_var_kernel(const __grid_constant__ Geom g,
                                                         const __grid_constant__ UnitList ul,
                                                         const float* __restrict__ partial,
                                                         double* __restrict__ var_ws) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int u = blockIdx.y;
  if (i >= g.N) return;
  const float* p = partial + (size_t)u * g.nch * g.N + i;
  double acc = 0.0;
  if (head_gains_on(g.flags)) {
    float* gains = reinterpret_cast<float*>(ul.u[u].payload + g.off_sigma) + i;
    const int cph = g.head_dim / kChunk;   // chunks of a head
    for (int h = 0; h < g.heads; ++h) {
      double acc_h = 0.0;
      for (int q = h * cph; q < (h + 1) * cph; ++q) {
        const double v = (double)__ldcs(p + (size_t)q * g.N);
        acc += v;
        acc_h += v;
      }
      gains[(size_t)h * g.N] = (float)sqrt(acc_h / (double)g.head_dim);
    }
  } else {
#pragma unroll 8
    for (int q = 0; q < g.nch; ++q) acc += (double)__ldcs(p + (size_t)q * g.N);
  }
  var_ws[(size_t)u * g.N + i] = acc / (double)g.n;
}

// Exclusive scan of s_slab[0..S) into out[0..S] (out[S] = total), by one warp.
__device__ void slab_scan(const uint32_t* s_slab, int S, uint32_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t run = 0;
  for (int k0 = 0; k0 < S; k0 += 32) {
    const uint32_t v = k0 + lane < S ? s_slab[k0 + lane] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (k0 + lane < S) out[k0 + lane] = run + incl - v;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) out[S] = run;
}

// Largest bucket D of hist[0..nb) with sum_{d >= D} hist[d] >= need (need >= 1, reached); returns D,
// puts sum_{d > D} hist[d] in *above and hist[D] in *count.  rev: scratch of nb words (may be the
// storage of another histogram, not hist itself).  All threads call it.
__device__ int select_bucket(const uint32_t* hist, int nb, uint32_t need, uint32_t* rev, uint32_t* s_warp,
                             int* s_pick, uint32_t* s_above, uint32_t* s_count, uint32_t* above, uint32_t* count) {
  for (int j = threadIdx.x; j < nb; j += blockDim.x) rev[j] = hist[nb - 1 - j];
  __syncthreads();
  block_exclusive_scan(rev, nb, s_warp);   // rev[j] = number of keys in buckets above nb-1-j
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const uint32_t pre = rev[j], here = hist[nb - 1 - j];
    if (pre < need && need <= pre + here) {
      *s_pick = nb - 1 - j;
      *s_above = pre;
      *s_count = here;
    }
  }
  __syncthreads();
  *above = *s_above;
  *count = *s_count;
  return *s_pick;
}

__global__ void __launch_bounds__(kAllocThreads) allocate_kernel(const __grid_constant__ Geom g,
                                                                 const __grid_constant__ UnitList ul,
                                                                 double* __restrict__ var_ws, bool var_in_smem,
                                                                 uint32_t* __restrict__ index, uint4* __restrict__ recs) {
  __shared__ long long s_ll[32];
  __shared__ uint32_t s_scan[33];
  __shared__ uint32_t s_cnt[kAllocThreads];
  __shared__ uint32_t s_slab[kMaxSlabs];
  __shared__ uint32_t s_nzslab[kMaxSlabs];
  __shared__ uint32_t s_P[kMaxSlabs + 1];
  __shared__ uint32_t s_NZ[kMaxSlabs + 1];
  __shared__ uint32_t s_hist[kExpBuckets], s_rev[kExpBuckets];
  __shared__ int s_pick;
  __shared__ uint32_t s_above, s_count;
  __shared__ unsigned long long s_mant;
  extern __shared__ __align__(16) unsigned char smem_var[];
  const int u = blockIdx.x;
  const UnitDev& ud = ul.u[u];
  unsigned char* pay = ud.payload;
  // the selection passes read every variance several times: keep them in shared memory when they fit
  double* var = var_in_smem ? reinterpret_cast<double*>(smem_var) : var_ws + (size_t)u * g.N;
  const bool raw = g.flags & TACTKV_NO_QUANT;
  // each thread owns a contiguous range of bins, so thread order is bin order
  const int per = (g.N + blockDim.x - 1) / blockDim.x;
  const int beg = min(g.N, (int)threadIdx.x * per), end = min(g.N, beg + per);

  // 1. sigma^2 (reduced over the channel chunks by reduce_var_kernel)
  long long act = 0;
  const double* var_g = var_ws + (size_t)u * g.N;
  // the counting passes take bins interleaved across threads (bin i to thread i mod blockDim):
  // consecutive threads read consecutive variances, without bank conflicts
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
    const double v = var_g[i];
    var[i] = v;
    act += v > 0.0;
  }
  act = block_sum<long long>(act, s_ll);
  const long long B = (long long)g.bits * g.N;
  const bool uniform = g.flags & TACTKV_UNIFORM_ALLOC;   // the ablation: bits for every active bin
  const bool select = !raw && !uniform && 8 * act > B;

  // 2. the B-th largest key K (counted with multiplicity): the largest pattern lo with
  // count(lo) >= B, so count(lo + 1) < B.  The keys of bin i are var_i * 4^-k: the mantissa of
  // var_i with the exponents e_i - 2k (all normal numbers, see the head of this file).  K is found
  // by radix selection: K's exponent from the histogram of all keys' exponents (the histogram of
  // the bins' exponents summed over the 8 shifts), then 11-bit digits of K's mantissa from the
  // keys with that exponent (at most one per bin), until one key is left.
  unsigned long long lo = 0, hi = 0;
  if (select) {
    for (int j = threadIdx.x; j < kExpBuckets; j += blockDim.x) s_hist[j] = 0;
    __syncthreads();
    const unsigned lt = (1u << (threadIdx.x & 31)) - 1u;
    for (int i0 = 0; i0 < g.N; i0 += blockDim.x) {   // warp-uniform rounds: bins with one exponent
      const int i = i0 + (int)threadIdx.x;           // are counted by one atomic per warp
      const double x = i < g.N ? var[i] : 0.0;
      const int e = x > 0.0 ? (int)(__double_as_longlong(x) >> 52) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && (peers & lt) == 0u) atomicAdd(&s_hist[e], (uint32_t)__popc(peers));
    }
    __syncthreads();
    for (int j = threadIdx.x; j < kExpBuckets; j += blockDim.x) {
      uint32_t c = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) c += j + 2 * k < kExpBuckets ? s_hist[j + 2 * k] : 0u;
      s_rev[j] = c;   // keys with exponent j
    }
    __syncthreads();
    uint32_t above = 0, here = 0;
    const int E = select_bucket(s_rev, kExpBuckets, (uint32_t)B, s_hist, s_scan, &s_pick, &s_above, &s_count,
                                &above, &here);
    uint32_t need = (uint32_t)B - above;      // K is the need-th largest key with exponent E
    unsigned long long prefix = 0;            // K's leading mantissa bits selected so far
    int done = 0;                             // how many of the 52 mantissa bits
    while (done < 52) {
      const int width = min(11, 52 - done), shift = 52 - done - width;
      __syncthreads();
      for (int j = threadIdx.x; j < (1 << width); j += blockDim.x) s_hist[j] = 0;
      __syncthreads();
      for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
        const unsigned long long bits = (unsigned long long)__double_as_longlong(var[i]);
        const int d = (int)(bits >> 52) - E;   // (var[i] > 0: its sign bit is 0)
        const unsigned long long m = bits & 0xFFFFFFFFFFFFFull;
        if (var[i] > 0.0 && d >= 0 && d <= 14 && !(d & 1) && (m >> (shift + width)) == prefix)
          atomicAdd(&s_hist[(m >> shift) & ((1u << width) - 1u)], 1u);
      }
      __syncthreads();
      uint32_t above_d = 0;
      const int digit = select_bucket(s_hist, 1 << width, need, s_rev, s_scan, &s_pick, &s_above, &s_count,
                                      &above_d, &here);
      need -= above_d;
      prefix = (prefix << width) | (unsigned long long)digit;
      done += width;
      if (here == 1u && done < 52) {   // a single key has these leading bits: it is K
        for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
          const unsigned long long bits = (unsigned long long)__double_as_longlong(var[i]);
          const int d = (int)(bits >> 52) - E;
          const unsigned long long m = bits & 0xFFFFFFFFFFFFFull;
          if (var[i] > 0.0 && d >= 0 && d <= 14 && !(d & 1) && (m >> shift) == prefix) s_mant = m;
        }
        __syncthreads();
        prefix = s_mant;
        done = 52;
      }
    }
    lo = ((unsigned long long)E << 52) | prefix;
    hi = lo + 1ull;
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
  for (int k = threadIdx.x; k < g.S; k += blockDim.x) {
    s_slab[k] = 0;
    s_nzslab[k] = 0;
  }
  __syncthreads();
  int ks = beg / g.HW, in_slab = beg - ks * g.HW;   // slab of bin i, walked incrementally
  uint32_t slab_sum = 0, slab_nz = 0, my_nz = 0;
  for (int i = beg; i < end; ++i) {
    const double x = var[i];
    int b = 0;
    if (!raw && x > 0.0) {
      if (!select) {
        b = uniform ? g.bits : 8;
      } else {
        b = key_count(x, v_hi);
        if (key_count(x, v_lo) > b) {
          if (rank < need) b += 1;
          rank += 1;
        }
      }
    }
    pay[kHeaderBytes + i] = (unsigned char)b;
    const float sg = (float)sqrt(x);
    if (!head_gains_on(g.flags)) reinterpret_cast<float*>(pay + g.off_sigma)[i] = sg;   // (else: per head, written)
    reinterpret_cast<uint2*>(var)[i] = make_uint2(__float_as_uint(sg), (uint32_t)b);   // for the records
    code_bits_local += b;
    slab_sum += b;
    slab_nz += b > 0;
    my_nz += b > 0;
    if (++in_slab == g.HW || i + 1 == end) {
      if (slab_sum) atomicAdd(&s_slab[ks], slab_sum);
      if (slab_nz) atomicAdd(&s_nzslab[ks], slab_nz);
      slab_sum = 0;
      slab_nz = 0;
      in_slab = 0;
      ++ks;
    }
  }
  // zero padding after the b[] and sigma[] arrays
  for (int i = kHeaderBytes + g.N + threadIdx.x; i < g.off_sigma; i += blockDim.x) pay[i] = 0;
  for (int i = g.off_sigma + 4 * g.N * gain_vectors(g.flags, g.heads) + threadIdx.x; i < g.off_codes; i += blockDim.x)
    pay[i] = 0;
  const long long code_bits = raw ? 32LL * g.N : block_sum<long long>(code_bits_local, s_ll);
  const long long cstride = pad16((code_bits + 7) / 8);
  // slab offsets P(k_s) and record offsets NZ(k_s)
  __syncthreads();
  if (threadIdx.x < 32) slab_scan(s_slab, g.S, s_P);
  else if (threadIdx.x < 64) slab_scan(s_nzslab, g.S, s_NZ);
  __syncthreads();
  uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  uint32_t* NZ = P + g.S + 2;
  for (int k = threadIdx.x; k <= g.S; k += blockDim.x) {
    P[k] = raw ? 0u : s_P[k];
    NZ[k] = raw ? 0u : s_NZ[k];
  }
  // the records of the bins with bits, in bin order: {bin, bits, P_i, 1/sigma_i}
  if (!raw) {
    s_cnt[threadIdx.x] = my_nz;
    __syncthreads();
    block_exclusive_scan(s_cnt, blockDim.x, s_scan);
    uint32_t slot = s_cnt[threadIdx.x];
    __syncthreads();
    s_cnt[threadIdx.x] = (uint32_t)code_bits_local;
    __syncthreads();
    block_exclusive_scan(s_cnt, blockDim.x, s_scan);
    uint32_t pos = s_cnt[threadIdx.x];
    uint4* urecs = recs + (size_t)u * g.N;
    for (int i = beg; i < end; ++i) {
      const uint2 sb = reinterpret_cast<const uint2*>(var)[i];   // {sigma_i, b_i} of this thread's bins
      const uint32_t b = sb.y;
      if (b) {
        urecs[slot++] = make_uint4((uint32_t)i, b, pos, __float_as_uint(__frcp_rn(__uint_as_float(sb.x))));
        pos += b;
      }
    }
  }
  if (threadIdx.x == 0) {
    uint32_t* h32 = reinterpret_cast<uint32_t*>(pay);
    int32_t* i32 = reinterpret_cast<int32_t*>(pay);
    h32[0] = kMagic;
    h32[1] = (uint32_t)kVersion | ((uint32_t)(g.flags & kPayloadFlags) << 16);
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

// ----------------------------------------------------------------------------- decode index ---
constexpr int kDecodeIndexThreads = 1024;   // a warp per slab (S <= 64): two slabs per warp at most

// One CTA per unit: the header must describe exactly the unit the caller asked for, every bit
// width must be <= 8 and their sum must equal the header's code_bits; then P(k_s), NZ(k_s) and the
// decoding records are rebuilt from the payload (one warp per slab, a scan gives every bin's stream
// position).  Decoding records are dense, one per (slab, row pair, column), so that the inverse
// kernel's warp for a row pair reads its two rows' bins in order: sigma and position << 8 | code
// mask for each of the two rows.  The 32 chunk CTAs that decode a bin do no index arithmetic of
// their own.
__global__ void __launch_bounds__(kDecodeIndexThreads) decode_index_kernel(const __grid_constant__ Geom g,
                                                           const __grid_constant__ UnitList ul,
                                                           uint32_t* __restrict__ index, uint4* __restrict__ recs,
                                                           unsigned int* status) {
  __shared__ int s_ok;    // header check: written by thread 0 before the first barrier, then only read
  __shared__ int s_bad;   // allocation check: set by any thread, read after the next barriers
  __shared__ uint32_t s_slab[kMaxSlabs];
  __shared__ uint32_t s_nzslab[kMaxSlabs];
  __shared__ uint32_t s_P[kMaxSlabs + 1];
  __shared__ uint32_t s_NZ[kMaxSlabs + 1];
  const int u = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const UnitDev& ud = ul.u[u];
  const unsigned char* pay = ud.payload;
  const bool raw = g.flags & TACTKV_NO_QUANT;
  if (threadIdx.x == 0) {
    const uint32_t* h32 = reinterpret_cast<const uint32_t*>(pay);
    const int32_t* i32 = reinterpret_cast<const int32_t*>(pay);
    const uint32_t ver_flags = h32[1], cb = h32[10], cs = h32[11];
    const unsigned long long total = *reinterpret_cast<const unsigned long long*>(pay + 48);
    bool ok = h32[0] == kMagic && (ver_flags & 0xffffu) == (uint32_t)kVersion &&
              (ver_flags >> 16) == ((uint32_t)g.flags & kPayloadFlags) && i32[2] == ud.layer &&
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
  __syncthreads();
  // Every thread takes the same branch below: s_ok is not written again, and the allocation check
  // reports through s_bad, which is read only after the barriers that follow every write to it.
  const bool header_ok = s_ok;
  bool ok = header_ok;
  const unsigned char* b = pay + kHeaderBytes;
  if (header_ok && !raw) {
    bool bad = false;
    for (int k = warp; k < g.S; k += nwarps) {
      uint32_t sum = 0, nz = 0;
      for (int i = lane; i < g.HW; i += 32) {
        const uint32_t v = b[(size_t)k * g.HW + i];
        bad |= v > 8;
        sum += v;
        nz += v > 0;
      }
      sum = __reduce_add_sync(0xffffffffu, sum);
      nz = __reduce_add_sync(0xffffffffu, nz);
      if (lane == 0) {
        s_slab[k] = sum;
        s_nzslab[k] = nz;
      }
    }
    if (bad) s_bad = 1;
    __syncthreads();
    if (warp == 0) slab_scan(s_slab, g.S, s_P);
    else if (warp == 1) slab_scan(s_nzslab, g.S, s_NZ);
    __syncthreads();
    if (threadIdx.x == 0 && s_P[g.S] != reinterpret_cast<const uint32_t*>(pay)[10]) s_bad = 1;
    __syncthreads();
    ok = s_bad == 0;
  }
  uint32_t* P = index + (size_t)u * unit_index_words(g.S);
  uint32_t* NZ = P + g.S + 2;
  for (int k = threadIdx.x; k <= g.S; k += blockDim.x) {
    P[k] = (ok && !raw) ? s_P[k] : 0u;
    NZ[k] = (ok && !raw) ? s_NZ[k] : 0u;
  }
  if (threadIdx.x == 0) {
    P[g.S + 1] = ok ? 1u : 0u;
    if (!ok) set_status(status, TACTKV_CORRUPT_PAYLOAD);
  }
  if (ok && !raw) {
    // dense decoding records, one per (slab, row pair kp, column t) at ks*HP*W + kp*W + t:
    // {sigma of row 2kp, sigma of row 2kp+1, shift << 26 | offset << 8 | code mask of each row}, the
    // offset (18 bits) of a code counted from the first bit of its slab's first stream word (P(k_s)
    // rounded down to 32), the shift (6 bits) counted from the first bit of the stream word that
    // holds the row's first code (the decoder's 64-bit window when the row's codes fit in it);
    // a bin without bits (and the padding row of an odd H) has sigma 0, mask 0 and an offset
    // inside its slab's span, so that the decoder may read its (empty) code like any other
    const float* sig = reinterpret_cast<const float*>(pay + g.off_sigma);
    const int HP = (g.H + 1) >> 1, RP = HP * g.W;
    uint32_t* urec32 = reinterpret_cast<uint32_t*>(recs + (size_t)u * g.N);
    for (int k = warp; k < g.S; k += nwarps) {
      uint32_t pos = s_P[k];
      const uint32_t wbase = pos & ~31u;   // first bit of the slab's first stream word
      for (int i0 = 0; i0 < g.HW; i0 += 32) {
        const int j = i0 + lane, i = k * g.HW + j;
        const uint32_t v = j < g.HW ? b[i] : 0u;
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (j < g.HW) {
          const int kh = j / g.W, t = j - kh * g.W;
          uint32_t* rec = urec32 + ((size_t)k * RP + (size_t)(kh >> 1) * g.W + t) * 4;
          rec[kh & 1] = v ? __float_as_uint(sig[i]) : 0u;
          rec[2 + (kh & 1)] = ((pos + incl - v - wbase) << 8) | ((1u << v) - 1u);
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (g.H & 1)   // the padding row H of the last row pair: no bits, at the slab's first bit
        for (int t = lane; t < g.W; t += 32) {
          uint32_t* rec = urec32 + ((size_t)k * RP + (size_t)(HP - 1) * g.W + t) * 4;
          rec[1] = 0u;
          rec[3] = (s_P[k] - wbase) << 8;
        }
      // the shifts: columns t > 0 from their row's first code (column 0, not yet changed), then
      // column 0 itself
      __syncwarp();
      for (int e = lane; e < RP; e += 32) {
        const int kp = e / g.W;
        if (e == kp * g.W) continue;
        uint32_t* rec = urec32 + ((size_t)k * RP + e) * 4;
        const uint32_t* first = urec32 + ((size_t)k * RP + (size_t)kp * g.W) * 4;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint32_t y = rec[2 + r], base = (first[2 + r] >> 8) & 0x3ffe0u;
          rec[2 + r] = y | (((((y >> 8) & 0x3ffffu) - base) & 63u) << 26);
        }
      }
      __syncwarp();
      for (int kp = lane; kp < HP; kp += 32) {
        uint32_t* rec = urec32 + ((size_t)k * RP + (size_t)kp * g.W) * 4;
#pragma unroll
        for (int r = 0; r < 2; ++r) rec[2 + r] |= ((rec[2 + r] >> 8) & 31u) << 26;
      }
    }
  }
}

}  // namespace

cudaError_t launch_decode_index(const Geom& g, const UnitList& ul, int nu, uint32_t* index, uint4* recs,
                                unsigned int* status, cudaStream_t st) {
  decode_index_kernel<<<nu, kDecodeIndexThreads, 0, st>>>(g, ul, index, recs, status);
  return cudaGetLastError();
}

cudaError_t launch_allocate_from_var(const Geom& g, const UnitList& ul, int nu, double* var, uint32_t* index,
                                     uint4* recs, cudaStream_t st) {
  const size_t var_bytes = (size_t)g.N * sizeof(double);
  const bool in_smem = var_bytes <= kAllocSmemVar;
  if (in_smem) cudaFuncSetAttribute(allocate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)var_bytes);
  allocate_kernel<<<nu, kAllocThreads, in_smem ? var_bytes : 0, st>>>(g, ul, var, in_smem, index, recs);
  return cudaGetLastError();
}

cudaError_t launch_allocate(const Geom& g, const UnitList& ul, int nu, const float* partial, double* var,
                            uint32_t* index, uint4* recs, cudaStream_t st) {
  reduce_var_kernel<<<dim3((g.N + 255) / 256, nu), 256, 0, st>>>(g, ul, partial, var);
  return launch_allocate_from_var(g, ul, nu, var, index, recs, st);
}

}  // namespace tactkv
