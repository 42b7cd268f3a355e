// TACT-KV codec C ABI (host side): argument checks, grouping of units into waves, launches.
//
// A compress wave (up to kMaxUnits units of identical shape) runs five kernels on the caller's
// stream: the forward DCT along S (axis_s.cu), the forward DCT along H and W, which writes the
// finished coefficients back into the workspace volume and sums the per-bin energies (axis_hw.cu),
// the variance reduction and the per-unit allocation with the payload header, slab offsets and
// the records of the bins with bits (allocate.cu), and the quantization and packing of those bins
// (pack.cu).  A decompress
// wave runs the decoding index (allocate.cu: header checks, slab offsets), the inverse H/W pass
// (dequantize + inverse DCT along W and H) and the inverse DCT along S.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "lloyd_max_tables.inc"

namespace tactkv {

cudaError_t launch_axis_s_16(bool, const Geom&, const UnitList&, int, float*, cudaStream_t);
cudaError_t launch_axis_s_32(bool, const Geom&, const UnitList&, int, float*, cudaStream_t);
cudaError_t launch_axis_s_64(bool, const Geom&, const UnitList&, int, float*, cudaStream_t);
#define TACTKV_DECL_HW(h, w)                                                                                 \
  cudaError_t launch_axis_hw_##h##_##w(bool, int, const Geom&, const UnitList&, int, float*, float*, const uint32_t*, \
                                       const uint4*, int, cudaStream_t);                                              \
  void axis_hw_shape_##h##_##w(const Geom&, bool, int, size_t*, int*);
TACTKV_DECL_HW(16, 16)
TACTKV_DECL_HW(16, 32)
TACTKV_DECL_HW(32, 16)
TACTKV_DECL_HW(32, 32)
#undef TACTKV_DECL_HW

cudaError_t launch_axis_s(int cls, bool inverse, const Geom& g, const UnitList& ul, int nu, float* buf,
                          cudaStream_t st) {
  if (cls == 16) return launch_axis_s_16(inverse, g, ul, nu, buf, st);
  if (cls == 32) return launch_axis_s_32(inverse, g, ul, nu, buf, st);
  return launch_axis_s_64(inverse, g, ul, nu, buf, st);
}

#define TACTKV_DECL_FUSED(s) \
  cudaError_t launch_fused_##s(const Geom&, const UnitList&, int, float*, float*, unsigned int*, cudaStream_t);
TACTKV_DECL_FUSED(8)
TACTKV_DECL_FUSED(16)
TACTKV_DECL_FUSED(32)
TACTKV_DECL_FUSED(64)
#undef TACTKV_DECL_FUSED
#define TACTKV_DECL_FUSED_INV(s)                                                                            \
  cudaError_t launch_fused_inv_##s(const Geom&, const UnitList&, int, float*, const uint32_t*, const uint4*, \
                                   unsigned int*, cudaStream_t);
TACTKV_DECL_FUSED_INV(16)
TACTKV_DECL_FUSED_INV(32)
TACTKV_DECL_FUSED_INV(64)
#undef TACTKV_DECL_FUSED_INV

// Decode and all three inverse DCTs in one launch (quantized payloads on the fused grids with S =
// 16, 32 or 64); cudaErrorNotSupported where the separate inverse kernels must run instead.
cudaError_t launch_fused_inv(const Geom& g, const UnitList& ul, int nu, float* big, const uint32_t* index,
                             const uint4* recs, unsigned int* status, cudaStream_t st) {
  switch (g.S) {
    case 16: return launch_fused_inv_16(g, ul, nu, big, index, recs, status, st);
    case 32: return launch_fused_inv_32(g, ul, nu, big, index, recs, status, st);
    case 64: return launch_fused_inv_64(g, ul, nu, big, index, recs, status, st);
    default: return cudaErrorNotSupported;
  }
}

// Grids with a fused three-axis forward kernel (one launch for the S and H/W passes, the volume
// kept in L2 between them).
bool fused_grid(const Geom& g) {
  const bool s = g.S == 8 || g.S == 16 || g.S == 32 || g.S == 64;
  return s && ((g.H == 16 && g.W == 16) || (g.H == 14 && g.W == 14) || (g.H == 8 && g.W == 8) ||
               (g.H == 24 && g.W == 24 && g.S <= 32));
}
cudaError_t launch_fused(const Geom& g, const UnitList& ul, int nu, float* buf, float* partial, unsigned int* status,
                         cudaStream_t st) {
  switch (g.S) {
    case 8: return launch_fused_8(g, ul, nu, buf, partial, status, st);
    case 16: return launch_fused_16(g, ul, nu, buf, partial, status, st);
    case 32: return launch_fused_32(g, ul, nu, buf, partial, status, st);
    case 64: return launch_fused_64(g, ul, nu, buf, partial, status, st);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_axis_hw(int hcls, int wcls, bool inverse, int mode, const Geom& g, const UnitList& ul, int nu,
                           float* buf, float* partial, const uint32_t* index, const uint4* recs, int spc,
                           cudaStream_t st) {
  if (hcls == 16 && wcls == 16) return launch_axis_hw_16_16(inverse, mode, g, ul, nu, buf, partial, index, recs, spc, st);
  if (hcls == 16) return launch_axis_hw_16_32(inverse, mode, g, ul, nu, buf, partial, index, recs, spc, st);
  if (wcls == 16) return launch_axis_hw_32_16(inverse, mode, g, ul, nu, buf, partial, index, recs, spc, st);
  return launch_axis_hw_32_32(inverse, mode, g, ul, nu, buf, partial, index, recs, spc, st);
}

void axis_hw_shape(int hcls, int wcls, const Geom& g, bool inverse, int mode, size_t* smem, int* threads) {
  if (hcls == 16 && wcls == 16) return axis_hw_shape_16_16(g, inverse, mode, smem, threads);
  if (hcls == 16) return axis_hw_shape_16_32(g, inverse, mode, smem, threads);
  if (wcls == 16) return axis_hw_shape_32_16(g, inverse, mode, smem, threads);
  return axis_hw_shape_32_32(g, inverse, mode, smem, threads);
}

size_t attention_scores_smem(const Geom& g, int q_heads);
size_t attention_values_smem(const Geom& g, int q_heads);
size_t attention_softmax_smem(const Geom& g);
cudaError_t launch_attention(const Geom& g, const UnitList& kl, const UnitList& vl, int nu, int q_heads,
                             const uint32_t* kidx, const uint4* krec, const uint32_t* vidx, const uint4* vrec,
                             const float* q, float* zp, float* part, float* out, float* m, float* l,
                             cudaStream_t st);

bool tc_s_pass_enabled() {
  static const bool on = [] {
    const char* e = getenv("TACTKV_TC_S");
    return e && e[0] == '1';
  }();
  return on;
}

bool fused_decode_enabled() {
  static const bool on = [] {
    const char* e = getenv("TACTKV_FUSED_DECODE");
    return e && e[0] == '1';
  }();
  return on;
}

namespace {

tactkv_status make_geom(const tactkv_unit& u, Geom& g) {
  if (u.bits < 1 || u.bits > 8) return TACTKV_INVALID_ARG;
  if (u.flags & ~kAllFlags) return TACTKV_INVALID_ARG;
  if (u.S < 1 || u.H < 1 || u.W < 1 || u.heads < 1 || u.head_dim < 1) return TACTKV_INVALID_ARG;
  if (!supported_length(u.S) || !supported_length(u.H) || !supported_length(u.W)) return TACTKV_UNSUPPORTED_SHAPE;
  if (u.H > 32 || u.W > 32 || u.H * u.W > kMaxHW) return TACTKV_UNSUPPORTED_SHAPE;
  const long long n = (long long)u.heads * u.head_dim;
  if (n % kChunk != 0 || u.head_dim % 2 != 0 || n > (1 << 16)) return TACTKV_UNSUPPORTED_SHAPE;
  // per-head gains: every 32-channel chunk lies inside one head
  if (head_gains_on((int)u.flags) && u.head_dim % kChunk != 0) return TACTKV_UNSUPPORTED_SHAPE;
  const long long N = (long long)u.S * u.H * u.W;
  g.S = u.S;
  g.H = u.H;
  g.W = u.W;
  g.HW = u.H * u.W;
  g.T = (int)N;
  g.heads = u.heads;
  g.head_dim = u.head_dim;
  g.n = (int)n;
  g.nch = (int)(n / kChunk);
  g.N = (int)N;
  g.bits = u.bits;
  g.flags = (int)u.flags;
  g.off_sigma = (int)(kHeaderBytes + pad16(g.N));
  g.off_codes = (int)(g.off_sigma + pad16(4LL * g.N * gain_vectors(g.flags, g.heads)));
  g.capacity = 0;
  g.unit0 = 0;
  return TACTKV_OK;
}

size_t payload_bytes_geom(const Geom& g) {
  const long long bits_per_chan = (g.flags & TACTKV_NO_QUANT) ? 32LL * g.N : (long long)g.bits * g.N;
  return (size_t)(g.off_codes + (long long)g.n * pad16((bits_per_chan + 7) / 8));
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// workspace of one unit: the transformed volume (fp32; Y and then X when compressing, V when
// decompressing), per-chunk energy sums, fp64 variances, the index block (P, ok, NZ) and the
// records of the bins with bits
size_t unit_ws_bytes(const Geom& g) {
  return round256((size_t)g.T * g.n * 4) + round256((size_t)g.nch * g.N * 4) + round256((size_t)g.N * 8) +
         round256((size_t)unit_index_words(g.S) * 4) + round256((size_t)g.N * 16);
}

struct WsView {
  unsigned int* status;
  float* big;         // nu * T * n floats: Y/X (compress) or V (decompress)
  float* partial;     // nu * nch * N floats
  double* var;        // nu * N doubles
  uint32_t* index;    // nu * unit_index_words(S) words
  uint4* recs;        // nu * N records
};

WsView view(unsigned char* ws, const Geom& g, int nu) {
  WsView v;
  v.status = reinterpret_cast<unsigned int*>(ws);
  size_t off = kStatusBytes;
  v.big = reinterpret_cast<float*>(ws + off);
  off += round256((size_t)nu * g.T * g.n * 4);
  v.partial = reinterpret_cast<float*>(ws + off);
  off += round256((size_t)nu * g.nch * g.N * 4);
  v.var = reinterpret_cast<double*>(ws + off);
  off += round256((size_t)nu * g.N * 8);
  v.index = reinterpret_cast<uint32_t*>(ws + off);
  off += round256((size_t)nu * unit_index_words(g.S) * 4);
  v.recs = reinterpret_cast<uint4*>(ws + off);
  return v;
}

// Slabs per CTA of the slab-walking kernels: whole units when the batch alone fills the GPU a
// couple of times over, shorter slab ranges (more CTAs) for small batches.
int slabs_per_cta_for(const Geom& g, int nu, size_t smem, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int by_smem = (int)((228 * 1024) / (smem + 1024));
  const int by_threads = 2048 / threads;
  const int occ = std::max(1, std::min(by_smem, by_threads));
  const long long target = 2LL * sms * occ;
  const long long have = (long long)g.nch * nu;
  const int ranges = (int)std::min<long long>(g.S, std::max<long long>(1, (target + have - 1) / have));
  return (g.S + ranges - 1) / ranges;
}
int slabs_per_cta(const Geom& g, int nu, bool inverse, int mode) {
  size_t smem = 0;
  int threads = 32;
  axis_hw_shape(length_class(g.H), length_class(g.W), g, inverse, mode, &smem, &threads);
  return slabs_per_cta_for(g, nu, smem, threads);
}

bool same_group(const tactkv_unit& a, const tactkv_unit& b) {
  return a.S == b.S && a.H == b.H && a.W == b.W && a.heads == b.heads && a.head_dim == b.head_dim &&
         a.bits == b.bits && a.flags == b.flags;
}

tactkv_status check_unit(const tactkv_unit& u, const Geom& g, bool compress) {
  const size_t elem = (u.flags & TACTKV_FP32_IO) ? 4 : 2;
  const void* io = compress ? u.kv_in : static_cast<const void*>(u.kv_out);
  if (!io || !u.payload) return TACTKV_INVALID_ARG;
  if (u.token_stride <= 0 || u.head_stride < 0) return TACTKV_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(io) % (2 * elem)) || (u.token_stride % 2) || (u.head_stride % 2))
    return TACTKV_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(u.payload) % 16) return TACTKV_ALIGNMENT;
  if (u.payload_capacity < payload_bytes_geom(g)) return TACTKV_CAPACITY;
  return TACTKV_OK;
}

thread_local int t_launches = 0;    // kernels launched by this thread's current or last call

template <class F>
tactkv_status for_each_wave(const tactkv_unit* units, int n_units, void* ws, size_t ws_bytes, bool compress,
                            F&& fn) {
  if (n_units < 0 || (n_units > 0 && !units)) return TACTKV_INVALID_ARG;
  if (n_units == 0) return TACTKV_OK;
  if (!ws || ws_bytes < kStatusBytes || reinterpret_cast<uintptr_t>(ws) % 256) return TACTKV_WORKSPACE;
  int i = 0;
  while (i < n_units) {
    int j = i + 1;
    while (j < n_units && same_group(units[i], units[j])) ++j;
    Geom g;
    tactkv_status st = make_geom(units[i], g);
    if (st != TACTKV_OK) return st;
    long long cap = -1;
    for (int k = i; k < j; ++k) {
      st = check_unit(units[k], g, compress);
      if (st != TACTKV_OK) return st;
      cap = cap < 0 ? (long long)units[k].payload_capacity : std::min(cap, (long long)units[k].payload_capacity);
    }
    g.capacity = cap;
    const size_t per = unit_ws_bytes(g);
    const int wave = (int)std::min<size_t>(kMaxUnits, (ws_bytes - kStatusBytes) / per);
    if (wave < 1) return TACTKV_WORKSPACE;
    for (int k = i; k < j; k += wave) {
      const int nu = std::min(wave, j - k);
      UnitList ul;
      memset(&ul, 0, sizeof(ul));
      for (int q = 0; q < nu; ++q) {
        const tactkv_unit& s = units[k + q];
        ul.u[q].in = s.kv_in;
        ul.u[q].out = s.kv_out;
        ul.u[q].payload = static_cast<unsigned char*>(s.payload);
        ul.u[q].tok_stride = s.token_stride;
        ul.u[q].head_stride = s.head_stride;
        ul.u[q].layer = s.layer;
        ul.u[q].kv = s.kv;
      }
      st = fn(g, ul, nu, static_cast<unsigned char*>(ws));
      if (st != TACTKV_OK) return st;
    }
    i = j;
  }
  return TACTKV_OK;
}

}  // namespace

// ------------------------------------------------------------- allocation-free compress scratch ---
// Scratch of tactkv_compress_noalloc: a fixed array in the library's device image, so the call
// needs no allocation from its caller.  Every device that loads the library holds it until exit.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the symbol names a
// host-side stand-in, not device memory, so the address is looked up once per device (with that
// device current) and cached.
cudaError_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}
}  // namespace
}  // namespace tactkv

using namespace tactkv;

extern "C" {

size_t tactkv_payload_bytes(const tactkv_unit* unit) {
  if (!unit) return 0;
  Geom g;
  if (make_geom(*unit, g) != TACTKV_OK) return 0;
  return payload_bytes_geom(g);
}

size_t tactkv_workspace_bytes(const tactkv_unit* units, int n_units) {
  size_t best = 0;
  int i = 0;
  while (units && i < n_units) {
    int j = i + 1;
    while (j < n_units && same_group(units[i], units[j])) ++j;
    Geom g;
    if (make_geom(units[i], g) == TACTKV_OK)
      best = std::max(best, (size_t)std::min(kMaxUnits, j - i) * unit_ws_bytes(g));
    i = j;
  }
  return kStatusBytes + best;
}

static tactkv_status compress_impl(const tactkv_unit* units, int n_units, void* workspace, size_t workspace_bytes,
                                   cudaStream_t st, void* const* events) {
  auto mark = [&](int k) {
    if (events && events[k]) cudaEventRecord(static_cast<cudaEvent_t>(events[k]), st);
  };
  t_launches = 0;
  return for_each_wave(units, n_units, workspace, workspace_bytes, true,
                       [&](const Geom& g, const UnitList& ul, int nu, unsigned char* ws) -> tactkv_status {
                         const WsView w = view(ws, g, nu);
                         const int cs = length_class(g.S), ch = length_class(g.H), cw = length_class(g.W);
                         mark(0);
                         if (fused_grid(g)) {
                           t_launches += 1;   // fdct3
                           if (launch_fused(g, ul, nu, w.big, w.partial, w.status, st) != cudaSuccess)
                             return TACTKV_CUDA;
                         } else {
                           t_launches += 2;   // fdct_s, fdct_hw
                           if (launch_axis_s(cs, false, g, ul, nu, w.big, st) != cudaSuccess) return TACTKV_CUDA;
                           if (launch_axis_hw(ch, cw, false, kStats, g, ul, nu, w.big, w.partial, w.index, nullptr,
                                              slabs_per_cta(g, nu, false, kStats), st) != cudaSuccess)
                             return TACTKV_CUDA;
                         }
                         mark(1);
                         t_launches += 3;   // reduce_var, allocate, pack
                         if (launch_allocate(g, ul, nu, w.partial, w.var, w.index, w.recs, st) != cudaSuccess)
                           return TACTKV_CUDA;
                         mark(2);
                         if (launch_pack(g, ul, nu, w.big, w.recs, w.index, st) != cudaSuccess)
                           return TACTKV_CUDA;
                         mark(3);
                         return TACTKV_OK;
                       });
}

static tactkv_status decompress_impl(const tactkv_unit* units, int n_units, void* workspace, size_t workspace_bytes,
                                     cudaStream_t st, void* const* events) {
  auto mark = [&](int k) {
    if (events && events[k]) cudaEventRecord(static_cast<cudaEvent_t>(events[k]), st);
  };
  t_launches = 0;
  return for_each_wave(units, n_units, workspace, workspace_bytes, false,
                       [&](const Geom& g, const UnitList& ul, int nu, unsigned char* ws) -> tactkv_status {
                         const WsView w = view(ws, g, nu);
                         const int cs = length_class(g.S), ch = length_class(g.H), cw = length_class(g.W);
                         const int mode = (g.flags & TACTKV_NO_QUANT) ? kRaw : kQuant;
                         mark(0);
                         t_launches += 1;   // decode_index
                         if (launch_decode_index(g, ul, nu, w.index, w.recs, w.status, st) != cudaSuccess)
                           return TACTKV_CUDA;
                         mark(1);
                         const cudaError_t fe = fused_grid(g) ? launch_fused_inv(g, ul, nu, w.big, w.index, w.recs,
                                                                                 w.status, st)
                                                              : cudaErrorNotSupported;
                         if (fe == cudaSuccess) {
                           t_launches += 1;   // idct3 (decode, inverse H/W, inverse S)
                           mark(2);
                         } else if (fe == cudaErrorNotSupported) {
                           t_launches += 2;   // idct_hw, idct_s
                           if (launch_axis_hw(ch, cw, true, mode, g, ul, nu, w.big, nullptr, w.index, w.recs,
                                              slabs_per_cta(g, nu, true, mode), st) != cudaSuccess)
                             return TACTKV_CUDA;
                           mark(2);
                           if (launch_axis_s(cs, true, g, ul, nu, w.big, st) != cudaSuccess) return TACTKV_CUDA;
                         } else {
                           return TACTKV_CUDA;
                         }
                         mark(3);
                         return TACTKV_OK;
                       });
}

tactkv_status tactkv_compress(const tactkv_unit* units, int n_units, void* workspace, size_t workspace_bytes,
                              struct CUstream_st* stream) {
  return compress_impl(units, n_units, workspace, workspace_bytes, stream, nullptr);
}

tactkv_status tactkv_decompress(const tactkv_unit* units, int n_units, void* workspace, size_t workspace_bytes,
                                struct CUstream_st* stream) {
  return decompress_impl(units, n_units, workspace, workspace_bytes, stream, nullptr);
}

tactkv_status tactkv_compress_profiled(const tactkv_unit* units, int n_units, void* workspace,
                                       size_t workspace_bytes, struct CUstream_st* stream, void* const* events) {
  return compress_impl(units, n_units, workspace, workspace_bytes, stream, events);
}

tactkv_status tactkv_decompress_profiled(const tactkv_unit* units, int n_units, void* workspace,
                                         size_t workspace_bytes, struct CUstream_st* stream, void* const* events) {
  return decompress_impl(units, n_units, workspace, workspace_bytes, stream, events);
}

tactkv_status tactkv_compress_noalloc(const tactkv_unit* units, int n_units, struct CUstream_st* stream) {
  if (n_units < 0 || (n_units > 0 && !units)) return TACTKV_INVALID_ARG;
  if (n_units == 0) return TACTKV_OK;
  for (int i = 0; i < n_units; ++i) {   // every unit must fit the fixed scratch on its own
    Geom g;
    const tactkv_status st = make_geom(units[i], g);
    if (st != TACTKV_OK) return st;
    if (kStatusBytes + unit_ws_bytes(g) > kNoAllocScratchBytes) return TACTKV_SCRATCH_LIMIT;
  }
  void* ws = nullptr;
  if (noalloc_scratch(&ws) != cudaSuccess) return TACTKV_CUDA;
  // the scratch keeps the previous call's contents: the status word is the part that must start at 0
  if (cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return TACTKV_CUDA;
  return compress_impl(units, n_units, ws, kNoAllocScratchBytes, stream, nullptr);
}

tactkv_status tactkv_allocate(const tactkv_unit* unit, const double* var, void* workspace, size_t workspace_bytes,
                              struct CUstream_st* stream) {
  t_launches = 0;
  if (!unit || !var || !unit->payload) return TACTKV_INVALID_ARG;
  Geom g;
  tactkv_status st = make_geom(*unit, g);
  if (st != TACTKV_OK) return st;
  if (head_gains_on(g.flags)) return TACTKV_INVALID_ARG;   // per-head gains need the channels, not variances
  if (reinterpret_cast<uintptr_t>(unit->payload) % 16 || reinterpret_cast<uintptr_t>(var) % 8) return TACTKV_ALIGNMENT;
  if (unit->payload_capacity < payload_bytes_geom(g)) return TACTKV_CAPACITY;
  g.capacity = (long long)unit->payload_capacity;
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < kStatusBytes + unit_ws_bytes(g))
    return TACTKV_WORKSPACE;
  UnitList ul;
  memset(&ul, 0, sizeof(ul));
  ul.u[0].in = unit->kv_in;
  ul.u[0].out = unit->kv_out;
  ul.u[0].payload = static_cast<unsigned char*>(unit->payload);
  ul.u[0].tok_stride = unit->token_stride;
  ul.u[0].head_stride = unit->head_stride;
  ul.u[0].layer = unit->layer;
  ul.u[0].kv = unit->kv;
  const WsView w = view(static_cast<unsigned char*>(workspace), g, 1);
  if (cudaMemcpyAsync(w.var, var, sizeof(double) * g.N, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return TACTKV_CUDA;
  t_launches = 1;
  if (launch_allocate_from_var(g, ul, 1, w.var, w.index, w.recs, stream) != cudaSuccess) return TACTKV_CUDA;
  return TACTKV_OK;
}

// ------------------------------------------------------------------ decode-time attention ---
namespace {
constexpr int kAttnMaxUnits = kMaxUnits / 2;   // K and V index blocks of one call share one launch

struct AttnWs {
  unsigned int* status;
  uint32_t* index;   // 2 nu index blocks: K units, then V units
  uint4* recs;       // 2 nu * N dense records
  float* zp;         // nu * q_heads * N: z, then dct3(p)
  float* part;       // nu * S * q_heads * head_dim
  size_t total;
};
AttnWs attn_view(unsigned char* ws, const Geom& g, int nu, int q_heads) {
  AttnWs a;
  size_t off = kStatusBytes;
  a.status = reinterpret_cast<unsigned int*>(ws);
  a.index = reinterpret_cast<uint32_t*>(ws + off);
  off += round256((size_t)2 * nu * unit_index_words(g.S) * 4);
  a.recs = reinterpret_cast<uint4*>(ws + off);
  off += round256((size_t)2 * nu * g.N * 16);
  a.zp = reinterpret_cast<float*>(ws + off);
  off += round256((size_t)nu * q_heads * g.N * 4);
  a.part = reinterpret_cast<float*>(ws + off);
  off += round256((size_t)nu * g.S * q_heads * g.head_dim * 4);
  a.total = off;
  return a;
}
tactkv_status attn_check(const tactkv_unit* k_units, const tactkv_unit* v_units, int n_units, int q_heads,
                         Geom& g) {
  if (n_units < 1 || n_units > kAttnMaxUnits || !k_units || !v_units) return TACTKV_INVALID_ARG;
  tactkv_status st = make_geom(k_units[0], g);
  if (st != TACTKV_OK) return st;
  if ((g.flags & TACTKV_NO_QUANT) || q_heads < g.heads || q_heads % g.heads || q_heads / g.heads > 16 ||
      g.head_dim % kChunk)
    return TACTKV_UNSUPPORTED_SHAPE;
  if (attention_softmax_smem(g) > 227 * 1024 || attention_scores_smem(g, q_heads) > 227 * 1024 ||
      attention_values_smem(g, q_heads) > 227 * 1024)
    return TACTKV_UNSUPPORTED_SHAPE;
  long long cap = -1;
  for (int i = 0; i < n_units; ++i)
    for (const tactkv_unit* u : {&k_units[i], &v_units[i]}) {
      if (!same_group(k_units[0], *u)) return TACTKV_INVALID_ARG;
      if (!u->payload) return TACTKV_INVALID_ARG;
      if (reinterpret_cast<uintptr_t>(u->payload) % 16) return TACTKV_ALIGNMENT;
      if (u->payload_capacity < payload_bytes_geom(g)) return TACTKV_CAPACITY;
      cap = cap < 0 ? (long long)u->payload_capacity : std::min(cap, (long long)u->payload_capacity);
    }
  g.capacity = cap;
  return TACTKV_OK;
}
}  // namespace

size_t tactkv_attention_workspace_bytes(const tactkv_unit* k_units, int n_units, int q_heads) {
  Geom g;
  if (!k_units || n_units < 1 || make_geom(k_units[0], g) != TACTKV_OK || q_heads < 1) return 0;
  return attn_view(nullptr, g, n_units, q_heads).total;
}

tactkv_status tactkv_attention_decode(const tactkv_unit* k_units, const tactkv_unit* v_units, int n_units,
                                      int q_heads, const float* q, float* out, float* m, float* l,
                                      void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
  t_launches = 0;
  Geom g;
  tactkv_status st = attn_check(k_units, v_units, n_units, q_heads, g);
  if (st != TACTKV_OK) return st;
  if (!q || !out || !m || !l) return TACTKV_INVALID_ARG;
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256) return TACTKV_WORKSPACE;
  const AttnWs a = attn_view(static_cast<unsigned char*>(workspace), g, n_units, q_heads);
  if (workspace_bytes < a.total) return TACTKV_WORKSPACE;
  UnitList both, kl, vl;
  memset(&both, 0, sizeof(both));
  memset(&kl, 0, sizeof(kl));
  memset(&vl, 0, sizeof(vl));
  for (int i = 0; i < n_units; ++i) {
    for (int side = 0; side < 2; ++side) {
      const tactkv_unit& s = side ? v_units[i] : k_units[i];
      UnitDev d;
      memset(&d, 0, sizeof(d));
      d.payload = static_cast<unsigned char*>(s.payload);
      d.layer = s.layer;
      d.kv = s.kv;
      both.u[side * n_units + i] = d;
      (side ? vl : kl).u[i] = d;
    }
  }
  t_launches = 5;   // decode_index (K and V), scores, softmax, values, reduce
  if (launch_decode_index(g, both, 2 * n_units, a.index, a.recs, a.status, stream) != cudaSuccess) return TACTKV_CUDA;
  const size_t iw = unit_index_words(g.S);
  if (launch_attention(g, kl, vl, n_units, q_heads, a.index, a.recs, a.index + n_units * iw,
                       a.recs + (size_t)n_units * g.N, q, a.zp, a.part, out, m, l, stream) != cudaSuccess)
    return TACTKV_CUDA;
  return TACTKV_OK;
}

tactkv_status tactkv_device_status(void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
  if (!workspace || workspace_bytes < kStatusBytes) return TACTKV_WORKSPACE;
  unsigned int v = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TACTKV_CUDA;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TACTKV_CUDA;
  if (cudaMemset(workspace, 0, sizeof(v)) != cudaSuccess) return TACTKV_CUDA;
  return static_cast<tactkv_status>(v);
}

const char* tactkv_status_string(tactkv_status s) {
  switch (s) {
    case TACTKV_OK: return "ok";
    case TACTKV_INVALID_ARG: return "invalid argument";
    case TACTKV_UNSUPPORTED_SHAPE: return "unsupported shape";
    case TACTKV_CAPACITY: return "payload capacity too small";
    case TACTKV_ALIGNMENT: return "misaligned pointer or stride";
    case TACTKV_CORRUPT_PAYLOAD: return "corrupt payload";
    case TACTKV_CUDA: return "CUDA error";
    case TACTKV_WORKSPACE: return "workspace missing or too small";
    case TACTKV_SCRATCH_LIMIT: return "unit larger than the fixed scratch of tactkv_compress_noalloc";
    case TACTKV_TIMEOUT: return "a kernel's bounded wait for a copy or a tensor-core operation expired";
    default: return "unknown status";
  }
}

int tactkv_lloyd_max_table(int bits, double* levels, double* thresholds) {
  if (bits < 1 || bits > 8) return 0;
  const int L = 1 << bits;
  if (levels) memcpy(levels, kLmLevels + lm_lv_offset(bits), sizeof(double) * L);
  if (thresholds) memcpy(thresholds, kLmThresholds + lm_thr_offset(bits), sizeof(double) * (L - 1));
  return L;
}

tactkv_status tactkv_occupancy(const void* payload, size_t bytes, tactkv_occupancy_t* out) {
  if (!payload || !out || bytes < (size_t)kHeaderBytes) return TACTKV_INVALID_ARG;
  const unsigned char* p = static_cast<const unsigned char*>(payload);
  uint32_t h32[16];
  memcpy(h32, p, sizeof(h32));
  int32_t i32[16];
  memcpy(i32, p, sizeof(i32));
  if (h32[0] != kMagic || (h32[1] & 0xffffu) != (uint32_t)kVersion) return TACTKV_CORRUPT_PAYLOAD;
  const long long S = i32[4], H = i32[5], W = i32[6], heads = i32[7], head_dim = i32[8];
  if (S < 1 || H < 1 || W < 1 || heads < 1 || head_dim < 1) return TACTKV_CORRUPT_PAYLOAD;
  const unsigned long long N = (unsigned long long)(S * H * W), n = (unsigned long long)(heads * head_dim);
  if (bytes < (size_t)kHeaderBytes + N) return TACTKV_INVALID_ARG;
  const bool raw = (h32[1] >> 16) & TACTKV_NO_QUANT;
  unsigned long long code_bits = 0;
  for (unsigned long long i = 0; i < N; ++i) {
    const unsigned b = p[kHeaderBytes + i];
    if (b > 8) return TACTKV_CORRUPT_PAYLOAD;
    code_bits += b;
  }
  if (raw) code_bits = 32ull * N;
  if (code_bits != h32[10]) return TACTKV_CORRUPT_PAYLOAD;
  unsigned long long total = 0;
  memcpy(&total, p + 48, sizeof(total));
  out->bins = N;
  out->channels = n;
  out->code_bits = code_bits;
  // one 32-bit gain per gain-shape vector: per bin, or per (bin, head) with per-head gains
  out->formula_bits = code_bits * n + 32ull * N * (unsigned long long)gain_vectors((int)(h32[1] >> 16), (int)heads);
  out->index_bits = 8ull * N;
  out->payload_bytes = total;
  out->bits_per_element = 8.0 * (double)total / ((double)N * (double)n);
  out->shrink_vs_bf16 = total ? 2.0 * (double)N * (double)n / (double)total : 0.0;
  return TACTKV_OK;
}

int64_t tactkv_max_batch(uint64_t hbm_bytes, uint64_t fixed_bytes, uint64_t per_request_bytes) {
  if (per_request_bytes == 0) return -1;
  if (fixed_bytes >= hbm_bytes) return 0;
  return (int64_t)((hbm_bytes - fixed_bytes) / per_request_bytes);
}

int tactkv_last_launches(void) { return t_launches; }

int tactkv_format_version(void) { return kVersion; }

}  // extern "C"
