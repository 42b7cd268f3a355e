/*
 * tactkv.h -- C ABI of the B200 TACT-KV visual-KV transform codec.
 *
 * The operations are those of the TACT-KV summary page ("TACT-KV: Tri-Axis Cosine Transform for
 * Compressing Volumetric KV Caches in Medical VLMs"), section "Methodology in Plain English":
 *   stage 1  the visual K or V of one layer of one sequence is laid out on its (S, H, W) grid;
 *   stage 2  a separable orthonormal 3D DCT-II runs along S, H and W (features untouched);
 *   stage 3  per-bin variances (over all heads x head_dim channels) drive a reverse
 *            water-filling split of the layer's bit budget: b_i = max(0, 1/2 log2(s_i^2/theta)),
 *            theta by bisection, integer rounding, +-1 greedy fix to hit the budget, cap 8 bits;
 *   stage 4  each surviving bin is scaled by its own gain s_i and every coordinate is quantized
 *            with a fixed Lloyd-Max table of a unit Gaussian at the bin's bit width;
 *   decoding reverses the stages (paragraph after stage 4).
 *
 * Terms.  A UNIT is one (sequence, layer, K|V) volume: T = S*H*W tokens by n = heads*head_dim
 * channels.  Token t = (s*H + h)*W + w; channel c = head*head_dim + d.  Frequency bin
 * i = (k_s*H + k_h)*W + k_w, N = T bins.  Nominal budget: bits*N bit slots per channel.
 *
 * Memory.  Every pointer in a unit descriptor and the workspace are DEVICE pointers owned by
 * the caller.  The library allocates nothing.  Its only state is the read-only tables in the CUDA
 * module (constant memory, and 16-byte-aligned copies in global memory that kernels stage into
 * shared memory) and the fixed device scratch array of tactkv_compress_noalloc (below); every other entry
 * point is safe to call from several host threads on different streams provided each call has
 * its own workspace.  Calls are asynchronous on `stream`; a status other than
 * TACTKV_OK means nothing was launched for the failing group of units (earlier groups of the
 * same call may already be queued).  Errors found by the kernels (a corrupt payload) are
 * recorded in the workspace and read back with tactkv_device_status().
 *
 * Payload format (version 1, little-endian), one self-describing blob per unit:
 *   [0, 64)             header: u32 magic 0x31564B54 ("TKV1"), u16 version = 1, u16 flags (the
 *                       unit's flags without TACTKV_FP32_IO),
 *                       i32 layer, kv, S, H, W, heads, head_dim, bits, u32 code_bits (sum b_i,
 *                       or 32*N with TACTKV_NO_QUANT), u32 chan_stride (bytes), u64 total_bytes,
 *                       u32 0, u32 0
 *   [64, +pad16(N))     u8 b[N]          bits of every bin (0..8; 0 = dropped)
 *   then pad16(4N)      f32 sigma[N]     gain of every bin, float32(sqrt(sigma^2)); with
 *                       TACTKV_HEAD_GAIN pad16(4*heads*N) bytes, f32 sigma[heads][N]
 *   then n streams      channel c at offset off_codes + c*chan_stride, chan_stride =
 *                       pad16(ceil(code_bits/8)); stream bit P_i + k is bit k (LSB first) of bin
 *                       i's code, P_i = sum_{j<i} b_j; stream bit q is bit (q&7) of byte q>>3.
 *                       With TACTKV_NO_QUANT a stream holds the N float32 coefficients instead.
 * pad16(x) rounds x up to a multiple of 16.  The gain/rate part is the pages' sum(b_i*d + 32)
 * bits per layer; the b[] bytes are the index the pages add on top of it.
 */
#ifndef TACTKV_H_
#define TACTKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st*`; NULL is the legacy default stream */

typedef enum {
  TACTKV_OK = 0,
  TACTKV_INVALID_ARG = 1,        /* null pointer, n_units < 0, bits outside 1..8, bad flags */
  TACTKV_UNSUPPORTED_SHAPE = 2,  /* an axis length or channel layout the kernels do not cover */
  TACTKV_CAPACITY = 3,           /* payload_capacity below tactkv_payload_bytes() */
  TACTKV_ALIGNMENT = 4,          /* a pointer or stride breaks the alignment rules below */
  TACTKV_CORRUPT_PAYLOAD = 5,    /* (device status) a payload header or allocation is invalid */
  TACTKV_CUDA = 6,               /* a CUDA launch or copy failed */
  TACTKV_WORKSPACE = 7,          /* workspace null or smaller than one unit needs */
  TACTKV_SCRATCH_LIMIT = 8,      /* a unit needs more scratch than tactkv_compress_noalloc has */
  TACTKV_TIMEOUT = 9             /* (device status) a kernel's bounded wait on a tensor-memory copy
                                    or a tensor-core operation expired; its outputs are undefined */
} tactkv_status;

/* flags */
#define TACTKV_NO_QUANT 1u /* transform only: store float32 coefficients (lossless round trip) */
#define TACTKV_FP32_IO  2u /* K/V are float32 instead of bfloat16 */
/* Variants of the summary page's "Main Findings" ablations and of stage 4's shape rotation, all
   recorded in the payload header (decompress must be given the same flags):
     TACTKV_SKIP_S / _H / _W  no DCT along that axis (2-axis, 1-axis and no-DCT transforms);
     TACTKV_UNIFORM_ALLOC     every bin with a nonzero variance gets the nominal bits (no
                              water-filling; the total stays within the budget);
     TACTKV_ROTATE            the fixed shared orthogonal rotation of each bin's shape vector before
                              scalar quantization, undone after dequantization: block-diagonal over
                              the 32-channel groups, H_32 diag(s) / sqrt(32) with H_32 the
                              Sylvester-Hadamard matrix and s_c = -1 exactly when bit 63 of output c
                              of SplitMix64 seeded with 0x544143544B56 is set (ignored with
                              TACTKV_NO_QUANT).  Gains and allocation are unchanged by it;
     TACTKV_HEAD_GAIN         one gain per (bin, head) instead of one per bin: the gain-shape
                              vectors of stage 4 are a bin's head_dim coordinates in one head
                              (the d of stage 4's occupancy sum), each scaled by
                              float32(sqrt(mean over the head's channels of X^2)) and decoded with
                              it (a zero gain scales by 0).  The bit allocation still uses the
                              variance pooled over all channels.  Needs head_dim a multiple of 32;
                              the payload then holds sigma[heads][N] (ignored with TACTKV_NO_QUANT). */
#define TACTKV_SKIP_S        4u
#define TACTKV_SKIP_H        8u
#define TACTKV_SKIP_W       16u
#define TACTKV_UNIFORM_ALLOC 32u
#define TACTKV_ROTATE       64u
#define TACTKV_HEAD_GAIN   128u

typedef struct {
  int32_t layer;          /* recorded in the header, checked by decompress */
  int32_t kv;             /* 0 = K, 1 = V; recorded and checked like layer */
  int32_t S, H, W;        /* token grid; lengths from the supported set below */
  int32_t heads, head_dim;/* n = heads*head_dim channels, n a multiple of 32, head_dim even */
  int32_t bits;           /* nominal bits per element, 1..8 */
  uint32_t flags;         /* TACTKV_NO_QUANT | TACTKV_FP32_IO | the variant flags above */
  const void* kv_in;      /* compress input: element (t, head, d) at
                             kv_in + t*token_stride + head*head_stride + d (elements) */
  void* kv_out;           /* decompress output, same indexing as kv_in */
  int64_t token_stride;   /* in elements; even, > 0 */
  int64_t head_stride;    /* in elements; even */
  void* payload;          /* compress writes, decompress reads; 16-byte aligned */
  size_t payload_capacity;/* bytes available at payload */
} tactkv_unit;

/* Supported shapes: S in {1..16, 20, 24, 28, 32, 40, 48, 56, 64}; H and W in {1..16, 20, 24, 28,
   32} with H*W <= 1024; heads*head_dim a multiple of 32 and at most 65536.  kv_in / kv_out must
   be 4-byte aligned (8-byte with TACTKV_FP32_IO); strides even.  Other shapes return
   TACTKV_UNSUPPORTED_SHAPE. */

/* Worst-case payload size of one unit (every bin budget used): the capacity to provide. */
size_t tactkv_payload_bytes(const tactkv_unit* unit);

/* Workspace bytes that let compress/decompress process the units in as few waves as possible
   (a wave is up to 256 units of one shape).  Any size of at least tactkv_workspace_bytes(units,
   1) works; the units are then processed in more, smaller waves. */
size_t tactkv_workspace_bytes(const tactkv_unit* units, int n_units);

/* Compress every unit: read kv_in, write the payload.  Units with identical shape, bits and
   flags that are adjacent in the array are batched into one set of launches.  Steps: forward
   DCT along S; forward DCT along H and W with per-bin energy sums; per-unit bit allocation and
   gains; quantization of the finished coefficients and bit packing. */
tactkv_status tactkv_compress(const tactkv_unit* units, int n_units, void* workspace,
                              size_t workspace_bytes, struct CUstream_st* stream);

/* Decompress every unit: read the payload, write kv_out (bfloat16, or float32 with
   TACTKV_FP32_IO) with the descriptor's strides.  The payload header must match the
   descriptor (layer, kv, shape, bits, flags); a mismatch or an invalid allocation is recorded
   as TACTKV_CORRUPT_PAYLOAD in the workspace and that unit's output is zero-filled. */
tactkv_status tactkv_decompress(const tactkv_unit* units, int n_units, void* workspace,
                                size_t workspace_bytes, struct CUstream_st* stream);

/* Profiling variants: the same work as tactkv_compress / tactkv_decompress, and, when `events`
   is not NULL, cudaEventRecord(events[k], stream) at the stage boundaries of every wave (so for
   a call that fits in one wave the events bracket each stage).  events[k] are cudaEvent_t
   handles created by the caller; a NULL entry is skipped.
   compress:   0 before the transforms, 1 after the DCTs along S and along H and W (with the
               energy sums) of every unit, 2 after the allocation, 3 after quantization and
               packing.
   decompress: 0 before the payload index, 1 after it, 2 after the inverse DCT along W and H
               (with the decoding), 3 after the inverse DCT along S (with the single-kernel decode
               2 and 3 mark the same point). */
tactkv_status tactkv_compress_profiled(const tactkv_unit* units, int n_units, void* workspace,
                                       size_t workspace_bytes, struct CUstream_st* stream,
                                       void* const* events);
tactkv_status tactkv_decompress_profiled(const tactkv_unit* units, int n_units, void* workspace,
                                         size_t workspace_bytes, struct CUstream_st* stream,
                                         void* const* events);

/* tactkv_compress without a workspace argument, for callers that cannot allocate device memory
   at the point where they compress: code recording a CUDA graph (a cudaMalloc there fails or
   breaks the capture), engines whose device memory is all handed out by their own pool, and
   latency-critical loops where an allocation could synchronize the device.  The TACT-KV pages
   have no counterpart of this call; it only changes where the scratch lives.
   The scratch is a fixed 16 MiB array inside the library's device image, which every GPU that
   loads the library holds until the process exits.  Each unit on its own must fit in it (its
   workspace, tactkv_workspace_bytes of that one unit, at most 16 MiB: e.g. 8x8x8 x 64 channels or
   64x16x16 x 128 channels, not 64x16x16 x 1024); otherwise TACTKV_SCRATCH_LIMIT is returned and
   nothing is launched.  The first call on a device looks the array's address up
   (cudaGetSymbolAddress), so make that first call before any stream capture.  All calls share
   the one array: calls that may overlap on the GPU (different streams, or several host threads)
   race on it and must be serialized by the caller.  Allocates nothing; output is identical to
   tactkv_compress. */
tactkv_status tactkv_compress_noalloc(const tactkv_unit* units, int n_units,
                                      struct CUstream_st* stream);

/* Stage 3 alone ("Methodology in Plain English", stage 3: reverse water-filling of the bit budget
   bits*N over the bins, cap 8 bits): the allocation compress runs, applied to the variances the
   caller gives instead of the ones compress measures.  var: DEVICE array of N = S*H*W doubles,
   var[i] >= 0 the variance of bin i (8-byte aligned; not modified).  Writes into unit->payload
   exactly what compress writes there from its own variances: the header, b[N] (the selection of
   the B = bits*N largest keys var_i * 4^-k, k = 0..7, ties to the lower bin index, every active bin
   at 8 bits when 8*#active <= B; b = 0 where var = 0), sigma[N] = float32(sqrt(var)) and the zero
   padding; the code area is left unspecified.  Only the unit's shape, bits, flags, layer, kv,
   payload and payload_capacity are read.  TACTKV_HEAD_GAIN is refused (TACTKV_INVALID_ARG): its
   gains come from the channels, which this call does not see.  workspace: at least tactkv_workspace_bytes(unit, 1)
   bytes, 256-byte aligned.  Asynchronous on `stream`; one kernel. */
tactkv_status tactkv_allocate(const tactkv_unit* unit, const double* var, void* workspace,
                              size_t workspace_bytes, struct CUstream_st* stream);

/* One decode step of attention over compressed visual K/V (the paragraph after stage 4: decoding
   runs inside the attention computation and the reconstructed cache never exists).  Unit i of
   k_units / v_units is the K / V payload of one (sequence, layer); all 2*n_units descriptors have
   the same shape, bits and flags (quantized, not TACTKV_NO_QUANT), and each unit's kv field must
   match its payload.  Only the payload pointers and the shape fields are read.
     q_heads   query heads, a multiple G of the K/V heads (G <= 16); query head j reads K/V head j/G;
     q         DEVICE float32 [n_units][q_heads][head_dim], the decode step's queries;
     out       DEVICE float32 [n_units][q_heads][head_dim]:
                 out_j = sum_t softmax_t(q_j . K[t] / sqrt(head_dim)) V[t] over the S*H*W visual tokens;
     m, l      DEVICE float32 [n_units][q_heads]: the scores' maximum and sum_t exp(score - m), so
               that a caller can merge these tokens with its bf16 text tokens.
   Limits: n_units <= 128, head_dim a multiple of 32, and shared memory for one slab's stream words
   of a head (head_dim * ((c*H*W + 31)/32 + 3, rounded up to odd) 4-byte words, c = min(8, 2*bits + 2)
   bits per bin; a slab whose codes span more is decoded from the payload directly) and for the
   score volume (S*H*(W rounded up to odd) floats) within 227 KB each; other shapes return
   TACTKV_UNSUPPORTED_SHAPE (every benchmark grid fits).  workspace: at least
   tactkv_attention_workspace_bytes(k_units, n_units, q_heads) bytes, 256-byte aligned.  A corrupt
   payload is recorded as TACTKV_CORRUPT_PAYLOAD (tactkv_device_status) and contributes no
   tokens of its unit: out = 0, m = -inf and l = 0 for that unit's query heads.  Asynchronous on
   `stream`; 5 kernels. */
size_t tactkv_attention_workspace_bytes(const tactkv_unit* k_units, int n_units, int q_heads);
tactkv_status tactkv_attention_decode(const tactkv_unit* k_units, const tactkv_unit* v_units, int n_units,
                                      int q_heads, const float* q, float* out, float* m, float* l,
                                      void* workspace, size_t workspace_bytes,
                                      struct CUstream_st* stream);

/* Synchronizes `stream`, returns the first error the kernels recorded in `workspace` since the
   previous call (TACTKV_OK if none), and clears it. */
tactkv_status tactkv_device_status(void* workspace, size_t workspace_bytes,
                                   struct CUstream_st* stream);

/* Human-readable status name. */
const char* tactkv_status_string(tactkv_status status);

/* The library's own Lloyd-Max codebook for `bits` (1..8): 2^bits levels and 2^bits - 1
   thresholds, increasing, written to the host arrays given.  Returns the number of levels, or
   0 for bits outside 1..8.  Host-only; needs no GPU. */
int tactkv_lloyd_max_table(int bits, double* levels, double* thresholds);

/* Occupancy of one compressed unit ("Methodology in Plain English", stage 4: a layer's cache takes
   sum_i (b_i * d + 32) bits plus a small index).  The sum runs over the gain-shape vectors: one per
   bin with d = n = heads*head_dim, or, with TACTKV_HEAD_GAIN, one per (bin, head) with
   d = head_dim.  The index is the byte b_i of every bin. */
typedef struct {
  uint64_t bins;            /* N */
  uint64_t channels;        /* n */
  uint64_t code_bits;       /* sum_i b_i, the bits of one channel stream */
  uint64_t formula_bits;    /* sum_i (b_i * n + 32 * gains per bin): codes and gains */
  uint64_t index_bits;      /* 8 * N: the bit widths */
  uint64_t payload_bytes;   /* the payload's actual size (header, padding and alignment included) */
  double bits_per_element;  /* 8 * payload_bytes / (N * n) */
  double shrink_vs_bf16;    /* 2 * N * n / payload_bytes: size of the bf16 volume over the payload */
} tactkv_occupancy_t;

/* Reads a HOST copy of a payload (at least its header and b[] array: 64 + N bytes) and fills
   *out.  Returns TACTKV_OK, TACTKV_INVALID_ARG (null pointers) or TACTKV_CORRUPT_PAYLOAD (bad
   magic or version, a bit width above 8, or a code_bits field that disagrees with b[]).
   Host-only; needs no GPU. */
tactkv_status tactkv_occupancy(const void* payload, size_t bytes, tactkv_occupancy_t* out);

/* Largest number of requests whose caches fit: floor((hbm_bytes - fixed_bytes) / per_request_bytes)
   (0 when fixed_bytes >= hbm_bytes, -1 when per_request_bytes is 0).  fixed_bytes: what every
   request shares (weights, activations, runtime reserve); per_request_bytes: one request's cache,
   e.g. the sum of its units' payload_bytes plus its uncompressed text KV.  Host-only. */
int64_t tactkv_max_batch(uint64_t hbm_bytes, uint64_t fixed_bytes, uint64_t per_request_bytes);

/* Version of the payload format this library writes and reads. */
int tactkv_format_version(void);

/* Number of kernels that the calling host thread's most recent tactkv_compress*,
   tactkv_decompress* call launched, over all its waves (0 after a call that failed before
   launching).  A compress wave launches 4 kernels when its grid has a fused three-axis forward
   transform kernel (H x W = 16 x 16, 14 x 14 or 8 x 8 with S = 8, 16, 32 or 64, 24 x 24 with S = 8, 16
   or 32) and 5 otherwise;
   a decompress wave launches 3. */
int tactkv_last_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* TACTKV_H_ */
