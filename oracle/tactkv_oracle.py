"""TACT-KV CPU oracle: plain, slow, obviously-correct fp64 NumPy restatement of the codec.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of the
benchmark may import this module.  It shares no code with the CUDA library (no kernels,
headers, tables or constant generators); the two meet only on the seeded inputs produced by
``dct_transform_coding_b200.workloads`` and on the documented payload format.

What it computes, step by step, following the TACT-KV summary page ("TACT-KV: Tri-Axis Cosine
Transform for Compressing Volumetric KV Caches in Medical VLMs", ai.info), section
"Methodology in Plain English", stages 1-4 and the decoding paragraph after them:

1. Reshape (stage 1): one layer's visual K (or V) of one sequence is viewed as an (S, H, W)
   token grid times n = heads * head_dim channels; token t = (s*H + h)*W + w.
2. Transform (stage 2): orthonormal separable 3D DCT-II along S, H and W, per channel; the
   feature axis is not transformed.  Frequency bin i = (k_s*H + k_h)*W + k_w.
3. Bit allocation (stage 3): per-bin variance sigma_i^2 = mean over the n channels of X[i,c]^2
   (estimated afresh for every layer of every sequence, "Key Contributions" item 3); reverse
   water-filling b_i = max(0, 1/2 log2(sigma_i^2 / theta)), theta by bisection, b_i rounded to
   integers, a +-1 greedy correction to hit the budget, cap 8 bits, b_i = 0 drops the bin.
4. Quantize (stage 4): gain-shape -- each bin is scaled by its own sigma_i and every coordinate
   is looked up in a fixed Lloyd-Max table for a unit Gaussian at the bin's bit width.
5. Decode (paragraph after stage 4): reverse the steps -- unpack, dequantize, inverse 3D DCT.

Readings taken where the pages are silent (each is listed in the design notes):
* sigma_i^2 is a second moment (no mean removal) pooled over all heads x head_dim channels;
  the stored gain is sigma_i = float32(sqrt(sigma_i^2)).
* The nominal budget is B = bits * N "bit slots per channel", so sum_i b_i * n = bits * N * n.
* If 8 * (#bins with sigma^2 > 0) <= B every such bin gets 8 bits and the total stays below B.
* Rounding is nearest with halves up, floor(r + 1/2); the greedy removes the cheapest last bit
  (least sigma_i^2 * 4^-(b_i-1), ties to the highest index) or adds the most valuable next bit
  (greatest sigma_i^2 * 4^-b_i, ties to the lowest index) one step at a time.
* A code is the number of thresholds t_j <= u with u = X / sigma_i; the decision is taken in
  float32 (the precision of the CUDA kernels), ties go to the upper cell, outer cells saturate.
* The fixed shared rotation of the shape vector named in stage 4 is optional (FLAG_ROTATE, off by
  default, as in the codec's specification).  Reading of the fixed, shared orthogonal rotation: the
  same orthogonal matrix R for every bin, layer and sequence, block-diagonal over groups of 32
  consecutive channels, R_g = (1/sqrt(32)) H_32 D_g with H_32 the Sylvester-Hadamard matrix and D_g
  a diagonal of signs drawn once from a counter-based SplitMix64 (see ``rotation_signs``).  It
  acts on each bin's vector of n coefficients after the gain is measured (R is orthogonal, so the
  gain is unchanged) and is undone after dequantization.
* Ablation variants ("Main Findings": fewer transformed axes, uniform allocation), also flags:
  FLAG_SKIP_S / _H / _W leave that axis untransformed (all three: no DCT); FLAG_UNIFORM gives every
  bin with sigma^2 > 0 the nominal bits (b_i = bits) instead of water-filling.
* Per-head gains (FLAG_HEAD_GAIN, off by default).  Stage 4 counts Sum(b_i * d + 32) bits with d
  the head dimension of the pages' models ("Main Findings" quotes absmax-to-std "at d=256"), which
  reads as one gain-shape vector, with its own 32-bit gain, per (bin, head).  With the flag, bin i
  of head h is scaled by g[h, i] = float32(sqrt(mean over the head's head_dim channels of
  X[i, c]^2)) and dequantized with it; a zero gain scales by 0 (every coordinate is then 0).  The
  bit allocation still uses the pooled sigma_i^2 of all channels, so b_i is shared by the heads.
* Payload layout: see ``FORMAT`` below (the pages fix only its size, stage 4:
  sum_i (b_i * d + 32) bits plus a small index).
"""
from __future__ import annotations

import math
import struct
from typing import Dict, Tuple

import numpy as np
from scipy.special import erfc, ndtri

# --------------------------------------------------------------------------------------------
# Payload format (version 1).  Little-endian throughout.
#
#   [0, 64)                     header, see HEADER_FMT
#   [64, 64 + pad16(N))         uint8  b[N]        bits of each frequency bin (0..8)
#   [off_sigma, +pad16(4N))     float32 sigma[N]   stored gain of each bin
#                               (FLAG_HEAD_GAIN: float32 sigma[heads][N], pad16(4 * heads * N))
#   [off_codes, ...)            n channel streams, channel c at off_codes + c * chan_stride
#       quantized:   stream bit P_i + k holds bit k (LSB first) of bin i's code, with
#                    P_i = sum_{j<i} b_j; stream bit q is bit (q & 7) of byte (q >> 3);
#                    chan_stride = pad16(ceil(sum_i b_i / 8))
#       NO_QUANT:    float32 X[i, c] for i = 0..N-1, chan_stride = pad16(4N)
# --------------------------------------------------------------------------------------------
MAGIC = 0x31564B54          # bytes 'T','K','V','1'
VERSION = 1
FLAG_NO_QUANT = 1
FLAG_SKIP_S = 4             # no DCT along S (ablation)
FLAG_SKIP_H = 8             # no DCT along H
FLAG_SKIP_W = 16            # no DCT along W
FLAG_UNIFORM = 32           # uniform allocation: b_i = bits for every bin with sigma^2 > 0
FLAG_ROTATE = 64            # fixed shared rotation of each bin's shape vector before quantization
FLAG_HEAD_GAIN = 128        # one gain per (bin, head) instead of one per bin
PAYLOAD_FLAGS = (FLAG_NO_QUANT | FLAG_SKIP_S | FLAG_SKIP_H | FLAG_SKIP_W | FLAG_UNIFORM | FLAG_ROTATE |
                 FLAG_HEAD_GAIN)
HEADER_FMT = "<IHHiiiiiiiiIIQII"   # magic ver flags layer kv S H W heads head_dim bits codebits stride total r0 r1
HEADER_BYTES = 64
assert struct.calcsize(HEADER_FMT) == HEADER_BYTES

MAX_BITS = 8


def _pad16(x: int) -> int:
    return (x + 15) // 16 * 16


# ------------------------------------------------------------------------------------- DCT ---
def dct_matrix(L: int) -> np.ndarray:
    """Orthonormal DCT-II matrix: C[k, t] = a_k cos(pi (2t+1) k / (2L)), a_0 = sqrt(1/L), a_k = sqrt(2/L).

    Stage 2 of the methodology: a separable 3D DCT-II whose basis is orthonormal, so the transform
    alone loses nothing.
    """
    k = np.arange(L, dtype=np.float64)[:, None]
    t = np.arange(L, dtype=np.float64)[None, :]
    C = np.cos(np.pi * (2.0 * t + 1.0) * k / (2.0 * L))
    C *= np.where(k == 0, math.sqrt(1.0 / L), math.sqrt(2.0 / L))
    return C


def dct3(x: np.ndarray, axes=(True, True, True)) -> np.ndarray:
    """Forward separable 3D DCT-II of x[S, H, W, n] along the first three axes (fp64); an axis whose
    entry in `axes` is False is left untransformed (the ablations with fewer axes)."""
    S, H, W, _ = x.shape
    y = x
    if axes[0]:
        y = np.einsum("ks,shwc->khwc", dct_matrix(S), y)
    if axes[1]:
        y = np.einsum("kh,shwc->skwc", dct_matrix(H), y)
    if axes[2]:
        y = np.einsum("kw,shwc->shkc", dct_matrix(W), y)
    return y


def idct3(X: np.ndarray, axes=(True, True, True)) -> np.ndarray:
    """Inverse of dct3: the transpose (DCT-III) along each transformed axis."""
    S, H, W, _ = X.shape
    y = X
    if axes[0]:
        y = np.einsum("ks,khwc->shwc", dct_matrix(S), y)
    if axes[1]:
        y = np.einsum("kh,skwc->shwc", dct_matrix(H), y)
    if axes[2]:
        y = np.einsum("kw,shkc->shwc", dct_matrix(W), y)
    return y


def axes_of(flags: int):
    return (not flags & FLAG_SKIP_S, not flags & FLAG_SKIP_H, not flags & FLAG_SKIP_W)


# ----------------------------------------------------------------- shared shape rotation ---
ROTATION_SEED = 0x544143544B56     # "TACTKV"
ROTATION_GROUP = 32


def splitmix64(seed: int, i: int) -> int:
    """Output i (0, 1, ...) of the SplitMix64 generator (Steele, Lea and Flood, "Fast splittable
    pseudorandom number generators", OOPSLA 2014) started from `seed`: state = seed + (i+1) gamma,
    gamma = 0x9E3779B97F4A7C15, then the variant-13 finalizer of MurmurHash3."""
    m = (1 << 64) - 1
    z = (seed + (i + 1) * 0x9E3779B97F4A7C15) & m
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
    return z ^ (z >> 31)


def rotation_signs(n: int) -> np.ndarray:
    """Sign of channel c: -1 when the top bit of SplitMix64 output c (seed ROTATION_SEED) is set."""
    return np.array([-1.0 if splitmix64(ROTATION_SEED, c) >> 63 else 1.0 for c in range(n)])


def hadamard(m: int) -> np.ndarray:
    """Sylvester-Hadamard matrix of order m (a power of two): H[i, j] = (-1)^popcount(i & j)."""
    i = np.arange(m)[:, None]
    j = np.arange(m)[None, :]
    pop = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(pop % 2 == 1, -1.0, 1.0)


def rotation_matrix(n: int) -> np.ndarray:
    """The fixed shared rotation R (n x n, orthogonal): block-diagonal over groups of 32 channels,
    block g = H_32 diag(signs of its channels) / sqrt(32).  A bin's shape vector v becomes R v."""
    if n % ROTATION_GROUP:
        raise ValueError("the rotation acts on whole groups of 32 channels")
    Hm = hadamard(ROTATION_GROUP) / math.sqrt(ROTATION_GROUP)
    sg = rotation_signs(n)
    R = np.zeros((n, n))
    for g0 in range(0, n, ROTATION_GROUP):
        R[g0:g0 + ROTATION_GROUP, g0:g0 + ROTATION_GROUP] = Hm * sg[None, g0:g0 + ROTATION_GROUP]
    return R


# -------------------------------------------------------------------------- bin variances ---
def bin_variances(X: np.ndarray) -> np.ndarray:
    """sigma_i^2 = (1/n) sum_c X[i, c]^2 for every frequency bin (X given as [N, n] or [S,H,W,n])."""
    Xf = X.reshape(-1, X.shape[-1])
    return np.mean(Xf * Xf, axis=1)


def stored_sigma(var: np.ndarray) -> np.ndarray:
    """The gain written to the payload: float32(sqrt(sigma^2))."""
    return np.sqrt(var).astype(np.float32)


# ------------------------------------------------------------------------- allocation -------
def waterfill_rate(var: np.ndarray, log2_theta: float) -> np.ndarray:
    """Continuous reverse water-filling rates r_i = clamp(1/2 log2(sigma_i^2 / theta), 0, 8)."""
    out = np.zeros_like(var)
    act = var > 0
    out[act] = np.clip(0.5 * (np.log2(var[act]) - log2_theta), 0.0, MAX_BITS)
    return out


def water_level(var: np.ndarray, B: float) -> float:
    """log2(theta) with sum_i clamp(1/2 log2(sigma_i^2 / theta), 0, 8) = B, found by bisection
    until the interval stops shrinking (needs 0 < B < 8 * #active bins).  The total rate is
    non-increasing in theta: it is 8 * #active at the lower end and 0 at the upper end."""
    act = var > 0
    lo = math.log2(var[act].min()) - 2 * MAX_BITS - 1
    hi = math.log2(var.max())
    while True:
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            return hi
        if waterfill_rate(var, mid).sum() > B:
            lo = mid
        else:
            hi = mid


def allocate_bits(var: np.ndarray, bits: int) -> np.ndarray:
    """Integer bits per bin by reverse water-filling with bisection and a +-1 greedy fix.

    Stage 3 of the methodology ("Methodology in Plain English" on the TACT-KV summary page): the
    water level theta comes from a bisection, the continuous rates are rounded, and single-bit
    greedy steps then bring the total exactly to the budget B = bits * N; no bin takes more than
    8 bits.
    """
    var = np.asarray(var, dtype=np.float64)
    N = var.size
    B = int(bits) * N
    act = var > 0
    n_act = int(np.count_nonzero(act))
    b = np.zeros(N, dtype=np.int64)
    if n_act == 0:
        return b
    if MAX_BITS * n_act <= B:                       # every active bin saturates: stay within budget
        b[act] = MAX_BITS
        return b
    r = waterfill_rate(var, water_level(var, B))
    b = np.clip(np.floor(r + 0.5), 0, MAX_BITS).astype(np.int64)
    b[~act] = 0
    idx = np.arange(N)
    while b.sum() > B:                              # drop the least valuable last bit
        cand = b > 0
        key = np.where(cand, var * np.power(4.0, -(b - 1).astype(np.float64)), np.inf)
        m = key.min()
        i = idx[key == m].max()                     # ties -> highest index
        b[i] -= 1
    while b.sum() < B:                              # add the most valuable next bit
        cand = act & (b < MAX_BITS)
        key = np.where(cand, var * np.power(4.0, -b.astype(np.float64)), -np.inf)
        m = key.max()
        i = idx[key == m].min()                     # ties -> lowest index
        b[i] += 1
    return b


def allocate_uniform(var: np.ndarray, bits: int) -> np.ndarray:
    """The uniform-allocation ablation ("Main Findings"): every bin with sigma^2 > 0 gets the nominal
    bits, every other bin none."""
    var = np.asarray(var, dtype=np.float64)
    return np.where(var > 0, int(bits), 0).astype(np.int64)


def allocate_bits_topk(var: np.ndarray, bits: int) -> np.ndarray:
    """Brute force used as a pin: b_i = number of bin i's keys sigma_i^2 4^-k (k = 0..7) among the
    B largest of all 8N keys (ties to the lower bin index), all active bins saturated if they fit."""
    var = np.asarray(var, dtype=np.float64)
    N = var.size
    B = int(bits) * N
    act = var > 0
    if MAX_BITS * int(act.sum()) <= B:
        return np.where(act, MAX_BITS, 0).astype(np.int64)
    keys = []
    for i in range(N):
        if var[i] > 0:
            for k in range(MAX_BITS):
                keys.append((-var[i] * 4.0 ** (-k), i, k))
    keys.sort()
    b = np.zeros(N, dtype=np.int64)
    for _, i, _ in keys[:B]:
        b[i] += 1
    return b


# ------------------------------------------------------------------------- Lloyd-Max --------
_SQ2 = math.sqrt(2.0)
_SQ2PI = math.sqrt(2.0 * math.pi)


def _upper_tail(x):
    return 0.5 * erfc(np.asarray(x, dtype=np.float64) / _SQ2)


def _pdf(x):
    x = np.asarray(x, dtype=np.float64)
    return np.exp(-0.5 * x * x) / _SQ2PI


def _centroids(levels: np.ndarray):
    """Centroid of every cell of the nearest-neighbour partition defined by `levels` (N(0,1))."""
    t = 0.5 * (levels[1:] + levels[:-1])
    a = np.concatenate([[-np.inf], t])
    b = np.concatenate([t, [np.inf]])
    # P(a < Z < b), taken from the tail on the cell's own side so no 1 - (1 - eps) cancellation
    mass = np.where(b <= 0, _upper_tail(-b) - _upper_tail(-a), _upper_tail(a) - _upper_tail(b))
    return (_pdf(a) - _pdf(b)) / mass, a, b, mass


def lloyd_max(bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """Lloyd-Max quantizer of a unit Gaussian with 2^bits levels (stage 4: the fixed codebook of
    each bit width): levels are the centroids of their cells and thresholds the midpoints of adjacent
    levels.  Lloyd's alternation is run from a companding start; because it converges slowly for
    many levels, Newton's method on the same two conditions finishes it.  Returns (levels,
    thresholds), increasing."""
    L = 1 << bits
    y = math.sqrt(3.0) * ndtri((np.arange(L) + 0.5) / L)
    for _ in range(200):                                  # Lloyd: midpoint step, centroid step
        y = _centroids(y)[0]
    for _ in range(60):                                   # Newton on F(y) = y - centroid(y)
        c, a, b, mass = _centroids(y)
        F = y - c
        if np.max(np.abs(F)) < 1e-15:
            break
        fa = np.where(np.isfinite(a), a, 0.0)
        fb = np.where(np.isfinite(b), b, 0.0)
        dca = np.where(np.isfinite(a), _pdf(a) * (c - fa) / mass, 0.0)   # d c_j / d a_j
        dcb = np.where(np.isfinite(b), _pdf(b) * (fb - c) / mass, 0.0)   # d c_j / d b_j
        J = np.eye(L)
        for j in range(L):
            if j > 0:            # a_j = (y_{j-1} + y_j) / 2
                J[j, j - 1] -= 0.5 * dca[j]
                J[j, j] -= 0.5 * dca[j]
            if j < L - 1:        # b_j = (y_j + y_{j+1}) / 2
                J[j, j] -= 0.5 * dcb[j]
                J[j, j + 1] -= 0.5 * dcb[j]
        y = y - np.linalg.solve(J, F)
    y = 0.5 * (y - y[::-1])                               # exact odd symmetry
    return y, 0.5 * (y[1:] + y[:-1])


_TABLES: Dict[int, Tuple[np.ndarray, np.ndarray]] = {}


def table(bits: int) -> Tuple[np.ndarray, np.ndarray]:
    if bits not in _TABLES:
        _TABLES[bits] = lloyd_max(bits)
    return _TABLES[bits]


def quantizer_mse(bits: int) -> float:
    """Mean squared error of the Lloyd-Max quantizer for N(0,1) (exact integral, per cell)."""
    y, _ = table(bits)
    c, a, b, mass = _centroids(y)
    # E[(Z - y_j)^2 ; cell j] = E[Z^2 ; cell] - 2 y_j E[Z ; cell] + y_j^2 P(cell)
    az = np.where(np.isfinite(a), np.where(np.isfinite(a), a, 0.0) * _pdf(a), 0.0)
    bz = np.where(np.isfinite(b), np.where(np.isfinite(b), b, 0.0) * _pdf(b), 0.0)
    ez2 = mass + az - bz
    ez = _pdf(a) - _pdf(b)
    return float(np.sum(ez2 - 2 * y * ez + y * y * mass))


def quantize(u: np.ndarray, bits: int) -> np.ndarray:
    """Code = number of thresholds t_j <= u, decided in float32 (ties to the upper cell)."""
    _, t = table(bits)
    return np.searchsorted(t.astype(np.float32), np.asarray(u, dtype=np.float32), side="right")


def dequantize(code: np.ndarray, bits: int) -> np.ndarray:
    y, _ = table(bits)
    return y[code]


# ------------------------------------------------------------------------------ payload -----
def payload_layout(N: int, n: int, code_bits: int, no_quant: bool = False, gains: int = 1) -> Dict[str, int]:
    """Byte offsets of the payload's parts; gains = gain vectors of N floats (heads with
    FLAG_HEAD_GAIN, else 1)."""
    off_sigma = HEADER_BYTES + _pad16(N)
    off_codes = off_sigma + _pad16(4 * N * gains)
    stride = _pad16(4 * N) if no_quant else _pad16((code_bits + 7) // 8)
    return dict(off_b=HEADER_BYTES, off_sigma=off_sigma, off_codes=off_codes, chan_stride=stride,
                total=off_codes + n * stride)


def payload_capacity(S: int, H: int, W: int, heads: int, head_dim: int, bits: int,
                     no_quant: bool = False, flags: int = 0) -> int:
    """Worst-case payload size: sum_i b_i <= bits * N."""
    N = S * H * W
    no_quant = no_quant or bool(flags & FLAG_NO_QUANT)
    return payload_layout(N, heads * head_dim, 32 * N if no_quant else bits * N, no_quant,
                          _gain_vectors(flags, heads))["total"]


def _gain_vectors(flags: int, heads: int) -> int:
    return heads if (flags & FLAG_HEAD_GAIN) and not (flags & FLAG_NO_QUANT) else 1


def head_gains(X: np.ndarray, heads: int, head_dim: int) -> np.ndarray:
    """Per-head gains g[h, i] = float32(sqrt(mean over head h's channels of X[i, c]^2)) (the
    per-head reading of stage 4's gain-shape vectors), as fp64 values of float32 numbers."""
    X = np.asarray(X, dtype=np.float64)
    hv = np.mean(X.reshape(X.shape[0], heads, head_dim) ** 2, axis=2).T     # [heads, N]
    return stored_sigma(hv)


def _pack_streams(codes: np.ndarray, b: np.ndarray, stride: int) -> np.ndarray:
    """codes[N, n] (bin-major) -> n channel streams of stride bytes, bit layout as in FORMAT."""
    N, n = codes.shape
    P = np.concatenate([[0], np.cumsum(b)])
    out = np.zeros((n, stride), dtype=np.uint8)
    for i in range(N):
        for k in range(int(b[i])):
            q = int(P[i]) + k
            bit = ((codes[i] >> k) & 1).astype(np.uint8)
            out[:, q >> 3] |= (bit << (q & 7)).astype(np.uint8)
    return out


def _unpack_streams(streams: np.ndarray, b: np.ndarray) -> np.ndarray:
    n = streams.shape[0]
    N = b.size
    P = np.concatenate([[0], np.cumsum(b)])
    codes = np.zeros((N, n), dtype=np.int64)
    for i in range(N):
        for k in range(int(b[i])):
            q = int(P[i]) + k
            codes[i] |= ((streams[:, q >> 3] >> (q & 7)) & 1).astype(np.int64) << k
    return codes


def compress_unit(x, S: int, H: int, W: int, heads: int, head_dim: int, bits: int,
                  layer: int = 0, kv: int = 0, no_quant: bool = False,
                  return_info: bool = False, flags: int = 0):
    """Compress one visual K or V, x[S*H*W, heads, head_dim] (any real dtype), to payload bytes.
    flags: FLAG_SKIP_* (axes left untransformed), FLAG_UNIFORM, FLAG_ROTATE, FLAG_HEAD_GAIN (see
    the head)."""
    n = heads * head_dim
    N = S * H * W
    if not 1 <= bits <= MAX_BITS:
        raise ValueError("bits must be 1..8")
    flags = (int(flags) | (FLAG_NO_QUANT if no_quant else 0)) & PAYLOAD_FLAGS
    no_quant = bool(flags & FLAG_NO_QUANT)
    xv = np.asarray(x, dtype=np.float64).reshape(S, H, W, n)
    X = dct3(xv, axes_of(flags)).reshape(N, n)
    var = bin_variances(X)
    sig = stored_sigma(var)
    Xq = X @ rotation_matrix(n).T if (flags & FLAG_ROTATE) and not no_quant else X   # row i: R X_i
    if no_quant:
        b = np.zeros(N, dtype=np.int64)
        lay = payload_layout(N, n, 32 * N, True)
        body = np.zeros((n, lay["chan_stride"]), dtype=np.uint8)
        body[:, :4 * N] = np.ascontiguousarray(X.T.astype("<f4")).view(np.uint8)
        code_bits = 32 * N
        codes = None
    else:
        b = allocate_uniform(var, bits) if flags & FLAG_UNIFORM else allocate_bits(var, bits)
        code_bits = int(b.sum())
        if flags & FLAG_HEAD_GAIN:
            sig = head_gains(X, heads, head_dim)                            # [heads, N]
        lay = payload_layout(N, n, code_bits, gains=_gain_vectors(flags, heads))
        codes = np.zeros((N, n), dtype=np.int64)
        for i in np.nonzero(b)[0]:
            # the gain of every channel of bin i: the bin's, or its head's (0 where a head is silent)
            g = np.repeat(sig[:, i], head_dim) if flags & FLAG_HEAD_GAIN else np.full(n, sig[i])
            g = g.astype(np.float64)
            u = np.divide(Xq[i], g, out=np.zeros(n), where=g > 0)
            codes[i] = quantize(u, int(b[i]))
        body = _pack_streams(codes, b, lay["chan_stride"])
    buf = bytearray(lay["total"])
    struct.pack_into(HEADER_FMT, buf, 0, MAGIC, VERSION, flags,
                     layer, kv, S, H, W, heads, head_dim, bits, code_bits, lay["chan_stride"],
                     lay["total"], 0, 0)
    buf[lay["off_b"]:lay["off_b"] + N] = b.astype(np.uint8).tobytes()
    sig_bytes = np.ascontiguousarray(sig, dtype="<f4").tobytes()
    buf[lay["off_sigma"]:lay["off_sigma"] + len(sig_bytes)] = sig_bytes
    buf[lay["off_codes"]:] = body.tobytes()
    if return_info:
        return bytes(buf), dict(X=X, Xq=Xq, var=var, sigma=sig, b=b, codes=codes)
    return bytes(buf)


def parse_payload(payload) -> Dict:
    buf = bytes(payload)
    f = struct.unpack_from(HEADER_FMT, buf, 0)
    (magic, ver, flags, layer, kv, S, H, W, heads, head_dim, bits, code_bits, stride, total,
     _, _) = f
    if magic != MAGIC or ver != VERSION:
        raise ValueError("not a TACT-KV payload")
    N = S * H * W
    n = heads * head_dim
    gains = _gain_vectors(flags, heads)
    lay = payload_layout(N, n, code_bits, bool(flags & FLAG_NO_QUANT), gains)
    if lay["chan_stride"] != stride or lay["total"] != total or len(buf) < total:
        raise ValueError("inconsistent payload header")
    b = np.frombuffer(buf, np.uint8, N, lay["off_b"]).astype(np.int64)
    sig = np.frombuffer(buf, "<f4", N * gains, lay["off_sigma"]).copy()
    if (flags & FLAG_HEAD_GAIN) and not (flags & FLAG_NO_QUANT):
        sig = sig.reshape(gains, N)                     # [heads, N]
    streams = np.frombuffer(buf, np.uint8, n * stride, lay["off_codes"]).reshape(n, stride)
    return dict(flags=flags, layer=layer, kv=kv, S=S, H=H, W=W, heads=heads, head_dim=head_dim,
                bits=bits, code_bits=code_bits, b=b, sigma=sig, streams=streams, N=N, n=n)


def decompress_unit(payload) -> np.ndarray:
    """Reverse of compress_unit: fp64 reconstruction [S*H*W, heads, head_dim] (not yet rounded)."""
    p = parse_payload(payload)
    N, n = p["N"], p["n"]
    if p["flags"] & FLAG_NO_QUANT:
        X = p["streams"][:, :4 * N].copy().view("<f4").astype(np.float64).T
    else:
        b = p["b"]
        if b.max(initial=0) > MAX_BITS or b.sum() > p["bits"] * N:
            raise ValueError("corrupt allocation")
        codes = _unpack_streams(p["streams"], b)
        X = np.zeros((N, n), dtype=np.float64)
        for i in np.nonzero(b)[0]:
            if p["flags"] & FLAG_HEAD_GAIN:
                g = np.repeat(p["sigma"][:, i].astype(np.float64), p["head_dim"])
            else:
                g = np.float64(p["sigma"][i])
            X[i] = g * dequantize(codes[i], int(b[i]))
        if p["flags"] & FLAG_ROTATE:
            X = X @ rotation_matrix(n)                  # row i: R^T (dequantized R X_i)
    x = idct3(X.reshape(p["S"], p["H"], p["W"], n), axes_of(p["flags"]))
    return x.reshape(N, p["heads"], p["head_dim"])


def attention_decode(q: np.ndarray, payload_k, payload_v):
    """One decode step of attention over a compressed visual K/V (the paragraph after stage 4:
    decoding can run inside the attention kernel, so the reconstructed cache never exists).

    The plain definition on the decompressed cache: for query head j (q[j], of head_dim D) and its
    key/value head j // G (G = query heads per K/V head),
        s_j[t] = q_j . K[t] / sqrt(D),  m_j = max_t s_j[t],  l_j = sum_t exp(s_j[t] - m_j),
        out_j  = sum_t exp(s_j[t] - m_j) V[t] / l_j,
    over the unit's T = S*H*W visual tokens, K and V the fp64 reconstructions of the payloads.
    Returns (out [Hq, D], m [Hq], l [Hq]); m and l let a caller merge these tokens with others."""
    pk, pv = parse_payload(payload_k), parse_payload(payload_v)
    K = decompress_unit(payload_k)            # [T, kv_heads, D]
    V = decompress_unit(payload_v)
    kv_heads, D = pk["heads"], pk["head_dim"]
    assert (pv["heads"], pv["head_dim"]) == (kv_heads, D)
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    G = Hq // kv_heads
    out = np.zeros((Hq, D))
    m = np.zeros(Hq)
    l = np.zeros(Hq)
    for j in range(Hq):
        h = j // G
        sc = K[:, h, :] @ q[j] / math.sqrt(D)
        m[j] = sc.max()
        e = np.exp(sc - m[j])
        l[j] = e.sum()
        out[j] = e @ V[:, h, :] / l[j]
    return out, m, l


def codes_of(payload) -> Tuple[np.ndarray, np.ndarray]:
    """(b[N], codes[N, n]) decoded from a payload (for code-level parity checks)."""
    p = parse_payload(payload)
    return p["b"], _unpack_streams(p["streams"], p["b"])


def occupancy_bits(b: np.ndarray, d: int, vectors: int = 1) -> int:
    """Stage 4's occupancy of one compressed layer: sum over the gain-shape vectors of
    (b_i * d + 32) bits, d the channels that share a gain and 32 bits for the gain.  By default a
    bin is one vector of all n = heads * head_dim channels (d = n); with per-head gains each bin
    holds `vectors` = heads vectors of d = head_dim channels."""
    b = np.asarray(b, dtype=np.int64)
    return int(vectors) * int(np.sum(b * int(d) + 32))


def index_bits(N: int) -> int:
    """The small index on top of the occupancy: one byte (the bit width) per bin."""
    return 8 * int(N)


def max_batch(hbm_bytes: int, fixed_bytes: int, per_request_bytes: int) -> int:
    """Requests whose caches fit in what is left of the device memory after the shared part."""
    if per_request_bytes <= 0:
        return -1
    return max(0, (int(hbm_bytes) - int(fixed_bytes)) // int(per_request_bytes))


def threshold_distance(u: np.ndarray, bits: int) -> np.ndarray:
    """Distance of u to the nearest decision threshold t_j of the b-bit codebook, each distance
    taken relative to max(1, |t_j|) (fp64).  This is the band of the code-parity rule: a code may
    differ from the oracle's only where this distance is at most 1e-5 (the middle threshold 0 of
    an even codebook gets the absolute distance)."""
    thresholds_b = table(bits)[1]
    gaps = np.abs(np.asarray(u, dtype=np.float64)[..., None] - thresholds_b)
    return np.min(gaps / np.maximum(1.0, np.abs(thresholds_b)), axis=-1)


def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bfloat16 (8 significant bits, round half to even) directly, no
    intermediate float32 rounding, and return them as fp64 (normal range only)."""
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
