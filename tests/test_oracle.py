"""Pins of the CPU oracle against what the TACT-KV pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed form, a library
routine that computes the same textbook transform, a brute-force search, a printed table, or
an invariant the summary page states (an orthonormal transform that alone loses nothing, an
allocation that meets the budget exactly with at most 8 bits per bin, Theorem 1's 1/gamma).  A dropped term, a wrong sign or index, or a
transposed operand anywhere in the oracle fails at least one of them.
"""
import math
import os
import struct

import numpy as np
import pytest
import scipy.fft

from oracle import tactkv_oracle as O

RNG = np.random.default_rng(20261202)


# ------------------------------------------------------------------------------------ DCT ---
@pytest.mark.parametrize("L", [1, 2, 3, 7, 8, 14, 16, 24, 64])
def test_dct_matrix_orthonormal(L):
    C = O.dct_matrix(L)
    assert np.allclose(C @ C.T, np.eye(L), atol=1e-13, rtol=0)


def test_dct_matrix_closed_form():
    # L = 2: the orthonormal DCT-II is the Haar butterfly [[1, 1], [1, -1]] / sqrt(2)
    assert np.allclose(O.dct_matrix(2), np.array([[1, 1], [1, -1]]) / math.sqrt(2), atol=1e-15)
    # DC row is constant 1/sqrt(L); row 1 of L = 4 is sqrt(1/2) * cos(pi (2t+1) / 8)
    C4 = O.dct_matrix(4)
    assert np.allclose(C4[0], 0.5, atol=1e-15)
    c1, c3 = math.cos(math.pi / 8), math.cos(3 * math.pi / 8)
    assert np.allclose(C4[1], math.sqrt(0.5) * np.array([c1, c3, -c3, -c1]), atol=1e-15)


@pytest.mark.parametrize("shape", [(8, 8, 8, 3), (3, 5, 7, 2), (6, 14, 14, 1), (4, 24, 2, 5), (1, 1, 9, 2)])
def test_dct3_matches_scipy_dctn(shape):
    x = RNG.standard_normal(shape)
    ref = scipy.fft.dctn(x, type=2, norm="ortho", axes=(0, 1, 2))
    assert np.allclose(O.dct3(x), ref, atol=1e-12, rtol=0)
    assert np.allclose(O.idct3(ref), scipy.fft.idctn(ref, type=2, norm="ortho", axes=(0, 1, 2)),
                       atol=1e-12, rtol=0)


def test_dct3_of_a_basis_function_is_a_delta():
    S, H, W = 6, 5, 4
    ks, kh, kw = 2, 4, 1
    x = np.einsum("s,h,w->shw", O.dct_matrix(S)[ks], O.dct_matrix(H)[kh], O.dct_matrix(W)[kw])
    X = O.dct3(x[..., None])[..., 0]
    want = np.zeros((S, H, W))
    want[ks, kh, kw] = 1.0
    assert np.allclose(X, want, atol=1e-14)


def test_parseval_dc_and_inverse():
    x = RNG.standard_normal((8, 6, 10, 4))
    X = O.dct3(x)
    assert np.allclose((X ** 2).sum(axis=(0, 1, 2)), (x ** 2).sum(axis=(0, 1, 2)), rtol=1e-13)
    assert np.allclose(X[0, 0, 0], x.sum(axis=(0, 1, 2)) / math.sqrt(8 * 6 * 10), rtol=1e-13)
    assert np.allclose(O.idct3(X), x, atol=1e-13)


def test_bin_variance_hand_example():
    X = np.array([[1.0, -2.0, 2.0], [0.0, 3.0, 4.0]])       # 2 bins x 3 channels
    assert np.allclose(O.bin_variances(X), [3.0, 25.0 / 3.0])
    assert O.stored_sigma(np.array([2.25]))[0] == np.float32(1.5)


# ------------------------------------------------------------------------------ Lloyd-Max ---
def test_lloyd_max_one_bit_closed_form():
    y, t = O.table(1)
    assert np.allclose(y, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-15)
    assert t[0] == 0.0
    assert abs(O.quantizer_mse(1) - (1 - 2 / math.pi)) < 1e-14


@pytest.mark.parametrize("bits", range(1, 9))
def test_lloyd_max_optimality_conditions(bits):
    y, t = O.table(bits)
    assert len(y) == 1 << bits and np.all(np.diff(y) > 0)
    assert np.allclose(t, 0.5 * (y[1:] + y[:-1]), atol=0)                # midpoint condition
    # centroid condition, each cell integrated numerically (independent of the closed form used)
    from scipy.integrate import quad
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    for j in range(len(y) // 2, len(y)):                                   # upper half (symmetry below)
        m1 = quad(lambda z: z * math.exp(-0.5 * z * z), edges[j], edges[j + 1], epsabs=0, epsrel=1e-13)[0]
        m0 = quad(lambda z: math.exp(-0.5 * z * z), edges[j], edges[j + 1], epsabs=0, epsrel=1e-13)[0]
        assert abs(m1 / m0 - y[j]) < 1e-11 * max(1.0, abs(y[j]))
    assert np.allclose(y, -y[::-1], atol=0)                                 # symmetry


def test_lloyd_max_matches_max_1960_table(golden_dir):
    rows = {}
    with open(os.path.join(golden_dir, "lloyd_max_max1960.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                parts = line.split()
                rows[(int(parts[0]), parts[1])] = parts[2:]

    def close(ours, printed):
        # half a unit of the last printed digit, plus 1e-4 for the table's own last-digit slips
        for v, txt in zip(ours, printed):
            dec = len(txt.split(".")[1]) if "." in txt else 0
            assert abs(v - float(txt)) <= 0.5 * 10.0 ** -dec + 1e-4, (v, txt)

    for bits in (1, 2, 3, 4):
        y, t = O.table(bits)
        half = len(y) // 2
        close(y[half:], rows[(bits, "levels")])
        close(t[half - 1:], rows[(bits, "thresholds")])
        assert abs(O.quantizer_mse(bits) / float(rows[(bits, "mse")][0]) - 1) < 1e-3


def test_lloyd_max_high_rate_panter_dite():
    # D(b) -> (sqrt(3) pi / 2) 4^-b from below as b grows; MSE strictly decreasing
    mse = [O.quantizer_mse(b) for b in range(1, 9)]
    assert all(a > b for a, b in zip(mse, mse[1:]))
    pd = [math.sqrt(3) * math.pi / 2 * 4.0 ** -b for b in range(1, 9)]
    ratio = [m / p for m, p in zip(mse, pd)]
    assert all(r < 1 for r in ratio) and abs(ratio[-1] - 1) < 0.01
    assert all(a < b for a, b in zip(ratio[1:], ratio[2:]))


@pytest.mark.parametrize("bits", [1, 3, 6])
def test_quantizer_empirical_mse(bits):
    z = np.random.default_rng(bits).standard_normal(400_000)
    zh = O.dequantize(O.quantize(z, bits), bits)
    emp = np.mean((z - zh) ** 2)
    assert abs(emp / O.quantizer_mse(bits) - 1) < 0.02


def test_quantize_decisions():
    _, t1 = O.table(1)
    assert list(O.quantize(np.array([-0.1, 0.0, 0.5, -1e30, 1e30]), 1)) == [0, 1, 1, 0, 1]
    y2, t2 = O.table(2)
    # thresholds of the 2-bit table are (-t, 0, t) with t = 0.9816; -t2[2] is the same value as t2[0]
    codes = O.quantize(np.array([-5.0, -t2[2], t2[0] - 1e-3, t2[0], 0.0, 0.1, t2[2], 7.0]), 2)
    assert list(codes) == [0, 1, 0, 1, 2, 2, 3, 3]
    # a threshold itself goes to the upper cell (decided in float32)
    assert O.quantize(np.array([np.float32(t2[2])]), 2)[0] == 3


def _max1960_thresholds(golden_dir, bits):
    with open(os.path.join(golden_dir, "lloyd_max_max1960.txt")) as f:
        for line in f:
            p = line.split()
            if p and not line.startswith("#") and int(p[0]) == bits and p[1] == "thresholds":
                return [float(v) for v in p[2:]]
    raise KeyError(bits)


def test_threshold_distance_hand_values(golden_dir):
    """The code-parity band: distance from u to the NEAREST decision threshold t_j, divided by
    max(1, |t_j|).  Pinned with thresholds printed by Max (1960) (4 significant digits, so every
    expected value below is checked to a relative 1e-2, far tighter than any of the planted
    alternatives: a squared divisor, the farthest threshold, the levels instead of thresholds)."""
    t2 = _max1960_thresholds(golden_dir, 2)          # 0, 0.9816 (and -0.9816)
    t3 = _max1960_thresholds(golden_dir, 3)          # 0, 0.5006, 1.050, 1.748
    # the middle threshold 0 of an even codebook: the absolute distance
    assert abs(O.threshold_distance(np.array([0.25]), 1)[0] - 0.25) < 1e-12
    assert abs(O.threshold_distance(np.array([-0.3]), 1)[0] - 0.3) < 1e-12
    assert abs(O.threshold_distance(np.array([0.01]), 2)[0] - 0.01) < 1e-12
    # a threshold below 1 in magnitude: absolute distance as well
    d = O.threshold_distance(np.array([t2[1] + 0.1, -(t2[1] + 0.1)]), 2)
    assert np.allclose(d, 0.1, rtol=1e-2)
    # a threshold above 1: the distance relative to |t_j| (not |t_j|^2)
    d = O.threshold_distance(np.array([t3[3] + 0.2]), 3)[0]
    assert abs(d / (0.2 / t3[3]) - 1) < 1e-2
    # between two thresholds the nearer one counts: 0.75 lies 0.2494 above 0.5006 and 0.30 below
    # 1.050 (0.2857 relative); the level 0.7560 in between is no decision boundary
    d = O.threshold_distance(np.array([0.75]), 3)[0]
    assert abs(d / (0.75 - t3[1]) - 1) < 1e-2
    # far outside the table the outermost threshold decides: 3 bits, u = 5 -> (5 - 1.748) / 1.748
    d = O.threshold_distance(np.array([5.0]), 3)[0]
    assert abs(d / ((5.0 - t3[3]) / t3[3]) - 1) < 1e-2
    # vectorised over any shape
    assert O.threshold_distance(np.zeros((3, 4)), 2).shape == (3, 4)


# ------------------------------------------------------------------------------ allocation ---
def _random_var(N, rng, spread=8.0):
    return np.exp(rng.uniform(-spread, spread, N))


@pytest.mark.parametrize("seed", range(12))
def test_allocation_equals_bruteforce_topk(seed):
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(1, 200))
    var = _random_var(N, rng, spread=float(rng.uniform(0.5, 9)))
    if seed % 3 == 0:                                      # inactive bins
        var[rng.random(N) < 0.2] = 0.0
    if seed % 4 == 1 and N > 4:                            # exact ties, also across powers of 4
        var[1] = var[0]
        var[2] = var[0] * 16.0
        var[3] = var[0] / 4.0
    for bits in (1, 2, 3, 4, 8):
        b = O.allocate_bits(var, bits)
        assert np.array_equal(b, O.allocate_bits_topk(var, bits)), (N, bits)
        assert b.min() >= 0 and b.max() <= 8 and np.all(b[var == 0] == 0)
        act = int((var > 0).sum())
        assert b.sum() == min(bits * N, 8 * act)           # budget hit exactly when feasible


def test_allocation_special_cases():
    assert np.array_equal(O.allocate_bits(np.zeros(5), 2), np.zeros(5))
    assert np.array_equal(O.allocate_bits(np.ones(4), 8), np.full(4, 8))
    # equal variances at 3 bits: everybody gets 3 (all keys tie, the top-B set is the first 3 per bin)
    assert np.array_equal(O.allocate_bits(np.ones(7), 3), np.full(7, 3))
    # one dominant bin: it saturates at 8, the rest share what is left
    b = O.allocate_bits(np.array([1e12, 1.0, 1.0, 1.0]), 3)
    assert b[0] == 8 and b.sum() == 12
    # sigma^2 = (1, 1, 16), B = 3: keys 16 and 4 (bin 2) are taken, then the value 1 ties three ways
    # (bin 0 k=0, bin 1 k=0, bin 2 k=2) and the lowest bin index takes the last slot
    assert O.allocate_bits(np.array([1.0, 1.0, 16.0]), 1).tolist() == [1, 0, 2]
    assert O.allocate_bits(np.array([1.0, 4.0, 4.0]), 1).tolist() == [1, 1, 1]
    # larger variance never gets fewer bits
    rng = np.random.default_rng(7)
    var = _random_var(300, rng)
    b = O.allocate_bits(var, 2)
    order = np.argsort(var)
    assert np.all(np.diff(b[order]) >= 0)


def test_theorem1_closed_form_continuous():
    """Theorem 1 (Key Contributions item 2): D_uniform / D_waterfilling = 1/gamma, gamma the spectral
    flatness GM/AM of the bin variances, for the continuous allocation with every rate inside (0, 8)
    and distortion sigma^2 4^-b per bin."""
    rng = np.random.default_rng(1)
    var = 10.0 ** rng.uniform(-1, 1, 500)                  # two decades: every bin stays active
    bits = 4
    B = bits * var.size
    r = O.waterfill_rate(var, O.water_level(var, B))
    assert r.min() > 0 and r.max() < 8
    assert abs(r.sum() - B) < 1e-8
    d_uniform = np.sum(var * 4.0 ** -bits)
    d_wf = np.sum(var * 4.0 ** -r)
    gamma = math.exp(np.mean(np.log(var))) / np.mean(var)
    assert abs((d_uniform / d_wf) * gamma - 1) < 1e-12


def test_theorem1_empirical_high_rate():
    """With integer bits and the real Lloyd-Max quantizer on Gaussian bins the ratio approaches
    1/gamma in the high-rate regime (the pages flag 1 bit as outside it)."""
    rng = np.random.default_rng(2)
    N, n, bits = 64, 4000, 5
    var = 10.0 ** rng.uniform(-1, 1, N)
    X = rng.standard_normal((N, n)) * np.sqrt(var)[:, None]
    sig = np.sqrt((X ** 2).mean(axis=1))

    def distortion(b):
        d = 0.0
        for i in range(N):
            u = X[i] / sig[i]
            xh = sig[i] * O.dequantize(O.quantize(u, int(b[i])), int(b[i])) if b[i] else 0 * u
            d += np.sum((X[i] - xh) ** 2)
        return d

    ratio = distortion(np.full(N, bits)) / distortion(O.allocate_bits(sig ** 2, bits))
    inv_gamma = np.mean(sig ** 2) / math.exp(np.mean(np.log(sig ** 2)))
    assert abs(ratio / inv_gamma - 1) < 0.10


# -------------------------------------------------------------------------- payload / codec ---
def test_pack_streams_hand_example():
    b = np.array([2, 0, 3])
    codes = np.array([[3, 1], [0, 0], [5, 2]])             # bins x channels
    s = O._pack_streams(codes, b, 16)
    # channel 0: bin0=3 -> bits 0,1 = 1,1; bin2=5 -> bits 2..4 = 1,0,1  => 0b10111
    # channel 1: bin0=1 -> bits 0,1 = 1,0; bin2=2 -> bits 2..4 = 0,1,0  => 0b01001
    assert s.shape == (2, 16) and s[0, 0] == 0x17 and s[1, 0] == 0x09 and not s[:, 1:].any()
    assert np.array_equal(O._unpack_streams(s, b), codes)


def test_pack_crosses_bytes():
    b = np.array([8, 8, 1, 7])
    codes = np.array([[0xA5], [0x3C], [1], [0x55]])
    s = O._pack_streams(codes, b, 16)
    assert list(s[0, :4]) == [0xA5, 0x3C, 0xAB, 0x00]      # 1 | 0x55 << 1 = 0xAB
    assert np.array_equal(O._unpack_streams(s, b), codes)


def test_compress_header_size_and_no_quant_roundtrip():
    S, H, W, heads, D = 4, 3, 5, 2, 8
    x = RNG.standard_normal((S * H * W, heads, D))
    p = O.compress_unit(x, S, H, W, heads, D, bits=3, layer=7, kv=1, no_quant=True)
    f = struct.unpack_from(O.HEADER_FMT, p, 0)
    assert f[0] == O.MAGIC and f[3:11] == (7, 1, S, H, W, heads, D, 3)
    assert np.allclose(O.decompress_unit(p), x, atol=1e-6)  # fp32 coefficient storage
    assert len(p) == O.payload_capacity(S, H, W, heads, D, 3, no_quant=True)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_compress_occupancy_and_reconstruction(bits):
    """Occupancy sum_i b_i * n bits of codes + 32 bits of gain per bin + 1 byte index (stage 4),
    and a reconstruction error consistent with the allocated rates."""
    S, H, W, heads, D = 6, 5, 4, 2, 32
    import torch
    from dct_transform_coding_b200.workloads import make_unit
    x = make_unit(S, H, W, heads, D, rho=(0.9, 0.8, 0.7), nu=4.0, seed=bits, dtype=torch.float32).numpy()
    p, info = O.compress_unit(x, S, H, W, heads, D, bits, return_info=True)
    N, n = S * H * W, heads * D
    b = info["b"]
    assert b.sum() == bits * N or b.sum() == 8 * N
    lay = O.payload_layout(N, n, int(b.sum()))
    assert len(p) == lay["total"] <= O.payload_capacity(S, H, W, heads, D, bits)
    assert lay["chan_stride"] * 8 - b.sum() < 128           # only 16-byte padding per channel
    xh = O.decompress_unit(p)
    # predicted distortion: sum_i sigma_i^2 * D(b_i) (dropped bins lose all their energy)
    pred = sum(info["var"][i] * (O.quantizer_mse(int(b[i])) if b[i] else 1.0) for i in range(N)) * n
    err = np.sum((xh.reshape(-1) - x.reshape(-1)) ** 2)
    assert 0.5 < err / pred < 2.0
    bb, codes = O.codes_of(p)
    assert np.array_equal(bb, b) and np.array_equal(codes, info["codes"])


def test_to_bf16_rounding():
    import torch
    # bf16 keeps 8 significant bits: spacing 2^-7 just above 1; halfway cases go to the even neighbour
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -9 + 2 ** -20), 3.14159, 0.0])
    got = O.to_bf16(v)
    assert got[0] == 1.0 and got[1] == 1.0 and got[2] == 1.0 + 2 ** -6 and got[3] == -1.0 and got[5] == 0.0
    r = np.random.default_rng(3).standard_normal(10000).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(r.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.to_bf16(r), ref)


# ------------------------------------------------------------------- occupancy and capacity ---
def test_occupancy_hand_example():
    """Stage 4: sum_i (b_i d + 32) bits, plus one index byte per bin."""
    assert O.occupancy_bits(np.array([2, 0, 3]), 2) == (2 * 2 + 32) + (0 + 32) + (3 * 2 + 32)
    assert O.occupancy_bits(np.zeros(5, int), 128) == 5 * 32
    assert O.index_bits(7) == 56


def test_occupancy_bounds_the_payload():
    """The payload holds exactly the occupancy and the index plus the header and 16-byte padding."""
    S, H, W, heads, D = 4, 3, 5, 2, 16
    x = RNG.standard_normal((S * H * W, heads, D))
    for bits in (1, 3):
        p, info = O.compress_unit(x, S, H, W, heads, D, bits, return_info=True)
        N, n = S * H * W, heads * D
        need_bits = O.occupancy_bits(info["b"], n) + O.index_bits(N)
        assert 8 * len(p) >= need_bits
        assert 8 * len(p) - need_bits < 8 * (64 + 16 + 16 + 16 * n)    # header and paddings only


def test_max_batch_hand_values():
    assert O.max_batch(100, 30, 7) == 10
    assert O.max_batch(10, 20, 1) == 0
    assert O.max_batch(10, 0, 0) == -1


# ----------------------------------------------------- variants: rotation, axis mask, uniform ---
def test_splitmix64_published_outputs():
    """SplitMix64 (Steele, Lea and Flood 2014) from seed 0: the first three outputs of the
    reference implementation (java.util.SplittableRandom's mix64 on the gamma sequence)."""
    assert [O.splitmix64(0, i) for i in range(3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_hadamard_matches_scipy():
    import scipy.linalg
    for m in (1, 2, 8, 32):
        assert np.array_equal(O.hadamard(m), scipy.linalg.hadamard(m))


def test_rotation_is_orthogonal_block_diagonal_and_keeps_the_gain():
    n = 96
    R = O.rotation_matrix(n)
    assert np.allclose(R @ R.T, np.eye(n), atol=1e-14, rtol=0)
    assert np.allclose(np.abs(R[:32, :32]), 1 / math.sqrt(32), atol=0)
    assert not R[:32, 32:].any() and not R[32:64, :32].any()          # groups of 32 channels
    s = O.rotation_signs(n)
    assert set(np.unique(s)) <= {-1.0, 1.0} and 20 < np.sum(s > 0) < 76
    X = RNG.standard_normal((10, n))
    assert np.allclose(O.bin_variances(X @ R.T), O.bin_variances(X), rtol=1e-13)   # gains unchanged


def test_rotation_round_trip_and_gaussianization():
    """With the rotation on, decompress(compress(x)) still reconstructs x (the decoder undoes R),
    and a bin whose energy sits in one channel per group is spread over all 32 of them."""
    S, H, W, heads, D = 2, 3, 4, 1, 64
    x = RNG.standard_normal((S * H * W, heads, D))
    p8 = O.compress_unit(x, S, H, W, heads, D, 8, flags=O.FLAG_ROTATE)
    assert O.parse_payload(p8)["flags"] & O.FLAG_ROTATE
    assert np.sqrt(np.mean((O.decompress_unit(p8) - x) ** 2)) < 0.02 * np.sqrt(np.mean(x ** 2))
    e = np.zeros((1, 64))
    e[0, 5] = 1.0
    v = (e @ O.rotation_matrix(64).T)[0]
    assert np.allclose(np.abs(v[:32]), 1 / math.sqrt(32)) and not v[32:].any()
    # same allocation and gains as without the rotation; the codes differ
    p0, i0 = O.compress_unit(x, S, H, W, heads, D, 2, return_info=True)
    p1, i1 = O.compress_unit(x, S, H, W, heads, D, 2, return_info=True, flags=O.FLAG_ROTATE)
    assert np.array_equal(i0["b"], i1["b"]) and np.array_equal(i0["sigma"], i1["sigma"])
    assert not np.array_equal(i0["codes"], i1["codes"])


@pytest.mark.parametrize("axes", [(True, False, False), (False, True, True), (False, False, True),
                                  (False, False, False)])
def test_axis_mask_matches_scipy_on_the_kept_axes(axes):
    x = RNG.standard_normal((5, 6, 7, 3))
    keep = tuple(a for a, k in zip((0, 1, 2), axes) if k)
    ref = scipy.fft.dctn(x, type=2, norm="ortho", axes=keep) if keep else x
    assert np.allclose(O.dct3(x, axes), ref, atol=1e-12, rtol=0)
    assert np.allclose(O.idct3(ref, axes), x, atol=1e-12, rtol=0)
    flags = (0 if axes[0] else O.FLAG_SKIP_S) | (0 if axes[1] else O.FLAG_SKIP_H) | (0 if axes[2] else O.FLAG_SKIP_W)
    assert O.axes_of(flags) == axes


def test_uniform_allocation_and_theorem1_through_the_codec():
    """FLAG_UNIFORM gives every active bin the nominal bits; on Gaussian bins with spread variances
    the distortion of the uniform payload over the water-filling payload approaches AM/GM of the
    variances (Theorem 1) at a high rate."""
    assert O.allocate_uniform(np.array([0.0, 2.0, 5.0]), 3).tolist() == [0, 3, 3]
    rng = np.random.default_rng(11)
    S, H, W, heads, D, bits = 4, 4, 4, 8, 250, 5
    N, n = S * H * W, heads * D
    var = 10.0 ** rng.uniform(-1, 1, N)
    X = rng.standard_normal((N, n)) * np.sqrt(var)[:, None]
    x = O.idct3(X.reshape(S, H, W, n)).reshape(N, heads, D)     # a field whose bins hold X
    d = {}
    for name, fl in (("uniform", O.FLAG_UNIFORM), ("wf", 0)):
        p, info = O.compress_unit(x, S, H, W, heads, D, bits, return_info=True, flags=fl)
        if fl:
            assert np.all(info["b"] == bits)
        d[name] = np.sum((O.decompress_unit(p) - x) ** 2)
    v = O.bin_variances(X)
    inv_gamma = np.mean(v) / math.exp(np.mean(np.log(v)))
    assert abs(d["uniform"] / d["wf"] / inv_gamma - 1) < 0.1


# -------------------------------------------------------------------------- per-head gains ---
def test_head_gain_one_head_is_the_pooled_gain():
    """With a single head the per-head gain is the bin's pooled gain: same b, gains, codes and
    reconstruction as the default payload; only the header's flag differs."""
    S, H, W, heads, D = 2, 4, 4, 1, 64
    x = RNG.standard_normal((S * H * W, heads, D))
    p0, i0 = O.compress_unit(x, S, H, W, heads, D, 3, return_info=True)
    p1, i1 = O.compress_unit(x, S, H, W, heads, D, 3, return_info=True, flags=O.FLAG_HEAD_GAIN)
    assert np.array_equal(i0["b"], i1["b"]) and np.array_equal(i0["codes"], i1["codes"])
    assert np.array_equal(O.parse_payload(p1)["sigma"], O.parse_payload(p0)["sigma"][None])
    assert np.array_equal(O.decompress_unit(p0), O.decompress_unit(p1))
    assert p0[:6] == p1[:6] and p0[8:] == p1[8:] and p1[6:8] != p0[6:8]


def test_head_gain_scaled_copy_of_a_head():
    """Gain-shape per head: head 1 = 4 x head 0 (exact in fp64) gives gains g1 = 4 g0 exactly and the
    very codes of head 0, and reconstructs to 4 x head 0's reconstruction; one gain per bin would
    quantize head 1 on another scale (different codes)."""
    S, H, W, D, bits = 2, 4, 4, 32, 3
    x0 = RNG.standard_normal((S * H * W, 1, D))
    x = np.concatenate([x0, 4.0 * x0], axis=1)
    p, info = O.compress_unit(x, S, H, W, 2, D, bits, return_info=True, flags=O.FLAG_HEAD_GAIN)
    g = O.parse_payload(p)["sigma"]
    assert g.shape == (2, S * H * W) and np.array_equal(g[1], 4 * g[0])
    act = info["b"] > 0
    assert np.array_equal(info["codes"][act][:, D:], info["codes"][act][:, :D])
    y = O.decompress_unit(p)
    assert np.array_equal(y[:, 1], 4 * y[:, 0])
    _, pooled = O.compress_unit(x, S, H, W, 2, D, bits, return_info=True)
    assert not np.array_equal(pooled["codes"][act][:, D:], pooled["codes"][act][:, :D])


def test_head_gain_silent_head_and_occupancy():
    """A head whose channels are all zero gets zero gains and an exactly zero reconstruction, the
    other head's gains are those of its own channels; the payload carries heads x N gains, and the
    stage-4 occupancy counts one 32-bit gain per (bin, head)."""
    S, H, W, D, bits = 2, 2, 4, 32, 2
    N = S * H * W
    x = np.concatenate([RNG.standard_normal((N, 1, D)), np.zeros((N, 1, D))], axis=1)
    p, info = O.compress_unit(x, S, H, W, 2, D, bits, return_info=True, flags=O.FLAG_HEAD_GAIN)
    g = O.parse_payload(p)["sigma"]
    assert not g[1].any()
    assert np.array_equal(g[0], np.sqrt(np.mean(info["X"][:, :D] ** 2, axis=1)).astype(np.float32))
    y = O.decompress_unit(p)
    assert not y[:, 1].any() and np.sqrt(np.mean((y[:, 0] - x[:, 0]) ** 2)) < 0.5
    # gains region: pad16(4 * heads * N) bytes; the codes follow it
    lay = O.payload_layout(N, 2 * D, int(info["b"].sum()), gains=2)
    assert lay["off_codes"] - lay["off_sigma"] == 4 * 2 * N and len(p) == lay["total"]
    b = info["b"]
    assert O.occupancy_bits(b, D, 2) == int(np.sum(b) * 2 * D + 32 * 2 * N)
    assert O.occupancy_bits(b, 2 * D) == int(np.sum(b) * 2 * D + 32 * N)


# ------------------------------------------------------------------- decode-time attention ---
def test_attention_decode_matches_torch_sdpa():
    """The oracle's attention over a compressed cache equals torch's scaled_dot_product_attention
    (fp64, grouped query heads expanded) applied to the decompressed K and V."""
    import torch
    S, H, W, kv_heads, D, G = 4, 3, 5, 2, 32, 3
    rng = np.random.default_rng(5)
    k = rng.standard_normal((S * H * W, kv_heads, D))
    v = rng.standard_normal((S * H * W, kv_heads, D))
    pk = O.compress_unit(k, S, H, W, kv_heads, D, 3)
    pv = O.compress_unit(v, S, H, W, kv_heads, D, 3, kv=1)
    q = rng.standard_normal((kv_heads * G, D))
    out, m, l = O.attention_decode(q, pk, pv)
    K = torch.from_numpy(O.decompress_unit(pk)).permute(1, 0, 2).repeat_interleave(G, 0)   # [Hq, T, D]
    V = torch.from_numpy(O.decompress_unit(pv)).permute(1, 0, 2).repeat_interleave(G, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q)[:, None, :], K, V)[:, 0, :]
    assert np.allclose(out, ref.numpy(), atol=1e-12, rtol=1e-12)
    s = torch.einsum("hd,htd->ht", torch.from_numpy(q), K) / math.sqrt(D)
    assert np.allclose(m, s.max(dim=1).values.numpy(), atol=1e-12)
    assert np.allclose(l, torch.exp(s - s.max(dim=1, keepdim=True).values).sum(1).numpy(), rtol=1e-12)


def test_attention_decode_special_cases():
    """A zero query attends uniformly (the output is the mean of the value rows, l = T); a query
    that picks one token out by a large margin returns that token's value row."""
    S, H, W, D = 2, 2, 4, 32
    T = S * H * W
    rng = np.random.default_rng(6)
    v = rng.standard_normal((T, 1, D))
    pv = O.compress_unit(v, S, H, W, 1, D, 8, kv=1)
    Vh = O.decompress_unit(pv)[:, 0, :]
    k = np.zeros((T, 1, D))
    k[5, 0, 0] = 1.0
    pk = O.compress_unit(k, S, H, W, 1, D, 8, no_quant=True)      # exact keys (float32 coefficients)
    out, m, l = O.attention_decode(np.zeros((1, D)), pk, pv)
    assert np.allclose(out[0], Vh.mean(axis=0), atol=1e-12) and abs(l[0] - T) < 1e-9
    q = np.zeros((1, D))
    q[0, 0] = 400.0 * math.sqrt(D)
    out, m, l = O.attention_decode(q, pk, pv)
    assert np.allclose(out[0], Vh[5], atol=1e-9) and abs(l[0] - 1) < 1e-9
