"""The C ABI library on a machine without a GPU: it loads, exports every symbol include/tactkv.h
declares, and its host-only functions and argument checks behave (no kernel is launched)."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import tactkv_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def T():
    from dct_transform_coding_b200 import tactkv
    return tactkv


def test_exports_every_declared_symbol(T):
    header = open(os.path.join(ROOT, "include", "tactkv.h")).read()
    declared = set(re.findall(r"^\w[\w\s\*]*?\b(tactkv_\w+)\s*\(", header, flags=re.M))
    assert declared >= set(T.EXPORTED)
    lib = ctypes.CDLL(T.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def test_format_version_and_status_strings(T):
    assert T.tactkv_format_version() == O.VERSION
    assert T.tactkv_status_string(T.TACTKV_OK) == "ok"
    assert T.tactkv_status_string(T.TACTKV_CORRUPT_PAYLOAD) == "corrupt payload"
    assert T.tactkv_status_string(99) == "unknown status"


@pytest.mark.parametrize("bits", range(1, 9))
def test_library_codebooks_match_oracle(T, bits):
    """Two independent Lloyd-Max solvers (library build step vs oracle) agree to 1e-12."""
    lv, th = T.tactkv_lloyd_max_table(bits)
    y, t = O.table(bits)
    assert np.max(np.abs(np.array(lv) - y)) < 1e-12
    assert np.max(np.abs(np.array(th) - t)) < 1e-12


def test_codebook_rejects_bad_bits(T):
    with pytest.raises(ValueError):
        T.tactkv_lloyd_max_table(0)
    with pytest.raises(ValueError):
        T.tactkv_lloyd_max_table(9)


@pytest.mark.parametrize("shape,bits,flags", [((64, 16, 16, 4, 256), 1, 0), ((32, 24, 24, 8, 128), 1, 0),
                                              ((64, 14, 14, 4, 128), 4, 0), ((8, 8, 8, 1, 64), 2, 0),
                                              ((8, 8, 8, 1, 64), 2, 1), ((5, 7, 3, 2, 32), 8, 0),
                                              ((64, 16, 16, 4, 256), 1, 128), ((5, 7, 3, 2, 32), 3, 128),
                                              ((8, 8, 8, 2, 64), 2, 129)])
def test_payload_capacity_matches_oracle_layout(T, shape, bits, flags):
    S, H, W, heads, D = shape
    cap = T.payload_capacity(S, H, W, heads, D, bits, flags)
    assert cap == O.payload_capacity(S, H, W, heads, D, bits, flags=flags)


def test_unsupported_shapes_report_zero_capacity(T):
    for S, H, W, heads, D in [(17, 8, 8, 1, 32), (8, 33, 8, 1, 32), (8, 8, 8, 1, 30), (8, 8, 8, 1, 48),
                              (65, 8, 8, 1, 32), (8, 32, 40, 1, 32)]:
        u = T.tactkv_unit(S=S, H=H, W=W, heads=heads, head_dim=D, bits=2)
        assert T.tactkv_payload_bytes(u) == 0, (S, H, W, heads, D)


def _unit(T, **kw):
    d = dict(S=8, H=8, W=8, heads=1, head_dim=32, bits=2, flags=0, kv_in=4096, kv_out=4096,
             token_stride=32, head_stride=32, payload=8192, payload_capacity=1 << 20)
    d.update(kw)
    return T.tactkv_unit(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(bits=0), "TACTKV_INVALID_ARG"), (dict(bits=9), "TACTKV_INVALID_ARG"),
    (dict(flags=256), "TACTKV_INVALID_ARG"), (dict(S=0), "TACTKV_INVALID_ARG"),
    (dict(flags=128, heads=2, head_dim=48), "TACTKV_UNSUPPORTED_SHAPE"),   # per-head gains: head_dim % 32
    (dict(kv_in=None), "TACTKV_INVALID_ARG"), (dict(payload=None), "TACTKV_INVALID_ARG"),
    (dict(token_stride=0), "TACTKV_INVALID_ARG"),
    (dict(S=17), "TACTKV_UNSUPPORTED_SHAPE"), (dict(head_dim=30), "TACTKV_UNSUPPORTED_SHAPE"),
    (dict(kv_in=4098), "TACTKV_ALIGNMENT"), (dict(token_stride=33), "TACTKV_ALIGNMENT"),
    (dict(payload=8200), "TACTKV_ALIGNMENT"), (dict(payload_capacity=100), "TACTKV_CAPACITY"),
])
def test_compress_argument_checks_without_gpu(T, kw, status):
    units = [_unit(T, **kw)]
    st = T.tactkv_compress(units, 1 << 20, 1 << 30, 0)
    assert st == getattr(T, status)


def test_workspace_checks_without_gpu(T):
    units = [_unit(T)]
    assert T.tactkv_compress(units, 0, 1 << 30, 0) == T.TACTKV_WORKSPACE
    assert T.tactkv_compress(units, 1 << 20, 16, 0) == T.TACTKV_WORKSPACE
    assert T.tactkv_compress(units, (1 << 20) + 8, 1 << 30, 0) == T.TACTKV_WORKSPACE
    assert T.tactkv_compress([], 1 << 20, 1 << 30, 0) == T.TACTKV_OK
    need = T.tactkv_workspace_bytes(units)
    assert need >= 8 * 8 * 8 * 32 * 4
    # a workspace one byte short of a single unit is refused before anything is launched
    assert T.tactkv_compress(units, 1 << 20, need - 1, 0) == T.TACTKV_WORKSPACE


def test_allocate_argument_checks_without_gpu(T):
    u = _unit(T)
    assert T.tactkv_allocate(u, 0, 1 << 20, 1 << 30, 0) == T.TACTKV_INVALID_ARG          # no variances
    assert T.tactkv_allocate(_unit(T, payload=None), 4096, 1 << 20, 1 << 30, 0) == T.TACTKV_INVALID_ARG
    assert T.tactkv_allocate(_unit(T, bits=9), 4096, 1 << 20, 1 << 30, 0) == T.TACTKV_INVALID_ARG
    assert T.tactkv_allocate(_unit(T, S=17), 4096, 1 << 20, 1 << 30, 0) == T.TACTKV_UNSUPPORTED_SHAPE
    assert T.tactkv_allocate(u, 4100, 1 << 20, 1 << 30, 0) == T.TACTKV_ALIGNMENT        # var not 8-aligned
    assert T.tactkv_allocate(_unit(T, payload_capacity=100), 4096, 1 << 20, 1 << 30, 0) == T.TACTKV_CAPACITY
    need = T.tactkv_workspace_bytes([u])
    assert T.tactkv_allocate(u, 4096, 1 << 20, need - 1, 0) == T.TACTKV_WORKSPACE
    assert T.tactkv_allocate(u, 4096, 0, need, 0) == T.TACTKV_WORKSPACE
    # per-head gains come from the channels, which the given variances do not carry
    assert T.tactkv_allocate(_unit(T, flags=128), 4096, 1 << 20, 1 << 30, 0) == T.TACTKV_INVALID_ARG


def _attention_status(T, S, H, W, heads, D, bits, q_heads, flags=0):
    """tactkv_attention_decode's host checks only: fake device pointers and a null workspace, so a
    call that passes the shape checks stops at TACTKV_WORKSPACE before anything is launched."""
    ku = (T.tactkv_unit * 1)(_unit(T, S=S, H=H, W=W, heads=heads, head_dim=D, bits=bits, flags=flags, kv=0,
                                   payload_capacity=1 << 40))
    vu = (T.tactkv_unit * 1)(_unit(T, S=S, H=H, W=W, heads=heads, head_dim=D, bits=bits, flags=flags, kv=1,
                                   payload_capacity=1 << 40))
    p = ctypes.c_void_p(4096)
    return int(T._lib.tactkv_attention_decode(ku, vu, 1, q_heads, p, p, p, p, None, 0, None))


@pytest.mark.parametrize("shape,bits,q_heads,flags,status", [
    ((64, 16, 16, 4, 256), 1, 8, 0, "TACTKV_WORKSPACE"),       # the benchmark layer: supported
    ((64, 16, 16, 4, 256), 1, 8, 1, "TACTKV_UNSUPPORTED_SHAPE"),   # NO_QUANT payloads
    ((64, 16, 16, 4, 256), 1, 6, 0, "TACTKV_UNSUPPORTED_SHAPE"),   # q_heads not a multiple of heads
    ((8, 8, 8, 1, 64), 2, 17, 0, "TACTKV_UNSUPPORTED_SHAPE"),      # more than 16 query heads per K/V head
    # the stream-word rows are sized for min(8, 2*bits + 2) bits per bin: a 32 x 32 slab of 256
    # channels fits at 1 bit per element (131 words per channel) but not at 4 (259 words, 265 KB)
    ((8, 32, 32, 1, 256), 1, 2, 0, "TACTKV_WORKSPACE"),
    ((8, 32, 32, 1, 256), 4, 2, 0, "TACTKV_UNSUPPORTED_SHAPE"),
])
def test_attention_shape_checks_without_gpu(T, shape, bits, q_heads, flags, status):
    S, H, W, heads, D = shape
    assert _attention_status(T, S, H, W, heads, D, bits, q_heads, flags) == getattr(T, status)


def test_decompress_checks_output_pointer(T):
    units = [_unit(T, kv_out=None)]
    assert T.tactkv_decompress(units, 1 << 20, 1 << 30, 0) == T.TACTKV_INVALID_ARG


# ------------------------------------------------------------ code lookup of the quantizer ---
def _gen_tables():
    import importlib.util
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "dct_transform_coding_b200", "csrc", "gen_tables.py")
    spec = importlib.util.spec_from_file_location("gen_tables", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _csrc_module(name):
    import importlib.util
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "dct_transform_coding_b200", "csrc", name + ".py")
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("L", [1, 2, 3, 5, 7, 8, 14, 16, 20, 24, 28, 32, 40, 48, 56, 64])
def test_generated_pencil_programs_match_scipy(L):
    """The library's generated DCT programs (forward and its transpose), evaluated in float64 and in
    float32, against scipy's orthonormal DCT-II / DCT-III: exact to rounding in float64, and within a
    few float32 ulps of the largest coefficient in float32 (the accuracy the codes rely on)."""
    import scipy.fft
    G = _csrc_module("gen_dct")
    g, outs = G.build_forward(L)
    tg, touts = G.transpose_graph(g, outs)
    x = np.random.default_rng(L).standard_normal((L, 64))
    ref_f = scipy.fft.dct(x, type=2, norm="ortho", axis=0)
    ref_i = scipy.fft.idct(x, type=2, norm="ortho", axis=0)
    assert np.max(np.abs(G.evaluate(g, outs, x) - ref_f)) < 1e-12
    assert np.max(np.abs(G.evaluate(tg, touts, x) - ref_i)) < 1e-12
    f32 = G.evaluate(g, outs, x.astype(np.float32), dtype=np.float32).astype(np.float64)
    assert np.max(np.abs(f32 - ref_f)) < 16 * np.finfo(np.float32).eps * np.max(np.abs(ref_f))


@pytest.mark.parametrize("L", [16, 32, 64])
def test_tensor_core_limbs_rebuild_the_dct_matrix(L):
    """The three bf16 limbs of the DCT matrix used by the tensor-core S pass: each limb exactly a
    bfloat16 value, their sum equal to scipy's orthonormal DCT-II matrix within 2^-24, and the
    rounding to bfloat16 ties to even."""
    import scipy.fft
    G = _csrc_module("gen_mma_tables")
    C = scipy.fft.dct(np.eye(L), type=2, norm="ortho", axis=0)
    parts = G.limbs(G.dct_matrix(L))
    for p in parts:
        assert np.array_equal(p, p.astype(np.float32).astype(np.float64))
        for v in p.ravel()[:64]:
            G.bf16_bits(float(v))              # raises unless the low 16 bits of the float32 are 0
    assert np.max(np.abs(parts[0] + parts[1] + parts[2] - C)) <= 2.0 ** -24
    assert G.round_bf16(1.0 + 2.0 ** -8) == 1.0 and G.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2 ** -6
    assert G.round_bf16(-(1.0 + 2.0 ** -8 + 2.0 ** -20)) == -(1.0 + 2.0 ** -7)


@pytest.mark.parametrize("bits", range(3, 9))
def test_cell_table_code_lookup_equals_threshold_count(bits):
    """The kernels' code lookup for b >= 3 (cell of u, table count, two compares), emulated in
    float32 exactly as the device computes it, equals the number of float32 thresholds <= u for
    values on, next to and between every threshold, far outside the range, and at +-0."""
    G = _gen_tables()
    lv, th = G.codebook(bits)
    th32 = np.array(th, dtype=np.float32)
    tab, scale, offset = G.code_table([float(t) for t in th32])
    tab = np.array(tab)
    padded = np.concatenate([th32, np.array([np.inf, np.inf], np.float32)])
    rng = np.random.default_rng(bits)
    u = [th32, np.nextafter(th32, np.float32(np.inf)), np.nextafter(th32, np.float32(-np.inf)),
         rng.uniform(-6, 6, 200000).astype(np.float32), rng.standard_normal(200000).astype(np.float32) * 3,
         np.array([0.0, -0.0, 4.5, -4.5, 1e30, -1e30, 1e-40, -1e-40], np.float32)]
    for k in range(2, 6):   # a few ulps on both sides of every threshold
        u.append(th32 + np.float32(k) * np.spacing(th32))
        u.append(th32 - np.float32(k) * np.spacing(th32))
    u = np.concatenate(u).astype(np.float32)
    # fmaf(u, scale, offset): u*scale + offset is exact in float64, so one rounding to float32
    jf = (u.astype(np.float64) * np.float64(np.float32(scale)) + np.float64(np.float32(offset))).astype(np.float32)
    j = np.clip(np.floor(jf.astype(np.float64)), 0, G.QK - 1).astype(np.int64)
    c = tab[j]
    code = c + (u >= padded[c]) + (u >= padded[c + 1])
    want = np.searchsorted(th32, u, side="right")
    assert np.array_equal(code, want)


def _c_array(text, name):
    """The initialiser of the C array `name` in generated source, as a list of numbers."""
    import re
    body = re.search(r"\b" + name + r"\[\] = \{(.*?)\};", text, re.S).group(1)
    vals = []
    for tok in body.replace("\n", " ").split(","):
        tok = tok.strip()
        if tok:
            vals.append(np.inf if tok == "INFINITY" else float(tok.rstrip("f")))
    return vals


def test_global_table_copies_match_the_constant_tables():
    """The 16-byte-vector copies of the codebook tables that kernels stage into shared memory: the
    levels behind a leading zero, the padded thresholds, the threshold pairs the packer compares
    against after its cell lookup, and the code cells, each equal to its constant-memory table and
    padded to whole 16-byte vectors."""
    G = _gen_tables()
    text = G.generate()
    lv, lv0 = _c_array(text, "c_lm_levels"), _c_array(text, "g_lm_levels0")
    thr, thr16 = _c_array(text, "c_thr_pad"), _c_array(text, "g_thr_pad")
    q, q16 = _c_array(text, "c_qcell"), _c_array(text, "g_qcell")
    assert len(lv) == 510 and lv0[0] == 0.0 and lv0[1:len(lv) + 1] == lv and len(lv0) % 4 == 0
    assert all(v == 0.0 for v in lv0[len(lv) + 1:])
    assert thr16[:len(thr)] == thr and len(thr16) % 4 == 0 and all(np.isinf(thr16[len(thr):]))
    assert q16[:len(q)] == q and len(q16) % 16 == 0
    # the pairs (t_c, t_c+1) of each width b >= 3 from pair 2^b - 8 on, c = 0 .. 2^b - 1
    pairs = _c_array(text, "g_thr_pairs")
    for b in range(3, 9):
        o = (1 << b) + b - 3          # width b's first threshold among the padded ones
        for c in range(1 << b):
            p = (1 << b) - 8 + c
            assert pairs[2 * p] == thr[o + c] and pairs[2 * p + 1] == thr[o + c + 1]
    assert np.isinf(thr[(1 << 8) + 8 - 3 + 255]) and np.isinf(pairs[2 * (504 - 1) + 1])
    for name, vals, per in (("LV0", lv0, 4), ("THR", thr16, 4), ("THR_PAIR", pairs, 4), ("QCELL", q16, 16)):
        assert f"#define TACTKV_{name}_VEC {len(vals) // per}" in text


# ------------------------------------------------------------------- occupancy and capacity ---
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_occupancy_of_an_oracle_payload(T, bits):
    """The library's occupancy report on a payload written by the oracle (no GPU needed)."""
    S, H, W, heads, D = 4, 6, 5, 1, 32
    x = np.random.default_rng(bits).standard_normal((S * H * W, heads, D))
    p, info = O.compress_unit(x, S, H, W, heads, D, bits, return_info=True)
    occ = T.tactkv_occupancy(p)
    N, n = S * H * W, heads * D
    assert occ["bins"] == N and occ["channels"] == n
    assert occ["code_bits"] == int(info["b"].sum())
    assert occ["formula_bits"] == O.occupancy_bits(info["b"], n)
    assert occ["index_bits"] == O.index_bits(N)
    assert occ["payload_bytes"] == len(p)
    assert abs(occ["bits_per_element"] - 8 * len(p) / (N * n)) < 1e-12
    assert abs(occ["shrink_vs_bf16"] - 2 * N * n / len(p)) < 1e-12


def test_occupancy_with_per_head_gains(T):
    """With per-head gains the stage-4 sum runs over (bin, head) vectors of head_dim channels: one
    32-bit gain per bin and head."""
    S, H, W, heads, D = 4, 6, 5, 3, 32
    x = np.random.default_rng(3).standard_normal((S * H * W, heads, D))
    p, info = O.compress_unit(x, S, H, W, heads, D, 2, return_info=True, flags=O.FLAG_HEAD_GAIN)
    occ = T.tactkv_occupancy(p)
    assert occ["formula_bits"] == O.occupancy_bits(info["b"], D, heads)
    assert occ["payload_bytes"] == len(p)
    assert occ["formula_bits"] - O.occupancy_bits(info["b"], heads * D) == 32 * (heads - 1) * S * H * W


@pytest.mark.parametrize("flags", [0, 128])
def test_payload_size_is_the_occupancy_formula_plus_header_index_and_padding(T, flags):
    """Stage 4's relation on real payloads: the payload's bytes are the formula's bits (codes and
    32-bit gains), the 64-byte header, one byte of bit width per bin, and nothing but the padding
    of each part to 16 bytes."""
    def pad16(v):
        return (v + 15) // 16 * 16
    S, H, W, heads, D = 3, 5, 6, 2, 32
    N, n = S * H * W, heads * D
    for bits in (1, 3, 8):
        x = np.random.default_rng(bits).standard_normal((N, heads, D))
        p = O.compress_unit(x, S, H, W, heads, D, bits, flags=flags)
        occ = T.tactkv_occupancy(p)
        g = heads if flags & 128 else 1
        stride = pad16((occ["code_bits"] + 7) // 8)
        padding_bits = 8 * (pad16(N) - N) + 8 * (pad16(4 * N * g) - 4 * N * g) + n * (8 * stride - occ["code_bits"])
        assert 8 * occ["payload_bytes"] == 8 * 64 + occ["index_bits"] + occ["formula_bits"] + padding_bits


def test_occupancy_rejects_corrupt_payloads(T):
    S, H, W, heads, D = 4, 6, 5, 1, 32
    p = bytearray(O.compress_unit(np.ones((S * H * W, heads, D)), S, H, W, heads, D, 2))
    bad = bytearray(p)
    bad[0] ^= 1                                      # magic
    with pytest.raises(T.TactkvError):
        T.tactkv_occupancy(bytes(bad))
    bad = bytearray(p)
    bad[64] = 9                                      # a bit width above 8
    with pytest.raises(T.TactkvError):
        T.tactkv_occupancy(bytes(bad))
    bad = bytearray(p)
    bad[64] = (bad[64] + 1) % 9 if bad[64] < 8 else 7  # widths no longer sum to the header's code_bits
    with pytest.raises(T.TactkvError):
        T.tactkv_occupancy(bytes(bad))


def test_max_batch_and_capacity(T):
    assert T.tactkv_max_batch(100, 30, 7) == O.max_batch(100, 30, 7) == 10
    assert T.tactkv_max_batch(10, 20, 1) == 0 and T.tactkv_max_batch(10, 0, 0) == -1
    cap = T.batch_capacity(hbm_bytes=1000, fixed_bytes=200, payload_bytes_per_request=10,
                           text_kv_bytes_per_request=6, visual_kv_bf16_bytes_per_request=154)
    assert cap == {"batch_bf16": 5, "batch_compressed": 50, "cache_shrink": 10.0}
