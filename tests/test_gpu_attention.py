"""GPU parity of decode-time attention over compressed K/V (the decoding paragraph after stage 4 of
"Methodology in Plain English": decoding inside the attention kernel, no reconstructed cache).

The GPU computes scores and outputs in the DCT domain from the payloads' codes; the oracle runs
plain softmax(q K^T / sqrt(D)) V on its own fp64 decompression of the SAME payloads, so the
comparison isolates the attention arithmetic.  Tolerance: 1e-4 of the largest output magnitude
(float32 sums over at most 256 channels, float32 3D DCTs of the score volume and of the
probabilities: errors of order 1e-6 relative in the scores, 1e-5 in the outputs).
"""
import numpy as np
import pytest
import torch

from oracle import tactkv_oracle as O
from dct_transform_coding_b200.workloads import make_unit

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from dct_transform_coding_b200 import tactkv as T

DEV = "cuda:0"
TOL = 1e-4


def _run(S, H, W, heads, D, G, bits, flags=0, units=2, qscale=1.0, seed=0, k=None, v=None):
    if k is None:
        k = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.85), nu=4.0, seed=seed + 2 * i, device=DEV)
                         for i in range(units)])
        v = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.85), nu=4.0, seed=seed + 2 * i + 1,
                                   device=DEV) for i in range(units)])
    layers = list(range(units))
    pk = T.compress(k, S, H, W, bits, layers=layers, kvs=[0] * units, flags=flags)
    pv = T.compress(v, S, H, W, bits, layers=layers, kvs=[1] * units, flags=flags)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed + 99)
    q = torch.randn((units, heads * G, D), generator=gen, device=DEV) * qscale
    out, m, l = T.attention_decode(q, pk, pv, S, H, W, bits, heads=heads, head_dim=D, layers=layers, flags=flags,
                                   check=True)
    torch.cuda.synchronize()
    for i in range(units):
        o_ref, m_ref, l_ref = O.attention_decode(q[i].double().cpu().numpy(), pk[i].cpu().numpy().tobytes(),
                                                 pv[i].cpu().numpy().tobytes())
        o = out[i].double().cpu().numpy()
        assert np.max(np.abs(o - o_ref)) <= TOL * np.max(np.abs(o_ref)), np.max(np.abs(o - o_ref))
        assert np.allclose(m[i].double().cpu().numpy(), m_ref, rtol=TOL, atol=TOL)
        assert np.allclose(l[i].double().cpu().numpy(), l_ref, rtol=10 * TOL)
    return out


@pytest.mark.parametrize("S,H,W,heads,D,G,bits", [
    (8, 8, 8, 1, 64, 1, 2),
    (16, 16, 16, 2, 64, 4, 1),
    (5, 7, 6, 2, 32, 3, 3),        # ragged grid
    (64, 16, 16, 4, 256, 2, 1),    # the 4B-class medical layout (one layer)
    (4, 24, 24, 2, 128, 4, 2),     # the 32B-class slab (24 x 24 cells, 128 channels per head)
    (8, 8, 8, 1, 64, 8, 2),        # eight query heads per K/V head (the wide values kernel)
    (8, 32, 32, 1, 256, 2, 1),     # the largest slab, 256 channels: rows fit only at a low rate
])
def test_attention_matches_oracle(S, H, W, heads, D, G, bits):
    _run(S, H, W, heads, D, G, bits)


@pytest.mark.parametrize("flags", [64, 4 | 32, 128, 128 | 64],
                         ids=["rotate", "skip_s_uniform", "head_gain", "head_gain_rotate"])
def test_attention_with_variant_flags(flags):
    _run(16, 8, 8, 2, 64, 2, 2, flags=flags, seed=5)


def test_attention_reads_slabs_too_wide_to_stage():
    """A slab whose codes span more stream words than the shared-memory rows hold (sized for
    2 * bits + 2 bits per bin) is decoded from the payload in global memory.  K and V constant along
    S put the whole budget into the first slab: 8 bits per bin there at 2 bits per element over 4
    slabs, 64 words per channel against rows of 51."""
    S, H, W, heads, D, G, bits, units = 4, 16, 16, 2, 64, 2, 2, 2
    gen = torch.Generator(device=DEV).manual_seed(23)

    def flat_along_s():
        one = torch.randn((units, 1, H * W, heads, D), generator=gen, device=DEV)
        return one.expand(units, S, H * W, heads, D).reshape(units, S * H * W, heads, D).to(torch.bfloat16)

    k, v = flat_along_s(), flat_along_s()
    _run(S, H, W, heads, D, G, bits, units=units, k=k, v=v, seed=23)
    pk = T.compress(k, S, H, W, bits, layers=[0, 1], kvs=[0, 0])
    b = O.parse_payload(pk[0].cpu().numpy().tobytes())["b"].reshape(S, H * W)
    assert b[0].sum() == 8 * H * W and b[1:].sum() == 0   # the first slab takes every bit


def test_attention_sharp_scores():
    """Large query norms make the softmax nearly one-hot: the max-subtraction must hold up."""
    _run(8, 8, 8, 1, 64, 2, 4, qscale=8.0, seed=11)


def test_attention_corrupt_unit_contributes_no_tokens():
    """A unit whose K (or V) payload is corrupt is reported as TACTKV_CORRUPT_PAYLOAD and contributes
    no tokens (out = 0, m = -inf, l = 0); the other units of the call are unaffected."""
    S, H, W, heads, D, G, bits, units = 8, 8, 8, 1, 64, 2, 2, 3
    k = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.85), nu=4.0, seed=40 + i, device=DEV)
                     for i in range(units)])
    v = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.85), nu=4.0, seed=50 + i, device=DEV)
                     for i in range(units)])
    layers = list(range(units))
    pk = T.compress(k, S, H, W, bits, layers=layers, kvs=[0] * units)
    pv = T.compress(v, S, H, W, bits, layers=layers, kvs=[1] * units)
    pk[1, 0] ^= 1                                   # unit 1: K magic broken
    pv[2, 64] = 9                                   # unit 2: a V bit width above 8
    q = torch.randn((units, heads * G, D), generator=torch.Generator(DEV).manual_seed(7), device=DEV)
    ku = T.make_units(None, S, H, W, bits, heads=heads, head_dim=D, payload=pk, layers=layers, kvs=[0] * units,
                      n_units=units)
    nbytes = T.tactkv_attention_workspace_bytes(ku, units, heads * G)
    ws = torch.zeros(nbytes + 256, dtype=torch.uint8, device=DEV)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + nbytes]
    out, m, l = T.attention_decode(q, pk, pv, S, H, W, bits, heads=heads, head_dim=D, layers=layers, workspace=ws)
    assert T.tactkv_device_status(ws.data_ptr(), ws.numel(), 0) == T.TACTKV_CORRUPT_PAYLOAD
    for i in (1, 2):
        assert not out[i].any() and not l[i].any() and torch.all(torch.isneginf(m[i]))
    o_ref, m_ref, l_ref = O.attention_decode(q[0].double().cpu().numpy(), pk[0].cpu().numpy().tobytes(),
                                             pv[0].cpu().numpy().tobytes())
    assert np.max(np.abs(out[0].double().cpu().numpy() - o_ref)) <= TOL * np.max(np.abs(o_ref))
