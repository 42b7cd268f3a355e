"""Parity checks of the CUDA codec against the CPU oracle (shared by the GPU tests and smoke()).

Acceptance, per unit (the codec's stated tolerances, with the readings needed to apply them):
* bit allocations equal the oracle's exactly, with no tolerance.  The report gives the relative
  gap between the B-th and the (B+1)-th largest key sigma^2 4^-k of the oracle ("alloc_margin"):
  the GPU's variances come from float32 coefficients, so a gap of the order of 1e-7 could let the
  two sides order those keys differently; a failure names that case, it is not forgiven;
* quantization codes equal the oracle's, except where the oracle's scaled coefficient
  u = X / sigma lies within 1e-5 * max(1, |t|) of a decision threshold t (distance taken in
  sigma-scaled units, because the middle threshold is 0);
* reconstructions: ||y_gpu - y_ref|| / ||y_ref|| <= 1e-3, both rounded to the I/O type, where y_ref
  is the oracle's decode of the GPU's own payload (so the decoder is compared on identical codes).
  The end-to-end figure against the oracle's own payload is asserted as well whenever the two
  payloads hold identical codes; a code inside the band moves one coefficient by about one
  quantization step, which in a small unit is alone above 1e-3 (one coefficient of 20,000 is
  already a relative RMS near 7e-3), so with band codes present it is only reported;
* with TACTKV_NO_QUANT the round trip matches the input within 1e-5 relative RMS.
"""
from __future__ import annotations

import numpy as np

from oracle import tactkv_oracle as O

CODE_BAND = 1e-5
RECON_TOL = 1e-3
ROUNDTRIP_TOL = 1e-5
NEAR_TIE = 1e-6


def rel_rms(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))


def selection_threshold(var: np.ndarray, bits: int) -> float:
    """The B-th largest key sigma_i^2 4^-k of the oracle's allocation (inf if all active bins saturate)."""
    act = var > 0
    B = bits * var.size
    if 8 * int(act.sum()) <= B:
        return np.inf
    keys = (var[act][:, None] * 4.0 ** -np.arange(8)[None, :]).ravel()
    return float(np.partition(keys, keys.size - B)[keys.size - B])


def allocation_margin(var: np.ndarray, bits: int) -> float:
    """Relative gap (K_B - K_{B+1}) / K_B between the B-th and the (B+1)-th largest keys (inf when
    every active bin saturates or no key is left out): how far the oracle's selection is from a tie."""
    act = var > 0
    B = bits * var.size
    keys = np.sort((var[act][:, None] * 4.0 ** -np.arange(8)[None, :]).ravel())[::-1]
    if 8 * int(act.sum()) <= B or keys.size <= B:
        return np.inf
    return float((keys[B - 1] - keys[B]) / keys[B - 1])


def compare_unit(x: np.ndarray, gpu_payload: bytes, gpu_recon: np.ndarray, *, S, H, W, heads, head_dim, bits,
                 layer=0, kv=0, flags=0, io_round=O.to_bf16, report=None):
    """Check one unit.  x: the input exactly as the GPU saw it; gpu_recon: the GPU decode of gpu_payload."""
    pflags = flags & O.PAYLOAD_FLAGS
    no_quant = bool(pflags & O.FLAG_NO_QUANT)
    p_o, info = O.compress_unit(x, S, H, W, heads, head_dim, bits, layer=layer, kv=kv, return_info=True,
                                flags=pflags)
    g = O.parse_payload(gpu_payload)
    assert (g["layer"], g["kv"], g["S"], g["H"], g["W"], g["heads"], g["head_dim"], g["bits"]) == \
        (layer, kv, S, H, W, heads, head_dim, bits)
    assert g["flags"] == pflags
    N = S * H * W
    var = info["var"]
    # gains: float32(sqrt(sigma^2)) from fp32 coefficients and fp64 sums
    # (per-head gains: [heads, N], each head's gains against the same relative floor)
    sig_o = info["sigma"].astype(np.float64)
    sig_g = g["sigma"].astype(np.float64)
    assert sig_g.shape == sig_o.shape
    big = sig_o > 1e-6 * max(sig_o.max(), 1e-300)
    assert np.all(np.abs(sig_g[big] - sig_o[big]) <= 2e-5 * sig_o[big]), "gain mismatch"
    out = dict(alloc_margin=np.inf, code_mismatch_band=0, codes=0)
    if no_quant:
        Xg = g["streams"][:, :4 * N].copy().view("<f4").astype(np.float64).T
        assert rel_rms(Xg, info["X"]) <= ROUNDTRIP_TOL
    else:
        b_o, b_g = info["b"], g["b"]
        out["alloc_margin"] = allocation_margin(var, bits)
        differ = np.nonzero(b_o != b_g)[0]
        if differ.size:
            thr = selection_threshold(var, bits)
            near = sum(abs(var[i] * 4.0 ** -min(b_o[i], b_g[i]) / thr - 1) < NEAR_TIE for i in differ)
            raise AssertionError(f"allocation differs at {differ.size} bins (first {differ[0]}: oracle "
                                 f"{b_o[differ[0]]}, GPU {b_g[differ[0]]}); {near} of them decide a key within "
                                 f"{NEAR_TIE} of the selection threshold (float32 vs fp64 near-tie)")
        assert b_g.sum() == g["code_bits"]
        _, codes_g = O.codes_of(gpu_payload)
        codes_o = info["codes"]
        X = info["Xq"]                                  # the (rotated, when FLAG_ROTATE) coefficients coded
        same = np.nonzero((b_o == b_g) & (b_o > 0))[0]
        for i in same:
            bad = codes_g[i] != codes_o[i]
            out["codes"] += codes_o.shape[1]
            if bad.any():
                gain = np.repeat(sig_o[:, i], head_dim) if sig_o.ndim == 2 else np.full(X.shape[1], sig_o[i])
                u = np.divide(X[i, bad], gain[bad], out=np.zeros(int(bad.sum())), where=gain[bad] > 0)
                d = O.threshold_distance(u, int(b_o[i]))
                assert np.all(d <= CODE_BAND), f"code mismatch outside the band at bin {i}: {d.max()}"
                out["code_mismatch_band"] += int(bad.sum())
    y_o = io_round(O.decompress_unit(p_o)).reshape(gpu_recon.shape)
    err = rel_rms(gpu_recon, y_o)
    out["recon_rel_rms"] = err
    if no_quant or out["code_mismatch_band"] == 0:
        assert err <= (ROUNDTRIP_TOL if no_quant else RECON_TOL), f"reconstruction rel RMS {err}"
    if not no_quant:
        y_same = io_round(O.decompress_unit(gpu_payload)).reshape(gpu_recon.shape)
        err_same = rel_rms(gpu_recon, y_same)
        out["decode_rel_rms"] = err_same
        assert err_same <= RECON_TOL, f"decoder rel RMS {err_same} on the same payload"
    if report is not None:
        report.append(out)
    return out
