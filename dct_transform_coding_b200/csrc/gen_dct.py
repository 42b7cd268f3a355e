#!/usr/bin/env python3
"""Generate straight-line CUDA code for orthonormal DCT-II / DCT-III pencils of fixed length.

Build step of the CUDA library (it writes ``dct_gen.cuh`` next to this file).  The transforms
are those of the TACT-KV methodology's stage 2 (separable orthonormal DCT-II along S, H and W)
and their inverses for decoding.  The oracle does not use this file.

Algorithm (for the un-normalised Z[k] = sum_t x[t] cos(pi (2t+1) k / (2L))):
  * even L: u[t] = x[t] + x[L-1-t], v[t] = x[t] - x[L-1-t] (t < L/2); the even outputs are the
    length-L/2 DCT-II of u and the odd outputs Z[2k+1] are the length-L/2 DCT-IV of v;
  * DCT-IV halves of power-of-two length >= 8: pre-twiddle, complex FFT of half the length,
    post-twiddle (see dct4_unnorm); other DCT-IV halves and odd-length DCT-IIs: the definition.
Orthonormal scaling a_0 = sqrt(1/L), a_k = sqrt(2/L) is applied to the outputs.  The inverse
(DCT-III) is emitted as the exact transpose of the forward flow graph (reverse-mode accumulation
of the same linear statements), so forward and inverse use the same constants.

Every generated program is checked here in float64 against the cosine definition before it
is written.
"""
from __future__ import annotations

import math
import os
import sys
from typing import Dict, List, Tuple

import numpy as np

FAST_LENGTHS = list(range(1, 17)) + [20, 24, 28, 32, 40, 48, 56, 64]


class Graph:
    """Linear straight-line program: each node is sum_j c_j * node_j (one or two terms)."""

    def __init__(self, n_in: int):
        self.ops: List[List[Tuple[float, int]]] = [[] for _ in range(n_in)]   # inputs: no terms
        self.n_in = n_in

    def lin(self, terms: List[Tuple[float, int]]) -> int:
        terms = [(c, s) for c, s in terms if c != 0.0]
        assert 1 <= len(terms) <= 2
        if len(terms) == 1 and terms[0][0] == 1.0:
            return terms[0][1]
        self.ops.append(terms)
        return len(self.ops) - 1

    def add(self, a, b):
        return self.lin([(1.0, a), (1.0, b)])

    def sub(self, a, b):
        return self.lin([(1.0, a), (-1.0, b)])

    def scale(self, a, c):
        return self.lin([(c, a)])


def dct2_unnorm(g: Graph, x: List[int]) -> List[int]:
    L = len(x)
    if L == 1:
        return [x[0]]
    if L % 2 == 0:
        h = L // 2
        u = [g.add(x[t], x[L - 1 - t]) for t in range(h)]
        v = [g.sub(x[t], x[L - 1 - t]) for t in range(h)]
        E = dct2_unnorm(g, u)
        O = dct4_unnorm(g, v)
        out = [None] * L
        for k in range(h):
            out[2 * k] = E[k]
            out[2 * k + 1] = O[k]
        return out
    return dense(g, x, lambda k, t: math.cos(math.pi * (2 * t + 1) * k / (2 * L)))


def cmul_const(g: Graph, z, w: complex):
    """z * w for a complex constant w (z a pair of nodes)."""
    a, b = z
    c, d = w.real, w.imag
    if abs(d) < 1e-15 and abs(c - 1) < 1e-15:
        return z
    if abs(c) < 1e-15:                                  # w = i d: (a + ib) i d = -b d + i a d
        return (g.scale(b, -d), g.scale(a, d))
    if abs(d) < 1e-15:
        return (g.scale(a, c), g.scale(b, c))
    return (g.lin([(c, a), (-d, b)]), g.lin([(d, a), (c, b)]))


def fft(g: Graph, z, sign: int):
    """Z[p] = sum_m z[m] exp(sign 2 pi i m p / M), radix 2 (len(z) a power of two)."""
    M = len(z)
    if M == 1:
        return list(z)
    E = fft(g, z[0::2], sign)
    O = fft(g, z[1::2], sign)
    out = [None] * M
    for p in range(M // 2):
        t = cmul_const(g, O[p], complex(math.cos(2 * math.pi * p / M), sign * math.sin(2 * math.pi * p / M)))
        out[p] = (g.add(E[p][0], t[0]), g.add(E[p][1], t[1]))
        out[p + M // 2] = (g.sub(E[p][0], t[0]), g.sub(E[p][1], t[1]))
    return out


def dct4_unnorm(g: Graph, v: List[int]) -> List[int]:
    """DCT-IV, Y[k] = sum_t v[t] cos(pi (2t+1)(2k+1) / (4N)).

    N a power of two >= 8: with a_m = v[2m], b_m = v[N-1-2m] (m < N/2),
        sum_m (a_m - i b_m) exp(i pi (4m+1)(4p+1) / (4N)) = Y[2p] + i Y[N-1-2p],
    and the exponent splits into exp(i pi m/N) (pre-twiddle), exp(2 pi i m p / (N/2)) (an
    N/2-point DFT, by FFT) and exp(i pi (p + 1/4)/N) (post-twiddle).  Every step is a rotation or
    a butterfly, so float32 rounding stays at the level of the dense product.  Other lengths: the
    definition.  (The shorter route through a pre-scaled DCT-II and the running difference
    Y[k] = Z'[k] - Y[k-1] carries the rounding error of the large low-frequency terms into the
    small high-frequency ones and is ~14x less accurate in float32: not used.)"""
    N = len(v)
    if N >= 8 and N & (N - 1) == 0:
        M = N // 2
        d = []
        for m in range(M):
            a, b = v[2 * m], v[N - 1 - 2 * m]
            al = math.pi * m / N
            ca, sa = math.cos(al), math.sin(al)
            if m == 0:
                d.append((a, g.scale(b, -1.0)))
            else:                                       # (a - i b)(cos al + i sin al)
                d.append((g.lin([(ca, a), (sa, b)]), g.lin([(sa, a), (-ca, b)])))
        D = fft(g, d, +1)
        Y = [None] * N
        for p in range(M):
            be = math.pi * (p + 0.25) / N
            re, im = cmul_const(g, D[p], complex(math.cos(be), math.sin(be)))
            Y[2 * p] = re
            Y[N - 1 - 2 * p] = im
        return Y
    return dense(g, v, lambda k, t: math.cos(math.pi * (2 * t + 1) * (2 * k + 1) / (4 * N)))


def dense(g: Graph, x: List[int], coef) -> List[int]:
    """Matrix-vector product, emitted term-major: every output advances by one multiply-add per
    step, so neighbouring statements are independent (L chains in flight, not one)."""
    L = len(x)
    acc = [g.scale(x[0], coef(k, 0)) for k in range(L)]
    for t in range(1, L):
        for k in range(L):
            c = coef(k, t)
            if abs(c) < 1e-15:
                continue
            acc[k] = g.lin([(c, x[t]), (1.0, acc[k])])
    return acc


def build_forward(L: int) -> Tuple[Graph, List[int]]:
    """Forward orthonormal DCT-II flow graph.  The recursion is built once, then transposed twice:
    the second transpose computes the same map with the scale factors folded into the
    multiply-adds (see transpose_graph), a few percent fewer statements."""
    g = Graph(L)
    Z = dct2_unnorm(g, list(range(L)))
    out = [g.scale(Z[k], math.sqrt((1.0 if k == 0 else 2.0) / L)) for k in range(L)]
    tg, touts = transpose_graph(g, out)
    return transpose_graph(tg, touts)


def evaluate(g: Graph, outs: List[int], x: np.ndarray, dtype=np.float64) -> np.ndarray:
    val: Dict[int, np.ndarray] = {}
    for i in range(g.n_in):
        val[i] = x[i].astype(dtype)
    for idx in range(g.n_in, len(g.ops)):
        terms = g.ops[idx]
        if len(terms) == 1:
            c, s = terms[0]
            val[idx] = (dtype(c) * val[s]).astype(dtype)
        else:
            (c1, s1), (c2, s2) = terms
            val[idx] = (dtype(c1) * val[s1] + dtype(c2) * val[s2]).astype(dtype)
    return np.stack([val[o] for o in outs])


def dct_matrix(L: int) -> np.ndarray:
    k = np.arange(L)[:, None]
    t = np.arange(L)[None, :]
    C = np.cos(np.pi * (2 * t + 1) * k / (2 * L)) * np.sqrt(2.0 / L)
    C[0] /= math.sqrt(2.0)
    return C


# ------------------------------------------------------------------------------ emission ---
def _fmt(c: float) -> str:
    return repr(float(np.float32(c))) + "f"


def emit_program(g: Graph, inputs: List[str], outs: List[int], out_names: List[str]) -> List[str]:
    """Emit statements computing `outs` from `inputs` (names of V lvalues)."""
    lines: List[str] = []
    name = {i: inputs[i] for i in range(g.n_in)}
    # materialise each op once into a fresh temporary
    for idx in range(g.n_in, len(g.ops)):
        terms = g.ops[idx]
        t = f"t{idx}"
        if len(terms) == 1:
            c, s = terms[0]
            if c == -1.0:
                lines.append(f"const V {t} = vneg({name[s]});")
            else:
                lines.append(f"const V {t} = vmul({name[s]}, {_fmt(c)});")
        else:
            (c1, s1), (c2, s2) = terms
            if c1 == 1.0 and c2 == 1.0:
                lines.append(f"const V {t} = vadd({name[s1]}, {name[s2]});")
            elif c1 == 1.0 and c2 == -1.0:
                lines.append(f"const V {t} = vsub({name[s1]}, {name[s2]});")
            elif c1 == -1.0 and c2 == 1.0:
                lines.append(f"const V {t} = vsub({name[s2]}, {name[s1]});")
            elif c2 == 1.0:
                lines.append(f"const V {t} = vfma({name[s1]}, {_fmt(c1)}, {name[s2]});")
            elif c1 == 1.0:
                lines.append(f"const V {t} = vfma({name[s2]}, {_fmt(c2)}, {name[s1]});")
            else:
                lines.append(f"const V {t} = vfma({name[s1]}, {_fmt(c1)}, vmul({name[s2]}, {_fmt(c2)}));")
        name[idx] = t
    for o, nm in zip(outs, out_names):
        lines.append(f"{nm} = {name[o]};")
    return lines


def transpose_graph(g: Graph, outs: List[int]) -> Tuple[Graph, List[int]]:
    """Adjoint program: inputs are the forward outputs' adjoints, outputs the inputs' adjoints.

    Adjoints are carried as (coefficient, node) pairs meaning coefficient * node, so a scale is
    only materialized when two contributions meet (c1 n1 + c2 n2 = c1 (n1 + (c2/c1) n2), one
    fused multiply-add) or at an output."""
    L = len(outs)
    tg = Graph(L)
    adj: Dict[int, List[Tuple[float, int]]] = {}

    def combine(terms: List[Tuple[float, int]]) -> Tuple[float, int]:
        c0, n0 = terms[0]
        for c, n in terms[1:]:
            n0 = tg.lin([(1.0, n0), (c / c0, n)])
        return c0, n0

    for j, o in enumerate(outs):
        adj.setdefault(o, []).append((1.0, j))
    for idx in range(len(g.ops) - 1, g.n_in - 1, -1):
        if idx not in adj:
            continue
        c, n = combine(adj.pop(idx))
        for cop, src in g.ops[idx]:
            adj.setdefault(src, []).append((c * cop, n))
    res = []
    for i in range(g.n_in):
        c, n = combine(adj[i])
        res.append(n if c == 1.0 else tg.scale(n, c))
    return tg, res


def generate(lengths=FAST_LENGTHS) -> str:
    rng = np.random.default_rng(0)
    parts = [
        "// Generated by gen_dct.py -- do not edit.  Orthonormal DCT-II (forward) and DCT-III",
        "// (inverse, the exact transpose of the forward flow graph) of fixed-length pencils held",
        "// in registers.  V is a value type with vadd/vsub/vneg/vmul(V, float)/vfma(V, float, V).",
        "#pragma once",
        "",
    ]
    stats = []
    for L in lengths:
        g, outs = build_forward(L)
        C = dct_matrix(L)
        x = rng.standard_normal((L, 8))
        err_f = np.max(np.abs(evaluate(g, outs, x) - C @ x))
        tg, touts = transpose_graph(g, outs)
        err_i = np.max(np.abs(evaluate(tg, touts, x) - C.T @ x))
        if err_f > 1e-12 or err_i > 1e-12:
            raise SystemExit(f"generated DCT of length {L} is wrong: {err_f} {err_i}")
        names = [f"x[{i}]" for i in range(L)]
        body_f = emit_program(g, names, outs, names)
        body_i = emit_program(tg, names, touts, names)
        stats.append((L, len(g.ops) - L, len(tg.ops) - L))
        for nm, body in (("fdct", body_f), ("idct", body_i)):
            parts.append(f"template <class V> __device__ __forceinline__ void {nm}_{L}(V* x) {{")
            parts.extend("  " + ln for ln in body)
            parts.append("}")
        parts.append("")
    parts.append("// ops per pencil (forward, inverse): " + ", ".join(f"{L}:{a}/{b}" for L, a, b in stats))
    parts.append(f"#define TACTKV_FAST_LENGTHS {', '.join(str(L) for L in lengths)}")
    return "\n".join(parts) + "\n"


if __name__ == "__main__":
    here = os.path.dirname(os.path.abspath(__file__))
    out = sys.argv[1] if len(sys.argv) > 1 else os.path.join(here, "dct_gen.cuh")
    text = generate()
    with open(out, "w") as f:
        f.write(text)
    print(f"wrote {out} ({len(text.splitlines())} lines)")
