#!/usr/bin/env python3
"""Generate straight-line CUDA code for orthonormal DCT-II / DCT-III pencils of fixed length.

Build step of the CUDA library (it writes ``dct_gen.cuh`` next to this file).  The transforms
are those of the TACT-KV methodology's stage 2 (separable orthonormal DCT-II along S, H and W)
and their inverses for decoding.  The oracle does not use this file.

Algorithm (for the un-normalised Z[k] = sum_t x[t] cos(pi (2t+1) k / (2L))):
  * even L: u[t] = x[t] + x[L-1-t], v[t] = x[t] - x[L-1-t] (t < L/2); the even outputs are the
    length-L/2 DCT-II of u and the odd outputs Z[2k+1] are the length-L/2 DCT-IV of v;
  * the DCT-IV halves and odd-length DCT-IIs: the definition, one multiply-add per term.
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


def dct4_unnorm(g: Graph, v: List[int]) -> List[int]:
    """DCT-IV by its definition.  (The shorter route through a pre-scaled DCT-II and the running
    difference Y[k] = Z'[k] - Y[k-1] carries the rounding error of the large low-frequency terms
    into the small high-frequency ones and is ~14x less accurate in float32, too much for the
    code-level parity the codec needs.)"""
    M = len(v)
    return dense(g, v, lambda k, t: math.cos(math.pi * (2 * t + 1) * (2 * k + 1) / (4 * M)))


def dense(g: Graph, x: List[int], coef) -> List[int]:
    L = len(x)
    out = []
    for k in range(L):
        acc = g.scale(x[0], coef(k, 0))
        for t in range(1, L):
            c = coef(k, t)
            if abs(c) < 1e-15:
                continue
            acc = g.lin([(c, x[t]), (1.0, acc)])
        out.append(acc)
    return out


def build_forward(L: int) -> Tuple[Graph, List[int]]:
    g = Graph(L)
    Z = dct2_unnorm(g, list(range(L)))
    out = [g.scale(Z[k], math.sqrt((1.0 if k == 0 else 2.0) / L)) for k in range(L)]
    return g, out


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
    """Adjoint program: inputs are the forward outputs' adjoints, outputs the inputs' adjoints."""
    L = len(outs)
    tg = Graph(L)
    adj: Dict[int, int] = {}

    def acc(node: int, src: int, c: float):
        if node not in adj:
            adj[node] = src if c == 1.0 else tg.scale(src, c)
        else:
            adj[node] = tg.lin([(1.0, adj[node]), (c, src)])     # one fused statement

    for j, o in enumerate(outs):
        acc(o, j, 1.0)
    for idx in range(len(g.ops) - 1, g.n_in - 1, -1):
        if idx not in adj:
            continue
        a = adj.pop(idx)
        for c, s in g.ops[idx]:
            acc(s, a, c)
    return tg, [adj[i] for i in range(g.n_in)]


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
