#!/usr/bin/env python3
"""Generate the CUDA library's fixed Lloyd-Max codebooks (build step; writes lloyd_max_tables.inc).

TACT-KV quantizes every coordinate of a surviving bin with a fixed Lloyd-Max codebook chosen by
the bin's bit width ("Methodology in Plain English", stage 4).  The codebook is the minimum-MSE
scalar quantizer of a unit Gaussian with 2^b levels, b = 1..8: every level is the centroid of
its cell and every threshold the midpoint of two neighbouring levels.

This generator works on the non-negative half only (the optimum is odd-symmetric; for an even
number of levels the middle threshold is 0).  Unknowns are the M = 2^(b-1) positive levels
y_1 < ... < y_M with cell edges e_0 = 0, e_j = (y_j + y_{j+1}) / 2, e_M = +inf.  It starts from
the companding approximation (levels at the quantiles of N(0, 3)), runs Lloyd updates, and
then solves G(y) = y - centroid(y) = 0 by Newton's method with the tridiagonal Jacobian and a
Thomas solve, in plain Python floats.  Tail probabilities use erfc on the cell's own side.
"""
from __future__ import annotations

import math
import os
import struct
import sys

INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def pdf(x: float) -> float:
    return 0.0 if math.isinf(x) else math.exp(-0.5 * x * x) * INV_SQRT_2PI


def upper(x: float) -> float:
    """P(Z > x)."""
    return 0.0 if x == math.inf else 0.5 * math.erfc(x / math.sqrt(2.0))


def inv_upper(p: float) -> float:
    """x with P(Z > x) = p, 0 < p <= 1/2, by bisection."""
    lo, hi = 0.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if upper(mid) > p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def cells(y):
    M = len(y)
    e = [0.0] + [0.5 * (y[j] + y[j + 1]) for j in range(M - 1)] + [math.inf]
    out = []
    for j in range(M):
        a, b = e[j], e[j + 1]
        mass = upper(a) - upper(b)
        out.append((a, b, mass, (pdf(a) - pdf(b)) / mass))
    return out


def solve_tridiag(lo, di, up, rhs):
    n = len(di)
    c = [0.0] * n
    d = [0.0] * n
    c[0] = up[0] / di[0] if n > 1 else 0.0
    d[0] = rhs[0] / di[0]
    for i in range(1, n):
        m = di[i] - lo[i] * c[i - 1]
        c[i] = up[i] / m if i < n - 1 else 0.0
        d[i] = (rhs[i] - lo[i] * d[i - 1]) / m
    x = [0.0] * n
    x[-1] = d[-1]
    for i in range(n - 2, -1, -1):
        x[i] = d[i] - c[i] * x[i + 1]
    return x


def codebook(bits: int):
    M = 1 << (bits - 1)
    L = 2 * M
    # companding start: positive quantiles of N(0, 3) at probabilities (M + j + 1/2) / L
    y = [math.sqrt(3.0) * inv_upper(1.0 - (M + j + 0.5) / L) for j in range(M)]
    for _ in range(100):
        y = [c[3] for c in cells(y)]
    for _ in range(100):
        cs = cells(y)
        G = [y[j] - cs[j][3] for j in range(M)]
        if max(abs(g) for g in G) < 1e-15:
            break
        lo = [0.0] * M
        di = [1.0] * M
        up = [0.0] * M
        for j, (a, b, mass, cen) in enumerate(cs):
            da = pdf(a) * (cen - a) / mass          # d centroid / d lower edge
            db = 0.0 if math.isinf(b) else pdf(b) * (b - cen) / mass
            if j > 0:                                # a = (y_{j-1} + y_j) / 2; the edge at 0 is fixed
                lo[j] -= 0.5 * da
                di[j] -= 0.5 * da
            if j < M - 1:                            # b = (y_j + y_{j+1}) / 2
                di[j] -= 0.5 * db
                up[j] -= 0.5 * db
        step = solve_tridiag(lo, di, up, G)
        y = [y[j] - step[j] for j in range(M)]
    levels = [-v for v in reversed(y)] + y
    thresholds = [0.5 * (levels[j] + levels[j + 1]) for j in range(L - 1)]
    return levels, thresholds


def f32(v: float) -> str:
    """C float literal of float32(v), rounded to nearest even (exact as printed)."""
    return repr(struct.unpack("<f", struct.pack("<f", v))[0]) + "f"


# Code lookup for b >= 3.  The range [-G, G) of u is cut into K equal cells; cell j of u is
# clamp(floor(fmaf(u, QSCALE, QOFFSET)), 0, K-1) in float32.  The table holds, per cell, the
# number c of thresholds below the cell's lower edge minus DELTA; the code of u is then
# c + [u >= t_c] + [u >= t_{c+1}], exact as long as every cell, widened by DELTA on both sides,
# holds at most two thresholds (checked here).  DELTA covers the float32 rounding of the cell
# index (|error| < 1e-4 cell widths).  Thresholds are padded with two +inf after the last one.
QK = 512
QG = 4.5
QDELTA = 1e-4


def f32v(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def code_table(th32):
    """Per-cell count of thresholds below (cell edge - DELTA), with the two-threshold check."""
    scale = f32v(QK / (2.0 * QG))
    offset = f32v(QK / 2.0)
    out = []
    for j in range(QK):
        lo = (j - offset) / scale
        hi = (j + 1 - offset) / scale
        c = sum(1 for t in th32 if t < lo - QDELTA)
        if j == 0:
            inside = [t for t in th32 if t < hi + QDELTA]
        elif j == QK - 1:
            inside = [t for t in th32 if t >= lo - QDELTA]
        else:
            inside = [t for t in th32 if lo - QDELTA <= t < hi + QDELTA]
        assert len(inside) <= 2, (len(th32), j, inside)
        assert c <= 255
        out.append(c)
    return out, scale, offset


def generate() -> str:
    lv_all, th_all, lv_off, th_off = [], [], [], []
    for b in range(1, 9):
        lv, th = codebook(b)
        lv_off.append(len(lv_all))
        th_off.append(len(th_all))
        lv_all += lv
        th_all += th
    lines = ["// Generated by gen_tables.py -- do not edit.  Lloyd-Max codebooks of N(0,1), 1..8 bits.",
             "#pragma once",
             f"#define TACTKV_LM_LEVELS_TOTAL {len(lv_all)}",
             f"#define TACTKV_LM_THRESH_TOTAL {len(th_all)}",
             "static const int kLmLevelOffset[9] = {" + ", ".join(map(str, lv_off + [len(lv_all)])) + "};",
             "static const int kLmThreshOffset[9] = {" + ", ".join(map(str, th_off + [len(th_all)])) + "};",
             "static const double kLmLevels[] = {"]
    lines += ["  " + ", ".join(repr(v) for v in lv_all[i:i + 4]) + "," for i in range(0, len(lv_all), 4)]
    lines += ["};", "static const double kLmThresholds[] = {"]
    lines += ["  " + ", ".join(repr(v) for v in th_all[i:i + 4]) + "," for i in range(0, len(th_all), 4)]
    lines += ["};", "#ifdef __CUDACC__", "static __constant__ float c_lm_levels[] = {"]
    lines += ["  " + ", ".join(f32(v) for v in lv_all[i:i + 4]) + "," for i in range(0, len(lv_all), 4)]
    lines += ["};", "static __constant__ float c_lm_thresholds[] = {"]
    lines += ["  " + ", ".join(f32(v) for v in th_all[i:i + 4]) + "," for i in range(0, len(th_all), 4)]
    lines += ["};"]
    # thresholds of each width followed by two +inf (width b starts at 2^b + b - 3), and the
    # per-cell code table for b >= 3
    pad_all, qtab = [], []
    for b in range(1, 9):
        th32 = [f32v(v) for v in th_all[th_off[b - 1]:th_off[b - 1] + (1 << b) - 1]]
        assert len(pad_all) == (1 << b) + b - 3
        pad_all += th32 + [math.inf, math.inf]
        if b >= 3:
            tab, scale, offset = code_table(th32)
            qtab += tab
    lines += [f"#define TACTKV_LM_T2 {f32(th_all[th_off[1] + 2])}   // the positive 2-bit threshold",
              f"#define TACTKV_Q_CELLS {QK}",
              f"#define TACTKV_Q_SCALE {f32(scale)}",
              f"#define TACTKV_Q_OFFSET {f32(offset)}",
              f"#define TACTKV_THR_PAD_TOTAL {len(pad_all)}",
              "static __constant__ float c_thr_pad[] = {"]
    lit = lambda v: "INFINITY" if math.isinf(v) else f32(v)
    lines += ["  " + ", ".join(lit(v) for v in pad_all[i:i + 4]) + "," for i in range(0, len(pad_all), 4)]
    lines += ["};", "static __constant__ unsigned char c_qcell[] = {"]
    lines += ["  " + ", ".join(str(v) for v in qtab[i:i + 32]) + "," for i in range(0, len(qtab), 32)]
    lines += ["};"]
    # The same tables in global memory, 16-byte aligned and padded to whole 16-byte vectors, for
    # kernels that copy them to shared memory: thread i reads vector i, where a copy out of
    # constant memory would serialise the warp's 32 different addresses.  The levels get a zero
    # in front (index 0 stands for "no bits").
    lv0 = [0.0] + [f32v(v) for v in lv_all]
    lv0 += [0.0] * (-len(lv0) % 4)
    thr16 = pad_all + [math.inf] * (-len(pad_all) % 4)
    q16 = qtab + [0] * (-len(qtab) % 16)
    # for b >= 3, the pair (t_c, t_{c+1}) of padded thresholds for every count c = 0 .. 2^b - 1,
    # width b's pairs from pair 2^b - 8 on: the two compares after the cell lookup take one load
    pairs = []
    for b in range(3, 9):
        o = (1 << b) + b - 3
        assert len(pairs) == 2 * ((1 << b) - 8)
        for c in range(1 << b):
            pairs += [pad_all[o + c], pad_all[o + c + 1]]
    pairs += [math.inf] * (-len(pairs) % 4)
    lines += [f"#define TACTKV_LV0_VEC {len(lv0) // 4}",
              f"#define TACTKV_THR_VEC {len(thr16) // 4}",
              f"#define TACTKV_THR_PAIR_VEC {len(pairs) // 4}",
              f"#define TACTKV_QCELL_VEC {len(q16) // 16}",
              "static __device__ __align__(16) const float g_lm_levels0[] = {"]
    lines += ["  " + ", ".join(lit(v) for v in lv0[i:i + 4]) + "," for i in range(0, len(lv0), 4)]
    lines += ["};", "static __device__ __align__(16) const float g_thr_pad[] = {"]
    lines += ["  " + ", ".join(lit(v) for v in thr16[i:i + 4]) + "," for i in range(0, len(thr16), 4)]
    lines += ["};", "static __device__ __align__(16) const float g_thr_pairs[] = {"]
    lines += ["  " + ", ".join(lit(v) for v in pairs[i:i + 4]) + "," for i in range(0, len(pairs), 4)]
    lines += ["};", "static __device__ __align__(16) const unsigned char g_qcell[] = {"]
    lines += ["  " + ", ".join(str(v) for v in q16[i:i + 32]) + "," for i in range(0, len(q16), 32)]
    lines += ["};", "#endif", ""]
    return "\n".join(lines)


if __name__ == "__main__":
    here = os.path.dirname(os.path.abspath(__file__))
    out = sys.argv[1] if len(sys.argv) > 1 else os.path.join(here, "lloyd_max_tables.inc")
    with open(out, "w") as f:
        f.write(generate())
    print("wrote", out)
