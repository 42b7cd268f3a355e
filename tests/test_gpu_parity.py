"""GPU parity of the CUDA codec (through the C ABI) against the CPU oracle.

Every case generates its input once (seeded), hands the same tensor to the CUDA path and to
the oracle, and applies the acceptance rules of tests/parity.py.  Sizes: small cases that span
several 32-channel chunks and S slabs with ragged (non power of two) axes, the exact shapes of
every benchmark workload on sampled units, and the degenerate inputs of the method.
"""
import numpy as np
import pytest
import torch

from oracle import tactkv_oracle as O
from dct_transform_coding_b200.workloads import WORKLOADS, make_unit, make_workload_unit

from parity import compare_unit, rel_rms

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from dct_transform_coding_b200 import tactkv as T

DEV = "cuda:0"


def _round_trip(x_dev, S, H, W, bits, layers=None, kvs=None, flags=0, workspace=None):
    U, _, heads, D = x_dev.shape
    pay = T.compress(x_dev, S, H, W, bits, layers=layers, kvs=kvs, flags=flags, workspace=workspace)
    out_dtype = x_dev.dtype
    y = T.decompress(pay, S, H, W, bits, heads=heads, head_dim=D, layers=layers, kvs=kvs, flags=flags,
                     dtype=out_dtype, workspace=workspace, check=True)
    torch.cuda.synchronize()
    return pay, y


def _check_batch(x_dev, S, H, W, bits, layers=None, kvs=None, flags=0, units=None, workspace=None):
    U, _, heads, D = x_dev.shape
    pay, y = _round_trip(x_dev, S, H, W, bits, layers, kvs, flags, workspace)
    fp32 = x_dev.dtype == torch.float32
    io_round = (lambda v: np.asarray(v, np.float32).astype(np.float64)) if fp32 else O.to_bf16
    reports = []
    for i in (range(U) if units is None else units):
        x = x_dev[i].double().cpu().numpy()
        gp = pay[i].cpu().numpy().tobytes()
        yr = y[i].double().cpu().numpy()
        compare_unit(x, gp, yr, S=S, H=H, W=W, heads=heads, head_dim=D, bits=bits,
                     layer=layers[i] if layers is not None else i, kv=kvs[i] if kvs is not None else 0,
                     flags=flags, io_round=io_round, report=reports)
    return reports, pay, y


# ------------------------------------------------------------------------------ small cases ---
def test_tiny_config_fp32_io():
    """The 8x8x8, 1 x 64, fp32, 2-bit oracle workload."""
    w = WORKLOADS["tiny"]
    x = make_workload_unit(w, 0, 0, 0, device=DEV)[None]
    reports, _, _ = _check_batch(x, w.S, w.H, w.W, 2)
    assert reports[0]["codes"] > 0


@pytest.mark.parametrize("shape,bits", [
    ((5, 7, 3, 2, 32), 3),      # ragged axes, two chunks
    ((12, 6, 10, 1, 96), 1),    # three chunks, odd-ish lengths
    ((16, 16, 16, 2, 64), 4),
    ((3, 14, 14, 4, 16), 2),    # the video grid's H, W with a short S; head_dim 16 < 32
    ((24, 5, 9, 1, 32), 8),     # 8 bits: every active bin saturates
    ((32, 2, 24, 1, 64), 2),    # S in the 32 class, W in the 32 class
    ((1, 1, 1, 1, 32), 5),      # a single token
    ((8, 14, 14, 1, 64), 3),    # fused three-axis kernels: S = 8 on the 14 x 14 grid
    ((32, 8, 8, 2, 32), 2),     # fused, S = 32 on the 8 x 8 grid
    ((64, 8, 8, 1, 32), 1),     # fused, S = 64 on the 8 x 8 grid
    ((16, 24, 24, 2, 64), 2),   # fused, S = 16 on the 24 x 24 grid (32-class H/W pencils)
    ((32, 24, 24, 1, 32), 1),   # fused, S = 32 on the 24 x 24 grid (the 32B-class medical layout)
    ((8, 24, 24, 1, 64), 4),    # fused, S = 8 on the 24 x 24 grid (one slab per CTA of the cluster)
    ((64, 24, 24, 1, 32), 2),   # S = 64 on the 24 x 24 grid: the separate transform kernels
    ((8, 16, 16, 2, 256), 2),   # 512 channels: the decode kernel with its channel count fixed
    ((8, 8, 8, 4, 256), 3),     # 1024 channels on the 8 x 8 grid, likewise
])
def test_small_shapes_bf16(shape, bits):
    S, H, W, heads, D = shape
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.8, 0.85), nu=4.0, seed=10 * i + bits, device=DEV)
                     for i in range(2)])
    reports, _, _ = _check_batch(x, S, H, W, bits, layers=[3, 4], kvs=[0, 1])
    assert all(r["recon_rel_rms"] <= 1e-3 for r in reports)


@pytest.mark.parametrize("bits,flags", [(1, 0), (8, 0), (2, 1)])
def test_maximum_grid(bits, flags):
    """S = 64 slabs of a 32 x 32 grid (the largest unit the codec takes): the shared-memory
    footprint of every kernel is at its largest here.  flags = 1 is TACTKV_NO_QUANT."""
    S, H, W, heads, D = 64, 32, 32, 1, 32
    x = make_unit(S, H, W, heads, D, rho=(0.95, 0.9, 0.9), nu=4.0, seed=7 + bits, device=DEV)[None]
    reports, _, _ = _check_batch(x, S, H, W, bits, flags=flags)
    assert reports[0]["recon_rel_rms"] <= (1e-5 if flags else 1e-3)


def test_no_quant_round_trip_is_lossless():
    S, H, W, heads, D = 16, 8, 12, 2, 32
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.9, 0.9), nu=4.0, seed=i, device=DEV) for i in range(3)])
    reports, pay, y = _check_batch(x, S, H, W, 2, flags=T.TACTKV_NO_QUANT)
    assert rel_rms(y.double().cpu(), x.double().cpu()) <= 1e-5
    # bf16 in, fp32 transform, bf16 out: all but the tiniest elements come back bit for bit
    # (an fp32 round-trip error of ~1e-7 can move a value of ~1e-5 across a bf16 rounding boundary)
    assert (y == x).double().mean().item() > 0.999


def test_no_quant_fp32_io():
    S, H, W, heads, D = 8, 8, 8, 1, 64
    x = make_unit(S, H, W, heads, D, rho=(0.9, 0.9, 0.9), seed=3, dtype=torch.float32, device=DEV)[None]
    _, _, y = _check_batch(x, S, H, W, 4, flags=T.TACTKV_NO_QUANT)
    assert rel_rms(y.double().cpu(), x.double().cpu()) <= 1e-6


@pytest.mark.parametrize("S,H,W", [(8, 6, 6), (8, 8, 8)])   # separate and fused transform kernels
def test_strided_input_and_output(S, H, W):
    """kv_in as a view into a larger [tokens, heads_total, head_dim] cache (only 2 of 4 heads)."""
    D = 32
    big = make_unit(S, H, W, 4, D, rho=(0.9, 0.9, 0.9), nu=4.0, seed=5, device=DEV)
    x = big[:, 1:3, :][None]                          # stride(2) = D, stride(1) = 4 * D
    assert not x.is_contiguous()
    reports, pay, y = _check_batch(x, S, H, W, 2)
    # decode into a strided output as well
    out_big = torch.zeros_like(big)[None]
    T.decompress(pay, S, H, W, 2, heads=2, head_dim=D, out=out_big[:, :, 1:3, :], check=True)
    torch.cuda.synchronize()
    assert torch.equal(out_big[0, :, 1:3, :], y[0])
    assert not out_big[0, :, 0, :].any() and not out_big[0, :, 3, :].any()


# --------------------------------------------------------------------------- degenerate inputs ---
def test_all_zero_input():
    S, H, W, heads, D = 8, 4, 4, 1, 32
    x = torch.zeros((1, S * H * W, heads, D), dtype=torch.bfloat16, device=DEV)
    pay, y = _round_trip(x, S, H, W, 2)
    p = O.parse_payload(pay[0].cpu().numpy().tobytes())
    assert p["code_bits"] == 0 and not p["b"].any() and not p["sigma"].any()
    assert not y.any()


def test_constant_field_keeps_dc():
    """A constant field has all its energy in the DC bin; the other bins hold only rounding noise
    (fp32 on the GPU, fp64 in the oracle) whose allocation is meaningless, so the DC allocation
    and the reconstruction are compared.  The DC coefficient scaled by its own gain is exactly 1
    in every channel, so even 8 bits leave the Lloyd-Max error of u = 1 (about 1%) on both sides."""
    S, H, W, heads, D = 8, 8, 8, 1, 32
    x = torch.full((1, S * H * W, heads, D), 0.75, dtype=torch.bfloat16, device=DEV)
    pay, y = _round_trip(x, S, H, W, 1)
    p = O.parse_payload(pay[0].cpu().numpy().tobytes())
    assert p["b"][0] == 8
    p_o = O.compress_unit(x[0].double().cpu().numpy(), S, H, W, heads, D, 1)
    assert O.parse_payload(p_o)["b"][0] == 8
    y_o = O.to_bf16(O.decompress_unit(p_o))
    assert rel_rms(y[0].double().cpu().numpy(), y_o) <= 1e-3
    assert rel_rms(y.double().cpu(), x.double().cpu()) < 0.02


# ---------------------------------------------------------------------- batching and waves ---
def test_many_units_and_small_workspace():
    """More units than one launch carries (256), processed again with a workspace of one unit."""
    S, H, W, heads, D = 4, 4, 4, 1, 32
    U = 260
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.8, 0.8, 0.8), seed=i, device=DEV) for i in range(U)])
    pay_a, y_a = _round_trip(x, S, H, W, 3)
    units = T.make_units(x, S, H, W, 3, heads=heads, head_dim=D, payload=pay_a)
    one = T.tactkv_workspace_bytes(units[:1])
    ws = torch.zeros(one + 256, dtype=torch.uint8, device=DEV)
    off = (-ws.data_ptr()) % 256
    pay_b, y_b = _round_trip(x, S, H, W, 3, workspace=ws[off:off + one])
    assert torch.equal(pay_a, pay_b) and torch.equal(y_a, y_b)
    _check_batch(x, S, H, W, 3, units=[0, 130, 256, 259])


def test_wave_splitting_and_launch_counts():
    """12 units in one wave (4 compress kernels: the 8 x 8 x 8 grid has the fused three-axis forward
    kernel; 3 decompress kernels) give the same payloads and outputs as 12 waves of one unit each
    (a one-unit workspace)."""
    S, H, W, heads, D = 8, 8, 8, 2, 32
    U = 12
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.8, 0.85), nu=4.0, seed=40 + i, device=DEV)
                     for i in range(U)])
    pay = T.compress(x, S, H, W, 2)
    assert T.tactkv_last_launches() == 4
    y = T.decompress(pay, S, H, W, 2, heads=heads, head_dim=D, check=False)
    assert T.tactkv_last_launches() == 3
    units = T.make_units(x, S, H, W, 2, heads=heads, head_dim=D, payload=pay)
    one = T.tactkv_workspace_bytes(units[:1])
    ws = torch.zeros(one + 256, dtype=torch.uint8, device=DEV)
    off = (-ws.data_ptr()) % 256
    pay1, y1 = _round_trip(x, S, H, W, 2, workspace=ws[off:off + one])
    assert T.tactkv_last_launches() == 3 * U
    torch.cuda.synchronize()
    assert torch.equal(pay, pay1) and torch.equal(y, y1)


def test_deterministic():
    S, H, W, heads, D = 16, 8, 8, 2, 64
    x = make_unit(S, H, W, heads, D, rho=(0.9, 0.9, 0.9), nu=4.0, seed=1, device=DEV)[None]
    a, _ = _round_trip(x, S, H, W, 2)
    b, _ = _round_trip(x, S, H, W, 2)
    assert torch.equal(a, b)


def test_cross_decode_oracle_payload_on_gpu():
    """The GPU decoder reads a payload written by the oracle (same format, independent writers)."""
    S, H, W, heads, D = 8, 6, 10, 1, 64
    x = make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.8), nu=4.0, seed=9, device=DEV)
    p_o = O.compress_unit(x.double().cpu().numpy(), S, H, W, heads, D, 3, layer=0, kv=0)
    cap = T.payload_capacity(S, H, W, heads, D, 3)
    pay = torch.zeros((1, (cap + 15) // 16 * 16), dtype=torch.uint8)
    pay[0, :len(p_o)] = torch.frombuffer(bytearray(p_o), dtype=torch.uint8)
    y = T.decompress(pay.to(DEV), S, H, W, 3, heads=heads, head_dim=D, layers=[0], kvs=[0], check=True)
    ref = O.to_bf16(O.decompress_unit(p_o))
    assert rel_rms(y[0].double().cpu().numpy(), ref) <= 1e-3


@pytest.mark.parametrize("shape,bits", [
    ((8, 8, 8, 1, 64), 2),     # two chunks: one channel per lane, one packing range
    ((8, 8, 8, 4, 32), 2),     # four chunks: four channels per lane, ranges of 256 records
    ((16, 8, 8, 4, 32), 1),    # likewise, more ranges at 1 bit
    ((16, 8, 8, 8, 32), 2),    # eight chunks: two CTAs of four channels per lane side by side
])
def test_payload_bytes_match_oracle_format(shape, bits):
    """Where allocations and codes agree, the GPU payload is byte-identical to the oracle's."""
    S, H, W, heads, D = shape
    x = make_unit(S, H, W, heads, D, rho=(0.9, 0.9, 0.9), nu=4.0, seed=21, device=DEV)[None]
    pay, _ = _round_trip(x, S, H, W, bits, layers=[0], kvs=[0])
    p_o, info = O.compress_unit(x[0].double().cpu().numpy(), S, H, W, heads, D, bits, return_info=True)
    g = pay[0].cpu().numpy().tobytes()[:len(p_o)]
    po = np.frombuffer(p_o, np.uint8)
    gg = np.frombuffer(g, np.uint8)
    lay = O.payload_layout(S * H * W, heads * D, int(info["b"].sum()))
    # header + bit allocation identical
    assert np.array_equal(gg[:lay["off_sigma"]], po[:lay["off_sigma"]])
    # code area: identical unless a code sits inside the tolerance band
    _, codes_g = O.codes_of(g)
    if np.array_equal(codes_g, info["codes"]):
        assert np.array_equal(gg[lay["off_codes"]:], po[lay["off_codes"]:])


@pytest.mark.parametrize("bits,flags", [(1, 0), (4, 0), (2, 64)])
def test_payload_independent_of_buffer_contents(bits, flags):
    """The packer clears the bit fields it owns in the stream words it shares with a neighbouring
    range instead of relying on zeroed memory: payload buffers filled with zeros, with ones and
    with random bytes give the same payload.  A benchmark-size unit (many packing ranges); flags 64
    (the rotation) takes the one-channel-per-lane packer."""
    S, H, W, heads, D = 64, 16, 16, 4, 256
    x = make_unit(S, H, W, heads, D, rho=(0.85, 0.9, 0.9), nu=4.0, seed=5 + bits, device=DEV)[None]
    cap = T.payload_capacity(S, H, W, heads, D, bits, flags)
    cap = (cap + 15) // 16 * 16
    fills = [torch.zeros((1, cap), dtype=torch.uint8, device=DEV),
             torch.full((1, cap), 255, dtype=torch.uint8, device=DEV),
             torch.randint(0, 256, (1, cap), dtype=torch.uint8, device=DEV,
                           generator=torch.Generator(device=DEV).manual_seed(bits))]
    outs = []
    for buf in fills:
        T.compress(x, S, H, W, bits, layers=[0], kvs=[0], flags=flags, payload=buf)
        torch.cuda.synchronize()
        outs.append(buf[0].cpu().numpy().tobytes())
    used = T.tactkv_occupancy(outs[0])["payload_bytes"]
    assert used > 0
    assert outs[1][:used] == outs[0][:used] and outs[2][:used] == outs[0][:used]


# ------------------------------------------------------------------------------- full sizes ---
@pytest.mark.parametrize("name,bits,pick", [
    ("med4b", 1, [0, 67]),
    ("med4b_b8", 2, [5, 300]),
    ("med4b_b8", 4, [77, 543]),
    ("med32b", 1, [0, 511]),
    ("video", 1, [0, 895]),
])
def test_full_size_sampled_units(name, bits, pick):
    """The benchmark workloads at full size: the whole batch is compressed and decompressed in the
    launch configuration the benchmark uses (one call, waves of up to 256 units, workspace sized
    by tactkv_workspace_bytes), and the oracle checks sampled units of it."""
    from dct_transform_coding_b200.workloads import make_batch
    w = WORKLOADS[name]
    all_units = list(w.units())
    x = make_batch(w, device=DEV)
    layers = [u[1] for u in all_units]
    kvs = [u[2] for u in all_units]
    pay, y = _round_trip(x, w.S, w.H, w.W, bits, layers=layers, kvs=kvs)
    heads, D = w.heads, w.head_dim
    fp32 = x.dtype == torch.float32
    io_round = (lambda v: np.asarray(v, np.float32).astype(np.float64)) if fp32 else O.to_bf16
    for u in pick:
        r = compare_unit(x[u].double().cpu().numpy(), pay[u].cpu().numpy().tobytes(), y[u].double().cpu().numpy(),
                         S=w.S, H=w.H, W=w.W, heads=heads, head_dim=D, bits=bits, layer=layers[u], kv=kvs[u],
                         io_round=io_round, report=[])
        print(name, bits, u, r)
    del x, y, pay
    torch.cuda.empty_cache()


# ------------------------------------------------------- tensor-core and CUDA-core S passes ---
@pytest.mark.parametrize("S,H,W", [(64, 16, 16), (32, 14, 14), (16, 8, 8)])
def test_tensor_core_and_cuda_core_s_pass_both_match_the_oracle(S, H, W):
    """With TACTKV_TC_S=1 the fused forward kernel runs its DCT along S on the tensor cores when
    one TMA tensor map can describe the whole wave (units evenly spaced in memory), and on the CUDA
    cores otherwise.  The same three units are compressed both ways (the second time listed in
    reverse memory order, which no single map describes) and both payloads must pass the oracle's
    acceptance rules (without the variable both runs take the CUDA-core form)."""
    heads, D = 2, 64
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.85), nu=4.0, seed=70 + i, device=DEV)
                     for i in range(3)])
    pay_tc, y_tc = _round_trip(x, S, H, W, 2, layers=[0, 1, 2], kvs=[0, 0, 0])
    cap = T.payload_capacity(S, H, W, heads, D, 2)
    pay_sm = torch.zeros((3, (cap + 15) // 16 * 16), dtype=torch.uint8, device=DEV)
    y_sm = torch.empty_like(x)
    cu = T.make_units(x, S, H, W, 2, heads=heads, head_dim=D, payload=pay_sm, layers=[0, 1, 2], kvs=[0, 0, 0])
    du = T.make_units(None, S, H, W, 2, heads=heads, head_dim=D, payload=pay_sm, out=y_sm, layers=[0, 1, 2],
                      kvs=[0, 0, 0], n_units=3)
    cu_rev = (T.tactkv_unit * 3)(*[cu[2 - i] for i in range(3)])
    ws = T.alloc_workspace(cu, DEV)
    sp = torch.cuda.current_stream().cuda_stream
    assert T.tactkv_compress(cu_rev, ws.data_ptr(), ws.numel(), sp) == T.TACTKV_OK
    assert T.tactkv_decompress(du, ws.data_ptr(), ws.numel(), sp) == T.TACTKV_OK
    assert T.tactkv_device_status(ws.data_ptr(), ws.numel(), sp) == T.TACTKV_OK
    torch.cuda.synchronize()
    for i in range(3):
        xi = x[i].double().cpu().numpy()
        for pay, y in ((pay_tc, y_tc), (pay_sm, y_sm)):
            compare_unit(xi, pay[i].cpu().numpy().tobytes(), y[i].double().cpu().numpy(), S=S, H=H, W=W,
                         heads=heads, head_dim=D, bits=2, layer=i, kv=0)
    # same allocation both ways (the code streams may differ only inside the parity band)
    assert torch.equal(pay_tc[:, :64 + S * H * W], pay_sm[:, :64 + S * H * W])


@pytest.mark.parametrize("S,H,W,flags,dtype", [
    (16, 8, 8, 0, torch.float32),     # fused decode on the tensor cores, float32 output
    (32, 16, 16, 1, torch.bfloat16),  # NO_QUANT on a fused grid: the separate (exact) inverse kernels
    (64, 14, 14, 1, torch.float32),
    (32, 24, 24, 0, torch.float32),   # fused forward on the 24 x 24 grid, float32 output
])
def test_fused_grid_output_variants(S, H, W, flags, dtype):
    """The fused decode kernel writes bf16 or float32; NO_QUANT payloads keep the separate inverse
    kernels (their round trip must stay within 1e-5), on the grids that have the fused kernels."""
    heads, D = 1, 64
    x = make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.85), nu=4.0, seed=90 + S, dtype=dtype, device=DEV)[None]
    reports, _, y = _check_batch(x, S, H, W, 3, flags=flags)
    if flags:
        assert rel_rms(y.double().cpu(), x.double().cpu()) <= 1e-5


# ---------------------------------------------------------------- ablation and rotation flags ---
@pytest.mark.parametrize("shape", [(16, 16, 16, 2, 64), (5, 7, 6, 3, 32)], ids=["fused-grid", "ragged-grid"])
@pytest.mark.parametrize("variant", ["no_dct", "hw_only", "s_only", "w_only", "uniform", "rotate",
                                     "rotate_uniform_hw", "head_gain", "head_gain_rotate"])
def test_variant_flags(shape, variant):
    """The summary page's ablations ("Main Findings": fewer transformed axes, uniform allocation),
    stage 4's fixed shared rotation and per-head gains, as flags: payload, codes and reconstruction
    against the oracle run with the same flags."""
    flags = {"no_dct": T.TACTKV_SKIP_S | T.TACTKV_SKIP_H | T.TACTKV_SKIP_W, "hw_only": T.TACTKV_SKIP_S,
             "s_only": T.TACTKV_SKIP_H | T.TACTKV_SKIP_W, "w_only": T.TACTKV_SKIP_S | T.TACTKV_SKIP_H,
             "uniform": T.TACTKV_UNIFORM_ALLOC, "rotate": T.TACTKV_ROTATE,
             "rotate_uniform_hw": T.TACTKV_ROTATE | T.TACTKV_UNIFORM_ALLOC | T.TACTKV_SKIP_S,
             "head_gain": T.TACTKV_HEAD_GAIN, "head_gain_rotate": T.TACTKV_HEAD_GAIN | T.TACTKV_ROTATE}[variant]
    S, H, W, heads, D = shape
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.8), nu=4.0, seed=300 + i, device=DEV)
                     for i in range(2)])
    reports, pay, _ = _check_batch(x, S, H, W, 2, layers=[0, 1], kvs=[1, 1], flags=flags)
    p = O.parse_payload(pay[0].cpu().numpy().tobytes())
    assert p["flags"] == flags
    if flags & T.TACTKV_UNIFORM_ALLOC:
        assert set(np.unique(p["b"])) <= {0, 2}
    # decoding with other flags than the payload's is refused
    with pytest.raises(T.TactkvError):
        T.decompress(pay, S, H, W, 2, heads=heads, head_dim=D, layers=[0, 1], kvs=[1, 1], flags=0, check=True)


def test_head_gain_scaled_copy_of_a_head():
    """Per-head gains on the GPU: head 1 = 4 x head 0 (exact in bf16 and in every float32 step)
    gives head 1 exactly 4 x head 0's gains and exactly head 0's codes, on a fused grid."""
    S, H, W, D = 16, 16, 16, 64
    x0 = make_unit(S, H, W, 1, D, rho=(0.9, 0.85, 0.85), nu=4.0, seed=77, device=DEV)
    x = torch.cat([x0, x0 * 4], dim=1)[None]
    reports, pay, _ = _check_batch(x, S, H, W, 3, flags=T.TACTKV_HEAD_GAIN)
    p = O.parse_payload(pay[0].cpu().numpy().tobytes())
    assert p["sigma"].shape == (2, S * H * W) and np.array_equal(p["sigma"][1], 4 * p["sigma"][0])
    b, codes = O.codes_of(pay[0].cpu().numpy().tobytes())
    act = b > 0
    assert np.array_equal(codes[act][:, D:], codes[act][:, :D])


@pytest.mark.parametrize("shape,bits,flags", [((16, 16, 16, 2, 64), 2, 0), ((5, 7, 6, 3, 32), 8, 0),
                                              ((16, 16, 16, 2, 64), 3, 64 | 128)],
                         ids=["fused-grid-2b", "ragged-8b", "fused-grid-rotate-headgain"])
def test_canaries_around_payloads_and_outputs(shape, bits, flags):
    """Compress writes exactly the payload's total_bytes (the bytes after it in a larger buffer keep
    their canary), and decompress into a strided view leaves the gaps between heads untouched."""
    S, H, W, heads, D = shape
    U = 2
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.8), nu=4.0, seed=500 + i, device=DEV)
                     for i in range(U)])
    cap = T.payload_capacity(S, H, W, heads, D, bits, flags)
    pay = torch.full((U, cap + 272), 0xA5, dtype=torch.uint8, device=DEV)
    T.compress(x, S, H, W, bits, layers=[0, 1], kvs=[0, 0], flags=flags, payload=pay)
    big = torch.full((U, S * H * W, heads, D + 8), 7.0, dtype=torch.bfloat16, device=DEV)
    T.decompress(pay, S, H, W, bits, heads=heads, head_dim=D, layers=[0, 1], kvs=[0, 0], flags=flags,
                 out=big[..., :D], check=True)
    torch.cuda.synchronize()
    for i in range(U):
        buf = pay[i].cpu().numpy()
        total = int.from_bytes(buf[48:56].tobytes(), "little")
        assert total <= cap and np.all(buf[total:] == 0xA5)
        assert total == len(O.compress_unit(x[i].double().cpu().numpy(), S, H, W, heads, D, bits, flags=flags))
    assert torch.all(big[..., D:] == 7.0)


def test_opt_in_tensor_core_kernels():
    """The opt-in tensor-core forms, read once per process: the forward kernel's DCT along S on
    tcgen05 (TACTKV_TC_S=1) and the single-kernel decode with the inverse S on tcgen05
    (TACTKV_FUSED_DECODE=1), on the fused-grid parity cases, in a child process."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, TACTKV_TC_S="1", TACTKV_FUSED_DECODE="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_gpu_parity.py", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider", "-k",
                        "tensor_core_and_cuda_core or fused_grid_output or small_shapes or variant_flags or "
                        "full_size_sampled_units and med4b-1"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


# ------------------------------------------------------------------------------ exact ties ---
def _gpu_allocation(var, grid, bits):
    S, H, W = grid
    v = torch.from_numpy(np.asarray(var, dtype=np.float64)).to(DEV)
    b = T.allocate(v, S, H, W, bits)
    torch.cuda.synchronize()
    return b.cpu().numpy().astype(np.int64)


@pytest.mark.parametrize("var,grid,bits,want", [
    ([1.0, 1.0, 16.0], (1, 1, 3), 1, [1, 0, 2]),       # three keys equal to 1 for the last slot
    ([1.0, 4.0, 4.0], (1, 1, 3), 1, [1, 1, 1]),
    ([8.0, 2.0], (1, 1, 2), 1, [2, 0]),                # keys 8 4^-(k+1) = 2 4^-k tie at every k
    ([8.0, 2.0], (1, 1, 2), 2, [3, 1]),
    ([2.0, 8.0], (1, 1, 2), 1, [1, 1]),                # key 2 of bin 0 ties key 8/4 of bin 1: bin 0 wins
    ([0.0, 5.0, 0.0, 5.0], (1, 2, 2), 3, [0, 6, 0, 6]),  # zero bins get nothing; budget 12 split evenly
    ([3.0, 0.0, 1.0, 2.0], (1, 1, 4), 8, [8, 0, 8, 8]),  # every active bin saturates below the budget
])
def test_allocation_kernel_exact_on_planted_ties(var, grid, bits, want):
    """Stage 3 ("Methodology in Plain English": the bisection, rounding and +-1 greedy steps up to
    the budget, capped at 8 bits, ties to the lower bin index) on variances given to the library
    directly, so the GPU and the oracle see the same fp64 numbers and exact ties are exact on both
    sides.  Compared with no tolerance against the oracle and the brute-force top-B selection."""
    var = np.asarray(var)
    assert O.allocate_bits(var, bits).tolist() == want
    assert O.allocate_bits_topk(var, bits).tolist() == want
    assert _gpu_allocation(var, grid, bits).tolist() == want


@pytest.mark.parametrize("grid,bits,seed", [((64, 16, 16), 1, 0), ((64, 16, 16), 2, 1), ((16, 16, 16), 4, 2),
                                             ((32, 24, 24), 1, 3), ((7, 5, 9), 3, 4), ((64, 32, 32), 1, 5)])
def test_allocation_kernel_exact_on_tie_heavy_variances(grid, bits, seed):
    """Thousands of exact key ties: variances drawn from four mantissas times powers of 4 (so
    sigma_i^2 4^-k of one bin equals that of many others), 10% of the bins empty.  The GPU's radix
    selection and its in-order tie fill must give the oracle's allocation bit for bit."""
    rng = np.random.default_rng(seed)
    N = grid[0] * grid[1] * grid[2]
    var = rng.choice([1.0, 1.5, 3.0, 0.75], N) * 4.0 ** rng.integers(-12, 12, N)
    var[rng.random(N) < 0.1] = 0.0
    b_gpu = _gpu_allocation(var, grid, bits)
    b_o = O.allocate_bits(var, bits)
    assert np.array_equal(b_gpu, b_o), np.nonzero(b_gpu != b_o)[0][:10]
    assert b_gpu.sum() == bits * N


# ------------------------------------------------------------------------------ error paths ---
def test_corrupt_header_is_reported_and_zero_filled():
    S, H, W, heads, D = 8, 4, 4, 1, 32
    x = make_unit(S, H, W, heads, D, seed=2, device=DEV)[None]
    pay = T.compress(x, S, H, W, 2)
    bad = pay.clone()
    bad[0, 16] ^= 1                                   # S field of the header
    units = T.make_units(None, S, H, W, 2, heads=heads, head_dim=D, payload=bad,
                         out=torch.ones_like(x), n_units=1)
    ws = T.alloc_workspace(units, DEV)
    out = torch.ones_like(x)
    T.decompress(bad, S, H, W, 2, heads=heads, head_dim=D, out=out, workspace=ws)
    st = T.tactkv_device_status(ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == T.TACTKV_CORRUPT_PAYLOAD
    assert not out.any()
    # status is cleared once read; a good payload decodes cleanly afterwards
    T.decompress(pay, S, H, W, 2, heads=heads, head_dim=D, workspace=ws, check=True)


def test_bit_width_above_8_is_reported_and_zero_filled():
    """A payload whose header is intact but whose allocation holds a bit width of 9 (the sum of
    the widths unchanged, so only the per-bin range check can catch it): the decoder's index
    kernel must flag it, zero-fill that unit and decode the next unit of the batch normally."""
    S, H, W, heads, D = 8, 4, 4, 1, 32
    x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.9, 0.9), seed=s, device=DEV) for s in (2, 3)])
    pay = T.compress(x, S, H, W, 2, layers=[0, 1])
    bad = pay.clone()
    b = bad[0, 64:64 + S * H * W].cpu().numpy().astype(np.int64)
    i_hi = int(np.argmax(b))
    donors = [j for j in np.argsort(-b) if j != i_hi and b[j] > 0]
    need = 9 - int(b[i_hi])
    for j in donors:                    # move bits from other bins so that the total is unchanged
        take = min(need, int(b[j]))
        b[j] -= take
        need -= take
        if need == 0:
            break
    assert need == 0
    b[i_hi] = 9
    bad[0, 64:64 + S * H * W] = torch.from_numpy(b.astype(np.uint8)).to(DEV)
    units = T.make_units(None, S, H, W, 2, heads=heads, head_dim=D, payload=bad, out=torch.ones_like(x),
                         layers=[0, 1], n_units=2)
    ws = T.alloc_workspace(units, DEV)
    out = torch.ones_like(x)
    T.decompress(bad, S, H, W, 2, heads=heads, head_dim=D, out=out, layers=[0, 1], workspace=ws)
    st = T.tactkv_device_status(ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == T.TACTKV_CORRUPT_PAYLOAD
    assert not out[0].any()
    good = T.decompress(pay, S, H, W, 2, heads=heads, head_dim=D, layers=[0, 1], check=True)
    torch.cuda.synchronize()
    assert torch.equal(out[1], good[1])


def test_wrong_layer_is_rejected():
    S, H, W, heads, D = 8, 4, 4, 1, 32
    x = make_unit(S, H, W, heads, D, seed=2, device=DEV)[None]
    pay = T.compress(x, S, H, W, 2, layers=[7])
    with pytest.raises(T.TactkvError):
        T.decompress(pay, S, H, W, 2, heads=heads, head_dim=D, layers=[8], check=True)
