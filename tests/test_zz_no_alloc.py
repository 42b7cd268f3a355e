"""tactkv_compress_noalloc: compression for callers that cannot allocate device memory.

Some callers cannot hand the codec a workspace: code that is recording a CUDA graph (cudaMalloc
is not allowed while a stream is being captured), serving engines whose device memory is owned
by their own pool, and latency-critical loops where an allocation may synchronize the device.
For them the library keeps a fixed device array as scratch.  These tests call that entry point
through the C ABI and compare its payloads with the workspace entry point's, on two calls in a
row (the second with other data and another shape, so contents left over from the first call
cannot leak into the result).  This file is collected last on purpose.
"""
import pytest
import torch

from dct_transform_coding_b200.workloads import make_unit

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _payloads_with_workspace(T, x, S, H, W, bits, layers, kvs):
    return T.compress(x, S, H, W, bits, layers=layers, kvs=kvs)


def _payloads_without_workspace(T, x, S, H, W, bits, layers, kvs, like):
    pay = torch.full_like(like, 0xA5)                           # stale bytes everywhere
    U, _, heads, D = x.shape
    units = T.make_units(x, S, H, W, bits, heads=heads, head_dim=D, payload=pay, layers=layers, kvs=kvs)
    st = T.tactkv_compress_noalloc(units, torch.cuda.current_stream().cuda_stream)
    assert st == T.TACTKV_OK, T.tactkv_status_string(st)
    return pay


def _total_bytes(pay_row):
    return int.from_bytes(bytes(pay_row[48:56].cpu().numpy()), "little")


@pytest.mark.parametrize("first,second", [
    ((8, 8, 8, 2, 32, 2, 3), (16, 6, 10, 1, 64, 4, 2)),
])
def test_noalloc_matches_workspace_entry_on_two_calls(first, second):
    from dct_transform_coding_b200 import tactkv as T
    for call, (S, H, W, heads, D, bits, U) in enumerate((first, second)):
        x = torch.stack([make_unit(S, H, W, heads, D, rho=(0.9, 0.85, 0.8), nu=4.0, seed=100 * call + i,
                                   device=DEV) for i in range(U)])
        layers, kvs = list(range(U)), [i % 2 for i in range(U)]
        ref = _payloads_with_workspace(T, x, S, H, W, bits, layers, kvs)
        got = _payloads_without_workspace(T, x, S, H, W, bits, layers, kvs, ref)
        torch.cuda.synchronize()
        for i in range(U):
            n = _total_bytes(ref[i])
            assert n == _total_bytes(got[i])
            assert torch.equal(got[i, :n], ref[i, :n]), f"call {call}, unit {i}"
        # and the payload decodes like the reference one
        y_ref = T.decompress(ref, S, H, W, bits, heads=heads, head_dim=D, layers=layers, kvs=kvs, check=True)
        y_got = T.decompress(got, S, H, W, bits, heads=heads, head_dim=D, layers=layers, kvs=kvs, check=True)
        torch.cuda.synchronize()
        assert torch.equal(y_ref, y_got)


def test_noalloc_rejects_units_beyond_its_scratch():
    from dct_transform_coding_b200 import tactkv as T
    S, H, W, heads, D = 64, 16, 16, 4, 256                       # 64 MiB of scratch per unit
    x = torch.zeros((1, S * H * W, heads, D), dtype=torch.bfloat16, device=DEV)
    cap = T.payload_capacity(S, H, W, heads, D, 1)
    pay = torch.zeros((1, cap), dtype=torch.uint8, device=DEV)
    units = T.make_units(x, S, H, W, 1, heads=heads, head_dim=D, payload=pay)
    st = T.tactkv_compress_noalloc(units, torch.cuda.current_stream().cuda_stream)
    assert st == T.TACTKV_SCRATCH_LIMIT
    assert "scratch" in T.tactkv_status_string(st)
    torch.cuda.synchronize()
    assert not pay.any()                                         # nothing was launched
