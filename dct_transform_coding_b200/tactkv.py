"""Thin Python binding of libtactkv.so (include/tactkv.h): argument marshalling only.

Every step of compression and decompression runs in the library's CUDA kernels.  PyTorch is
used for device memory and streams: the helpers below allocate payload, output and workspace
tensors and pass their device pointers to the C ABI.  If the shared library is missing the
import fails; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtactkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m dct_transform_coding_b200.build` "
                      "(or __graft_entry__.build()); the codec has no CPU path")
_lib = ctypes.CDLL(LIB_PATH)

TACTKV_OK = 0
TACTKV_INVALID_ARG = 1
TACTKV_UNSUPPORTED_SHAPE = 2
TACTKV_CAPACITY = 3
TACTKV_ALIGNMENT = 4
TACTKV_CORRUPT_PAYLOAD = 5
TACTKV_CUDA = 6
TACTKV_WORKSPACE = 7
TACTKV_SCRATCH_LIMIT = 8
TACTKV_TIMEOUT = 9

TACTKV_NO_QUANT = 1
TACTKV_FP32_IO = 2
TACTKV_SKIP_S = 4
TACTKV_SKIP_H = 8
TACTKV_SKIP_W = 16
TACTKV_UNIFORM_ALLOC = 32
TACTKV_ROTATE = 64
TACTKV_HEAD_GAIN = 128

HEADER_BYTES = 64
EXPORTED = ("tactkv_payload_bytes", "tactkv_workspace_bytes", "tactkv_compress", "tactkv_decompress",
            "tactkv_compress_profiled", "tactkv_decompress_profiled", "tactkv_compress_noalloc",
            "tactkv_allocate", "tactkv_device_status", "tactkv_occupancy", "tactkv_max_batch",
            "tactkv_attention_workspace_bytes", "tactkv_attention_decode",
            "tactkv_status_string", "tactkv_lloyd_max_table", "tactkv_format_version", "tactkv_last_launches")


class tactkv_unit(ctypes.Structure):
    _fields_ = [
        ("layer", ctypes.c_int32), ("kv", ctypes.c_int32),
        ("S", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
        ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("bits", ctypes.c_int32), ("flags", ctypes.c_uint32),
        ("kv_in", ctypes.c_void_p), ("kv_out", ctypes.c_void_p),
        ("token_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64),
        ("payload", ctypes.c_void_p), ("payload_capacity", ctypes.c_size_t),
    ]


class tactkv_occupancy_t(ctypes.Structure):
    _fields_ = [("bins", ctypes.c_uint64), ("channels", ctypes.c_uint64), ("code_bits", ctypes.c_uint64),
                ("formula_bits", ctypes.c_uint64), ("index_bits", ctypes.c_uint64),
                ("payload_bytes", ctypes.c_uint64), ("bits_per_element", ctypes.c_double),
                ("shrink_vs_bf16", ctypes.c_double)]


_P = ctypes.POINTER(tactkv_unit)
_lib.tactkv_payload_bytes.restype = ctypes.c_size_t
_lib.tactkv_payload_bytes.argtypes = [_P]
_lib.tactkv_workspace_bytes.restype = ctypes.c_size_t
_lib.tactkv_workspace_bytes.argtypes = [_P, ctypes.c_int]
for _name in ("tactkv_compress", "tactkv_decompress"):
    getattr(_lib, _name).restype = ctypes.c_int
    getattr(_lib, _name).argtypes = [_P, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
for _name in ("tactkv_compress_profiled", "tactkv_decompress_profiled"):
    getattr(_lib, _name).restype = ctypes.c_int
    getattr(_lib, _name).argtypes = [_P, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                     ctypes.POINTER(ctypes.c_void_p)]
_lib.tactkv_compress_noalloc.restype = ctypes.c_int
_lib.tactkv_compress_noalloc.argtypes = [_P, ctypes.c_int, ctypes.c_void_p]
_lib.tactkv_allocate.restype = ctypes.c_int
_lib.tactkv_allocate.argtypes = [_P, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
_lib.tactkv_device_status.restype = ctypes.c_int
_lib.tactkv_device_status.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
_lib.tactkv_occupancy.restype = ctypes.c_int
_lib.tactkv_occupancy.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(tactkv_occupancy_t)]
_lib.tactkv_max_batch.restype = ctypes.c_int64
_lib.tactkv_max_batch.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
_lib.tactkv_attention_workspace_bytes.restype = ctypes.c_size_t
_lib.tactkv_attention_workspace_bytes.argtypes = [_P, ctypes.c_int, ctypes.c_int]
_lib.tactkv_attention_decode.restype = ctypes.c_int
_lib.tactkv_attention_decode.argtypes = [_P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_void_p]
_lib.tactkv_status_string.restype = ctypes.c_char_p
_lib.tactkv_status_string.argtypes = [ctypes.c_int]
_lib.tactkv_lloyd_max_table.restype = ctypes.c_int
_lib.tactkv_lloyd_max_table.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
_lib.tactkv_format_version.restype = ctypes.c_int
_lib.tactkv_format_version.argtypes = []
_lib.tactkv_last_launches.restype = ctypes.c_int
_lib.tactkv_last_launches.argtypes = []


class TactkvError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {tactkv_status_string(status)} ({status})")


# ------------------------------------------------------------------------- raw C entry points ---
def tactkv_payload_bytes(unit: tactkv_unit) -> int:
    return int(_lib.tactkv_payload_bytes(ctypes.byref(unit)))


def tactkv_workspace_bytes(units) -> int:
    arr = _as_array(units)
    return int(_lib.tactkv_workspace_bytes(arr, len(arr)))


def tactkv_compress(units, workspace_ptr: int, workspace_bytes: int, stream_ptr: int) -> int:
    arr = _as_array(units)
    return int(_lib.tactkv_compress(arr, len(arr), ctypes.c_void_p(workspace_ptr), workspace_bytes,
                                    ctypes.c_void_p(stream_ptr)))


def tactkv_decompress(units, workspace_ptr: int, workspace_bytes: int, stream_ptr: int) -> int:
    arr = _as_array(units)
    return int(_lib.tactkv_decompress(arr, len(arr), ctypes.c_void_p(workspace_ptr), workspace_bytes,
                                      ctypes.c_void_p(stream_ptr)))


def _events_array(events):
    if events is None:
        return None
    return (ctypes.c_void_p * len(events))(*[int(e) if e else None for e in events])


def tactkv_compress_profiled(units, workspace_ptr: int, workspace_bytes: int, stream_ptr: int, events) -> int:
    """events: sequence of 5 cudaEvent_t handles (ints, e.g. torch.cuda.Event().cuda_event) or None."""
    arr = _as_array(units)
    return int(_lib.tactkv_compress_profiled(arr, len(arr), ctypes.c_void_p(workspace_ptr), workspace_bytes,
                                             ctypes.c_void_p(stream_ptr), _events_array(events)))


def tactkv_decompress_profiled(units, workspace_ptr: int, workspace_bytes: int, stream_ptr: int, events) -> int:
    """events: sequence of 4 cudaEvent_t handles or None."""
    arr = _as_array(units)
    return int(_lib.tactkv_decompress_profiled(arr, len(arr), ctypes.c_void_p(workspace_ptr), workspace_bytes,
                                               ctypes.c_void_p(stream_ptr), _events_array(events)))


def tactkv_compress_noalloc(units, stream_ptr: int) -> int:
    """Compress with the library's fixed device scratch instead of a caller workspace (for callers
    that cannot allocate, e.g. while recording a CUDA graph).  Calls share that scratch: serialize
    calls that could overlap on the GPU."""
    arr = _as_array(units)
    return int(_lib.tactkv_compress_noalloc(arr, len(arr), ctypes.c_void_p(stream_ptr)))


def tactkv_allocate(unit: tactkv_unit, var_ptr: int, workspace_ptr: int, workspace_bytes: int,
                    stream_ptr: int) -> int:
    """Stage 3 on given fp64 variances (device pointer var_ptr, N doubles): header, b[] and sigma[]
    of unit.payload as compress would write them."""
    return int(_lib.tactkv_allocate(ctypes.byref(unit), ctypes.c_void_p(var_ptr), ctypes.c_void_p(workspace_ptr),
                                    workspace_bytes, ctypes.c_void_p(stream_ptr)))


def allocate(var: torch.Tensor, S: int, H: int, W: int, bits: int, *, heads: int = 1, head_dim: int = 32,
             stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Bit allocation of the fp64 variances var [S*H*W] (on the GPU): returns b [S*H*W] uint8."""
    var = var.to(torch.float64).contiguous()
    cap = payload_capacity(S, H, W, heads, head_dim, bits)
    payload = torch.zeros(((cap + 15) // 16 * 16,), dtype=torch.uint8, device=var.device)
    u = tactkv_unit(S=S, H=H, W=W, heads=heads, head_dim=head_dim, bits=bits, payload=payload.data_ptr(),
                    payload_capacity=payload.numel(), token_stride=heads * head_dim, head_stride=head_dim)
    ws = alloc_workspace([u], var.device)
    st = tactkv_allocate(u, var.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    if st != TACTKV_OK:
        raise TactkvError(st, "tactkv_allocate")
    N = S * H * W
    return payload[HEADER_BYTES:HEADER_BYTES + N]


def tactkv_attention_workspace_bytes(k_units, n_units: int, q_heads: int) -> int:
    return int(_lib.tactkv_attention_workspace_bytes(_as_array(k_units), n_units, q_heads))


def tactkv_device_status(workspace_ptr: int, workspace_bytes: int, stream_ptr: int) -> int:
    return int(_lib.tactkv_device_status(ctypes.c_void_p(workspace_ptr), workspace_bytes, ctypes.c_void_p(stream_ptr)))


def tactkv_occupancy(payload) -> dict:
    """Occupancy of one payload (a host bytes-like object or a CPU uint8 tensor)."""
    buf = bytes(payload.numpy().tobytes()) if isinstance(payload, torch.Tensor) else bytes(payload)
    out = tactkv_occupancy_t()
    st = int(_lib.tactkv_occupancy(ctypes.c_char_p(buf), len(buf), ctypes.byref(out)))
    if st != TACTKV_OK:
        raise TactkvError(st, "tactkv_occupancy")
    return {name: getattr(out, name) for name, _ in tactkv_occupancy_t._fields_}


def tactkv_max_batch(hbm_bytes: int, fixed_bytes: int, per_request_bytes: int) -> int:
    return int(_lib.tactkv_max_batch(int(hbm_bytes), int(fixed_bytes), int(per_request_bytes)))


def batch_capacity(hbm_bytes: int, fixed_bytes: int, payload_bytes_per_request: int, text_kv_bytes_per_request: int,
                   visual_kv_bf16_bytes_per_request: int) -> dict:
    """Decode batch that fits with the visual KV compressed versus kept in bf16 (the text KV stays
    bf16 either way), and the per-request cache shrink."""
    comp = payload_bytes_per_request + text_kv_bytes_per_request
    full = visual_kv_bf16_bytes_per_request + text_kv_bytes_per_request
    return {"batch_bf16": tactkv_max_batch(hbm_bytes, fixed_bytes, full),
            "batch_compressed": tactkv_max_batch(hbm_bytes, fixed_bytes, comp),
            "cache_shrink": full / comp if comp else float("inf")}


def tactkv_status_string(status: int) -> str:
    return _lib.tactkv_status_string(int(status)).decode()


def tactkv_lloyd_max_table(bits: int):
    """The library's own codebook: (levels, thresholds) as lists of floats (host only)."""
    L = 1 << bits
    lv = (ctypes.c_double * L)()
    th = (ctypes.c_double * max(1, L - 1))()
    n = _lib.tactkv_lloyd_max_table(bits, lv, th)
    if n != L:
        raise ValueError("bits must be 1..8")
    return list(lv), list(th)[:L - 1]


def tactkv_format_version() -> int:
    return int(_lib.tactkv_format_version())


def tactkv_last_launches() -> int:
    """Kernels launched by this thread's most recent compress / decompress call."""
    return int(_lib.tactkv_last_launches())


def _as_array(units):
    if isinstance(units, ctypes.Array):
        return units
    units = list(units)
    arr = (tactkv_unit * len(units))(*units)
    return arr


# ------------------------------------------------------------------------------ torch helpers ---
def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def make_units(x: Optional[torch.Tensor], S: int, H: int, W: int, bits: int, *, heads: int, head_dim: int,
               payload: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
               layers: Optional[Sequence[int]] = None, kvs: Optional[Sequence[int]] = None,
               flags: int = 0, n_units: Optional[int] = None):
    """Descriptors for a batch laid out as [units, tokens, heads, head_dim] (strided views allowed).

    x is the compress input (or None for decompress), out the decompress output, payload a
    [units, capacity] uint8 tensor."""
    ref = x if x is not None else out
    U = ref.shape[0] if n_units is None else n_units
    arr = (tactkv_unit * U)()
    for i in range(U):
        u = arr[i]
        u.layer = int(layers[i]) if layers is not None else i
        u.kv = int(kvs[i]) if kvs is not None else 0
        u.S, u.H, u.W, u.heads, u.head_dim, u.bits, u.flags = S, H, W, heads, head_dim, bits, flags
        if x is not None:
            u.kv_in = x[i].data_ptr()
            u.token_stride, u.head_stride = x.stride(1), x.stride(2)
        if out is not None:
            u.kv_out = out[i].data_ptr()
            u.token_stride, u.head_stride = out.stride(1), out.stride(2)
        if payload is not None:
            u.payload = payload[i].data_ptr()
            u.payload_capacity = payload.shape[1]
    return arr


def payload_capacity(S: int, H: int, W: int, heads: int, head_dim: int, bits: int, flags: int = 0) -> int:
    u = tactkv_unit(S=S, H=H, W=W, heads=heads, head_dim=head_dim, bits=bits, flags=flags)
    cap = tactkv_payload_bytes(u)
    if cap == 0:
        raise TactkvError(TACTKV_UNSUPPORTED_SHAPE, "payload_capacity")
    return cap


def alloc_workspace(units, device) -> torch.Tensor:
    nbytes = tactkv_workspace_bytes(units)
    ws = torch.zeros(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + nbytes]


def compress(x: torch.Tensor, S: int, H: int, W: int, bits: int, *, layers=None, kvs=None, flags: int = 0,
             payload: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Compress x [units, S*H*W, heads, head_dim] (bf16, or fp32 with TACTKV_FP32_IO) on its device.
    Returns the [units, capacity] uint8 payload tensor (asynchronous on the stream)."""
    U, T, heads, D = x.shape
    if x.dtype == torch.float32:
        flags |= TACTKV_FP32_IO
    cap = payload_capacity(S, H, W, heads, D, bits, flags)
    if payload is None:
        payload = torch.empty((U, (cap + 15) // 16 * 16), dtype=torch.uint8, device=x.device)
    units = make_units(x, S, H, W, bits, heads=heads, head_dim=D, payload=payload, layers=layers, kvs=kvs,
                       flags=flags)
    if workspace is None:
        workspace = alloc_workspace(units, x.device)
    st = tactkv_compress(units, workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    if st != TACTKV_OK:
        raise TactkvError(st, "tactkv_compress")
    return payload


def decompress(payload: torch.Tensor, S: int, H: int, W: int, bits: int, *, heads: int, head_dim: int,
               layers=None, kvs=None, flags: int = 0, dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
               check: bool = False) -> torch.Tensor:
    """Decompress [units, capacity] payloads into [units, S*H*W, heads, head_dim]."""
    U = payload.shape[0]
    if dtype == torch.float32:
        flags |= TACTKV_FP32_IO
    if out is None:
        out = torch.empty((U, S * H * W, heads, head_dim), dtype=dtype, device=payload.device)
    units = make_units(None, S, H, W, bits, heads=heads, head_dim=head_dim, payload=payload, out=out,
                       layers=layers, kvs=kvs, flags=flags, n_units=U)
    if workspace is None:
        workspace = alloc_workspace(units, payload.device)
    st = tactkv_decompress(units, workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    if st != TACTKV_OK:
        raise TactkvError(st, "tactkv_decompress")
    if check:
        ds = tactkv_device_status(workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
        if ds != TACTKV_OK:
            raise TactkvError(ds, "tactkv_decompress (device)")
    return out


def attention_decode(q: torch.Tensor, k_payload: torch.Tensor, v_payload: torch.Tensor, S: int, H: int, W: int,
                     bits: int, *, heads: int, head_dim: int, layers=None, flags: int = 0,
                     workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                     check: bool = False):
    """One decode step of attention over compressed K/V: q [units, q_heads, head_dim] float32 on the
    GPU, k_payload / v_payload [units, capacity] (compressed with kv 0 / 1).  Returns (out, m, l):
    out [units, q_heads, head_dim] = softmax(q K^T / sqrt(head_dim)) V over the visual tokens, m and
    l the scores' maximum and exp-sum per query head."""
    U, q_heads, D = q.shape
    q = q.contiguous().to(torch.float32)
    ku = make_units(None, S, H, W, bits, heads=heads, head_dim=head_dim, payload=k_payload, layers=layers,
                    kvs=[0] * U, flags=flags, n_units=U)
    vu = make_units(None, S, H, W, bits, heads=heads, head_dim=head_dim, payload=v_payload, layers=layers,
                    kvs=[1] * U, flags=flags, n_units=U)
    out = torch.empty((U, q_heads, D), dtype=torch.float32, device=q.device)
    m = torch.empty((U, q_heads), dtype=torch.float32, device=q.device)
    l = torch.empty((U, q_heads), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = tactkv_attention_workspace_bytes(ku, U, q_heads)
        ws = torch.zeros(nbytes + 256, dtype=torch.uint8, device=q.device)
        off = (-ws.data_ptr()) % 256
        workspace = ws[off:off + nbytes]
    st = int(_lib.tactkv_attention_decode(ku, vu, U, q_heads, ctypes.c_void_p(q.data_ptr()),
                                          ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(m.data_ptr()),
                                          ctypes.c_void_p(l.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
                                          workspace.numel(), ctypes.c_void_p(_stream_ptr(stream))))
    if st != TACTKV_OK:
        raise TactkvError(st, "tactkv_attention_decode")
    if check:
        ds = tactkv_device_status(workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
        if ds != TACTKV_OK:
            raise TactkvError(ds, "tactkv_attention_decode (device)")
    return out, m, l
