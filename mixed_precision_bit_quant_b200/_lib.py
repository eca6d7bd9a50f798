"""ctypes binding of libthrift (include/thrift.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels; this module only
allocates output tensors with PyTorch, passes device pointers and the
current stream, and turns status codes into exceptions.  There is no CPU
fallback: if the library is missing, :func:`lib` raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libthrift.so")

THRIFT_OK, THRIFT_ERR_INVALID, THRIFT_ERR_UNSUPPORTED, THRIFT_ERR_CUDA, THRIFT_ERR_TIMEOUT = range(5)
OP_QUANTIZE, OP_SELECT, OP_ATTN, OP_SELECT_VERTICAL, OP_QUANTIZE_MX = range(5)
FORMATS = ("nvfp4", "mxfp4")
QUANT_FIELDS = ["q_fp4", "q_sf", "q_sf_mma", "q_gs", "k_fp4", "k_sf", "k_sf_mma", "k_gs",
                "v_fp8t", "v_st", "v_exp"]
_FIELD_DTYPES = {"q_gs": torch.float32, "k_gs": torch.float32, "v_st": torch.bfloat16,
                 "v_exp": torch.int8}


class ThriftError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]


class QuantStruct(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in QUANT_FIELDS]


DECODE_FIELDS = ["kc", "ksc", "vc", "vsc"]


class DecodeShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("L", ctypes.c_int32), ("d", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


class DecodeCacheStruct(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in DECODE_FIELDS]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libthrift.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libthrift.so not found at {LIB_PATH}; build it with "
                               "`python -m mixed_precision_bit_quant_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S, I32, U64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64
        SP = ctypes.POINTER(Shape)
        QP = ctypes.POINTER(QuantStruct)
        L.thrift_quant_bytes.argtypes = [SP, ctypes.c_int]
        L.thrift_quant_bytes.restype = S
        L.thrift_workspace_bytes.argtypes = [SP, ctypes.c_int]
        L.thrift_workspace_bytes.restype = S
        L.thrift_quantize.argtypes = [SP, P, P, P, QP, P, S, P]
        L.thrift_quantize.restype = ctypes.c_int
        L.thrift_select.argtypes = [SP, P, P, I32, I32, P, P, P, S, P]
        L.thrift_select.restype = ctypes.c_int
        L.thrift_quantize_mx.argtypes = [SP, P, P, P, QP, P, S, P]
        L.thrift_quantize_mx.restype = ctypes.c_int
        L.thrift_attn_fwd_mx.argtypes = [SP, QP, P, P, P, P, P, P]
        L.thrift_attn_fwd_mx.restype = ctypes.c_int
        L.thrift_select_vertical.argtypes = [SP, P, P, I32, I32, P, P, P, S, P]
        L.thrift_select_vertical.restype = ctypes.c_int
        L.thrift_attn_fwd.argtypes = [SP, QP, P, P, P, P, P, P, S, P]
        L.thrift_attn_fwd.restype = ctypes.c_int
        L.thrift_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
        L.thrift_device_status.restype = ctypes.c_int
        L.thrift_status_string.argtypes = [ctypes.c_int]
        L.thrift_status_string.restype = ctypes.c_char_p
        L.thrift_debug_withhold_v_load.argtypes = [I32]
        L.thrift_debug_withhold_v_load.restype = ctypes.c_int
        DSP = ctypes.POINTER(DecodeShape)
        DCP = ctypes.POINTER(DecodeCacheStruct)
        L.thrift_decode_cache_bytes.argtypes = [DSP, ctypes.c_int]
        L.thrift_decode_cache_bytes.restype = S
        L.thrift_decode_workspace_bytes.argtypes = [DSP]
        L.thrift_decode_workspace_bytes.restype = S
        L.thrift_decode_quantize_cache.argtypes = [DSP, P, P, DCP, I32, I32, P]
        L.thrift_decode_quantize_cache.restype = ctypes.c_int
        L.thrift_decode_step.argtypes = [DSP, P, P, P, DCP, P, P, P, S, P]
        L.thrift_decode_step.restype = ctypes.c_int
        L.thrift_probe_mma.argtypes = [I32, I32, I32, I32, ctypes.POINTER(ctypes.c_float), P, P]
        L.thrift_probe_mma.restype = ctypes.c_int
        L.thrift_launch_count.argtypes = []
        L.thrift_launch_count.restype = U64
        L.thrift_version.argtypes = []
        L.thrift_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().thrift_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != THRIFT_OK:
        raise ThriftError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


# The C ABI takes plain pointers and reads every buffer as dense and of the size
# its shape implies, so a strided view, another dtype, a host tensor or a buffer
# sized for another problem would be read or written out of bounds.  These checks
# run before any call into the library.
def _want(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, device=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    _on_device(t, name, device)


def _on_device(t: torch.Tensor, name: str, device=None) -> None:
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor (got {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor] = None) -> None:
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q: expected a [B, Hq, N, d] tensor")
    if not isinstance(k, torch.Tensor) or k.dim() != 4:
        raise ValueError("k: expected a [B, Hkv, N, d] tensor")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    _want(q, "q", torch.bfloat16)
    _want(k, "k", torch.bfloat16, (B, Hkv, N, d), q.device)
    if v is not None:
        _want(v, "v", torch.bfloat16, (B, Hkv, N, d), q.device)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def make_shape(B, Hq, Hkv, N, d, causal, softmax_scale: float = 0.0) -> Shape:
    return Shape(int(B), int(Hq), int(Hkv), int(N), int(d), int(bool(causal)), float(softmax_scale))


def shape_of(q: torch.Tensor, k: torch.Tensor, causal: bool, softmax_scale: float = 0.0) -> Shape:
    B, Hq, N, d = q.shape
    return make_shape(B, Hq, k.shape[1], N, d, causal, softmax_scale)


def quant_bytes(shape: Shape, field: int) -> int:
    return int(lib().thrift_quant_bytes(ctypes.byref(shape), field))


def workspace_bytes(shape: Shape, op: int) -> int:
    return int(lib().thrift_workspace_bytes(ctypes.byref(shape), op))


@dataclasses.dataclass
class Quantized:
    """The quantised operands (device tensors), in thrift_quant field order, and their FP4 format."""
    tensors: dict
    fmt: str = "nvfp4"

    def struct(self) -> QuantStruct:
        return QuantStruct(*[self.tensors[f].data_ptr() for f in QUANT_FIELDS])

    def __getitem__(self, k):
        return self.tensors[k]


def _check_quantized(quant: "Quantized", shape: Shape, device) -> None:
    for idx, f in enumerate(QUANT_FIELDS):
        t = quant.tensors.get(f)
        if t is None:
            raise ValueError(f"quantized operands: missing {f}")
        _want(t, f, _FIELD_DTYPES.get(f, torch.uint8), device=device)
        if t.numel() * t.element_size() < quant_bytes(shape, idx):
            raise ValueError(f"{f}: {t.numel() * t.element_size()} bytes, the shape needs {quant_bytes(shape, idx)}")


def alloc_quantized(shape: Shape, device) -> Quantized:
    out = {}
    for idx, f in enumerate(QUANT_FIELDS):
        nbytes = quant_bytes(shape, idx)
        if nbytes == 0:
            raise ThriftError(THRIFT_ERR_INVALID, "thrift_quant_bytes")
        dt = _FIELD_DTYPES.get(f, torch.uint8)
        out[f] = torch.empty(nbytes // torch.empty((), dtype=dt).element_size(), dtype=dt, device=device)
    return Quantized(out)


def _workspace(shape: Shape, op: int, device) -> Optional[torch.Tensor]:
    n = workspace_bytes(shape, op)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device) if n > 0 else None


def _want_fmt(fmt: str) -> None:
    if fmt not in FORMATS:
        raise ValueError(f"fmt: {fmt!r}, expected one of {FORMATS}")


def quantize(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
             out: Optional[Quantized] = None, ws: Optional[torch.Tensor] = None, fmt: str = "nvfp4") -> Quantized:
    """thrift_quantize (fmt "nvfp4") or thrift_quantize_mx (fmt "mxfp4"): FP4 Q, K and FP8 V
    (all device tensors)."""
    _want_fmt(fmt)
    _check_qkv(q, k, v)
    shape = shape_of(q, k, causal)
    if out is None:
        out = alloc_quantized(shape, q.device)
    else:
        _check_quantized(out, shape, q.device)
    op = OP_QUANTIZE if fmt == "nvfp4" else OP_QUANTIZE_MX
    if ws is not None:
        _want(ws, "ws", torch.uint8, device=q.device)
        if ws.numel() < workspace_bytes(shape, op):
            raise ValueError(f"ws: {ws.numel()} bytes, the shape needs {workspace_bytes(shape, op)}")
    ws = ws if ws is not None else _workspace(shape, op, q.device)
    st = out.struct()
    fn = lib().thrift_quantize if fmt == "nvfp4" else lib().thrift_quantize_mx
    _check(fn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(st), _ptr(ws),
              0 if ws is None else ws.numel(), _stream()),
           "thrift_quantize" if fmt == "nvfp4" else "thrift_quantize_mx")
    out.fmt = fmt
    return out


def select(q: torch.Tensor, k: torch.Tensor, causal: bool, budget_bp: int = 500, budget_tiles: int = 0,
           mask: Optional[torch.Tensor] = None, counts: Optional[torch.Tensor] = None,
           ws: Optional[torch.Tensor] = None, mode: str = "score"):
    """thrift_select (mode "score") or thrift_select_vertical (mode "vertical"):
    returns (mask[B,Hq,T,W] int32 view of the uint32 words, counts[B,Hq,T])."""
    if mode not in ("score", "vertical"):
        raise ValueError(f"mode: {mode!r}, expected 'score' or 'vertical'")
    _check_qkv(q, k)
    shape = shape_of(q, k, causal)
    B, Hq, N, _ = q.shape
    T = (N + 127) // 128
    W = (T + 31) // 32
    if mask is None:
        mask = torch.empty((B, Hq, T, W), dtype=torch.int32, device=q.device)
    else:
        _want(mask, "mask", torch.int32, (B, Hq, T, W), q.device)
    if counts is None:
        counts = torch.empty((B, Hq, T), dtype=torch.int32, device=q.device)
    else:
        _want(counts, "counts", torch.int32, (B, Hq, T), q.device)
    op = OP_SELECT if mode == "score" else OP_SELECT_VERTICAL
    if ws is not None:
        _want(ws, "ws", torch.uint8, device=q.device)
    ws = ws if ws is not None else _workspace(shape, op, q.device)
    fn = lib().thrift_select if mode == "score" else lib().thrift_select_vertical
    _check(fn(ctypes.byref(shape), _ptr(q), _ptr(k), int(budget_bp), int(budget_tiles), _ptr(mask), _ptr(counts),
              _ptr(ws), 0 if ws is None else ws.numel(), _stream()),
           "thrift_select" if mode == "score" else "thrift_select_vertical")
    return mask, counts


def attn_fwd(q: torch.Tensor, k: torch.Tensor, quant: Quantized, mask: torch.Tensor, causal: bool,
             softmax_scale: float = 0.0, o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             want_lse: bool = False):
    """thrift_attn_fwd (NVFP4 operands) or thrift_attn_fwd_mx (MXFP4 operands, by quant.fmt):
    returns (o[B,Hq,N,d] bf16, lse[B,Hq,N] fp32 or None)."""
    _want_fmt(quant.fmt)
    _check_qkv(q, k)
    shape = shape_of(q, k, causal, softmax_scale)
    B, Hq, N, _ = q.shape
    T = (N + 127) // 128
    _check_quantized(quant, shape, q.device)
    _want(mask, "mask", torch.int32, (B, Hq, T, (T + 31) // 32), q.device)
    if o is None:
        o = torch.empty_like(q)
    else:
        _want(o, "o", torch.bfloat16, tuple(q.shape), q.device)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    elif lse is not None:
        _want(lse, "lse", torch.float32, tuple(q.shape[:3]), q.device)
    st = quant.struct()
    if quant.fmt == "nvfp4":
        _check(lib().thrift_attn_fwd(ctypes.byref(shape), ctypes.byref(st), _ptr(q), _ptr(k), _ptr(mask),
                                     _ptr(o), _ptr(lse), None, 0, _stream()), "thrift_attn_fwd")
    else:
        _check(lib().thrift_attn_fwd_mx(ctypes.byref(shape), ctypes.byref(st), _ptr(q), _ptr(k), _ptr(mask),
                                        _ptr(o), _ptr(lse), _stream()), "thrift_attn_fwd_mx")
    return o, lse


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool, budget_bp: int = 500,
              budget_tiles: int = 0, softmax_scale: float = 0.0, want_lse: bool = False, mode: str = "score",
              fmt: str = "nvfp4"):
    """The whole forward pass: quantize (NVFP4 or MXFP4) -> select (score or vertical mode) ->
    fused mixed attention."""
    quant = quantize(q, k, v, causal, fmt=fmt)
    mask, _ = select(q, k, causal, budget_bp, budget_tiles, mode=mode)
    return attn_fwd(q, k, quant, mask, causal, softmax_scale, want_lse=want_lse)


def decode_shape(q: torch.Tensor, k: torch.Tensor, softmax_scale: float = 0.0) -> DecodeShape:
    B, Hq, d = q.shape
    return DecodeShape(int(B), int(Hq), int(k.shape[1]), int(k.shape[2]), int(d), float(softmax_scale))


def _check_decode_kv(k: torch.Tensor, v: torch.Tensor) -> None:
    if not isinstance(k, torch.Tensor) or k.dim() != 4:
        raise ValueError("k: expected a [B, Hkv, L, d] tensor")
    _want(k, "k", torch.bfloat16)
    _want(v, "v", torch.bfloat16, tuple(k.shape), k.device)


def decode_quantize_cache(k: torch.Tensor, v: torch.Tensor, cache: Optional[dict] = None, t_begin: int = 0,
                          t_end: Optional[int] = None) -> dict:
    """thrift_decode_quantize_cache: per-token MXFP4 K / MXFP8 V of cache rows [t_begin, t_end).
    Returns the cache dict (kc, ksc, vc, vsc uint8 device tensors), allocated when not given."""
    _check_decode_kv(k, v)
    B, Hkv, L, d = k.shape
    shape = DecodeShape(int(B), int(Hkv), int(Hkv), int(L), int(d), 0.0)
    if cache is None:
        cache = {}
        for idx, f in enumerate(DECODE_FIELDS):
            n = int(lib().thrift_decode_cache_bytes(ctypes.byref(shape), idx))
            if n == 0:
                raise ThriftError(THRIFT_ERR_INVALID, "thrift_decode_cache_bytes")
            cache[f] = torch.empty(n, dtype=torch.uint8, device=k.device)
    else:
        for idx, f in enumerate(DECODE_FIELDS):
            _want(cache[f], f, torch.uint8, device=k.device)
            if cache[f].numel() < int(lib().thrift_decode_cache_bytes(ctypes.byref(shape), idx)):
                raise ValueError(f"{f}: buffer too small for the cache shape")
    st = DecodeCacheStruct(*[cache[f].data_ptr() for f in DECODE_FIELDS])
    t_end = L if t_end is None else t_end
    _check(lib().thrift_decode_quantize_cache(ctypes.byref(shape), _ptr(k), _ptr(v), ctypes.byref(st),
                                              int(t_begin), int(t_end), _stream()), "thrift_decode_quantize_cache")
    return cache


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cache: dict, softmax_scale: float = 0.0,
                o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = False,
                ws: Optional[torch.Tensor] = None):
    """thrift_decode_step: q[B,Hq,d] against the cache -> (o[B,Hq,d] bf16, lse[B,Hq] fp32 or None)."""
    _check_decode_kv(k, v)
    if not isinstance(q, torch.Tensor) or q.dim() != 3:
        raise ValueError("q: expected a [B, Hq, d] tensor")
    _want(q, "q", torch.bfloat16, device=k.device)
    B, Hkv, L, d = k.shape
    if q.shape[0] != B or q.shape[2] != d:
        raise ValueError(f"q: shape {tuple(q.shape)} does not match the cache {tuple(k.shape)}")
    shape = decode_shape(q, k, softmax_scale)
    for idx, f in enumerate(DECODE_FIELDS):
        _want(cache[f], f, torch.uint8, device=k.device)
        if cache[f].numel() < int(lib().thrift_decode_cache_bytes(ctypes.byref(shape), idx)):
            raise ValueError(f"{f}: buffer too small for the cache shape")
    if o is None:
        o = torch.empty_like(q)
    else:
        _want(o, "o", torch.bfloat16, tuple(q.shape), k.device)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=k.device)
    elif lse is not None:
        _want(lse, "lse", torch.float32, tuple(q.shape[:2]), k.device)
    need = int(lib().thrift_decode_workspace_bytes(ctypes.byref(shape)))
    if need == 0:
        raise ThriftError(THRIFT_ERR_UNSUPPORTED, "thrift_decode_workspace_bytes")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=k.device)
    else:
        _want(ws, "ws", torch.uint8, device=k.device)
    st = DecodeCacheStruct(*[cache[f].data_ptr() for f in DECODE_FIELDS])
    _check(lib().thrift_decode_step(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(st), _ptr(o),
                                    _ptr(lse), _ptr(ws), ws.numel(), _stream()), "thrift_decode_step")
    return o, lse


def device_status() -> tuple:
    """Synchronise the current stream and read (status, raw word) of the device watchdog."""
    w = ctypes.c_uint32(0)
    s = lib().thrift_device_status(_stream(), ctypes.byref(w))
    return int(s), int(w.value)


def debug_withhold_v_load(tile: int) -> None:
    """Watchdog test hook: later attention launches skip key tile `tile`'s V load (-1: off)."""
    _check(lib().thrift_debug_withhold_v_load(int(tile)), "thrift_debug_withhold_v_load")


def probe_mma(kind: int, n: int = 128, iters: int = 20000, ctas: Optional[int] = None) -> dict:
    """thrift_probe_mma: dense tensor-core rate of one MMA form (kind 0 NVFP4, 1 e4m3 with A in
    tensor memory, 2 BF16), one CTA per SM by default.  Returns TFLOP/s and cycle figures."""
    if ctas is None:
        ctas = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    cyc = torch.zeros(ctas, dtype=torch.int64, device="cuda")
    ms = ctypes.c_float(0.0)
    _check(lib().thrift_probe_mma(int(kind), int(n), int(iters), int(ctas), ctypes.byref(ms), cyc.data_ptr(),
                                  _stream()), "thrift_probe_mma")
    flops = 2.0 * 128 * n * 128 * iters * ctas
    c = cyc.cpu().double()
    return {"tflops": flops / (ms.value * 1e-3) / 1e12, "ms": float(ms.value),
            "flop_per_clk_per_sm": 2.0 * 128 * n * 128 * iters / float(c.max()),
            "cycles_max": float(c.max()), "ctas": ctas, "iters": iters}


def launch_count() -> int:
    return int(lib().thrift_launch_count())


def version() -> str:
    return lib().thrift_version().decode()
