"""B200-native rotary position embedding fused into FlashAttention forward.

Thin ctypes binding over librfa.so (C ABI in include/rfa.h).  This module only
marshals arguments: it checks that every tensor of a call sits on one CUDA
device (and runs the call with that device current), checks dtypes and
contiguity, passes raw pointers and torch's current CUDA stream of that
device, and turns status codes into exceptions.  Every step of the computation runs in the library's CUDA
kernels.  There is no CPU fallback: if librfa.so is missing the import fails.

Entry points (C name without the ``rfa_`` prefix):
    rope_sincos(position_ids, inv_freq, seq_lens, head_size, out_dtype)
    rope_apply(q, k, sin, cos, ...)   rotated q, k (and a KV-cache write)
    kv_rms_norm_rope_cache(k, v, gamma, eps, sin, cos, slots, k_cache, v_cache)
    decode_rope_attention(q, k_cache, v_cache, q_pos, kv_lens, ...)
    fused_rope_attention(q, k, v, position, ...)
    fused_rope_attention_workspace(...)
    get_device_status()
    status_string(code)
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "RfaError", "LIB_PATH", "CHECKED_LIB_PATH", "EXPORTS", "load_library", "use_library", "rope_sincos", "fused_rope_attention",
    "fused_rope_attention_workspace", "rope_attention_table", "fused_rope_attention_with_table",
    "fused_rope_attention_noalloc", "rope_apply", "kv_rms_norm_rope_cache", "KvCacheParams",
    "decode_rope_attention", "DecodeParams",
    "get_device_status", "set_wait_limit_ns", "set_hold_items", "status_string", "AttnParams", "RopeApplyParams",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librfa.so")
# the bounds-checked build of the same sources (see use_library)
CHECKED_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librfa_checked.so")

# Every symbol include/rfa.h declares.
EXPORTS = (
    "rfa_rope_sincos",
    "rfa_rope_apply",
    "rfa_kv_rms_norm_rope_cache",
    "rfa_decode_rope_attention_workspace",
    "rfa_decode_rope_attention",
    "rfa_fused_rope_attention_workspace",
    "rfa_fused_rope_attention",
    "rfa_rope_attention_table",
    "rfa_fused_rope_attention_with_table",
    "rfa_fused_rope_attention_noalloc",
    "rfa_get_device_status",
    "rfa_set_wait_limit_ns",
    "rfa_set_hold_items",
    "rfa_status_string",
    "rfa_version",
)

RFA_OK, RFA_ERR_INVALID_ARG, RFA_ERR_UNSUPPORTED, RFA_ERR_WORKSPACE, RFA_ERR_CUDA, RFA_ERR_TIMEOUT = range(6)
DT_UNDEFINED, DT_FP16, DT_BF16, DT_FP32 = range(4)
LAYOUT_BNSD, LAYOUT_TND = 0, 1
_TORCH_DT = {torch.float16: DT_FP16, torch.bfloat16: DT_BF16, torch.float32: DT_FP32}


class RfaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {status_string(code)} ({code})")


class AttnParams(ctypes.Structure):
    """Mirror of rfa_attn_params."""
    _fields_ = [
        ("B", ctypes.c_int32),
        ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("S", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("layout", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("rope_interleaved", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("ntk_enable", ctypes.c_int32),
        ("ntk_train_len", ctypes.c_int32),
        ("ntk_factor", ctypes.c_double),
    ]


class RopeApplyParams(ctypes.Structure):
    """Mirror of rfa_rope_apply_params."""
    _fields_ = [
        ("layout", ctypes.c_int32),
        ("T", ctypes.c_int32),
        ("B", ctypes.c_int32),
        ("S", ctypes.c_int32),
        ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32),
        ("table_dtype", ctypes.c_int32),
        ("interleaved", ctypes.c_int32),
    ]


class KvCacheParams(ctypes.Structure):
    """Mirror of rfa_kv_cache_params."""
    _fields_ = [
        ("T", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32),
        ("table_dtype", ctypes.c_int32),
        ("interleaved", ctypes.c_int32),
        ("eps", ctypes.c_float),
    ]


class DecodeParams(ctypes.Structure):
    """Mirror of rfa_decode_params."""
    _fields_ = [
        ("B", ctypes.c_int32),
        ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("Sq", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("Smax", ctypes.c_int32),
        ("max_kv_len", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32),
        ("rope_interleaved", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("num_splits", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
    ]


_lib = None


def load_library():
    """Load librfa.so (built in-tree by __graft_entry__.build())."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _open(LIB_PATH)
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Run this module's calls against another build of the library for the
    duration of the block -- e.g. librfa_checked.so, the same sources compiled
    with every device-side index bounds-checked (RFA_CHECKED)."""
    global _lib
    prev = load_library()
    _lib = _open(path)
    try:
        yield _lib
    finally:
        _lib = prev


def _open(path: str):
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} is not built ({path}); run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.rfa_rope_sincos.argtypes = [P, P, P, I32, I32, I32, ctypes.c_int, P, P, P]
    lib.rfa_rope_sincos.restype = ctypes.c_int
    lib.rfa_fused_rope_attention_workspace.argtypes = [ctypes.POINTER(AttnParams), I64]
    lib.rfa_fused_rope_attention_workspace.restype = SZ
    lib.rfa_fused_rope_attention.argtypes = [ctypes.POINTER(AttnParams), P, P, P, P, P, P, P, P, SZ, P]
    lib.rfa_fused_rope_attention.restype = ctypes.c_int
    lib.rfa_rope_attention_table.argtypes = [ctypes.POINTER(AttnParams), P, P, P, P, SZ, P]
    lib.rfa_rope_attention_table.restype = ctypes.c_int
    lib.rfa_fused_rope_attention_with_table.argtypes = [ctypes.POINTER(AttnParams), P, P, P, P, P, P, SZ, P]
    lib.rfa_fused_rope_attention_with_table.restype = ctypes.c_int
    lib.rfa_fused_rope_attention_noalloc.argtypes = [ctypes.POINTER(AttnParams), P, P, P, P, P, P, P, P]
    lib.rfa_fused_rope_attention_noalloc.restype = ctypes.c_int
    lib.rfa_rope_apply.argtypes = [ctypes.POINTER(RopeApplyParams), P, P, P, P, P, P, P, P, I64, P]
    lib.rfa_rope_apply.restype = ctypes.c_int
    lib.rfa_kv_rms_norm_rope_cache.argtypes = [ctypes.POINTER(KvCacheParams), P, P, P, P, P, P, P, P, I64, P]
    lib.rfa_kv_rms_norm_rope_cache.restype = ctypes.c_int
    lib.rfa_decode_rope_attention_workspace.argtypes = [ctypes.POINTER(DecodeParams)]
    lib.rfa_decode_rope_attention_workspace.restype = SZ
    lib.rfa_decode_rope_attention.argtypes = [ctypes.POINTER(DecodeParams), P, P, P, P, P, P, P, P, SZ, P]
    lib.rfa_decode_rope_attention.restype = ctypes.c_int
    lib.rfa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.rfa_set_wait_limit_ns.restype = ctypes.c_int
    lib.rfa_set_hold_items.argtypes = [I32]
    lib.rfa_set_hold_items.restype = ctypes.c_int
    lib.rfa_get_device_status.argtypes = [P]
    lib.rfa_get_device_status.restype = ctypes.c_int
    lib.rfa_status_string.argtypes = [ctypes.c_int]
    lib.rfa_status_string.restype = ctypes.c_char_p
    lib.rfa_version.argtypes = []
    lib.rfa_version.restype = I32
    return lib


def set_wait_limit_ns(ns: int) -> None:
    """Kernel role-to-role wait limit on the current device (0: default 2 s);
    for failure-detection tests (rfa_set_wait_limit_ns)."""
    _check(load_library().rfa_set_wait_limit_ns(int(ns)), "rfa_set_wait_limit_ns")


def set_hold_items(on: bool) -> None:
    """Failure-detection switch on the current device (rfa_set_hold_items): while
    on, the attention kernels publish no work item and their waits run out."""
    _check(load_library().rfa_set_hold_items(1 if on else 0), "rfa_set_hold_items")


def status_string(code: int) -> str:
    return load_library().rfa_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != RFA_OK:
        raise RfaError(code, where)


def _stream_ptr(stream=None, device: Optional[torch.device] = None):
    """The stream the library enqueues on: `stream`, else torch's current
    stream of `device`.  A stream of another device is refused (the library
    launches on the current device, which _on_device makes `device`)."""
    s = stream if stream is not None else torch.cuda.current_stream(device)
    if device is not None and s.device != device:
        raise ValueError(f"stream is on {s.device}, the tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _same_device(**tensors) -> torch.device:
    """The one CUDA device every given tensor (None entries skipped) lives on.

    The library reads its pointers on the current device (TMA tensor maps
    included), so a tensor on another GPU would be dereferenced as peer
    memory; such a call is refused here instead."""
    pairs = []
    for name, t in tensors.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        pairs.append((name, t.device))
    return _one_device(pairs)


def _one_device(pairs) -> torch.device:
    """The device shared by every (name, device) pair; raises if they differ."""
    dev = None
    first = None
    for name, d in pairs:
        if dev is None:
            dev, first = d, name
        elif d != dev:
            raise ValueError(f"{name} is on {d}, {first} on {dev}: all tensors must be on one GPU")
    if dev is None:
        raise ValueError("no CUDA tensor given")
    return dev


def rope_sincos(position_ids: torch.Tensor, inv_freq: torch.Tensor, seq_lens: torch.Tensor, head_size: int,
                out_dtype=torch.float16, sin_out: Optional[torch.Tensor] = None,
                cos_out: Optional[torch.Tensor] = None, stream=None):
    """sin, cos [ntokens, head_size] of cat(outer(pos_b, invFreq_b), same).

    position_ids int32 [ntokens], inv_freq fp32 [batch, head_size/2] and
    seq_lens int32 [batch] live on the GPU (as on the DynamicNTK operator).
    """
    T = position_ids.numel()
    batch = seq_lens.numel()
    dev = _same_device(position_ids=position_ids, inv_freq=inv_freq, seq_lens=seq_lens, sin_out=sin_out,
                       cos_out=cos_out)
    if sin_out is None:
        sin_out = torch.empty((T, head_size), dtype=out_dtype, device=dev)
    if cos_out is None:
        cos_out = torch.empty((T, head_size), dtype=out_dtype, device=dev)
    with torch.cuda.device(dev):
        code = load_library().rfa_rope_sincos(
            _dev(position_ids, "position_ids", torch.int32), _dev(inv_freq, "inv_freq", torch.float32),
            _dev(seq_lens, "seq_lens", torch.int32), batch, T, int(head_size),
            _TORCH_DT.get(sin_out.dtype, DT_UNDEFINED), _dev(sin_out, "sin_out"), _dev(cos_out, "cos_out"),
            _stream_ptr(stream, dev))
    _check(code, "rfa_rope_sincos")
    return sin_out, cos_out


def rope_apply(q: Optional[torch.Tensor], k: Optional[torch.Tensor], sin: torch.Tensor, cos: torch.Tensor, *,
               layout: str = "TND", interleaved: bool = False, inplace: bool = False,
               q_out: Optional[torch.Tensor] = None, k_out: Optional[torch.Tensor] = None,
               cache_slots: Optional[torch.Tensor] = None, k_cache: Optional[torch.Tensor] = None,
               keys_out: bool = True, stream=None):
    """Rotated (q, k) from sin/cos tables [tokens, D] (rfa_rope_apply).

    layout "TND": q [T, Hq, D], k [T, Hkv, D]; "BNSD": q [B, Hq, S, D],
    k [B, Hkv, S, D] with table row b*S + s.  Either of q, k may be None.
    inplace writes over q and k.  cache_slots (int32 [tokens]) and k_cache
    ([rows, Hkv, D]) also write the rotated keys to k_cache[cache_slots[t]]
    (negative slots skipped); keys_out=False then skips the separate k output.
    Returns (q_out, k_out) (None where not produced).
    """
    x0 = q if q is not None else k
    if x0 is None:
        raise ValueError("q or k is required")
    if layout == "TND":
        if x0.dim() != 3:
            raise ValueError("TND tensors are [T, H, D]")
        T, D = x0.shape[0], x0.shape[2]
        B = S = 0
        rows = T
    elif layout == "BNSD":
        if x0.dim() != 4:
            raise ValueError("BNSD tensors are [B, H, S, D]")
        B, S, D = x0.shape[0], x0.shape[2], x0.shape[3]
        T = 0
        rows = B * S
    else:
        raise ValueError(f"layout {layout!r}")
    io = _TORCH_DT.get(x0.dtype)
    if io not in (DT_FP16, DT_BF16):
        raise TypeError("q/k must be float16 or bfloat16")
    tab = _TORCH_DT.get(sin.dtype)
    if tab is None or cos.dtype != sin.dtype:
        raise TypeError("sin/cos must share one of float16, bfloat16, float32")
    if tuple(sin.shape) != (rows, D) or tuple(cos.shape) != (rows, D):
        raise ValueError(f"sin/cos must be [{rows}, {D}]")
    hax = 1
    Hq = int(q.shape[hax]) if q is not None else 0
    Hkv = int(k.shape[hax]) if k is not None else 0
    for t, name in ((q, "q"), (k, "k")):
        if t is not None and (t.dtype != x0.dtype or t.dim() != x0.dim()):
            raise ValueError(f"{name} must match the other input's dtype and layout")
    if q is not None:
        q_out = q if inplace else (q_out if q_out is not None else torch.empty_like(q))
    if k is not None and (keys_out or k_cache is None):
        k_out = k if inplace else (k_out if k_out is not None else torch.empty_like(k))
    else:
        k_out = None
    p = RopeApplyParams(LAYOUT_TND if layout == "TND" else LAYOUT_BNSD, T, B, S, Hq, Hkv, D, io, tab,
                        1 if interleaved else 0)
    dev = _same_device(q=q, k=k, sin=sin, cos=cos, q_out=q_out if q is not None else None, k_out=k_out,
                       cache_slots=cache_slots, k_cache=k_cache)
    nul = ctypes.c_void_p(None)
    slots_p = _dev(cache_slots, "cache_slots", torch.int32) if cache_slots is not None else nul
    cache_p = _dev(k_cache, "k_cache", x0.dtype) if k_cache is not None else nul
    rows_cache = int(k_cache.shape[0]) if k_cache is not None else 0
    with torch.cuda.device(dev):
        code = load_library().rfa_rope_apply(
            ctypes.byref(p), _dev(q, "q") if q is not None else nul, _dev(k, "k") if k is not None else nul,
            _dev(sin, "sin"), _dev(cos, "cos"), _dev(q_out, "q_out") if q is not None else nul,
            _dev(k_out, "k_out") if k_out is not None else nul, slots_p, cache_p, rows_cache,
            _stream_ptr(stream, dev))
    _check(code, "rfa_rope_apply")
    return (q_out if q is not None else None), k_out


def _params(q, k, layout, seq_lens, causal, scale, rope_base, ntk_train_len, ntk_factor,
            interleaved=False) -> AttnParams:
    if layout == "BNSD":
        B, Hq, S, D = q.shape
        Hkv = k.shape[1]
        lay = LAYOUT_BNSD
    elif layout == "TND":
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        B, S, lay = len(seq_lens), 0, LAYOUT_TND
    else:
        raise ValueError("layout must be 'BNSD' or 'TND'")
    p = AttnParams()
    p.B, p.Hq, p.Hkv, p.S, p.D, p.layout = B, Hq, Hkv, S, D, lay
    p.causal = 1 if causal else 0
    p.io_dtype = _TORCH_DT.get(q.dtype, DT_UNDEFINED)
    p.scale = 0.0 if scale is None else float(scale)
    p.rope_base = float(rope_base)
    p.ntk_enable = 1 if ntk_train_len else 0
    p.ntk_train_len = int(ntk_train_len or 0)
    p.ntk_factor = float(ntk_factor)
    p.rope_interleaved = 1 if interleaved else 0
    return p


def fused_rope_attention_workspace(q, k, *, layout="BNSD", seq_lens=None, causal=True, scale=None,
                                   rope_base=10000.0, ntk_train_len=0, ntk_factor=1.0, interleaved=False) -> int:
    p = _params(q, k, layout, seq_lens, causal, scale, rope_base, ntk_train_len, ntk_factor, interleaved)
    T = p.B * p.S if layout == "BNSD" else int(sum(int(x) for x in seq_lens))
    return int(load_library().rfa_fused_rope_attention_workspace(ctypes.byref(p), T))


def _lens_arg(layout, seq_lens, p):
    if layout != "TND":
        return None, p.B * p.S
    arr = (ctypes.c_int32 * p.B)(*[int(x) for x in seq_lens])
    return arr, sum(int(x) for x in seq_lens)


def _need(p, T) -> int:
    need = int(load_library().rfa_fused_rope_attention_workspace(ctypes.byref(p), T))
    if need == 0:
        _check(RFA_ERR_INVALID_ARG if p.io_dtype == DT_UNDEFINED else RFA_ERR_UNSUPPORTED,
               "rfa_fused_rope_attention_workspace")
    return need


def _ptr_or_null(arr):
    return None if arr is None else ctypes.cast(arr, ctypes.c_void_p)


def kv_rms_norm_rope_cache(k: torch.Tensor, v: torch.Tensor, gamma: torch.Tensor, eps: float, sin: torch.Tensor,
                           cos: torch.Tensor, slots: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, *,
                           interleaved: bool = False, stream=None):
    """RMSNorm(k) * gamma, rotated with the token's sin/cos row, into
    k_cache[slots[t]]; v into v_cache[slots[t]] (rfa_kv_rms_norm_rope_cache).
    k, v [T, Hkv, D]; gamma fp32 [D]; sin/cos [T, D]; slots int32 [T];
    caches [rows, Hkv, D].  Writes the caches in place and returns them."""
    if k.dim() != 3 or v.shape != k.shape:
        raise ValueError("k and v must both be [T, Hkv, D]")
    T, Hkv, D = k.shape
    io = _TORCH_DT.get(k.dtype)
    if io not in (DT_FP16, DT_BF16):
        raise TypeError("k/v must be float16 or bfloat16")
    tab = _TORCH_DT.get(sin.dtype)
    if tab is None or cos.dtype != sin.dtype:
        raise TypeError("sin/cos must share one of float16, bfloat16, float32")
    if tuple(sin.shape) != (T, D) or tuple(cos.shape) != (T, D):
        raise ValueError(f"sin/cos must be [{T}, {D}]")
    if k_cache.dim() != 3 or tuple(k_cache.shape[1:]) != (Hkv, D) or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [rows, Hkv, D]")
    p = KvCacheParams(T, Hkv, D, io, tab, 1 if interleaved else 0, float(eps))
    dev = _same_device(k=k, v=v, gamma=gamma, sin=sin, cos=cos, slots=slots, k_cache=k_cache, v_cache=v_cache)
    with torch.cuda.device(dev):
        code = load_library().rfa_kv_rms_norm_rope_cache(
            ctypes.byref(p), _dev(k, "k"), _dev(v, "v", k.dtype), _dev(gamma, "gamma", torch.float32),
            _dev(sin, "sin"), _dev(cos, "cos"), _dev(slots, "slots", torch.int32), _dev(k_cache, "k_cache", k.dtype),
            _dev(v_cache, "v_cache", k.dtype), int(k_cache.shape[0]), _stream_ptr(stream, dev))
    _check(code, "rfa_kv_rms_norm_rope_cache")
    return k_cache, v_cache


def decode_rope_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, q_pos: torch.Tensor,
                          kv_lens: torch.Tensor, *, max_kv_len: Optional[int] = None, causal: bool = True,
                          scale: Optional[float] = None, rope_base: float = 10000.0,
                          inv_freq: Optional[torch.Tensor] = None, interleaved: bool = False,
                          num_splits: int = 0, out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """A decode step over a KV cache (rfa_decode_rope_attention).

    q [B, Hq, Sq, D] new tokens (rotated in the kernel at q_pos [B, Sq]);
    k_cache / v_cache [B, Smax, Hkv, D] with keys already rotated; kv_lens
    int32 [B] on the GPU (each in [Sq, max_kv_len]; max_kv_len defaults to
    Smax).  num_splits: parts each sequence's keys are split into across CTAs
    (0: the library's plan).  Returns out [B, Hq, Sq, D].
    """
    if q.dim() != 4 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q [B, Hq, Sq, D]; caches [B, Smax, Hkv, D]")
    B, Hq, Sq, D = q.shape
    Smax, Hkv = int(k_cache.shape[1]), int(k_cache.shape[2])
    p = DecodeParams(B, Hq, Hkv, Sq, D, Smax, int(max_kv_len if max_kv_len is not None else Smax), 1 if causal else 0,
                     _TORCH_DT.get(q.dtype, DT_UNDEFINED), 1 if interleaved else 0,
                     0.0 if scale is None else float(scale), int(num_splits), float(rope_base))
    lib = load_library()
    dev = _same_device(q=q, k_cache=k_cache, v_cache=v_cache, q_pos=q_pos, kv_lens=kv_lens, inv_freq=inv_freq,
                       out=out, workspace=workspace)
    with torch.cuda.device(dev):
        need = int(lib.rfa_decode_rope_attention_workspace(ctypes.byref(p)))
        if need == 0:
            _check(RFA_ERR_INVALID_ARG, "rfa_decode_rope_attention_workspace")
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        if out is None:
            out = torch.empty_like(q)
        io = (torch.bfloat16, torch.float16)
        code = lib.rfa_decode_rope_attention(
            ctypes.byref(p), _dev(q, "q", io), _dev(k_cache, "k_cache", q.dtype), _dev(v_cache, "v_cache", q.dtype),
            _dev(q_pos, "q_pos", torch.int32), _dev(kv_lens, "kv_lens", torch.int32),
            None if inv_freq is None else _dev(inv_freq, "inv_freq", torch.float32), _dev(out, "out", q.dtype),
            _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream_ptr(stream, dev))
    _check(code, "rfa_decode_rope_attention")
    return out


def rope_attention_table(q, k, position: torch.Tensor, *, layout: str = "BNSD", seq_lens=None, causal=True,
                         scale=None, rope_base: float = 10000.0, ntk_train_len: int = 0, ntk_factor: float = 1.0,
                         inv_freq: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                         interleaved: bool = False, stream=None) -> torch.Tensor:
    """Build the cos/sin table of this batch's positions into a workspace
    tensor (returned), for reuse by fused_rope_attention_with_table (the table
    is the same for both pairings)."""
    p = _params(q, k, layout, seq_lens, causal, scale, rope_base, ntk_train_len, ntk_factor, interleaved)
    lens, T = _lens_arg(layout, seq_lens, p)
    dev = _same_device(q=q, k=k, position=position, inv_freq=inv_freq, workspace=workspace)
    need = _need(p, T)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        code = load_library().rfa_rope_attention_table(
            ctypes.byref(p), _dev(position, "position", torch.int32), _ptr_or_null(lens),
            None if inv_freq is None else _dev(inv_freq, "inv_freq", torch.float32), _dev(workspace, "workspace"),
            workspace.numel() * workspace.element_size(), _stream_ptr(stream, dev))
    _check(code, "rfa_rope_attention_table")
    return workspace


def fused_rope_attention_with_table(q, k, v, table: torch.Tensor, *, layout: str = "BNSD", seq_lens=None,
                                    causal=True, scale=None, rope_base: float = 10000.0, ntk_train_len: int = 0,
                                    ntk_factor: float = 1.0, out: Optional[torch.Tensor] = None,
                                    interleaved: bool = False, stream=None) -> torch.Tensor:
    """The attention kernel alone, reading a table from rope_attention_table."""
    p = _params(q, k, layout, seq_lens, causal, scale, rope_base, ntk_train_len, ntk_factor, interleaved)
    lens, T = _lens_arg(layout, seq_lens, p)
    dev = _same_device(q=q, k=k, v=v, table=table, out=out)
    if out is None:
        out = torch.empty_like(q)
    io = (torch.bfloat16, torch.float16)
    with torch.cuda.device(dev):
        code = load_library().rfa_fused_rope_attention_with_table(
            ctypes.byref(p), _dev(q, "q", io), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype), _ptr_or_null(lens),
            _dev(out, "out", q.dtype), _dev(table, "table"), table.numel() * table.element_size(),
            _stream_ptr(stream, dev))
    _check(code, "rfa_fused_rope_attention_with_table")
    return out


def fused_rope_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, position: torch.Tensor, *,
                         layout: str = "BNSD", seq_lens: Optional[Sequence[int]] = None, causal: bool = True,
                         scale: Optional[float] = None, rope_base: float = 10000.0, ntk_train_len: int = 0,
                         ntk_factor: float = 1.0, inv_freq: Optional[torch.Tensor] = None,
                         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                         interleaved: bool = False, stream=None) -> torch.Tensor:
    """softmax(rope(q) rope(k)^T * scale) v, rotated q/k kept on chip.

    BNSD: q [B,Hq,S,D], k/v [B,Hkv,S,D], position int32 [B,S].
    TND : q [T,Hq,D], k/v [T,Hkv,D], position int32 [T], seq_lens (host ints).
    ntk_train_len > 0 enables dynamic NTK with factor ntk_factor.
    interleaved: adjacent pairs (2i, 2i+1) instead of rotate-half pairs.
    inv_freq: optional fp32 [B, D/2] on the GPU.
    """
    p = _params(q, k, layout, seq_lens, causal, scale, rope_base, ntk_train_len, ntk_factor, interleaved)
    lens, T = _lens_arg(layout, seq_lens, p)
    dev = _same_device(q=q, k=k, v=v, position=position, inv_freq=inv_freq, out=out, workspace=workspace)
    need = _need(p, T)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty_like(q)
    io = (torch.bfloat16, torch.float16)
    with torch.cuda.device(dev):
        code = load_library().rfa_fused_rope_attention(
            ctypes.byref(p), _dev(q, "q", io), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype),
            _dev(position, "position", torch.int32), _ptr_or_null(lens),
            None if inv_freq is None else _dev(inv_freq, "inv_freq", torch.float32),
            _dev(out, "out", q.dtype), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
            _stream_ptr(stream, dev))
    _check(code, "rfa_fused_rope_attention")
    return out


def fused_rope_attention_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, position: torch.Tensor, *,
                                 layout: str = "BNSD", seq_lens: Optional[Sequence[int]] = None, causal: bool = True,
                                 scale: Optional[float] = None, rope_base: float = 10000.0, ntk_train_len: int = 0,
                                 ntk_factor: float = 1.0, inv_freq: Optional[torch.Tensor] = None,
                                 out: Optional[torch.Tensor] = None, interleaved: bool = False, stream=None) -> torch.Tensor:
    """fused_rope_attention with the library's fixed internal scratch instead of
    a caller workspace (for callers that cannot allocate device memory; see
    rfa_fused_rope_attention_noalloc in include/rfa.h for limits and the
    one-scratch-per-device rule)."""
    p = _params(q, k, layout, seq_lens, causal, scale, rope_base, ntk_train_len, ntk_factor, interleaved)
    lens, _ = _lens_arg(layout, seq_lens, p)
    dev = _same_device(q=q, k=k, v=v, position=position, inv_freq=inv_freq, out=out)
    if out is None:
        out = torch.empty_like(q)
    io = (torch.bfloat16, torch.float16)
    with torch.cuda.device(dev):
        code = load_library().rfa_fused_rope_attention_noalloc(
            ctypes.byref(p), _dev(q, "q", io), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype),
            _dev(position, "position", torch.int32), _ptr_or_null(lens),
            None if inv_freq is None else _dev(inv_freq, "inv_freq", torch.float32), _dev(out, "out", q.dtype),
            _stream_ptr(stream, dev))
    _check(code, "rfa_fused_rope_attention_noalloc")
    return out


def get_device_status(stream=None, device=None) -> int:
    """Synchronise the stream and return/clear the status word of its device
    (the stream's device, else `device`, else the current device)."""
    if stream is not None:
        device = stream.device
    if device is None:
        return int(load_library().rfa_get_device_status(_stream_ptr(stream)))
    with torch.cuda.device(device):
        return int(load_library().rfa_get_device_status(_stream_ptr(stream, torch.device(device))))


# C names, for callers that prefer them.
rfa_rope_sincos = rope_sincos
rfa_fused_rope_attention = fused_rope_attention
rfa_fused_rope_attention_workspace = fused_rope_attention_workspace
rfa_rope_attention_table = rope_attention_table
rfa_fused_rope_attention_with_table = fused_rope_attention_with_table
rfa_fused_rope_attention_noalloc = fused_rope_attention_noalloc
rfa_get_device_status = get_device_status
rfa_status_string = status_string


def attention_flops(lens, Hq: int, D: int, causal: bool = True) -> float:
    """Algorithmic FLOPs of the two attention GEMMs: 4*D*Hq*sum(S_b(S_b+1)/2)
    causal (masked work not counted), 4*D*Hq*sum(S_b^2) otherwise."""
    tot = 0
    for s in lens:
        s = int(s)
        tot += s * (s + 1) // 2 if causal else s * s
    return 4.0 * D * Hq * tot


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
