"""fp64 CPU oracle for fused RoPE + attention and the DynamicNTK sin/cos table.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The product library never
imports this package and this package never loads the product library.

The arithmetic lives in ``rfa_oracle.c`` (plain loops, fp64, pthreads); this
module only compiles it with gcc and marshals numpy arrays.  What each call
computes, with the passage it follows:

* ``inv_freq``     invFreq_j = base^(-2j/D) -- page "RoPE fused into attention
  on Ascend", section 1.2 (the freqs line of the RoPE snippet).
* ``ntk_base``     base' = base*((f*S/L)-(f-1))^(D/(D-2)) when S > L, else base --
  page "DynamicNTKOperation", function description (no interpolation up to the
  training length, an enlarged base beyond it).  The closed form itself is not
  printed on that page (its InvFreqs formula was lost); this is the dynamic-NTK
  form named for the long-context workload.
* ``rope_sincos``  freq = outer(positionIds_b, invFreq_b); emb = cat(freq, freq);
  sin/cos of emb -- page "DynamicNTKOperation", computation process.
* ``rope_rotate``  rotate-half: x' = x*cos + rotate_half(x)*sin.
* ``rope_apply``   the Rope operator on given sin/cos tables: q, k, sin, cos
  in, rotated q, k out -- page "DynamicNTKOperation", operator context;
  out = x*cos + rot(x)*sin with rotate-half pairs, or adjacent pairs
  (x1,x2),(x3,x4),... -- page "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE", sec. 6.
* ``rms_norm``     gamma * x / sqrt(mean(x^2) + eps) -- same page, sec. 8.
* ``decode_attention``  the decode step over a KV cache (page "RoPE, RMSNorm,
  GQA/MQA, SwiGLU, MoE", sec. 12-13: every decode step reads the cached K/V,
  shared by a group of query heads): the Sq new tokens' queries, rotated at
  their positions, attend to the cached keys (rotated when written) and
  values; new token s of a sequence with L cached keys sees keys [0, L-Sq+s]
  (its own and earlier positions: the new tokens are the last Sq entries).
  Plain numpy in fp64, full score rows, two-pass softmax.
* ``kv_rms_norm_rope_cache``  the fused cache-write op named on page "RoPE
  fused into attention on Ascend" (sec. 5.2, kv_rms_norm_rope_cache): per
  token and kv head, RMSNorm of k, then the Rope operator, into the K cache at
  the token's slot; v into the V cache at the same slot; negative slots are
  skipped.  Its composition is the reading taken (the page names the op only).
* ``attention_rows`` / ``attention_probs``  softmax(Q'K'^T * scale) V with the
  full score row, two passes -- page "FlashAttention in ops-transformer", the
  attention formula; GQA grouping from page "RoPE, RMSNorm, GQA/MQA", sec. 12.

Pinned by tests/test_oracle_*.py against closed forms, mpmath, numpy's complex
exponential, torch's CPU scaled_dot_product_attention and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rfa_oracle.c")
_LIB = os.path.join(_HERE, "librfa_oracle.so")
_lock = threading.Lock()
_lib = None

BF16, FP16 = 0, 1
BNSD, TND = 0, 1


# Test hook for the mutation tests only: a prebuilt library (a copy of
# rfa_oracle.c with one planted mistake) to load instead of this one.  It is a
# module attribute, not read from the environment: only the mutation tests'
# pytest plugin sets it, in the subprocesses that run the pins against a
# mutant, so no other process can have its checker swapped.
_lib_override = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (only if missing or stale)."""
    if _lib_override:
        return _lib_override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread", _SRC, "-lm", "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class _Desc(ctypes.Structure):
    _fields_ = [
        ("layout", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("B", ctypes.c_int32),
        ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("S", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("scale", ctypes.c_double),
        ("nthreads", ctypes.c_int32),
        ("interleaved", ctypes.c_int32),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            lib.oracle_inv_freq.argtypes = [ctypes.c_double, ctypes.c_int32, P]
            lib.oracle_inv_freq.restype = None
            lib.oracle_ntk_base.argtypes = [ctypes.c_double, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_double]
            lib.oracle_ntk_base.restype = ctypes.c_double
            lib.oracle_rope_sincos.argtypes = [P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P]
            lib.oracle_rope_sincos.restype = ctypes.c_int
            lib.oracle_rope_rotate.argtypes = [P, ctypes.c_int64, ctypes.c_int32, P, P, P]
            lib.oracle_rope_rotate.restype = None
            lib.oracle_rope_apply.argtypes = [P, ctypes.c_int64, ctypes.c_int32, P, P, P, ctypes.c_int32, P]
            lib.oracle_rope_apply.restype = None
            lib.oracle_rms_norm.argtypes = [P, ctypes.c_int64, ctypes.c_int32, P, ctypes.c_double, P]
            lib.oracle_rms_norm.restype = None
            lib.oracle_attention_rows.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, P, P, P, ctypes.c_int64, P]
            lib.oracle_attention_rows.restype = ctypes.c_int
            lib.oracle_attention_probs.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, P, ctypes.c_int32,
                                                   ctypes.c_int32, ctypes.c_int32, P]
            lib.oracle_attention_probs.restype = ctypes.c_int
            lib.oracle_widen16.argtypes = [ctypes.c_uint16, ctypes.c_int]
            lib.oracle_widen16.restype = ctypes.c_double
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def widen16(bits: int, dtype: int = BF16) -> float:
    return _load().oracle_widen16(int(bits), int(dtype))


def inv_freq(base: float, D: int) -> np.ndarray:
    out = np.empty(D // 2, np.float64)
    _load().oracle_inv_freq(float(base), int(D), _ptr(out))
    return out


def ntk_base(base: float, D: int, S: int, L: int, factor: float) -> float:
    return float(_load().oracle_ntk_base(float(base), int(D), int(S), int(L), float(factor)))


def rope_sincos(position_ids, inv_freq_rows, seq_lens, head_size: int):
    """sin, cos [ntokens, head_size] in fp64.  inv_freq_rows [batch, head_size/2]
    (fp32 inputs are widened exactly).  Raises ValueError on bad lengths."""
    pos = _c(position_ids, np.int32)
    inv = _c(inv_freq_rows, np.float64)
    sl = _c(seq_lens, np.int32)
    batch, T = sl.shape[0], pos.shape[0]
    assert inv.shape == (batch, head_size // 2)
    s = np.empty((T, head_size), np.float64)
    c = np.empty((T, head_size), np.float64)
    rc = _load().oracle_rope_sincos(_ptr(pos), _ptr(inv), _ptr(sl), batch, T, head_size, _ptr(s), _ptr(c))
    if rc != 0:
        raise ValueError("seqLens must be positive and sum to ntokens")
    return s, c


def rope_rotate(x, pos, inv_freq_row):
    """Rotate-half RoPE of rows x [n, D] (fp64) at positions pos [n]."""
    x = _c(x, np.float64)
    n, D = x.shape
    p = _c(pos, np.int32)
    inv = _c(inv_freq_row, np.float64)
    assert p.shape == (n,) and inv.shape == (D // 2,)
    out = np.empty_like(x)
    _load().oracle_rope_rotate(_ptr(x), n, D, _ptr(p), _ptr(inv), _ptr(out))
    return out


def rope_apply(x, sin_t, cos_t, table_rows, interleaved: bool = False):
    """Rows x [n, D] (fp64) rotated with table rows sin_t/cos_t[table_rows[r]]
    ([*, D], fp64; 16-bit tables are widened exactly by the caller)."""
    x = _c(x, np.float64)
    n, D = x.shape
    s = _c(sin_t, np.float64)
    c = _c(cos_t, np.float64)
    tr = _c(table_rows, np.int64)
    assert s.shape == c.shape and s.shape[1] == D and tr.shape == (n,)
    assert n == 0 or (tr.min() >= 0 and tr.max() < s.shape[0])
    out = np.empty_like(x)
    _load().oracle_rope_apply(_ptr(x), n, D, _ptr(s), _ptr(c), _ptr(tr), 1 if interleaved else 0, _ptr(out))
    return out


def rms_norm(x, gamma, eps: float):
    """Rows x [n, D] (fp64) -> gamma * x / sqrt(mean(x^2) + eps)."""
    x = _c(x, np.float64)
    n, D = x.shape
    g = _c(gamma, np.float64)
    assert g.shape == (D,)
    out = np.empty_like(x)
    _load().oracle_rms_norm(_ptr(x), n, D, _ptr(g), float(eps), _ptr(out))
    return out


def kv_rms_norm_rope_cache(k, v, gamma, eps, sin_t, cos_t, slots, k_cache, v_cache, interleaved=False):
    """k, v [T, Hkv, D] (fp64 values), tables [T, D]; writes rows into copies
    of k_cache / v_cache [rows, Hkv, D] and returns them (fp64)."""
    k = _c(k, np.float64)
    v = _c(v, np.float64)
    T, H, D = k.shape
    kc = np.array(k_cache, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    kn = rms_norm(k.reshape(T * H, D), gamma, eps)
    kr = rope_apply(kn, sin_t, cos_t, np.repeat(np.arange(T), H), interleaved).reshape(T, H, D)
    for t in range(T):
        sl = int(slots[t])
        if sl >= 0:
            kc[sl] = kr[t]
            vc[sl] = v[t]
    return kc, vc


def decode_attention(q, k_cache, v_cache, q_pos, kv_lens, inv_freq_rows, *, causal=True, scale=None,
                     interleaved=False) -> np.ndarray:
    """q [B, Hq, Sq, D] (new tokens, not rotated), caches [B, Smax, Hkv, D]
    (keys already rotated), q_pos [B, Sq], kv_lens [B], inv_freq_rows [B, D/2]
    -> out [B, Hq, Sq, D] in fp64."""
    qf = _f64_values(q)
    kf = _f64_values(k_cache)
    vf = _f64_values(v_cache)
    B, Hq, Sq, D = qf.shape
    Hkv = kf.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    pos = np.asarray(q_pos, np.int64).reshape(B, Sq)
    inv = np.asarray(inv_freq_rows, np.float64).reshape(B, D // 2)
    out = np.zeros((B, Hq, Sq, D), np.float64)
    for b in range(B):
        L = int(kv_lens[b])
        for h in range(Hq):
            kvh = h // G
            K = kf[b, :L, kvh, :]
            V = vf[b, :L, kvh, :]
            for s in range(Sq):
                th = pos[b, s] * inv[b]  # angle of pair i
                x = qf[b, h, s]
                if interleaved:
                    z = (x[0::2] + 1j * x[1::2]) * np.exp(1j * th)
                    qr = np.empty(D)
                    qr[0::2], qr[1::2] = z.real, z.imag
                else:
                    z = (x[: D // 2] + 1j * x[D // 2:]) * np.exp(1j * th)
                    qr = np.concatenate([z.real, z.imag])
                sc = (K @ qr) * scale
                if causal:
                    sc[L - Sq + s + 1:] = -np.inf
                p = np.exp(sc - sc.max())
                out[b, h, s] = (p / p.sum()) @ V
    return out


def _f64_values(t) -> np.ndarray:
    """bf16/fp16 torch tensors (or numpy arrays) as fp64 values, widened exactly."""
    if hasattr(t, "float"):
        return t.float().cpu().numpy().astype(np.float64)
    return np.asarray(t, np.float64)


def _bits16(t) -> np.ndarray:
    """Raw 16-bit patterns of a bf16/fp16 torch tensor or a uint16 numpy array."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch

    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _dtype_code(t) -> int:
    import torch

    if isinstance(t, np.ndarray):
        raise TypeError("pass torch tensors so the 16-bit format is known")
    return BF16 if t.dtype == torch.bfloat16 else FP16


def _desc(layout, dtype, B, Hq, Hkv, S, D, causal, scale, nthreads, interleaved=False):
    return _Desc(layout, dtype, B, Hq, Hkv, S, D, int(bool(causal)), float(scale),
                 int(nthreads or default_threads()), int(bool(interleaved)))


def attention_rows(q, k, v, position, inv_freq_rows, rows, *, layout=BNSD, seq_lens=None, causal=True,
                   scale=None, nthreads=None, interleaved=False) -> np.ndarray:
    """fp64 attention output for the given (b, h, i) rows -> [nrows, D].

    BNSD: q [B,Hq,S,D], k/v [B,Hkv,S,D], position [B,S].
    TND : q [T,Hq,D],   k/v [T,Hkv,D],   position [T], seq_lens [B].
    inv_freq_rows: [B, D/2] per sequence (float values; fp32 widened exactly).
    """
    dt = _dtype_code(q)
    if layout == BNSD:
        B, Hq, S, D = q.shape
        Hkv = k.shape[1]
        sl = np.zeros(1, np.int32)
    else:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        sl = _c(seq_lens, np.int32)
        B, S = sl.shape[0], 0
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    d = _desc(layout, dt, B, Hq, Hkv, S, D, causal, scale, nthreads, interleaved)
    qb, kb, vb = _bits16(q), _bits16(k), _bits16(v)
    pos = _c(np.asarray(position), np.int32).reshape(-1)
    inv = _c(inv_freq_rows, np.float64).reshape(B, D // 2)
    r = _c(rows, np.int32).reshape(-1, 3)
    out = np.zeros((r.shape[0], D), np.float64)
    rc = _load().oracle_attention_rows(ctypes.byref(d), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(pos), _ptr(sl), _ptr(inv),
                                       _ptr(r), r.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("invalid attention rows or descriptor")
    return out


def attention_probs(q, k, position, inv_freq_rows, b, h, i, *, layout=BNSD, seq_lens=None, causal=True,
                    scale=None, interleaved=False) -> np.ndarray:
    """One full softmax row P[b,h,i,:] in fp64."""
    dt = _dtype_code(q)
    if layout == BNSD:
        B, Hq, S, D = q.shape
        Hkv = k.shape[1]
        sl = np.zeros(1, np.int32)
        L = S
    else:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        sl = _c(seq_lens, np.int32)
        B, S = sl.shape[0], 0
        L = int(sl[b])
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    d = _desc(layout, dt, B, Hq, Hkv, S, D, causal, scale, 1, interleaved)
    qb, kb = _bits16(q), _bits16(k)
    pos = _c(np.asarray(position), np.int32).reshape(-1)
    inv = _c(inv_freq_rows, np.float64).reshape(B, D // 2)
    p = np.zeros(L, np.float64)
    rc = _load().oracle_attention_probs(ctypes.byref(d), _ptr(qb), _ptr(kb), _ptr(pos), _ptr(sl), _ptr(inv), b, h, i,
                                        _ptr(p))
    if rc != 0:
        raise ValueError("invalid row")
    return p


def all_rows(B: int, Hq: int, lens) -> np.ndarray:
    """Every (b, h, i) row of a problem with per-sequence lengths lens."""
    out = []
    for b in range(B):
        L = int(lens[b])
        i = np.arange(L, dtype=np.int32)
        for h in range(Hq):
            out.append(np.stack([np.full(L, b, np.int32), np.full(L, h, np.int32), i], axis=1))
    return np.concatenate(out, axis=0) if out else np.zeros((0, 3), np.int32)


def attention_full(q, k, v, position, inv_freq_rows, *, layout=BNSD, seq_lens=None, causal=True, scale=None,
                   nthreads=None, interleaved=False) -> np.ndarray:
    """Full fp64 output in the layout of q."""
    if layout == BNSD:
        B, Hq, S, D = q.shape
        rows = all_rows(B, Hq, [S] * B)
        out = attention_rows(q, k, v, position, inv_freq_rows, rows, layout=layout, causal=causal, scale=scale,
                             nthreads=nthreads, interleaved=interleaved)
        return out.reshape(B, Hq, S, D)
    T, Hq, D = q.shape
    sl = np.asarray(seq_lens, np.int64)
    rows = all_rows(len(sl), Hq, sl)
    out = attention_rows(q, k, v, position, inv_freq_rows, rows, layout=layout, seq_lens=seq_lens, causal=causal,
                         scale=scale, nthreads=nthreads, interleaved=interleaved)
    full = np.zeros((T, Hq, D), np.float64)
    t0 = np.concatenate([[0], np.cumsum(sl)])
    tok = t0[rows[:, 0]] + rows[:, 2]
    full[tok, rows[:, 1]] = out
    return full
