"""TEST INFRASTRUCTURE -- the fp64 CPU oracle for GQA decode and multi-token (prefill) attention.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference arm may import this package.  The product library
(``gqa_mqa_kv_b200``) never imports it, and the two share no code.

The arithmetic lives in ``gqa_oracle.cpp`` (plain C++17, double precision,
``std::thread`` over (batch, query-head) pairs); this module only compiles it
with g++ and marshals arguments through ctypes.  See the header comment of
``gqa_oracle.cpp`` for what is computed and which page passage each step
follows.

Every function is pinned by tests in ``tests/test_oracle_pins.py``
(printed KV-cache table, closed forms, library special cases, brute force).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.cpp")
_LIB = os.path.join(_HERE, "libgqa_oracle.so")
_lock = threading.Lock()
_lib = None

IN_BF16, IN_F32, IN_F64, IN_E4M3 = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile gqa_oracle.cpp into libgqa_oracle.so next to it (g++, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp],
            check=True,
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # ORACLE_LIB points the wrapper at another build of gqa_oracle.cpp
            # (the mutation tests use it to run the pins against planted mistakes).
            lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
            vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_gqa_decode.argtypes = [vp, i32, vp, vp, i32, vp, i32, i32, i32, i32, i64,
                                              dbl, vp, i64, vp, i32]
            lib.oracle_gqa_decode.restype = i32
            lib.oracle_attention_weights.argtypes = [vp, i32, vp, i32, vp, i32, i32, i32, i32, i64,
                                                     dbl, i32, i32, vp]
            lib.oracle_attention_weights.restype = i32
            lib.oracle_partial.argtypes = [vp, i32, vp, vp, i32, vp, i32, i32, i32, i32, i64, dbl,
                                           i32, i32, i64, i64, vp, vp]
            lib.oracle_partial.restype = i32
            lib.oracle_lse_combine.argtypes = [i64, vp, vp, i32, vp]
            lib.oracle_lse_combine.restype = i32
            lib.oracle_kv_cache_bytes.argtypes = [i64, i64, i64, i64, i64]
            lib.oracle_kv_cache_bytes.restype = dbl
            lib.oracle_rope.argtypes = [vp, i32, i32, i32, i32, vp, dbl, i32, vp]
            lib.oracle_gqa_decode_scaled.argtypes = [vp, i32, vp, vp, i32, vp, vp, vp, i32, i32, i32,
                                                     i32, i64, dbl, vp, i64, vp, i32]
            lib.oracle_gqa_decode_scaled.restype = i32
            lib.oracle_e4m3_table.argtypes = [vp]
            lib.oracle_e4m3_table.restype = None
            lib.oracle_rope.restype = i32
            lib.oracle_gqa_prefill.argtypes = [vp, i32, vp, vp, i32, vp, vp, i32, i32, i32, i32, i64,
                                               dbl, vp, i64, vp, i32]
            lib.oracle_gqa_prefill.restype = i32
            lib.oracle_hardware_threads.argtypes = []
            lib.oracle_hardware_threads.restype = i32
            _lib = lib
    return _lib


def _as_array(x):
    """Return (contiguous numpy array, oracle dtype code) for a torch tensor or ndarray.

    bf16 tensors are passed as their raw 16-bit patterns; the oracle widens
    them to double exactly.
    """
    try:
        import torch
    except ImportError:  # pragma: no cover - torch is always present here
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), IN_BF16
        if x.dtype == torch.float32:
            return x.numpy(), IN_F32
        if x.dtype == torch.float64:
            return x.numpy(), IN_F64
        if x.dtype == torch.float8_e4m3fn:
            return x.view(torch.uint8).numpy(), IN_E4M3
        raise TypeError(f"oracle: unsupported dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, IN_BF16
    if x.dtype == np.float32:
        return x, IN_F32
    if x.dtype == np.float64:
        return x, IN_F64
    raise TypeError(f"oracle: unsupported dtype {x.dtype}")


def _lens(seq_lens):
    try:
        import torch
        if isinstance(seq_lens, torch.Tensor):
            seq_lens = seq_lens.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def gqa_decode(q, k, v, seq_lens, scale, pairs=None, n_threads=0):
    """fp64 decode attention.

    q [B,H_Q,D]; k, v [B,S_max,H_KV,D] (logical contiguous cache); seq_lens [B].
    Returns float64 [B,H_Q,D], or [n,D] for an explicit list of (b, h) pairs.
    """
    qa, qt = _as_array(q)
    ka, kt = _as_array(k)
    va, vt = _as_array(v)
    if kt != vt:
        raise TypeError("oracle: k and v must share a dtype")
    lens = _lens(seq_lens)
    B, H_Q, D = qa.shape
    Bk, S_max, H_KV, Dk = ka.shape
    if Bk != B or Dk != D or va.shape != ka.shape or lens.shape != (B,):
        raise ValueError("oracle: inconsistent shapes")
    if pairs is None:
        out = np.zeros((B, H_Q, D), dtype=np.float64)
        pp, n = None, 0
    else:
        pa = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        out = np.zeros((pa.shape[0], D), dtype=np.float64)
        pp, n = _ptr(pa), pa.shape[0]
    rc = _load().oracle_gqa_decode(_ptr(qa), qt, _ptr(ka), _ptr(va), kt, _ptr(lens), B, H_Q, H_KV,
                                   D, S_max, float(scale), pp, n, _ptr(out), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_gqa_decode rejected its arguments")
    return out


def gqa_prefill(q, k, v, seq_lens, cu_q, scale, rows=None, n_threads=0):
    """fp64 multi-token causal attention.

    q [total_q, H_Q, D] (rows cu_q[b] .. cu_q[b+1]-1 belong to sequence b);
    k, v [B, S_max, H_KV, D] logical contiguous cache; seq_lens [B]; cu_q [B+1].
    Query row j of sequence b sits at position seq_lens[b] - n_b + j and sees
    cache positions t <= that position.  Returns float64 [total_q, H_Q, D], or
    [n, D] for an explicit list of (row, head) pairs.
    """
    qa, qt = _as_array(q)
    ka, kt = _as_array(k)
    va, vt = _as_array(v)
    if kt != vt:
        raise TypeError("oracle: k and v must share a dtype")
    lens = _lens(seq_lens)
    cu = _lens(cu_q)
    T, H_Q, D = qa.shape
    B, S_max, H_KV, Dk = ka.shape
    if Dk != D or va.shape != ka.shape or lens.shape != (B,) or cu.shape != (B + 1,) or int(cu[-1]) != T:
        raise ValueError("oracle: inconsistent shapes")
    if rows is None:
        out = np.zeros((T, H_Q, D), dtype=np.float64)
        rp, n = None, 0
    else:
        ra = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 2))
        out = np.zeros((ra.shape[0], D), dtype=np.float64)
        rp, n = _ptr(ra), ra.shape[0]
    rc = _load().oracle_gqa_prefill(_ptr(qa), qt, _ptr(ka), _ptr(va), kt, _ptr(lens), _ptr(cu), B, H_Q,
                                    H_KV, D, S_max, float(scale), rp, n, _ptr(out), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_gqa_prefill rejected its arguments")
    return out


def gqa_decode_scaled(q, k, v, seq_lens, scale, k_scale, v_scale, pairs=None, n_threads=0):
    """fp64 decode over a cache whose stored K/V are multiplied by per-KV-head
    factors (k_scale, v_scale [H_KV]); k, v may be torch.float8_e4m3fn."""
    qa, qt = _as_array(q)
    ka, kt = _as_array(k)
    va, vt = _as_array(v)
    if kt != vt:
        raise TypeError("oracle: k and v must share a dtype")
    ks = np.ascontiguousarray(np.asarray(k_scale, dtype=np.float64))
    vs = np.ascontiguousarray(np.asarray(v_scale, dtype=np.float64))
    lens = _lens(seq_lens)
    B, H_Q, D = qa.shape
    Bk, S_max, H_KV, Dk = ka.shape
    if Bk != B or Dk != D or va.shape != ka.shape or ks.shape != (H_KV,) or vs.shape != (H_KV,):
        raise ValueError("oracle: inconsistent shapes")
    if pairs is None:
        out = np.zeros((B, H_Q, D), dtype=np.float64)
        pp, n = None, 0
    else:
        pa = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        out = np.zeros((pa.shape[0], D), dtype=np.float64)
        pp, n = _ptr(pa), pa.shape[0]
    rc = _load().oracle_gqa_decode_scaled(_ptr(qa), qt, _ptr(ka), _ptr(va), kt, _ptr(ks), _ptr(vs),
                                          _ptr(lens), B, H_Q, H_KV, D, S_max, float(scale), pp, n,
                                          _ptr(out), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_gqa_decode_scaled rejected its arguments")
    return out


def e4m3_table():
    """float64 [256]: the oracle's decoded value of every E4M3 byte."""
    out = np.zeros(256, dtype=np.float64)
    _load().oracle_e4m3_table(_ptr(out))
    return out


def attention_weights(q, k, seq_lens, scale, b, h):
    """Normalised softmax weights (float64 [L_b]) of query head h in batch row b."""
    qa, qt = _as_array(q)
    ka, kt = _as_array(k)
    lens = _lens(seq_lens)
    B, H_Q, D = qa.shape
    _, S_max, H_KV, _ = ka.shape
    w = np.zeros(max(int(lens[b]), 1), dtype=np.float64)
    rc = _load().oracle_attention_weights(_ptr(qa), qt, _ptr(ka), kt, _ptr(lens), B, H_Q, H_KV, D,
                                          S_max, float(scale), int(b), int(h), _ptr(w))
    if rc != 0:
        raise ValueError("oracle_attention_weights rejected its arguments")
    return w[: int(lens[b])]


def partial(q, k, v, seq_lens, scale, b, h, t0, t1):
    """(lse, o) of one (b, h) over tokens [t0, t1): natural-log LSE, normalised o [D]."""
    qa, qt = _as_array(q)
    ka, kt = _as_array(k)
    va, _ = _as_array(v)
    lens = _lens(seq_lens)
    B, H_Q, D = qa.shape
    _, S_max, H_KV, _ = ka.shape
    lse = np.zeros(1, dtype=np.float64)
    o = np.zeros(D, dtype=np.float64)
    rc = _load().oracle_partial(_ptr(qa), qt, _ptr(ka), _ptr(va), kt, _ptr(lens), B, H_Q, H_KV, D,
                                S_max, float(scale), int(b), int(h), int(t0), int(t1), _ptr(lse),
                                _ptr(o))
    if rc != 0:
        raise ValueError("oracle_partial rejected its arguments")
    return float(lse[0]), o


def lse_combine(lse, o):
    """Merge partials: lse [n], o [n, D] -> out [D] (float64)."""
    la = np.ascontiguousarray(np.asarray(lse, dtype=np.float64))
    oa = np.ascontiguousarray(np.asarray(o, dtype=np.float64))
    n, D = oa.shape
    out = np.zeros(D, dtype=np.float64)
    rc = _load().oracle_lse_combine(n, _ptr(la), _ptr(oa), D, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_lse_combine rejected its arguments")
    return out


def kv_cache_bytes(layers, tokens, h_kv, d, elem_bytes=2):
    """2 x layers x tokens x KV heads x head dim x bytes per element."""
    return _load().oracle_kv_cache_bytes(int(layers), int(tokens), int(h_kv), int(d),
                                         int(elem_bytes))


def rope(x, positions, base=10000.0, pairing="adjacent"):
    """fp64 rotary embedding of x [B, H, D] at positions [B] -> float64 [B, H, D].

    pairing "adjacent" rotates (2i, 2i+1); "halves" rotates (i, i + D/2).
    """
    xa, xt = _as_array(x)
    pa = _lens(positions)
    B, H, D = xa.shape
    out = np.zeros((B, H, D), dtype=np.float64)
    code = {"adjacent": 0, "halves": 1}[pairing]
    rc = _load().oracle_rope(_ptr(xa), xt, B, H, D, _ptr(pa), float(base), code, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_rope rejected its arguments")
    return out


def hardware_threads() -> int:
    """Threads the oracle uses by default (std::thread::hardware_concurrency)."""
    return int(_load().oracle_hardware_threads())
