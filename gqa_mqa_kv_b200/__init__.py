"""B200-native grouped-query attention (GQA): decode and multi-token (prefill) steps.

A thin ctypes binding over ``libgqa_decode.so`` (the C ABI in
``include/gqa_decode.h``).  Every step of the computation runs in the
library's CUDA kernels; this module only checks tensor shapes, fills the
parameter struct, hands over device pointers and the current CUDA stream,
and translates status codes into exceptions.  PyTorch provides the device
memory and the stream.

    out = gqa_decode(q, k_cache, v_cache, seq_lens)                 # contiguous
    out = gqa_decode(q, k_pages, v_pages, seq_lens, block_table)    # paged

There is no fallback: if the library is missing or was not built for this
GPU the call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading

__all__ = [
    "GqaError", "Params", "gqa_decode", "gqa_decode_timed", "gqa_decode_static_workspace",
    "gqa_rope_append", "gqa_decode_fp8kv", "gqa_prefill", "FLAG_BAD_POSITION", "FLAG_BAD_QUERY_SPAN",
    "workspace_bytes", "make_workspace",
    "read_status", "static_workspace_status", "kv_cache_bytes", "library", "LIB_PATH", "FLAG_SEQ_LEN_CLAMPED",
    "FLAG_BAD_BLOCK", "FLAG_TIMEOUT", "PAGE_SIZE",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgqa_decode.so")
PAGE_SIZE = 64
GQA_BF16, GQA_F32 = 0, 1
# gqa_kernel: which split kernel serves a call (all compute the same result)
KERNELS = {"auto": 0, "mma_sync": 1, "tcgen05": 2}
FLAG_SEQ_LEN_CLAMPED, FLAG_BAD_BLOCK, FLAG_TIMEOUT, FLAG_BAD_POSITION, FLAG_BAD_QUERY_SPAN = 1, 2, 4, 8, 16
ROPE_PAIRING = {"adjacent": 0, "halves": 1}

EXPORTED = (
    "gqa_decode_workspace_size", "gqa_decode", "gqa_decode_timed", "gqa_read_status",
    "gqa_kv_cache_bytes", "gqa_status_string", "gqa_version", "gqa_decode_static_workspace",
    "gqa_rope_append", "gqa_decode_fp8kv", "gqa_wait_selftest", "gqa_prefill_workspace_size",
    "gqa_prefill", "gqa_static_workspace_status",
)


class GqaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_status_string(status)} (status {status})")


class Params(ctypes.Structure):
    """Mirror of gqa_decode_params."""

    _fields_ = [
        ("B", ctypes.c_int32), ("H_Q", ctypes.c_int32), ("H_KV", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("qkv_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("kernel", ctypes.c_int32),
    ]

    def key(self):
        return tuple(getattr(self, f) for f, _ in self._fields_)


_lib = None
_lock = threading.Lock()


def library() -> ctypes.CDLL:
    """Load libgqa_decode.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m gqa_mqa_kv_b200.build` "
                    "(there is no CPU fallback)")
            lib = ctypes.CDLL(LIB_PATH)
            vp, sz = ctypes.c_void_p, ctypes.c_size_t
            pp = ctypes.POINTER(Params)
            lib.gqa_decode_workspace_size.argtypes = [pp, ctypes.POINTER(sz)]
            lib.gqa_decode_workspace_size.restype = ctypes.c_int
            lib.gqa_decode.argtypes = [pp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, sz, vp]
            lib.gqa_decode.restype = ctypes.c_int
            lib.gqa_decode_timed.argtypes = [pp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, sz,
                                             vp, vp, vp]
            lib.gqa_decode_timed.restype = ctypes.c_int
            lib.gqa_read_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
            lib.gqa_read_status.restype = ctypes.c_int
            lib.gqa_kv_cache_bytes.argtypes = [ctypes.c_int64] * 5
            lib.gqa_kv_cache_bytes.restype = ctypes.c_uint64
            lib.gqa_status_string.argtypes = [ctypes.c_int]
            lib.gqa_status_string.restype = ctypes.c_char_p
            lib.gqa_version.argtypes = []
            lib.gqa_version.restype = ctypes.c_int
            lib.gqa_decode_static_workspace.argtypes = [pp, vp, vp, vp, vp, vp, ctypes.c_float, vp,
                                                        vp]
            lib.gqa_decode_static_workspace.restype = ctypes.c_int
            lib.gqa_static_workspace_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
            lib.gqa_static_workspace_status.restype = ctypes.c_int
            lib.gqa_rope_append.argtypes = [pp, vp, vp, vp, vp, vp, ctypes.c_double, ctypes.c_int, vp,
                                            vp, vp, vp, vp, vp]
            lib.gqa_rope_append.restype = ctypes.c_int
            lib.gqa_decode_fp8kv.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, sz,
                                             vp]
            lib.gqa_decode_fp8kv.restype = ctypes.c_int
            lib.gqa_prefill_workspace_size.argtypes = [pp, ctypes.POINTER(sz)]
            lib.gqa_prefill_workspace_size.restype = ctypes.c_int
            lib.gqa_prefill.argtypes = [pp, vp, vp, ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp,
                                        ctypes.c_float, vp, vp, sz, vp]
            lib.gqa_prefill.restype = ctypes.c_int
            lib.gqa_wait_selftest.argtypes = [ctypes.c_uint64, ctypes.c_int, vp, vp, vp]
            lib.gqa_wait_selftest.restype = ctypes.c_int
            _lib = lib
    return _lib


def _status_string(status: int) -> str:
    try:
        return library().gqa_status_string(status).decode()
    except Exception:  # pragma: no cover - only when the library itself is missing
        return "unknown"


def _dtype_code(dtype) -> int:
    import torch

    if dtype == torch.bfloat16:
        return GQA_BF16
    if dtype == torch.float32:
        return GQA_F32
    raise TypeError(f"unsupported dtype {dtype}: use torch.bfloat16 or torch.float32")


def make_params(q, k_cache, seq_lens, block_table=None, out_dtype=None, max_seq_len=None,
                kernel="auto") -> Params:
    """Fill gqa_decode_params from tensor shapes (no device work)."""
    import torch

    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, H_Q, D]; caches must be 4-D")
    B, H_Q, D = q.shape
    p = Params()
    p.B, p.H_Q, p.head_dim = B, H_Q, D
    p.H_KV = k_cache.shape[2]
    if k_cache.shape[3] != D:
        raise ValueError("cache head_dim differs from q")
    if block_table is None:
        if k_cache.shape[0] != B:
            raise ValueError("contiguous cache must be [B, S_max, H_KV, D]")
        p.max_seq_len = k_cache.shape[1] if max_seq_len is None else int(max_seq_len)
        p.page_size = p.max_blocks_per_seq = p.num_blocks = 0
    else:
        if k_cache.shape[1] != PAGE_SIZE:
            raise ValueError(f"paged cache must be [num_blocks, {PAGE_SIZE}, H_KV, D]")
        if block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError("block_table must be [B, max_blocks_per_seq]")
        p.page_size = PAGE_SIZE
        p.max_blocks_per_seq = block_table.shape[1]
        p.num_blocks = k_cache.shape[0]
        p.max_seq_len = (p.max_blocks_per_seq * PAGE_SIZE if max_seq_len is None
                         else int(max_seq_len))
    p.qkv_dtype = _dtype_code(q.dtype)
    p.out_dtype = _dtype_code(torch.float32 if out_dtype is None else out_dtype)
    if kernel not in KERNELS:
        raise ValueError(f"kernel must be one of {sorted(KERNELS)}")
    p.kernel = KERNELS[kernel]
    return p


def workspace_bytes(params: Params) -> int:
    n = ctypes.c_size_t(0)
    st = library().gqa_decode_workspace_size(ctypes.byref(params), ctypes.byref(n))
    if st != 0:
        raise GqaError(st, "gqa_decode_workspace_size")
    return int(n.value)


_ws_cache: dict = {}


def make_workspace(params: Params, device) -> "torch.Tensor":
    """A zero-filled workspace for these parameters (cached per device and shape)."""
    import torch

    dev = torch.device(device)
    key = (dev.index, params.key())
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(workspace_bytes(params), dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def _check_inputs(q, k_cache, v_cache, seq_lens, block_table):
    import torch

    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("seq_lens", seq_lens)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype:
        raise ValueError("k_cache and v_cache must match in shape and dtype")
    if q.dtype != k_cache.dtype:
        raise ValueError("q and the caches must share a dtype")
    if seq_lens.dtype != torch.int32 or seq_lens.shape != (q.shape[0],):
        raise ValueError("seq_lens must be int32 [B]")
    if block_table is not None:
        if not block_table.is_cuda or not block_table.is_contiguous() or block_table.dtype != torch.int32:
            raise ValueError("block_table must be a contiguous int32 CUDA tensor")


def _call(q, k_cache, v_cache, seq_lens, block_table, scale, out, out_dtype, workspace, stream,
          events, max_seq_len, kernel="auto"):
    import torch

    _check_inputs(q, k_cache, v_cache, seq_lens, block_table)
    params = make_params(q, k_cache, seq_lens, block_table, out_dtype if out is None else out.dtype,
                         max_seq_len, kernel)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or torch.float32, device=q.device)
    elif out.shape != q.shape or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor shaped like q")
    if workspace is None:
        workspace = make_workspace(params, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    bt = ctypes.c_void_p(block_table.data_ptr() if block_table is not None else None)
    args = [ctypes.byref(params), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k_cache.data_ptr()),
            ctypes.c_void_p(v_cache.data_ptr()), ctypes.c_void_p(seq_lens.data_ptr()), bt,
            ctypes.c_float(scale), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(workspace.numel()), sp]
    lib = library()
    if events is None:
        st = lib.gqa_decode(*args)
    else:
        for ev in events:  # torch creates the CUDA event on its first record
            if ev.cuda_event == 0:
                ev.record(stream)
        st = lib.gqa_decode_timed(*args, ctypes.c_void_p(events[0].cuda_event),
                                  ctypes.c_void_p(events[1].cuda_event))
    if st != 0:
        raise GqaError(st, "gqa_decode")
    return out


def gqa_decode(q, k_cache, v_cache, seq_lens, block_table=None, scale=None, out=None,
               out_dtype=None, workspace=None, stream=None, max_seq_len=None, kernel="auto"):
    """One GQA decode step on the GPU.

    q            [B, H_Q, D] bf16 or f32 (CUDA)
    k_cache,     contiguous [B, S_max, H_KV, D], or paged [num_blocks, 64, H_KV, D]
    v_cache
    seq_lens     int32 [B] cached tokens per sequence (newest included)
    block_table  int32 [B, max_blocks_per_seq] for a paged cache
    scale        softmax scale (default 1/sqrt(D))
    out          optional [B, H_Q, D] output (f32 default, or bf16)
    kernel       "auto", "mma_sync" or "tcgen05" (gqa_kernel)
    Returns out.  Enqueued on ``stream`` (default: the current stream); no sync.
    """
    return _call(q, k_cache, v_cache, seq_lens, block_table, scale, out, out_dtype, workspace,
                 stream, None, max_seq_len, kernel)


def gqa_decode_timed(events, q, k_cache, v_cache, seq_lens, block_table=None, scale=None,
                     out=None, out_dtype=None, workspace=None, stream=None, max_seq_len=None,
                     kernel="auto"):
    """gqa_decode with torch.cuda.Event pair ``events`` recorded around the split kernel."""
    return _call(q, k_cache, v_cache, seq_lens, block_table, scale, out, out_dtype, workspace,
                 stream, events, max_seq_len, kernel)


def gqa_decode_static_workspace(q, k_cache, v_cache, seq_lens, block_table=None, scale=None,
                                out=None, out_dtype=None, stream=None, max_seq_len=None):
    """gqa_decode on the library's built-in 8 MiB workspace: this call allocates nothing.

    For callers that cannot call cudaMalloc (a plugin whose host application
    owns all device memory, a loop that must not take cudaMalloc's implicit
    device synchronisation).  ``out`` must be given for a call that allocates
    nothing; without it a fresh output tensor is created here.  Calls whose
    kernels overlap on the GPU share the one built-in workspace and race; the
    first call on a device should come before any stream capture.
    """
    import torch

    _check_inputs(q, k_cache, v_cache, seq_lens, block_table)
    params = make_params(q, k_cache, seq_lens, block_table, out_dtype if out is None else out.dtype,
                         max_seq_len)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or torch.float32, device=q.device)
    elif out.shape != q.shape or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor shaped like q")
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    bt = ctypes.c_void_p(block_table.data_ptr() if block_table is not None else None)
    st = library().gqa_decode_static_workspace(
        ctypes.byref(params), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k_cache.data_ptr()),
        ctypes.c_void_p(v_cache.data_ptr()), ctypes.c_void_p(seq_lens.data_ptr()), bt,
        ctypes.c_float(scale), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
    if st != 0:
        raise GqaError(st, "gqa_decode_static_workspace")
    return out


def gqa_rope_append(q, k_new, v_new, positions, k_cache, v_cache, block_table=None,
                    rope_base=10000.0, pairing="adjacent", q_out=None, seq_lens_out=None,
                    workspace=None, stream=None, max_seq_len=None):
    """RoPE on the new token's query heads (returned) and key heads, appended with
    its value rows to the cache at positions[b]; optionally seq_lens_out[b] = positions[b] + 1.

    q [B, H_Q, D]; k_new, v_new [B, H_KV, D]; positions int32 [B]; caches as in
    gqa_decode.  q_out may be q itself.  Enqueued on the current stream.
    """
    import torch

    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("positions", positions),
                    ("k_cache", k_cache), ("v_cache", v_cache)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    B, H_Q, D = q.shape
    H_KV = k_cache.shape[2]
    if k_new.shape != (B, H_KV, D) or v_new.shape != k_new.shape:
        raise ValueError("k_new and v_new must be [B, H_KV, D]")
    if positions.dtype != torch.int32 or positions.shape != (B,):
        raise ValueError("positions must be int32 [B]")
    if not (q.dtype == k_new.dtype == v_new.dtype == k_cache.dtype == v_cache.dtype):
        raise ValueError("q, k_new, v_new and the caches must share a dtype")
    params = make_params(q, k_cache, positions, block_table, None, max_seq_len)
    if q_out is None:
        q_out = torch.empty_like(q)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    opt = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else None)  # noqa: E731
    st = library().gqa_rope_append(
        ctypes.byref(params), opt(q), opt(k_new), opt(v_new), opt(positions), opt(block_table),
        ctypes.c_double(rope_base), ROPE_PAIRING[pairing], opt(q_out), opt(k_cache), opt(v_cache),
        opt(seq_lens_out), opt(workspace), ctypes.c_void_p(stream.cuda_stream))
    if st != 0:
        raise GqaError(st, "gqa_rope_append")
    return q_out


def gqa_decode_fp8kv(q, k_cache, v_cache, k_scale, v_scale, seq_lens, block_table=None,
                     scale=None, out=None, out_dtype=None, workspace=None, stream=None,
                     max_seq_len=None, kernel="auto"):
    """gqa_decode over an 8-bit cache: k_cache, v_cache hold E4M3 values
    (torch.float8_e4m3fn or their uint8 bytes) multiplied by per-KV-head
    k_scale, v_scale (float32 [H_KV]).  q is bf16."""
    import torch

    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("seq_lens", seq_lens),
                    ("k_scale", k_scale), ("v_scale", v_scale)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if q.dtype != torch.bfloat16:
        raise ValueError("q must be bf16 for an 8-bit cache")
    if k_cache.dtype not in (torch.float8_e4m3fn, torch.uint8) or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache must be float8_e4m3fn (or uint8 bytes)")
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache must match in shape")
    H_KV = k_cache.shape[2]
    for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        if t.dtype != torch.float32 or t.shape != (H_KV,):
            raise ValueError(f"{name} must be float32 [H_KV]")
    if seq_lens.dtype != torch.int32 or seq_lens.shape != (q.shape[0],):
        raise ValueError("seq_lens must be int32 [B]")
    params = make_params(q, k_cache, seq_lens, block_table, out_dtype if out is None else out.dtype,
                         max_seq_len, kernel)
    params.qkv_dtype = GQA_BF16
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or torch.float32, device=q.device)
    if workspace is None:
        workspace = make_workspace(params, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    opt = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else None)  # noqa: E731
    st = library().gqa_decode_fp8kv(
        ctypes.byref(params), opt(q), opt(k_cache), opt(v_cache), opt(k_scale), opt(v_scale),
        opt(seq_lens), opt(block_table), ctypes.c_float(scale), opt(out), opt(workspace),
        ctypes.c_size_t(workspace.numel()), ctypes.c_void_p(stream.cuda_stream))
    if st != 0:
        raise GqaError(st, "gqa_decode_fp8kv")
    return out


def gqa_prefill(q, k_cache, v_cache, seq_lens, cu_q_lens, max_q_len=None, block_table=None, scale=None,
                out=None, out_dtype=None, workspace=None, stream=None, max_seq_len=None, kernel="auto"):
    """Multi-token causal GQA (prefill, or a prompt chunk after a cached prefix) on the GPU.

    q            [total_q, H_Q, 128] bf16: the new query tokens of every
                 sequence, back to back (rows cu_q_lens[b] .. cu_q_lens[b+1]-1)
    k_cache,     as in gqa_decode, already holding the new tokens' keys and
    v_cache      values as the last n_b of each sequence's seq_lens[b] tokens
    seq_lens     int32 [B]
    cu_q_lens    int32 [B + 1], cu_q_lens[0] = 0, cu_q_lens[B] = total_q
    max_q_len    host bound on every n_b (read from cu_q_lens, with a
                 synchronisation, when not given)
    Token j of sequence b sits at position seq_lens[b] - n_b + j and attends to
    cache positions <= it.  Returns out [total_q, H_Q, 128] (f32 default, or
    bf16), enqueued on ``stream`` (default: the current stream).
    """
    import torch

    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("seq_lens", seq_lens),
                    ("cu_q_lens", cu_q_lens)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [total_q, H_Q, D]; caches must be 4-D")
    if k_cache.shape != v_cache.shape or not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise ValueError("q and the caches must share a dtype; k_cache and v_cache a shape")
    B = seq_lens.shape[0]
    if seq_lens.dtype != torch.int32 or seq_lens.dim() != 1:
        raise ValueError("seq_lens must be int32 [B]")
    if cu_q_lens.dtype != torch.int32 or cu_q_lens.shape != (B + 1,):
        raise ValueError("cu_q_lens must be int32 [B + 1]")
    if block_table is not None and (not block_table.is_cuda or not block_table.is_contiguous()
                                    or block_table.dtype != torch.int32):
        raise ValueError("block_table must be a contiguous int32 CUDA tensor")
    total_q = q.shape[0]
    if max_q_len is None:
        cu = cu_q_lens.cpu()
        max_q_len = int((cu[1:] - cu[:-1]).max().item()) if B > 0 else 0
    # gqa_decode_params from the cache geometry; B comes from seq_lens.
    proxy = torch.empty((B, q.shape[1], q.shape[2]), dtype=q.dtype, device="meta")
    params = make_params(proxy, k_cache, seq_lens, block_table, out_dtype if out is None else out.dtype,
                         max_seq_len, kernel)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or torch.float32, device=q.device)
    elif out.shape != q.shape or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor shaped like q")
    if workspace is None:
        workspace = make_workspace(params, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    opt = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else None)  # noqa: E731
    st = library().gqa_prefill(
        ctypes.byref(params), opt(q), opt(cu_q_lens), int(total_q), int(max_q_len), opt(k_cache), opt(v_cache),
        opt(seq_lens), opt(block_table), ctypes.c_float(scale), opt(out), opt(workspace),
        ctypes.c_size_t(workspace.numel()), ctypes.c_void_p(stream.cuda_stream))
    if st != 0:
        raise GqaError(st, "gqa_prefill")
    return out


def wait_selftest(timeout_ns: int, abort_early: bool = False, device=None):
    """Run the library's bounded-wait self test (gqa_wait_selftest) on the GPU
    and return (flags, elapsed_ns); synchronises the stream."""
    import torch

    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    flags = torch.zeros(1, dtype=torch.int32, device=device)
    elapsed = torch.zeros(1, dtype=torch.int64, device=device)
    stream = torch.cuda.current_stream(device)
    st = library().gqa_wait_selftest(ctypes.c_uint64(int(timeout_ns)), int(bool(abort_early)),
                                     ctypes.c_void_p(flags.data_ptr()), ctypes.c_void_p(elapsed.data_ptr()),
                                     ctypes.c_void_p(stream.cuda_stream))
    if st != 0:
        raise GqaError(st, "gqa_wait_selftest")
    stream.synchronize()
    return int(flags.item()) & 0xFFFFFFFF, int(elapsed.item())


def read_status(workspace, stream=None, clear=False) -> int:
    """GQA_FLAG_* bits accumulated in a workspace (synchronises the stream)."""
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    flags = ctypes.c_uint32(0)
    st = library().gqa_read_status(ctypes.c_void_p(workspace.data_ptr()),
                                   ctypes.c_void_p(stream.cuda_stream), ctypes.byref(flags),
                                   int(bool(clear)))
    if st != 0:
        raise GqaError(st, "gqa_read_status")
    return int(flags.value)


def static_workspace_status(stream=None, clear=False, device=None) -> int:
    """GQA_FLAG_* bits accumulated in the built-in workspace that
    gqa_decode_static_workspace uses on the current device (synchronises the
    stream); ``clear`` resets them."""
    import torch

    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(device):
        st = library().gqa_static_workspace_status(ctypes.c_void_p(stream.cuda_stream), ctypes.byref(flags),
                                                   int(bool(clear)))
    if st != 0:
        raise GqaError(st, "gqa_static_workspace_status")
    return int(flags.value)


def kv_cache_bytes(layers, tokens, h_kv, head_dim, elem_bytes=2) -> int:
    """2 x layers x tokens x H_KV x head_dim x bytes per element (host-side formula)."""
    return int(library().gqa_kv_cache_bytes(int(layers), int(tokens), int(h_kv), int(head_dim),
                                            int(elem_bytes)))
