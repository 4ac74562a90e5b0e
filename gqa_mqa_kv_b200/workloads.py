"""Seeded synthetic decode workloads (inputs only; no attention arithmetic here).

The shapes are the production head layouts the GQA pages tabulate ("Grouped-
Query Attention (GQA) and Multi-Query Attention (MQA): Mathematical
Foundations, Arithmetic Intensity, and KV-Cache Scaling Mechanics",
section 5, "Attention architectures in production": Llama 3 8B with 32/8
heads, Llama 2 70B with 64/8 heads) plus a grouping sweep from MHA to MQA.

Values are N(0, 1).  Each tensor is generated in fixed-size chunks; chunk j of
stream s draws from ``numpy.random.PCG64(SeedSequence((seed, s, ..., j)))``,
so the values do not depend on how many threads generate them.  bf16 tensors
are the round-to-nearest-even bf16 of the float32 draws.

This module is imported by the tests and the benchmark, for the GPU path and
for the CPU oracle alike.  It holds no part of the method's arithmetic.
"""

from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

PAGE_SIZE = 64
_CHUNK = 1 << 22  # elements per independently seeded chunk

# stream ids
_S_Q, _S_K, _S_V, _S_LENS, _S_TABLE = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """One decode step of one attention layer.

    seq_len is the cache length of every sequence, or the upper bound of the
    uniform length draw when ``ragged``.  ``page_size`` 0 means a contiguous
    cache [B, S_max, H_KV, D]; 64 means a paged cache [num_blocks, 64, H_KV, D]
    addressed through a block table.
    """

    name: str
    B: int
    H_Q: int
    H_KV: int
    D: int
    seq_len: int
    dtype: str = "bf16"  # "bf16" or "f32": dtype of q, k and v
    ragged: bool = False
    page_size: int = 0
    seed: int = 0
    scale: float | None = None  # None -> 1/sqrt(D)
    kv8: bool = False  # cache stored as OCP E4M3 bytes with per-KV-head scales

    @property
    def R(self) -> int:
        return self.H_Q // self.H_KV

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    @property
    def max_blocks_per_seq(self) -> int:
        return -(-self.seq_len // self.page_size) if self.page_size else 0

    @property
    def num_blocks(self) -> int:
        return self.B * self.max_blocks_per_seq


def _wl(name, B, H_Q, H_KV, D, L, seed, **kw):
    return Workload(name, B, H_Q, H_KV, D, L, seed=seed, **kw)


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        _wl("tiny", 1, 8, 2, 64, 256, 1, dtype="f32"),
        _wl("llama3_8b", 16, 32, 8, 128, 4096, 2),
        _wl("sweep_hkv32", 32, 32, 32, 128, 8192, 3),
        _wl("sweep_hkv8", 32, 32, 8, 128, 8192, 3),
        _wl("sweep_hkv4", 32, 32, 4, 128, 8192, 3),
        _wl("sweep_hkv2", 32, 32, 2, 128, 8192, 3),
        _wl("sweep_hkv1", 32, 32, 1, 128, 8192, 3),
        _wl("llama2_70b_ragged", 32, 64, 8, 128, 32768, 4, ragged=True),
        _wl("paged_long", 8, 64, 8, 128, 131072, 5, page_size=PAGE_SIZE),
        _wl("llama3_8b_fp8", 16, 32, 8, 128, 4096, 2, kv8=True),
        _wl("llama2_70b_ragged_fp8", 32, 64, 8, 128, 32768, 4, ragged=True, kv8=True),
        _wl("paged_long_fp8", 8, 64, 8, 128, 131072, 5, page_size=PAGE_SIZE, kv8=True),
    ]
}


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _fill_normal(out: torch.Tensor, key: tuple) -> None:
    """Fill a contiguous CPU tensor (bf16/f32/f64) with seeded N(0,1) draws."""
    flat = out.view(-1)
    n = flat.numel()
    nchunks = -(-n // _CHUNK)

    def work(j):
        lo, hi = j * _CHUNK, min(n, (j + 1) * _CHUNK)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(key + (j,))))
        x = rng.standard_normal(hi - lo, dtype=np.float32)
        flat[lo:hi].copy_(torch.from_numpy(x))

    if nchunks <= 1:
        for j in range(nchunks):
            work(j)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))


def _torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def seq_lens_for(w: Workload) -> torch.Tensor:
    """int32 [B]: every sequence at seq_len, or U[1, seq_len] per sequence when ragged."""
    if not w.ragged:
        return torch.full((w.B,), w.seq_len, dtype=torch.int32)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence((w.seed, _S_LENS))))
    return torch.from_numpy(rng.integers(1, w.seq_len + 1, size=w.B).astype(np.int32))


def block_table_for(w: Workload) -> torch.Tensor:
    """int32 [B, max_blocks_per_seq]: a seeded random permutation of all pages."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence((w.seed, _S_TABLE))))
    perm = rng.permutation(w.num_blocks).astype(np.int32)
    return torch.from_numpy(perm).view(w.B, w.max_blocks_per_seq)


def kv_scales(w: Workload) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-KV-head float32 factors of an 8-bit cache (distinct per head)."""
    g = torch.arange(w.H_KV, dtype=torch.float32)
    return (5.0 + 0.5 * g) / 448.0, (5.5 + 0.25 * g) / 448.0


def _quantize_e4m3(x: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """E4M3 bytes of x / scale[head] (heads on dim -2), saturated at +-448."""
    y = (x.float() / scale[:, None]).clamp(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn)


def make_inputs(w: Workload, pad_value: float = 0.0, seq_lens: torch.Tensor | None = None):
    """Generate one decode step's inputs on the host.

    Returns a dict with
      q          [B, H_Q, D]
      k, v       [B, S_max, H_KV, D] logical contiguous cache; rows t >= L_b
                 hold ``pad_value`` (use NaN to prove they are never read)
      seq_lens   int32 [B]
      block_table, k_paged, v_paged   (paged workloads only):
                 k_paged[block_table[b, t // 64], t % 64] == k[b, t]
    """
    dt = _torch_dtype(w.dtype)
    lens = seq_lens_for(w) if seq_lens is None else seq_lens.to(torch.int32).cpu()
    S_max = w.max_blocks_per_seq * w.page_size if w.page_size else w.seq_len
    q = torch.empty(w.B, w.H_Q, w.D, dtype=dt)
    _fill_normal(q, (w.seed, _S_Q))
    k = torch.full((w.B, S_max, w.H_KV, w.D), pad_value, dtype=dt)
    v = torch.full((w.B, S_max, w.H_KV, w.D), pad_value, dtype=dt)
    for b in range(w.B):
        L = int(lens[b])
        if L > 0:
            _fill_normal(k[b, :L], (w.seed, _S_K, b))
            _fill_normal(v[b, :L], (w.seed, _S_V, b))
    out = {"q": q, "k": k, "v": v, "seq_lens": lens}
    if w.kv8:
        # The draws above are in bf16; quantise them per KV head to E4M3 bytes.
        ks, vs = kv_scales(w)
        k8 = torch.zeros(k.shape, dtype=torch.uint8)
        v8 = torch.zeros(v.shape, dtype=torch.uint8)
        if pad_value != 0.0:
            k8.fill_(0x7F)  # E4M3 NaN
            v8.fill_(0x7F)
        for b in range(w.B):
            L = int(lens[b])
            if L > 0:
                k8[b, :L] = _quantize_e4m3(k[b, :L], ks).view(torch.uint8)
                v8[b, :L] = _quantize_e4m3(v[b, :L], vs).view(torch.uint8)
        out.update(k=k8.view(torch.float8_e4m3fn), v=v8.view(torch.float8_e4m3fn), k_scale=ks, v_scale=vs)
        k, v = out["k"], out["v"]
    if w.page_size:
        table = block_table_for(w)
        out["block_table"] = table
        out["k_paged"] = to_pages(k, table, w.page_size)
        out["v_paged"] = to_pages(v, table, w.page_size)
    return out


def to_pages(x: torch.Tensor, table: torch.Tensor, page_size: int) -> torch.Tensor:
    """Scatter a logical cache [B, S, H, D] into pages [num_blocks, page, H, D].

    Page j of sequence b (tokens [64j, 64j+64)) lands in physical page
    table[b, j].  Physical pages that no table entry names stay zero.
    """
    B, S, H, D = x.shape
    nb = S // page_size
    assert nb * page_size == S and table.shape == (B, nb)
    num_blocks = int(table.max()) + 1 if table.numel() else 0
    byte_view = x.dtype == torch.float8_e4m3fn
    src = x.view(torch.uint8) if byte_view else x
    pages = torch.zeros(num_blocks, page_size, H, D, dtype=src.dtype)
    pages[table.reshape(-1).long()] = src.reshape(B * nb, page_size, H, D)
    return pages.view(torch.float8_e4m3fn) if byte_view else pages


def algorithmic_bytes(w: Workload, seq_lens: torch.Tensor, out_bytes: int = 4) -> int:
    """Bytes the step must move at minimum: K and V rows actually cached, plus Q and O."""
    e = 2 if w.dtype == "bf16" else 4
    e_kv = 1 if w.kv8 else e
    kv = int(seq_lens.to(torch.int64).sum()) * w.H_KV * w.D * e_kv * 2
    return kv + w.B * w.H_Q * w.D * e + w.B * w.H_Q * w.D * out_bytes


# ---------------------------------------------------------------- multi-token (prefill) steps

_S_QLEN, _S_PREFIX = 5, 6


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    """One multi-token step of one attention layer.

    Every sequence brings ``q_len`` new query tokens (U[1, q_len] when
    ``ragged``) after a cached prefix of ``prefix`` tokens (U[0, prefix] when
    ragged); the new tokens' keys and values are already the last n_b of its
    L_b = prefix_b + n_b cached tokens.  prefix 0 is a fresh prompt.
    """

    name: str
    B: int
    H_Q: int
    H_KV: int
    D: int
    q_len: int
    prefix: int
    seed: int
    ragged: bool = False
    page_size: int = 0

    @property
    def R(self) -> int:
        return self.H_Q // self.H_KV

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def capacity(self) -> int:
        """Cache positions per sequence (a whole number of pages when paged)."""
        n = self.prefix + self.q_len
        return -(-n // self.page_size) * self.page_size if self.page_size else n


PREFILL_WORKLOADS: dict[str, PrefillWorkload] = {
    w.name: w
    for w in [
        # Llama 3 8B heads (32 / 8): four fresh 4096-token prompts.
        PrefillWorkload("prefill_llama3_8b", 4, 32, 8, 128, 4096, 0, seed=11),
        # Llama 2 70B heads (64 / 8): the last 2048-token chunk of 32K-token prompts.
        PrefillWorkload("prefill_llama2_70b_chunk", 4, 64, 8, 128, 2048, 30720, seed=12),
        # Mixed chunk lengths and prefixes over a paged cache.
        PrefillWorkload("prefill_ragged_paged", 8, 64, 8, 128, 1024, 8192, seed=13, ragged=True,
                        page_size=PAGE_SIZE),
    ]
}


def prefill_lengths(w: PrefillWorkload) -> tuple[np.ndarray, np.ndarray]:
    """(n_b, L_b) as int32 arrays [B]."""
    if not w.ragged:
        n = np.full(w.B, w.q_len, dtype=np.int32)
        pre = np.full(w.B, w.prefix, dtype=np.int32)
    else:
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence((w.seed, _S_QLEN))))
        n = rng.integers(1, w.q_len + 1, size=w.B).astype(np.int32)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence((w.seed, _S_PREFIX))))
        pre = rng.integers(0, w.prefix + 1, size=w.B).astype(np.int32)
    return n, (n + pre).astype(np.int32)


def make_prefill_inputs(w: PrefillWorkload, pad_value: float = 0.0, lengths=None):
    """Generate one multi-token step's inputs on the host.

    ``lengths`` = (n_b, L_b) overrides the workload's length draw.

    Returns a dict with
      q          [total_q, H_Q, D] bf16, sequence b's rows at cu_q[b] .. cu_q[b+1]-1
      k, v       [B, capacity, H_KV, D] bf16 logical contiguous cache; rows
                 t >= L_b hold ``pad_value``
      seq_lens   int32 [B];  cu_q  int32 [B + 1];  max_q  int
      block_table, k_paged, v_paged   (paged workloads only), as make_inputs
    """
    if lengths is None:
        n, lens = prefill_lengths(w)
    else:
        n, lens = (np.asarray(x, dtype=np.int32) for x in lengths)
        assert n.shape == lens.shape == (w.B,) and (n <= lens).all()
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = torch.empty(int(cu[-1]), w.H_Q, w.D, dtype=torch.bfloat16)
    _fill_normal(q, (w.seed, _S_Q))
    S = max(w.capacity, int(lens.max()) if w.B else 0)
    if w.page_size:
        S = -(-S // w.page_size) * w.page_size
    k = torch.full((w.B, S, w.H_KV, w.D), pad_value, dtype=torch.bfloat16)
    v = torch.full((w.B, S, w.H_KV, w.D), pad_value, dtype=torch.bfloat16)
    for b in range(w.B):
        L = int(lens[b])
        _fill_normal(k[b, :L], (w.seed, _S_K, b))
        _fill_normal(v[b, :L], (w.seed, _S_V, b))
    out = {"q": q, "k": k, "v": v, "seq_lens": torch.from_numpy(lens), "cu_q": torch.from_numpy(cu),
           "max_q": int(n.max()) if w.B else 0}
    if w.page_size:
        nb = S // w.page_size
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence((w.seed, _S_TABLE))))
        table = torch.from_numpy(rng.permutation(w.B * nb).astype(np.int32)).view(w.B, nb)
        out["block_table"] = table
        out["k_paged"] = to_pages(k, table, w.page_size)
        out["v_paged"] = to_pages(v, table, w.page_size)
    return out


def prefill_flops(w: PrefillWorkload, n: np.ndarray, lens: np.ndarray) -> int:
    """Algorithmic FLOPs: 4 D per (query head, visible key) pair -- 2 D for the
    score, 2 D for the weighted value -- where query token j of sequence b sees
    L_b - n_b + j + 1 keys."""
    pairs = 0
    for n_b, L in zip(n.tolist(), lens.tolist()):
        first = L - n_b + 1  # keys seen by the first new token
        pairs += n_b * first + n_b * (n_b - 1) // 2
    return 4 * w.D * w.H_Q * pairs
