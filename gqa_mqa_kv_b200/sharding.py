"""Host-side partitioning of one decode step across ranks.

Two ways to split the step, neither of which needs an exchange on the data
path:

* batch sharding: each rank owns a contiguous block of sequences;
* tensor-parallel head sharding ("Grouped-Query Attention (GQA) and
  Multi-Query Attention (MQA): Mathematical Foundations, ...", section 4,
  "Tensor Parallelism (TP) Head Partitioning"): rank j of N holds KV heads
  [j H_KV/N, (j+1) H_KV/N) and the query heads that read them,
  [j H_Q/N, (j+1) H_Q/N); this requires H_KV mod N = 0.  Because the group map
  is contiguous, every query head of a rank's slice reads a KV head of the
  same slice, so each rank runs an ordinary GQA decode on its slice.  When
  N > H_KV (the same section: the KV heads are then duplicated), N must be a
  multiple of H_KV: rank j holds the single KV head j H_KV / N, replicated on
  N / H_KV ranks, and the query heads [j H_Q/N, (j+1) H_Q/N), which all belong
  to that head's group, so each rank runs an MQA decode (H_KV = 1) on its
  slice.
"""

from __future__ import annotations


def batch_shard(B: int, world: int, rank: int) -> slice:
    """Contiguous block of sequences for `rank` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    lo = rank * B // world
    hi = (rank + 1) * B // world
    return slice(lo, hi)


def tp_head_shard(H_Q: int, H_KV: int, world: int, rank: int) -> tuple[slice, slice]:
    """(query-head slice, KV-head slice) of `rank` under tensor parallelism.

    world <= H_KV: H_KV % world == 0, each rank owns H_KV / world KV heads.
    world > H_KV: world % H_KV == 0, each rank holds one (duplicated) KV head.
    """
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    if H_Q % H_KV != 0:
        raise ValueError("H_Q must be a multiple of H_KV")
    if H_Q % world != 0:
        raise ValueError("H_Q must be a multiple of the tensor-parallel size")
    q_per = H_Q // world
    qs = slice(rank * q_per, (rank + 1) * q_per)
    if H_KV % world == 0:
        kv_per = H_KV // world
        return qs, slice(rank * kv_per, (rank + 1) * kv_per)
    if world % H_KV == 0:
        kv = rank * H_KV // world
        return qs, slice(kv, kv + 1)
    raise ValueError("tensor parallelism needs H_KV % world == 0 or world % H_KV == 0")
