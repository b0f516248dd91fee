"""Head-sharded SparsePR over the ranks of a torch.distributed group.

Every step of the call (sampled responses, both k-means, routing, permutation, block-sparse
attention, probes, fit and write-back) works on one KV head at a time, so the heads split across
GPUs with no exchange between them. Rank r of W takes the contiguous range of flattened KV heads
z = b * Hkv + hk that head_range(P, W, r) gives (shard sizes differ by at most one) and runs one
handle configured as a single batch of those KV heads: their query heads are the contiguous rows
z * g .. z * g + g - 1 of the flattened [B * Hq] query heads, so a shard is a plain slice of the
inputs. The only collective is gather_output, for a caller that needs all of O on every device:
each rank's O is padded to the largest shard and one all_gather_into_tensor (NCCL over
NVLink/NVSwitch on GPUs) collects them; the padding is dropped afterwards.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def head_range(P: int, world: int, rank: int) -> tuple[int, int]:
    """Flattened KV heads [lo, hi) of `rank`: P heads in `world` contiguous shards whose sizes
    differ by at most one (the first P mod world shards take one more)."""
    if world < 1 or not 0 <= rank < world or P < 0:
        raise ValueError(f"bad shard request P={P} world={world} rank={rank}")
    base, extra = divmod(P, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def local_heads(x: torch.Tensor, per_head: int, lo: int, hi: int) -> torch.Tensor:
    """Rows [lo * per_head, hi * per_head) of x [B, H, N, d] viewed as [B * H, N, d]: the query
    heads (per_head = g) or the key / value heads (per_head = 1) of KV heads [lo, hi)."""
    return x.reshape(-1, *x.shape[2:])[lo * per_head: hi * per_head]


def gather_output(O_local: torch.Tensor, P: int, g: int, group=None) -> torch.Tensor:
    """Every rank's output [n_r * g, N, d] in head order as [P * g, N, d], on every rank."""
    world = dist.get_world_size(group)
    smax = -(-P // world)
    rows = smax * g
    buf = O_local.new_zeros((rows, *O_local.shape[1:]))
    buf[: O_local.shape[0]] = O_local
    out = O_local.new_empty((world * rows, *O_local.shape[1:]))
    dist.all_gather_into_tensor(out, buf, group=group)
    pieces = []
    for r in range(world):
        lo, hi = head_range(P, world, r)
        pieces.append(out[r * rows: r * rows + (hi - lo) * g])
    return torch.cat(pieces)


class ShardedSparsePR:
    """This rank's share of one SparsePR call: the KV heads head_range(B * Hkv, world, rank).

    compute, when given, replaces the CUDA path for the local heads (a callable
    (q [n*g, N, d], k [n, N, d], v [n, N, d]) -> O [n*g, N, d]); host-side tests use it to drive
    the sharding and the gather on CPU ranks. Otherwise a SparsePR handle serves the local heads
    (keyword arguments as for SparsePR, except B, Hq and Hkv). world and rank may be given to run
    one shard outside a process group (no gather then).
    """

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, d: int, group=None, compute=None, world=None, rank=None,
                 **kw):
        self.group = group
        # world / rank default to the group's; given explicitly, one process can run any shard
        self.world = world if world is not None else (dist.get_world_size(group) if dist.is_initialized() else 1)
        self.rank = rank if rank is not None else (dist.get_rank(group) if dist.is_initialized() else 0)
        self.P, self.g, self.N, self.d = B * Hkv, Hq // Hkv, N, d
        self.lo, self.hi = head_range(self.P, self.world, self.rank)
        self.n = self.hi - self.lo
        self.compute = compute
        self.handle = None
        if compute is None and self.n > 0:
            from . import SparsePR

            self.handle = SparsePR(B=1, Hq=self.n * self.g, Hkv=self.n, N=N, d=d, **kw)

    def close(self):
        if self.handle is not None:
            self.handle.close()
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def attention_local(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
        """O [n*g, N, d] of this rank's heads from its own q [n*g, N, d], k, v [n, N, d]."""
        if self.n == 0:
            return q.new_empty((0, self.N, self.d))
        if self.compute is not None:
            return self.compute(q, k, v)
        shape_q, shape_kv = (1, self.n * self.g, self.N, self.d), (1, self.n, self.N, self.d)
        O = self.handle.attention(q.reshape(shape_q), k.reshape(shape_kv), v.reshape(shape_kv))
        return O.reshape(self.n * self.g, self.N, self.d)

    def attention(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, gather: bool = False) -> torch.Tensor:
        """From the full inputs Q [B, Hq, N, d], K, V [B, Hkv, N, d]: this rank's O, or (gather)
        the whole O [B * Hq, N, d] on every rank."""
        O = self.attention_local(local_heads(Q, self.g, self.lo, self.hi),
                                 local_heads(K, 1, self.lo, self.hi), local_heads(V, 1, self.lo, self.hi))
        if not gather:
            return O
        if self.world == 1:
            return O
        return gather_output(O, self.P, self.g, self.group)
