"""Token-split decode: one sequence's KV cache spread over ranks by token ranges.

Each rank's cache holds a contiguous shard of the prompt's tokens; the last
rank also takes every appended token (its residual is the sequence's
residual).  A decode step computes each rank's unnormalised partial
(kvq_decode_attention_partial), gathers the partials of all ranks and merges
them with a log-sum-exp (kvq_merge_partials): attention over a concatenation
does not depend on the order of its parts ("Resumo Técnico: LogQuant",
section 4), so the merged result is the attention over the whole cache.

Every shard but the last holds a multiple of R tokens, so it is quantized
exactly as those tokens are in a single cache (key groups of G tokens never
straddle a shard boundary, R being a multiple of G).

The exchange is the only collective: an all-gather of B*Hq*(d + 2) floats per
rank and decode step.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import kvq


def shard_bounds(T: int, world: int, R: int) -> list[tuple[int, int]]:
    """Token range [lo, hi) of a T-token prompt held by each of `world` ranks: every
    shard but the last a multiple of R tokens (possibly empty), the last the rest."""
    if T < 0 or world < 1 or R < 1:
        raise ValueError("T >= 0, world >= 1 and R >= 1 required")
    per = -(-T // world)
    per = -(-per // R) * R
    top = (T // R) * R            # shards before the last end on multiples of R
    bounds, lo = [], 0
    for k in range(world):
        hi = T if k == world - 1 else min(top, lo + per)
        bounds.append((lo, hi))
        lo = hi
    return bounds


def exchange_partials(o: torch.Tensor, m: torch.Tensor, l: torch.Tensor, group=None):
    """All-gather the ranks' partials (o [*rows, d], m and l [*rows], float32): returns
    o_all [world, *rows, d], m_all and l_all [world, *rows] in rank order."""
    world = dist.get_world_size(group)
    nm, no = m.numel(), o.numel()
    buf = torch.cat([o.reshape(-1), m.reshape(-1), l.reshape(-1)]).contiguous()
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=group)
    allp = torch.stack(parts)
    return (allp[:, :no].reshape(world, *o.shape), allp[:, no:no + nm].reshape(world, *m.shape),
            allp[:, no + nm:].reshape(world, *l.shape))


class TokenSplitCache:
    """This rank's part of a KV cache whose tokens are split across the ranks of `group`."""

    def __init__(self, batch, q_heads, kv_heads, head_dim, group_k, group_v, residual, bits,
                 symmetric, dtype, prompt_tokens: int, max_new_tokens: int, device, group=None):
        self.group = group
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        self.bounds = shard_bounds(prompt_tokens, self.world, residual)
        lo, hi = self.bounds[self.rank]
        self.last = self.rank == self.world - 1
        tokens = (hi - lo) + (max_new_tokens if self.last else 0)
        capacity = max(residual, -(-tokens // residual) * residual)
        self.cache = kvq.KVQCache(batch, q_heads, kv_heads, head_dim, group_k, group_v, residual, bits,
                                  symmetric, dtype, capacity, device)

    def prefill_quantize(self, X_K: torch.Tensor, X_V: torch.Tensor, stream=None):
        """X_K, X_V: the whole prompt [B, Hkv, T, d]; this rank keeps its token shard."""
        lo, hi = self.bounds[self.rank]
        if hi > lo:
            self.cache.prefill_quantize(X_K[:, :, lo:hi].contiguous(), X_V[:, :, lo:hi].contiguous(), stream)
        return self

    def append(self, t_K: torch.Tensor, t_V: torch.Tensor, stream=None):
        """New tokens go to the last rank."""
        if self.last:
            self.cache.append(t_K, t_V, stream)
        return self

    def decode_attention(self, t_Q: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        """The attention output over all ranks' tokens, on every rank."""
        c = self.cache.cfg
        if self.cache.state() == (0, 0):   # an empty shard weighs nothing in the merge
            o = torch.zeros((c.batch, c.q_heads, c.head_dim), dtype=torch.float32, device=self.cache.device)
            m = torch.full((c.batch, c.q_heads), float("-inf"), dtype=torch.float32, device=self.cache.device)
            l = torch.zeros((c.batch, c.q_heads), dtype=torch.float32, device=self.cache.device)
        else:
            o, m, l = self.cache.decode_attention_partial(t_Q, stream)
        o_all, m_all, l_all = exchange_partials(o, m, l, self.group)
        return kvq.merge_partials(o_all, m_all, l_all, out, stream)
