"""One layer on several GPUs: token-sharded H and row-sharded prunes.

One process per GPU; torch.distributed (NCCL between GPUs) carries the one exchange.
Both shardings are exact by the structure of the problem:

* Tokens.  H = 2 X X^T is a sum over calibration tokens ("Pruning LLMs with Thanos",
  "The layer-reconstruction lens"; the weight-pruning blog page, "SparseGPT:
  Second-Order Reconstruction at Scale"), so rank r builds 2 X_r X_r^T from its own
  token shard on the tensor cores and one all-reduce (sum) leaves H on every rank.
* Rows.  The reconstruction loss is a sum of independent per-row terms (same section of
  the Thanos page).  With H on every rank, each rank factors it and prunes its own slice
  of W's rows, which reproduces the rows of a one-GPU prune on that H wherever nothing
  couples rows: N:M patterns (every group lies inside one row) and the per-row quotas
  of Wanda and magnitude.
* The unstructured global budget of Thanos and SparseGPT ties every row to each block's
  threshold ("Contribution two: keep the budget global and the execution local"), and only
  through it: ``prune_rows_global`` runs the block sweep step by step (``Sweep``) and, per
  block, sums the level-1 selection histogram (with each rank's removal count) and the
  level-2 histograms over ranks and gathers the per-column counts of tied entries, so
  every rank picks the same exact threshold and its own share of the ties in (column,
  row) order, lower ranks' rows first.  Three collectives per block, all on the
  prune's stream.

Without an initialised process group every function acts as a single rank.
"""
from __future__ import annotations

from . import MAGNITUDE, METHODS, NM, WANDA, hessian_accumulate, prune_layer
from . import _stream_ctx

__all__ = ["token_range", "row_range", "rows_independent", "allreduce_hessian", "hessian_sharded",
           "prune_rows", "gather_rows", "TorchComm", "LocalComm", "global_sweep", "prune_rows_global"]


def _dist():
    import torch.distributed as dist
    return dist


def _world(group=None):
    dist = _dist()
    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def _split(total: int, world: int, rank: int):
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError(f"bad split: total={total} world={world} rank={rank}")
    base, extra = divmod(total, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def token_range(n: int, world: int, rank: int):
    """[t0, t1): this rank's calibration tokens; shards differ in size by at most one."""
    return _split(n, world, rank)


def row_range(c: int, world: int, rank: int):
    """[r0, r1): this rank's rows of W; shards differ in size by at most one."""
    return _split(c, world, rank)


def rows_independent(method="thanos", pattern="unstructured") -> bool:
    """True where a prune of a row slice gives exactly those rows of the whole-layer prune."""
    m = METHODS[method] if isinstance(method, str) else int(method)
    p = ({"unstructured": 0, "nm": NM}[pattern] if isinstance(pattern, str) else int(pattern))
    return p == NM or m in (WANDA, MAGNITUDE)


def allreduce_hessian(H, group=None):
    """In place: every rank's partial 2 X_r X_r^T becomes the sum over ranks."""
    world, _ = _world(group)
    if world > 1:
        dist = _dist()
        dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    return H


def hessian_sharded(X_local, group=None, stream=None):
    """H = 2 X X^T over the tokens of all ranks: this rank's token shard X_local ([n_r, b],
    bf16/fp32 CUDA tensor) on the tensor cores, then one all-reduce.  Every rank must pass
    the same b; a rank may hold no tokens (n_r = 0)."""
    H = hessian_accumulate(X_local, stream=stream)
    if stream is None:
        return allreduce_hessian(H, group)
    with _stream_ctx(stream):                  # the collective waits for the H build on this stream
        return allreduce_hessian(H, group)


def prune_rows(W_local, H, *, method="thanos", pattern="nm", group=None, **kw):
    """Prune this rank's rows W_local ([c_r, b]) against the whole layer's H (destroyed
    as in ``prune_layer``).  Only where ``rows_independent(method, pattern)`` (else use
    ``prune_rows_global``); returns ``prune_layer``'s (W_hat, mask, stats) for the local rows."""
    if not rows_independent(method, pattern):
        raise ValueError("unstructured Thanos/SparseGPT couples the rows through each block's threshold: "
                         "use prune_rows_global")
    if H is None and (METHODS[method] if isinstance(method, str) else int(method)) != MAGNITUDE:
        raise ValueError("give the layer's H (hessian_sharded)")
    return prune_layer(W_local, H=H, method=method, pattern=pattern, **kw)


def gather_rows(local, c: int, group=None):
    """Concatenate every rank's row slice (as cut by ``row_range``) into the [c, ...]
    tensor on every rank."""
    import torch
    world, rank = _world(group)
    r0, r1 = row_range(c, world, rank)
    if local.shape[0] != r1 - r0:
        raise ValueError(f"rank {rank} holds {local.shape[0]} rows, row_range gives {r1 - r0}")
    if world == 1:
        return local
    rows = -(-c // world)                      # the largest shard
    padded = torch.zeros((rows,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    padded[: r1 - r0].copy_(local)
    parts = [torch.empty_like(padded) for _ in range(world)]
    _dist().all_gather(parts, padded, group=group)
    return torch.cat([p[: row_range(c, world, r)[1] - row_range(c, world, r)[0]] for r, p in enumerate(parts)])


# --------------------------------------------------------------------------- the global budget

class TorchComm:
    """Sums and gathers over the ranks of a torch.distributed group, one sweep per process."""

    def __init__(self, group=None):
        self.group = group

    def sum(self, tensors):
        for t in tensors:
            _dist().all_reduce(t, op=_dist().ReduceOp.SUM, group=self.group)

    def gather(self, tensors, outs):
        for t, out in zip(tensors, outs):
            parts = list(out.unbind(0))
            _dist().all_gather(parts, t, group=self.group)


class LocalComm:
    """Ranks emulated in one process (every sweep in the list is one rank, in rank order):
    sums and gathers across the list."""

    def sum(self, tensors):
        total = tensors[0].clone()
        for t in tensors[1:]:
            total += t.to(total.device)
        for t in tensors:
            t.copy_(total)

    def gather(self, tensors, outs):
        import torch
        stacked = torch.stack([t.to(outs[0].device) for t in tensors])
        for out in outs:
            out.copy_(stacked)


def global_sweep(sweeps, comm):
    """Drive the block loop of row-sharded prunes under one global budget: ``sweeps`` holds
    this process's ranks (``Sweep`` objects or anything with the same steps and buffers),
    ``comm`` sums and gathers their buffers over all ranks between the steps."""
    for sw in sweeps:
        sw.step("setup")
    for t in range(sweeps[0].nblk):
        for sw in sweeps:
            sw.step("score", t)
        comm.sum([sw.level1 for sw in sweeps])             # level-1 counts and removals so far
        for sw in sweeps:
            sw.step("pick_bin", t)
            sw.step("reread", t)
        comm.sum([sw.level2 for sw in sweeps])             # level-2 counts of the chosen bin
        for sw in sweeps:
            sw.step("pick_key", t)
            sw.step("count_ties", t)
        comm.gather([sw.ties for sw in sweeps], [sw.ties_all for sw in sweeps])
        for sw in sweeps:
            sw.step("cut_ties", t)
            sw.step("solve", t)
    for sw in sweeps:
        sw.step("finish")
    return sweeps


def prune_rows_global(W_local, H, c_total=None, *, method="thanos", group=None, stream=None, **kw):
    """This rank's rows of a layer pruned with the unstructured budget over every rank's
    rows (W_local: the rows of ``row_range`` in rank order; H: the whole layer's H, e.g.
    from ``hessian_sharded``, destroyed).  Returns (W_hat, mask, Stats) of the local rows;
    the removals summed over ranks meet floor(sparsity * c_total * b)."""
    world, rank = _world(group)
    if c_total is None:
        import torch
        t = torch.tensor([W_local.shape[0]], dtype=torch.int64, device=W_local.device)
        if world > 1:
            _dist().all_reduce(t, group=group)
        c_total = int(t.item())
    from . import Sweep
    sw = Sweep(W_local, H, c_total, world, rank, method=method, stream=stream, **kw)
    comm = TorchComm(group) if world > 1 else LocalComm()
    if stream is None:
        global_sweep([sw], comm)
    else:
        with _stream_ctx(stream):   # the exchanges are ordered with the steps on this stream
            global_sweep([sw], comm)
    return sw.result()
