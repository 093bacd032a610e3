"""Host logic of the multi-GPU layer prune (CPU): the token and row splits, the
all-reduce of per-rank Hessians and the row gather over gloo ranks (world size 2), and,
on the oracle, the property that makes row sharding exact -- for N:M patterns and the
per-row quotas of Wanda and magnitude a prune of a row slice gives exactly those rows of
the whole-layer prune, while the unstructured global budget couples the rows."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from post_weight_pruning_b200 import sharded


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("total,world", [(0, 1), (7, 2), (16384, 3), (5, 8), (11008, 8)])
def test_splits_partition_and_balance(total, world):
    for split in (sharded.token_range, sharded.row_range):
        ranges = [split(total, world, r) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == total
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        sizes = [hi - lo for lo, hi in ranges]
        assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1


def test_split_rejects_bad_rank():
    with pytest.raises(ValueError):
        sharded.row_range(10, 2, 2)


@pytest.mark.parametrize("method,pattern,want", [
    ("thanos", "nm", True), ("sparsegpt", "nm", True), ("wanda", "unstructured", True),
    ("magnitude", "unstructured", True), ("thanos", "unstructured", False), ("sparsegpt", "unstructured", False),
])
def test_rows_independent(method, pattern, want):
    assert sharded.rows_independent(method, pattern) is want


def test_prune_rows_sends_the_global_budget_to_the_sweep():
    W = torch.zeros(8, 16)
    with pytest.raises(ValueError, match="prune_rows_global"):
        sharded.prune_rows(W, torch.zeros(16, 16), method="thanos", pattern="unstructured")


def _layer(c=24, b=64, n=256, seed=5):
    wl = synth.custom(c, b, n, dtype="fp32", outlier_frac=0.05, outlier_scale=10.0, seed=seed)
    W = synth.to_f64(synth.make_W(wl), "fp32")
    Xt = synth.to_f64(synth.make_X_tokens(wl), "fp32")
    return W, Xt


@pytest.mark.parametrize("method,pattern,nm", [
    ("thanos", "nm", (2, 4)), ("thanos", "nm", (4, 8)), ("sparsegpt", "nm", (2, 4)),
])
def test_oracle_row_slices_reproduce_the_layer_nm(method, pattern, nm):
    W, Xt = _layer()
    H = oracle.hessian(Xt)
    full = oracle.prune_layer(W, H=H, method=method, pattern=pattern, nm=nm, block=16)
    for world in (2, 3):
        for r in range(world):
            r0, r1 = sharded.row_range(W.shape[0], world, r)
            part = oracle.prune_layer(W[r0:r1], H=H, method=method, pattern=pattern, nm=nm, block=16)
            assert np.array_equal(part["mask"], full["mask"][r0:r1])
            np.testing.assert_allclose(part["W"], full["W"][r0:r1], rtol=0, atol=1e-12)


@pytest.mark.parametrize("method,pattern", [("wanda", "unstructured"), ("magnitude", "unstructured"),
                                            ("wanda", "nm")])
def test_oracle_row_slices_reproduce_the_layer_no_update(method, pattern):
    W, Xt = _layer(c=21)
    full = oracle.prune_no_update(W, Xt=Xt, method=method, pattern=pattern, sparsity=0.4)
    for r in range(3):
        r0, r1 = sharded.row_range(W.shape[0], 3, r)
        part = oracle.prune_no_update(W[r0:r1], Xt=Xt, method=method, pattern=pattern, sparsity=0.4)
        assert np.array_equal(part["mask"], full["mask"][r0:r1])
        assert np.array_equal(part["W"], full["W"][r0:r1])


def test_oracle_unstructured_budget_couples_rows():
    # rows of very different scale: the global budget takes most removals from the small
    # rows, a per-slice budget cannot
    W, Xt = _layer(c=24)
    W[:12] *= 10.0
    H = oracle.hessian(Xt)
    full = oracle.prune_layer(W, H=H, method="thanos", sparsity=0.5, block=16)
    part = oracle.prune_layer(W[:12], H=H, method="thanos", sparsity=0.5, block=16)
    assert full["mask"][:12].sum() < part["mask"].sum()


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, Xt = _layer(c=7, n=250)
        t0, t1 = sharded.token_range(Xt.shape[0], world, rank)
        H = torch.from_numpy(oracle.hessian(Xt[t0:t1]))       # this rank's 2 X_r X_r^T
        sharded.allreduce_hessian(H)
        r0, r1 = sharded.row_range(W.shape[0], world, rank)
        G = sharded.gather_rows(torch.from_numpy(W[r0:r1]).contiguous(), W.shape[0])
        out[rank] = (H.numpy(), G.numpy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_h_and_gather_rows():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    W, Xt = _layer(c=7, n=250)
    H_ref = oracle.hessian(Xt)
    for r in range(world):
        H, G = out[r]
        np.testing.assert_allclose(H, H_ref, rtol=1e-12, atol=1e-12 * np.abs(H_ref).max())
        assert np.array_equal(G, W)
    assert np.array_equal(out[0][0], out[1][0])


def test_single_rank_without_process_group():
    W = torch.arange(12.0).reshape(4, 3)
    assert sharded.gather_rows(W, 4) is W
    H = torch.ones(3, 3)
    assert sharded.allreduce_hessian(H) is H


# --------------------------------------------------------------------------------------
# The exchange the unstructured global budget needs under row sharding (not built on the
# GPU): per block, every rank histograms its own keys, the histograms are summed across
# ranks, and the per-column counts of keys equal to the threshold are gathered so that
# every rank knows how many tied entries precede its own in (column, row) order.  Checked
# here with the selection's two radix levels (13 + 18 bits of the fp32 key) and gloo ranks:
# the union of the ranks' masks must be the oracle's lowest-r selection.

LO_BITS = 18


def _find_bin(hist, rank_1based):
    """(bin holding the rank-th smallest key, number of keys in lower bins)."""
    cum = np.cumsum(hist, dtype=np.int64)
    b = int(np.searchsorted(cum, rank_1based))
    return b, int(cum[b - 1]) if b > 0 else 0


def _sharded_select(S_local, r, world):
    """This rank's part of the lowest-r selection over all ranks' rows (rank order = row
    order), with the exchanges a row-sharded GPU sweep would make."""
    keys = S_local.astype(np.float32).view(np.uint32)
    h1 = torch.from_numpy(np.bincount((keys >> LO_BITS).ravel(), minlength=1 << (31 - LO_BITS)).astype(np.int64))
    dist.all_reduce(h1)                                              # exchange 1: level-1 counts
    b1, below1 = _find_bin(h1.numpy(), r)
    in_b1 = (keys >> LO_BITS) == b1
    h2 = torch.from_numpy(np.bincount((keys[in_b1] & ((1 << LO_BITS) - 1)).ravel(),
                                      minlength=1 << LO_BITS).astype(np.int64))
    dist.all_reduce(h2)                                              # exchange 2: level-2 counts
    b2, below2 = _find_bin(h2.numpy(), r - below1)
    T = np.uint32((b1 << LO_BITS) | b2)
    need = r - below1 - below2                                       # tied entries to take
    tied = keys == T
    t_local = torch.from_numpy(tied.sum(axis=0).astype(np.int64))   # per column
    gathered = [torch.zeros_like(t_local) for _ in range(world)]
    dist.all_gather(gathered, t_local)                               # exchange 3: tie counts
    t_all = torch.stack(gathered).numpy()                            # [world, columns]
    me = dist.get_rank()
    before = np.concatenate([[0], np.cumsum(t_all.sum(axis=0))[:-1]]) + t_all[:me].sum(axis=0)
    take = np.clip(need - before, 0, t_all[me])                      # this rank's ties per column
    mask = keys < T
    for q in np.flatnonzero(take):
        rows = np.flatnonzero(tied[:, q])[: take[q]]
        mask[rows, q] = True
    return mask


def _select_worker(rank, world, port, S32, r, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r0, r1 = sharded.row_range(S32.shape[0], world, rank)
        out[rank] = _sharded_select(S32[r0:r1], r, world)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,ties", [(2, False), (3, True)])
def test_global_budget_exchange_reproduces_the_global_selection(world, ties):
    rng = np.random.default_rng(40 + world)
    W = rng.normal(0, 0.02, size=(29, 48))
    if ties:
        W = np.round(W * 64) / 64                  # large groups of equal scores
    g = rng.uniform(0.5, 2.0, size=48) if not ties else np.ones(48)
    S32 = oracle.wanda_scores(W, g).astype(np.float32)
    r = int(0.45 * S32.size)
    want, t_last, _ = oracle.lowest_global(S32.astype(np.float64), 0, r)
    if ties:
        assert (S32 == np.float32(t_last)).sum() > 10            # the boundary really is tied
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_select_worker, args=(world, _free_port(), S32, r, out), nprocs=world, start_method="spawn")
    got = np.concatenate([out[k] for k in range(world)])
    assert got.sum() == r
    assert np.array_equal(got, want)


# ----------------------------------------------------------------------------- the stepwise sweep

def _sweep_worker(rank, world, port, W, H, out, kw):
    from tests._sweep_standin import NumpySweep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r0, r1 = sharded.row_range(W.shape[0], world, rank)
        sw = NumpySweep(W[r0:r1], H, W.shape[0], world, rank, **kw)
        sharded.global_sweep([sw], sharded.TorchComm())
        out[rank] = (sw.W, sw.mask, sw.pruned)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,ties", [(2, False), (3, True)])
def test_global_sweep_over_gloo_ranks_reproduces_the_whole_layer(world, ties):
    """The real host loop (sharded.global_sweep with its torch.distributed collectives) over
    gloo ranks, each holding a row slice of one layer under the global budget: the ranks'
    masks and weights together are the oracle's whole-layer prune.  With ties, the first
    block's threshold falls inside large groups of equal scores spread over the ranks."""
    rng = np.random.default_rng(70 + world)
    c, b, n = 29, 32, 96
    if ties:
        W = np.round(rng.normal(0, 0.02, size=(c, b)) * 64) / 64
        Xt = rng.choice([-1.0, 1.0], size=(n, b))              # every feature the same norm
    else:
        W = rng.normal(0, 0.02, size=(c, b))
        Xt = rng.normal(size=(n, b)) * rng.uniform(0.5, 2.0, size=b)
    H = oracle.hessian(Xt)
    kw = dict(sparsity=0.5, block=8, damp=0.01)
    want = oracle.prune_layer(W, H=H, **kw)
    if ties:
        S0 = oracle.wanda_scores(W, np.diag(H) / 2)
        assert (S0 == want["blocks"][0]["t_last"]).sum() > 10     # the boundary really is tied
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_sweep_worker, args=(world, _free_port(), W, H, out, kw), nprocs=world, start_method="spawn")
    got_W = np.concatenate([out[r][0] for r in range(world)])
    got_m = np.concatenate([out[r][1] for r in range(world)])
    assert sum(out[r][2] for r in range(world)) == want["zstar"]
    assert np.array_equal(got_m, want["mask"])
    assert np.allclose(got_W, want["W"], rtol=1e-9, atol=1e-12)


def test_global_sweep_drops_the_cross_rank_tie_order_and_fails():
    """A plant in the stand-in, not the library: if a rank ignored the lower ranks' tied
    entries (rank 0's cut-off used by every rank), the union would take too many ties."""
    from tests._sweep_standin import NumpySweep

    class Careless(NumpySweep):
        def _cut_ties(self, t):
            keep = self.rank
            self.rank = 0
            self.ties_all.numpy()[:] = 0
            self.ties_all.numpy()[0, :] = self.ties.numpy()
            super()._cut_ties(t)
            self.rank = keep

    rng = np.random.default_rng(72)
    W = np.round(rng.normal(0, 0.02, size=(20, 16)) * 64) / 64
    Xt = rng.choice([-1.0, 1.0], size=(48, 16))
    H = oracle.hessian(Xt)
    sweeps = [Careless(W[r0:r1], H, 20, 2, r, sparsity=0.5, block=8)
              for r, (r0, r1) in enumerate(sharded.row_range(20, 2, r) for r in range(2))]
    sharded.global_sweep(sweeps, sharded.LocalComm())
    want = oracle.prune_layer(W, H=H, sparsity=0.5, block=8)
    got = np.concatenate([sw.mask for sw in sweeps])
    assert not np.array_equal(got, want["mask"])


def test_local_comm_emulates_ranks_in_one_process():
    """The in-process communicator on the CPU stand-in reproduces the whole layer too."""
    from tests._sweep_standin import NumpySweep
    rng = np.random.default_rng(73)
    W = rng.normal(0, 0.02, size=(21, 24))
    Xt = rng.normal(size=(60, 24))
    H = oracle.hessian(Xt)
    sweeps = [NumpySweep(W[r0:r1], H, 21, 3, r, sparsity=0.4, block=8)
              for r, (r0, r1) in enumerate(sharded.row_range(21, 3, r) for r in range(3))]
    sharded.global_sweep(sweeps, sharded.LocalComm())
    want = oracle.prune_layer(W, H=H, sparsity=0.4, block=8)
    assert np.array_equal(np.concatenate([sw.mask for sw in sweeps]), want["mask"])
    assert np.allclose(np.concatenate([sw.W for sw in sweeps]), want["W"], rtol=1e-9, atol=1e-12)


def test_global_budget_exchanges_run_on_the_callers_stream(monkeypatch):
    """prune_rows_global given a stream: every step and every exchange between the steps
    happens with that stream current (one rank, the in-process communicator)."""
    import post_weight_pruning_b200 as pwp
    from tests._sweep_standin import NumpySweep
    current = []

    class Ctx:
        def __init__(self, s):
            self.s = s

        def __enter__(self):
            current.append(self.s)

        def __exit__(self, *exc):
            current.pop()

    seen = []

    class Recording(NumpySweep):
        def __init__(self, W_local, H, c_total, world, rank, *, method="thanos", stream=None, **kw):
            super().__init__(W_local, H, c_total, world, rank, **kw)

        def step(self, name, t=0):
            seen.append(("step", current[-1] if current else None))
            super().step(name, t)

        def result(self):
            return self.W, self.mask, None

    orig_sum = sharded.LocalComm.sum

    def rec_sum(self, tensors):
        seen.append(("sum", current[-1] if current else None))
        return orig_sum(self, tensors)

    monkeypatch.setattr(sharded, "_stream_ctx", Ctx)
    monkeypatch.setattr(pwp, "Sweep", Recording)
    monkeypatch.setattr(sharded.LocalComm, "sum", rec_sum)
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, size=(6, 16))
    H = oracle.hessian(rng.normal(size=(40, 16)))
    s = object()
    W_hat, mask, _ = sharded.prune_rows_global(W, H, 6, stream=s, sparsity=0.5, block=8)
    assert seen and all(who is s for _, who in seen)
    assert {kind for kind, _ in seen} == {"step", "sum"} and not current
    want = oracle.prune_layer(W, H=H, sparsity=0.5, block=8)
    assert np.array_equal(mask, want["mask"])
