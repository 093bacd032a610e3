"""Parity at the full sizes of the benchmark workloads (4096x4096 at 50% unstructured,
11008x4096 at 2:4, 4096x11008 at 4:8; n = 16384 or 32768 bf16 tokens; and the seven
layers of a LLaMA-7B-shaped decoder block on 128 x 2048 tokens), in the configuration
bench.py times.  Checked: properties that hold at any size (removed weights
exactly 0, the exact removal count or every N:M group keeping n); sampled entries of H
against fp64 dot products of the activation columns; and the first block's selection
against the oracle, which at that point depends only on W and the column norms
(tests/_fullsize.py), except within 2e-5 (relative) of the selection boundary."""
import os

import numpy as np
import pytest

import synth
from tests import _fullsize as F
from tests import _parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.fullsize]

TIE_TOL = 2e-5
# over 262144 tokens the fp32 accumulation of diag(H) drifts by up to ~6e-6 relative
BLOCK_TIE_TOL = 5e-5


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("name", ["q_proj4096x4096", "up_proj11008x4096_2of4", "down_proj4096x11008_4of8"])
def test_full_size_workload(name):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl = synth.workload(name)
    W, X = synth.make_W(wl), synth.make_X_tokens(wl, threads=max(1, min(16, os.cpu_count() or 1)))
    Wt, Xt = P.torch_inputs(W, X, wl.dtype)
    g = F.column_norms_sq(X, wl.dtype)

    # sampled entries of H = 2 X X^T (diagonal ones included)
    H = pwp.hessian_accumulate(Xt)
    torch.cuda.synchronize()
    rng = np.random.default_rng(77)
    ii = rng.integers(0, wl.b, 48)
    jj = rng.integers(0, wl.b, 48)
    ii = np.concatenate([ii, ii[:16]])
    jj = np.concatenate([jj, ii[:16]])
    Hs = H[torch.from_numpy(ii).cuda(), torch.from_numpy(jj).cuda()].cpu().numpy().astype(np.float64)
    del H
    ref = 2.0 * np.einsum("tk,tk->k", synth.to_f64(X[:, ii], wl.dtype), synth.to_f64(X[:, jj], wl.dtype))
    scale = 2.0 * np.sqrt(g[ii] * g[jj])
    assert np.max(np.abs(Hs - ref) / scale) < 1e-4

    # the prune
    nm = wl.nm if wl.pattern == "nm" else (0, 0)
    W_hat, mask, st = pwp.prune_layer(Wt, X=Xt, method="thanos", pattern=wl.pattern, nm=nm, sparsity=wl.sparsity,
                                      block=wl.block, damp=wl.damp)
    torch.cuda.synchronize()
    assert st.status == 0
    assert bool(torch.all(W_hat[mask.bool()] == 0).item())
    m = mask.cpu().numpy().astype(bool)
    c, b = m.shape
    if wl.pattern == "unstructured":
        want = int(np.floor(float(np.float32(wl.sparsity)) * c * b))
        assert int(m.sum()) == st.pruned == st.target == want
    else:
        n_keep, mm = nm
        assert np.all(m.reshape(c, -1, mm).sum(axis=2) == mm - n_keep)
        assert st.pruned == st.target == int(m.sum())

    # the first block's decisions
    W64 = synth.to_f64(W, wl.dtype)
    m0, decided = F.block0_expected(W64, g, pattern=wl.pattern, nm=nm, sparsity=wl.sparsity, block=wl.block,
                                    tol=TIE_TOL)
    B = min(wl.block, b)
    assert decided.mean() > 0.99
    assert np.array_equal(m[:, :B][decided], m0[decided])


def _sampled_h_error(H, wl, g, rng):
    """Largest error of 64 sampled entries of H (16 on the diagonal) against fp64 dot
    products of the regenerated activation columns, relative to 2 sqrt(G_ii G_jj)."""
    torch = _torch()
    ii = rng.integers(0, wl.b, 48)
    jj = rng.integers(0, wl.b, 48)
    ii = np.concatenate([ii, ii[:16]])
    jj = np.concatenate([jj, ii[:16]])
    Hs = H[torch.from_numpy(ii).cuda(), torch.from_numpy(jj).cuda()].cpu().numpy().astype(np.float64)
    cols = sorted(set(ii.tolist()) | set(jj.tolist()))
    row = {q: r for r, q in enumerate(cols)}
    Xc = synth.to_f64(synth.make_X_features(wl, cols), wl.dtype)        # [len(cols), n]
    ref = 2.0 * np.einsum("in,in->i", Xc[[row[i] for i in ii]], Xc[[row[j] for j in jj]])
    return float(np.max(np.abs(Hs - ref) / (2.0 * np.sqrt(g[ii] * g[jj]))))


def test_decoder_block_full_size():
    """q, k, v, o 4096x4096, gate, up 11008x4096 and down 4096x11008 pruned to 50%
    (Thanos, global budget per layer) through prune_block, one H per input: exact zeros
    and counts for every layer, sampled H entries of every input, and every layer's
    first-block selection against the oracle."""
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    blk = synth.decoder_block()
    threads = max(1, min(16, os.cpu_count() or 1))
    inputs = {}
    for inp, wl in blk.values():
        inputs.setdefault(inp, wl)
    acts, norms = {}, {}
    rng = np.random.default_rng(78)
    for inp, wl in inputs.items():
        X = synth.make_X_tokens(wl, threads=threads)
        norms[inp] = F.column_norms_sq(X, wl.dtype)
        acts[inp] = pwp.from_bf16_bits(X)
        del X
        H = pwp.hessian_accumulate(acts[inp])
        torch.cuda.synchronize()
        assert _sampled_h_error(H, wl, norms[inp], rng) < 1e-4, inp
        del H

    weights = {layer: pwp.from_bf16_bits(synth.make_W(wl)) for layer, (_, wl) in blk.items()}
    feeds = {layer: inp for layer, (inp, _) in blk.items()}
    res = pwp.prune_block(weights, acts, feeds, method="thanos", pattern="unstructured", sparsity=0.5,
                          block=128, damp=0.01)
    torch.cuda.synchronize()
    del acts
    for layer, (inp, wl) in blk.items():
        W_hat, mask, st = res[layer]
        assert st.status == 0, layer
        assert bool(torch.all(W_hat[mask.bool()] == 0).item()), layer
        m = mask.cpu().numpy().astype(bool)
        want = int(np.floor(float(np.float32(wl.sparsity)) * wl.c * wl.b))
        assert int(m.sum()) == st.pruned == st.target == want, layer
        W64 = synth.to_f64(synth.make_W(wl), wl.dtype)
        m0, decided = F.block0_expected(W64, norms[inp], pattern="unstructured", nm=(0, 0), sparsity=wl.sparsity,
                                        block=wl.block, tol=BLOCK_TIE_TOL)
        assert decided.mean() > 0.99, layer
        assert np.array_equal(m[:, :wl.block][decided], m0[decided]), layer
