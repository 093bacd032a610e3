"""Expected first-block decisions at full size.  Before any update the scores depend only
on W and the activation norms, so the oracle can give the first block's mask of a layer
too large for a full oracle run: for the global budget, the floor(s*c*b) smallest Wanda
scores over the whole layer intersected with block 0; for N:M, the groups of block 0.
Entries near the selection boundary (relative gap <= tol) are left undecided."""
import numpy as np

import oracle
import synth


def column_norms_sq(X_store, dtype, chunk=4096):
    """G_qq = sum_t X_tq^2 in fp64, over token chunks."""
    n, b = X_store.shape
    g = np.zeros(b)
    for s in range(0, n, chunk):
        xs = synth.to_f64(X_store[s:s + chunk], dtype)
        g += np.einsum("tq,tq->q", xs, xs)
    return g


def block0_expected(W64, g, *, pattern, nm, sparsity, block, tol):
    """(mask of block 0, boolean array of decided positions) for a Thanos prune."""
    c, b = W64.shape
    B = min(block, b)
    S = oracle.wanda_scores(W64, g)
    if pattern == "unstructured":
        count = int(np.floor(float(np.float32(sparsity)) * c * b))
        mask, t_last, _ = oracle.lowest_global(S, 0, count)
        decided = np.abs(S[:, :B] - t_last) > tol * max(abs(t_last), 1e-300)
        return mask[:, :B], decided
    n_keep, m = nm
    mask, gaps = oracle.nm_mask(S[:, :B], n_keep, m)
    decided = np.repeat(gaps > tol, m, axis=1)
    return mask, decided
