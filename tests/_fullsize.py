"""Helpers of the full-size parity tests.

* ``column_norms_sq`` / ``hessian64``: fp64 statistics of activations too large for one
  conversion, summed over token chunks.
* ``block0_expected``: before any update the scores depend only on W and the activation
  norms, so the oracle can give the first block's mask of a layer too large for a full
  oracle run: for the global budget, the floor(s*c*b) smallest Wanda scores over the
  whole layer intersected with block 0; for N:M, the groups of block 0.  Entries near the
  selection boundary (relative gap <= tol) are left undecided.
* ``compare_rows``: a GPU result on a subset of rows against an oracle run on the same rows.
"""
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


def hessian64(X_store, dtype, chunk=8192):
    """The undamped H = 2 X X^T in fp64 from token-major activations, over token chunks
    (independent of the GPU: only the stored activations are read)."""
    n, b = X_store.shape
    H = np.zeros((b, b))
    for s in range(0, n, chunk):
        xs = synth.to_f64(X_store[s:s + chunk], dtype)
        H += xs.T @ xs
    return 2.0 * H


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


def u_rel_error(U_gpu_storage, H64, damp):
    """Relative Frobenius error of the GPU's factor (the upper triangle of the prune's H
    storage after the call) against the fp64 U with (H + lambda I)^-1 = U^T U."""
    Hd, _ = oracle.damp_hessian(H64, damp)
    U64 = oracle.inverse_cholesky_upper(Hd)
    Ug = np.triu(np.asarray(U_gpu_storage, dtype=np.float64))
    return float(np.linalg.norm(Ug - U64) / np.linalg.norm(U64))


def compare_rows(W64_rows, W_hat_rows, mask_rows, orc, G, *, nm=None, tie_tol):
    """Element-wise comparison of the GPU's rows with an oracle run on the same rows.
    N:M disagreements are ties when the group's own score gap is within tie_tol; for a
    fixed-mask replay (nm None) the masks are equal by construction."""
    Wo, Mo = orc["W"], orc["mask"]
    dis = np.argwhere(mask_rows != Mo)
    gaps = []
    n_not_tie = 0
    if nm is not None and len(dis):
        m = nm[1]
        for k, q in dis:
            gap = float(orc["nm_gap"][k, q // m])
            gaps.append(gap)
            n_not_tie += gap > tie_tol
    else:
        n_not_tie = len(dis)
    lg = oracle.recon_loss(W64_rows, W_hat_rows, G)
    return {
        "agree": 1.0 - len(dis) / Mo.size,
        "n_dis": int(len(dis)),
        "n_dis_not_tie": int(n_not_tie),
        "dis_gaps": sorted(gaps)[-8:],
        "w_rel": float(np.linalg.norm(W_hat_rows - Wo) / np.linalg.norm(Wo)),
        "loss_gpu": lg,
        "loss_oracle": float(orc["loss"]),
        "loss_rel": abs(lg - orc["loss"]) / max(orc["loss"], 1e-300),
        "zeros_exact": bool(np.all(W_hat_rows[mask_rows] == 0.0)),
    }
