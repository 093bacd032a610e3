"""Plain fp64 CPU oracle for one-layer reconstruction pruning (Thanos; SparseGPT as
its column-sequential special case).

TEST INFRASTRUCTURE ONLY.  This module is imported by the tests, by the smoke
check and by the benchmark's CPU-baseline leg, and by nothing on the product
path.  It shares no code with the CUDA library and imports nothing from it.

Sources (web pages, cited by title and section):

* [THANOS] "Pruning LLMs with Thanos" -- sections "The layer-reconstruction
  lens", "Why magnitude alone misses important weights", "One deletion with
  compensation: the OBS view", "The scaling problem, and what SparseGPT
  changes", "Contribution one: solve a selected set directly", "Contribution
  two: keep the budget global and the execution local", "Making irregular row
  masks batchable".  The display equations of this page did not survive text
  extraction; the formulas below are rebuilt from its prose and from [BLOG].
* [BLOG] "Weight Pruning in Large Language Models: How SparseGPT, Wanda, and
  Semi-Structured 2:4 Sparsity Compress Neural Networks Without Retraining" --
  sections "SparseGPT: Second-Order Reconstruction at Scale" (objective,
  H = 2XX^T + lambda*I, the column update, Cholesky of H^-1), "Wanda: Pruning by
  Weights and Activations" (score |W_ij| * ||X_j||_2) and "N:M Semi-Structured
  Sparsity".
* [README] "Thanos - Method of Pruning LLMs" -- section "Usage" (methods
  thanos / sparsegpt, sparsity types unstructured / 2:4 / 4:8).
* [BLOG] also for the no-update baselines: "Wanda: Pruning by Weights and
  Activations" (per-row thresholds, no weight update) and "The Failure of
  Magnitude Pruning in Large Transformers" (rank by |W_ij|).

Everything is fp64.  Library primitives used as single steps: matrix product,
``numpy.linalg.inv``, ``numpy.linalg.cholesky``, ``numpy.linalg.solve``,
``numpy.partition`` / ``numpy.lexsort`` / ``numpy.argsort``.  There is no
blocking, fusion or reordering beyond what the pages' algorithm states.

Parity status: every function is pinned by the tests in tests/test_oracle.py, except that
the rule by which ``outlier_rows`` chooses its rows is a reading of a page that does not
state it -- parity unpinned for that rule (its count, tie order and the resulting sparsity
are pinned).

Notation follows [THANOS]: W is c x b (rows = outputs, columns = input
features), X is b x n with calibration examples as columns.  Activations are
passed token-major, ``Xt = X^T`` with shape [n, b].
"""
from __future__ import annotations

import math
import numpy as np

__all__ = [
    "gram", "hessian", "damp_hessian", "inverse_cholesky_upper", "active_inverse",
    "conditioned_diag", "wanda_scores", "obs_scores", "lowest_global", "nm_mask",
    "thanos_row_update", "sparsegpt_block", "prune_layer", "recon_loss", "row_losses",
    "row_quota_mask", "prune_no_update", "bf16_bits_rne", "pack_24", "outlier_rows", "prune_layer_alpha",
]


# ----------------------------------------------------------------------------- statistics

def gram(Xt: np.ndarray) -> np.ndarray:
    """G = X X^T for X (b x n) given as Xt = X^T ([n, b]).  [THANOS] "One deletion with
    compensation: the OBS view" (activation Gram matrix)."""
    Xt = np.asarray(Xt, dtype=np.float64)
    return Xt.T @ Xt


def hessian(Xt: np.ndarray) -> np.ndarray:
    """Undamped H = 2 X X^T.  [BLOG] "SparseGPT: Second-Order Reconstruction at Scale"."""
    return 2.0 * gram(Xt)


def damp_hessian(H: np.ndarray, damp: float):
    """H_d = H + lambda*I with lambda = damp * mean(diag H) of the undamped H.

    [BLOG] "SparseGPT..." gives H = 2XX^T + lambda*I; [THANOS] "One deletion with
    compensation" calls lambda*I the stabilising damping.  lambda relative to the
    mean diagonal is the reading adopted where the pages give no value."""
    H = np.asarray(H, dtype=np.float64)
    lam = float(damp) * float(np.mean(np.diag(H)))
    return H + lam * np.eye(H.shape[0]), lam


def inverse_cholesky_upper(Hd: np.ndarray) -> np.ndarray:
    """Upper-triangular U with H_d^-1 = U^T U: the Cholesky factor of the inverse
    Hessian, computed once per layer.  [BLOG] "SparseGPT..." ("Cholesky decomposition
    of H^-1 once per layer")."""
    Hinv = np.linalg.inv(Hd)
    Hinv = 0.5 * (Hinv + Hinv.T)
    L = np.linalg.cholesky(Hinv)          # Hinv = L L^T, L lower
    return L.T                            # U = L^T upper, Hinv = U^T U


def active_inverse(Hd: np.ndarray, j: int) -> np.ndarray:
    """inv(H_d[A, A]) for the active region A = [j, b): the inverse Hessian of the
    row problem once columns < j are frozen.  [THANOS] "The scaling problem..."
    (freeze completed columns, compensate only into active ones) and "Contribution
    one" (rows R and block R-hat are taken from this inverse)."""
    return np.linalg.inv(Hd[j:, j:])


def conditioned_diag(Hd: np.ndarray, q: int) -> float:
    """[inv(H_d[q:, q:])]_{qq}: the OBS denominator of column q once the columns
    before it are frozen.  [BLOG] "SparseGPT..." ([H^-1]_jj in the column update)."""
    return float(np.linalg.inv(Hd[q:, q:])[0, 0])


# ----------------------------------------------------------------------------- scores

def wanda_scores(W_region: np.ndarray, g_diag: np.ndarray) -> np.ndarray:
    """|W_kq| * ||X_q,:||_2 with ||X_q,:||_2 = sqrt(G_qq).  [BLOG] "Wanda..." and
    [THANOS] "Why magnitude alone misses important weights"; used by Thanos to rescore
    the active region ([THANOS] "Contribution two", step 2)."""
    return np.abs(W_region) * np.sqrt(g_diag)[None, :]


def obs_scores(W_region: np.ndarray, hinv_diag: np.ndarray) -> np.ndarray:
    """W_kq^2 / [H^-1]_qq, the OBS loss increase of removing one weight, with [H^-1]_qq the
    diagonal of the inverse Hessian conditioned on the frozen columns (= U_qq^2 in
    factored form).  [THANOS] "One deletion with compensation: the OBS view" (increase
    proportional to W_kq^2 / [H^-1]_qq); [BLOG] "SparseGPT..." (denominator of the
    column update)."""
    return W_region ** 2 / hinv_diag[None, :]


# ----------------------------------------------------------------------------- selection

def lowest_global(S: np.ndarray, col0: int, count: int):
    """Choose the ``count`` smallest entries of the score array S (rows k, columns
    col0 + q) in ascending (score, column, row) order.

    Returns (selected mask, score of the last selected entry, score of the first
    unselected entry).  The order among equal scores is not given by the pages; the
    lower column is taken first, then the lower row."""
    c, m = S.shape
    N = c * m
    count = int(min(max(count, 0), N))
    sel = np.zeros(N, dtype=bool)
    if count == 0:
        first_out = float(np.min(S)) if N else math.inf
        return sel.reshape(c, m), -math.inf, first_out
    flat_cm = S.T.ravel()                 # column-major: index = q * c + k, i.e. (column, row) order
    if count == N:
        sel[:] = True
        return sel.reshape(c, m), float(np.max(S)), math.inf
    # value of the count-th smallest score
    part = np.partition(flat_cm, [count - 1, count])
    t_last, t_next = float(part[count - 1]), float(part[count])
    below = flat_cm < t_last
    ties = np.flatnonzero(flat_cm == t_last)       # ascending column-major index = (column, row) order
    need = count - int(below.sum())
    chosen = below.copy()
    chosen[ties[:need]] = True
    mask = chosen.reshape(m, c).T
    return np.ascontiguousarray(mask), t_last, t_next


def nm_mask(S_block: np.ndarray, n: int, m: int):
    """N:M mask on a block whose width is a multiple of m and whose first column is
    group-aligned: in every group of m consecutive weights of a row, the m - n lowest
    scores are removed and exactly n kept.  Among equal scores the lower column goes
    first.  [THANOS] "The compression target" (N:M keeps exactly N of every M);
    [BLOG] "N:M Semi-Structured Sparsity".

    Returns (mask, relative gap) where the gap, per row and group, is the relative
    difference between the largest removed and the smallest kept score."""
    c, w = S_block.shape
    assert w % m == 0
    mask = np.zeros((c, w), dtype=bool)
    gaps = np.zeros((c, w // m))
    for g in range(0, w, m):
        grp = S_block[:, g:g + m]
        order = np.argsort(grp, axis=1, kind="stable")
        drop = order[:, : m - n]
        np.put_along_axis(mask[:, g:g + m], drop, True, axis=1)
        srt = np.take_along_axis(grp, order, axis=1)
        lo, hi = srt[:, m - n - 1], srt[:, m - n]
        gaps[:, g // m] = (hi - lo) / np.maximum(np.abs(hi), 1e-300)
    return mask, gaps


# ----------------------------------------------------------------------------- updates

def thanos_row_update(w_A: np.ndarray, Q: np.ndarray, K_QA: np.ndarray) -> np.ndarray:
    """Joint multi-constraint update of one row over the active region A.

    u = w[Q] (current values of the coordinates to remove), R = K[Q, A] (rows of the
    active inverse Hessian), R-hat = K[Q, Q]; the constrained optimum is
    delta = -u^T R-hat^-1 R, which zeroes every coordinate in Q and moves the rest of
    A to minimise the damped quadratic model.  [THANOS] "Contribution one: solve a
    selected set directly".  Entries in Q are then set to exactly 0."""
    w = np.array(w_A, dtype=np.float64)
    Q = np.asarray(Q, dtype=np.int64)
    if Q.size == 0:
        return w
    u = w[Q]
    Rhat = K_QA[:, Q]
    z = np.linalg.solve(Rhat, u)
    w = w - z @ K_QA
    w[Q] = 0.0
    return w


def sparsegpt_block(W: np.ndarray, j0: int, j1: int, mask_J: np.ndarray, *, U=None, Hd=None):
    """Column-sequential OBS sweep over block [j0, j1), in place on W.

    For each column q in order: e = W[:, q] / [H^-1]_qq on the masked rows (0
    elsewhere) and W[:, q:] -= e * H^-1[q, q:], with H^-1 the inverse of H_d[q:, q:]
    (columns before q frozen for every row at once).  [BLOG] "SparseGPT..." (column
    update); [THANOS] "The scaling problem, and what SparseGPT changes" (steps 1-4).

    Factored form (``U`` given): [inv(H_d[q:,q:])]_{q,q:} = U_qq * U[q, q:], so the
    update is W[:, q:] -= (W[:, q] / U_qq) * U[q, q:] on masked rows.
    Definitional form (``Hd`` given): the inverse is formed for every column."""
    c, b = W.shape
    for q in range(j0, j1):
        m = mask_J[:, q - j0]
        if U is not None:
            e = np.where(m, W[:, q] / U[q, q], 0.0)
            W[:, q:] -= np.outer(e, U[q, q:])
        else:
            K = np.linalg.inv(Hd[q:, q:])
            e = np.where(m, W[:, q] / K[0, 0], 0.0)
            W[:, q:] -= np.outer(e, K[0, :])
        W[m, q] = 0.0


# ----------------------------------------------------------------------------- losses

def row_losses(W: np.ndarray, What: np.ndarray, G: np.ndarray) -> np.ndarray:
    """||(W-hat_k - W_k) X||^2 = Delta_k G Delta_k^T per row.  [THANOS] "The
    layer-reconstruction lens" (the loss decomposes over rows)."""
    D = np.asarray(What, np.float64) - np.asarray(W, np.float64)
    return np.einsum("kq,kq->k", D @ G, D)


def recon_loss(W: np.ndarray, What: np.ndarray, G: np.ndarray) -> float:
    """||(W-hat - W) X||_F^2 = sum_k Delta_k G Delta_k^T.  [THANOS] "The layer-reconstruction lens"."""
    return float(np.sum(row_losses(W, What, G)))


# ----------------------------------------------------------------------------- the layer

def prune_layer(W, *, Xt=None, H=None, sparsity=0.5, pattern="unstructured", nm=(2, 4),
                block=128, damp=0.01, method="thanos", mode="factored", rows=None, fixed_mask=None):
    """Prune one linear layer.

    W: c x b weights (any float dtype, widened exactly to fp64).  Xt: [n, b]
    token-major activations, or H: the undamped 2XX^T (b x b).  ``rows``: optional
    subset of rows of W to process -- valid only where rows do not interact (N:M
    patterns and the per-row work of a fixed mask); the unstructured global budget
    couples all rows and needs every row.  ``fixed_mask``: optional c x b boolean mask
    (for the processed rows) used as every block's selection instead of choosing one
    (Thanos only; for the global budget over all rows, each block also records in
    ``blocks`` the selection the budget loop would have made on the replayed state --
    ``chosen``, with its residual count and thresholds; for N:M, the groups' ``chosen``
    removals and their ``nm_gap`` on the replayed state).  Once the masks are given the rows do not interact -- the loss is a sum
    of per-row terms ([THANOS] "The layer-reconstruction lens") and each row's update
    depends only on its own selected set ([THANOS] "Contribution one") -- so any subset of
    rows of a layer pruned elsewhere can be replayed exactly, also under the global budget.

    Thanos (method="thanos"), per block J = [j, j+B) with active region A = [j, b):
      1. K = inv(H_d[A, A]) (mode "definitional") or K[J, A] = U[J,J]^T U[J,A] with
         U the upper Cholesky factor of H_d^-1 (mode "factored"; the two agree because
         inv(H_d[A,A]) = U[A,A]^T U[A,A] for a trailing block A).
      2. Unstructured: r = floor(s*c*b) - pruned so far; rescore the whole active
         region with |W|*||X_q||; the r lowest form the provisional candidate set; the
         block mask is its intersection with J.  [THANOS] "Contribution two", steps 1-5.
         N:M: groups of m inside J, m - n lowest removed.  [THANOS] "Contribution two"
         (last paragraph).
      3. Each row solves its joint system on its selected set and updates the whole
         active part of the row.  [THANOS] "Contribution one".
    SparseGPT (method="sparsegpt"): per block the mask is chosen at the block start by
    W^2/[H^-1]_qq^2 (unstructured: the floor(s*c*|J|) lowest of the c x |J| block;
    N:M: per group), then the column-sequential sweep of ``sparsegpt_block`` runs.
    [THANOS] "The scaling problem..." (step 5: refresh decisions block by block).

    Returns a dict with W_hat (fp64), mask (bool, True = pruned), loss, lam, U and
    per-block diagnostics used to classify near-tie mask differences."""
    W0 = np.array(W, dtype=np.float64)
    if rows is not None:
        W0 = W0[np.asarray(rows)]
    c, b = W0.shape
    if H is None:
        H = hessian(Xt)
    H = np.asarray(H, dtype=np.float64)
    G = 0.5 * H
    g_diag = np.diag(G).copy()
    Hd, lam = damp_hessian(H, damp)
    U = inverse_cholesky_upper(Hd) if mode == "factored" else None
    B = int(block)
    unstructured = pattern == "unstructured"
    if not unstructured:
        n_keep, m_grp = nm
        assert b % m_grp == 0 and B % m_grp == 0
    if unstructured and method == "thanos" and rows is not None and fixed_mask is None:
        raise ValueError("the global budget couples rows; a row subset is not defined")
    if fixed_mask is not None:
        if method != "thanos":
            raise ValueError("fixed_mask replays Thanos row updates only")
        fixed_mask = np.asarray(fixed_mask, dtype=bool)
        assert fixed_mask.shape == (c, b)

    What = W0.copy()
    mask = np.zeros((c, b), dtype=bool)
    dscore = np.zeros((c, b))            # score of each weight in the block where its column was decided
    nm_gap = None if unstructured else np.zeros((c, b // nm[1]))
    zstar = int(math.floor(sparsity * c * b))
    pruned = 0
    blocks = []
    shortfall = False

    for j in range(0, b, B):
        j1 = min(j + B, b)
        nJ = j1 - j
        info = {"j": j}
        if method == "thanos":
            if mode == "factored":
                K_JA = U[j:j1, j:j1].T @ U[j:j1, j:]
            else:
                K_JA = active_inverse(Hd, j)[:nJ, :]
            if fixed_mask is not None:
                M = fixed_mask[:, j:j1]
                dscore[:, j:j1] = wanda_scores(What[:, j:j1], g_diag[j:j1])
                if not unstructured:
                    # the groups the N:M rule would remove on this (replayed) state
                    chosen, gaps = nm_mask(dscore[:, j:j1], n_keep, m_grp)
                    info.update(chosen=chosen, nm_gap=gaps)
                if unstructured and rows is None:
                    # what step 3 of the budget loop would choose on this (replayed) state,
                    # with the residual count left by the given mask's earlier blocks
                    S = wanda_scores(What[:, j:], g_diag[j:])
                    r = zstar - pruned
                    chosen, t_last, t_next = lowest_global(S, j, min(max(r, 0), c * (b - j)))
                    info.update(r=r, chosen=chosen[:, :nJ], t_last=t_last, t_next=t_next)
            elif unstructured:
                S = wanda_scores(What[:, j:], g_diag[j:])
                r = zstar - pruned
                take = min(r, c * (b - j))
                if take < r:
                    shortfall = True
                sel, t_last, t_next = lowest_global(S, j, take)
                M = sel[:, :nJ]
                info.update(r=r, take=take, t_last=t_last, t_next=t_next)
                dscore[:, j:j1] = S[:, :nJ]
            else:
                S = wanda_scores(What[:, j:j1], g_diag[j:j1])
                M, gaps = nm_mask(S, n_keep, m_grp)
                nm_gap[:, j // m_grp: j1 // m_grp] = gaps
                dscore[:, j:j1] = S
            for k in range(c):
                Q = np.flatnonzero(M[k])
                if Q.size:
                    What[k, j:] = thanos_row_update(What[k, j:], Q, K_JA[Q, :])
        elif method == "sparsegpt":
            if mode == "factored":
                hd = np.diag(U)[j:j1] ** 2
            else:
                hd = np.array([conditioned_diag(Hd, q) for q in range(j, j1)])
            S = obs_scores(What[:, j:j1], hd)
            if unstructured:
                quota = int(math.floor(sparsity * c * nJ))
                M, t_last, t_next = lowest_global(S, j, quota)
                info.update(take=quota, t_last=t_last, t_next=t_next)
            else:
                M, gaps = nm_mask(S, n_keep, m_grp)
                nm_gap[:, j // m_grp: j1 // m_grp] = gaps
            dscore[:, j:j1] = S
            if mode == "factored":
                sparsegpt_block(What, j, j1, M, U=U)
            else:
                sparsegpt_block(What, j, j1, M, Hd=Hd)
        else:
            raise ValueError(method)
        mask[:, j:j1] = M
        pruned += int(M.sum())
        info["pruned"] = int(M.sum())
        blocks.append(info)

    return {
        "W": What, "mask": mask, "loss": recon_loss(W0, What, G), "lam": lam, "U": U,
        "g_diag": g_diag, "blocks": blocks, "dscore": dscore, "nm_gap": nm_gap,
        "zstar": zstar, "pruned": pruned, "shortfall": shortfall,
    }


# ----------------------------------------------------------------------------- no-update baselines

def row_quota_mask(S: np.ndarray, count: int) -> np.ndarray:
    """Per output row, remove the ``count`` lowest scores; among equal scores the lower
    column goes first.  [BLOG] "Wanda: Pruning by Weights and Activations" (the pruning
    threshold is set independently for each output row, and the lowest s% of the row's
    scores are zeroed)."""
    c, b = S.shape
    mask = np.zeros((c, b), dtype=bool)
    if count <= 0:
        return mask
    cols = np.arange(b)
    for k in range(c):
        order = np.lexsort((cols, S[k]))      # by score, then by column
        mask[k, order[:count]] = True
    return mask


def prune_no_update(W, *, Xt=None, H=None, sparsity=0.5, pattern="unstructured", nm=(2, 4),
                    method="wanda"):
    """Wanda or magnitude pruning of one layer: a score per weight, a per-row mask, and no
    compensation -- kept weights are returned unchanged, removed ones are exactly 0.

    method "wanda": S_kq = |W_kq| * ||X_q||_2 with ||X_q||^2 = G_qq = (X X^T)_qq, taken
      from Xt ([n, b]) or from an undamped H = 2 X X^T as H_qq / 2.  [BLOG] "Wanda:
      Pruning by Weights and Activations".
    method "magnitude": S_kq = |W_kq|.  [BLOG] "The Failure of Magnitude Pruning in Large
      Transformers"; [THANOS] "Why magnitude alone misses important weights".  The pages
      do not say whether its quota is per row or per layer; the per-row quota of Wanda
      is used.
    pattern "unstructured": floor(sparsity * b) removed per row; "nm": in every aligned
      group of m consecutive weights of a row, the m - n lowest removed (nm_mask).
    Returns a dict with W (fp64), mask, pruned, target and the scores S."""
    W = np.asarray(W, dtype=np.float64)
    c, b = W.shape
    if method == "wanda":
        if Xt is not None:
            g = np.einsum("tq,tq->q", np.asarray(Xt, dtype=np.float64), np.asarray(Xt, dtype=np.float64))
        else:
            g = 0.5 * np.diag(np.asarray(H, dtype=np.float64))
        S = wanda_scores(W, g)
    elif method == "magnitude":
        S = np.abs(W)
    else:
        raise ValueError(method)
    if pattern == "unstructured":
        count = int(np.floor(float(sparsity) * b))
        mask = row_quota_mask(S, count)
        target = c * count
    else:
        n, m = nm
        mask, _ = nm_mask(S, n, m)
        target = c * (b // m) * (m - n)
    What = np.where(mask, 0.0, W)
    return {"W": What, "mask": mask, "pruned": int(mask.sum()), "target": target, "S": S}


# ----------------------------------------------------------------------------- 2:4 storage

def bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns of fp32 values, rounded to nearest with ties to even (the
    upper 16 bits of the fp32 pattern after adding 0x7fff plus the kept half's lowest
    bit).  Finite inputs only."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def pack_24(What: np.ndarray, mask: np.ndarray):
    """Compressed 2:4 storage of a pruned layer: in every aligned group of four weights of
    a row exactly two are kept; store those two values at 16-bit precision (bfloat16, in
    column order) and their 2-bit positions in the group.  [BLOG] "N:M Semi-Structured
    Sparsity (2:4 Pattern)": only the 2 non-zero values and 2-bit index metadata are
    stored.  The pages do not give the metadata layout the tensor cores read; here each
    group's positions form one 4-bit field idx0 | idx1 << 2 (idx0 < idx1), eight groups per
    32-bit word, the first group in the lowest bits, words row-major (ceil(b/32) per row).
    Returns (values: uint16 c x b/2, meta: uint32 c x ceil(b/32))."""
    What = np.asarray(What, dtype=np.float32)
    mask = np.asarray(mask, dtype=bool)
    c, b = What.shape
    assert b % 4 == 0
    groups = b // 4
    values = np.zeros((c, 2 * groups), dtype=np.uint16)
    meta = np.zeros((c, (groups + 7) // 8), dtype=np.uint32)
    bits = bf16_bits_rne(What)
    for k in range(c):
        for g in range(groups):
            kept = [e for e in range(4) if not mask[k, 4 * g + e]]
            assert len(kept) == 2, (k, g)
            values[k, 2 * g] = bits[k, 4 * g + kept[0]]
            values[k, 2 * g + 1] = bits[k, 4 * g + kept[1]]
            meta[k, g // 8] |= np.uint32((kept[0] | (kept[1] << 2)) << (4 * (g % 8)))
    return values, meta



# ----------------------------------------------------------------------------- outlier rows (alpha)

def outlier_rows(W, g_diag, alpha):
    """The rows kept dense by the alpha variant: floor(alpha * c) rows of W with the largest
    sum over q of (W_kq * ||X_q||)^2 = W_kq^2 G_qq (ties: the lower row first).

    [THANOS] "Thanos versus SparseGPT on LLaMA-3 8B": the alpha = 0.1 variant keeps 10% of
    the rows as outliers, which lowers the total N:M sparsity from 50% to 45%.  The page does
    not say how the rows are chosen; the reading here ranks a row by the squared norm of its
    activation-aware scores (the scores of [BLOG] "Wanda..." that Thanos rescores with,
    [THANOS] "Contribution two").  Returns a boolean array over rows."""
    W = np.asarray(W, dtype=np.float64)
    c = W.shape[0]
    n_out = int(math.floor(float(alpha) * c))
    score = (W ** 2) @ np.asarray(g_diag, dtype=np.float64)
    order = np.lexsort((np.arange(c), -score))      # by score descending, then row ascending
    out = np.zeros(c, dtype=bool)
    out[order[:n_out]] = True
    return out


def prune_layer_alpha(W, *, Xt=None, H=None, alpha=0.0, **kw):
    """The alpha variant of ``prune_layer``: the outlier rows (``outlier_rows``) keep their
    weights, and the other rows are pruned as a layer of their own with the same
    configuration (for the unstructured global budget: floor(sparsity * rows * b) of their
    weights).  Returns ``prune_layer``'s dict for the whole layer (W, mask, loss, pruned,
    zstar) plus "outliers" and "inner", the pruned rows' own result."""
    W0 = np.array(W, dtype=np.float64)
    if H is None:
        H = hessian(Xt)
    H = np.asarray(H, dtype=np.float64)
    g = 0.5 * np.diag(H)
    out = outlier_rows(W0, g, alpha)
    keep = ~out
    inner = prune_layer(W0[keep], H=H, **kw)
    What = W0.copy()
    What[keep] = inner["W"]
    mask = np.zeros(W0.shape, dtype=bool)
    mask[keep] = inner["mask"]
    return {"W": What, "mask": mask, "loss": recon_loss(W0, What, 0.5 * H), "outliers": out, "inner": inner,
            "pruned": inner["pruned"], "zstar": inner["zstar"]}
