"""Pins for the fp64 oracle: each test checks the oracle against something other than
itself -- hand-derived values, closed forms, brute force on tiny inputs, textbook
special cases and invariants the pages state.  CPU only, seconds.

Page titles cited: "Pruning LLMs with Thanos" (THANOS) and "Weight Pruning in Large
Language Models: How SparseGPT, Wanda, and Semi-Structured 2:4 Sparsity ..." (BLOG).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(seed, c=6, b=10, n=24, outlier=True):
    rng = np.random.default_rng(seed)
    Xt = rng.normal(size=(n, b))
    if outlier:
        Xt[:, rng.integers(b)] *= 7.0
    W = rng.normal(scale=0.5, size=(c, b))
    return W, Xt


def _brute_gram(Xt):
    n, b = Xt.shape
    G = np.zeros((b, b))
    for i in range(b):
        for j in range(b):
            s = 0.0
            for t in range(n):
                s += Xt[t, i] * Xt[t, j]
            G[i, j] = s
    return G


# --------------------------------------------------------------------------- statistics

def test_gram_matches_triple_loop():
    _, Xt = _rand_problem(0, b=5, n=7)
    assert np.allclose(oracle.gram(Xt), _brute_gram(Xt), rtol=1e-13, atol=1e-13)
    assert np.allclose(oracle.hessian(Xt), 2.0 * _brute_gram(Xt), rtol=1e-13, atol=1e-13)


def test_damping_is_relative_to_mean_undamped_diagonal():
    H = np.diag([1.0, 2.0, 3.0, 6.0])
    Hd, lam = oracle.damp_hessian(H, 0.5)
    assert lam == pytest.approx(0.5 * 3.0)
    assert np.allclose(np.diag(Hd), [2.5, 3.5, 4.5, 7.5])


def test_inverse_cholesky_upper_is_upper_and_factors_inverse():
    W, Xt = _rand_problem(1)
    Hd, _ = oracle.damp_hessian(oracle.hessian(Xt), 0.01)
    U = oracle.inverse_cholesky_upper(Hd)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.all(np.diag(U) > 0)
    assert np.allclose(U.T @ U @ Hd, np.eye(Hd.shape[0]), atol=1e-10)
    # trailing principal inverses come from U's trailing block (what the factored mode relies on)
    for j in range(Hd.shape[0]):
        assert np.allclose(U[j:, j:].T @ U[j:, j:], np.linalg.inv(Hd[j:, j:]), rtol=1e-9, atol=1e-12)


# --------------------------------------------------------------------------- single deletion (I1)

def test_single_deletion_error_closed_form():
    """THANOS 'Why magnitude alone misses important weights': deleting W_kq with the rest
    frozen costs W_kq^2 ||X_q||^2; with H it is W_kq^2 H_qq."""
    W, Xt = _rand_problem(2)
    G = oracle.gram(Xt)
    H = oracle.hessian(Xt)
    c, b = W.shape
    for k in range(c):
        for q in range(b):
            Wd = W.copy()
            Wd[k, q] = 0.0
            direct = float(np.sum(((Wd - W) @ Xt.T) ** 2))
            closed = W[k, q] ** 2 * np.sum(Xt[:, q] ** 2)
            assert oracle.recon_loss(W, Wd, G) == pytest.approx(closed, rel=1e-12)
            assert direct == pytest.approx(closed, rel=1e-12)
            d = np.zeros(b)
            d[q] = -W[k, q]
            assert d @ H @ d == pytest.approx(W[k, q] ** 2 * H[q, q], rel=1e-12)
    # Wanda's score squared orders weights exactly like the deletion error
    S = oracle.wanda_scores(W, np.diag(G))
    assert np.allclose(S ** 2, W ** 2 * np.diag(G)[None, :], rtol=1e-12)


# --------------------------------------------------------------------------- row decomposition (I2)

def test_loss_decomposes_over_rows():
    W, Xt = _rand_problem(3, c=8)
    r = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=4)
    direct = float(np.sum(((r["W"] - W) @ Xt.T) ** 2))
    per_row = oracle.row_losses(W, r["W"], oracle.gram(Xt))
    assert r["loss"] == pytest.approx(direct, rel=1e-10)
    assert per_row.sum() == pytest.approx(direct, rel=1e-10)
    for k in range(W.shape[0]):
        assert per_row[k] == pytest.approx(float(np.sum(((r["W"][k] - W[k]) @ Xt.T) ** 2)), rel=1e-10)


# --------------------------------------------------------------------------- joint update (I3, I13)

def _lstsq_row(w, Xt, lam, j, Q_abs):
    """min over delta supported on [j, b) with delta_Q = -w_Q of
    ||sqrt2 X^T delta||^2 + lam ||delta||^2, solved as a least-squares problem."""
    n, b = Xt.shape
    A = np.arange(j, b)
    F = np.array([q for q in A if q not in set(Q_abs)], dtype=int)
    M = np.vstack([math.sqrt(2.0) * Xt, math.sqrt(lam) * np.eye(b)])
    dQ = -w[Q_abs]
    rhs = -(M[:, Q_abs] @ dQ)
    dF = np.linalg.lstsq(M[:, F], rhs, rcond=None)[0] if F.size else np.zeros(0)
    out = w.copy()
    out[Q_abs] = 0.0
    out[F] += dF
    return out


@pytest.mark.parametrize("seed", range(4))
def test_row_update_equals_constrained_least_squares(seed):
    W, Xt = _rand_problem(10 + seed, c=3, b=9, n=20)
    damp = 0.05
    H = oracle.hessian(Xt)
    Hd, lam = oracle.damp_hessian(H, damp)
    rng = np.random.default_rng(seed)
    for j in (0, 2, 5):
        K = oracle.active_inverse(Hd, j)
        for size in range(1, 4):
            Q_rel = np.sort(rng.choice(min(4, 9 - j), size=min(size, 9 - j), replace=False))
            w = W[0]
            got = w.copy()
            got[j:] = oracle.thanos_row_update(w[j:], Q_rel, K[Q_rel, :])
            want = _lstsq_row(w, Xt, lam, j, Q_rel + j)
            assert np.allclose(got, want, rtol=1e-9, atol=1e-11)
            assert np.all(got[Q_rel + j] == 0.0)
            assert np.array_equal(got[:j], w[:j])


def test_single_block_is_optimal_over_every_mask_exhaustive():
    """c=1, b=6, one block: for every 3-of-6 mask, the joint update reaches the least-squares
    optimum of the damped objective, so no other choice of kept values does better."""
    W, Xt = _rand_problem(20, c=1, b=6, n=15)
    H = oracle.hessian(Xt)
    Hd, lam = oracle.damp_hessian(H, 0.01)
    K = oracle.active_inverse(Hd, 0)
    w = W[0]
    for Q in itertools.combinations(range(6), 3):
        Q = np.array(Q)
        got = oracle.thanos_row_update(w, Q, K[Q, :])
        want = _lstsq_row(w, Xt, lam, 0, Q)
        assert np.allclose(got, want, rtol=1e-9, atol=1e-11)
        d = got - w
        rng = np.random.default_rng(0)
        for _ in range(5):       # random feasible perturbations never lower the damped loss
            p = rng.normal(size=6) * 1e-3
            p[Q] = 0.0
            assert (d + p) @ Hd @ (d + p) >= d @ Hd @ d - 1e-12


# --------------------------------------------------------------------------- hand-derived goldens

def _golden_cases():
    with open(os.path.join(GOLDEN, "obs_hand_examples.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_derived_examples(case):
    s = case.get("sparsity")
    if s is None:
        s = case["sparsity_num"] / case["sparsity_den"]
    r = oracle.prune_layer(np.array(case["W"]), H=np.array(case["H"], float), sparsity=s,
                           block=case["block"], damp=0.0, method=case["method"])
    assert np.allclose(r["W"], case["W_hat"], rtol=0, atol=1e-12)
    assert np.array_equal(r["mask"].astype(int), np.array(case["mask"]))
    assert r["loss"] == pytest.approx(case["loss"], rel=1e-12)
    r2 = oracle.prune_layer(np.array(case["W"]), H=np.array(case["H"], float), sparsity=s,
                            block=case["block"], damp=0.0, method=case["method"], mode="definitional")
    assert np.allclose(r2["W"], case["W_hat"], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- invariants (I4, I5)

@pytest.mark.parametrize("method", ["thanos", "sparsegpt"])
@pytest.mark.parametrize("c,b,B", [(7, 24, 8), (5, 30, 8), (9, 17, 5), (1, 12, 12)])
def test_unstructured_budget_and_exact_zeros(method, c, b, B):
    rng = np.random.default_rng(c * b)
    Xt = rng.normal(size=(3 * b, b))
    W = rng.normal(size=(c, b))
    for s in (0.0, 0.3, 0.5, 0.9):
        r = oracle.prune_layer(W, Xt=Xt, sparsity=s, block=B, method=method)
        assert np.all(r["W"][r["mask"]] == 0.0)
        if method == "thanos":
            assert int(r["mask"].sum()) == math.floor(s * c * b)
        else:
            want = sum(math.floor(s * c * (min(j + B, b) - j)) for j in range(0, b, B))
            assert int(r["mask"].sum()) == want


@pytest.mark.parametrize("method", ["thanos", "sparsegpt"])
@pytest.mark.parametrize("nm", [(2, 4), (4, 8), (1, 4)])
def test_nm_groups_keep_exactly_n(method, nm):
    n_keep, m = nm
    rng = np.random.default_rng(5)
    b = 32
    Xt = rng.normal(size=(80, b))
    W = rng.normal(size=(6, b))
    r = oracle.prune_layer(W, Xt=Xt, pattern="nm", nm=nm, block=16, method=method)
    groups = r["mask"].reshape(6, b // m, m)
    assert np.all(groups.sum(axis=2) == m - n_keep)
    assert np.all(r["W"][r["mask"]] == 0.0)


def test_nm_ties_prune_lower_column_first():
    S = np.array([[1.0, 1.0, 1.0, 1.0, 3.0, 2.0, 2.0, 1.0]])
    mask, _ = oracle.nm_mask(S, 2, 4)
    assert mask.astype(int).tolist() == [[1, 1, 0, 0, 0, 1, 0, 1]]


@pytest.mark.parametrize("n,m", [(1, 4), (2, 4), (4, 8), (3, 8)])
def test_nm_mask_by_exhaustive_subsets(n, m):
    """Brute force over every removal set of size m - n in each group: exactly one set has
    every removed (score, column) below every kept one, and nm_mask removes that set; the
    reported gap is that of the boundary pair.  Small integer scores make ties common."""
    rng = np.random.default_rng(100 + 10 * n + m)
    S = rng.integers(0, 4, size=(5, 2 * m)).astype(float) + 1.0
    mask, gaps = oracle.nm_mask(S, n, m)
    for k in range(S.shape[0]):
        for g in range(0, S.shape[1], m):
            cols = range(g, g + m)
            valid = []
            for R in itertools.combinations(cols, m - n):
                kept = [q for q in cols if q not in R]
                if max((S[k, q], q) for q in R) < min((S[k, q], q) for q in kept):
                    valid.append(set(R))
            assert len(valid) == 1
            assert {q for q in cols if mask[k, q]} == valid[0]
            hi = min(S[k, q] for q in cols if q not in valid[0])
            lo = max(S[k, q] for q in valid[0])
            assert gaps[k, g // m] == pytest.approx((hi - lo) / abs(hi))


def test_global_selection_tie_order():
    S = np.array([[1.0, 0.5, 1.0],
                  [1.0, 2.0, 1.0]])
    # order by (score, column, row): (0.5,1,0), (1,0,0), (1,0,1), (1,2,0), (1,2,1), (2,1,1)
    m, t_last, t_next = oracle.lowest_global(S, 0, 3)
    assert m.astype(int).tolist() == [[1, 1, 0], [1, 0, 0]]
    assert (t_last, t_next) == (1.0, 1.0)
    m, _, _ = oracle.lowest_global(S, 0, 4)
    assert m.astype(int).tolist() == [[1, 1, 1], [1, 0, 0]]


# --------------------------------------------------------------------------- diagonal Hessian (I6)

def test_orthogonal_features_reduce_to_static_wanda_selection():
    """With X X^T diagonal no update reaches another coordinate, so the dynamic global
    budget picks exactly the static lowest floor(s c b) Wanda scores."""
    rng = np.random.default_rng(7)
    c, b, n = 9, 20, 40
    Qo, _ = np.linalg.qr(rng.normal(size=(n, b)))
    d = rng.uniform(0.5, 3.0, size=b)
    Xt = Qo * d[None, :]                      # columns orthogonal -> X X^T = diag(d^2)
    W = rng.normal(size=(c, b))
    r = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=4)
    score = np.abs(W) * d[None, :]
    k = math.floor(0.5 * c * b)
    idx = np.argsort(score.ravel(), kind="stable")[:k]
    static = np.zeros(c * b, bool)
    static[idx] = True
    assert np.array_equal(r["mask"], static.reshape(c, b))
    assert np.allclose(r["W"], np.where(r["mask"], 0.0, W), atol=1e-12)


# --------------------------------------------------------------------------- padding (I7)

def test_identity_padding_leaves_updates_unchanged():
    """THANOS 'Making irregular row masks batchable': padded u (zeros), R (zero rows) and
    R-hat (identity fill) give the same updates as the unpadded per-row solves."""
    W, Xt = _rand_problem(30, c=5, b=12, n=30)
    Hd, _ = oracle.damp_hessian(oracle.hessian(Xt), 0.01)
    K = oracle.active_inverse(Hd, 0)
    rng = np.random.default_rng(1)
    Qs = [np.sort(rng.choice(6, size=s, replace=False)) for s in (0, 1, 3, 2, 5)]
    smax = max(len(q) for q in Qs)
    U_pad = np.zeros((5, smax))
    R_pad = np.zeros((5, smax, 12))
    Rh_pad = np.tile(np.eye(smax), (5, 1, 1))
    for k, Q in enumerate(Qs):
        s = len(Q)
        U_pad[k, :s] = W[k, Q]
        R_pad[k, :s] = K[Q, :]
        Rh_pad[k, :s, :s] = K[np.ix_(Q, Q)]
    Z = np.linalg.solve(Rh_pad, U_pad[..., None])[..., 0]
    D_pad = -np.einsum("ks,ksa->ka", Z, R_pad)
    for k, Q in enumerate(Qs):
        got = oracle.thanos_row_update(W[k], Q, K[Q, :])
        want = W[k] + D_pad[k]
        want[Q] = 0.0
        assert np.allclose(got, want, atol=1e-12)


# --------------------------------------------------------------------------- sequential OBS (I8)

@pytest.mark.parametrize("seed", range(3))
def test_joint_update_equals_correctly_conditioned_sequential_obs(seed):
    """THANOS 'The scaling problem...': sequential OBS with the inverse downdated after each
    removal (other coordinates stay free) represents the same fixed constraint set."""
    W, Xt = _rand_problem(40 + seed, c=1, b=10, n=25)
    Hd, _ = oracle.damp_hessian(oracle.hessian(Xt), 0.02)
    K = oracle.active_inverse(Hd, 0)
    Q = np.array([1, 4, 5, 8])
    joint = oracle.thanos_row_update(W[0], Q, K[Q, :])
    rng = np.random.default_rng(seed)
    for _ in range(3):
        w = W[0].copy()
        Kc = K.copy()
        for q in rng.permutation(Q):
            w = w - (w[q] / Kc[q, q]) * Kc[q, :]
            Kc = Kc - np.outer(Kc[:, q], Kc[q, :]) / Kc[q, q]
        w[Q] = 0.0
        assert np.allclose(w, joint, atol=1e-10)


# --------------------------------------------------------------------------- loss ordering (I9)

def test_joint_update_is_below_every_other_update_for_the_same_mask():
    """With one block and a fixed mask the joint update is the exact minimiser of the damped
    objective (THANOS 'Contribution one'), so the column-sequential update and the no-update
    (Wanda-style) result -- both feasible for the same mask -- can only be worse.  Between
    those two there is no fixed order: each sequential step is measured from the already
    compensated weights, not from W."""
    W, Xt = _rand_problem(50, c=6, b=16, n=40)
    H = oracle.hessian(Xt)
    Hd, _ = oracle.damp_hessian(H, 0.01)
    U = oracle.inverse_cholesky_upper(Hd)
    r = oracle.prune_layer(W, H=H, sparsity=0.5, block=16)        # one block
    mask = r["mask"]
    Ws = W.copy()
    oracle.sparsegpt_block(Ws, 0, 16, mask, U=U)
    Wz = np.where(mask, 0.0, W)

    def damped(Wx):
        D = Wx - W
        return np.einsum("kq,kq->k", D @ Hd, D)
    assert np.all(damped(r["W"]) <= damped(Ws) + 1e-12)
    assert np.all(damped(r["W"]) <= damped(Wz) + 1e-12)
    assert np.any(damped(r["W"]) < damped(Ws) - 1e-6)


# --------------------------------------------------------------------------- scale (I10)

@pytest.mark.parametrize("method,pattern", [("thanos", "unstructured"), ("thanos", "nm"),
                                            ("sparsegpt", "unstructured"), ("sparsegpt", "nm")])
def test_scaling_activations_leaves_result_unchanged(method, pattern):
    W, Xt = _rand_problem(60, c=6, b=16, n=40)
    a = oracle.prune_layer(W, Xt=Xt, block=8, method=method, pattern=pattern)
    b_ = oracle.prune_layer(W, Xt=3.7 * Xt, block=8, method=method, pattern=pattern)
    assert np.array_equal(a["mask"], b_["mask"])
    assert np.allclose(a["W"], b_["W"], rtol=1e-9, atol=1e-12)


# --------------------------------------------------------------------------- factored form (I11)

@pytest.mark.parametrize("method,pattern,B", [("thanos", "unstructured", 5), ("thanos", "nm", 8),
                                              ("sparsegpt", "unstructured", 6), ("sparsegpt", "nm", 4)])
def test_definitional_and_factored_modes_agree(method, pattern, B):
    W, Xt = _rand_problem(70, c=7, b=24, n=50)
    a = oracle.prune_layer(W, Xt=Xt, block=B, method=method, pattern=pattern, mode="factored")
    d = oracle.prune_layer(W, Xt=Xt, block=B, method=method, pattern=pattern, mode="definitional")
    assert np.array_equal(a["mask"], d["mask"])
    assert np.allclose(a["W"], d["W"], rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------- B = 1 (I12)

def test_thanos_with_unit_block_is_the_sparsegpt_column_update():
    W, Xt = _rand_problem(80, c=5, b=12, n=30)
    Hd, _ = oracle.damp_hessian(oracle.hessian(Xt), 0.01)
    U = oracle.inverse_cholesky_upper(Hd)
    mask = np.random.default_rng(0).random(W.shape) < 0.5
    Wt = W.copy()
    for q in range(12):
        K_row = oracle.active_inverse(Hd, q)[:1, :]        # the single block row of inv(H_d[q:, q:])
        for k in range(5):
            if mask[k, q]:
                Wt[k, q:] = oracle.thanos_row_update(Wt[k, q:], np.array([0]), K_row)
    Ws = W.copy()
    oracle.sparsegpt_block(Ws, 0, 12, mask, U=U)
    Wd = W.copy()
    oracle.sparsegpt_block(Wd, 0, 12, mask, Hd=Hd)
    assert np.allclose(Wt, Ws, atol=1e-11)
    assert np.allclose(Wd, Ws, atol=1e-11)


def test_sparsegpt_uses_conditioned_diagonal():
    W, Xt = _rand_problem(90, c=3, b=8, n=20)
    Hd, _ = oracle.damp_hessian(oracle.hessian(Xt), 0.01)
    U = oracle.inverse_cholesky_upper(Hd)
    for q in range(8):
        assert U[q, q] ** 2 == pytest.approx(oracle.conditioned_diag(Hd, q), rel=1e-10)


def test_obs_score_is_the_compensated_single_removal_loss():
    """"Pruning LLMs with Thanos", "One deletion with compensation: the OBS view": removing
    W_kq and letting the row's other weights compensate raises the loss by an amount
    proportional to W_kq^2 / [H^-1]_qq.  Brute force: the best compensation is a least-squares
    fit of W_kq X_q by the other feature rows; its residual is the loss.  With H = 2 X X^T
    the score is exactly twice that loss, for every weight (so it ranks them the same)."""
    W, Xt = _rand_problem(91, c=3, b=7, n=30)
    X = Xt.T                                             # b x n, features as rows
    H = oracle.hessian(Xt)
    S = oracle.obs_scores(W, np.diag(np.linalg.inv(H)))
    for k in range(W.shape[0]):
        for q in range(W.shape[1]):
            rest = [t for t in range(W.shape[1]) if t != q]
            target = W[k, q] * X[q]
            coef, *_ = np.linalg.lstsq(X[rest].T, target, rcond=None)
            loss = float(np.sum((target - coef @ X[rest]) ** 2))
            assert S[k, q] == pytest.approx(2.0 * loss, rel=1e-8)


# ----------------------------------------------------------------------------- no-update baselines

def test_row_quota_mask_is_the_per_row_order_statistic():
    """Properties that fix the mask: exactly `count` per row; every removed score <= every
    kept score of its row; at the boundary value the removed ties sit left of the kept."""
    rng = np.random.default_rng(11)
    S = rng.integers(0, 6, size=(40, 37)).astype(np.float64)   # many exact ties
    for count in (0, 1, 9, 18, 36, 37):
        M = oracle.row_quota_mask(S, count)
        assert np.all(M.sum(axis=1) == count)
        for k in range(S.shape[0]):
            rem, kep = S[k, M[k]], S[k, ~M[k]]
            if rem.size and kep.size:
                assert rem.max() <= kep.min()
                v = rem.max()
                if v == kep.min():
                    assert np.flatnonzero(M[k] & (S[k] == v)).max() < np.flatnonzero(~M[k] & (S[k] == v)).min()


def test_no_update_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "no_update_hand_example.json")))
    W = np.array(g["W"])
    Xt = np.array(g["Xt"], dtype=np.float64)
    for method in ("wanda", "magnitude"):
        want = np.array(g[method + "_mask"])
        r = oracle.prune_no_update(W, Xt=Xt, sparsity=g["sparsity"], method=method)
        assert np.array_equal(r["mask"], want)
        r = oracle.prune_no_update(W, Xt=Xt, pattern="nm", nm=(2, 4), method=method)
        assert np.array_equal(r["mask"], want)
        # H = 2 X X^T gives the same norms
        r = oracle.prune_no_update(W, H=oracle.hessian(Xt), sparsity=g["sparsity"], method=method)
        assert np.array_equal(r["mask"], want)


def test_no_update_leaves_kept_weights_and_zeroes_removed():
    rng = np.random.default_rng(12)
    W = rng.normal(0, 0.02, size=(16, 64))
    Xt = rng.normal(size=(100, 64))
    r = oracle.prune_no_update(W, Xt=Xt, sparsity=0.6, method="wanda")
    assert np.all(r["W"][r["mask"]] == 0.0)
    assert np.array_equal(r["W"][~r["mask"]], W[~r["mask"]])
    assert r["pruned"] == r["target"] == 16 * int(np.floor(0.6 * 64))


def test_wanda_with_equal_feature_norms_is_magnitude():
    """With every ||X_q|| equal the Wanda score is |W| times a constant, so the masks of the
    two methods coincide (the special case in which activations carry no information)."""
    rng = np.random.default_rng(13)
    W = rng.normal(0, 0.02, size=(24, 96))
    Xt = rng.choice([-1.0, 1.0], size=(50, 96))
    for pattern, nm in (("unstructured", (0, 0)), ("nm", (2, 4)), ("nm", (4, 8))):
        a = oracle.prune_no_update(W, Xt=Xt, sparsity=0.5, pattern=pattern, nm=nm, method="wanda")
        b = oracle.prune_no_update(W, Xt=Xt, sparsity=0.5, pattern=pattern, nm=nm, method="magnitude")
        assert np.array_equal(a["mask"], b["mask"])


def test_wanda_scale_of_activations_does_not_change_the_mask():
    rng = np.random.default_rng(14)
    W = rng.normal(0, 0.02, size=(8, 40))
    Xt = rng.normal(size=(30, 40))
    a = oracle.prune_no_update(W, Xt=Xt, sparsity=0.3, method="wanda")
    b = oracle.prune_no_update(W, Xt=7.0 * Xt, sparsity=0.3, method="wanda")
    assert np.array_equal(a["mask"], b["mask"])


# ----------------------------------------------------------------------------- 2:4 storage

def test_pack24_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "pack24_hand_example.json")))
    v, m = oracle.pack_24(np.array(g["What"], dtype=np.float32), np.array(g["mask"]))
    assert v.tolist() == g["values"] and m.tolist() == g["meta"]


def test_bf16_rne_known_patterns():
    x = np.array([1.0, -2.0, 0.5, 3.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9, 65504.0, 0.0], dtype=np.float32)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0; 1 + 3*2^-9 rounds up
    assert oracle.bf16_bits_rne(x).tolist() == [0x3F80, 0xC000, 0x3F00, 0x4040, 0x3F80, 0x3F81, 0x4780, 0x0000]


def test_pack24_roundtrip_restores_the_rounded_layer():
    """Unpacking by the stated layout gives back W-hat rounded to bfloat16 with the
    removed weights zero, for a 2:4 mask from the oracle itself."""
    rng = np.random.default_rng(15)
    W = rng.normal(0, 0.02, size=(12, 72))
    r = oracle.prune_no_update(W, pattern="nm", nm=(2, 4), method="magnitude")
    What = r["W"].astype(np.float32)
    v, m = oracle.pack_24(What, r["mask"])
    c, b = What.shape
    back = np.zeros((c, b), dtype=np.float32)
    for k in range(c):
        for g in range(b // 4):
            field = (int(m[k, g // 8]) >> (4 * (g % 8))) & 0xF
            for slot, pos in enumerate((field & 3, field >> 2)):
                back[k, 4 * g + pos] = (np.uint32(v[k, 2 * g + slot]) << np.uint32(16)).view(np.float32)
    want = (oracle.bf16_bits_rne(What).astype(np.uint32) << 16).view(np.float32)
    want[r["mask"]] = 0.0
    assert np.array_equal(back, want)


def test_block0_expectation_matches_the_full_oracle():
    """The full-size check's first-block expectation (scores of the untouched W, the global
    candidate set or the N:M groups) equals block 0 of a complete oracle prune."""
    from tests import _fullsize
    import synth
    for pattern, nm in (("unstructured", (0, 0)), ("nm", (2, 4)), ("nm", (4, 8))):
        wl = synth.custom(48, 96, 160, dtype="bf16", outlier_frac=0.02, outlier_scale=20.0, block=32,
                          sparsity=0.5, seed=31)
        W, X = synth.make_W(wl), synth.make_X_tokens(wl)
        W64, X64 = synth.to_f64(W, "bf16"), synth.to_f64(X, "bf16")
        full = oracle.prune_layer(W64, Xt=X64, sparsity=float(np.float32(0.5)), pattern=pattern, nm=nm, block=32,
                                  damp=0.01, method="thanos")
        g = _fullsize.column_norms_sq(X, "bf16", chunk=50)
        m0, decided = _fullsize.block0_expected(W64, g, pattern=pattern, nm=nm, sparsity=0.5, block=32, tol=0.0)
        assert np.array_equal(m0, full["mask"][:, :32])
        assert decided.shape == m0.shape


def test_dead_features_go_first_and_undamped_singular_h_is_refused():
    """A feature that is zero on every token has G_qq = 0, so its weights score 0 and the
    global budget takes all of them first; the damping keeps H_d positive definite.  With
    damp 0 the same H is singular and the factor refuses it."""
    rng = np.random.default_rng(8)
    Xt = rng.normal(size=(64, 16))
    Xt[:, [3, 7]] = 0.0
    W = rng.normal(0, 0.02, size=(8, 16))
    r = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=16, damp=0.01)
    assert r["mask"][:, [3, 7]].all()
    assert r["pruned"] == 64
    with pytest.raises(np.linalg.LinAlgError):
        oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=16, damp=0.0)


# --------------------------------------------------------------------------- fixed-mask replay

def test_fixed_mask_replay_equals_sequential_least_squares():
    """Replaying a given mask over three blocks equals, block after block, the brute-force
    constrained least squares on [sqrt(2) X^T; sqrt(lambda) I] over that block's active
    region with the block's selected weights forced to 0 and earlier columns frozen."""
    W, Xt = _rand_problem(41, c=2, b=12, n=30)
    damp = 0.03
    B = 4
    H = oracle.hessian(Xt)
    _, lam = oracle.damp_hessian(H, damp)
    mask = np.zeros((2, 12), dtype=bool)
    mask[0, [1, 2, 5, 9, 10]] = True
    mask[1, [0, 7, 11]] = True
    r = oracle.prune_layer(W, H=H, block=B, damp=damp, fixed_mask=mask)
    for k in range(2):
        w = W[k].copy()
        for j in range(0, 12, B):
            Q = np.flatnonzero(mask[k, j:j + B]) + j
            if Q.size:
                w = _lstsq_row(w, Xt, lam, j, Q)
        assert np.allclose(r["W"][k], w, rtol=1e-9, atol=1e-11)
    assert np.array_equal(r["mask"], mask)


@pytest.mark.parametrize("pattern,nm", [("unstructured", (0, 0)), ("nm", (2, 4))])
def test_fixed_mask_replay_reproduces_full_runs_on_row_subsets(pattern, nm):
    """With the full run's own mask given, every row -- and any subset of rows, also under
    the global budget that couples them through the selection -- comes out as in the full
    run, in both the factored and the definitional mode."""
    rng = np.random.default_rng(17)
    Xt = rng.normal(size=(60, 24))
    Xt[:, 5] *= 9.0
    W = rng.normal(0, 0.02, size=(10, 24))
    for mode in ("factored", "definitional"):
        full = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, pattern=pattern, nm=nm, block=8, mode=mode)
        again = oracle.prune_layer(W, Xt=Xt, block=8, mode=mode, fixed_mask=full["mask"])
        assert np.allclose(again["W"], full["W"], rtol=1e-12, atol=1e-15)
        rows = np.array([1, 4, 8])
        sub = oracle.prune_layer(W, Xt=Xt, block=8, mode=mode, rows=rows, fixed_mask=full["mask"][rows])
        assert np.allclose(sub["W"], full["W"][rows], rtol=1e-12, atol=1e-15)
        assert np.isclose(sub["loss"], float(np.sum(oracle.row_losses(W[rows], full["W"][rows],
                                                                         0.5 * oracle.hessian(Xt)))))


def test_fixed_mask_replay_records_the_selection_of_the_replayed_state():
    """Replaying the full run's own mask, every block's recorded choice is the mask itself;
    with one block-0 decision flipped, block 0's recorded choice shows the flip (and only
    that), since the choice is made before the block's update."""
    rng = np.random.default_rng(23)
    Xt = rng.normal(size=(50, 20))
    W = rng.normal(0, 0.02, size=(9, 20))
    full = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=5)
    again = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=5, fixed_mask=full["mask"])
    for blk in again["blocks"]:
        j = blk["j"]
        assert np.array_equal(blk["chosen"], full["mask"][:, j:j + 5])
        assert blk["r"] == full["zstar"] - int(full["mask"][:, :j].sum())
    flipped = full["mask"].copy()
    k, q = np.argwhere(flipped[:, :5])[0]
    flipped[k, q] = False
    other = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=5, fixed_mask=flipped)
    diff = np.argwhere(other["blocks"][0]["chosen"] != flipped[:, :5])
    assert diff.tolist() == [[k, q]]


def test_fixed_mask_replay_records_the_nm_choice_of_the_replayed_state():
    """N:M: replaying the full run's own mask, every block's recorded choice is the mask
    itself with the run's own group gaps; with one group of block 0 changed, block 0's
    recorded choice is still the rule's (the choice precedes the block's update), so it
    differs from the replayed mask exactly in that group."""
    rng = np.random.default_rng(29)
    Xt = rng.normal(size=(40, 16))
    W = rng.normal(0, 0.02, size=(6, 16))
    full = oracle.prune_layer(W, Xt=Xt, pattern="nm", nm=(2, 4), block=8)
    again = oracle.prune_layer(W, Xt=Xt, pattern="nm", nm=(2, 4), block=8, fixed_mask=full["mask"])
    for blk in again["blocks"]:
        j = blk["j"]
        assert np.array_equal(blk["chosen"], full["mask"][:, j:j + 8])
        assert np.allclose(blk["nm_gap"], full["nm_gap"][:, j // 4: j // 4 + 2])
    changed = full["mask"].copy()
    k = 3
    changed[k, 0:4] = ~changed[k, 0:4]          # the other two of the group's four
    other = oracle.prune_layer(W, Xt=Xt, pattern="nm", nm=(2, 4), block=8, fixed_mask=changed)
    diff = np.argwhere(other["blocks"][0]["chosen"] != changed[:, :8])
    assert sorted(diff.tolist()) == [[k, q] for q in range(4)]


# --------------------------------------------------------------------------- outlier rows (alpha)

def test_alpha_keeps_floor_alpha_c_rows_dense_and_gives_the_stated_total_sparsity():
    """alpha = 0.1 keeps 10% of the rows dense; with 2:4 and 4:8 on the other rows the total
    sparsity is 45% instead of 50% ("Thanos versus SparseGPT on LLaMA-3 8B")."""
    rng = np.random.default_rng(61)
    c, b = 40, 16
    Xt = rng.normal(size=(48, b))
    W = rng.normal(0, 0.02, size=(c, b))
    for nm in ((2, 4), (4, 8)):
        r = oracle.prune_layer_alpha(W, Xt=Xt, alpha=0.1, pattern="nm", nm=nm, block=8)
        assert int(r["outliers"].sum()) == 4
        assert np.array_equal(r["W"][r["outliers"]], W[r["outliers"]])
        assert not r["mask"][r["outliers"]].any()
        assert r["mask"].sum() / r["mask"].size == pytest.approx(0.45)
    r = oracle.prune_layer_alpha(W, Xt=Xt, alpha=0.1, sparsity=0.5, block=8)
    assert int(r["mask"].sum()) == math.floor(0.5 * 36 * b) == r["zstar"]


def test_alpha_outlier_rows_are_the_largest_activation_weighted_rows():
    """The dense rows are those with the largest sum of (W_kq ||X_q||)^2, by brute force over
    the rows (ties between equal rows: the lower row first); alpha = 0 changes nothing."""
    rng = np.random.default_rng(62)
    c, b = 23, 10
    Xt = rng.normal(size=(30, b)) * rng.uniform(0.2, 3.0, size=b)
    W = rng.normal(size=(c, b))
    W[7] = W[3]                                  # an exact tie between two rows
    g = np.einsum("tq,tq->q", Xt, Xt)
    out = oracle.outlier_rows(W, g, 0.2)         # floor(4.6) = 4 rows
    score = [sum((W[k, q] * math.sqrt(g[q])) ** 2 for q in range(b)) for k in range(c)]
    ranked = sorted(range(c), key=lambda k: (-score[k], k))
    assert sorted(np.flatnonzero(out).tolist()) == sorted(ranked[:4])
    tied = oracle.outlier_rows(W[[3, 7]], g, 0.5)
    assert tied.tolist() == [True, False]
    plain = oracle.prune_layer(W, Xt=Xt, sparsity=0.5, block=5)
    zero = oracle.prune_layer_alpha(W, Xt=Xt, alpha=0.0, sparsity=0.5, block=5)
    assert np.array_equal(zero["W"], plain["W"]) and np.array_equal(zero["mask"], plain["mask"])
