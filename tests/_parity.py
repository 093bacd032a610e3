"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and the
fp64 oracle on the same seeded inputs, and compare them element by element."""
import numpy as np

import oracle
import synth

# Ŵ relative Frobenius, loss relative, mask agreement (the stated acceptance bars)
W_REL_TOL = 1e-3
LOSS_REL_TOL = 1e-2
MASK_AGREE = 0.9999


def torch_inputs(W_store, X_store, dtype, device="cuda"):
    import torch
    import post_weight_pruning_b200 as pwp
    if dtype == "bf16":
        return pwp.from_bf16_bits(W_store, device), pwp.from_bf16_bits(X_store, device)
    return torch.from_numpy(W_store).to(device), torch.from_numpy(X_store).to(device)


def run_gpu(W_store, X_store, dtype, *, method, pattern, nm, block, sparsity, damp):
    import torch
    import post_weight_pruning_b200 as pwp
    Wt, Xt = torch_inputs(W_store, X_store, dtype)
    W_hat, mask, st = pwp.prune_layer(Wt, X=Xt, method=method, pattern=pattern, nm=nm, block=block,
                                      sparsity=sparsity, damp=damp)
    torch.cuda.synchronize()
    return W_hat.cpu().numpy().astype(np.float64), mask.cpu().numpy().astype(bool), st


def run_oracle(W_store, X_store, dtype, *, method, pattern, nm, block, sparsity, damp):
    W64 = synth.to_f64(W_store, dtype)
    X64 = synth.to_f64(X_store, dtype)
    # the library receives sparsity as fp32; give the oracle the same number
    s32 = float(np.float32(sparsity))
    return oracle.prune_layer(W64, Xt=X64, sparsity=s32, pattern=pattern, nm=nm, block=block,
                              damp=damp, method=method)


def compare(W_store, dtype, gpu, orc, *, pattern, nm, block, tie_tol):
    """Element-wise comparison.  Returns a dict of figures; mask disagreements are
    classified as ties when the oracle's own decision score sits within tie_tol
    (relative) of its selection boundary."""
    W_hat, mask, st = gpu
    Wo, Mo = orc["W"], orc["mask"]
    c, b = Wo.shape
    dis = np.argwhere(mask != Mo)
    tie_ok = np.zeros(len(dis), dtype=bool)
    gaps = np.zeros(len(dis))
    if pattern == "unstructured":
        thr = {}
        for blk in orc["blocks"]:
            thr[blk["j"]] = blk.get("t_last", 0.0)
        for i, (k, q) in enumerate(dis):
            j = (q // block) * block
            t = thr[j]
            gaps[i] = abs(orc["dscore"][k, q] - t) / max(abs(t), 1e-300)
            tie_ok[i] = gaps[i] <= tie_tol
    else:
        m = nm[1]
        for i, (k, q) in enumerate(dis):
            gaps[i] = orc["nm_gap"][k, q // m]
            tie_ok[i] = gaps[i] <= tie_tol
    res = {
        "agree": 1.0 - len(dis) / (c * b),
        "n_dis": int(len(dis)),
        "n_dis_not_tie": int((~tie_ok).sum()),
        "dis_gaps": sorted(gaps.tolist())[-8:],       # the largest relative score gaps that flipped
        # rows whose first (lowest-column) disagreement is not a tie: a later one in a row
        # follows from that row's earlier flip
        "rows_first_not_tie": int(sum(1 for k in np.unique(dis[:, 0]) if
                                      not tie_ok[np.flatnonzero(dis[:, 0] == k)[np.argmin(dis[dis[:, 0] == k, 1])]]))
        if len(dis) else 0,
        "w_rel": float(np.linalg.norm(W_hat - Wo) / np.linalg.norm(Wo)),
        "zeros_exact": bool(np.all(W_hat[mask] == 0.0)),
        "n_mask": int(mask.sum()),
        "n_mask_oracle": int(Mo.sum()),
        "stats_pruned": int(st.pruned),
        "status": int(st.status),
    }
    return res


def loss_of(W_store, dtype, W_hat, G):
    W0 = synth.to_f64(W_store, dtype)
    return oracle.recon_loss(W0, W_hat, G)
