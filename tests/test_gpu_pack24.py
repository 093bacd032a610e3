"""GPU parity of the compressed 2:4 storage against the oracle: bit-exact values and
metadata on the same host-built inputs, and a reported (not faulting) error for a
group that does not keep exactly two entries."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _random_24(c, b, seed):
    rng = np.random.default_rng(seed)
    W = rng.normal(0, 0.05, size=(c, b)).astype(np.float32)
    mask = np.ones((c, b), dtype=bool)
    for k in range(c):
        for g in range(b // 4):
            keep = rng.choice(4, size=2, replace=False)
            mask[k, 4 * g + keep] = False
    W[mask] = 0.0
    return W, mask


def _gpu_pack(W, mask):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    Wd = torch.from_numpy(W).cuda()
    Md = torch.from_numpy(mask.astype(np.uint8)).cuda()
    v, m, st = pwp.pack_24(Wd, Md, check=False)
    torch.cuda.synchronize()
    return v.cpu().numpy().view(np.uint16), m.cpu().numpy().view(np.uint32), pwp.read_stats(st)


@pytest.mark.parametrize("c,b", [(1, 4), (3, 32), (17, 100), (64, 4096)])   # partial last word at b = 100
def test_pack24_matches_oracle(c, b):
    W, mask = _random_24(c, b, seed=c * 1000 + b)
    v, m, st = _gpu_pack(W, mask)
    vo, mo = oracle.pack_24(W, mask)
    assert st.status == 0
    assert np.array_equal(v, vo) and np.array_equal(m, mo)


def test_pack24_of_an_oracle_2of4_layer():
    rng = np.random.default_rng(21)
    W = rng.normal(0, 0.02, size=(40, 256))
    r = oracle.prune_no_update(W, pattern="nm", nm=(2, 4), method="magnitude")
    What = r["W"].astype(np.float32)
    v, m, st = _gpu_pack(What, r["mask"])
    vo, mo = oracle.pack_24(What, r["mask"])
    assert st.status == 0
    assert np.array_equal(v, vo) and np.array_equal(m, mo)


def test_pack24_reports_a_group_that_is_not_2of4():
    W, mask = _random_24(4, 64, seed=3)
    mask[2, 8:12] = [True, False, False, False]     # three kept in one group
    v, m, st = _gpu_pack(W, mask)
    assert st.status == 1                            # PWP_EINVAL, recorded by the kernel
