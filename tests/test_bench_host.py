"""Host side of bench.py: the roofline object's algorithmic work of each kernel class for a
small workload, against values worked out by hand from the stated definitions, and the
reference arm's contract line."""
import os

import numpy as np

import bench
import synth


def _wl():
    return synth.custom(8, 20, 12, dtype="fp32", block=8, sparsity=0.5)   # c=8, b=20, n=12, B=8


def test_stream_bytes():
    # blocks j = 0, 8, 16: 8c(b-j) = 64*20, 64*12, 64*4; K rows 4*B*(b-j) for t > 0: 32*12, 32*4
    want = 64 * (20 + 12 + 4) + 32 * (12 + 4)
    work, unit, bound = bench.algorithmic_work(bench.K_STREAM, _wl(), [1.0, 1.0, 1.0])
    assert (work, unit, bound) == (want, "byte", "hbm")


def test_select_and_hessian_and_factor():
    wl = _wl()
    assert bench.algorithmic_work(bench.K_SELECT, wl, [1.0] * 3) == (4 * 8 * (20 + 12 + 4), "byte", "hbm")
    assert bench.algorithmic_work(bench.K_HESSIAN, wl, [1.0]) == (20 * 20 * 12, "flop", "tensor")
    assert bench.algorithmic_work(bench.K_FACTOR, wl, [1.0]) == (2 * 20 ** 3 / 3, "flop", "alu")


def test_solve_flops_from_the_mask():
    """s = the selected count of a row in a block; per row and block s^3/3 + 2 s^2 (the
    Cholesky and the two triangular solves)."""
    wl = synth.custom(8, 24, 12, dtype="fp32", block=8, sparsity=0.5)    # three whole blocks
    mask = np.zeros((8, 24), dtype=np.uint8)
    mask[0, 0:3] = 1          # row 0, block 0: s = 3
    mask[1, 8:10] = 1         # row 1, block 1: s = 2
    want = (27 / 3 + 2 * 9) + (8 / 3 + 2 * 4)
    work, unit, bound = bench.algorithmic_work(bench.K_SOLVE, wl, [1.0] * 3, mask)
    assert np.isclose(work, want) and unit == "flop" and bound == "alu"


def test_no_update_bytes():
    wl = _wl()
    assert bench.algorithmic_work(bench.K_ROWPRUNE, wl, [1.0], method="wanda") == (8 * 20 * 7 + 4 * 20, "byte", "hbm")
    assert bench.algorithmic_work(bench.K_ROWPRUNE, wl, [1.0, 1.0], method="magnitude") == (2 * 8 * 20 * 7, "byte", "hbm")
    assert bench.algorithmic_work(bench.K_COLNORM, wl, [1.0]) == (2 * 12 * 20, "byte", "hbm")


def test_alu_peak_formula():
    assert np.isclose(bench.fp32_alu_peak_tflops(1965.0), 148 * 128 * 2 * 1965e6 / 1e12)


def test_reference_arm_prints_the_contract_line():
    """The reference arm (the fp64 oracle on the host cores) runs without a GPU: its one
    JSON line carries the keys of the benchmark contract."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                          "--cpu-rows", "64"], cwd=root, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "weights/s" and d["value"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 1, 3)
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"].startswith("q_proj4096x4096")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert abs(d["ms_per_step"] - 4096 * 64 / d["value"] * 1e3) < 1e-6 * d["ms_per_step"]
    assert "64 of 4096 rows" in cb["sample"]


def test_reference_arm_other_ranks_exit_quietly():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2"], cwd=root, env=env,
                         capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_block_phase_bytes_and_phase_fractions():
    """Block phase bytes: 8 c sum(b - j) + 4 B sum over blocks after the first of (b - j) +
    7 c b; each phase's fraction is its work over its time over its peak."""
    wl = _wl()                                   # c=8, b=20, B=8: j = 0, 8, 16
    want = 8 * 8 * (20 + 12 + 4) + 4 * 8 * (12 + 4) + 7 * 8 * 20
    assert bench.block_phase_bytes(wl) == want
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 2250.0, "sm_max_mhz": 1000.0}
    mask = np.zeros((8, 20), dtype=np.uint8)
    mask[:, :4] = 1                              # s = 4 in block 0 for every row
    ph = bench.phase_rooflines(wl, {"hessian_xxt": 1.0, "factor": 2.0, "stream_update_score": 1.0,
                                    "select": 0.5, "row_solve": 0.5}, mask, peaks)
    assert np.isclose(ph["hessian_xxt"]["achieved"], 20 * 20 * 12 / 1e-3 / 1e12)
    assert np.isclose(ph["hessian_xxt"]["frac"], ph["hessian_xxt"]["achieved"] / 2250.0)
    assert np.isclose(ph["row_solve"]["achieved"], 8 * (64 / 3 + 32) / 0.5e-3 / 1e12)
    assert np.isclose(ph["block_phase"]["ms"], 2.0)
    assert np.isclose(ph["block_phase"]["achieved"], want / 2e-3 / 1e9)
    # trailing update: block t's 2 c |J_t| (b - j_t) flops, applied by the next pass (the
    # last block's by the final pass): j = 0, 8 with |J| = 8, and j = 16 with |J| = 4
    assert np.isclose(ph["trailing_update_tensor"]["achieved"], 2 * 8 * (8 * 20 + 8 * 12 + 4 * 4) / 1e-3 / 1e12)
    assert np.isclose(ph["trailing_update_tensor"]["peak"], 2250.0 * 1.1 / 2.25)
