"""The seeded input generators: the stated recipe (per-row streams), the decoder block's
seven layers and four shared inputs, and that feature subsets and threaded generation
give the same bytes as the serial token-major draw."""
import numpy as np

import synth


def test_weight_rows_follow_their_streams():
    wl = synth.custom(6, 40, 8, dtype="fp32", seed=3)
    W = synth.make_W(wl)
    for k in (0, 5):
        want = np.random.default_rng([3, 0, k]).normal(0.0, 0.02, 40).astype(np.float32)
        assert np.array_equal(W[k], want)
    blk = synth.decoder_block(n=16)
    _, wl_v = blk["v_proj"]                                     # layer 2 of the block
    want = np.random.default_rng([0, 102, 7]).normal(0.0, 0.02, wl_v.b)
    assert np.array_equal(synth.make_W(wl_v, rows=[7])[0], synth.f64_to_bf16_bits(want))


def test_decoder_block_layers_and_inputs():
    blk = synth.decoder_block()
    assert list(blk) == ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj"]
    shapes = {k: (wl.c, wl.b) for k, (_, wl) in blk.items()}
    assert shapes["q_proj"] == shapes["o_proj"] == (4096, 4096)
    assert shapes["gate_proj"] == shapes["up_proj"] == (11008, 4096)
    assert shapes["down_proj"] == (4096, 11008)
    assert {k: inp for k, (inp, _) in blk.items()} == {
        "q_proj": "attn_in", "k_proj": "attn_in", "v_proj": "attn_in", "o_proj": "o_in",
        "gate_proj": "mlp_in", "up_proj": "mlp_in", "down_proj": "down_in"}
    for _, wl in blk.values():
        assert wl.n == 128 * 2048 and wl.dtype == "bf16" and wl.pattern == "unstructured"
        assert wl.sparsity == 0.5 and wl.block == 128
    assert blk["down_proj"][1].x_dist == "laplace" and blk["down_proj"][1].outlier_frac == 0.0
    assert len({wl.w_id for _, wl in blk.values()}) == 7
    assert len({wl.input_id for _, wl in blk.values()}) == 4


def test_layers_sharing_an_input_draw_one_x_and_distinct_w():
    blk = synth.decoder_block(n=64)
    _, q = blk["q_proj"]
    _, k = blk["k_proj"]
    _, o = blk["o_proj"]
    Xq, Xk, Xo = (synth.make_X_features(wl, range(0, 32)) for wl in (q, k, o))
    assert np.array_equal(Xq, Xk) and not np.array_equal(Xq, Xo)
    assert not np.array_equal(synth.make_W(q, rows=[0]), synth.make_W(k, rows=[0]))


def test_threaded_and_subset_draws_match_the_serial_draw():
    wl = synth.custom(4, 300, 96, dtype="bf16", x_dist="laplace", input_id=2)
    X = synth.make_X_tokens(wl)
    assert np.array_equal(synth.make_X_tokens(wl, threads=4), X)
    cols = [0, 7, 64, 299]
    assert np.array_equal(synth.make_X_features(wl, cols), X[:, cols].T)


def test_bf16_storage_rounds_fp64_once_to_nearest_even():
    """Inputs are stored as bfloat16 rounded once from fp64 (no detour through fp32, whose
    own rounding could move a value that sits just off a halfway point onto it)."""
    rng = np.random.default_rng(7)
    x = rng.normal(size=3000) * 10.0 ** rng.integers(-20, 20, size=3000)
    # exact halfway points between neighbouring bfloat16 values (even and odd lower
    # neighbour), and points one fp64 step either side of them
    v = synth.bf16_bits_to_f64(np.arange(0x3F80, 0x3F80 + 64, dtype=np.uint16))
    mid = 0.5 * (v[:-1] + v[1:])
    x = np.concatenate([x, mid, -mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf)])
    u = synth.f64_to_bf16_bits(x)
    y = synth.bf16_bits_to_f64(u)
    up = synth.bf16_bits_to_f64(u + np.uint16(1))       # the neighbours of y in magnitude
    dn = synth.bf16_bits_to_f64(u - np.uint16(1))
    d = np.abs(y - x)
    assert np.all(d <= np.abs(up - x)) and np.all(d <= np.abs(dn - x))
    tie = (d == np.abs(up - x)) | (d == np.abs(dn - x))
    assert tie.sum() == 2 * len(mid)                     # only the exact halfway points tie
    assert np.all((u[tie] & 1) == 0)                     # and they go to the even pattern
    n = len(mid)
    above, below = x[-2 * n:-n], x[-n:]
    assert np.all(synth.bf16_bits_to_f64(synth.f64_to_bf16_bits(above)) == v[1:])
    assert np.all(synth.bf16_bits_to_f64(synth.f64_to_bf16_bits(below)) == v[:-1])
