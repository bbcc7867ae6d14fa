"""Host-side pieces of block-by-block tuning: the minibatch draws, the preset
modes, and the oracle's driver pinned to properties the pages fix."""
import numpy as np
import pytest

import synth
from oracle import autoround_oracle as O


def test_schedule_draws_distinct_samples_per_step_and_is_seeded():
    s = synth.make_schedule(128, 8, 50, seed=3)
    assert s.shape == (50, 8) and s.dtype == np.int32
    assert all(len(set(row)) == 8 for row in s)
    assert s.min() >= 0 and s.max() < 128
    assert np.array_equal(s, synth.make_schedule(128, 8, 50, seed=3))
    assert not np.array_equal(s, synth.make_schedule(128, 8, 50, seed=4))
    # uniform draws: over many steps every sample is used about equally often
    counts = np.bincount(synth.make_schedule(16, 4, 4000, seed=1).ravel(), minlength=16)
    assert counts.min() > 0.9 * 1000 and counts.max() < 1.1 * 1000
    with pytest.raises(ValueError):
        synth.make_schedule(4, 5, 1)


def test_presets_follow_the_table():
    """[AR] §8 preset table: batch, iterations, sequence length, calibration samples; lr 5e-3 in all."""
    import json, os
    from post_weight_quantization_autoround_b200 import driver

    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "preset_modes.json")))
    assert set(driver.PRESETS) == set(gold["modes"])
    for name, row in gold["modes"].items():
        assert driver.PRESETS[name] == row, name
    assert driver.LR == gold["lr"]


def _tiny_model(n_blocks=2, H=64, F=128, S=6, L=4, seed=0):
    blocks = []
    for b in range(n_blocks):
        d = synth.make_mlp(H, F, 1, seed=seed + b)
        blocks.append(tuple(synth.bf16_bits_to_f32(d[k]) for k in ("Wg", "Wu", "Wd")))
    X0 = synth.bf16_bits_to_f32(synth.make_activations(S * L, H, seed=seed + 10)).reshape(S, L, H)
    return blocks, X0


def test_oracle_driver_chains_blocks_through_quantized_outputs():
    """[AR] §3 "Algorithm Flow" step 7: block b+1 starts from block b's quantized output."""
    cfg = O.QConfig(bits=4, group_size=32)
    blocks, X0 = _tiny_model()
    sched = synth.make_schedule(6, 3, 4, seed=2)
    both = O.tune_blocks_mlp(blocks, X0, cfg, sched)
    second = O.tune_blocks_mlp(blocks[1:], both[0]["x_out"], cfg, sched)
    assert np.array_equal(both[1]["losses"], second[0]["losses"])
    assert np.array_equal(both[1]["x_out"], second[0]["x_out"])
    for (V1, a1, b1), (V2, a2, b2) in zip(both[1]["states"], second[0]["states"]):
        assert np.array_equal(V1, V2) and np.array_equal(a1, a2) and np.array_equal(b1, b2)


def test_oracle_driver_first_loss_is_the_rtn_loss_of_the_drawn_samples():
    """Step 3-4 at the start state (V = 0, alpha = beta = 1) on exactly the drawn samples."""
    cfg = O.QConfig(bits=4, group_size=32)
    blocks, X0 = _tiny_model(n_blocks=1)
    sched = synth.make_schedule(6, 2, 1, seed=5)
    res = O.tune_blocks_mlp(blocks, X0, cfg, sched)
    Ws = blocks[0]
    H = X0.shape[2]
    Y = O.mlp_reference(X0.reshape(-1, H), *Ws).reshape(X0.shape)
    idx = sched[0]
    st0 = [(np.zeros(W.shape, np.float32), np.ones((W.shape[0], W.shape[1] // 32), np.float32),
            np.ones((W.shape[0], W.shape[1] // 32), np.float32)) for W in Ws]
    ref = O.eval_loss_mlp(Ws, X0[idx].reshape(-1, H), Y[idx].reshape(-1, H), st0, cfg)
    assert res[0]["losses"][0] == pytest.approx(ref, rel=1e-12)


def test_oracle_driver_with_every_sample_each_step_is_the_full_batch_trajectory():
    cfg = O.QConfig(bits=4, group_size=32)
    blocks, X0 = _tiny_model(n_blocks=1)
    S, L, H = X0.shape
    steps = 3
    sched = np.tile(np.arange(S, dtype=np.int32), (steps, 1))
    res = O.tune_blocks_mlp(blocks, X0, cfg, sched)
    Ws = blocks[0]
    Xf = X0.reshape(-1, H)
    Y = O.mlp_reference(Xf, *Ws)
    st = [(np.zeros(W.shape, np.float32), np.ones((W.shape[0], W.shape[1] // 32), np.float32),
           np.ones((W.shape[0], W.shape[1] // 32), np.float32)) for W in Ws]
    for t in range(steps):
        loss, st, _, _, _ = O.tune_step_mlp(Ws, Xf, Y, st, cfg)
        assert res[0]["losses"][t] == loss
    for (V1, a1, b1), (V2, a2, b2) in zip(res[0]["states"], st):
        assert np.array_equal(V1, V2) and np.array_equal(a1, a2) and np.array_equal(b1, b2)


def test_int4_checkpoint_round_trip(tmp_path):
    import torch

    from post_weight_quantization_autoround_b200 import QConfig, driver

    rng = np.random.default_rng(0)
    results = []
    for b in range(2):
        layers = []
        for N, K in ((64, 32), (64, 32), (32, 64)):
            layers.append((torch.from_numpy(rng.integers(0, 2**31, (N, K // 8), dtype=np.int64).astype(np.int32)),
                           torch.from_numpy(rng.standard_normal((N, K // 32)).astype(np.float16)),
                           torch.from_numpy(rng.integers(0, 16, (N, K // 32)).astype(np.float16))))
        results.append({"int4": layers})
    cfg = QConfig(4, 32, 0, 0.005, 200, -0.5, 0.5, 0.5, 1.0)
    path = str(tmp_path / "ckpt.npz")
    driver.save_int4_checkpoint(path, results, cfg)
    meta, arrays = driver.load_int4_checkpoint(path)
    assert meta["bits"] == 4 and meta["group_size"] == 32 and meta["blocks"] == 2
    for b, r in enumerate(results):
        for name, (p, s, z) in zip(("gate", "up", "down"), r["int4"]):
            assert np.array_equal(arrays[f"b{b}.{name}.packed"], p.numpy().view(np.uint32))
            assert np.array_equal(arrays[f"b{b}.{name}.scale"], s.numpy())
            assert np.array_equal(arrays[f"b{b}.{name}.zero"], z.numpy())


def test_tuning_state_file_round_trips(tmp_path):
    """save_tuning_state / load_tuning_state keep every array bit for bit, the step count and the settings."""
    import os

    import torch

    import post_weight_quantization_autoround_b200 as ar
    from post_weight_quantization_autoround_b200 import driver

    if not os.path.exists(ar.library_path):
        pytest.skip("libautoround.so not built")
    cfg = ar.ar_qconfig_default(bits=2, group_size=32, lr=0.002)
    layers = [tuple(torch.from_numpy(x) for x in synth.make_state(n, k, 32, seed=n, spread=True))
              for n, k in ((64, 128), (128, 64))]
    path = str(tmp_path / "s.npz")
    driver.save_tuning_state(path, layers, 37, cfg, names=["gate", "down"])
    step, cfg2, back, names = driver.load_tuning_state(path, device="cpu")
    assert step == 37 and names == ["gate", "down"]
    for f in driver._CFG_FIELDS:
        assert getattr(cfg2, f) == getattr(cfg, f), f
    for (V, a, b), (V2, a2, b2) in zip(layers, back):
        for x, y in ((V, V2), (a, a2), (b, b2)):
            assert x.dtype == y.dtype and torch.equal(x, y)
