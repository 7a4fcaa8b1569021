"""Seeded input generator (bf16 rounding, shapes, determinism) and the oracle
regression fixture."""
import json
import os

import numpy as np
import torch

import oracle
from invariant_lm_head_gemm_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_rounding_matches_torch_on_f32_inputs():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * s for s in (1e-3, 0.02, 1.0, 300.0)])
    x = x.astype(np.float32).astype(np.float64)        # float32-exact, so no double rounding
    ours = wl.f64_to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours, ref.view(np.uint16))


def test_bf16_rounding_ties_to_even_and_subnormals():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0
    assert wl.f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even) -> 1+2^-6
    assert wl.f64_to_bf16_bits(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82
    # just above the tie rounds up (a float32 detour would lose this)
    assert wl.f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81
    # bf16 subnormal grid is 2^-133
    v = np.array([3 * 2.0 ** -133, -5 * 2.0 ** -133])
    assert np.array_equal(wl.bf16_bits_to_f64(wl.f64_to_bf16_bits(v)), v)


def test_generator_is_deterministic_and_shaped():
    a, b = wl.tiny(0), wl.tiny(0)
    assert np.array_equal(a.hidden, b.hidden) and np.array_equal(a.W, b.W)
    assert a.hidden.shape == (64, 256) and a.W.shape == (1024, 256)
    assert a.targets.min() >= 0 and a.targets.max() < 1024
    lens = wl.rl_seq_lens(3)
    assert len(lens) == 8 and lens.min() >= 256 and lens.max() <= 1024
    # W of one seed does not depend on how many rows are drawn
    w1 = wl.make_weight(7, 5000, 64)
    w2 = wl.make_weight(7, 4100, 64)
    assert np.array_equal(w1[:4100], w2)
    # RMS-normalised rows have unit RMS before rounding
    h = wl.rms_normalise(np.random.default_rng(1).standard_normal((4, 4096)))
    assert np.allclose(np.sqrt((h * h).mean(axis=1)), 1.0, atol=1e-6)


def test_sweep_batches_embed_probes():
    probes = wl.sweep_probes(4, H=64, V=1000)
    for T in (1, 7, 64, 513):
        h, t, dl, de, pidx, pos = wl.sweep_batch(T, probes, 100 + T, H=64, V=1000)
        assert h.shape == (T, 64)
        assert np.array_equal(h[pos], probes[0][pidx])
        assert np.array_equal(t[pos], probes[1][pidx])
        assert len(set(pos.tolist())) == len(pos)


def test_oracle_matches_regression_fixture():
    with open(os.path.join(GOLDEN, "oracle_tiny_rows.json")) as f:
        g = json.load(f)
    w = wl.tiny(0)
    n = g["rows"]
    assert w.targets[:n].tolist() == g["targets"]
    lp, en, ls = oracle.forward(w.hidden, w.W, w.targets, w.temperature)
    for name, got in (("logp", lp), ("entropy", en), ("lse", ls)):
        want = np.array([float(x) for x in g[name]])
        assert np.max(np.abs(got[:n] - want)) <= 1e-13 * np.max(np.abs(want))
    dH, dW = oracle.backward(w.hidden, w.W, w.targets, w.temperature, w.dlogp, w.dentropy)
    assert abs(np.linalg.norm(dH) - float(g["dHidden_fro"])) <= 1e-12 * float(g["dHidden_fro"])
    assert abs(np.linalg.norm(dW) - float(g["dW_fro"])) <= 1e-12 * float(g["dW_fro"])
