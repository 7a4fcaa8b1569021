"""The bitwise claims: results are identical run to run, independent of
batch size, of a row's position and of the other rows in the batch.

The pages hold the train/rollout logp comparison to zero bitwise mismatches
(h100-cp-gradient.json, runs[0].validation.train_rollout_logprob:
bitwise_equal, mismatch_count 0 over element_count 8192) and report
batch_invariant / strict_bitwise_repeatable gates (h3-runtime-integration-b200
report, transition[] and model_checks); the tests below compare at least
that many elements with zero mismatches."""
import json
import os

import numpy as np
import pytest
import torch

from invariant_lm_head_gemm_b200 import binding
from invariant_lm_head_gemm_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

with open(os.path.join(os.path.dirname(__file__), "golden", "pages_claims.json")) as _f:
    CLAIMS = json.load(_f)
EXPOSURE = CLAIMS["train_rollout_logprob"]["element_count"]       # 8192


@pytest.fixture(scope="module")
def W4():
    return gu.dev_bf16(wl.make_weight(4, wl.QWEN_V, wl.QWEN_H))


def _count_mismatch(a, b):
    return int((a.view(torch.int32) != b.view(torch.int32)).sum())


def _bits_equal(a, b):
    it = {torch.float32: torch.int32, torch.bfloat16: torch.int16}[a.dtype]
    return a.shape == b.shape and torch.equal(a.view(it), b.view(it))


def test_batch_size_sweep_is_bitwise(W4):
    probes = wl.sweep_probes(4)
    ref = None
    compared = 0
    for i, T in enumerate(wl.SWEEP_T):
        h, t, dl, de, pidx, pos = wl.sweep_batch(T, probes, 100 + i)
        out = gu.run(h, W4, t, 1.0, dl, de)
        assert out["err"] == 0
        posd = torch.from_numpy(pos).cuda()
        got = {k: out[k][posd] for k in ("logp", "entropy", "lse")}
        got["dH"] = out["dH"][posd]
        if ref is None:
            ref = {k: {} for k in got}
        for k, v in got.items():
            for j, p in enumerate(pidx.tolist()):
                if p in ref[k]:
                    a, b = ref[k][p], v[j]
                    if k == "dH":
                        mism = int((a.view(torch.int16) != b.view(torch.int16)).sum())
                    else:
                        mism = _count_mismatch(a.reshape(1), b.reshape(1))
                    assert mism == 0, "probe %d %s differs at T=%d" % (p, k, T)
                    compared += a.numel()
                else:
                    ref[k][p] = v[j].clone()
    print("sweep: elements compared bitwise", compared)
    assert compared > 0


def test_repeats_and_permutations_are_bitwise():
    w = wl.rl_step(3)
    W_dev = gu.dev_bf16(w.W)
    ws = binding.make_workspace(w.T, w.H, w.V, True)
    base = gu.run(w.hidden, W_dev, w.targets, 1.0, w.dlogp, w.dentropy, ws=ws)
    assert base["err"] == 0
    keep = {k: base[k].clone() for k in ("logp", "entropy", "lse", "dH", "dW")}
    del base
    compared = 0
    for rep in range(10):
        out = gu.run(w.hidden, W_dev, w.targets, 1.0, w.dlogp, w.dentropy, ws=ws)
        for k in ("logp", "entropy", "lse"):
            assert _count_mismatch(out[k], keep[k]) == 0, (rep, k)
            compared += out[k].numel()
        assert _bits_equal(out["dH"], keep["dH"]), rep
        assert _bits_equal(out["dW"], keep["dW"]), rep     # fixed order, no atomics
        del out
    assert compared >= EXPOSURE
    rng = np.random.default_rng(7)
    for k in range(3):
        perm = rng.permutation(w.T)
        out = gu.run(w.hidden[perm], W_dev, w.targets[perm], 1.0, w.dlogp[perm],
                     w.dentropy[perm], ws=ws)
        pd = torch.from_numpy(perm).cuda()
        for key in ("logp", "entropy", "lse", "dH"):
            assert _bits_equal(out[key], keep[key][pd]), (k, key)
        del out
    print("repeat: elements compared bitwise", compared)
