"""GPU path vs the fp64 oracle, element by element, on the tiny and small
workloads and on edge shapes (ragged T, V not a multiple of the tile, a
one-entry vocabulary, several backward vocab chunks with a one-column tail),
plus the fail-closed behaviour for out-of-range targets and empty batches."""
import numpy as np
import pytest
import torch

import oracle
from invariant_lm_head_gemm_b200 import binding
from invariant_lm_head_gemm_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _parity(w, check_bwd=True):
    lp, en, ls = oracle.forward(w.hidden, w.W, w.targets, w.temperature)
    W_dev = gu.dev_bf16(w.W)
    out = gu.run(w.hidden, W_dev, w.targets, w.temperature,
                 w.dlogp if check_bwd else None, w.dentropy if check_bwd else None)
    assert out["err"] == 0
    report = dict(logp=gu.assert_close_vec(out["logp"].cpu(), lp, "logp"),
                  entropy=gu.assert_close_vec(out["entropy"].cpu(), en, "entropy"),
                  lse=gu.assert_close_vec(out["lse"].cpu(), ls, "lse"))
    if check_bwd:
        dH, dW = oracle.backward(w.hidden, w.W, w.targets, w.temperature, w.dlogp, w.dentropy)
        gdH = gu.bf16_to_f64(out["dH"])
        gdW = out["dW"].double().cpu().numpy()
        if np.linalg.norm(dH) == 0:
            assert np.max(np.abs(gdH)) <= 1e-6 and np.max(np.abs(gdW)) <= 1e-6
        else:
            report["dHidden"] = gu.rel_frob(gdH, dH)
            report["dW"] = gu.rel_frob(gdW, dW)
            assert report["dHidden"] <= gu.FROB_TOL, report
            assert report["dW"] <= gu.FROB_TOL, report
    return report


def test_tiny_parity():
    r = _parity(wl.tiny(0))
    print("tiny", r)


def test_small_parity():
    r = _parity(wl.small(1))
    print("small", r)


EDGE = [
    (1, 64, 1, 1.0),        # one-entry vocabulary: logp = 0, entropy = 0, zero gradients
    (1, 64, 300, 1.0),      # a single row
    (7, 64, 129, 0.7),      # V one past a 128 boundary
    (130, 128, 1000, 1.3),  # two M tiles, ragged V
    (3, 4096, 300, 1.0),    # long K
    (257, 192, 8193, 1.0),  # two backward chunks, the second one column wide
    (300, 256, 20000, 0.9), # three backward chunks, ragged tail
    (33, 8192, 700, 0.25),  # long K (128 blocks) on the short-batch forward, sharp softmax
    (300, 8192, 3000, 4.0), # long K on the pair kernels, 32 dHidden column blocks, flat softmax
]


@pytest.mark.parametrize("T,H,V,tau", EDGE, ids=lambda *a: None)
def test_edge_shapes(T, H, V, tau):
    w = gu.random_case(T, H, V, tau, seed=T * 31 + V)
    r = _parity(w)
    print((T, H, V, tau), r)


def test_out_of_range_targets_fail_closed():
    w = gu.random_case(16, 64, 500, 1.0, seed=77)
    bad = w.targets.copy()
    bad[3] = 500
    bad[5] = -1
    W_dev = gu.dev_bf16(w.W)
    out = gu.run(w.hidden, W_dev, bad, 1.0, w.dlogp, w.dentropy)
    assert out["err"] & binding.RLK_DEVERR_TARGET
    logp = out["logp"].cpu().numpy()
    assert np.isnan(logp[3]) and np.isnan(logp[5])
    good = [i for i in range(16) if i not in (3, 5)]
    lp, en, ls = oracle.forward(w.hidden[good], w.W, w.targets[good], 1.0)
    gu.assert_close_vec(logp[good], lp, "logp")
    gu.assert_close_vec(out["entropy"].cpu().numpy()[good], en, "entropy")
    assert np.isfinite(out["entropy"].cpu().numpy()).all()
    # rows with valid targets keep their exact gradient rows (row independence)
    dH, _ = oracle.backward(w.hidden[good], w.W, w.targets[good], 1.0, w.dlogp[good],
                            w.dentropy[good])
    assert gu.rel_frob(gu.bf16_to_f64(out["dH"])[good], dH) <= gu.FROB_TOL


def test_empty_batch():
    V, H = 300, 64
    W = gu.dev_bf16(wl.make_weight(3, V, H))
    hid = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    tg = torch.empty(0, dtype=torch.int64, device="cuda")
    ws = binding.make_workspace(0, H, V, True)
    logp, ent, lse = binding.rlk_linear_logp_fwd(hid, W, tg, 1.0, ws)
    assert logp.numel() == 0
    e = torch.empty(0, dtype=torch.float32, device="cuda")
    dW = torch.full((V, H), 7.0, device="cuda")
    dH = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    binding.rlk_linear_logp_bwd(hid, W, tg, 1.0, e, e, e, e, ws, out=(dH, dW))
    torch.cuda.synchronize()
    assert float(dW.abs().max()) == 0.0


def test_provenance_counts_calls():
    c0, c1 = binding.call_count(0), binding.call_count(1)
    w = gu.random_case(4, 64, 100, 1.0, seed=5)
    gu.run(w.hidden, gu.dev_bf16(w.W), w.targets, 1.0, w.dlogp, w.dentropy)
    assert binding.call_count(0) == c0 + 1 and binding.call_count(1) == c1 + 1
    assert binding.backend_id() == "rlk.linear_logp.bitwise.sm100a.v1"


def test_wrong_workspace_is_refused():
    w = gu.random_case(4, 64, 100, 1.0, seed=6)
    hid, W = gu.dev_bf16(w.hidden), gu.dev_bf16(w.W)
    tg = gu.dev(w.targets, torch.int64)
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.RlkError) as e:
        binding.rlk_linear_logp_fwd(hid, W, tg, 1.0, small)
    assert e.value.status == 4


def test_temperature_identity_is_bitwise():
    """(tau = 0.5, W) and (tau = 1, 2W) give the same logits exactly (scaling
    by two is exact in bf16 and fp32), so the outputs must match bit for bit."""
    w = gu.random_case(70, 256, 3000, 0.5, seed=9)
    W2 = wl.f64_to_bf16_bits(2.0 * wl.bf16_bits_to_f64(w.W))
    a = gu.run(w.hidden, gu.dev_bf16(w.W), w.targets, 0.5)
    b = gu.run(w.hidden, gu.dev_bf16(W2), w.targets, 1.0)
    for k in ("logp", "entropy", "lse"):
        assert torch.equal(a[k].view(torch.int32), b[k].view(torch.int32)), k
