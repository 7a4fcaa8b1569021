"""Guard bands around every buffer the library writes (a stand-in for a memory
sanitizer): each output, each workspace and each exchange buffer is carved out
of a larger allocation whose 4 KB on both sides hold a byte pattern, and after
the calls every guard byte must be unchanged.  The kernels write past ragged
edges with TMA stores and vector stores (dX boxes at T and at chunk tails, dW
rows at V, the dHidden accumulator, split partials), so the shapes are ragged
on purpose: T on both sides of the switch between the two short-batch MMA
forms (32 / 33), at the short-batch kernel's N = 224 / 256 (T = 224 / 225)
and on both sides of the switch to the pair kernel's 256-row tiles (256 /
257), V on both sides of the 8192-row backward chunk, H at its
smallest and at the model's size.  The guarded results must also equal the
results of the same calls on plain allocations bit for bit, and the fp64
oracle within the parity tolerances (fail closed, zero mismatches: VIME
Qwen3-8B TP4/CP2 page, "Required gates")."""
import numpy as np
import pytest
import torch

import oracle
from invariant_lm_head_gemm_b200 import binding, tp
from invariant_lm_head_gemm_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """nbytes of device memory with GUARD bytes of PATTERN on each side; the
    interior is filled with `fill` (a byte value)."""

    def __init__(self, nbytes, fill=0x5A):
        self.n = int(nbytes)
        self.buf = torch.full((self.n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.buf[GUARD:GUARD + self.n] = fill

    def view(self, dtype, *shape):
        return self.buf[GUARD:GUARD + self.n].view(dtype).view(*shape)

    def intact(self):
        return bool((self.buf[:GUARD] == PATTERN).all()) and \
            bool((self.buf[GUARD + self.n:] == PATTERN).all())


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def _inputs(case):
    return (gu.dev_bf16(case.hidden), gu.dev_bf16(case.W), gu.dev(case.targets, torch.int64),
            gu.dev(case.dlogp, torch.float32), gu.dev(case.dentropy, torch.float32))


def _guarded_step(hid, W, tg, dl, de, tau):
    T, H = hid.shape
    V = W.shape[0]
    g_ws = Guarded(binding.workspace_bytes(T, H, V, True), fill=0)
    g_out = [Guarded(4 * T) for _ in range(3)]
    g_dH = Guarded(2 * T * H)
    g_dW = Guarded(4 * V * H)
    ws = g_ws.view(torch.uint8, g_ws.n)
    logp, ent, lse = (g.view(torch.float32, T) for g in g_out)
    binding.rlk_linear_logp_fwd(hid, W, tg, tau, ws, out=(logp, ent, lse))
    dH = g_dH.view(torch.bfloat16, T, H)
    dW = g_dW.view(torch.float32, V, H)
    binding.rlk_linear_logp_bwd(hid, W, tg, tau, lse, ent, dl, de, ws, out=(dH, dW))
    torch.cuda.synchronize()
    err = binding.rlk_read_device_error(ws)
    guards = [g_ws] + g_out + [g_dH, g_dW]
    return dict(logp=logp, entropy=ent, lse=lse, dH=dH, dW=dW), guards, err


def _plain_step(hid, W, tg, dl, de, tau):
    logp, ent, lse = binding.rlk_linear_logp_fwd(hid, W, tg, tau)
    dH, dW = binding.rlk_linear_logp_bwd(hid, W, tg, tau, lse, ent, dl, de)
    torch.cuda.synchronize()
    return dict(logp=logp, entropy=ent, lse=lse, dH=dH, dW=dW)


CASES = [(1, 64, 1), (32, 64, 1537), (33, 64, 8193), (127, 64, 1537), (129, 64, 8193),
         (224, 4096, 1537), (225, 64, 8193), (256, 64, 8193), (257, 4096, 8193),
         (1, 4096, 151936), (129, 64, 151936)]


@pytest.mark.parametrize("T,H,V", CASES)
def test_fwd_bwd_write_nothing_outside_their_buffers(T, H, V):
    tau = 0.9
    case = gu.random_case(T, H, V, tau, seed=7 * T + V + H)
    args = _inputs(case)
    got, guards, err = _guarded_step(*args, tau)
    assert err == 0
    assert all(g.intact() for g in guards)
    ref = _plain_step(*args, tau)
    for k in ref:
        assert torch.equal(_bits(got[k]), _bits(ref[k])), k
    # the oracle, in full (these sizes stay small for an fp64 CPU pass)
    z = oracle.logits(case.hidden, case.W, tau)
    lp, en, ls = oracle.softmax_stats(z, case.targets)
    for k, r in (("logp", lp), ("entropy", en), ("lse", ls)):
        gu.assert_close_vec(got[k].cpu().numpy(), r, k)
    dx = oracle.dlogits(z, case.targets, tau, case.dlogp, case.dentropy)
    assert gu.rel_frob(gu.bf16_to_f64(got["dH"]), oracle.dhidden(dx, case.W)) <= gu.FROB_TOL
    # dW in full where it is small, else on sampled vocab rows (the targets,
    # both ends and a random set)
    if V * H <= 50_000_000:
        vs = np.arange(V)
    else:
        rng = np.random.default_rng(T + V)
        vs = np.unique(np.concatenate([case.targets, rng.choice(V, 512, replace=False),
                                       [0, V - 1]]))
    gdW = got["dW"][torch.from_numpy(vs).cuda()].double().cpu().numpy()
    assert gu.rel_frob(gdW, oracle.dw(dx[:, vs], case.hidden)) <= gu.FROB_TOL


def test_full_size_step_writes_nothing_outside_its_buffers():
    """The bench's launch configuration: the RL actor step (T = 5980, H = 4096,
    V = 151936), guarded, equal bit for bit to the same step on plain
    allocations; sampled rows against the oracle."""
    w = wl.rl_step(3)
    W = gu.dev_bf16(w.W)
    args = (gu.dev_bf16(w.hidden), W, gu.dev(w.targets, torch.int64),
            gu.dev(w.dlogp, torch.float32), gu.dev(w.dentropy, torch.float32))
    got, guards, err = _guarded_step(*args, 1.0)
    assert err == 0
    assert all(g.intact() for g in guards)
    ref = _plain_step(*args, 1.0)
    for k in ref:
        assert torch.equal(_bits(got[k]), _bits(ref[k])), k
    del ref
    rows = np.array([0, 1, 255, 256, 2989, w.T - 2, w.T - 1])
    lp, en, ls = oracle.forward(w.hidden[rows], w.W, w.targets[rows], 1.0)
    for k, r in (("logp", lp), ("entropy", en), ("lse", ls)):
        gu.assert_close_vec(got[k].cpu().numpy()[rows], r, k)


def test_shard_calls_write_nothing_outside_their_buffers():
    """Vocab-parallel calls at TP = 3 with every exchange buffer guarded; the
    merged results equal the single-GPU calls bit for bit."""
    T, H, V, tau, world = 300, 256, 40000, 0.9, 3
    case = gu.random_case(T, H, V, tau, seed=77)
    hid, W, tg, dl, de = _inputs(case)
    ref = _plain_step(hid, W, tg, dl, de, tau)
    align = tp.shard_alignment(V)
    split = binding.fwd_split_width()
    Gs = -(-tp.per_shard(V, world, align) // split)
    guards = []
    g_parts = [Guarded(4 * world * T * Gs, fill=0) for _ in range(3)]
    g_yt = Guarded(4 * T, fill=0)
    guards += g_parts + [g_yt]
    parts = [g.view(torch.float32, world, T, Gs) for g in g_parts]
    ytgt = g_yt.view(torch.float32, T)
    chunk = binding.bwd_chunk_width(V)
    nchunks = -(-V // chunk)
    R = -(-T // world)
    cps = -(-tp.per_shard(V, world, align) // chunk)
    g_dW = Guarded(4 * V * H)
    guards.append(g_dW)
    dW = g_dW.view(torch.float32, V, H)
    sent = []
    for r in range(world):
        v0, v1 = tp.shard_rows(V, world, r, align)
        g_ws = Guarded(binding.workspace_bytes(T, H, V, True), fill=0)
        g_dp = Guarded(4 * world * cps * R * H, fill=0)
        guards += [g_ws, g_dp]
        ws = g_ws.view(torch.uint8, g_ws.n)
        dp = g_dp.view(torch.float32, world, cps, R, H)
        if v1 > v0:
            Ws = W[v0:v1].contiguous()
            binding.rlk_linear_logp_fwd_shard(hid, Ws, tg, V, v0, tau, [p[r] for p in parts],
                                              ytgt, workspace=ws)
            binding.rlk_linear_logp_bwd_shard(hid, Ws, tg, V, v0, tau, ref["lse"],
                                              ref["entropy"], dl, de, dp, R, dW_shard=dW[v0:v1],
                                              workspace=ws)
        sent.append(dp)
    nshards = -(-(-(-V // split)) // Gs)
    g_out = [Guarded(4 * T) for _ in range(3)]
    g_cws = Guarded(256, fill=0)
    guards += g_out + [g_cws]
    out = tuple(g.view(torch.float32, T) for g in g_out)
    binding.rlk_linear_logp_combine([p[:nshards].contiguous() for p in parts], nshards, Gs, ytgt,
                                    tg, V, out=out, workspace=g_cws.view(torch.uint8, 256))
    slices = []
    for q in range(world):
        recv = torch.stack([sent[r][q] for r in range(world)]).contiguous()
        g_s = Guarded(2 * R * H)
        guards.append(g_s)
        slices.append(binding.rlk_dhidden_combine(recv, nchunks, g_s.view(torch.bfloat16, R, H)))
    torch.cuda.synchronize()
    assert all(g.intact() for g in guards)
    for a, k in zip(out, ("logp", "entropy", "lse")):
        assert torch.equal(_bits(a), _bits(ref[k])), k
    assert torch.equal(_bits(torch.cat(slices)[:T]), _bits(ref["dH"]))
    assert torch.equal(_bits(dW), _bits(ref["dW"]))


@pytest.mark.parametrize("T,H,V", [(1, 64, 1537), (129, 4096, 8193), (300, 256, 20000)])
def test_noalloc_forward_writes_nothing_outside_its_outputs(T, H, V):
    case = gu.random_case(T, H, V, 1.0, seed=T + 3 * V)
    hid, W, tg, _, _ = _inputs(case)
    g_out = [Guarded(4 * T) for _ in range(3)]
    out = tuple(g.view(torch.float32, T) for g in g_out)
    binding.rlk_linear_logp_fwd_noalloc(hid, W, tg, 1.0, out=out)
    ref = binding.rlk_linear_logp_fwd(hid, W, tg, 1.0)
    torch.cuda.synchronize()
    assert all(g.intact() for g in g_out)
    for a, b in zip(out, ref):
        assert torch.equal(_bits(a), _bits(b))


def test_transition_step_writes_nothing_outside_its_buffers():
    B, n = 3, 257 * 96
    tw = wl.transition_case(0, B, n)
    x, v, eps, a, c, s = (torch.from_numpy(np.ascontiguousarray(q)).cuda()
                          for q in (tw.x, tw.v, tw.eps, tw.a, tw.c, tw.s))
    ws_ref = binding.transition_workspace(B, n)
    g_ws = Guarded(ws_ref.numel(), fill=0)
    g_mean, g_prev, g_lp = Guarded(4 * B * n), Guarded(4 * B * n), Guarded(4 * B)
    out = (g_mean.view(torch.float32, B, n), g_prev.view(torch.float32, B, n),
           g_lp.view(torch.float32, B))
    binding.rlk_transition_sample(x, v, eps, a, c, s, out=out,
                                  workspace=g_ws.view(torch.uint8, g_ws.n))
    ref = binding.rlk_transition_sample(x, v, eps, a, c, s, workspace=ws_ref)
    torch.cuda.synchronize()
    assert all(g.intact() for g in (g_ws, g_mean, g_prev, g_lp))
    for p, q in zip(out, ref):
        assert torch.equal(_bits(p), _bits(q))


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (33, 520, 136), (224, 264, 4096), (225, 264, 136),
                                   (70, 512, 384), (128, 8192, 64), (100, 8200, 72)])
def test_dense_gemm_writes_nothing_outside_its_output(M, N, K):
    """The dense GEMM's paths (the short-batch kernel's store mode up to 224
    rows, in its half-height form up to 128 rows and 8192 columns; the pair
    tiles above) with ragged M, N and K: C and the workspace
    guarded, C equal to the same call on plain allocations bit for bit and to
    an fp64 matmul within 1e-5."""
    g = torch.Generator().manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    g_c = Guarded(4 * M * N)
    g_ws = Guarded(int(binding.lib().rlk_gemm_workspace_bytes()), fill=0)
    C = g_c.view(torch.float32, M, N)
    binding.rlk_gemm_bf16_f32(A, B, out=C, workspace=g_ws.view(torch.uint8, g_ws.n))
    ref, ws = binding.rlk_gemm_bf16_f32(A, B)
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    assert g_c.intact() and g_ws.intact()
    assert torch.equal(_bits(C), _bits(ref))
    exact = A.double() @ B.double().t()
    assert float((C.double() - exact).norm() / exact.norm()) < 1e-5
