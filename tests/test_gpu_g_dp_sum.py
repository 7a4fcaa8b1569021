"""The fixed-order sum behind the data-parallel dW exchange, on one GPU:
bitwise equal to adding the parts one after another in list order."""
import pytest
import torch

from invariant_lm_head_gemm_b200 import binding

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [1, 2, 3, 8])
@pytest.mark.parametrize("count,offset", [(4096 * 37, 0), (1001, 0), (4096, 1)])
def test_sum_ordered_is_sequential(n, count, offset):
    g = torch.Generator(device="cuda").manual_seed(n * 7 + count)
    base = [torch.randn(count + offset, device="cuda", generator=g) * (10.0 ** k)
            for k in range(n)]
    parts = [b[offset:] for b in base]          # offset 1: 4-byte aligned only -> scalar path
    out = torch.empty(count, device="cuda")
    binding.rlk_sum_ordered(parts, out)
    ref = parts[0].clone()
    for p in parts[1:]:
        ref = ref + p
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))


def test_sum_ordered_depends_on_order():
    # fp32 addition is not associative: the library keeps the given order
    a = torch.tensor([1e8, 1.0, -1e8, 0.5], device="cuda")
    parts = [a[0:1].repeat(4).contiguous(), torch.full((4,), 1.0, device="cuda"),
             torch.full((4,), -1e8, device="cuda")]
    out = binding.rlk_sum_ordered(parts)
    rev = binding.rlk_sum_ordered(parts[::-1])
    torch.cuda.synchronize()
    assert float(out[0]) == float((parts[0][0] + parts[1][0]) + parts[2][0])
    assert float(rev[0]) == float((parts[2][0] + parts[1][0]) + parts[0][0])


def test_signalling_backward_and_overlapped_exchange_on_one_rank():
    """The backward that publishes each vocab chunk's completion gives the
    plain backward's bits and sets every chunk word to the call's sequence
    number; the exchange that waits on those words on a second stream (a
    one-rank NCCL group: the only size one GPU holds) returns dW itself, bit
    for bit, in its group pieces; T = 0 publishes every word as well."""
    import os
    import socket

    import torch.distributed as dist

    from invariant_lm_head_gemm_b200 import dp
    from tests import gpu_util as gu

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        tau = 0.9
        T, H, V = 300, 256, 40000
        case = gu.random_case(T, H, V, tau, seed=515)
        hid, W = gu.dev_bf16(case.hidden), gu.dev_bf16(case.W)
        tg = gu.dev(case.targets, torch.int64)
        dl, de = gu.dev(case.dlogp, torch.float32), gu.dev(case.dentropy, torch.float32)
        ws = binding.make_workspace(T, H, V, True)
        lp, en, ls = binding.rlk_linear_logp_fwd(hid, W, tg, tau, ws)
        dH_ref, dW_ref = (t.clone() for t in binding.rlk_linear_logp_bwd(hid, W, tg, tau, ls, en,
                                                                         dl, de, ws))
        chunk = binding.bwd_chunk_width(V)
        nchunks = -(-V // chunk)
        words = torch.zeros(nchunks, dtype=torch.int32, device="cuda")
        comm = torch.cuda.Stream()
        out = (torch.empty_like(dH_ref), torch.empty_like(dW_ref))
        for seq in (1, 2):
            binding.rlk_linear_logp_bwd_signal(hid, W, tg, tau, ls, en, dl, de, ws, out, words,
                                               seq)
            got, pieces = dp.reduce_scatter_dw_overlapped(out[1], chunk, chunk_done=words,
                                                          seq=seq, group_chunks=2, stream=comm)
            torch.cuda.current_stream().wait_stream(comm)
            torch.cuda.synchronize()
            assert binding.rlk_read_device_error(ws) == 0
            assert torch.equal(out[0].view(torch.int16), dH_ref.view(torch.int16))
            assert torch.equal(out[1].view(torch.int32), dW_ref.view(torch.int32))
            assert (words == seq).all()
            rows = torch.cat([dW_ref[a:b] for a, b in pieces])
            assert torch.equal(got[: rows.shape[0]].view(torch.int32), rows.view(torch.int32))
        # T = 0: dW zeroed, every word published in stream order
        binding.rlk_linear_logp_bwd_signal(hid[:0], W, tg[:0], tau, ls[:0], en[:0], dl[:0],
                                           de[:0], ws, (out[0][:0], out[1]), words, 3)
        torch.cuda.synchronize()
        assert (words == 3).all() and not out[1].any()
    finally:
        dist.destroy_process_group()
