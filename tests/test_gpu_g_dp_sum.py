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
