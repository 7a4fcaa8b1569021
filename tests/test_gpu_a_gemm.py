"""The tensor-core mainloop on its own (self-check entry rlk_gemm_bf16_f32),
against a float64 matmul of the same bf16 inputs, for all four operand
majorness combinations and ragged shapes."""
import pytest
import torch

from invariant_lm_head_gemm_b200 import binding

pytestmark = pytest.mark.gpu

SHAPES = [(128, 256, 64), (8, 8, 8), (200, 264, 136), (136, 520, 4096), (1024, 1024, 1024),
          (256, 768, 8192)]


def _diagnose(C, ref):
    d = (C - ref).abs()
    i = int(d.argmax())
    return ("max|d|=%.3g at %s; C[:3,:3]=%s ref[:3,:3]=%s; rel err vs ref^T-shaped=%s" % (
        float(d.max()), divmod(i, C.shape[1]), C[:3, :3].tolist(), ref[:3, :3].tolist(),
        "n/a" if C.shape[0] != C.shape[1] else
        "%.3g" % float((C - ref.t()).norm() / ref.norm())))


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "M%dN%dK%d" % s)
@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
def test_gemm_matches_fp64(shape, a_mn, b_mn):
    M, N, K = shape
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K + 11 * a_mn + 13 * b_mn)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    A_st = A.t().contiguous() if a_mn else A
    B_st = B.t().contiguous() if b_mn else B
    C, ws = binding.rlk_gemm_bf16_f32(A_st.cuda(), B_st.cuda(), bool(a_mn), bool(b_mn))
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    ref = A.double() @ B.double().t()
    Cc = C.cpu().double()
    err = float((Cc - ref).norm() / ref.norm())
    assert err < 1e-5, _diagnose(Cc, ref)


def test_gemm_repeatable():
    g = torch.Generator().manual_seed(5)
    A = torch.randn(512, 2048, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(768, 2048, generator=g).to(torch.bfloat16).cuda()
    C0, _ = binding.rlk_gemm_bf16_f32(A, B)
    for _ in range(3):
        C1, _ = binding.rlk_gemm_bf16_f32(A, B)
        assert torch.equal(C0, C1)


@pytest.mark.parametrize("N,K", [(264, 136), (520, 4096), (8, 8), (5120, 640), (8448, 64)])
def test_short_row_counts_equal_rows_of_a_long_gemm(N, K):
    """GEMMs of at most 224 rows (row-major operands) run the short-batch kernel
    with the operands swapped and a plain store epilogue; every row must equal
    that row of a 300-row GEMM, which runs the pair tiles, bit for bit.  Up to
    128 rows and 8192 columns that is the half-height (M = 64) form; N = 8448
    and the counts above 128 take the 128-row forms."""
    g = torch.Generator().manual_seed(N + K)
    A = torch.randn(300, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    full, ws = binding.rlk_gemm_bf16_f32(A, B)
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    gen = torch.Generator().manual_seed(K)
    for T in (1, 16, 17, 32, 33, 64, 100, 224):
        rows = torch.randperm(300, generator=gen)[:T].cuda()
        sub, ws = binding.rlk_gemm_bf16_f32(A[rows].contiguous(), B)
        torch.cuda.synchronize()
        assert binding.rlk_read_device_error(ws) == 0
        assert torch.equal(sub.view(torch.int32), full[rows].view(torch.int32)), T
