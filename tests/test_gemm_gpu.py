"""The batched bf16 tensor-core GEMM (the backward pass's building block) against a plain
PyTorch fp32 matmul of the same bf16 operands: every operand layout, ragged M, N, K, batches,
accumulation, scaling and bf16 output."""
import pytest
import torch

from hybrid_softmax_linear_chunked_b200 import binding as rb

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_softmax_linear_chunked_b200 import build
    build.build()
    rb.load()
    return torch.device("cuda", 0)


def operands(dev, batch, M, N, K, a_mn, b_mn, seed):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(batch, M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(batch, K, N, generator=g).to(torch.bfloat16)
    want = A.float() @ B.float()
    A_st = A.transpose(1, 2).contiguous() if a_mn else A.contiguous()       # [K][M] or [M][K]
    B_st = B.contiguous() if b_mn else B.transpose(1, 2).contiguous()       # [K][N] or [N][K]
    return A_st.to(dev), B_st.to(dev), want


@pytest.mark.parametrize("a_mn", [False, True])
@pytest.mark.parametrize("b_mn", [False, True])
@pytest.mark.parametrize("M,N,K,batch", [(128, 128, 64, 1), (200, 136, 72, 3), (384, 256, 520, 2),
                                          (8, 16, 8, 1)])
def test_gemm_layouts(dev, a_mn, b_mn, M, N, K, batch):
    A, B, want = operands(dev, batch, M, N, K, a_mn, b_mn, seed=M + N + K)
    got = rb.gemm(A, B, a_mn=a_mn, b_mn=b_mn)
    rb.sync_status(dev)
    err = (got.cpu() - want).abs().max() / want.abs().max()
    assert err <= 1e-5, f"max rel err {err:.2e}"


def test_gemm_accumulate_alpha_bf16(dev):
    A, B, want = operands(dev, 2, 256, 192, 136, False, True, seed=7)
    C0 = torch.randn(2, 256, 192, generator=torch.Generator().manual_seed(8)).to(dev)
    got = rb.gemm(A, B, b_mn=True, out=C0.clone(), accumulate=True, alpha=0.5)
    rb.sync_status(dev)
    ref = C0.cpu() + 0.5 * want
    assert ((got.cpu() - ref).abs().max() / ref.abs().max()) <= 1e-5
    got16 = rb.gemm(A, B, b_mn=True, out_dtype=torch.bfloat16)
    rb.sync_status(dev)
    ref16 = want.to(torch.bfloat16).float()
    # one bf16 rounding of an fp32 sum whose last bits may differ from torch's: at most one bf16
    # ulp apart (2^-7 relative at most)
    assert ((got16.float().cpu() - ref16).abs() <= ref16.abs() * 2 ** -7 + 1e-6).all()
