"""Diagnostics of the tcgen05 operand staging and of the bounded waits."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    from block_sparse_attention_09_b200 import msa
    return msa


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_umma_staging_matches_matmul(msa, mode, N, K):
    g = torch.Generator().manual_seed(1000 * mode + N + K)
    A = torch.randn(128, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    ref = A.float() @ B.float().T
    D = msa.diag_umma(mode, A.cuda(), B.cuda()).cpu()
    err = (D - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item() + 1e-3, (mode, N, K, err)


def test_bounded_wait_gives_up(msa):
    # a barrier nothing arrives on: the wait must end by itself with a timeout status
    rc = msa.diag_wait_timeout(20_000_000)
    assert rc == -6
    # and the context is still usable afterwards
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0
