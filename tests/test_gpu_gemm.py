"""The tcgen05 projection GEMM on its own (GPU): against a plain PyTorch fp32
product of the same bf16 operands, against the SIMT kernel, and for row
results that do not depend on how many rows share the launch."""
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402

SHAPES = [(1, 256, 256), (5, 384, 256), (16, 1024, 1024), (17, 2560, 2560), (64, 3584, 2560),
          (80, 2560, 10240), (128, 20480, 2560), (200, 1024, 512), (2560, 3584, 2560), (1, 131072, 2560)]


def operands(M, N, K, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    X = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
    return X, W


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_tcgen05_matches_fp32_reference(M, N, K):
    X, W = operands(M, N, K, M + N + K)
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y, S = dory.gemm_bf16(X, W, batch_hint=1, invariant=M <= 128, impl=2, err=err)
    ref = X.float() @ W.float().T
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    scale = ref.abs().max().item()
    assert (Y - ref).abs().max().item() <= 2e-5 * K ** 0.5 * max(scale, 1.0), (S, (Y - ref).abs().max().item())
    assert 1 <= S <= 8


@pytest.mark.parametrize("M,N,K", [(3, 384, 256), (33, 2560, 2560)])
def test_simt_matches_fp32_reference(M, N, K):
    X, W = operands(M, N, K, 7)
    Y, S = dory.gemm_bf16(X, W, impl=1)
    ref = X.float() @ W.float().T
    assert S == 1 and (Y - ref).abs().max().item() <= 2e-5 * K ** 0.5 * max(ref.abs().max().item(), 1.0)


@pytest.mark.parametrize("N,K", [(3584, 2560), (2560, 10240), (20480, 2560), (384, 256)])
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_rows_bit_identical_across_M(N, K, batch):
    """A decode row alone and the same row inside a speculative verify chunk
    (at any position) must give bit-identical products."""
    X, W = operands(96, N, K, 11)
    alone, s1 = dory.gemm_bf16(X[:1].contiguous(), W, batch_hint=batch, invariant=True, impl=2)
    for M, at in ((batch, batch - 1), (5 * batch, 5 * batch - 3), (80, 37), (96, 95)):
        Xm = X[:M].clone()
        Xm[at] = X[0]
        full, s2 = dory.gemm_bf16(Xm, W, batch_hint=batch, invariant=True, impl=2)
        assert s1 == s2
        assert torch.equal(full[at], alone[0]), (M, at)


@pytest.mark.parametrize("M,N,K", [(1, 2560, 10240), (3, 20480, 2560), (40, 3584, 2560)])
def test_stage_width_does_not_change_bits(M, N, K):
    """One 64-column sub-tile per stage (impl 3) and the default wide stages
    (impl 2) accumulate the same K-steps in the same order."""
    X, W = operands(M, N, K, 3)
    a, s1 = dory.gemm_bf16(X, W, batch_hint=1, invariant=True, impl=2)
    b, s2 = dory.gemm_bf16(X, W, batch_hint=1, invariant=True, impl=3)
    assert s1 == s2 and torch.equal(a, b)


@pytest.mark.parametrize("M,N,K", [(1, 2560, 10240), (3, 3584, 2560), (20, 20480, 2560), (300, 1024, 512)])
def test_packed_weights_same_bits(M, N, K):
    """Weights in the packed tile layout (bulk copies) give the same bits as
    row-major weights read through tensor maps."""
    X, W = operands(M, N, K, 4)
    Wp = dory.pack_weight_bf16(W)
    a, s1 = dory.gemm_bf16(X, W, batch_hint=1, invariant=M <= 128, impl=2)
    b, s2 = dory.gemm_bf16(X, Wp, batch_hint=1, invariant=M <= 128, impl=4)
    assert s1 == s2 and torch.equal(a, b)
