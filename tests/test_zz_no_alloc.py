"""dory_gemm_bf16_noalloc: the projection GEMM for callers that cannot
allocate device memory (code recording a CUDA graph, servers whose device
memory is an arena owned elsewhere, allocation-free real-time paths).  It keeps
its split-K partial sums in a fixed array inside the library, so the caller
passes only X, W and the output Y.

Its result must equal, bit for bit, the allocating entry point's
(dory_gemm_bf16, whose partial slices the binding adds in the same order) on
two calls in a row with different inputs: the second call finds the array
holding the first call's partial sums, which are wrong values for it, so a
partial value it failed to write would show.  The status entry point must
report no timeout afterwards.  This file is collected last so a stopping run
has already run every other test; it also passes alone in a fresh process."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402


def noalloc(X, W, Y, batch_hint=1):
    M, K = X.shape
    N = W.shape[0]
    return dory.lib.dory_gemm_bf16_noalloc(M, N, K, ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                                           ctypes.c_void_p(Y.data_ptr()), batch_hint,
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def status():
    return dory.lib.dory_gemm_bf16_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K", [(1, 3584, 2560), (5, 2560, 10240), (16, 16384, 2560)])
def test_noalloc_matches_allocating_entry_point(M, N, K):
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    W = (torch.randn((N, K), generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
    for call in range(2):  # the second call starts from the first call's leftovers
        X = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
        ref, splits = dory.gemm_bf16(X, W, batch_hint=1, invariant=True, impl=2)
        Y = torch.full((M, N), float("nan"), device="cuda")
        assert noalloc(X, W, Y) == 0, dory.lib.dory_last_error(None)
        torch.cuda.synchronize()
        assert torch.equal(Y, ref), (call, splits, (Y - ref).abs().max().item())
    assert status() == 0, dory.lib.dory_last_error(None)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    X = torch.zeros((64, 2560), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((131072, 2560), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((64, 131072), device="cuda")
    assert noalloc(X, W, Y) == 2  # DORY_ERR_CAPACITY, before any work is queued
    assert b"2097152" in dory.lib.dory_last_error(None)
    assert status() == 0
