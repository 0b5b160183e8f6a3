"""NVFP4 weights on the GPU against the oracle's format (oracle/nvfp4.py).

* Quantiser: codes, block scales, the tensor scale and the bf16
  dequantisation must equal the oracle's bit for bit.  The oracle keeps one
  code per byte; the GPU packs two, the even k in the low nibble.
* GEMM (tcgen05, fed by TMA): |y - y_ref| <= 2e-5 * sum_k |x_k w_k| per
  element, and a row's bits must not depend on M.
* Decode with NVFP4 copies attached must follow the oracle's forward on the
  dequantised weights: logits relative L2 <= 2e-2, and greedy tokens
  identical except at near ties.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from oracle import nvfp4 as F

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402
from gpu_util import check_bf16_tokens, gpu_generate, rel_l2  # noqa: E402

CAP = dict(max_batch=4, max_seq=160, k_max=4, gamma_max=4, max_chunk=128)


def bf16_cuda(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def pack(codes: np.ndarray) -> np.ndarray:
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("K", [256, 1024, 2560])
def test_quantiser_matches_oracle_bit_for_bit(K):
    rng = np.random.default_rng(K)
    w = rng.standard_normal((45, K)).astype(np.float32) * 0.03
    w[1] = 0.0                      # a zero row
    w[2, ::16] = 5.0                # the tensor maximum sits in row 2
    w[3] *= 1e-6                    # blocks whose scale underflows E4M3 or rounds to small values
    w[4] = -np.abs(w[4]) * 1e-4     # small negatives: signed zeros
    wb = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w))
    q, s, g, deq = dory.quantize_nvfp4(bf16_cuda(synth.f32_to_bf16_bits(wb)))
    torch.cuda.synchronize()
    codes, scodes, gref = F.quantize(wb)
    assert float(g[0]) == gref
    assert np.array_equal(s.cpu().numpy(), scodes)
    assert np.array_equal(q.cpu().numpy(), pack(codes))
    want = synth.f32_to_bf16_bits(F.dequantize(codes, scodes, gref).astype(np.float32))
    assert np.array_equal(deq.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("M,N,K", [(1, 384, 256), (5, 2560, 2560), (16, 1024, 1024), (21, 256, 512),
                                   (1, 2560, 10240)])
def test_gemm_matches_oracle(M, N, K):
    rng = np.random.default_rng(M + N + K)
    w = rng.standard_normal((N, K)).astype(np.float32)
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    wb = synth.f32_to_bf16_bits(w)
    xb = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) / np.sqrt(K))
    q, s, g, _ = dory.quantize_nvfp4(bf16_cuda(wb), dequantised=False)
    X = bf16_cuda(xb)
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    y = dory.gemm_nvfp4(X, q, s, g, err=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    codes, scodes, gref = F.quantize(synth.bf16_bits_to_f32(wb))
    x64 = synth.bf16_bits_to_f32(xb).astype(np.float64)
    ref = F.gemv(x64, codes, scodes, gref)
    bound = 2e-5 * (np.abs(x64) @ np.abs(F.dequantize(codes, scodes, gref)).T) + 1e-30
    got = y.cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
    for m in sorted({0, M - 1}):
        one = dory.gemm_nvfp4(X[m:m + 1].contiguous(), q, s, g)
        assert torch.equal(one[0], y[m])


@pytest.fixture(scope="module", params=["tiny_bf16", "small128"])
def nv_model(request):
    shape = synth.SHAPES[request.param]
    w = synth.make_weights(shape, 0)
    nv = dory.NvWeights(dory.DeviceWeights(shape, w))
    h = dory.Handle(dory.make_config(shape, **CAP), nv.dequantised, dory.PER_LOOP)
    h.attach_nvfp4(nv)
    return shape, O.Model(shape, F.quantized_weights(w)), h


@pytest.mark.parametrize("k", [1, 2, 4])
@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
def test_decode_with_nvfp4_matches_oracle(nv_model, k, mode):
    shape, model, h = nv_model
    prompt = synth.make_prompt(8, 40, shape.vocab)
    om, cm = (O.LAST_LOOP, dory.LAST_LOOP) if mode == "last_loop" else (O.PER_LOOP, dory.PER_LOOP)
    h.reset()
    toks, lg = gpu_generate(h, prompt, 9, k, cm)
    h.synchronize()
    _, ora = O.generate(model, prompt, 9, k, om, forced=toks[:-1])
    errs = [rel_l2(lg[i], ora[i]) for i in range(len(toks))]
    assert max(errs) <= 2e-2, errs
    check_bf16_tokens(toks, ora)


def test_speculative_decoding_with_nvfp4_is_token_identical(nv_model):
    shape, _, h = nv_model
    tok = torch.tensor(synth.make_prompt(9, 30, shape.vocab), dtype=torch.int32, device="cuda")
    h.reset()
    nxt = h.prefill([0], tok, [30], 4, dory.PER_LOOP)
    plain = [int(nxt[0])]
    for _ in range(7):
        nxt = h.decode_step([0], nxt, 4, dory.PER_LOOP)
        plain.append(int(nxt[0]))
    first = h.prefill([1], tok, [30], 4, dory.PER_LOOP)
    out, _, _ = h.spec_decode([1], first, 1, 4, 4, dory.PER_LOOP, 7)
    assert [int(first[0])] + out[0].cpu().tolist() == plain
