"""MXFP8 weights on the GPU against the oracle's format (GPU).

* Quantiser: integer work on exact power-of-two scalings.  Codes, scale bytes
  and the bf16 dequantisation must equal the oracle's bit for bit, edge
  blocks included.
* GEMV, both implementations (CUDA cores; tensor cores with f16 operands and
  fp32 accumulators): |y - y_ref| <= 2e-5 * sum_k |x_k w_k| per element,
  where y_ref is the oracle's float64 product.  A row's bits must not depend
  on how many rows share the call.
* Decode with MXFP8 copies attached must follow the oracle's forward on the
  dequantised weights, within the bf16 path's tolerances: logits relative L2
  <= 2e-2, and greedy tokens identical except at near ties.
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth
from oracle import mxfp8 as MX

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402
from gpu_util import MODES, check_bf16_tokens, gpu_generate, rel_l2  # noqa: E402

CAP = dict(max_batch=4, max_seq=160, k_max=4, gamma_max=4, max_chunk=128)


def bf16_cuda(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def edge_rows(K: int, rng) -> np.ndarray:
    """Weight rows (float32, exactly bf16) with the quantiser's edge cases."""
    rows = []
    g = rng.standard_normal((6, K)).astype(np.float32)
    rows += list(g / np.linalg.norm(g, axis=1, keepdims=True))
    r = np.zeros(K, np.float32)
    rows.append(r)  # zero blocks: scale byte 0
    r = rng.standard_normal(K).astype(np.float32) * 1e-5
    r[::32] = 1.0
    rows.append(r)  # one large value per block, the rest in E4M3's subnormal range or below it
    r = -np.abs(rng.standard_normal(K).astype(np.float32)) * 1e-7
    r[5::32] = 0.5
    rows.append(r)  # negatives that round to zero: code 0x80
    r = rng.uniform(-1, 1, K).astype(np.float32)
    r[::32] = 1.9
    r[1::32] = -1.9
    rows.append(r)  # block maxima clamped to 448
    r = rng.standard_normal(K).astype(np.float32) * np.float32(2.0 ** -131)
    rows.append(r)  # bf16 subnormals: the scale clamps at 2^-127
    r = rng.standard_normal(K).astype(np.float32) * np.float32(2.0 ** 70)
    rows.append(r)  # large weights (scale byte 197 or so)
    pos = np.sort(MX.e4m3_table()[:0x7F])
    mids = ((pos[1:] + pos[:-1]) / 2)[-(K // 2):].astype(np.float32)
    r = np.zeros(K, np.float32)
    r[: len(mids)] = mids[: K]
    r[::32] = 256.0  # scale 1: the midpoints are exact ties
    rows.append(r)
    a = np.stack(rows)
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(a))


@pytest.mark.parametrize("K", [256, 1056, 2560])
def test_quantiser_matches_oracle_bit_for_bit(K):
    rng = np.random.default_rng(K)
    w = np.concatenate([edge_rows(K, rng), synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        rng.standard_normal((37, K)).astype(np.float32) * 0.03))])
    q, s, deq = dory.quantize_mxfp8(bf16_cuda(synth.f32_to_bf16_bits(w)))
    torch.cuda.synchronize()
    codes, scales = MX.quantize(w)
    got_q, got_s = q.cpu().numpy(), s.cpu().numpy()
    bad = np.argwhere(got_q != codes)
    assert bad.size == 0, [(int(i), int(j), w[i, j], got_q[i, j], codes[i, j]) for i, j in bad[:8]]
    assert np.array_equal(got_s, scales)
    want = synth.f32_to_bf16_bits(MX.dequantize(codes, scales).astype(np.float32))
    assert np.array_equal(deq.view(torch.int16).cpu().numpy().view(np.uint16), want)


def test_quantiser_flags_non_finite_weights():
    w = np.ones((4, 64), np.float32)
    w[2, 7] = np.inf
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    dory.quantize_mxfp8(bf16_cuda(synth.f32_to_bf16_bits(w)), err=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 4  # DEV_ERR_RANGE


GEMV_CASES = [(1, 37, 256), (2, 1000, 1056), (3, 384, 2560), (5, 2560, 2560), (1, 2560, 10240),
              (13, 300, 10240), (8, 4096, 2560)]


@pytest.mark.parametrize("impl", [1, 2, 4])
@pytest.mark.parametrize("M,N,K", GEMV_CASES)
def test_gemv_matches_oracle(M, N, K, impl):
    rng = np.random.default_rng(M * 7 + N + K)
    w = rng.standard_normal((N, K)).astype(np.float32)
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    w[0, 1:32] *= 1e-4  # subnormal codes in row 0
    wb = synth.f32_to_bf16_bits(w)
    xb = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) / np.sqrt(K))
    q, s, _ = dory.quantize_mxfp8(bf16_cuda(wb), dequantised=False)
    X = bf16_cuda(xb)
    y = dory.gemv_mxfp8(X, q, s, impl=impl)
    torch.cuda.synchronize()
    codes, scales = MX.quantize(synth.bf16_bits_to_f32(wb))
    x64 = synth.bf16_bits_to_f32(xb).astype(np.float64)
    ref = MX.gemv(x64, codes, scales)
    bound = 2e-5 * (np.abs(x64) @ np.abs(MX.dequantize(codes, scales)).T) + 1e-30
    got = y.cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
    # each row's bits do not depend on M
    for m in sorted({0, M // 2, M - 1}):
        one = dory.gemv_mxfp8(X[m:m + 1].contiguous(), q, s, impl=impl)
        assert torch.equal(one[0], y[m])


@pytest.mark.parametrize("M,N,K", [(1, 3584, 2560), (3, 512, 2048), (8, 4096, 2560), (2, 272, 640)])
def test_gemv_bulk_fed_same_bits_as_cuda_cores(M, N, K):
    """impl 4 streams the rows by bulk copies but keeps impl 1's arithmetic:
    the same bits."""
    rng = np.random.default_rng(M + N + K)
    w = rng.standard_normal((N, K)).astype(np.float32)
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    xb = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) / np.sqrt(K))
    q, s, _ = dory.quantize_mxfp8(bf16_cuda(synth.f32_to_bf16_bits(w)), dequantised=False)
    X = bf16_cuda(xb)
    assert torch.equal(dory.gemv_mxfp8(X, q, s, impl=4), dory.gemv_mxfp8(X, q, s, impl=1))


@pytest.mark.parametrize("impl", [1, 2])
def test_gemv_strided_operands_and_range_flag(impl):
    rng = np.random.default_rng(5)
    K, N = 512, 96
    w = synth.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.04)
    q, s, _ = dory.quantize_mxfp8(bf16_cuda(w), dequantised=False)
    xfull = bf16_cuda(synth.f32_to_bf16_bits(rng.standard_normal((3, K + 64)).astype(np.float32)))
    X = xfull[:, 32:32 + K]  # row stride K + 64
    Y = torch.full((3, N + 8), 7.0, device="cuda")
    dory.gemv_mxfp8(X, q, s, Y=Y[:, :N], impl=impl)
    ref = dory.gemv_mxfp8(X.contiguous(), q, s, impl=impl)
    torch.cuda.synchronize()
    assert torch.equal(Y[:, :N], ref) and bool((Y[:, N:] == 7.0).all())
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    big = X.contiguous().clone()
    big[1, 3] = 2.0 ** 70 if impl == 1 else float("inf")  # outside each kernel's range
    dory.gemv_mxfp8(big, q, s, impl=impl, err=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 4


def test_tensor_core_gemv_scales_each_token():
    # tokens of very different magnitudes in one call: each is staged with its own power of two
    rng = np.random.default_rng(6)
    K, N = 1024, 160
    w = synth.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.03)
    q, s, _ = dory.quantize_mxfp8(bf16_cuda(w), dequantised=False)
    x = rng.standard_normal((4, K)).astype(np.float32)
    x *= np.array([1e-20, 1.0, 3e10, 2.0 ** -60], np.float32)[:, None]
    xb = synth.f32_to_bf16_bits(x)
    y = dory.gemv_mxfp8(bf16_cuda(xb), q, s, impl=2).cpu().numpy()
    codes, scales = MX.quantize(synth.bf16_bits_to_f32(w))
    x64 = synth.bf16_bits_to_f32(xb).astype(np.float64)
    ref = MX.gemv(x64, codes, scales)
    bound = 2e-5 * (np.abs(x64) @ np.abs(MX.dequantize(codes, scales)).T)
    assert np.all(np.abs(y - ref) <= bound)


def mx_handle(shape, seed=0, alloc="per_loop"):
    w = synth.make_weights(shape, seed)
    dw = dory.DeviceWeights(shape, w)
    mx = dory.MxWeights(dw)
    h = dory.Handle(dory.make_config(shape, **CAP), mx.dequantised, dory.MODES[alloc])
    h.attach_mxfp8(mx)
    return w, h, mx


@pytest.fixture(scope="module", params=["tiny_bf16", "small128"])
def mx_model(request):
    shape = synth.SHAPES[request.param]
    w, h, mx = mx_handle(shape)
    return shape, O.Model(shape, MX.quantized_weights(w)), h, mx


@pytest.mark.parametrize("impl", [2, 1, 4])
@pytest.mark.parametrize("k", [1, 2, 4])
@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
def test_decode_with_mxfp8_matches_oracle(mx_model, k, mode, impl):
    shape, model, h, _ = mx_model
    prompt = synth.make_prompt(3, 40, shape.vocab)
    h.set_option(dory.OPT_MX_GEMV, impl)
    h.reset()
    om, cm = MODES[mode]
    toks, lg = gpu_generate(h, prompt, 13, k, cm)
    _, ora = O.generate(model, prompt, 13, k, om, forced=toks[:-1])
    errs = [rel_l2(lg[i], ora[i]) for i in range(len(toks))]
    assert max(errs) <= 2e-2, errs
    check_bf16_tokens(toks, ora)
    h.set_option(dory.OPT_MX_GEMV, 0)


def test_decode_reads_the_mxfp8_copies(mx_model):
    shape, _, h, _ = mx_model
    prompt = synth.make_prompt(4, 16, shape.vocab)
    h.reset()
    nxt = h.prefill([0], torch.tensor(prompt, dtype=torch.int32, device="cuda"), [16], 2, dory.LAST_LOOP)
    h.set_option(dory.OPT_PROFILE, 1)
    h.profile_reset()
    h.decode_step([0], nxt, 2, dory.LAST_LOOP)
    prof = h.profile_read()
    h.set_option(dory.OPT_PROFILE, 0)
    n, kk = shape.d_model, shape.q_dim
    per_launch = prof["gemm_o"]["bytes"] / prof["gemm_o"]["launches"]
    assert per_launch < 1.2 * n * kk  # 1 + 1/32 bytes per weight, not bf16's 2


@pytest.mark.parametrize("impl", [2, 1, 4])
def test_graph_replay_and_speculative_decoding_with_mxfp8(mx_model, impl):
    shape, _, h, _ = mx_model
    h.set_option(dory.OPT_MX_GEMV, impl)
    prompt = synth.make_prompt(5, 30, shape.vocab)
    tok = torch.tensor(prompt, dtype=torch.int32, device="cuda")

    def plain(graphs, n=10):
        h.set_option(dory.OPT_CUDA_GRAPHS, graphs)
        h.reset()
        nxt = h.prefill([0], tok, [30], 4, dory.PER_LOOP)
        out = [int(nxt[0])]
        for _ in range(n - 1):
            nxt = h.decode_step([0], nxt, 4, dory.PER_LOOP)
            out.append(int(nxt[0]))
        return out

    ref = plain(0)
    assert plain(1) == ref  # captured steps read the same copies
    h.reset()
    first = h.prefill([1], tok, [30], 4, dory.PER_LOOP)
    out, out_len, _ = h.spec_decode([1], first, 1, 4, 4, dory.PER_LOOP, 9)
    spec = [int(first[0])] + out[0].cpu().tolist()
    assert spec == ref  # per-loop speculative decoding is token-identical to plain k=4
    h.set_option(dory.OPT_CUDA_GRAPHS, 1)
    h.set_option(dory.OPT_MX_GEMV, 0)


def test_attach_validation():
    shape = synth.TINY_BF16
    _, h, mx = mx_handle(shape)
    bad = dory.MxWeightsC.from_buffer_copy(mx.c)
    bad.lm_head_s = None  # codes without scales
    with pytest.raises(dory.DoryError) as e:
        dory._check(dory.lib.dory_attach_mxfp8(h.h, bad))
    assert e.value.status == 1
    h.attach_mxfp8(None)  # detach; decoding goes back to the bf16 weights
    prompt = synth.make_prompt(6, 8, shape.vocab)
    nxt = h.prefill([0], torch.tensor(prompt, dtype=torch.int32, device="cuda"), [8], 1, dory.LAST_LOOP)
    h.decode_step([0], nxt, 1, dory.LAST_LOOP)
    h.synchronize()
    f32 = dory.Handle(dory.make_config(synth.TINY, **CAP), dory.DeviceWeights(synth.TINY, synth.make_weights(
        synth.TINY, 0)), dory.PER_LOOP)
    with pytest.raises(dory.DoryError) as e:
        f32.attach_mxfp8(mx)
    assert e.value.status == 7


# The TMA-fed tcgen05 GEMM (impl 3).


@pytest.mark.parametrize("M,N,K", [(1, 384, 256), (5, 2560, 2560), (16, 1024, 1024), (3, 128, 10240)])
def test_tma_tcgen05_gemm_matches_oracle(M, N, K):
    rng = np.random.default_rng(M + N + K)
    w = rng.standard_normal((N, K)).astype(np.float32)
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    w[0, 1:32] *= 1e-4
    wb = synth.f32_to_bf16_bits(w)
    xb = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) / np.sqrt(K))
    q, s, _ = dory.quantize_mxfp8(bf16_cuda(wb), dequantised=False)
    X = bf16_cuda(xb)
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    y = dory.gemv_mxfp8(X, q, s, impl=3, err=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    codes, scales = MX.quantize(synth.bf16_bits_to_f32(wb))
    x64 = synth.bf16_bits_to_f32(xb).astype(np.float64)
    ref = MX.gemv(x64, codes, scales)
    bound = 2e-5 * (np.abs(x64) @ np.abs(MX.dequantize(codes, scales)).T) + 1e-30
    got = y.cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
    for m in sorted({0, M - 1}):
        one = dory.gemv_mxfp8(X[m:m + 1].contiguous(), q, s, impl=3)
        assert torch.equal(one[0], y[m])


@pytest.mark.parametrize("k", [1, 4])
def test_decode_with_tma_tcgen05_gemm_matches_oracle(mx_model, k):
    shape, model, h, _ = mx_model
    prompt = synth.make_prompt(7, 40, shape.vocab)
    h.set_option(dory.OPT_MX_GEMV, 3)
    h.reset()
    toks, lg = gpu_generate(h, prompt, 9, k, dory.LAST_LOOP)
    h.synchronize()
    _, ora = O.generate(model, prompt, 9, k, O.LAST_LOOP, forced=toks[:-1])
    errs = [rel_l2(lg[i], ora[i]) for i in range(len(toks))]
    assert max(errs) <= 2e-2, errs
    check_bf16_tokens(toks, ora)
    # per-loop speculative decoding stays token-identical (draft and verify passes fit 16 rows)
    tok = torch.tensor(prompt[:30], dtype=torch.int32, device="cuda")
    h.reset()
    nxt = h.prefill([0], tok, [30], 4, dory.PER_LOOP)
    plain = [int(nxt[0])]
    for _ in range(7):
        nxt = h.decode_step([0], nxt, 4, dory.PER_LOOP)
        plain.append(int(nxt[0]))
    first = h.prefill([1], tok, [30], 4, dory.PER_LOOP)
    out, _, _ = h.spec_decode([1], first, 1, 4, 4, dory.PER_LOOP, 7)
    assert [int(first[0])] + out[0].cpu().tolist() == plain
    h.set_option(dory.OPT_MX_GEMV, 0)
