"""Paged full-attention cache (GPU).

The full-attention layers' positions live in pages drawn from a pool
(kv_page, kv_pages in the config); the pages only change where K/V sit, so a
paged handle must compute exactly what a linear one computes, and both must
follow the oracle (which stores the cache by absolute position) across page
boundaries.  The full-attention layer pattern is moved so a recurrent layer
and an output-block layer attend fully (the digest, onedev.kr "How it works",
interleaves full and sliding-window attention; the phase is a reading).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402
from gpu_util import MODES, check_bf16_tokens, check_tokens, gpu_generate, rel_l2  # noqa: E402

F32_TOL = 1e-4
TINY_FULL = synth.TINY.with_(name="tiny_full2", full_every=2, full_phase=1)
SMALL_FULL = synth.SMALL128.with_(name="small128_full2", full_every=2, full_phase=1)


def handles(shape, pages, **cap):
    w = synth.make_weights(shape, 3)
    dw = dory.DeviceWeights(shape, w)
    lin = dory.Handle(dory.make_config(shape, **cap), dw, dory.PER_LOOP)
    pag = dory.Handle(dory.make_config(shape, kv_page=16, kv_pages=pages, **cap), dw, dory.PER_LOOP)
    return O.Model(shape, w), dw, lin, pag


@pytest.fixture(scope="module")
def tiny():
    return handles(TINY_FULL, 24, max_batch=3, max_seq=128, k_max=4, gamma_max=4, max_chunk=96)


@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
@pytest.mark.parametrize("k", [1, 2])
def test_paged_matches_linear_and_oracle(tiny, mode, k):
    model, _, lin, pag = tiny
    om, cm = MODES[mode]
    prompt = synth.make_prompt(4, 40, TINY_FULL.vocab)
    lin.reset()
    pag.reset()
    t_lin, l_lin = gpu_generate(lin, prompt, 31, k, cm)
    t_pag, l_pag = gpu_generate(pag, prompt, 31, k, cm)  # positions 0..70: five 16-position pages
    assert np.array_equal(t_pag, t_lin) and np.array_equal(l_pag, l_lin)
    _, ora = O.generate(model, prompt, 31, k, om, forced=t_pag[:-1])
    assert np.abs(l_pag - ora).max() <= F32_TOL
    check_tokens(t_pag, ora, tol=2 * F32_TOL)
    # the full-attention recurrent layer's cache read back through the page table
    for p in (0, 15, 16, 47, 69):
        a = pag.read_kv(2, 0, 0, p, 1)
        b = lin.read_kv(2, 0, 0, p, 1)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_pages_return_to_the_pool_on_reset():
    """Two sequences of 64 tokens take all 8 pages of a small pool; a decode
    step that needs a ninth page is refused before any work (the sequence's
    length stays), a reset returns pages, and recycled pages (still holding
    the old sequence's keys) give the results of a linear cache (sequence 1
    ends on 5 pages, the new sequence 0 on 3)."""
    model, _, lin, pag = handles(TINY_FULL, 8, max_batch=2, max_seq=128, k_max=4, gamma_max=4, max_chunk=128)
    prompts = [synth.make_prompt(10 + i, n, TINY_FULL.vocab) for i, n in enumerate((64, 64, 40))]
    tok = torch.tensor(np.concatenate(prompts[:2]), dtype=torch.int32, device="cuda")
    nxt = pag.prefill([0, 1], tok, [64, 64], 2, dory.LAST_LOOP)
    with pytest.raises(dory.DoryError) as e:
        pag.decode_step([1], nxt[1:], 2, dory.LAST_LOOP)
    assert e.value.status == 2
    assert pag.seq_len(1) == 64
    pag.reset(0)
    got = [int(nxt[1])]
    cur = nxt[1:].clone()
    for _ in range(5):
        cur = pag.decode_step([1], cur, 2, dory.LAST_LOOP)
        got.append(int(cur[0]))
    again = gpu_generate(pag, prompts[2], 6, 2, dory.LAST_LOOP, seq=0)  # on recycled pages
    lin.reset()
    ref1 = gpu_generate(lin, prompts[1], 6, 2, dory.LAST_LOOP, seq=1)
    ref0 = gpu_generate(lin, prompts[2], 6, 2, dory.LAST_LOOP, seq=0)
    assert got == list(ref1[0])
    assert np.array_equal(again[0], ref0[0]) and np.array_equal(again[1], ref0[1])
    lin.close()
    pag.close()


def test_speculative_decoding_on_paged_cache(tiny):
    _, _, _, pag = tiny
    pag.reset()
    prompt = synth.make_prompt(6, 30, TINY_FULL.vocab)
    plain, _ = gpu_generate(pag, prompt, 20, 4, dory.PER_LOOP, seq=0)
    tok = torch.tensor(prompt, dtype=torch.int32, device="cuda")
    first = pag.prefill([1], tok, [30], 4, dory.PER_LOOP)
    out, out_len, _ = pag.spec_decode([1], first, 1, 4, 4, dory.PER_LOOP, 19)
    assert [int(first[0])] + out[0].cpu().tolist() == list(plain)


def test_paged_bf16_chunked_prefill_on_tensor_core_attention():
    """bf16 with 128-wide heads: the tcgen05 prefill attention reads the
    earlier chunk's keys through the page table, then decode steps."""
    model, _, lin, pag = handles(SMALL_FULL, 16, max_batch=2, max_seq=160, k_max=4, gamma_max=4, max_chunk=128)
    prompt = synth.make_prompt(5, 100, SMALL_FULL.vocab)
    lg = torch.empty((1, SMALL_FULL.vocab), device="cuda")
    outs = []
    for h in (lin, pag):
        h.reset()
        for off, n in ((0, 70), (70, 30)):
            t = torch.tensor(prompt[off:off + n], dtype=torch.int32, device="cuda")
            nxt = h.prefill([0], t, [n], 2, dory.LAST_LOOP, logits=lg)
        toks, logits = [int(nxt[0])], [lg[0].cpu().numpy().copy()]
        for _ in range(8):
            nxt = h.decode_step([0], nxt, 2, dory.LAST_LOOP, logits=lg)
            toks.append(int(nxt[0]))
            logits.append(lg[0].cpu().numpy().copy())
        h.synchronize()
        outs.append((np.array(toks), np.stack(logits)))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    _, ora = O.generate(model, prompt, 9, 2, O.LAST_LOOP, chunks=[70, 30], forced=outs[1][0][:-1])
    assert max(rel_l2(outs[1][1][i], ora[i]) for i in range(9)) <= 2e-2
    check_bf16_tokens(outs[1][0], ora)
    lin.close()
    pag.close()
