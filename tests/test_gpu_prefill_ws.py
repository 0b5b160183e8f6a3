"""The warp-specialised tcgen05 prefill attention (GPU) on the paths its
loader and its slot pairing take.

The model has five query heads per KV head (the 4B model's grouping), so one
head of every group is paired across two consecutive row tiles while the
others pair on the same rows; its window (160) makes the sliding-window ring
(160 + 16 slots) wrap inside key tiles, and its recurrent block attends fully.
A prompt prefilled in two chunks then reads, in the second chunk, key tiles
that lie wholly in the cache (copied by TMA), a tile that straddles the chunk
start and ring tiles that wrap (copied row by row), and tiles of the chunk
itself.  The kernel must follow the oracle within the bf16 bar (logits
relative L2 <= 2e-2, final-state cosine >= 0.999, greedy tokens identical up
to near ties), agree with the one-slot tcgen05 kernel within the same bar,
and give the same bits whether a full layer's cache is linear or paged
(pages of 128 positions are copied by TMA, pages of 64 row by row).
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
from gpu_util import MODES, check_bf16_tokens, cosine_rows, rel_l2  # noqa: E402

G5 = synth.Shape("g5_w160", 640, 2048, 5, 128, 1, 1024, 2, 2, 2, 160, full_every=2, full_phase=1, dtype="bf16")
CAP = dict(max_batch=3, max_seq=1024, k_max=4, gamma_max=4, max_chunk=640)


@pytest.fixture(scope="module")
def g5():
    w = synth.make_weights(G5, 11)
    dw = dory.DeviceWeights(G5, w)
    h = dory.Handle(dory.make_config(G5, **CAP), dw, dory.PER_LOOP)
    return O.Model(G5, w), dw, h


def prefill_chunks(h, prompt, chunks, k, cm, seq=0, steps=4):
    lg = torch.empty((1, G5.vocab), device="cuda")
    off = 0
    for c in chunks:
        nxt = h.prefill([seq], torch.tensor(prompt[off:off + c], dtype=torch.int32, device="cuda"), [c], k, cm,
                        logits=lg)
        off += c
    toks, logits = [int(nxt[0])], [lg[0].cpu().numpy().copy()]
    for _ in range(steps - 1):
        nxt = h.decode_step([seq], nxt, k, cm, logits=lg)
        toks.append(int(nxt[0]))
        logits.append(lg[0].cpu().numpy().copy())
    h.synchronize()
    return np.array(toks), np.stack(logits)


@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
def test_ws_chunked_prefill_matches_oracle(g5, mode):
    model, _, h = g5
    om, cm = MODES[mode]
    prompt = synth.make_prompt(31, 700, G5.vocab)
    chunks = [300, 400]
    h.set_option(dory.OPT_PREFILL_TC, 3)
    h.reset()
    toks, lg = prefill_chunks(h, prompt, chunks, 2, cm)
    _, ora = O.generate(model, prompt, len(toks), 2, om, chunks=chunks, forced=toks[:-1])
    errs = [rel_l2(lg[i], ora[i]) for i in range(len(toks))]
    assert max(errs) <= 2e-2, errs
    check_bf16_tokens(toks, ora)


def test_ws_agrees_with_one_slot_kernel(g5):
    model, _, h = g5
    prompt = synth.make_prompt(32, 600, G5.vocab)
    states = {}
    for tc in (2, 3):
        h.set_option(dory.OPT_PREFILL_TC, tc)
        h.reset()
        h.prefill([0], torch.tensor(prompt, dtype=torch.int32, device="cuda"), [600], 2, dory.LAST_LOOP)
        states[tc] = h.read_state("s", 600).cpu().numpy()
    h.set_option(dory.OPT_PREFILL_TC, 3)
    assert cosine_rows(states[2], states[3]).min() >= 0.999
    tr = {}
    O.forward_chunk(model, O.Cache(model, 610), prompt, 2, O.LAST_LOOP, trace=tr)
    assert cosine_rows(states[3], tr["s"][-1]).min() >= 0.999


def test_ws_ragged_batch(g5):
    """Three sequences in one call (one shorter than a tile): tiles of
    different sequences never share a work item."""
    model, _, h = g5
    h.set_option(dory.OPT_PREFILL_TC, 3)
    h.reset()
    lens = (300, 5, 260)
    prompts = [synth.make_prompt(40 + b, n, G5.vocab) for b, n in enumerate(lens)]
    ids = [2, 0, 1]
    lg = torch.empty((3, G5.vocab), device="cuda")
    tok = torch.tensor(np.concatenate(prompts), dtype=torch.int32, device="cuda")
    h.prefill(ids, tok, list(lens), 2, dory.PER_LOOP, logits=lg)
    got = lg.cpu().numpy()
    for b, p in enumerate(prompts):
        ora = O.forward_chunk(model, O.Cache(model, len(p) + 8), p, 2, O.PER_LOOP)
        assert rel_l2(got[b], ora[-1]) <= 2e-2, b


@pytest.mark.parametrize("page", [128, 64])
def test_ws_paged_cache_same_bits(g5, page):
    model, dw, lin = g5
    pag = dory.Handle(dory.make_config(G5, kv_page=page, kv_pages=2 * (1024 // page), **CAP), dw, dory.PER_LOOP)
    prompt = synth.make_prompt(33, 520, G5.vocab)
    chunks = [260, 260]  # the second chunk reads two whole cached 128-key tiles
    out = []
    for h in (lin, pag):
        h.set_option(dory.OPT_PREFILL_TC, 3)
        h.reset()
        out.append(prefill_chunks(h, prompt, chunks, 2, dory.LAST_LOOP))
    assert np.array_equal(out[0][0], out[1][0]) and np.array_equal(out[0][1], out[1][1])
    _, ora = O.generate(model, prompt, len(out[1][0]), 2, O.LAST_LOOP, chunks=chunks, forced=out[1][0][:-1])
    assert max(rel_l2(out[1][1][i], ora[i]) for i in range(len(out[1][0]))) <= 2e-2
    pag.close()


def test_ws_deterministic(g5):
    """Repeated prefills agree bit for bit (no result depends on which CTA
    finishes first)."""
    _, _, h = g5
    h.set_option(dory.OPT_PREFILL_TC, 3)
    prompt = synth.make_prompt(34, 640, G5.vocab)
    outs = []
    for _ in range(3):
        h.reset()
        lg = torch.empty((1, G5.vocab), device="cuda")
        h.prefill([0], torch.tensor(prompt, dtype=torch.int32, device="cuda"), [640], 2, dory.LAST_LOOP, logits=lg)
        outs.append(np.concatenate([lg.cpu().numpy().ravel(), h.read_state("s", 640).cpu().numpy().ravel()]))
    assert all(np.array_equal(outs[0], o) for o in outs[1:])
