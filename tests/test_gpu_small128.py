"""bf16 model with 128-wide heads and a 32-key window (GPU): long prefill
chunks take the tensor-core attention, sliding-window rings wrap, and the
result must match the oracle within the bf16 bar (logits relative L2 error
<= 2e-2, final-state cosine >= 0.999, greedy tokens identical up to near ties)."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402
from gpu_util import MODES, check_bf16_tokens, cosine_rows, make, rel_l2  # noqa: E402

SHAPE = synth.SMALL128


@pytest.fixture(scope="module")
def small():
    w, dw, h = make(SHAPE, seed=3, max_batch=4, max_seq=256, k_max=4, gamma_max=4, max_chunk=200)
    return O.Model(SHAPE, w), dw, h


def run_chunks(h, prompt, chunks, k, cm, seq=0, steps=6):
    lg = torch.empty((1, SHAPE.vocab), device="cuda")
    off = 0
    for c in chunks:
        h.prefill([seq], torch.tensor(prompt[off:off + c], dtype=torch.int32, device="cuda"), [c], k, cm, logits=lg)
        off += c
    nxt = torch.tensor([int(torch.argmax(lg[0]))], dtype=torch.int32, device="cuda")
    toks, logits = [int(nxt[0])], [lg[0].cpu().numpy().copy()]
    for _ in range(steps - 1):
        nxt = h.decode_step([seq], nxt, k, cm, logits=lg)
        toks.append(int(nxt[0]))
        logits.append(lg[0].cpu().numpy().copy())
    return np.array(toks), np.stack(logits)


@pytest.mark.parametrize("k", [1, 2, 4])
@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
def test_small128_chunked_prefill_and_decode(small, k, mode):
    model, _, h = small
    om, cm = MODES[mode]
    prompt = synth.make_prompt(5, 100, SHAPE.vocab)
    h.reset()
    toks, lg = run_chunks(h, prompt, [70, 30], k, cm)
    _, ora = O.generate(model, prompt, 6, k, om, chunks=[70, 30], forced=toks[:-1])
    errs = [rel_l2(lg[i], ora[i]) for i in range(len(toks))]
    assert max(errs) <= 2e-2, errs
    check_bf16_tokens(toks, ora)


@pytest.mark.parametrize("tc", [0, 1, 2, 3])  # CUDA cores, mma.sync, tcgen05 one slot, warp-specialised
def test_small128_prefill_state_both_attention_kernels(small, tc):
    model, _, h = small
    prompt = synth.make_prompt(6, 150, SHAPE.vocab)
    h.set_option(dory.OPT_PREFILL_TC, tc)
    h.reset()
    h.prefill([0], torch.tensor(prompt, dtype=torch.int32, device="cuda"), [150], 2, dory.LAST_LOOP)
    s = h.read_state("s", 150).cpu().numpy()
    h.set_option(dory.OPT_PREFILL_TC, 3)
    tr = {}
    O.forward_chunk(model, O.Cache(model, 160), prompt, 2, O.LAST_LOOP, trace=tr)
    assert cosine_rows(s, tr["s"][-1]).min() >= 0.999


def test_small128_ragged_batch(small):
    model, _, h = small
    h.reset()
    prompts = [synth.make_prompt(20 + b, n, SHAPE.vocab) for b, n in enumerate((65, 3, 120))]
    ids = [1, 3, 0]
    lg = torch.empty((3, SHAPE.vocab), device="cuda")
    tok = torch.tensor(np.concatenate(prompts), dtype=torch.int32, device="cuda")
    h.prefill(ids, tok, [len(p) for p in prompts], 2, dory.PER_LOOP, logits=lg)
    got = lg.cpu().numpy()
    for b, p in enumerate(prompts):
        ora = O.forward_chunk(model, O.Cache(model, 130), p, 2, O.PER_LOOP)
        assert rel_l2(got[b], ora[-1]) <= 2e-2
