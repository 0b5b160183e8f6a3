"""Mixed-k batched decode (GPU): one decode step in which every sequence runs
its own loop count (sequences grouped by non-increasing k; loop t runs only
on the sequences with k >= t).  Each sequence must match the oracle run of
that sequence alone at its own k: within 1e-4 (max abs logit error) for the
tiny fp32 model, and within the bf16 bar (logits relative L2 error <= 2e-2)
for the bf16 model with 128-wide heads."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402
from gpu_util import MODES, make, rel_l2  # noqa: E402

KS = [4, 2, 2, 1]
STEPS = 4


@pytest.fixture(scope="module", params=["tiny", "small128"])
def setup(request):
    shape = synth.TINY if request.param == "tiny" else synth.SMALL128
    w, dw, h = make(shape, seed=7, max_batch=4, max_seq=96, k_max=4, gamma_max=4, max_chunk=128)
    return shape, O.Model(shape, w), dw, h


@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
def test_mixed_k_decode_matches_oracle_per_sequence(setup, mode):
    shape, model, _, h = setup
    om, cm = MODES[mode]
    h.reset()
    prompts = [synth.make_prompt(30 + i, 20 + 3 * i, shape.vocab) for i in range(len(KS))]
    ids = list(range(len(KS)))
    lg = torch.empty((1, shape.vocab), device="cuda")
    first, pre_logits = [], []
    for i, (p, k) in enumerate(zip(prompts, KS)):  # each sequence prefilled at its own k
        t = h.prefill([i], torch.tensor(p, dtype=torch.int32, device="cuda"), [len(p)], k, cm, logits=lg)
        first.append(int(t[0]))
        pre_logits.append(lg[0].cpu().numpy().copy())
    tok = torch.tensor(first, dtype=torch.int32, device="cuda")
    L = torch.empty((len(KS), shape.vocab), device="cuda")
    toks, logits = [np.array(first)], []
    for _ in range(STEPS):
        tok = h.decode_step_mixed(ids, tok, KS, cm, logits=L)
        toks.append(tok.cpu().numpy().copy())
        logits.append(L.cpu().numpy().copy())
    h.synchronize()
    for i, (p, k) in enumerate(zip(prompts, KS)):
        forced = [int(toks[s][i]) for s in range(STEPS)]
        _, ora = O.generate(model, p, STEPS + 1, k, om, forced=forced)
        got = np.stack([pre_logits[i]] + [logits[s][i] for s in range(STEPS)])
        if shape.dtype == "f32":
            assert np.abs(got - ora).max() <= 1e-4, (i, k)
        else:
            assert max(rel_l2(got[s], ora[s]) for s in range(STEPS + 1)) <= 2e-2, (i, k)
