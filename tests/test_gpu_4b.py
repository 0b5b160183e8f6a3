"""4B-shaped bf16 model against the oracle on shortened workloads (GPU).

The oracle runs in float32 here (the float64 copy of 4.07B weights would not
fit in host memory); bf16 rounding on the GPU path dominates the error.
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
from gpu_util import MODES, check_tokens, cosine_rows, gpu_generate, rel_l2  # noqa: E402

SHAPE = synth.DORY_4B


@pytest.fixture(scope="module")
def model():
    w = synth.make_weights(SHAPE, 1)
    dw = dory.DeviceWeights(SHAPE, w)
    h = dory.Handle(dory.make_config(SHAPE, max_batch=2, max_seq=512, k_max=4, gamma_max=4, max_chunk=256), dw,
                    dory.PER_LOOP)
    om = O.Model(SHAPE, w, dtype=np.float32)
    del w
    return om, dw, h


@pytest.mark.parametrize("k,mode,n_new", [(2, "last_loop", 17), (1, "last_loop", 9), (4, "per_loop", 9)])
def test_4b_decode_matches_oracle(model, k, mode, n_new):
    om, _, h = model
    h.reset()
    prompt = synth.make_prompt(1, 32, SHAPE.vocab)
    o_mode, c_mode = MODES[mode]
    toks, lg = gpu_generate(h, prompt, n_new, k, c_mode)
    _, ora = O.generate(om, prompt, n_new, k, o_mode, forced=toks[:-1])
    errs = [rel_l2(lg[i], ora[i]) for i in range(n_new)]
    assert max(errs) <= 2e-2, errs
    tol = 4 * max(float(np.abs(lg[i] - ora[i]).max()) for i in range(n_new))
    check_tokens(toks, ora, tol)


def test_4b_prefill_final_state(model):
    om, _, h = model
    h.reset()
    prompt = synth.make_prompt(1, 64, SHAPE.vocab)
    h.prefill([0], torch.tensor(prompt, dtype=torch.int32, device="cuda"), [64], 2, dory.LAST_LOOP)
    s = h.read_state("s", 64).cpu().numpy()
    tr = {}
    O.forward_chunk(om, O.Cache(om, 64), prompt, 2, O.LAST_LOOP, trace=tr)
    assert cosine_rows(s, tr["s"][-1]).min() >= 0.999
