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
from gpu_util import MODES, check_bf16_tokens, cosine_rows, gpu_generate, rel_l2  # noqa: E402

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
    ties = check_bf16_tokens(toks, ora)
    print(f"4B k={k} {mode}: near-tie exemptions {ties}")


@pytest.mark.parametrize("n", [64, 256])  # 256 rows: the warp-per-row add + norm
def test_4b_prefill_final_state(model, n):
    om, _, h = model
    h.reset()
    prompt = synth.make_prompt(1, n, SHAPE.vocab)
    h.prefill([0], torch.tensor(prompt, dtype=torch.int32, device="cuda"), [n], 2, dory.LAST_LOOP)
    s = h.read_state("s", n).cpu().numpy()
    tr = {}
    O.forward_chunk(om, O.Cache(om, n), prompt, 2, O.LAST_LOOP, trace=tr)
    assert cosine_rows(s, tr["s"][-1]).min() >= 0.999


def _oracle_layer0_kv(om, tok):
    """Layer 0's K and V of one token, from the oracle's attention sublayer on
    a one-position cache (no positional encoding: the same at every position)."""
    cache = O.Cache(om, 1)
    O.attention(om, cache, 0, 0, om.w["embed"][np.array([tok])], np.array([0]))
    K, V, _ = cache.arrays(0, 0)
    return K[0], V[0]


def test_4b_bench_configuration(model):
    """The configuration the bench times (2560-token prefill, k=2, last_loop,
    graph-replayed decode steps), checked where the oracle can follow one
    value at a time: layer-0 K/V at sampled positions, unit-norm states,
    and graph replay bit-identical to eager launches."""
    om, dw, _ = model
    P, n = 2560, 6
    cfg = dory.make_config(SHAPE, max_batch=1, max_seq=P + 64, k_max=4, gamma_max=4, max_chunk=P)
    h = dory.Handle(cfg, dw, dory.LAST_LOOP)
    prompt = synth.make_prompt(1, P, SHAPE.vocab)
    tok = torch.tensor(prompt, dtype=torch.int32, device="cuda")

    def run(graphs):
        h.set_option(dory.OPT_CUDA_GRAPHS, graphs)
        h.reset()
        nxt = h.prefill([0], tok, [P], 2, dory.LAST_LOOP)
        out = [int(nxt[0])]
        for _ in range(n):
            nxt = h.decode_step([0], nxt, 2, dory.LAST_LOOP)
            out.append(int(nxt[0]))
        h.synchronize()
        return out

    eager = run(0)
    graph = run(1)
    h.set_option(dory.OPT_CUDA_GRAPHS, 1)
    assert graph == eager
    s = h.read_state("s", 1).cpu().numpy()
    assert abs(float(np.linalg.norm(s[0])) - 1.0) < 1e-5
    # layer 0 (sliding window, ring of 4112 positions: all of them retained)
    inputs = list(prompt) + graph[:n]
    for p in (0, 1, 1000, P - 1, P, P + n - 1):
        k, v = h.read_kv(0, 0, 0, p, 1)
        ko, vo = _oracle_layer0_kv(om, int(inputs[p]))
        for got, ref in ((k[0].float().cpu().numpy(), ko), (v[0].float().cpu().numpy(), vo)):
            assert np.abs(got - ref).max() <= 2.0 ** -7 * np.abs(ref).max(), p
    h.close()
