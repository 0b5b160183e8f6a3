"""Decode attention at larger batch (GPU).  The tensor-core decode attention
shares each row's keys among 16, 8 or 4 blocks of a cluster, chosen from the
number of sequences in the call.  Every size must match the oracle within the
bf16 bar (logits relative L2 error <= 2e-2), and per_loop speculative decoding
must stay token-identical to plain k=4 decoding at a batch that selects a
smaller cluster (plain decode and the verify chunk of the same sequences
split every row's keys the same way)."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import looped_ngpt_lm_b200 as dory  # noqa: E402
from gpu_util import make, rel_l2  # noqa: E402

SHAPE = synth.SMALL128  # one KV head: a batch of b sequences gives b (row, KV head) pairs
P = 24


@pytest.fixture(scope="module")
def big():
    w, dw, h = make(SHAPE, seed=4, max_batch=80, max_seq=96, k_max=4, gamma_max=4, max_chunk=80 * P)
    return O.Model(SHAPE, w), dw, h


def prompts(n):
    return [synth.make_prompt(100 + b, P, SHAPE.vocab) for b in range(n)]


@pytest.mark.parametrize("batch", [36, 40, 80])  # 16, 8 and 4 blocks per row
def test_batched_decode_matches_oracle(big, batch):
    model, _, h = big
    h.reset()
    ps = prompts(batch)
    ids = list(range(batch))
    tok = torch.tensor(np.concatenate(ps), dtype=torch.int32, device="cuda")
    nxt = h.prefill(ids, tok, [P] * batch, 2, dory.LAST_LOOP)
    lg = torch.empty((batch, SHAPE.vocab), device="cuda")
    toks, logits = [nxt.cpu().numpy().copy()], []
    for _ in range(3):
        nxt = h.decode_step(ids, nxt, 2, dory.LAST_LOOP, logits=lg)
        toks.append(nxt.cpu().numpy().copy())
        logits.append(lg.cpu().numpy().copy())
    h.synchronize()
    # the oracle on a sample of the sequences, fed the GPU's tokens
    for b in sorted({0, batch // 2, batch - 1}):
        forced = [int(toks[i][b]) for i in range(3)]
        _, ora = O.generate(model, ps[b], 4, 2, O.LAST_LOOP, forced=forced)
        errs = [rel_l2(logits[i][b], ora[i + 1]) for i in range(3)]
        assert max(errs) <= 2e-2, (b, errs)


def test_spec_identity_with_smaller_cluster(big):
    _, _, h = big
    B, n_new = 40, 10
    ps = prompts(B)
    tok = torch.tensor(np.concatenate(ps), dtype=torch.int32, device="cuda")
    ids_plain, ids_spec = list(range(B)), list(range(B, 2 * B))
    h.reset()
    first_p = h.prefill(ids_plain, tok, [P] * B, 4, dory.PER_LOOP)
    first_s = h.prefill(ids_spec, tok, [P] * B, 4, dory.PER_LOOP)
    plain, nxt = [first_p.cpu().numpy().copy()], first_p
    for _ in range(n_new - 1):
        nxt = h.decode_step(ids_plain, nxt, 4, dory.PER_LOOP)
        plain.append(nxt.cpu().numpy().copy())
    plain = np.stack(plain, 1)
    out, out_len, _ = h.spec_decode(ids_spec, first_s, 1, 4, 4, dory.PER_LOOP, n_new - 1)
    spec = np.concatenate([first_s.cpu().numpy()[:, None], out.cpu().numpy()], 1)
    assert (out_len.cpu().numpy() == n_new - 1).all()
    assert np.array_equal(spec, plain)
