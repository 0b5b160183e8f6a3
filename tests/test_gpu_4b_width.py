"""The kernels' full-size paths against the oracle, on a cut model of the 4B
width (GPU).

The 4B-shaped model keeps its width (d 2560, 20 query heads x 128, 4 KV
heads, SwiGLU 10240, vocab 131072) and gets 2 + 4 + 2 physical layers with the
full-attention phase moved so the recurrent block holds one full and one
sliding-window layer (window 4096).  The layer structure and the last-loop
cache follow the Dory1.0-4B digest (onedev.kr, "How it works": 27 SWA and 9
full attention layers interleaved; "Premises & limits": each loop overwrites
the previous loop's cache).  The oracle finishes this model in minutes, so the
paths the bench configuration takes can be compared with it directly:

* a 2600-token prompt in one chunk (the tcgen05 prefill attention on 21 tiles
  of 128 rows, the last one ragged), then 16 greedy decode steps at k = 2 in
  both cache modes; at batch 1 each of the 16 blocks of a decode attention
  cluster holds more than 128 keys, so its second key chunk is used;
* a 4300-token prompt: the sliding-window ring (4096 + 16 slots) wraps during
  the prefill commit and again during decoding, and the full layer's blocks
  refill their key chunks three times;
* 20 sequences of about 1040 tokens decoded together, which selects clusters
  of 4 blocks (over 256 keys per block: three key chunks);
* self-speculative decoding where the verifier rejects drafts.

Tolerances are those of the bf16 configurations: logits relative L2 <= 2e-2,
final-state cosine >= 0.999, greedy tokens identical except at near ties
under a threshold fixed by that tolerance (gpu_util.check_bf16_tokens).
Cached K/V of a recurrent layer are compared position by position (relative
L2 <= 2e-2): a wrong slot, loop or ring index gives unrelated vectors.
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
import oracle_jobs  # noqa: E402
from gpu_util import MODES, check_bf16_tokens, cosine_rows, rel_l2  # noqa: E402

CUT = synth.DORY_4B.with_(name="dory4b_cut", n_in=2, n_rec=4, n_out=2, full_phase=1)
SEED = 1
LOGITS_TOL = 2e-2
KV_TOL = 2e-2
COS_MIN = 0.999
N_DEC = 16
P_LONG = 2600
P_WRAP = 4300
BATCH = 20
BATCH_SAMPLE = (0, 9, 19)
SPEC_PROMPT, SPEC_NEW = 48, 24
REC_FULL, REC_SWA = 2, 4  # recurrent attention layers (global attention index 1 is full)


def batch_lens():
    return [1040 + 3 * i for i in range(BATCH)]


def batch_prompt(i):
    return synth.make_prompt(100 + i, batch_lens()[i], CUT.vocab)


@pytest.fixture(scope="module")
def env():
    # the oracle's prefills start in worker processes before any GPU work
    ex, saved = oracle_jobs.pool(workers=4, threads_each=4)
    jobs = {}
    cap = P_WRAP + N_DEC + 8
    try:
        jobs["wrap"] = ex.submit(oracle_jobs.prefill, CUT, SEED, synth.make_prompt(2, P_WRAP, CUT.vocab), 2,
                                 O.LAST_LOOP, cap)
        for mode in ("last_loop", "per_loop"):
            jobs[f"long_{mode}"] = ex.submit(oracle_jobs.prefill, CUT, SEED, synth.make_prompt(1, P_LONG, CUT.vocab),
                                             2, MODES[mode][0], cap)
        for i in BATCH_SAMPLE:
            jobs[f"batch{i}"] = ex.submit(oracle_jobs.prefill, CUT, SEED, batch_prompt(i), 1, O.LAST_LOOP, cap)
        jobs["spec"] = ex.submit(oracle_jobs.spec, CUT, SEED, synth.make_prompt(10, SPEC_PROMPT, CUT.vocab),
                                 SPEC_NEW, 4, O.LAST_LOOP)
    finally:
        oracle_jobs.release_env(saved)
    w = synth.make_weights(CUT, SEED)
    dw = dory.DeviceWeights(CUT, w)
    om = O.Model(CUT, w, dtype=np.float32)
    del w
    cfg = dory.make_config(CUT, max_batch=BATCH, max_seq=P_WRAP + N_DEC + 16, k_max=4, gamma_max=4,
                           max_chunk=P_WRAP + 100)
    h = dory.Handle(cfg, dw, dory.PER_LOOP)
    yield {"om": om, "h": h, "jobs": jobs}
    h.close()
    ex.shutdown(cancel_futures=True)


def oracle_slot(l, gpu_slot, mode):
    """The oracle numbers per-loop slots of recurrent layers 1..k; the
    library numbers them 0..k-1."""
    return gpu_slot + 1 if mode == O.PER_LOOP and CUT.n_in <= l < CUT.n_in + CUT.n_rec else gpu_slot


def check_kv(h, cache, layer, gpu_slot, mode, seq, positions):
    K, V, written = cache.arrays(layer, oracle_slot(layer, gpu_slot, mode))
    for p in positions:
        k, v = h.read_kv(layer, gpu_slot, seq, p, 1)
        assert written[p], (layer, p)
        for got, ref in ((k[0], K[p]), (v[0], V[p])):
            err = rel_l2(got.float().cpu().numpy().astype(np.float64), ref.astype(np.float64))
            assert err <= KV_TOL, (layer, gpu_slot, p, err)


def run_case(env, key, prompt, k, mode):
    om, h = env["om"], env["h"]
    o_mode, c_mode = MODES[mode]
    P = len(prompt)
    h.reset()
    lg = torch.empty((1, CUT.vocab), device="cuda")
    tok = torch.tensor(prompt, dtype=torch.int32, device="cuda")
    nxt = h.prefill([0], tok, [P], k, c_mode, logits=lg)
    s_pre = h.read_state("s", P).cpu().numpy()
    toks, logits, s_dec = [int(nxt[0])], [lg[0].cpu().numpy().copy()], []
    for _ in range(N_DEC):
        nxt = h.decode_step([0], nxt, k, c_mode, logits=lg)
        toks.append(int(nxt[0]))
        logits.append(lg[0].cpu().numpy().copy())
        s_dec.append(h.read_state("s", 1).cpu().numpy()[0])
    h.synchronize()

    res = env["jobs"][key].result()
    cos = cosine_rows(s_pre.astype(np.float64), res["s"].astype(np.float64))
    assert cos.min() >= COS_MIN, (int(np.argmin(cos)), float(cos.min()))
    cache = oracle_jobs.restore(om, res)
    ora, ora_s = [res["logits"]], []
    for i in range(N_DEC):
        tr = {}
        ora.append(O.forward_chunk(om, cache, [toks[i]], k, o_mode, trace=tr)[-1])
        ora_s.append(tr["s"][-1][0])
    errs = [rel_l2(logits[i].astype(np.float64), ora[i].astype(np.float64)) for i in range(N_DEC + 1)]
    assert max(errs) <= LOGITS_TOL, errs
    cos_dec = cosine_rows(np.stack(s_dec).astype(np.float64), np.stack(ora_s).astype(np.float64))
    assert cos_dec.min() >= COS_MIN, cos_dec
    ties = check_bf16_tokens(toks, ora)
    print(f"{key}: max logits rel L2 {max(errs):.2e}, min cosine {cos.min():.6f}/{cos_dec.min():.6f}, "
          f"near-tie exemptions {ties['exempt']} (min oracle margin {ties['min_margin']:.2e}, "
          f"threshold {ties['threshold']:.2e})")
    return h, cache, toks


@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
def test_prompt_2600_then_16_decode_steps(env, mode):
    k = 2
    h, cache, _ = run_case(env, f"long_{mode}", synth.make_prompt(1, P_LONG, CUT.vocab), k, mode)
    o_mode = MODES[mode][0]
    end = P_LONG + N_DEC  # positions written: 0 .. end - 1
    pos = [0, 1, 777, P_LONG - 1, P_LONG, end - 1]
    # last_loop: the one slot holds each token's final-loop K/V; per_loop: one slot per loop
    for layer in (REC_FULL, REC_SWA):
        for slot in ([0] if mode == "last_loop" else range(k)):
            check_kv(h, cache, layer, slot, o_mode, 0, pos)
    check_kv(h, cache, 0, 0, o_mode, 0, pos)  # input block


def test_prompt_4300_wraps_the_window_ring(env):
    h, cache, _ = run_case(env, "wrap", synth.make_prompt(2, P_WRAP, CUT.vocab), 2, "last_loop")
    end = P_WRAP + N_DEC
    ring = CUT.swa_window + 16  # window + slack of the speculative writes (gamma_max 4)
    assert end > ring
    # still in the ring: the last `ring` positions
    check_kv(h, cache, REC_SWA, 0, O.LAST_LOOP, 0, [end - ring, P_WRAP - 1, P_WRAP, end - 1])
    check_kv(h, cache, REC_FULL, 0, O.LAST_LOOP, 0, [0, 2047, P_WRAP - 1, end - 1])


def test_batched_decode_on_four_block_clusters(env):
    om, h = env["om"], env["h"]
    h.reset()
    lens = batch_lens()
    prompts = [batch_prompt(i) for i in range(BATCH)]
    lg = torch.empty((BATCH, CUT.vocab), device="cuda")
    first = torch.empty(BATCH, dtype=torch.int32, device="cuda")
    pre = np.empty((BATCH, CUT.vocab), np.float32)
    for g in range(0, BATCH, 4):  # four sequences per prefill call (ragged rows)
        ids = list(range(g, g + 4))
        tok = torch.tensor(np.concatenate(prompts[g:g + 4]), dtype=torch.int32, device="cuda")
        part = torch.empty((4, CUT.vocab), device="cuda")
        first[g:g + 4] = h.prefill(ids, tok, lens[g:g + 4], 1, dory.LAST_LOOP, logits=part)
        pre[g:g + 4] = part.cpu().numpy()
    ids = list(range(BATCH))
    toks, logits = [first.cpu().numpy().copy()], [pre]
    nxt = first
    steps = 6
    for _ in range(steps):
        nxt = h.decode_step(ids, nxt, 1, dory.LAST_LOOP, logits=lg)
        toks.append(nxt.cpu().numpy().copy())
        logits.append(lg.cpu().numpy().copy())
    h.synchronize()
    for i in BATCH_SAMPLE:
        res = env["jobs"][f"batch{i}"].result()
        cache = oracle_jobs.restore(om, res)
        ora = [res["logits"]]
        for s in range(steps):
            ora.append(O.forward_chunk(om, cache, [int(toks[s][i])], 1, O.LAST_LOOP)[-1])
        errs = [rel_l2(logits[s][i].astype(np.float64), ora[s].astype(np.float64)) for s in range(steps + 1)]
        assert max(errs) <= LOGITS_TOL, (i, errs)
        ties = check_bf16_tokens([toks[s][i] for s in range(steps + 1)], ora)
        print(f"batch seq {i}: max logits rel L2 {max(errs):.2e}, near-tie exemptions {ties['exempt']}")


def test_speculative_decoding_with_rejections(env):
    """The verifier rejects drafts on this model (the oracle accepts fewer
    than gamma drafts in most steps), so the rollback of lengths and ring
    slots runs at the 4B width.  per_loop: token-identical to plain k = 4
    decoding on the GPU.  last_loop: token-identical to the oracle running
    the same draft / verify schedule."""
    h = env["h"]
    prompt = synth.make_prompt(10, SPEC_PROMPT, CUT.vocab)
    tok = torch.tensor(prompt, dtype=torch.int32, device="cuda")
    h.reset()
    nxt = h.prefill([0], tok, [SPEC_PROMPT], 4, dory.PER_LOOP)
    plain = [int(nxt[0])]
    for _ in range(SPEC_NEW - 1):
        nxt = h.decode_step([0], nxt, 4, dory.PER_LOOP)
        plain.append(int(nxt[0]))
    first = h.prefill([1], tok, [SPEC_PROMPT], 4, dory.PER_LOOP)
    out, out_len, st = h.spec_decode([1], first, 1, 4, 4, dory.PER_LOOP, SPEC_NEW - 1)
    assert int(out_len[0]) == SPEC_NEW - 1
    assert [int(first[0])] + out[0].cpu().tolist() == plain
    assert st["accepted"] < st["drafted"], st

    first = h.prefill([2], tok, [SPEC_PROMPT], 4, dory.LAST_LOOP)
    out, out_len, st = h.spec_decode([2], first, 1, 4, 4, dory.LAST_LOOP, SPEC_NEW - 1)
    h.synchronize()
    spec = [int(first[0])] + out[0].cpu().tolist()
    ref = env["jobs"]["spec"].result()
    assert spec == list(ref["tokens"]), (spec, list(ref["tokens"]))
    assert st["accepted"] == sum(ref["accepted_per_step"]), (st, ref["accepted_per_step"])
    assert st["accepted"] < st["drafted"], st
    print(f"spec last_loop: {st}, oracle accepted per step {ref['accepted_per_step']}")
