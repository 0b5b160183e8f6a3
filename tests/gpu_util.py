"""Helpers shared by the GPU tests: drive the C ABI and compare with the oracle."""
import numpy as np
import torch

import looped_ngpt_lm_b200 as dory
import oracle as O
import synth

MODES = {"last_loop": (O.LAST_LOOP, dory.LAST_LOOP), "per_loop": (O.PER_LOOP, dory.PER_LOOP)}


def make(shape, seed=0, alloc="per_loop", **cap):
    w = synth.make_weights(shape, seed)
    dw = dory.DeviceWeights(shape, w)
    cfg = dory.make_config(shape, **cap)
    h = dory.Handle(cfg, dw, dory.MODES[alloc])
    return w, dw, h


def gpu_generate(h, prompt, n_new, k, mode, seq=0):
    """Prefill + greedy decode through the C ABI; returns tokens and logits
    (numpy) of each of the n_new steps."""
    V = h.cfg.vocab
    tok = torch.tensor(np.asarray(prompt), dtype=torch.int32, device="cuda")
    lg = torch.empty((1, V), dtype=torch.float32, device="cuda")
    nxt = h.prefill([seq], tok, [len(prompt)], k, mode, logits=lg)
    toks, logits = [int(nxt[0])], [lg[0].cpu().numpy().copy()]
    for _ in range(1, n_new):
        nxt = h.decode_step([seq], nxt, k, mode, logits=lg)
        toks.append(int(nxt[0]))
        logits.append(lg[0].cpu().numpy().copy())
    h.synchronize()
    return np.array(toks), np.stack(logits)


def check_tokens(gpu_toks, ora_logits, tol):
    """Every GPU choice must be the oracle's argmax, unless the oracle's best
    and the GPU's choice are within `tol` (a near tie both sides may break
    either way).  Returns the number of near-tie steps."""
    ties = 0
    for i, t in enumerate(gpu_toks):
        best = int(np.argmax(ora_logits[i]))
        if t == best:
            continue
        gap = ora_logits[i][best] - ora_logits[i][t]
        assert gap <= tol, f"step {i}: gpu chose {t}, oracle {best}, gap {gap}"
        ties += 1
    return ties


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def cosine_rows(a, b):
    return np.sum(a * b, -1) / (np.linalg.norm(a, axis=-1) * np.linalg.norm(b, axis=-1))
