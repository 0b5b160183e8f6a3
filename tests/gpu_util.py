"""Helpers shared by the GPU tests: drive the C ABI and compare with the oracle."""
import numpy as np
import torch

import looped_ngpt_lm_b200 as dory
import oracle as O
import synth

MODES = {"last_loop": (O.LAST_LOOP, dory.LAST_LOOP), "per_loop": (O.PER_LOOP, dory.PER_LOOP)}

# bf16 configurations must keep the logits within relative L2 2e-2 of the
# oracle's.  Spread evenly, that error is about 2e-2 * rms(logits) per logit;
# two logits moving that far in opposite directions can swap only when the
# oracle's margin between them is below twice that.  A greedy choice that
# differs from the oracle's argmax is accepted only under that margin.  The
# threshold is fixed by the stated tolerance and the oracle's own logits; it
# never grows with the error the run under test happens to make.
BF16_LOGITS_TOL = 2e-2
BF16_TIE_FRAC = 2 * BF16_LOGITS_TOL


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


def top2_margin(row):
    """Oracle logit of the best token minus that of the runner-up."""
    part = np.partition(np.asarray(row, dtype=np.float64), -2)
    return float(part[-1] - part[-2])


def check_tokens(gpu_toks, ora_logits, tol=None, rel=None):
    """Every GPU choice must be the oracle's argmax, except at a near tie:
    the oracle's logit of its best token exceeds that of the GPU's choice by
    at most `tol` (absolute) or `rel` * rms(oracle logits of that step).
    Returns {"exempt": steps excused as near ties, "min_margin": smallest
    top-2 margin of the oracle over the steps, "threshold": largest
    threshold used}; the caller may assert on them."""
    assert (tol is None) != (rel is None)
    exempt, min_margin, thr_max = 0, float("inf"), 0.0
    for i, t in enumerate(gpu_toks):
        row = np.asarray(ora_logits[i], dtype=np.float64)
        thr = tol if tol is not None else rel * float(np.sqrt(np.mean(row * row)))
        thr_max = max(thr_max, thr)
        min_margin = min(min_margin, top2_margin(row))
        best = int(np.argmax(row))
        if int(t) == best:
            continue
        gap = float(row[best] - row[int(t)])
        assert gap <= thr, (f"step {i}: gpu chose {int(t)}, oracle {best}; oracle margin {gap:.3e} "
                            f"above the near-tie threshold {thr:.3e}")
        exempt += 1
    return {"exempt": exempt, "min_margin": min_margin, "threshold": thr_max}


def check_bf16_tokens(gpu_toks, ora_logits):
    """check_tokens at the bf16 near-tie threshold."""
    return check_tokens(gpu_toks, ora_logits, rel=BF16_TIE_FRAC)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def cosine_rows(a, b):
    return np.sum(a * b, -1) / (np.linalg.norm(a, axis=-1) * np.linalg.norm(b, axis=-1))
