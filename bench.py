#!/usr/bin/env python
"""Benchmark of the looped nGPT hot path on B200.

Workload: the 4B-shaped model (d=2560, vocab 131072, 20 q-heads x 128, 4 KV
heads, SwiGLU 10240, 16 + 40 + 16 physical layers, window 4096) in bf16 with
seeded random weights; batch 1, a 2560-token uniform-random prompt, then
greedy decode at k=2 with the last-loop KV cache.  One "step" is one decode
step (every row of the hot path: embed, the input block, k passes of the
recurrent block with re-injection, the output block, the LM head and the
argmax).  The decode steps stream ~11.2 GB of weights each, far above the
126 MB L2, so no flush is needed between steps.

Default: 1 GPU.  Under torchrun each rank runs an independent replica (the
path shards over sequences with no exchange), so scaling is weak; the time is
the max over ranks.  --impl reference times the oracle on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s at k=1/2/4 (last-loop KV), % HBM roofline; prefill TFLOP/s"


class Ranks:
    """Rank plumbing: one process per GPU under torchrun (RANK, WORLD_SIZE,
    LOCAL_RANK, MASTER_* from the environment), process group over NCCL;
    backend "gloo" keeps every tensor on the host (used by the CPU tests).
    Every rank takes the same collective steps in the same order."""

    def __init__(self, backend="nccl", timeout_s=300):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.dist = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.dist = dist

    def _sync(self):
        if self.backend != "gloo":
            import torch
            torch.cuda.synchronize()

    def barrier(self):
        """Device work finished here and on every rank."""
        self._sync()
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x: float) -> float:
        """Maximum of x over the ranks (device times: the slowest rank)."""
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device="cpu" if self.backend == "gloo" else "cuda")
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def job_throughput(world: int, units_per_rank: int, max_ms: float) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1e3)


def peaks():
    try:
        p = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 1400.0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- algorithmic work
# DRAM bytes (read + write) per decode-GEMM launch from one ncu capture of the
# decode GEMMs of a 2+2+2-layer model of the 4B width (every launch's counters,
# weighted by the full step's launch counts: 56 each of QKV, O, gate-up, down
# and one LM head).  Each launch's count includes the 8 MiB of the next
# weights it prefetches into L2 (the look-ahead), which ncu's flush between
# launches makes the next launch read again.
GEMM_TRAFFIC_PER_LAUNCH = 58.40e6


def weight_bytes(shape, k):
    """Weight bytes one decode step streams at loop count k (bf16)."""
    d, q, kv, f = shape.d_model, shape.q_dim, shape.kv_dim, shape.d_ff
    attn = (q + 2 * kv) * d + d * q
    mlp = 3 * f * d
    def block(n):
        return (n // 2) * attn + (n - n // 2) * mlp
    per = block(shape.n_in) + k * block(shape.n_rec) + block(shape.n_out)
    return 2 * (per + shape.vocab * d + d)  # + LM head + one embedding row


def kv_read_bytes(shape, k, ctx):
    """KV bytes one decode step at context ctx reads (all attention
    applications; each key is K+V of every KV head)."""
    per_key = 2 * shape.kv_dim * 2
    tot = 0
    j = 0
    for l in range(shape.n_layers):
        if l % 2:
            continue
        full = (j % shape.full_every) == shape.full_phase
        j += 1
        rec = shape.n_in <= l < shape.n_in + shape.n_rec
        keys = ctx if full else min(ctx, shape.swa_window)
        tot += (k if rec else 1) * keys * per_key
    return tot


def proj_flops(shape, k, tokens):
    return 2 * tokens * (weight_bytes(shape, k) / 2 - shape.vocab * shape.d_model - shape.d_model)


def attn_flops_prefill(shape, k, T):
    pairs_full = T * (T + 1) // 2
    W = shape.swa_window
    pairs_swa = sum(min(p + 1, W) for p in range(T))
    per = 4 * shape.n_heads * shape.head_dim
    tot = 0
    j = 0
    for l in range(shape.n_layers):
        if l % 2:
            continue
        full = (j % shape.full_every) == shape.full_phase
        j += 1
        rec = shape.n_in <= l < shape.n_in + shape.n_rec
        tot += (k if rec else 1) * (pairs_full if full else pairs_swa) * per
    return tot


# ---------------------------------------------------------------- clocks
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = [r.split(", ") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows if len(r) >= 9 for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle
def sweep_modes(dory, torch, shape, dw, args, prompt_len=128, n_new=1024):
    """Batch 1, 128-token prompt, greedy decode at k = 1/2/4 in both cache
    modes: tokens/s, KV bytes per token, and how far last_loop logits drift
    from per_loop logits on the same tokens (teacher-forced over all n_new
    steps: the last_loop run's logits are kept on the device, then the
    per_loop replay is compared step by step)."""
    import synth
    cfg = dory.make_config(shape, max_batch=2, max_seq=prompt_len + n_new + 8, k_max=4, gamma_max=4,
                           max_chunk=prompt_len)
    h = dory.Handle(cfg, dw, dory.PER_LOOP)
    prompt = torch.tensor(synth.make_prompt(2, prompt_len, shape.vocab), dtype=torch.int32, device="cuda")
    out = {}
    for k in (1, 2, 4):
        toks = {}
        for mode in ("last_loop", "per_loop"):
            md = dory.MODES[mode]
            seq = 0 if mode == "last_loop" else 1
            h.reset(seq)
            t = h.prefill([seq], prompt, [prompt_len], k, md)
            bufs = [torch.empty(1, dtype=torch.int32, device="cuda") for _ in range(2)]
            for i in range(3):
                t = h.decode_step([seq], t, k, md, next_tokens=bufs[i % 2])
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            n = n_new - 4
            for i in range(n):
                t = h.decode_step([seq], t, k, md, next_tokens=bufs[i % 2])
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / n
            ctx = h.seq_len(seq)
            out[f"k{k}_{mode}"] = {"tokens_per_s": round(1e3 / ms, 2),
                                   "kv_bytes_per_token": round(h.kv_bytes(k, md, ctx) / ctx, 1), "ctx": ctx}
        # logits drift: replay one greedy last_loop run in both modes on the same tokens
        L = torch.empty((1, shape.vocab), device="cuda")
        ref = torch.empty((n_new, shape.vocab), device="cuda")
        tok_seq = torch.empty(n_new, dtype=torch.int32, device="cuda")
        drift = torch.empty(n_new, device="cuda")
        agree = torch.empty(n_new, device="cuda")
        for mode in ("last_loop", "per_loop"):
            md = dory.MODES[mode]
            seq = 0 if mode == "last_loop" else 1
            h.reset(seq)
            t = h.prefill([seq], prompt, [prompt_len], k, md, logits=L)
            for i in range(n_new):
                if mode == "last_loop":
                    ref[i] = L[0]
                    tok_seq[i] = t[0]
                else:
                    drift[i] = (L[0] - ref[i]).norm() / ref[i].norm()
                    agree[i] = (L[0].argmax() == ref[i].argmax()).float()
                if i + 1 < n_new:
                    t = h.decode_step([seq], tok_seq[i:i + 1], k, md, logits=L)
        drift, agree = drift.cpu(), float(agree.mean())
        out[f"k{k}_logits_drift"] = {"rel_l2_max": round(float(drift.max()), 5), "rel_l2_mean": round(float(drift.mean()), 5),
                                     "argmax_agreement": round(agree, 4), "steps": n_new}
    h.close()
    return out


def spec_leg(dory, torch, shape, dw, args, prompt_len=512, n_new=512, gamma=4):
    """Self-speculative decoding (draft k=1, verify k=4, gamma=4, last_loop)
    at batch 1, 4 and 16 against plain k=4 greedy decoding of the same
    prompts: accepted draft tokens per verify step, output tokens/s, speed-up,
    and agreement with the plain k=4 tokens."""
    import synth
    res = {}
    for B in (1, 4, 16):
        cfg = dory.make_config(shape, max_batch=2 * B, max_seq=prompt_len + n_new + 2 * gamma + 8, k_max=4,
                               gamma_max=gamma, max_chunk=2 * B * prompt_len)
        h = dory.Handle(cfg, dw, dory.LAST_LOOP)
        prompts = [synth.make_prompt(100 + b, prompt_len, shape.vocab) for b in range(B)]
        tok = torch.tensor(np.concatenate(prompts), dtype=torch.int32, device="cuda")
        md = dory.LAST_LOOP
        # plain k=4
        ids = list(range(B))
        first = h.prefill(ids, tok, [prompt_len] * B, 4, md)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t = first
        plain = [t.clone()]
        a.record()
        for i in range(n_new - 1):
            t = h.decode_step(ids, t, 4, md)
            plain.append(t.clone())
        b.record()
        torch.cuda.synchronize()
        plain_ms = a.elapsed_time(b)
        plain_tok = torch.stack(plain, 1).cpu()
        # speculative on other sequence slots
        sids = list(range(B, 2 * B))
        first = h.prefill(sids, tok, [prompt_len] * B, 4, md)
        torch.cuda.synchronize()
        a.record()
        out, out_len, st = h.spec_decode(sids, first, 1, 4, gamma, md, n_new - 1)
        b.record()
        torch.cuda.synchronize()
        spec_ms = a.elapsed_time(b)
        spec_tok = torch.cat([first.cpu()[:, None], out.cpu()], 1)
        agree = (spec_tok == plain_tok).float().mean().item()
        res[f"batch{B}"] = {
            "accepted_per_verify_step": round(st["accepted"] / max(st["steps"] * B, 1), 3),
            "tokens_per_verify_step": round((B * (n_new - 1)) / max(st["steps"] * B, 1), 3),
            "spec_tokens_per_s": round(B * (n_new - 1) / (spec_ms / 1e3), 1),
            "plain_k4_tokens_per_s": round(B * (n_new - 1) / (plain_ms / 1e3), 1),
            "speedup_vs_plain_k4": round(plain_ms / spec_ms, 3),
            "token_agreement_with_plain_k4": round(agree, 4),
        }
        h.close()
    res["workload"] = f"prompt {prompt_len}, {n_new} output tokens, gamma {gamma}, last_loop, greedy"
    return res


def mixed_leg(dory, torch, shape, dw, args, prompt_len=512, steps=32):
    """Mixed-k batched decode at batch 16 (k = 4 for 4 sequences, 2 for 4, 1
    for 8; last_loop): one dory_decode_step_mixed call per step, against the
    same sequences decoded as three per-k groups (three graph-replayed
    decode_step calls per step)."""
    import synth
    ks = [4] * 4 + [2] * 4 + [1] * 8
    B = len(ks)
    cfg = dory.make_config(shape, max_batch=2 * B, max_seq=prompt_len + 2 * steps + 16, k_max=4, gamma_max=4,
                           max_chunk=B * prompt_len)
    h = dory.Handle(cfg, dw, dory.LAST_LOOP)
    md = dory.LAST_LOOP
    prompts = [synth.make_prompt(200 + b, prompt_len, shape.vocab) for b in range(B)]
    tok = torch.tensor(np.concatenate(prompts), dtype=torch.int32, device="cuda")
    ev = lambda: torch.cuda.Event(enable_timing=True)
    # mixed: sequences 0..B-1
    ids = list(range(B))
    t = h.prefill(ids, tok, [prompt_len] * B, 4, md)
    for _ in range(3):
        t = h.decode_step_mixed(ids, t, ks, md)
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    for _ in range(steps):
        t = h.decode_step_mixed(ids, t, ks, md)
    b.record()
    torch.cuda.synchronize()
    mixed_ms = a.elapsed_time(b) / steps
    # grouped: sequences B..2B-1, one call per k group
    groups = [(4, list(range(B, B + 4))), (2, list(range(B + 4, B + 8))), (1, list(range(B + 8, 2 * B)))]
    t2 = h.prefill(list(range(B, 2 * B)), tok, [prompt_len] * B, 4, md)
    cur = {k: t2[(g[0] - B):(g[0] - B) + len(g)].clone() for k, g in groups}
    for _ in range(3):
        for k, g in groups:
            cur[k] = h.decode_step(g, cur[k], k, md)
    torch.cuda.synchronize()
    a.record()
    for _ in range(steps):
        for k, g in groups:
            cur[k] = h.decode_step(g, cur[k], k, md)
    b.record()
    torch.cuda.synchronize()
    grouped_ms = a.elapsed_time(b) / steps
    h.close()
    return {"ks": ks, "mixed_tokens_per_s": round(B * 1e3 / mixed_ms, 1), "mixed_ms_per_step": round(mixed_ms, 3),
            "grouped_tokens_per_s": round(B * 1e3 / grouped_ms, 1), "grouped_ms_per_step": round(grouped_ms, 3),
            "speedup_vs_grouped": round(grouped_ms / mixed_ms, 3),
            "workload": f"batch {B}, prompt {prompt_len}, {steps} steps, last_loop; mixed: one call per step "
                        f"(eager launches); grouped: one graph-replayed call per k group"}


def sampling_leg(dory, torch, h, tok, args, mode, steps=64):
    """Batch-1 decode at k = args.k with top-p sampling (temperature 1.0,
    top-p 0.95, the released model's settings) against greedy choice, on the
    bench's own handle and sequence."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    out = {}
    bufs = [torch.empty(1, dtype=torch.int32, device="cuda") for _ in range(2)]
    for name, T in (("greedy", 0.0), ("top_p_0.95_T_1.0", 1.0)):
        h.set_sampling(T, 0.95 if T > 0 else 1.0, 1234)
        for i in range(3):
            tok = h.decode_step([0], tok, args.k, mode, next_tokens=bufs[i % 2])
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        for i in range(steps):
            tok = h.decode_step([0], tok, args.k, mode, next_tokens=bufs[i % 2])
        b.record()
        torch.cuda.synchronize()
        out[name] = {"tokens_per_s": round(steps * 1e3 / a.elapsed_time(b), 2),
                     "ms_per_step": round(a.elapsed_time(b) / steps, 4)}
    h.set_sampling(0.0, 1.0, 0)
    out["sampler_ms_per_step"] = round(out["top_p_0.95_T_1.0"]["ms_per_step"] - out["greedy"]["ms_per_step"], 4)
    return out, tok


def lowbit_leg(dory, torch, shape, dw, args, mode, bf16_sweep, fmt, steps=32):
    """Batch-1 decode with low-bit weight copies made on the GPU from the
    bench's bf16 weights, at k = 1, 2, 4 on a handle of its own: prefill reads
    the exact bf16 dequantisation, decode GEMMs the copies.  fmt "mxfp8":
    E4M3 codes with one E8M0 scale per 32 weights, timed with the CUDA-core
    GEMV (option 1), the same GEMV fed by bulk copies (option 4) and the
    TMA-fed tcgen05 GEMM (option 3); fmt "nvfp4":
    E2M1 codes, one E4M3 scale per 16 weights and a tensor scale, on the
    tcgen05 GEMM.  Reports tokens/s, the speed-up over the bf16 k sweep at
    the same context, and the low-bit GEMMs' HBM rate from a profiled pass."""
    import synth
    ev = lambda: torch.cuda.Event(enable_timing=True)
    wq = dory.MxWeights(dw) if fmt == "mxfp8" else dory.NvWeights(dw)
    n_impl = 3 if fmt == "mxfp8" else 1
    # every implementation decodes (3 warm-up + steps) tokens at each k, then 2 profiled steps
    cfg = dory.make_config(shape, max_batch=1, max_seq=args.prompt + n_impl * (3 * (steps + 3) + 2) + 64, k_max=4,
                           gamma_max=4, max_chunk=args.prompt)
    h = dory.Handle(cfg, wq.dequantised, dory.LAST_LOOP if args.mode == "last_loop" else dory.PER_LOOP)
    (h.attach_mxfp8 if fmt == "mxfp8" else h.attach_nvfp4)(wq)
    prompt = torch.tensor(synth.make_prompt(1, args.prompt, shape.vocab), dtype=torch.int32, device="cuda")
    tok = h.prefill([0], prompt, [args.prompt], args.k, mode)
    bufs = [torch.empty(1, dtype=torch.int32, device="cuda") for _ in range(2)]
    out = {}
    impls = (((1, "cuda_core_gemv"), (4, "cuda_core_gemv_bulk_fed"), (3, "tcgen05_gemm")) if fmt == "mxfp8"
             else ((0, "tcgen05_gemm"),))
    hbm = peaks()[0]
    for impl, label in impls:
        if fmt == "mxfp8":
            h.set_option(dory.OPT_MX_GEMV, impl)
        res = {}
        for kk in (1, 2, 4):
            if args.mode == "per_loop" and kk != args.k:
                continue
            for i in range(3):
                tok = h.decode_step([0], tok, kk, mode, next_tokens=bufs[i % 2])
            torch.cuda.synchronize()
            a, b = ev(), ev()
            a.record()
            for i in range(steps):
                tok = h.decode_step([0], tok, kk, mode, next_tokens=bufs[i % 2])
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
            r = {"tokens_per_s": round(1e3 / ms, 2), "ms_per_token": round(ms, 4), "ctx": h.seq_len(0)}
            ref = (bf16_sweep or {}).get(f"k{kk}")
            if ref:
                r["speedup_vs_bf16"] = round(r["tokens_per_s"] / ref["tokens_per_s"], 3)
            res[f"k{kk}"] = r
        # the low-bit GEMMs' own time: CUDA events around every launch of two steps
        h.profile_reset()
        h.set_option(dory.OPT_PROFILE, 1)
        for i in range(2):
            tok = h.decode_step([0], tok, args.k, mode, next_tokens=bufs[i % 2])
        prof = h.profile_read()
        h.set_option(dory.OPT_PROFILE, 0)
        g = {n: v for n, v in prof.items() if n.startswith("gemm")}
        g_ms = sum(v["ms"] for v in g.values())
        g_bytes = sum(v["bytes"] for v in g.values())
        g_launch = sum(v["launches"] for v in g.values())
        tot_ms = sum(v["ms"] for v in prof.values())
        achieved = g_bytes / (g_ms / 1e3) / 1e9 if g_ms > 0 else 0.0
        res["gemm_hbm"] = {"achieved_GBs": round(achieved, 1), "frac": round(achieved / hbm, 4),
                           "avg_launch_us": round(1e3 * g_ms / max(g_launch, 1), 2),
                           "share_of_profiled_step": round(g_ms / tot_ms, 4) if tot_ms else None}
        out[label] = res
    out["weight_bytes"] = wq.nbytes()
    out["workload"] = (f"batch 1, prompt {args.prompt}, {steps} timed steps per k, {args.mode}; {fmt} copies of "
                       f"every projection and the LM head (embedding bf16)")
    out["pages_ratio"] = ("over BF16 at batch 1 on a DGX Spark: MXFP8 1.69x / NVFP4 2.17x (in 2560 / out 300), "
                          "MXFP8 1.84x / NVFP4 2.44x (in 128 / out 1024)")
    h.close()
    del wq
    torch.cuda.empty_cache()
    return out


def gemm_stream(dory, torch, shape, dw, k, reps=5):
    """The decode step's projection GEMMs alone, in the step's order and
    shapes (one token row; the weights of the input block, k passes over the
    recurrent block, the output block and the LM head), recorded into one
    CUDA graph and replayed back to back: the GEMM kernel's own streaming
    rate inside a step-length launch sequence with PDL.  Returns (ms per
    pass, launches per pass, algorithmic bytes per pass)."""
    mats = []
    def layer(l):
        if dw.qkv[l] is not None:
            mats.extend([dw.qkv[l], dw.o[l]])
        else:
            mats.extend([dw.gu[l], dw.down[l]])
    for l in range(shape.n_in):
        layer(l)
    for _ in range(k):
        for l in range(shape.n_in, shape.n_in + shape.n_rec):
            layer(l)
    for l in range(shape.n_in + shape.n_rec, shape.n_layers):
        layer(l)
    mats.append(dw.tensors["lm_head"])
    Ks = sorted({int(w.shape[1]) for w in mats})
    X = {K: torch.randn((1, K), device="cuda").div_(K ** 0.5).to(torch.bfloat16) for K in Ks}
    Y = torch.empty((8, 1, max(int(w.shape[0]) for w in mats)), dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    splits = [dory.gemm_bf16_into(X[int(w.shape[1])], w, Y, 1, True, 2, stream=side) for w in mats]
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for w in mats:
            dory.gemm_bf16_into(X[int(w.shape[1])], w, Y, 1, True, 2, stream=side)
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        graph.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    by = sum(int(w.shape[0]) * int(w.shape[1]) * 2 + int(w.shape[1]) * 2 + s * int(w.shape[0]) * 4
             for w, s in zip(mats, splits))
    del graph
    return ms, len(mats), by


def leg(fn, *a):
    """One auxiliary measurement.  An exception is recorded in the JSON line
    (as {"error": ...}) instead of costing the headline."""
    try:
        return fn(*a)
    except Exception as e:  # noqa: BLE001 - any failure of an extra leg is reported, not raised
        return {"error": f"{type(e).__name__}: {e}"[:400]}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(i.get("num_threads", 1) for i in threadpool_info()) or (os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def host_mem_gb():
    try:
        for line in open("/proc/meminfo"):
            if line.startswith("MemAvailable"):
                return int(line.split()[1]) / 1e6
    except Exception:
        pass
    return 0.0


def oracle_decode_rate(shape, weights, k, mode, prompt_len, steps, seed=1, model=None):
    """Oracle (float32 on the host) decode tokens/s on a bounded sample:
    prefill a short prompt, then time `steps` greedy decode steps."""
    import oracle as O
    m = model if model is not None else O.Model(shape, weights, dtype=np.float32)
    prompt = __import__("synth").make_prompt(seed, prompt_len, shape.vocab)
    cache = O.Cache(m, prompt_len + steps + 2)
    lg = O.forward_chunk(m, cache, prompt, k, mode)
    tok = int(np.argmax(lg[-1]))
    t0 = time.perf_counter()
    for _ in range(steps):
        lg = O.forward_chunk(m, cache, [tok], k, mode)
        tok = int(np.argmax(lg[-1]))
    dt = time.perf_counter() - t0
    return steps / dt, dt


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--gemm-impl", dest="gemm_variant", type=int, default=2,
                    help="--kernel gemm: 2 tcgen05 (default stages), 3 tcgen05 one sub-tile per stage, "
                         "4 tcgen05 with packed weights, 1 SIMT")
    ap.add_argument("--prompt", type=int, default=2560)
    ap.add_argument("--k", type=int, default=2)
    ap.add_argument("--mode", default="last_loop", choices=["last_loop", "per_loop"])
    ap.add_argument("--no-aux", action="store_true", help="skip the k sweep, e2e and CPU baseline legs")
    ap.add_argument("--profile-steps", type=int, default=3)
    ap.add_argument("--kernel", default=None, choices=["gemm", "mxgemv", "nvgemm"],
                    help="time one kernel alone instead of the decode step (prints its own JSON line)")
    ap.add_argument("--shape", default="qkv,o,gate_up,down,lm_head", help="GEMM shapes for --kernel gemm / mxgemv")
    ap.add_argument("--mx-impl", dest="mx_impl", type=int, default=1,
                    help="--kernel mxgemv: 1 CUDA cores (default), 2 mma.sync, 3 TMA-fed tcgen05 (one slice), "
                         "4 CUDA cores fed by bulk copies")
    ap.add_argument("--m", type=int, default=1, help="token rows for --kernel gemm")
    ap.add_argument("--l2-lookahead-mb", dest="l2_mb", type=int, default=None,
                    help="bytes of upcoming weights each decode GEMM prefetches into L2 (MiB; 0 = off; "
                         "default: the library's)")
    ap.add_argument("--attn-lookahead-mb", dest="attn_mb", type=int, default=None,
                    help="bytes of upcoming weights each decode attention launch prefetches into L2 (MiB)")
    ap.add_argument("--fused-rows", dest="fused_rows", type=int, default=None,
                    help="operand stages for decode passes of at most this many rows (0 = off; default: the "
                         "library's)")
    ap.add_argument("--l2-own", dest="l2_own", type=int, default=None,
                    help="own weight tiles each decode GEMM CTA prefetches into L2 before its wait (DORY_OPT_L2_OWN)")
    ap.add_argument("--prefill-tc", dest="prefill_tc", type=int, default=None,
                    help="prefill attention kernel (DORY_OPT_PREFILL_TC; default: the library's)")
    ap.add_argument("--attn-cluster", dest="attn_cluster", type=int, default=None,
                    help="decode attention cluster size (4, 8, 16; 1 = chosen from the batch; 0 = none)")
    ap.add_argument("--batched", action="store_true",
                    help="run the batched workload instead (--batch sequences of --prompt-batched tokens, "
                         "chunked prefill, then --steps decode steps) and print its own JSON line")
    ap.add_argument("--batch", type=int, default=64)
    ap.add_argument("--prompt-batched", dest="prompt_batched", type=int, default=32768)
    ap.add_argument("--chunk", type=int, default=8192, help="prefill chunk of the batched workload")
    ap.add_argument("--layers", default=None,
                    help="I,R,O physical layers (a narrower model of the same width, for small profiling captures)")
    args = ap.parse_args()
    if args.batched:
        batched_leg(args)
        return
    if args.kernel == "gemm":
        gemm_probe(args)
        return
    if args.kernel in ("mxgemv", "nvgemm"):
        mx_gemv_probe(args)
        return
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    import synth
    shape = synth.DORY_4B
    workload = f"dory4b_bf16_batch1_prompt{args.prompt}_decode_k{args.k}_{args.mode}"
    if args.layers:
        n_in, n_rec, n_out = (int(v) for v in args.layers.split(","))
        shape = shape.with_(name="dory4b_cut", n_in=n_in, n_rec=n_rec, n_out=n_out)
        workload += f"_layers{n_in}-{n_rec}-{n_out}"
    hbm, tc, tc_sus, peak_src = peaks()

    if args.impl == "reference":
        if rank != 0:
            return
        run_reference(args, shape, workload)
        return

    import torch
    import looped_ngpt_lm_b200 as dory

    torch.cuda.set_device(local)
    ranks = Ranks("nccl")

    w_np = synth.make_weights(shape, 1)
    dw = dory.DeviceWeights(shape, w_np)
    if rank != 0 or args.no_aux:
        del w_np
        w_np = None
    max_seq = args.prompt + args.warmup + args.steps + args.profile_steps + 512
    cfg = dory.make_config(shape, max_batch=1, max_seq=max_seq, k_max=4, gamma_max=4, max_chunk=args.prompt)
    h = dory.Handle(cfg, dw, dory.LAST_LOOP if args.mode == "last_loop" else dory.PER_LOOP)
    if args.l2_mb is not None:
        h.set_option(dory.OPT_L2_LOOKAHEAD, args.l2_mb << 20)
    if args.attn_mb is not None:
        h.set_option(dory.OPT_ATTN_LOOKAHEAD, args.attn_mb << 20)
    if args.fused_rows is not None:
        h.set_option(dory.OPT_FUSED_OPERANDS, args.fused_rows)
    if args.attn_cluster is not None:
        h.set_option(dory.OPT_ATTN_CLUSTER, args.attn_cluster)
    if args.prefill_tc is not None:
        h.set_option(dory.OPT_PREFILL_TC, args.prefill_tc)
    if args.l2_own is not None:
        h.set_option(dory.OPT_L2_OWN, args.l2_own)
    mode = dory.MODES[args.mode]
    stream = torch.cuda.current_stream()
    prompt = torch.tensor(synth.make_prompt(1, args.prompt, shape.vocab), dtype=torch.int32, device="cuda")

    barrier, max_over_ranks = ranks.barrier, ranks.max

    # ---- prefill (timed on its own: projection + attention TFLOP/s)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    pre_ms = []
    for rep in range(2):
        h.reset()
        barrier()
        a, b = ev(), ev()
        a.record(stream)
        first = h.prefill([0], prompt, [args.prompt], args.k, mode)
        b.record(stream)
        torch.cuda.synchronize()
        pre_ms.append(a.elapsed_time(b))
    h.synchronize()
    pre_ms = max_over_ranks(min(pre_ms))
    pf = proj_flops(shape, args.k, args.prompt)
    af = attn_flops_prefill(shape, args.k, args.prompt)
    # one more prefill with CUDA events around every launch: the projection
    # GEMMs' and the attention kernel's own time
    h.reset()
    h.profile_reset()
    h.set_option(dory.OPT_PROFILE, 1)
    first = h.prefill([0], prompt, [args.prompt], args.k, mode)
    torch.cuda.synchronize()
    pprof = h.profile_read()
    h.set_option(dory.OPT_PROFILE, 0)
    h.profile_reset()
    proj_ms = sum(v["ms"] for n, v in pprof.items() if n.startswith("gemm") and n != "gemm_lm_head")
    attn_ms = sum(v["ms"] for n, v in pprof.items() if n.startswith("attn"))

    # ---- decode: warm-up, then exactly K timed steps
    bufs = [torch.empty(1, dtype=torch.int32, device="cuda") for _ in range(2)]
    tok = first
    for i in range(args.warmup):
        tok = h.decode_step([0], tok, args.k, mode, next_tokens=bufs[i % 2])
    barrier()
    clocks = Clocks(local)
    clocks.start()
    t0, t1 = ev(), ev()
    t0.record(stream)
    for i in range(args.steps):
        tok = h.decode_step([0], tok, args.k, mode, next_tokens=bufs[i % 2])
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    h.synchronize()
    dec_ms = max_over_ranks(t0.elapsed_time(t1))
    ms_step = dec_ms / args.steps
    value = job_throughput(world, args.steps, dec_ms)
    ctx_mid = args.prompt + args.warmup + args.steps // 2
    step_bytes = weight_bytes(shape, args.k) + kv_read_bytes(shape, args.k, ctx_mid)

    # ---- per-kernel timing (CUDA events around every launch, same stream)
    h.profile_reset()
    h.set_option(dory.OPT_PROFILE, 1)
    for i in range(args.profile_steps):
        tok = h.decode_step([0], tok, args.k, mode, next_tokens=bufs[i % 2])
    prof = h.profile_read()
    h.set_option(dory.OPT_PROFILE, 0)
    launches_per_step = sum(v["launches"] for v in prof.values()) / args.profile_steps
    gemm = {n: v for n, v in prof.items() if n.startswith("gemm")}
    g_ms = sum(v["ms"] for v in gemm.values())
    g_bytes = sum(v["bytes"] for v in gemm.values())
    g_launch = sum(v["launches"] for v in gemm.values())
    tot_ms = sum(v["ms"] for v in prof.values())
    # the dominant kernel (the projection GEMM) timed live: the step's GEMM
    # sequence replayed as one graph on the same stream, CUDA events around it
    gs_ms, gs_n, gs_bytes = gemm_stream(dory, torch, shape, dw, args.k)
    achieved = gs_bytes / (gs_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": "k_gemm_tc (decode projections + LM head, one token row)",
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "peak_source": peak_src,
                "traffic": GEMM_TRAFFIC_PER_LAUNCH if (shape.name == "dory4b" and args.k == 2) else None,
                "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum per decode GEMM launch "
                                "(algorithmic bytes + the 8 MiB L2 look-ahead of the next weights)",
                "bytes_per_launch": round(gs_bytes / gs_n),
                "avg_launch_us": round(1e3 * gs_ms / gs_n, 2), "launches_per_step": gs_n,
                "gemm_ms_per_step": round(gs_ms, 4), "share_of_step": round(gs_ms / ms_step, 4),
                "method": "the step's GEMM sequence (same weights, order, shapes and split choice) recorded into one "
                          "CUDA graph and replayed; CUDA events on its stream; bytes = weights + operand + "
                          "split-K partial sums per launch",
                "event_timed_profile": {"achieved": round(g_bytes / (g_ms / 1e3) / 1e9, 1) if g_ms > 0 else None,
                                        "avg_launch_us": round(1e3 * g_ms / max(g_launch, 1), 2),
                                        "share_of_profiled_step": round(g_ms / tot_ms, 4) if tot_ms else None}}
    kernel_share = {n: round(v["ms"] / tot_ms, 4) for n, v in sorted(prof.items(), key=lambda kv: -kv[1]["ms"])}

    aux = {}
    e2e = None
    cpu = None
    if not args.no_aux and world == 1:
        # ---- k sweep (short runs, same context)
        sweep = {}
        for kk in (1, 2, 4):
            n = 32
            a, b = ev(), ev()
            for i in range(3):
                tok = h.decode_step([0], tok, kk, mode, next_tokens=bufs[i % 2])
            torch.cuda.synchronize()
            a.record(stream)
            for i in range(n):
                tok = h.decode_step([0], tok, kk, mode, next_tokens=bufs[i % 2])
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / n
            ctx = h.seq_len(0)
            by = weight_bytes(shape, kk) + kv_read_bytes(shape, kk, ctx)
            sweep[f"k{kk}"] = {"tokens_per_s": round(1e3 / ms, 2), "ms_per_token": round(ms, 4),
                               "hbm_frac_of_peak": round(by / (ms / 1e3) / 1e9 / hbm, 4),
                               "bytes_per_token": by, "ctx": ctx}
        aux["decode_k_sweep_last_loop" if args.mode == "last_loop" else "decode_k_sweep"] = sweep
        r = leg(sampling_leg, dory, torch, h, tok, args, mode)
        if isinstance(r, tuple):
            aux["sampling"], tok = r
        else:
            aux["sampling"] = r
        aux["mxfp8_decode"] = leg(lowbit_leg, dory, torch, shape, dw, args, mode, sweep, "mxfp8")
        aux["nvfp4_decode"] = leg(lowbit_leg, dory, torch, shape, dw, args, mode, sweep, "nvfp4")
        # ---- end to end: every step copies its input token from pinned host
        # memory and reads the chosen token back, through the public API
        pin_in = torch.empty(1, dtype=torch.int32).pin_memory()
        pin_out = torch.empty(1, dtype=torch.int32).pin_memory()
        d_in = torch.empty(1, dtype=torch.int32, device="cuda")
        pin_in[0] = int(tok[0])
        n = min(args.steps, 100)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record(stream)
        for i in range(n):
            d_in.copy_(pin_in, non_blocking=True)
            out = h.decode_step([0], d_in, args.k, mode, next_tokens=bufs[i % 2])
            pin_out.copy_(out, non_blocking=True)
            stream.synchronize()
            pin_in[0] = pin_out[0]
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b)
        e2e = {"value": round(n / (e_ms / 1e3), 2), "unit": "tokens/s", "h2d_bytes_per_step": 4,
               "d2h_bytes_per_step": 4, "steps": n,
               "note": "host-driven greedy loop: pinned H2D of the input token, decode step, D2H of the choice, sync"}
        # ---- CPU oracle baseline (bounded sample)
        if rank == 0 and w_np is not None:
            if host_mem_gb() > 40:
                import oracle as O
                om = O.Model(shape, w_np, dtype=np.float32)
                per_k, secs_all = {}, 0.0
                for kk in (1, 2, 4):
                    rate_k, secs = oracle_decode_rate(shape, None, kk, args.mode, 128, 8, model=om)
                    per_k[f"k{kk}"] = round(rate_k, 4)
                    secs_all += secs
                del om
                cpu = {"value": per_k[f"k{args.k}"] if f"k{args.k}" in per_k else None, "unit": "tokens/s",
                       "cores": blas_threads(), "kind": "oracle", "per_k": per_k,
                       "sample": f"float32 oracle, 4B shape, 128-token prompt then 8 timed greedy decode steps at "
                                 f"each of k = 1, 2, 4 ({args.mode}; {secs_all:.1f} s timed in all)"}
            else:
                cpu = {"value": None, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                       "sample": f"skipped: {host_mem_gb():.0f} GB host memory available, the fp32 oracle needs ~40"}

    if not args.no_aux and world == 1:
        aux["k_mode_sweep"] = leg(sweep_modes, dory, torch, shape, dw, args)
        aux["spec_decode"] = leg(spec_leg, dory, torch, shape, dw, args)
        aux["mixed_k_decode"] = leg(mixed_leg, dory, torch, shape, dw, args)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) weights with L2-normalised rows (bf16), uniform random prompt ids",
            "config": {"workload": workload, "model": "looped nGPT 4B-shaped", "global_batch": world,
                       "seq_len": args.prompt, "k": args.k, "cache_mode": args.mode,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2: each step streams ~11 GB of weights"},
            "hbm": {"bytes_per_step": step_bytes, "achieved_GBs": round(step_bytes / (ms_step / 1e3) / 1e9, 1),
                    "frac_of_peak": round(step_bytes / (ms_step / 1e3) / 1e9 / hbm, 4),
                    "frac_of_8TBs": round(step_bytes / (ms_step / 1e3) / 8e12, 4)},
            "prefill": {"tokens": args.prompt, "ms": round(pre_ms, 3),
                        "wall_tflops": round((pf + af) / (pre_ms / 1e3) / 1e12, 2),
                        "proj_tflops": round(pf / (proj_ms / 1e3) / 1e12, 2),
                        "proj_frac_of_peak_bf16": round(pf / (proj_ms / 1e3) / 1e12 / tc, 4),
                        "attn_tflops": round(af / (attn_ms / 1e3) / 1e12, 2),
                        "proj_tflop": round(pf / 1e12, 3), "attn_tflop": round(af / 1e12, 3),
                        "note": "proj/attn TFLOP/s: algorithmic FLOPs over the event-timed GEMM / attention "
                                "kernels of one prefill; wall: all FLOPs over the whole prefill",
                        "kernel_ms": {n: round(v["ms"], 3) for n, v in
                                      sorted(pprof.items(), key=lambda kv: -kv[1]["ms"])}},
            "roofline": roofline,
            "kernel_share": kernel_share,
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        line.update(aux)
        print(json.dumps(line))
    ranks.close()


def batched_leg(args):
    """64 sequences with 32768-token prompts at k=2, last-loop cache: chunked
    prefill (TFLOP/s), then batched decode steps (aggregate tokens/s, HBM GB/s).
    Prints one JSON line of its own."""
    import torch
    import synth
    import looped_ngpt_lm_b200 as dory

    hbm, tc, _, peak_src = peaks()
    shape = synth.DORY_4B
    B, P, k, chunk = args.batch, args.prompt_batched, 2, args.chunk
    steps, warm = args.steps, max(args.warmup, 3)
    torch.cuda.set_device(0)
    w_np = synth.make_weights(shape, 1)
    dw = dory.DeviceWeights(shape, w_np)
    del w_np
    cfg = dory.make_config(shape, max_batch=B, max_seq=P + steps + warm + 64, k_max=2, gamma_max=0,
                           max_chunk=chunk)
    h = dory.Handle(cfg, dw, dory.LAST_LOOP)
    if args.prefill_tc is not None:
        h.set_option(dory.OPT_PREFILL_TC, args.prefill_tc)
    ws_gb = dory.workspace_size(cfg, dory.LAST_LOOP) / 1e9
    prompts = torch.tensor(synth.make_prompt(1, B * P, shape.vocab), dtype=torch.int32).view(B, P).cuda()
    ev = lambda: torch.cuda.Event(enable_timing=True)

    # kernel-level split of one sequence's chunked prefill (events around every launch)
    h.reset()
    h.profile_reset()
    h.set_option(dory.OPT_PROFILE, 1)
    for c0 in range(0, P, chunk):
        n = min(chunk, P - c0)
        h.prefill([0], prompts[0, c0:c0 + n], [n], k, dory.LAST_LOOP)
    torch.cuda.synchronize()
    pprof = h.profile_read()
    h.set_option(dory.OPT_PROFILE, 0)
    h.profile_reset()
    pf1 = proj_flops(shape, k, P)
    af1 = attn_flops_prefill(shape, k, P)
    proj_ms = sum(v["ms"] for n_, v in pprof.items() if n_.startswith("gemm") and n_ != "gemm_lm_head")
    attn_ms = sum(v["ms"] for n_, v in pprof.items() if n_.startswith("attn"))

    # the whole batch, timed
    h.reset()
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    last = torch.empty(B, dtype=torch.int32, device="cuda")
    for s in range(B):
        for c0 in range(0, P, chunk):
            n = min(chunk, P - c0)
            t = h.prefill([s], prompts[s, c0:c0 + n], [n], k, dory.LAST_LOOP)
        last[s] = t[0]
    b.record()
    torch.cuda.synchronize()
    h.synchronize()
    pre_ms = a.elapsed_time(b)

    ids = list(range(B))
    bufs = [torch.empty(B, dtype=torch.int32, device="cuda") for _ in range(2)]
    tok = last
    for i in range(warm):
        tok = h.decode_step(ids, tok, k, dory.LAST_LOOP, next_tokens=bufs[i % 2])
    torch.cuda.synchronize()
    clocks = Clocks(0)
    clocks.start()
    a, b = ev(), ev()
    a.record()
    for i in range(steps):
        tok = h.decode_step(ids, tok, k, dory.LAST_LOOP, next_tokens=bufs[i % 2])
    b.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    h.synchronize()
    dec_ms = a.elapsed_time(b)
    ctx_mid = P + warm + steps // 2
    step_bytes = weight_bytes(shape, k) + B * kv_read_bytes(shape, k, ctx_mid)
    ms_step = dec_ms / steps
    line = {
        "leg": "batched", "config": {"workload": f"dory4b_bf16_batch{B}_prompt{P}_decode{steps}_k2_last_loop",
                                     "prefill_chunk": chunk, "workspace_GB": round(ws_gb, 2),
                                     "data": "synthetic: seeded weights, uniform random prompt ids"},
        "prefill": {"tokens": B * P, "s": round(pre_ms / 1e3, 3),
                    "wall_tflops": round(B * (pf1 + af1) / (pre_ms / 1e3) / 1e12, 2),
                    "proj_tflops": round(pf1 / (proj_ms / 1e3) / 1e12, 2),
                    "proj_frac_of_peak_bf16": round(pf1 / (proj_ms / 1e3) / 1e12 / tc, 4),
                    "attn_tflops": round(af1 / (attn_ms / 1e3) / 1e12, 2),
                    "pflop": round(B * (pf1 + af1) / 1e15, 3),
                    "kernel_ms_one_sequence": {n_: round(v["ms"], 2) for n_, v in
                                               sorted(pprof.items(), key=lambda kv: -kv[1]["ms"])[:8]}},
        "decode": {"steps": steps, "ms_per_step": round(ms_step, 3),
                   "tokens_per_s": round(B * steps / (dec_ms / 1e3), 1),
                   "bytes_per_step": step_bytes,
                   "hbm_GBs": round(step_bytes / (ms_step / 1e3) / 1e9, 1),
                   "hbm_frac_of_peak": round(step_bytes / (ms_step / 1e3) / 1e9 / hbm, 4)},
        "peaks": {"hbm_GBs": hbm, "bf16_tflops": tc, "source": peak_src},
        "clocks": clk,
    }
    print(json.dumps(line))


def gemm_probe(args):
    """Decode-projection GEMMs of the 4B shape at M token rows, each timed
    alone with CUDA events over launches that rotate through enough weight
    copies (> 4x L2) that every launch streams its weights from HBM."""
    import torch
    import looped_ngpt_lm_b200 as dory
    import synth
    s = synth.DORY_4B
    shapes = {"qkv": (s.q_dim + 2 * s.kv_dim, s.d_model), "o": (s.d_model, s.q_dim),
              "gate_up": (2 * s.d_ff, s.d_model), "down": (s.d_model, s.d_ff), "lm_head": (s.vocab, s.d_model)}
    hbm = peaks()[0]
    out = {}
    for name in args.shape.split(","):
        N, K = shapes[name]
        wbytes = N * K * 2
        copies = max(2, -(-512_000_000 // wbytes))
        g = torch.Generator(device="cuda").manual_seed(0)
        Ws = [(torch.randn((N, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16) for _ in range(copies)]
        if args.gemm_variant == 4:  # packed tile layout
            Ws = [dory.pack_weight_bf16(w) for w in Ws]
        X = torch.randn((args.m, K), generator=g, device="cuda").to(torch.bfloat16)
        Y = torch.empty((8, args.m, N), dtype=torch.float32, device="cuda")
        S = 1
        for i in range(3):
            S = dory.gemm_bf16_into(X, Ws[i % copies], Y, 1, True, args.gemm_variant)
        torch.cuda.synchronize()
        # replay the launches from a CUDA graph so the host does not pace them
        iters = max(30, 3 * copies)
        side = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for i in range(iters):
                dory.gemm_bf16_into(X, Ws[i % copies], Y, 1, True, args.gemm_variant, stream=side)
        graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        us = 1e3 * a.elapsed_time(b) / iters
        by = wbytes + args.m * K * 2 + S * args.m * N * 4
        out[name] = {"N": N, "K": K, "splits": S, "us": round(us, 2), "GBs": round(by / us / 1e3, 1),
                     "frac_of_peak": round(by / us / 1e3 / hbm, 4)}
        del Ws
    print(json.dumps({"kernel": "gemm_tc", "impl": args.gemm_variant, "m": args.m, "results": out,
                      "hbm_peak_GBs": hbm, "peak_source": peaks()[3],
                      "note": "graph-replayed back-to-back launches, weights cold in L2"}))


def mx_gemv_probe(args):
    """The MXFP8 decode GEMV (dory_gemv_mxfp8) on the 4B decode shapes at M
    token rows, each timed alone like --kernel gemm: graph-replayed launches
    rotating through weight copies (> 2x L2) of random E4M3 codes (NaN codes
    excluded) and scale bytes 110..124.  --mx-impl 1: CUDA cores, 2: mma.sync,
    3: TMA-fed tcgen05 without split-K.  --kernel nvgemm: the NVFP4 GEMM
    (dory_gemm_nvfp4) on random E2M1 code pairs, E4M3 scales 0x30..0x37 and
    g = 2^-9."""
    nv = args.kernel == "nvgemm"
    import ctypes
    import torch
    import looped_ngpt_lm_b200 as dory
    import synth
    s = synth.DORY_4B
    shapes = {"qkv": (s.q_dim + 2 * s.kv_dim, s.d_model), "o": (s.d_model, s.q_dim),
              "gate_up": (2 * s.d_ff, s.d_model), "down": (s.d_model, s.d_ff), "lm_head": (s.vocab, s.d_model)}
    hbm = peaks()[0]
    out = {}
    for name in args.shape.split(","):
        N, K = shapes[name]
        wbytes = N * K // 2 + N * K // 16 if nv else N * K + N * K // 32
        copies = max(2, -(-300_000_000 // wbytes))
        g = torch.Generator(device="cuda").manual_seed(0)
        qs, ss = [], []
        gscale = torch.tensor([2.0 ** -9], dtype=torch.float32, device="cuda")
        for _ in range(copies):
            if nv:
                qs.append(torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8, device="cuda"))
                ss.append(torch.randint(0x30, 0x38, (N, K // 16), generator=g, dtype=torch.uint8, device="cuda"))
                continue
            q = torch.randint(0, 0x7E, (N, K), generator=g, dtype=torch.uint8, device="cuda")
            q |= torch.randint(0, 2, (N, K), generator=g, dtype=torch.uint8, device="cuda") << 7
            qs.append(q)
            ss.append(torch.randint(110, 125, (N, K // 32), generator=g, dtype=torch.uint8, device="cuda"))
        X = (torch.randn((args.m, K), generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
        Y = torch.empty((args.m, N), dtype=torch.float32, device="cuda")

        def one(i, st):
            if nv:
                dory._check(dory.lib.dory_gemm_nvfp4(args.m, N, K, ctypes.c_void_p(X.data_ptr()), K,
                                                      ctypes.c_void_p(qs[i].data_ptr()),
                                                      ctypes.c_void_p(ss[i].data_ptr()),
                                                      ctypes.c_void_p(gscale.data_ptr()), ctypes.c_void_p(Y.data_ptr()),
                                                      N, None, ctypes.c_void_p(st.cuda_stream)))
                return
            dory._check(dory.lib.dory_gemv_mxfp8(args.m, N, K, ctypes.c_void_p(X.data_ptr()), K,
                                                  ctypes.c_void_p(qs[i].data_ptr()), ctypes.c_void_p(ss[i].data_ptr()),
                                                  ctypes.c_void_p(Y.data_ptr()), N, args.mx_impl, None,
                                                  ctypes.c_void_p(st.cuda_stream)))

        for i in range(3):
            one(i % copies, torch.cuda.current_stream())
        torch.cuda.synchronize()
        iters = max(30, 3 * copies)
        side = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for i in range(iters):
                one(i % copies, side)
        graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        us = 1e3 * a.elapsed_time(b) / iters
        by = wbytes + args.m * K * 2 + args.m * N * 4
        out[name] = {"N": N, "K": K, "us": round(us, 2), "GBs": round(by / us / 1e3, 1),
                     "frac_of_peak": round(by / us / 1e3 / hbm, 4)}
        del qs, ss, graph
        torch.cuda.empty_cache()
    print(json.dumps({"kernel": "nv_gemm" if nv else "mx_gemv", "mx_impl": None if nv else args.mx_impl,
                      "m": args.m, "results": out, "hbm_peak_GBs": hbm, "peak_source": peaks()[3],
                      "note": "graph-replayed back-to-back launches, weights cold in L2; one K split (S = 1), "
                              "which a decode step does not use for the QKV, O and down shapes (it splits K: "
                              "see the mxfp8_decode / nvfp4_decode legs for the in-step kernels)"}))


def run_reference(args, shape, workload):
    """Reference arm: the oracle on the host cores, one greedy decode step of
    the 4B shape per step (a bounded sample of the workload: an 8-token prompt
    instead of 2560, so each step's attention is shorter; the weights, which
    dominate a step, are the same), exactly --steps timed after --warmup."""
    import synth
    w = synth.make_weights(shape, 1)
    if host_mem_gb() < 40:
        print(json.dumps({"impl": "reference", "unavailable": "the float32 oracle of the 4B shape needs ~40 GB of host memory"}))
        return
    import oracle as O
    m = O.Model(shape, w, dtype=np.float32)
    del w
    prompt = synth.make_prompt(1, 8, shape.vocab)
    steps = max(1, args.steps)
    warm = max(0, args.warmup)
    cache = O.Cache(m, 8 + steps + warm + 2)
    lg = O.forward_chunk(m, cache, prompt, args.k, args.mode)
    tok = int(np.argmax(lg[-1]))
    for _ in range(warm):
        tok = int(np.argmax(O.forward_chunk(m, cache, [tok], args.k, args.mode)[-1]))
    t0 = time.perf_counter()
    for _ in range(steps):
        tok = int(np.argmax(O.forward_chunk(m, cache, [tok], args.k, args.mode)[-1]))
    dt = time.perf_counter() - t0
    v = steps / dt
    sample = (f"float32 oracle, 4B shape, {steps} timed greedy decode steps at k={args.k} {args.mode} after an "
              f"8-token prompt (a bounded sample of the {args.prompt}-token workload)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "tokens/s", "n_gpus": 1,
        "steps": steps, "warmup": warm, "ms_per_step": round(1e3 * dt / steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": workload, "model": "looped nGPT 4B-shaped", "global_batch": 1,
                   "seq_len": args.prompt, "k": args.k, "cache_mode": args.mode, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


if __name__ == "__main__":
    main()
