"""Oracle for the looped normalized-GPT forward -- TEST INFRASTRUCTURE ONLY.

This is a plain, slow, CPU implementation written to be checked by eye against
the sources.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference legs may import it; the CUDA library never does, and
this module shares no code with it (inputs come from the ``synth`` package).

Sources (web pages about Dory1.0-4B; section names translated):

* onedev.kr paper digest "Dory1.0-4B는 반복 횟수로 추론 연산과 정확도를
  조절한다", section "How it works": input block, shared recurrent block
  applied k times, output block; ``s0 = x``, ``u_t = N(s_{t-1} + x)``,
  ``s_t = N(F(u_t))``; ``s_k`` goes to the output block and the LM head; no
  adapter and no outer residual; 72/112/192 layer applications at k=1/2/4;
  36 MLP-only, 27 sliding-window and 9 full-attention layers, attention 3:1.
* same digest, section "Premises & limits" (and the trawling.dev / lucasainews
  articles, "KV cache" sections): last-loop KV caching, where every loop
  overwrites the previous loop's cache so its size stays at the k=1 size, and
  queries of earlier loops see the *final-loop* keys/values of earlier tokens;
  per-loop caching keeps one cache per loop.  Self-speculative decoding drafts
  at k=1, verifies at k=4, proposes gamma=4 tokens and reuses KV/activations.
* blog.secrett2633.cloud review "Dory1.0-4B: A Looped Normalized-GPT", §1 Key
  Terms: nGPT keeps hidden states L2-normalised.

Readings where the pages are silent (each also listed with the design notes):

* Per-layer update ``h = N(h + sublayer(h))``; no nGPT eigen learning rates,
  scale vectors or biases; softmax scale ``1/sqrt(head_dim)``.
* Physical layers alternate attention and MLP, attention first; attention
  layer j (counted over the whole stack) is full causal iff
  ``j % full_every == full_phase`` (4 and 3), otherwise sliding window.
* Sliding window of W keys including the query itself: keys ``p-W < j <= p``.
* No positional encoding; causal and window masks carry the order.
* SwiGLU MLP ``W_down (silu(W_g h) * (W_u h))``; GQA head ``h`` reads KV head
  ``h // (n_heads / n_kv_heads)``; untied LM head; greedy argmax, lowest id
  wins ties.
* Chunk semantics for last_loop: inside one forward call over several new
  tokens, loop t of every chunk position writes its loop-t K/V into the shared
  slot and attends to the chunk's loop-t K/V plus the cached (final-loop) K/V
  of earlier calls.  Decode calls are one-token chunks.
* ``N(v) = v / max(||v||_2, 1e-12)``.

Arithmetic is float64 by default; ``dtype=np.float32`` is accepted for the
4B-shaped model, whose float64 weights would not fit in host memory.

Pins (tests/test_oracle_pins.py) fix the pages' numbers, the invariants and
the closed forms of the recurrence, the attention and the MLP, and the
composition through relabelling invariances: renaming hidden units, MLP units
or heads consistently must leave the logits unchanged.  No external
reference value exists for a whole forward pass: the pages print no worked
example.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

LAST_LOOP = "last_loop"
PER_LOOP = "per_loop"
NORM_EPS = 1e-12


def l2n(v: np.ndarray) -> np.ndarray:
    """N(v): divide each last-axis vector by its L2 norm (floored at 1e-12)."""
    n = np.sqrt(np.sum(v * v, axis=-1, keepdims=True))
    return v / np.maximum(n, NORM_EPS)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def argmax_lowest(logits: np.ndarray) -> np.ndarray:
    """Greedy choice per row; numpy's argmax returns the first (lowest) id."""
    return np.argmax(logits, axis=-1)


class Model:
    """Weights (converted to the arithmetic dtype) plus the layer rules."""

    def __init__(self, shape, weights: dict, dtype=np.float64):
        self.shape = shape
        self.dtype = np.dtype(dtype)
        self.w = {}
        for name, arr in weights.items():
            if arr.dtype == np.uint16:  # bf16 bit patterns: widen exactly
                arr = (arr.astype(np.uint32) << 16).view(np.float32)
            self.w[name] = np.ascontiguousarray(arr, dtype=self.dtype)
        self.applications = 0  # (layer, token) sublayer applications so far

    # -- layer rules ---------------------------------------------------
    def kind(self, l: int) -> str:
        return "attn" if l % 2 == 0 else "mlp"

    def is_full(self, l: int) -> bool:
        s = self.shape
        return (l // 2) % s.full_every == s.full_phase

    def block(self, name: str) -> range:
        s = self.shape
        if name == "I":
            return range(0, s.n_in)
        if name == "R":
            return range(s.n_in, s.n_in + s.n_rec)
        if name == "O":
            return range(s.n_in + s.n_rec, s.n_layers)
        raise ValueError(name)

    def is_recurrent(self, l: int) -> bool:
        return l in self.block("R")

    def schedule(self, k: int) -> list[tuple[int, int]]:
        """(physical layer, loop) in the order one token applies them; loop 0
        marks the input and output blocks, 1..k the recurrent passes."""
        out = [(l, 0) for l in self.block("I")]
        for t in range(1, k + 1):
            out += [(l, t) for l in self.block("R")]
        out += [(l, 0) for l in self.block("O")]
        return out

    def slot(self, l: int, loop: int, mode: str) -> int:
        """Cache slot: last_loop shares slot 0 across loops; per_loop gives
        each recurrent loop t its own slot t."""
        if mode == PER_LOOP and self.is_recurrent(l):
            return loop
        return 0


@dataclass
class Cache:
    """One sequence's KV cache, addressed by absolute position (no ring).

    ``kv[(layer, slot)]`` holds ``K``, ``V`` of shape
    ``[capacity, n_kv_heads, head_dim]`` and a written-mask.  ``length`` is
    the number of committed positions.
    """

    model: Model
    capacity: int
    length: int = 0
    kv: dict = field(default_factory=dict)

    def arrays(self, l: int, slot: int):
        key = (l, slot)
        if key not in self.kv:
            s = self.model.shape
            shp = (self.capacity, s.n_kv_heads, s.head_dim)
            self.kv[key] = (np.zeros(shp, self.model.dtype), np.zeros(shp, self.model.dtype),
                            np.zeros(self.capacity, bool))
        return self.kv[key]

    def footprint_bytes(self, elem_bytes: int) -> int:
        """Bytes a cache must retain for future tokens: every slot that was
        written, times the positions still visible to a future query
        (the last W for a sliding-window layer, all of them for a full one)."""
        s = self.model.shape
        total = 0
        for (l, _slot) in self.kv:
            keep = self.length if self.model.is_full(l) else min(self.length, s.swa_window)
            total += keep * 2 * s.kv_dim * elem_bytes
        return total


def kv_bytes(model: Model, k: int, mode: str, ctx: int, elem_bytes: int) -> int:
    """Retained KV bytes for one sequence of ``ctx`` tokens run at loop count
    k: one slot per attention layer, except per_loop recurrent layers, which
    keep one slot per loop."""
    s = model.shape
    slots = set((l, model.slot(l, t, mode)) for (l, t) in model.schedule(k) if model.kind(l) == "attn")
    total = 0
    for (l, _slot) in slots:
        keep = ctx if model.is_full(l) else min(ctx, s.swa_window)
        total += keep * 2 * s.kv_dim * elem_bytes
    return total


def attention(model: Model, cache: Cache, l: int, slot: int, h: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """One attention sublayer over a chunk of rows ``h`` at positions ``pos``.

    The chunk's K/V are written into the cache first, then each query reads
    keys j with ``lo <= j <= p`` from the cache (``lo = 0`` for full
    attention, ``p - W + 1`` for the sliding window), so in-chunk keys are
    this pass's values and earlier keys are whatever the cache holds.
    """
    s = model.shape
    w = model.w
    C = h.shape[0]
    H, KV, hd = s.n_heads, s.n_kv_heads, s.head_dim
    group = H // KV
    q = (h @ w[f"L{l}.wq"].T).reshape(C, H, hd)
    k = (h @ w[f"L{l}.wk"].T).reshape(C, KV, hd)
    v = (h @ w[f"L{l}.wv"].T).reshape(C, KV, hd)
    K, V, written = cache.arrays(l, slot)
    K[pos] = k
    V[pos] = v
    written[pos] = True
    kv_of_head = np.arange(H) // group
    scale = 1.0 / math.sqrt(hd)
    out = np.empty((C, H, hd), model.dtype)
    full = model.is_full(l)
    for i, p in enumerate(pos):
        lo = 0 if full else max(0, p - s.swa_window + 1)
        if not written[lo:p + 1].all():
            raise RuntimeError(f"layer {l} slot {slot}: key in [{lo},{p}] was never written")
        keys = K[lo:p + 1][:, kv_of_head, :]  # [J, H, hd]
        vals = V[lo:p + 1][:, kv_of_head, :]
        scores = np.einsum("hd,jhd->hj", q[i], keys) * scale
        scores = scores - scores.max(axis=1, keepdims=True)
        e = np.exp(scores)
        pr = e / e.sum(axis=1, keepdims=True)
        out[i] = np.einsum("hj,jhd->hd", pr, vals)
    return out.reshape(C, H * hd) @ w[f"L{l}.wo"].T


def mlp(model: Model, l: int, h: np.ndarray) -> np.ndarray:
    """SwiGLU: W_down (silu(W_g h) * (W_u h))."""
    w = model.w
    return (silu(h @ w[f"L{l}.wg"].T) * (h @ w[f"L{l}.wu"].T)) @ w[f"L{l}.wdown"].T


def run_layers(model: Model, cache: Cache, layers, h, pos, loop: int, mode: str):
    """Apply physical layers in order, each as h <- N(h + sublayer(h))."""
    for l in layers:
        if model.kind(l) == "attn":
            y = attention(model, cache, l, model.slot(l, loop, mode), h, pos)
        else:
            y = mlp(model, l, h)
        h = l2n(h + y)
        model.applications += h.shape[0]
    return h


def forward_chunk(model: Model, cache: Cache, tokens, k: int, mode: str,
                  head: str = "last", trace: dict | None = None) -> np.ndarray:
    """Forward a chunk of new tokens of one sequence at loop count k.

    Returns logits for the last chunk position (``head='last'``) or for every
    position (``head='all'``).  ``trace`` (optional) receives x, every u_t and
    s_t, and the output-block result.
    """
    if mode not in (LAST_LOOP, PER_LOOP):
        raise ValueError(mode)
    if k < 1:
        raise ValueError("k must be >= 1")
    tokens = np.asarray(tokens, dtype=np.int64)
    C = tokens.shape[0]
    p0 = cache.length
    if p0 + C > cache.capacity:
        raise ValueError("cache capacity exceeded")
    pos = p0 + np.arange(C)
    h = model.w["embed"][tokens]
    h = run_layers(model, cache, model.block("I"), h, pos, 0, mode)
    x = h
    s = x
    if trace is not None:
        trace["x"] = x.copy()
        trace["u"], trace["s"] = [], []
    for t in range(1, k + 1):
        u = l2n(s + x)
        h = run_layers(model, cache, model.block("R"), u, pos, t, mode)
        s = l2n(h)
        if trace is not None:
            trace["u"].append(u.copy())
            trace["s"].append(s.copy())
    h = run_layers(model, cache, model.block("O"), s, pos, 0, mode)
    if trace is not None:
        trace["out"] = h.copy()
    cache.length = p0 + C
    rows = h[-1:] if head == "last" else h
    return rows @ model.w["lm_head"].T


def generate(model: Model, prompt, n_new: int, k: int, mode: str, capacity: int | None = None,
             chunks: list[int] | None = None, forced=None):
    """Greedy generation: prefill the prompt (in ``chunks`` if given), then
    decode one token per call.  Returns (tokens[n_new], logits[n_new, vocab]).

    With ``forced`` the decode inputs are the given tokens instead of the
    model's own choices (teacher forcing), so the logits can be compared step
    by step with another implementation that chose them.
    """
    prompt = np.asarray(prompt)
    cap = capacity or (len(prompt) + n_new + 1)
    cache = Cache(model, cap)
    if chunks is None:
        chunks = [len(prompt)]
    off = 0
    for c in chunks:
        lg = forward_chunk(model, cache, prompt[off:off + c], k, mode)
        off += c
    assert off == len(prompt)
    toks, logits = [], []
    cur = int(argmax_lowest(lg[-1]))
    toks.append(cur)
    logits.append(lg[-1])
    for i in range(1, n_new):
        inp = cur if forced is None else int(forced[i - 1])
        lg = forward_chunk(model, cache, [inp], k, mode)
        cur = int(argmax_lowest(lg[-1]))
        toks.append(cur)
        logits.append(lg[-1])
    return np.array(toks, dtype=np.int64), np.stack(logits)


@dataclass
class SpecStats:
    steps: int = 0
    drafted: int = 0
    accepted: int = 0
    accepted_per_step: list = field(default_factory=list)


def spec_generate(model: Model, prompt, n_new: int, k_draft: int = 1, k_verify: int = 4,
                  gamma: int = 4, mode: str = LAST_LOOP, capacity: int | None = None):
    """Self-speculative greedy generation (draft at k_draft, verify at k_verify).

    Each step, with y0 the pending token: forward y0, d1, ..., d_{gamma-1} one
    at a time at k_draft, producing drafts d1..d_gamma; then forward the chunk
    [y0, d1..d_gamma] at k_verify, giving choices a_0..a_gamma; accept the
    longest prefix with a_i == d_{i+1}, emit d1..d_n and the verifier's a_n,
    and keep y0, d1..d_n as committed positions.

    The verify pass here recomputes the input block and loop 1 of the chunk;
    that is the same arithmetic as reusing the drafts' values, because loop 1
    sees the same keys in both (committed final-loop K/V plus the chunk's
    loop-1 K/V) and ``u_1 = N(x + x) = x`` does not depend on k.
    """
    prompt = np.asarray(prompt)
    cap = capacity or (len(prompt) + n_new + gamma + 2)
    cache = Cache(model, cap)
    lg = forward_chunk(model, cache, prompt, k_verify, mode)
    y0 = int(argmax_lowest(lg[-1]))
    out = [y0]
    st = SpecStats()
    while len(out) < n_new:
        p0 = cache.length
        drafts = []
        cur = y0
        for _ in range(gamma):
            lg = forward_chunk(model, cache, [cur], k_draft, mode)
            cur = int(argmax_lowest(lg[-1]))
            drafts.append(cur)
        cache.length = p0
        lg = forward_chunk(model, cache, [y0] + drafts, k_verify, mode, head="all")
        a = argmax_lowest(lg)
        n = 0
        while n < gamma and int(a[n]) == drafts[n]:
            n += 1
        out += drafts[:n] + [int(a[n])]
        cache.length = p0 + n + 1
        y0 = int(a[n])
        st.steps += 1
        st.drafted += gamma
        st.accepted += n
        st.accepted_per_step.append(n)
    return np.array(out[:n_new], dtype=np.int64), st
