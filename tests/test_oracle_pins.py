"""Pins for the oracle: page facts, invariants, closed forms and brute force.

None of these re-types the oracle's code: each checks it against a number the
pages print (tests/golden/page_facts.json), a property the pages or the
mathematics fix, or an explicit loop-by-loop computation of a special case.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")
FACTS = json.load(open(GOLDEN))


@pytest.fixture(scope="module")
def tiny():
    return O.Model(synth.TINY, synth.make_weights(synth.TINY, 0))


@pytest.fixture(scope="module")
def prompt():
    return synth.make_prompt(0, 64, synth.TINY.vocab)


def micro_shape(**kw):
    base = dict(name="micro", d_model=8, vocab=16, n_heads=2, head_dim=4, n_kv_heads=1, d_ff=6,
                n_in=2, n_rec=2, n_out=2, swa_window=4, full_every=4, full_phase=3, dtype="f32")
    base.update(kw)
    return synth.Shape(**base)


# ---------------------------------------------------------------- page facts
def test_layer_counts_match_pages():
    m = O.Model(synth.DORY_4B, {})
    f = FACTS["physical_layers"]["value"]
    assert (len(m.block("I")), len(m.block("R")), len(m.block("O"))) == (f["input"], f["recurrent"], f["output"])
    mix = FACTS["layer_mix"]["value"]
    L = range(synth.DORY_4B.n_layers)
    attn = [l for l in L if m.kind(l) == "attn"]
    assert sum(m.kind(l) == "mlp" for l in L) == mix["mlp_only"]
    assert sum(m.is_full(l) for l in attn) == mix["full_attention"]
    assert sum(not m.is_full(l) for l in attn) == mix["sliding_window"]
    # 3:1 interleave: every run of four consecutive attention layers has one full layer
    for i in range(0, len(attn), 4):
        assert sum(m.is_full(l) for l in attn[i:i + 4]) == 1


@pytest.mark.parametrize("k", [1, 2, 4])
def test_layer_applications_match_pages(k):
    m = O.Model(synth.DORY_4B, {})
    assert len(m.schedule(k)) == FACTS["layer_applications_per_token"]["value"][str(k)]


def test_parameter_count_is_4b():
    n = sum(r * c for _, (r, c) in synth.weight_specs(synth.DORY_4B))
    assert round(n / 1e9) == FACTS["parameters_billion"]["value"]


@pytest.mark.parametrize("k", [1, 2, 4])
def test_forward_applies_the_schedule(tiny, prompt, k):
    tiny.applications = 0
    O.generate(tiny, prompt[:10], 3, k, O.LAST_LOOP)
    # 10 prompt tokens + 2 decoded tokens, each through every scheduled layer
    assert tiny.applications == 12 * len(tiny.schedule(k)) == 12 * (2 + 4 * k + 2)


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("k", [1, 2, 4])
@pytest.mark.parametrize("mode", [O.LAST_LOOP, O.PER_LOOP])
def test_states_unit_norm_and_u1_equals_x(tiny, prompt, k, mode):
    cache = O.Cache(tiny, 128)
    tr = {}
    O.forward_chunk(tiny, cache, prompt[:40], k, mode, trace=tr)
    for v in [tr["x"], tr["out"], *tr["u"], *tr["s"]]:
        assert np.abs(np.linalg.norm(v, axis=-1) - 1).max() < 1e-12
    # s0 = x, so u_1 = N(x + x) = x
    assert np.abs(tr["u"][0] - tr["x"]).max() < 4e-16
    assert len(tr["u"]) == k


def test_k1_modes_identical(tiny, prompt):
    t_a, l_a = O.generate(tiny, prompt, 8, 1, O.LAST_LOOP)
    t_b, l_b = O.generate(tiny, prompt, 8, 1, O.PER_LOOP)
    assert np.array_equal(t_a, t_b) and np.array_equal(l_a, l_b)
    ca, cb = O.Cache(tiny, 80), O.Cache(tiny, 80)
    O.forward_chunk(tiny, ca, prompt, 1, O.LAST_LOOP)
    O.forward_chunk(tiny, cb, prompt, 1, O.PER_LOOP)
    for (l, s), (K, V, _) in ca.kv.items():
        sb = tiny.slot(l, 1, O.PER_LOOP)
        assert np.array_equal(K, cb.kv[(l, sb)][0]) and np.array_equal(V, cb.kv[(l, sb)][1])


def test_last_loop_kv_size_constant_in_k(tiny, prompt):
    assert FACTS["last_loop_kv_size_independent_of_k"]["value"]
    sizes = {}
    for mode in (O.LAST_LOOP, O.PER_LOOP):
        for k in (1, 2, 4):
            c = O.Cache(tiny, 80)
            O.forward_chunk(tiny, c, prompt, k, mode)
            sizes[mode, k] = c.footprint_bytes(4)
            assert sizes[mode, k] == O.kv_bytes(tiny, k, mode, 64, 4)
    assert sizes[O.LAST_LOOP, 1] == sizes[O.LAST_LOOP, 2] == sizes[O.LAST_LOOP, 4]
    assert sizes[O.PER_LOOP, 1] == sizes[O.LAST_LOOP, 1]
    step = sizes[O.PER_LOOP, 2] - sizes[O.PER_LOOP, 1]
    assert step > 0 and sizes[O.PER_LOOP, 4] - sizes[O.PER_LOOP, 1] == 3 * step


def test_4b_kv_bytes_per_token():
    m = O.Model(synth.DORY_4B, {})
    # 9 full layers x 2 (K,V) x 4 heads x 128 x 2 bytes per token once ctx > window is irrelevant
    full_per_tok = 9 * 2 * 4 * 128 * 2
    ctx = 5000
    want = full_per_tok * ctx + 27 * 2 * 4 * 128 * 2 * 4096
    for k in (1, 2, 4):
        assert O.kv_bytes(m, k, O.LAST_LOOP, ctx, 2) == want
    # per_loop: the 5 recurrent full and 15 recurrent SWA layers gain a slot per extra loop
    extra = 5 * 2048 * ctx + 15 * 2048 * 4096
    assert O.kv_bytes(m, 4, O.PER_LOOP, ctx, 2) == want + 3 * extra


def test_input_block_independent_of_k_and_mode(tiny, prompt):
    ref = None
    for mode in (O.LAST_LOOP, O.PER_LOOP):
        for k in (1, 2, 4):
            c = O.Cache(tiny, 80)
            tr = {}
            O.forward_chunk(tiny, c, prompt, k, mode, trace=tr)
            ikv = {key: (K.copy(), V.copy()) for key, (K, V, _) in c.kv.items() if key[0] in tiny.block("I")}
            if ref is None:
                ref = (tr["x"], ikv)
            else:
                assert np.array_equal(tr["x"], ref[0])
                for key in ikv:
                    assert np.array_equal(ikv[key][0], ref[1][key][0])


@pytest.mark.parametrize("k", [2, 4])
def test_single_chunk_prefill_same_in_both_modes(tiny, prompt, k):
    la = O.forward_chunk(tiny, O.Cache(tiny, 80), prompt, k, O.LAST_LOOP, head="all")
    lb = O.forward_chunk(tiny, O.Cache(tiny, 80), prompt, k, O.PER_LOOP, head="all")
    assert np.array_equal(la, lb)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_per_loop_chunking_is_invisible(tiny, prompt, k):
    """per_loop keeps every loop's keys, so splitting the prompt into chunks
    (or single tokens) cannot change anything."""
    one = O.forward_chunk(tiny, O.Cache(tiny, 80), prompt, k, O.PER_LOOP, head="all")
    c = O.Cache(tiny, 80)
    parts = []
    for a, b in [(0, 20), (20, 21), (21, 51), (51, 64)]:
        parts.append(O.forward_chunk(tiny, c, prompt[a:b], k, O.PER_LOOP, head="all"))
    assert np.abs(np.concatenate(parts) - one).max() < 1e-12
    c = O.Cache(tiny, 80)
    steps = [O.forward_chunk(tiny, c, prompt[i:i + 1], k, O.PER_LOOP) for i in range(64)]
    assert np.abs(np.concatenate(steps) - one).max() < 1e-12


def test_last_loop_differs_from_per_loop_at_k2(tiny, prompt):
    """Last-loop caching shows earlier loops the final-loop keys: a real
    difference from per-loop caching once a token has context and k > 1."""
    ca, cb = O.Cache(tiny, 80), O.Cache(tiny, 80)
    la = [O.forward_chunk(tiny, ca, prompt[i:i + 1], 2, O.LAST_LOOP) for i in range(8)]
    lb = [O.forward_chunk(tiny, cb, prompt[i:i + 1], 2, O.PER_LOOP) for i in range(8)]
    assert np.array_equal(la[0], lb[0])  # first token: no context, no difference
    assert np.abs(la[7] - lb[7]).max() > 1e-6


def test_causality(tiny, prompt):
    a = O.forward_chunk(tiny, O.Cache(tiny, 80), prompt, 2, O.LAST_LOOP, head="all")
    p2 = prompt.copy()
    p2[40] = (p2[40] + 1) % synth.TINY.vocab
    b = O.forward_chunk(tiny, O.Cache(tiny, 80), p2, 2, O.LAST_LOOP, head="all")
    assert np.array_equal(a[:40], b[:40])
    assert np.abs(a[40:] - b[40:]).max() > 1e-6


def test_window_at_least_context_equals_full(tiny, prompt):
    w = tiny.w
    wide = O.Model(synth.TINY.with_(swa_window=1000), {})
    wide.w = w
    full = O.Model(synth.TINY.with_(full_every=1, full_phase=0), {})
    full.w = w
    a = O.forward_chunk(wide, O.Cache(wide, 80), prompt, 2, O.LAST_LOOP, head="all")
    b = O.forward_chunk(full, O.Cache(full, 80), prompt, 2, O.LAST_LOOP, head="all")
    assert np.array_equal(a, b)


def test_gqa_with_duplicated_kv_equals_mha(tiny, prompt):
    s = synth.TINY
    G = s.n_heads // s.n_kv_heads
    mha = O.Model(s.with_(n_kv_heads=s.n_heads), {})
    mha.w = dict(tiny.w)
    for l in range(s.n_layers):
        if tiny.kind(l) != "attn":
            continue
        for nm in ("wk", "wv"):
            W = tiny.w[f"L{l}.{nm}"].reshape(s.n_kv_heads, s.head_dim, s.d_model)
            mha.w[f"L{l}.{nm}"] = np.repeat(W, G, axis=0).reshape(s.q_dim, s.d_model)
    a = O.forward_chunk(tiny, O.Cache(tiny, 80), prompt, 2, O.PER_LOOP, head="all")
    b = O.forward_chunk(mha, O.Cache(mha, 80), prompt, 2, O.PER_LOOP, head="all")
    assert np.abs(a - b).max() < 1e-13


# ---------------------------------------------------------------- brute force
def brute_attention(q, K, V, lo_hi, H, KV, hd):
    """Loop-by-loop softmax attention for one query: q[H*hd], K/V[j][KV*hd]."""
    G = H // KV
    out = [0.0] * (H * hd)
    lo, hi = lo_hi
    for h in range(H):
        g = h // G
        scores = []
        for j in range(lo, hi + 1):
            dot = 0.0
            for e in range(hd):
                dot += q[h * hd + e] * K[j][g * hd + e]
            scores.append(dot / math.sqrt(hd))
        mx = max(scores)
        ex = [math.exp(x - mx) for x in scores]
        tot = sum(ex)
        for e in range(hd):
            acc = 0.0
            for jj, j in enumerate(range(lo, hi + 1)):
                acc += ex[jj] / tot * V[j][g * hd + e]
            out[h * hd + e] = acc
    return out


@pytest.mark.parametrize("full", [False, True])
def test_attention_brute_force(full):
    s = micro_shape(n_heads=4, n_kv_heads=2, head_dim=3, d_model=6, swa_window=3,
                    full_every=1 if full else 4, full_phase=0 if full else 3)
    rng = np.random.default_rng(5)
    w = {f"L0.{n}": rng.standard_normal(shape) for n, shape in
         [("wq", (12, 6)), ("wk", (6, 6)), ("wv", (6, 6)), ("wo", (6, 12))]}
    m = O.Model(s, w)
    cache = O.Cache(m, 16)
    hs = rng.standard_normal((9, 6))
    # two calls: a chunk of 5 then a chunk of 4 at p0 = 5
    outs = [O.attention(m, cache, 0, 0, hs[:5], np.arange(5)),
            O.attention(m, cache, 0, 0, hs[5:], np.arange(5, 9))]
    got = np.concatenate(outs)
    Ks = [list(w["L0.wk"] @ h) for h in hs]
    Vs = [list(w["L0.wv"] @ h) for h in hs]
    for p in range(9):
        q = list(w["L0.wq"] @ hs[p])
        lo = 0 if full else max(0, p - 3 + 1)
        a = brute_attention(q, Ks, Vs, (lo, p), 4, 2, 3)
        y = [sum(w["L0.wo"][r][c] * a[c] for c in range(12)) for r in range(6)]
        assert np.allclose(got[p], y, rtol=0, atol=1e-12), p


def test_one_key_returns_v_and_window_one():
    s = micro_shape(swa_window=1)
    w = synth.make_weights(s, 3)
    m = O.Model(s, w)
    h = O.l2n(np.random.default_rng(1).standard_normal((5, 8)))
    # window 1: every query sees only its own key, so the softmax weight is 1
    y = O.attention(m, O.Cache(m, 8), 0, 0, h, np.arange(5))
    G = s.n_heads // s.n_kv_heads
    v = h @ m.w["L0.wv"].T  # [5, kv_dim]
    v_heads = np.concatenate([v[:, (hh // G) * s.head_dim:(hh // G + 1) * s.head_dim] for hh in range(s.n_heads)], 1)
    assert np.abs(y - v_heads @ m.w["L0.wo"].T).max() < 1e-13


def test_mlp_brute_force():
    s = micro_shape()
    rng = np.random.default_rng(2)
    w = {"L1.wg": rng.standard_normal((6, 8)), "L1.wu": rng.standard_normal((6, 8)),
         "L1.wdown": rng.standard_normal((8, 6))}
    m = O.Model(s, w)
    h = rng.standard_normal((3, 8))
    got = O.mlp(m, 1, h)
    for r in range(3):
        a = []
        for i in range(6):
            g = sum(w["L1.wg"][i][c] * h[r][c] for c in range(8))
            u = sum(w["L1.wu"][i][c] * h[r][c] for c in range(8))
            a.append(g / (1 + math.exp(-g)) * u)
        for o in range(8):
            assert abs(got[r][o] - sum(w["L1.wdown"][o][i] * a[i] for i in range(6))) < 1e-12


# ---------------------------------------------------------------- closed forms
def _zero_io(m: O.Model):
    """Zero the output projections of the input and output blocks, so every
    layer there computes N(h + 0) = h."""
    for l in list(m.block("I")) + list(m.block("O")):
        m.w[f"L{l}.wo" if m.kind(l) == "attn" else f"L{l}.wdown"][:] = 0.0


def test_identity_blocks_give_back_the_token_and_ties_go_low():
    s = micro_shape(n_rec=2)
    m = O.Model(s, synth.make_weights(s, 4))
    for l in range(s.n_layers):
        m.w[f"L{l}.wo" if m.kind(l) == "attn" else f"L{l}.wdown"][:] = 0.0
    m.w["lm_head"] = m.w["embed"].copy()
    for tok in range(s.vocab):
        for k in (1, 3):
            lg = O.forward_chunk(m, O.Cache(m, 4), [tok], k, O.LAST_LOOP)
            assert int(O.argmax_lowest(lg[-1])) == tok
    m.w["lm_head"][3] = m.w["embed"][9]
    m.w["lm_head"][7] = m.w["embed"][9]
    lg = O.forward_chunk(m, O.Cache(m, 4), [9], 2, O.LAST_LOOP)
    assert int(O.argmax_lowest(lg[-1])) == 3


def _heads_matrix(m, l):
    """[q_dim, d] matrix that maps h to the per-head value vectors when each
    query head sees exactly one key (its own token)."""
    s = m.shape
    G = s.n_heads // s.n_kv_heads
    Wv = m.w[f"L{l}.wv"].reshape(s.n_kv_heads, s.head_dim, s.d_model)
    return np.concatenate([Wv[hh // G] for hh in range(s.n_heads)], 0)


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_loop_recurrence_closed_form(k):
    """One token, input/output blocks zeroed, recurrent block = one attention
    layer (one key, so attention returns v) + one zeroed MLP layer:
    F(u) = N(u + A u) with A = W_o V, and s_t follows the recurrence."""
    s = micro_shape(n_rec=2, full_every=1, full_phase=0)
    m = O.Model(s, synth.make_weights(s, 7))
    _zero_io(m)
    m.w["L3.wdown"][:] = 0.0
    A = m.w["L2.wo"] @ _heads_matrix(m, 2)
    tok = 5
    nrm = lambda v: v / np.linalg.norm(v)
    x = nrm(m.w["embed"][tok])  # the zeroed input block still applies N
    st = x
    for _ in range(k):
        u = nrm(st + x)
        st = nrm(u + A @ u)
    want = m.w["lm_head"] @ st
    for mode in (O.LAST_LOOP, O.PER_LOOP):
        got = O.forward_chunk(m, O.Cache(m, 4), [tok], k, mode)[-1]
        assert np.abs(got - want).max() < 1e-13


@pytest.mark.parametrize("mode", [O.LAST_LOOP, O.PER_LOOP])
def test_two_token_loop_cache_semantics(mode):
    """Token a, then token b decoded at k=2.  In loop t, b sees a's keys from
    the final loop (last_loop) or from loop t (per_loop), plus its own."""
    s = micro_shape(n_rec=2, full_every=1, full_phase=0, n_heads=2, n_kv_heads=2)
    m = O.Model(s, synth.make_weights(s, 11))
    _zero_io(m)
    m.w["L3.wdown"][:] = 0.0
    Wq, Wk, Wv, Wo = (m.w[f"L2.{n}"] for n in ("wq", "wk", "wv", "wo"))
    nrm = lambda v: v / np.linalg.norm(v)
    hd = s.head_dim

    def attn(u, keys, vals):
        q = Wq @ u
        out = np.zeros(s.q_dim)
        for h in range(2):
            sc = [float(q[h * hd:(h + 1) * hd] @ kk[h * hd:(h + 1) * hd]) / math.sqrt(hd) for kk in keys]
            mx = max(sc)
            e = [math.exp(c - mx) for c in sc]
            for j, vv in enumerate(vals):
                out[h * hd:(h + 1) * hd] += e[j] / sum(e) * vv[h * hd:(h + 1) * hd]
        return Wo @ out

    a_tok, b_tok = 2, 9
    xa, xb = nrm(m.w["embed"][a_tok]), nrm(m.w["embed"][b_tok])
    # token a alone: per-loop K/V of a
    kv_a = []
    st = xa
    for _ in range(2):
        u = nrm(st + xa)
        kv_a.append((Wk @ u, Wv @ u))
        st = nrm(u + attn(u, [Wk @ u], [Wv @ u]))
    st = xb
    for t in range(2):
        u = nrm(st + xb)
        ka, va = kv_a[1] if mode == O.LAST_LOOP else kv_a[t]
        st = nrm(u + attn(u, [ka, Wk @ u], [va, Wv @ u]))
    want = m.w["lm_head"] @ st
    c = O.Cache(m, 4)
    O.forward_chunk(m, c, [a_tok], 2, mode)
    got = O.forward_chunk(m, c, [b_tok], 2, mode)[-1]
    assert np.abs(got - want).max() < 1e-13


# ---------------------------------------------------------------- speculative
def test_spec_per_loop_equals_plain_verify_k(tiny, prompt):
    sp = FACTS["self_speculative"]["value"]
    toks, st = O.spec_generate(tiny, prompt, 24, sp["k_draft"], sp["k_verify"], sp["gamma"], O.PER_LOOP)
    plain, _ = O.generate(tiny, prompt, 24, sp["k_verify"], O.PER_LOOP)
    assert np.array_equal(toks, plain)
    assert all(0 <= n <= sp["gamma"] for n in st.accepted_per_step)


def test_spec_last_loop_runs_and_counts(tiny, prompt):
    toks, st = O.spec_generate(tiny, prompt[:30], 20, 1, 4, 4, O.LAST_LOOP)
    assert len(toks) == 20 and st.steps >= 4
    assert st.accepted == sum(st.accepted_per_step) and st.drafted == 4 * st.steps


def test_unwritten_key_is_an_error(tiny, prompt):
    """per_loop slots of loops a call did not run hold nothing to read."""
    c = O.Cache(tiny, 80)
    O.forward_chunk(tiny, c, prompt[:8], 1, O.PER_LOOP)
    with pytest.raises(RuntimeError):
        O.forward_chunk(tiny, c, prompt[8:9], 2, O.PER_LOOP)


def test_norm_floor():
    assert np.array_equal(O.l2n(np.zeros((2, 3))), np.zeros((2, 3)))


# ---------------------------------------------------------------- relabelling invariances
def relabelled(model, perm_d=None, perm_ff=None, perm_kv=None, perm_in_group=None):
    """The same network with its hidden units renamed: perm_d on the model width
    (embedding and head columns, every input column and every output row onto
    the residual stream), perm_ff on the MLP hidden units (gate and up rows,
    down columns), perm_kv on the KV heads together with their query groups,
    perm_in_group on the query heads inside every group.  The logits must not
    change."""
    s = model.shape
    d, hd, G = s.d_model, s.head_dim, s.n_heads // s.n_kv_heads
    w = {k: v.copy() for k, v in model.w.items()}
    qh = np.arange(s.n_heads)
    if perm_kv is not None or perm_in_group is not None:
        kv = perm_kv if perm_kv is not None else np.arange(s.n_kv_heads)
        ig = perm_in_group if perm_in_group is not None else np.arange(G)
        qh = np.array([kv[h // G] * G + ig[h % G] for h in range(s.n_heads)])  # new head h <- old head qh[h]
    else:
        kv = np.arange(s.n_kv_heads)
    q_rows = np.concatenate([np.arange(o * hd, (o + 1) * hd) for o in qh])
    kv_rows = np.concatenate([np.arange(o * hd, (o + 1) * hd) for o in kv])
    for l in range(s.n_layers):
        if model.kind(l) == "attn":
            w[f"L{l}.wq"] = w[f"L{l}.wq"][q_rows]
            w[f"L{l}.wk"] = w[f"L{l}.wk"][kv_rows]
            w[f"L{l}.wv"] = w[f"L{l}.wv"][kv_rows]
            w[f"L{l}.wo"] = w[f"L{l}.wo"][:, q_rows]
        elif perm_ff is not None:
            w[f"L{l}.wg"] = w[f"L{l}.wg"][perm_ff]
            w[f"L{l}.wu"] = w[f"L{l}.wu"][perm_ff]
            w[f"L{l}.wdown"] = w[f"L{l}.wdown"][:, perm_ff]
    if perm_d is not None:
        for name in list(w):
            if name in ("embed", "lm_head") or name.endswith((".wq", ".wk", ".wv", ".wg", ".wu")):
                w[name] = w[name][:, perm_d]
            elif name.endswith((".wo", ".wdown")):
                w[name] = w[name][perm_d]
    m = O.Model(s, {})
    m.w = w
    return m


@pytest.mark.parametrize("what", ["width", "mlp_hidden", "kv_heads", "heads_in_group", "all"])
@pytest.mark.parametrize("mode", [O.LAST_LOOP, O.PER_LOOP])
def test_renaming_hidden_units_leaves_the_logits_unchanged(tiny, prompt, what, mode):
    s = synth.TINY
    rng = np.random.default_rng(11)
    kw = {}
    if what in ("width", "all"):
        kw["perm_d"] = rng.permutation(s.d_model)
    if what in ("mlp_hidden", "all"):
        kw["perm_ff"] = rng.permutation(s.d_ff)
    if what in ("kv_heads", "all"):  # a cyclic shift: never the identity
        kw["perm_kv"] = np.roll(np.arange(s.n_kv_heads), 1)
    if what in ("heads_in_group", "all"):
        kw["perm_in_group"] = np.roll(np.arange(s.n_heads // s.n_kv_heads), 1)
    other = relabelled(tiny, **kw)
    a = O.forward_chunk(tiny, O.Cache(tiny, 40), prompt[:24], 2, mode, head="all")
    b = O.forward_chunk(other, O.Cache(other, 40), prompt[:24], 2, mode, head="all")
    assert np.abs(a - b).max() < 1e-12
