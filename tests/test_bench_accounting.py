"""The bench's roofline numerators (CPU): weight bytes, KV bytes and FLOPs per
step, checked against independent enumerations.  Weights come from the
synthetic tensor list, layer kinds and loops from the oracle's layer rules,
and visible attention pairs from brute force.  The layer-application counts
are pinned to the pages' 72 / 112 / 192."""
import numpy as np
import pytest

import bench
import oracle as O
import synth

SHAPES = [synth.DORY_4B, synth.TINY_BF16, synth.SMALL128]


def applications(model, k):
    """How many times one token applies each physical layer at loop count k."""
    n = np.zeros(model.shape.n_layers, dtype=np.int64)
    for l, _ in model.schedule(k):
        n[l] += 1
    return n


@pytest.mark.parametrize("k,total", [(1, 72), (2, 112), (4, 192)])
def test_layer_applications_match_the_pages(k, total):
    assert int(applications(O.Model(synth.DORY_4B, {}), k).sum()) == total


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("k", [1, 2, 4])
def test_weight_bytes_per_decode_step(shape, k):
    model = O.Model(shape, {})
    apps = applications(model, k)
    elems = 0
    for name, (rows, cols) in synth.weight_specs(shape):
        if name == "embed":
            elems += cols  # one gathered row per token
        elif name == "lm_head":
            elems += rows * cols
        else:
            elems += int(apps[int(name[1:].split(".")[0])]) * rows * cols
    assert bench.weight_bytes(shape, k) == 2 * elems


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("k", [1, 2, 4])
@pytest.mark.parametrize("ctx", [1, 17, 4096, 5000])
def test_kv_read_bytes_per_decode_step(shape, k, ctx):
    model = O.Model(shape, {})
    apps = applications(model, k)
    want = 0
    for l in range(shape.n_layers):
        if model.kind(l) != "attn":
            continue
        keys = ctx if model.is_full(l) else min(ctx, shape.swa_window)
        want += int(apps[l]) * keys * 2 * shape.n_kv_heads * shape.head_dim * 2  # K and V, bf16
    assert bench.kv_read_bytes(shape, k, ctx) == want


@pytest.mark.parametrize("k", [1, 2, 4])
def test_projection_flops(k):
    shape = synth.DORY_4B
    apps = applications(O.Model(shape, {}), k)
    macs = 0
    for name, (rows, cols) in synth.weight_specs(shape):
        if name.startswith("L"):
            macs += int(apps[int(name[1:].split(".")[0])]) * rows * cols
    assert bench.proj_flops(shape, k, 3) == 2 * 3 * macs


@pytest.mark.parametrize("T", [1, 5, 16, 40])
@pytest.mark.parametrize("k", [1, 2])
def test_prefill_attention_flops_by_brute_force(T, k):
    shape = synth.TINY_BF16  # window 16
    model = O.Model(shape, {})
    apps = applications(model, k)
    want = 0
    for l in range(shape.n_layers):
        if model.kind(l) != "attn":
            continue
        for p in range(T):
            for j in range(T):
                visible = j <= p and (model.is_full(l) or p - j < shape.swa_window)
                if visible:
                    want += int(apps[l]) * 4 * shape.n_heads * shape.head_dim  # QK^T and PV, 2 FLOP per MAC
    assert bench.attn_flops_prefill(shape, k, T) == want


def test_4b_decode_step_bytes_at_the_bench_context():
    # 7.47 / 11.24 / 18.79 GB of weights per token at k = 1 / 2 / 4 (2560-token prompt context)
    gb = [bench.weight_bytes(synth.DORY_4B, k) / 1e9 for k in (1, 2, 4)]
    assert [round(v, 2) for v in gb] == [7.47, 11.24, 18.79]
