"""C-ABI checks that need no GPU: exported symbols, workspace sizing, KV byte
accounting against the oracle, and argument validation (which runs before
any device work, so a fake workspace address is enough)."""
import ctypes
import os
import re

import pytest

import oracle as O
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

dory = pytest.importorskip("looped_ngpt_lm_b200")
lib = dory.lib
FAKE_WS = 1 << 40  # never dereferenced: validation fails before any launch


def header_functions():
    src = open(os.path.join(ROOT, "include", "dory.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dory_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_function_is_exported():
    names = header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(dory.SYMBOLS) == names


def cfg_for(shape, **kw):
    args = dict(max_batch=2, max_seq=128, k_max=4, gamma_max=4, max_chunk=96)
    args.update(kw)
    return dory.make_config(shape, **args)


def fake_handle(shape, alloc=dory.PER_LOOP, **kw):
    cfg = cfg_for(shape, **kw)
    n = dory.workspace_size(cfg, alloc)
    L = shape.n_layers
    arr = ctypes.c_void_p * L
    fake = arr(*([FAKE_WS] * L))
    w = dory.Weights(FAKE_WS, FAKE_WS, fake, fake, fake, fake)
    h = ctypes.c_void_p()
    st = lib.dory_create(ctypes.byref(cfg), ctypes.byref(w), alloc, ctypes.c_void_p(FAKE_WS), n, ctypes.byref(h))
    assert st == 0, lib.dory_last_error(None)
    return h, cfg, (cfg, w, fake)


def test_workspace_grows_with_per_loop_slots():
    a = dory.workspace_size(cfg_for(synth.TINY), dory.LAST_LOOP)
    b = dory.workspace_size(cfg_for(synth.TINY), dory.PER_LOOP)
    c = dory.workspace_size(cfg_for(synth.TINY, k_max=2), dory.PER_LOOP)
    assert 0 < a < c < b


def test_4b_workspace_is_kv_dominated_and_fits():
    cfg = cfg_for(synth.DORY_4B, max_batch=1, max_seq=2560 + 300 + 16, max_chunk=2560)
    n = dory.workspace_size(cfg, dory.LAST_LOOP)
    assert n < 16e9


@pytest.mark.parametrize("shape", [synth.TINY, synth.DORY_4B])
def test_kv_bytes_match_oracle(shape):
    h, cfg, keep = fake_handle(shape, max_seq=8192, max_chunk=64)
    m = O.Model(shape, {})
    esz = 2 if shape.dtype == "bf16" else 4
    for mode, cmode in ((O.LAST_LOOP, dory.LAST_LOOP), (O.PER_LOOP, dory.PER_LOOP)):
        for k in (1, 2, 4):
            for ctx in (1, 15, 16, 17, 100, 5000):
                n = ctypes.c_int64()
                assert lib.dory_kv_bytes(h, k, cmode, ctx, ctypes.byref(n)) == 0
                assert n.value == O.kv_bytes(m, k, mode, ctx, esz), (mode, k, ctx)
    lib.dory_destroy(h)


def status_name(s):
    return dory.STATUS[s]


def test_argument_validation():
    h, cfg, keep = fake_handle(synth.TINY, alloc=dory.LAST_LOOP)
    ids = (ctypes.c_int32 * 2)(0, 1)
    lens = (ctypes.c_int32 * 2)(4, 4)
    tok = ctypes.c_void_p(FAKE_WS)
    nt = ctypes.c_void_p(FAKE_WS)
    P = lambda *a: status_name(lib.dory_prefill(h, *a))
    assert P(2, ids, tok, lens, 0, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"       # k = 0
    assert P(2, ids, tok, lens, 5, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"       # k > k_max
    assert P(2, ids, tok, lens, 2, 1, None, nt, None) == "DORY_ERR_STATE"             # per_loop on last_loop handle
    assert P(3, ids, tok, lens, 2, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"       # batch > max_batch
    dup = (ctypes.c_int32 * 2)(1, 1)
    assert P(2, dup, tok, lens, 2, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"       # repeated id
    bad = (ctypes.c_int32 * 2)(0, 7)
    assert P(2, bad, tok, lens, 2, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"       # id out of range
    big = (ctypes.c_int32 * 2)(60, 60)
    assert P(2, ids, tok, big, 2, 0, None, nt, None) == "DORY_ERR_CAPACITY"           # > max_chunk
    zero = (ctypes.c_int32 * 2)(0, 3)
    assert P(2, ids, tok, zero, 2, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"       # empty sequence
    over = (ctypes.c_int32 * 1)(129)
    assert P(1, ids, tok, over, 2, 0, None, nt, None) == "DORY_ERR_CAPACITY"          # > max_seq
    S = lambda *a: status_name(lib.dory_spec_decode(h, *a))
    out = ctypes.c_void_p(FAKE_WS)
    assert S(1, ids, tok, 2, 4, 4, 0, 8, out, out, None, None) == "DORY_ERR_UNSUPPORTED"  # k_draft != 1
    assert S(1, ids, tok, 1, 4, 5, 0, 8, out, out, None, None) == "DORY_ERR_INVALID_ARG"  # gamma > gamma_max
    assert S(1, ids, tok, 1, 4, 4, 0, 8, out, out, None, None) == "DORY_ERR_STATE"        # no prefill yet
    D = lambda *a: status_name(lib.dory_decode_step(h, *a))
    assert D(1, ids, tok, 9, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"
    assert D(1, ids, None, 2, 0, None, nt, None) == "DORY_ERR_INVALID_ARG"
    X = lambda ks, mode=0: status_name(lib.dory_decode_step_mixed(h, len(ks), ids, tok, (ctypes.c_int32 * len(ks))(*ks),
                                                                  mode, None, nt, None))
    assert X([1, 2]) == "DORY_ERR_INVALID_ARG"      # k increases along the batch
    assert X([5, 1]) == "DORY_ERR_INVALID_ARG"      # k > k_max
    assert X([2, 0]) == "DORY_ERR_INVALID_ARG"      # k = 0
    assert X([2, 1], 1) == "DORY_ERR_STATE"         # per_loop on a last_loop handle
    assert status_name(lib.dory_decode_step_mixed(h, 2, dup, tok, (ctypes.c_int32 * 2)(2, 1), 0, None, nt,
                                                  None)) == "DORY_ERR_INVALID_ARG"  # repeated id
    assert lib.dory_set_option(h, 99, 1) == 1
    n = ctypes.c_int32()
    assert lib.dory_seq_len(h, 0, ctypes.byref(n)) == 0 and n.value == 0
    assert lib.dory_read_state(h, 0, ctypes.c_void_p(FAKE_WS), 1, None) == 1  # nothing computed yet
    assert b"rows" in lib.dory_last_error(None)
    lib.dory_destroy(h)


def test_mxfp8_argument_validation():
    F, F8 = ctypes.c_void_p(FAKE_WS), ctypes.c_void_p(FAKE_WS + 8)
    G = lambda *a, impl=0: status_name(lib.dory_gemv_mxfp8(*a, impl, None, None))
    assert G(1, 8, 48, F, 48, F, F, F, 8) == "DORY_ERR_UNSUPPORTED"    # K % 32
    assert G(1, 8, 40992, F, 40992, F, F, F, 8) == "DORY_ERR_UNSUPPORTED"  # staged activations too large
    assert G(1, 8, 10272, F, 10272, F, F, F, 8, impl=2) == "DORY_ERR_UNSUPPORTED"  # tensor cores: K <= 10240
    assert G(1, 8, 64, F, 64, F, F, F, 8, impl=5) == "DORY_ERR_INVALID_ARG"
    assert G(1, 100, 128, F, 128, F, F, F, 100, impl=3) == "DORY_ERR_UNSUPPORTED"   # N % 128
    assert G(1, 128, 96, F, 96, F, F, F, 128, impl=3) == "DORY_ERR_UNSUPPORTED"    # K % 128
    assert G(1, 128, 128, F8, 128, F, F, F, 128, impl=3) == "DORY_ERR_UNSUPPORTED"  # x not 16-byte aligned
    assert G(1, 8, 64, F, 32, F, F, F, 8) == "DORY_ERR_INVALID_ARG"    # ldx < K
    assert G(1, 8, 64, F, 64, F, F, F, 4) == "DORY_ERR_INVALID_ARG"    # ldy < N
    assert G(1, 8, 64, F, 64, F8, F, F, 8) == "DORY_ERR_INVALID_ARG"   # codes not 16-byte aligned
    assert G(0, 8, 64, F, 64, F, F, F, 8) == "DORY_ERR_INVALID_ARG"    # no rows
    Q = lambda *a: status_name(lib.dory_quantize_mxfp8(*a, None, None))
    assert Q(F, 4, 40, F, F, None) == "DORY_ERR_UNSUPPORTED"           # K % 32
    assert Q(F8, 4, 64, F, F, None) == "DORY_ERR_INVALID_ARG"          # weights not 16-byte aligned
    assert Q(F, 4, 64, F, F, F8) == "DORY_ERR_INVALID_ARG"             # dequantised output not aligned
    assert Q(F, 0, 64, F, F, None) == "DORY_ERR_INVALID_ARG"
    A = lambda h, mx: status_name(lib.dory_attach_mxfp8(h, mx))
    h32, _, keep32 = fake_handle(synth.TINY)
    L = synth.TINY.n_layers
    arr = (ctypes.c_void_p * L)(*([FAKE_WS] * L))
    full = dory.MxWeightsC(FAKE_WS, FAKE_WS, *([arr] * 8))
    assert A(h32, full) == "DORY_ERR_UNSUPPORTED"  # fp32 weights
    assert A(h32, None) == "DORY_OK"
    hb, _, keepb = fake_handle(synth.TINY_BF16)
    assert A(hb, dory.MxWeightsC(FAKE_WS, None, *([arr] * 8))) == "DORY_ERR_INVALID_ARG"  # codes without scales
    assert A(hb, dory.MxWeightsC(FAKE_WS + 8, FAKE_WS, *([arr] * 8))) == "DORY_ERR_INVALID_ARG"  # misaligned
    assert A(hb, full) == "DORY_OK"
    assert A(hb, dory.MxWeightsC(None, None, None, None, None, None, None, None, None, None)) == "DORY_OK"
    assert A(hb, None) == "DORY_OK"
    assert lib.dory_set_option(hb, dory.OPT_MX_GEMV, 3) == 0
    assert lib.dory_set_option(hb, dory.OPT_MX_GEMV, 4) == 0
    assert lib.dory_set_option(hb, dory.OPT_MX_GEMV, 5) == 1
    # NVFP4
    NQ = lambda *a: status_name(lib.dory_quantize_nvfp4(*a, None, None))
    assert NQ(F, 4, 40, F, F, F, None) == "DORY_ERR_UNSUPPORTED"       # K % 16
    assert NQ(F8, 4, 64, F, F, F, None) == "DORY_ERR_INVALID_ARG"      # weights not 16-byte aligned
    assert NQ(F, 4, 64, F, F, None, None) == "DORY_ERR_INVALID_ARG"    # no tensor scale
    NG = lambda *a: status_name(lib.dory_gemm_nvfp4(*a, None, None))
    assert NG(1, 100, 256, F, 256, F, F, F, F, 100) == "DORY_ERR_UNSUPPORTED"  # N % 128
    assert NG(1, 128, 128, F, 128, F, F, F, F, 128) == "DORY_ERR_UNSUPPORTED"  # K % 256
    assert NG(1, 128, 256, F, 256, F, F, None, F, 128) == "DORY_ERR_INVALID_ARG"  # no tensor scale
    NA = lambda h, nv: status_name(lib.dory_attach_nvfp4(h, nv))
    nv_full = dory.NvWeightsC(FAKE_WS, FAKE_WS, FAKE_WS, *([arr] * 12))
    assert NA(h32, nv_full) == "DORY_ERR_UNSUPPORTED"  # fp32 weights
    assert NA(hb, dory.NvWeightsC(FAKE_WS, FAKE_WS, None, *([arr] * 12))) == "DORY_ERR_INVALID_ARG"  # no g
    assert NA(hb, nv_full) == "DORY_OK"
    assert NA(hb, None) == "DORY_OK"
    lib.dory_destroy(h32)
    lib.dory_destroy(hb)


def test_create_rejects_bad_workspace_and_config():
    cfg = cfg_for(synth.TINY)
    n = dory.workspace_size(cfg, dory.LAST_LOOP)
    L = synth.TINY.n_layers
    fake = (ctypes.c_void_p * L)(*([FAKE_WS] * L))
    w = dory.Weights(FAKE_WS, FAKE_WS, fake, fake, fake, fake)
    h = ctypes.c_void_p()
    assert lib.dory_create(ctypes.byref(cfg), ctypes.byref(w), 0, ctypes.c_void_p(FAKE_WS), n - 1,
                           ctypes.byref(h)) == 4
    assert lib.dory_create(ctypes.byref(cfg), ctypes.byref(w), 0, ctypes.c_void_p(FAKE_WS + 8), n,
                           ctypes.byref(h)) == 4
    bad = dory.make_config(synth.TINY.with_(head_dim=48))
    assert lib.dory_workspace_size(ctypes.byref(bad), 0, ctypes.byref(ctypes.c_size_t())) == 7
    bad = dory.make_config(synth.TINY.with_(n_kv_heads=3))
    assert lib.dory_workspace_size(ctypes.byref(bad), 0, ctypes.byref(ctypes.c_size_t())) == 1


def test_paged_full_attention_cache_sizes_the_pool_not_every_slot():
    """A page pool for the full-attention layers replaces max_batch linear
    arrays of max_seq positions: 8 slots of 262,144 positions with a pool for
    one such sequence (plus short ones) is several times smaller."""
    s = synth.DORY_4B  # 9 full-attention layers, one cache slot each in last_loop mode
    big = dict(max_batch=8, max_seq=262144, max_chunk=8192)
    pages = 262144 // 64 + 7 * 64
    linear = dory.workspace_size(cfg_for(s, **big), dory.LAST_LOOP)
    paged = dory.workspace_size(cfg_for(s, kv_page=64, kv_pages=pages, **big), dory.LAST_LOOP)
    full = dory.workspace_size(cfg_for(s, kv_page=64, **big), dory.LAST_LOOP)  # default pool: every slot full
    per_pos = 2 * s.kv_dim * 2  # K and V bytes of one position in one layer
    saved = 9 * (8 * 262144 - pages * 64) * per_pos
    table = 8 * (262144 // 64) * 4
    assert abs((linear - paged) - (saved - table)) < 64 * 1024
    assert abs(full - linear - table) < 64 * 1024
    assert paged < linear / 3


@pytest.mark.parametrize("page", [8, 48, 8192])
def test_bad_page_sizes_are_rejected(page):
    cfg = cfg_for(synth.TINY, kv_page=page)
    n = ctypes.c_size_t()
    assert lib.dory_workspace_size(ctypes.byref(cfg), dory.LAST_LOOP, ctypes.byref(n)) == 1
    assert b"kv_page" in lib.dory_last_error(None)


def test_page_pool_exhaustion_is_a_capacity_error_before_any_work():
    """Two 16-position pages for a 48-token prompt: refused before launch,
    with nothing changed (the same call then fits after a reset frees pages)."""
    h, cfg, keep = fake_handle(synth.TINY, kv_page=16, kv_pages=2)
    ids = (ctypes.c_int32 * 1)(0)
    lens = (ctypes.c_int32 * 1)(48)
    st = lib.dory_prefill(h, 1, ids, ctypes.c_void_p(FAKE_WS), lens, 1, dory.LAST_LOOP, None,
                          ctypes.c_void_p(FAKE_WS), None)
    assert st == 2, lib.dory_last_error(None)
    assert b"pages" in lib.dory_last_error(None)
    n = ctypes.c_int32()
    assert lib.dory_seq_len(h, 0, ctypes.byref(n)) == 0 and n.value == 0
    lib.dory_destroy(h)
