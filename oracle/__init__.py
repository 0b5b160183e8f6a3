"""Oracle (test infrastructure only): plain CPU definition of the looped nGPT
forward.  Imported by tests, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU legs; never by the CUDA library or its binding."""
from .looped_ngpt import (  # noqa: F401
    LAST_LOOP,
    PER_LOOP,
    Cache,
    Model,
    SpecStats,
    argmax_lowest,
    attention,
    forward_chunk,
    generate,
    kv_bytes,
    l2n,
    mlp,
    run_layers,
    silu,
    spec_generate,
)
