"""Python binding of libdory.so (the looped nGPT C ABI declared in include/dory.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  PyTorch supplies device memory and streams.  Importing this
package fails loudly when the compiled library is missing; there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdory.so")

LAST_LOOP = 0
PER_LOOP = 1
F32 = 0
BF16 = 1
MODES = {"last_loop": LAST_LOOP, "per_loop": PER_LOOP, LAST_LOOP: LAST_LOOP, PER_LOOP: PER_LOOP}

OPT_CUDA_GRAPHS = 1
OPT_PROFILE = 2
OPT_GEMM_IMPL = 3
OPT_PDL = 4
OPT_PREFILL_TC = 5
OPT_ATTN_CLUSTER = 6
OPT_L2_LOOKAHEAD = 7
OPT_MX_GEMV = 8
OPT_FUSED_OPERANDS = 9
OPT_ATTN_LOOKAHEAD = 10
OPT_L2_OWN = 11

STATUS = {0: "DORY_OK", 1: "DORY_ERR_INVALID_ARG", 2: "DORY_ERR_CAPACITY", 3: "DORY_ERR_STATE",
          4: "DORY_ERR_WORKSPACE", 5: "DORY_ERR_CUDA", 6: "DORY_ERR_TIMEOUT", 7: "DORY_ERR_UNSUPPORTED"}

# Every entry point include/dory.h declares.
SYMBOLS = ["dory_workspace_size", "dory_create", "dory_destroy", "dory_reset", "dory_prefill",
           "dory_decode_step", "dory_decode_step_mixed", "dory_spec_decode", "dory_kv_bytes", "dory_seq_len", "dory_read_state",
           "dory_read_kv", "dory_synchronize", "dory_set_option", "dory_profile_read", "dory_profile_reset",
           "dory_last_error", "dory_gemm_bf16", "dory_gemm_bf16_noalloc", "dory_gemm_bf16_noalloc_status",
           "dory_pack_weight_bf16",
           "dory_set_sampling", "dory_sample", "dory_quantize_mxfp8", "dory_gemv_mxfp8", "dory_attach_mxfp8",
           "dory_quantize_nvfp4", "dory_gemm_nvfp4", "dory_attach_nvfp4"]


class DoryError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "d_model", "vocab", "n_heads", "head_dim", "n_kv_heads", "d_ff", "n_in", "n_rec", "n_out",
        "swa_window", "full_every", "full_phase", "dtype", "max_batch", "max_seq", "k_max", "gamma_max",
        "max_chunk", "kv_page", "kv_pages")]


class Weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("w_qkv", ctypes.POINTER(ctypes.c_void_p)), ("w_o", ctypes.POINTER(ctypes.c_void_p)),
                ("w_gu", ctypes.POINTER(ctypes.c_void_p)), ("w_down", ctypes.POINTER(ctypes.c_void_p))]


class MxWeightsC(ctypes.Structure):
    _fields_ = [("lm_head_q", ctypes.c_void_p), ("lm_head_s", ctypes.c_void_p)] + [
        (n, ctypes.POINTER(ctypes.c_void_p)) for n in (
            "qkv_q", "qkv_s", "o_q", "o_s", "gu_q", "gu_s", "down_q", "down_s")]


class NvWeightsC(ctypes.Structure):
    _fields_ = [("lm_head_q", ctypes.c_void_p), ("lm_head_s", ctypes.c_void_p), ("lm_head_g", ctypes.c_void_p)]
    for _n in ("qkv", "o", "gu", "down"):
        _fields_ += [(f"{_n}_q", ctypes.POINTER(ctypes.c_void_p)), (f"{_n}_s", ctypes.POINTER(ctypes.c_void_p)),
                     (f"{_n}_g", ctypes.POINTER(ctypes.c_void_p))]
    del _n


class SpecStats(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_int64), ("drafted", ctypes.c_int64), ("accepted", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python looped_ngpt_lm_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    IP = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "dory_workspace_size": [ctypes.POINTER(Config), I32, ctypes.POINTER(SZ)],
        "dory_create": [ctypes.POINTER(Config), ctypes.POINTER(Weights), I32, P, SZ, ctypes.POINTER(P)],
        "dory_destroy": [P],
        "dory_reset": [P, I32, P],
        "dory_prefill": [P, I32, IP, P, IP, I32, I32, P, P, P],
        "dory_decode_step": [P, I32, IP, P, I32, I32, P, P, P],
        "dory_decode_step_mixed": [P, I32, IP, P, IP, I32, P, P, P],
        "dory_spec_decode": [P, I32, IP, P, I32, I32, I32, I32, I32, P, P, ctypes.POINTER(SpecStats), P],
        "dory_kv_bytes": [P, I32, I32, I64, ctypes.POINTER(I64)],
        "dory_seq_len": [P, I32, IP],
        "dory_read_state": [P, I32, P, I32, P],
        "dory_read_kv": [P, I32, I32, I32, I32, I32, P, P, P],
        "dory_synchronize": [P, P],
        "dory_set_option": [P, I32, I64],
        "dory_profile_read": [P, I32, P, ctypes.POINTER(I64), ctypes.POINTER(ctypes.c_double),
                              ctypes.POINTER(ctypes.c_double), IP],
        "dory_profile_reset": [P],
        "dory_gemm_bf16": [I32, I32, I32, P, P, P, I32, I32, I32, IP, P, P],
        "dory_gemm_bf16_noalloc": [I32, I32, I32, P, P, P, I32, P],
        "dory_gemm_bf16_noalloc_status": [P],
        "dory_pack_weight_bf16": [P, P, I32, I32, P],
        "dory_set_sampling": [P, ctypes.c_float, ctypes.c_float, ctypes.c_uint64],
        "dory_sample": [P, I32, I32, P, P, ctypes.c_float, ctypes.c_float, ctypes.c_uint64, P, P, P],
        "dory_quantize_mxfp8": [P, I32, I32, P, P, P, P, P],
        "dory_gemv_mxfp8": [I32, I32, I32, P, I32, P, P, P, I32, I32, P, P],
        "dory_attach_mxfp8": [P, ctypes.POINTER(MxWeightsC)],
        "dory_quantize_nvfp4": [P, I32, I32, P, P, P, P, P, P],
        "dory_gemm_nvfp4": [I32, I32, I32, P, I32, P, P, P, P, I32, P, P],
        "dory_attach_nvfp4": [P, ctypes.POINTER(NvWeightsC)],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.dory_last_error.argtypes = [ctypes.c_void_p]
    lib.dory_last_error.restype = ctypes.c_char_p
    return lib


lib = _load()


def _check(status: int) -> None:
    if status != 0:
        raise DoryError(status, lib.dory_last_error(None).decode())


def make_config(shape, max_batch=1, max_seq=256, k_max=4, gamma_max=4, max_chunk=None, kv_page=0,
                kv_pages=0) -> Config:
    """C config for a synth.Shape plus capacity (kv_page > 0: paged
    full-attention cache with a pool of kv_pages pages)."""
    return Config(shape.d_model, shape.vocab, shape.n_heads, shape.head_dim, shape.n_kv_heads, shape.d_ff,
                  shape.n_in, shape.n_rec, shape.n_out, shape.swa_window, shape.full_every, shape.full_phase,
                  BF16 if shape.dtype == "bf16" else F32, max_batch, max_seq, k_max, gamma_max,
                  max_chunk if max_chunk is not None else max_seq, kv_page, kv_pages)


def _ptr(t) -> int:
    return t.data_ptr() if t is not None else None


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class DeviceWeights:
    """Model weights in device memory, packed into the C ABI's layout
    (q|k|v rows stacked into w_qkv, gate|up rows into w_gu)."""

    def __init__(self, shape, weights: dict, device="cuda"):
        import torch
        self.shape = shape
        self.bf16 = shape.dtype == "bf16"

        def up(a):
            if self.bf16:
                t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
            else:
                t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
            return t.to(device, non_blocking=False)

        self.tensors = {"embed": up(weights["embed"]), "lm_head": up(weights["lm_head"])}
        L = shape.n_layers
        self.qkv, self.o, self.gu, self.down = [None] * L, [None] * L, [None] * L, [None] * L
        for l in range(L):
            if f"L{l}.wq" in weights:
                self.qkv[l] = up(np.concatenate([weights[f"L{l}.wq"], weights[f"L{l}.wk"], weights[f"L{l}.wv"]]))
                self.o[l] = up(weights[f"L{l}.wo"])
            else:
                self.gu[l] = up(np.concatenate([weights[f"L{l}.wg"], weights[f"L{l}.wu"]]))
                self.down[l] = up(weights[f"L{l}.wdown"])
        self._bind()

    @classmethod
    def from_tensors(cls, shape, embed, lm_head, qkv, o, gu, down):
        """Device weights from CUDA tensors already in the ABI layout."""
        self = cls.__new__(cls)
        self.shape = shape
        self.bf16 = shape.dtype == "bf16"
        self.tensors = {"embed": embed, "lm_head": lm_head}
        self.qkv, self.o, self.gu, self.down = list(qkv), list(o), list(gu), list(down)
        self._bind()
        return self

    def matrices(self):
        """(name, tensor) of every projection matrix and the LM head."""
        out = [("lm_head", self.tensors["lm_head"])]
        for l in range(self.shape.n_layers):
            for name, t in (("qkv", self.qkv[l]), ("o", self.o[l]), ("gu", self.gu[l]), ("down", self.down[l])):
                if t is not None:
                    out.append((f"{name}{l}", t))
        return out

    def _bind(self):
        L = self.shape.n_layers
        arr = ctypes.c_void_p * L
        self._qkv = arr(*[_ptr(t) for t in self.qkv])
        self._o = arr(*[_ptr(t) for t in self.o])
        self._gu = arr(*[_ptr(t) for t in self.gu])
        self._down = arr(*[_ptr(t) for t in self.down])
        self.c = Weights(self.tensors["embed"].data_ptr(), self.tensors["lm_head"].data_ptr(),
                         self._qkv, self._o, self._gu, self._down)


def gemm_bf16(X, W, batch_hint=1, invariant=True, impl=0, err=None, stream=None):
    """Y = X . W^T through dory_gemm_bf16 (X [M, K], W [N, K] bf16 CUDA
    tensors).  Returns (Y fp32 [M, N], splits); Y is the in-order sum of the
    kernel's split-K slices."""
    import torch
    M, K = X.shape
    N = W.shape[0]
    Y = torch.empty((8, M, N), dtype=torch.float32, device=X.device)
    s = ctypes.c_int32()
    _check(lib.dory_gemm_bf16(M, N, K, ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                              ctypes.c_void_p(Y.data_ptr()), batch_hint, int(invariant), impl, ctypes.byref(s),
                              ctypes.c_void_p(_ptr(err)), _stream(stream)))
    out = Y[0].clone()
    for i in range(1, s.value):
        out += Y[i]
    return out, s.value


def gemm_bf16_into(X, W, Y, batch_hint=1, invariant=True, impl=0, err=None, stream=None) -> int:
    """dory_gemm_bf16 into a caller buffer Y (fp32, >= 8*M*N); returns the
    number of split slices."""
    M, K = X.shape
    N = W.shape[0]
    s = ctypes.c_int32()
    _check(lib.dory_gemm_bf16(M, N, K, ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                              ctypes.c_void_p(Y.data_ptr()), batch_hint, int(invariant), impl, ctypes.byref(s),
                              ctypes.c_void_p(_ptr(err)), _stream(stream)))
    return s.value


def pack_weight_bf16(W, stream=None):
    """Packed tile layout copy of a row-major [N, K] bf16 CUDA tensor."""
    import torch
    N, K = W.shape
    out = torch.empty((N, K), dtype=torch.bfloat16, device=W.device)
    _check(lib.dory_pack_weight_bf16(ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(out.data_ptr()), N, K,
                                     _stream(stream)))
    return out


def quantize_mxfp8(W, dequantised=True, err=None, stream=None):
    """MXFP8 copy of a row-major [N, K] bf16 CUDA tensor: (codes uint8 [N, K],
    scales uint8 [N, K/32], dequantised bf16 [N, K] or None)."""
    import torch
    N, K = W.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    sc = torch.empty((N, K // 32), dtype=torch.uint8, device=W.device)
    deq = torch.empty((N, K), dtype=torch.bfloat16, device=W.device) if dequantised else None
    _check(lib.dory_quantize_mxfp8(ctypes.c_void_p(W.data_ptr()), N, K, ctypes.c_void_p(q.data_ptr()),
                                   ctypes.c_void_p(sc.data_ptr()), ctypes.c_void_p(_ptr(deq)),
                                   ctypes.c_void_p(_ptr(err)), _stream(stream)))
    return q, sc, deq


def gemv_mxfp8(X, q, scales, Y=None, impl=0, err=None, stream=None):
    """Y = X . dequantize(q, scales)^T through dory_gemv_mxfp8 (X bf16 [M, K];
    impl 0 default (= 1), 1 CUDA cores, 2 tensor cores)."""
    import torch
    M, K = X.shape
    N = q.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    _check(lib.dory_gemv_mxfp8(M, N, K, ctypes.c_void_p(X.data_ptr()), X.stride(0), ctypes.c_void_p(q.data_ptr()),
                               ctypes.c_void_p(scales.data_ptr()), ctypes.c_void_p(Y.data_ptr()), Y.stride(0),
                               impl, ctypes.c_void_p(_ptr(err)), _stream(stream)))
    return Y


class MxWeights:
    """MXFP8 copies of a DeviceWeights' projection matrices and LM head
    (made on the GPU by dory_quantize_mxfp8), plus `dequantised`: a
    DeviceWeights holding their exact bf16 dequantisation (same embedding)
    for the handle's prefill GEMMs."""

    def __init__(self, dw: DeviceWeights, stream=None):
        self.shape = dw.shape
        L = dw.shape.n_layers
        self.q, self.s = {}, {}
        deq = {}
        for name, t in dw.matrices():
            self.q[name], self.s[name], deq[name] = quantize_mxfp8(t, stream=stream)
        pick = lambda kind: [deq.get(f"{kind}{l}") for l in range(L)]  # noqa: E731
        self.dequantised = DeviceWeights.from_tensors(dw.shape, dw.tensors["embed"], deq["lm_head"], pick("qkv"),
                                                      pick("o"), pick("gu"), pick("down"))
        arr = ctypes.c_void_p * L

        def ptrs(d, kind):
            return arr(*[_ptr(d.get(f"{kind}{l}")) for l in range(L)])

        self._keep = {f"{k}_{x}": ptrs(d, k) for k in ("qkv", "o", "gu", "down") for x, d in (("q", self.q),
                                                                                                ("s", self.s))}
        self.c = MxWeightsC(self.q["lm_head"].data_ptr(), self.s["lm_head"].data_ptr(),
                            *[self._keep[f"{k}_{x}"] for k in ("qkv", "o", "gu", "down") for x in ("q", "s")])

    def nbytes(self) -> int:
        return sum(t.numel() for t in self.q.values()) + sum(t.numel() for t in self.s.values())


def quantize_nvfp4(W, dequantised=True, err=None, stream=None):
    """NVFP4 copy of a row-major [N, K] bf16 CUDA tensor: (code pairs uint8
    [N, K/2], E4M3 scales uint8 [N, K/16], tensor scale float32 [1] on the
    device, dequantised bf16 [N, K] or None)."""
    import torch
    N, K = W.shape
    q = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    sc = torch.empty((N, K // 16), dtype=torch.uint8, device=W.device)
    g = torch.empty(1, dtype=torch.float32, device=W.device)
    deq = torch.empty((N, K), dtype=torch.bfloat16, device=W.device) if dequantised else None
    _check(lib.dory_quantize_nvfp4(ctypes.c_void_p(W.data_ptr()), N, K, ctypes.c_void_p(q.data_ptr()),
                                   ctypes.c_void_p(sc.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                                   ctypes.c_void_p(_ptr(deq)), ctypes.c_void_p(_ptr(err)), _stream(stream)))
    return q, sc, g, deq


def gemm_nvfp4(X, q, scales, g, Y=None, err=None, stream=None):
    """Y = X . dequantize(q, scales, g)^T through dory_gemm_nvfp4 (X bf16 [M, K])."""
    import torch
    M, K = X.shape
    N = q.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    _check(lib.dory_gemm_nvfp4(M, N, K, ctypes.c_void_p(X.data_ptr()), X.stride(0), ctypes.c_void_p(q.data_ptr()),
                               ctypes.c_void_p(scales.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                               ctypes.c_void_p(Y.data_ptr()), Y.stride(0), ctypes.c_void_p(_ptr(err)),
                               _stream(stream)))
    return Y


class NvWeights:
    """NVFP4 copies of a DeviceWeights' projection matrices and LM head, plus
    `dequantised` (their exact bf16 dequantisation, same embedding)."""

    def __init__(self, dw: DeviceWeights, stream=None):
        self.shape = dw.shape
        L = dw.shape.n_layers
        self.q, self.s, self.g = {}, {}, {}
        deq = {}
        for name, t in dw.matrices():
            self.q[name], self.s[name], self.g[name], deq[name] = quantize_nvfp4(t, stream=stream)
        pick = lambda kind: [deq.get(f"{kind}{l}") for l in range(L)]  # noqa: E731
        self.dequantised = DeviceWeights.from_tensors(dw.shape, dw.tensors["embed"], deq["lm_head"], pick("qkv"),
                                                      pick("o"), pick("gu"), pick("down"))
        arr = ctypes.c_void_p * L
        self._keep = {f"{k}_{x}": arr(*[_ptr(d.get(f"{k}{l}")) for l in range(L)])
                      for k in ("qkv", "o", "gu", "down") for x, d in (("q", self.q), ("s", self.s), ("g", self.g))}
        self.c = NvWeightsC(self.q["lm_head"].data_ptr(), self.s["lm_head"].data_ptr(), self.g["lm_head"].data_ptr(),
                            *[self._keep[f"{k}_{x}"] for k in ("qkv", "o", "gu", "down") for x in ("q", "s", "g")])

    def nbytes(self) -> int:
        return sum(t.numel() for d in (self.q, self.s) for t in d.values()) + 4 * len(self.g)


def workspace_size(cfg: Config, alloc_mode=LAST_LOOP) -> int:
    n = ctypes.c_size_t()
    _check(lib.dory_workspace_size(ctypes.byref(cfg), MODES[alloc_mode], ctypes.byref(n)))
    return n.value


class Handle:
    """One dory_handle over a torch-allocated workspace."""

    def __init__(self, cfg: Config, weights: DeviceWeights, alloc_mode=LAST_LOOP, device="cuda"):
        import torch
        self.cfg = cfg
        self.weights = weights
        self.alloc_mode = MODES[alloc_mode]
        nbytes = workspace_size(cfg, self.alloc_mode)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        h = ctypes.c_void_p()
        _check(lib.dory_create(ctypes.byref(cfg), ctypes.byref(weights.c), self.alloc_mode,
                               ctypes.c_void_p(self.workspace.data_ptr()), nbytes, ctypes.byref(h)))
        self.h = h
        self.reset()

    def close(self):
        if self.h:
            lib.dory_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _ids(seq_ids):
        a = (ctypes.c_int32 * len(seq_ids))(*[int(s) for s in seq_ids])
        return a

    def reset(self, seq=-1, stream=None):
        _check(lib.dory_reset(self.h, seq, _stream(stream)))

    def set_option(self, opt, value):
        _check(lib.dory_set_option(self.h, opt, int(value)))

    def attach_mxfp8(self, mx: "MxWeights | None"):
        """Decode GEMMs read these MXFP8 copies (None detaches)."""
        self.mx = mx
        _check(lib.dory_attach_mxfp8(self.h, ctypes.byref(mx.c) if mx is not None else None))

    def attach_nvfp4(self, nv: "NvWeights | None"):
        """Decode GEMMs read these NVFP4 copies (None detaches)."""
        self.mx = nv
        _check(lib.dory_attach_nvfp4(self.h, ctypes.byref(nv.c) if nv is not None else None))

    def prefill(self, seq_ids, tokens, lens, k, mode, logits=None, next_tokens=None, stream=None):
        import torch
        ids = self._ids(seq_ids)
        ln = (ctypes.c_int32 * len(lens))(*[int(x) for x in lens])
        if next_tokens is None:
            next_tokens = torch.empty(len(seq_ids), dtype=torch.int32, device=tokens.device)
        _check(lib.dory_prefill(self.h, len(seq_ids), ids, ctypes.c_void_p(tokens.data_ptr()), ln, k, MODES[mode],
                                ctypes.c_void_p(_ptr(logits)), ctypes.c_void_p(next_tokens.data_ptr()),
                                _stream(stream)))
        return next_tokens

    def decode_step(self, seq_ids, tokens_in, k, mode, logits=None, next_tokens=None, stream=None):
        import torch
        ids = self._ids(seq_ids)
        if next_tokens is None:
            next_tokens = torch.empty(len(seq_ids), dtype=torch.int32, device=tokens_in.device)
        _check(lib.dory_decode_step(self.h, len(seq_ids), ids, ctypes.c_void_p(tokens_in.data_ptr()), k,
                                    MODES[mode], ctypes.c_void_p(_ptr(logits)),
                                    ctypes.c_void_p(next_tokens.data_ptr()), _stream(stream)))
        return next_tokens

    def set_sampling(self, temperature: float, top_p: float = 1.0, seed: int = 0):
        """temperature 0: greedy; > 0: top-p sampling with seeded per-token draws."""
        _check(lib.dory_set_sampling(self.h, temperature, top_p, seed))

    def decode_step_mixed(self, seq_ids, tokens_in, ks, mode, logits=None, next_tokens=None, stream=None):
        """One decode step with loop count ks[i] for sequence seq_ids[i] (ks non-increasing)."""
        import torch
        ids = self._ids(seq_ids)
        karr = (ctypes.c_int32 * len(ks))(*ks)
        if next_tokens is None:
            next_tokens = torch.empty(len(seq_ids), dtype=torch.int32, device=tokens_in.device)
        _check(lib.dory_decode_step_mixed(self.h, len(seq_ids), ids, ctypes.c_void_p(tokens_in.data_ptr()), karr,
                                          MODES[mode], ctypes.c_void_p(_ptr(logits)),
                                          ctypes.c_void_p(next_tokens.data_ptr()), _stream(stream)))
        return next_tokens

    def spec_decode(self, seq_ids, last_tokens, k_draft, k_verify, gamma, mode, max_new, stream=None):
        import torch
        ids = self._ids(seq_ids)
        B = len(seq_ids)
        out = torch.zeros((B, max_new), dtype=torch.int32, device=last_tokens.device)
        out_len = torch.zeros(B, dtype=torch.int32, device=last_tokens.device)
        st = SpecStats()
        _check(lib.dory_spec_decode(self.h, B, ids, ctypes.c_void_p(last_tokens.data_ptr()), k_draft, k_verify,
                                    gamma, MODES[mode], max_new, ctypes.c_void_p(out.data_ptr()),
                                    ctypes.c_void_p(out_len.data_ptr()), ctypes.byref(st), _stream(stream)))
        return out, out_len, {"steps": st.steps, "drafted": st.drafted, "accepted": st.accepted}

    def kv_bytes(self, k, mode, ctx) -> int:
        n = ctypes.c_int64()
        _check(lib.dory_kv_bytes(self.h, k, MODES[mode], ctx, ctypes.byref(n)))
        return n.value

    def seq_len(self, seq) -> int:
        n = ctypes.c_int32()
        _check(lib.dory_seq_len(self.h, seq, ctypes.byref(n)))
        return n.value

    def read_state(self, which, rows, stream=None):
        import torch
        out = torch.empty((rows, self.cfg.d_model), dtype=torch.float32, device=self.workspace.device)
        sel = {"x": 0, "s": 1, "out": 2}[which] if isinstance(which, str) else which
        _check(lib.dory_read_state(self.h, sel, ctypes.c_void_p(out.data_ptr()), rows, _stream(stream)))
        return out

    def read_kv(self, layer, slot, seq, pos0, n, stream=None):
        import torch
        dt = torch.bfloat16 if self.cfg.dtype == BF16 else torch.float32
        k = torch.empty((n, self.cfg.n_kv_heads, self.cfg.head_dim), dtype=dt, device=self.workspace.device)
        v = torch.empty_like(k)
        _check(lib.dory_read_kv(self.h, layer, slot, seq, pos0, n, ctypes.c_void_p(k.data_ptr()),
                                ctypes.c_void_p(v.data_ptr()), _stream(stream)))
        return k, v

    def synchronize(self, stream=None):
        _check(lib.dory_synchronize(self.h, _stream(stream)))

    def profile_reset(self):
        _check(lib.dory_profile_reset(self.h))

    def profile_read(self):
        n = 64
        names = (ctypes.c_char * 48 * n)()
        launches = (ctypes.c_int64 * n)()
        ms = (ctypes.c_double * n)()
        by = (ctypes.c_double * n)()
        cnt = ctypes.c_int32()
        _check(lib.dory_profile_read(self.h, n, ctypes.cast(names, ctypes.c_void_p), launches, ms, by,
                                     ctypes.byref(cnt)))
        out = {}
        for i in range(min(cnt.value, n)):
            out[bytes(names[i]).split(b"\0")[0].decode()] = {"launches": launches[i], "ms": ms[i], "bytes": by[i]}
        return out
