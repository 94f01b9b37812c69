"""ctypes binding of libhgx_attn.so: argument marshalling only.

Tensors are passed as raw device pointers (torch is used for device memory and streams);
segment descriptors are passed as host int32 arrays. Every step of the path runs in the
library's kernels.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np

HGX_OK, HGX_ERR_INVALID_ARG, HGX_ERR_UNSUPPORTED, HGX_ERR_OOM, HGX_ERR_CUDA, HGX_ERR_TIMEOUT = range(6)
HGX_SEG_CAUSAL, HGX_SEG_FULL_SEQUENCE, HGX_SEG_FULL_IN_SEGMENT, HGX_SEG_GEN_IMAGE = 0, 1, 2, 3
HGX_TILE_SKIP, HGX_TILE_PARTIAL, HGX_TILE_FULL = 0, 1, 2
HGX_DEBUG_CHECKED, HGX_DEBUG_STALL_TEST, HGX_DEBUG_FAIL_ALLOC, HGX_DEBUG_SPLIT_TEST = 1, 2, 4, 8
HGX_ROPE_MROPE_INTERLEAVED, HGX_ROPE_2D_ALTERNATING, HGX_ROPE_2D_HALVES = 0, 1, 2

_STATUS = {0: "HGX_OK", 1: "HGX_ERR_INVALID_ARG", 2: "HGX_ERR_UNSUPPORTED", 3: "HGX_ERR_OOM",
           4: "HGX_ERR_CUDA", 5: "HGX_ERR_TIMEOUT"}

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhgx_attn.so")


class HgxError(RuntimeError):
    def __init__(self, status: int, message: str = ""):
        self.status = status
        super().__init__(f"{_STATUS.get(status, status)}: {message}")


class AttnConfig(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
        ("mrope_section", ctypes.c_int32 * 3),
        ("rms_eps", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("rope_layout", ctypes.c_int32),
    ]


_lib = None

_SIGS = {
    "hgx_attn_default_config": (None, [ctypes.c_void_p]),
    "hgx_attn_create": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)]),
    "hgx_attn_destroy": (None, [ctypes.c_void_p]),
    "hgx_attn_last_error": (ctypes.c_char_p, [ctypes.c_void_p]),
    "hgx_attn_forward": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int32] + [ctypes.c_void_p] * 3),
    "hgx_attn_forward_from": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int32] + [ctypes.c_void_p] * 4),
    "hgx_attn_prologue": (ctypes.c_int, [ctypes.c_void_p] * 7 + [ctypes.c_int32]),
    "hgx_attn_qkv_projection": (ctypes.c_int, [ctypes.c_void_p] * 10 + [ctypes.c_int32]),
    "hgx_attn_out_projection": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int32]),
    "hgx_attn_layer_forward": (ctypes.c_int, [ctypes.c_void_p] * 13 + [ctypes.c_int32] + [ctypes.c_void_p] * 3),
    "hgx_attn_attention": (ctypes.c_int, [ctypes.c_void_p] * 6 + [ctypes.c_int32] + [ctypes.c_void_p] * 3),
    "hgx_attn_row_limits": (ctypes.c_int, [ctypes.c_int32] + [ctypes.c_void_p] * 4 + [ctypes.c_size_t]),
    "hgx_attn_classify": (ctypes.c_int, [ctypes.c_int32] + [ctypes.c_void_p] * 6 + [ctypes.c_size_t, ctypes.c_void_p]),
    "hgx_attn_visible_pairs": (ctypes.c_int, [ctypes.c_int32] + [ctypes.c_void_p] * 4),
    "hgx_attn_schedule": (ctypes.c_int, [ctypes.c_int32] + [ctypes.c_void_p] * 3 + [ctypes.c_int32, ctypes.c_int32,
                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "hgx_attn_sync_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "hgx_attn_kernel_clock": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint64),
                                             ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_double)]),
    "hgx_attn_set_debug": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint64]),
}


def lib() -> ctypes.CDLL:
    """Loads libhgx_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise HgxError(HGX_ERR_UNSUPPORTED, f"{library_path} is missing: run "
                           "`python -m unified_text_pixel_b200.build` (there is no fallback)")
        L = ctypes.CDLL(library_path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a.size else None


def _descriptor(cu_seqlens, segs, cu_segs):
    cu = _i32(cu_seqlens).reshape(-1)
    sg = _i32(segs).reshape(-1, 3)
    cs = _i32(cu_segs).reshape(-1)
    return cu, sg, cs


def row_limits(cu_seqlens, segs, cu_segs) -> np.ndarray:
    """Exclusive key limit of every packed row (host-side planner of the library)."""
    cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
    T = int(cu[-1]) if cu.size else 0
    out = np.zeros(T, dtype=np.int32)
    st = lib().hgx_attn_row_limits(len(cu) - 1, _ptr(cu), _ptr(sg), _ptr(cs), _ptr(out), T)
    if st != HGX_OK:
        raise HgxError(st, "hgx_attn_row_limits")
    return out


def schedule(cu_seqlens, segs, cu_segs, ctas: int, mode: int = 0) -> np.ndarray:
    """The attention kernel's persistent-CTA schedule: int32 [items, 8] rows of
    (cta, q0, kv_head, kb0, n_total, part, n_full, list_off) in execution order. mode 0: the
    library's policy; 1: split items whenever that balances better; 2: split every item."""
    cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
    n = ctypes.c_size_t()
    L = lib()
    st = L.hgx_attn_schedule(len(cu) - 1, _ptr(cu), _ptr(sg), _ptr(cs), int(ctas), int(mode), None, 0,
                             ctypes.byref(n))
    if st != HGX_OK:
        raise HgxError(st, "hgx_attn_schedule")
    out = np.zeros((n.value, 8), dtype=np.int32)
    st = L.hgx_attn_schedule(len(cu) - 1, _ptr(cu), _ptr(sg), _ptr(cs), int(ctas), int(mode), _ptr(out),
                             n.value, ctypes.byref(n))
    if st != HGX_OK:
        raise HgxError(st, "hgx_attn_schedule")
    return out


def visible_pairs(cu_seqlens, segs, cu_segs) -> int:
    """Visible (query, key) pairs of the packed batch, Gen Image holes excluded."""
    cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
    out = ctypes.c_uint64()
    st = lib().hgx_attn_visible_pairs(len(cu) - 1, _ptr(cu), _ptr(sg), _ptr(cs), ctypes.byref(out))
    if st != HGX_OK:
        raise HgxError(st, "hgx_attn_visible_pairs")
    return int(out.value)


def classify(cu_seqlens, segs, cu_segs) -> Tuple[int, int, np.ndarray]:
    """(bm_tokens, bn_keys, classes uint8) at the attention kernel's tile size."""
    cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
    bm, bn, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_size_t()
    L = lib()
    st = L.hgx_attn_classify(len(cu) - 1, _ptr(cu), _ptr(sg), _ptr(cs), ctypes.byref(bm),
                             ctypes.byref(bn), None, 0, ctypes.byref(n))
    if st != HGX_OK:
        raise HgxError(st, "hgx_attn_classify")
    out = np.zeros(n.value, dtype=np.uint8)
    st = L.hgx_attn_classify(len(cu) - 1, _ptr(cu), _ptr(sg), _ptr(cs), ctypes.byref(bm),
                             ctypes.byref(bn), _ptr(out), out.size, ctypes.byref(n))
    if st != HGX_OK:
        raise HgxError(st, "hgx_attn_classify")
    return bm.value, bn.value, out


def _dev_ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _expect(name, t, dtype, tail, rows):
    """Marshalling check of one device tensor argument: a contiguous CUDA tensor of the
    given dtype whose trailing dimensions are `tail` and that holds at least `rows` rows
    (leading dimension; None = no leading dimension). Raises HgxError(INVALID_ARG)."""
    import torch

    if not isinstance(t, torch.Tensor):
        raise HgxError(HGX_ERR_INVALID_ARG, f"{name}: expected a torch tensor, got {type(t).__name__}")
    if not t.is_cuda:
        raise HgxError(HGX_ERR_INVALID_ARG, f"{name}: must be a CUDA tensor (device {t.device})")
    want = {"bf16": torch.bfloat16, "i32": torch.int32}[dtype]
    if t.dtype != want:
        raise HgxError(HGX_ERR_INVALID_ARG, f"{name}: dtype {t.dtype}, expected {want}")
    if not t.is_contiguous():
        raise HgxError(HGX_ERR_INVALID_ARG, f"{name}: must be contiguous (strides {tuple(t.stride())})")
    shape = tuple(t.shape)
    if rows is None:
        ok = shape == tuple(tail)
    else:
        ok = len(shape) == 1 + len(tail) and shape[1:] == tuple(tail) and shape[0] >= rows
    if not ok:
        want_shape = list(tail) if rows is None else [f">={rows}", *tail]
        raise HgxError(HGX_ERR_INVALID_ARG, f"{name}: shape {list(shape)}, expected {want_shape}")


def _check_path(T, q=None, k=None, v=None, out=None, pos=None, wq=None, wk=None):
    """Checks the tensors of the attention path for T packed tokens (nothing when T == 0:
    the library then does no device work)."""
    if T == 0:
        return
    for name, t, dt, tail in (("q", q, "bf16", (32, 128)), ("k", k, "bf16", (8, 128)), ("v", v, "bf16", (8, 128)),
                              ("out", out, "bf16", (32, 128)), ("pos", pos, "i32", (3,))):
        if t is not None:
            _expect(name, t, dt, tail, T)
    for name, t in (("wq", wq), ("wk", wk)):
        if t is not None:
            _expect(name, t, "bf16", (128,), None)


def _stream_ptr(stream):
    """torch.cuda.Stream, a raw cudaStream_t integer, or None for torch's current stream."""
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    if stream is None:
        import torch

        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Attention:
    """Owns one hgx_attn_handle. Methods take torch CUDA tensors (bf16 / int32)."""

    def __init__(self, config: Optional[AttnConfig] = None, **overrides):
        L = lib()
        cfg = AttnConfig()
        L.hgx_attn_default_config(ctypes.byref(cfg))
        if config is not None:
            cfg = config
        for name, value in overrides.items():
            setattr(cfg, name, value)
        self.config = cfg
        h = ctypes.c_void_p()
        st = L.hgx_attn_create(ctypes.byref(cfg), ctypes.byref(h))
        if st != HGX_OK:
            raise HgxError(st, "hgx_attn_create")
        self._h = h

    @staticmethod
    def default_config() -> AttnConfig:
        cfg = AttnConfig()
        lib().hgx_attn_default_config(ctypes.byref(cfg))
        return cfg

    def close(self):
        if getattr(self, "_h", None):
            lib().hgx_attn_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st: int, what: str):
        if st != HGX_OK:
            msg = lib().hgx_attn_last_error(self._h) or b""
            raise HgxError(st, f"{what}: {msg.decode(errors='replace')}")

    def forward(self, q, k, v, out, pos, wq, wk, cu_seqlens, segs, cu_segs, stream=None):
        """hgx_attn_forward: q, k overwritten with q', k'; out written."""
        cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
        _check_path(int(cu[-1]) if cu.size else 0, q, k, v, out, pos, wq, wk)
        st = lib().hgx_attn_forward(self._h, _stream_ptr(stream), _dev_ptr(q), _dev_ptr(k), _dev_ptr(v),
                                    _dev_ptr(out), _dev_ptr(pos), _dev_ptr(wq), _dev_ptr(wk), len(cu) - 1,
                                    _ptr(cu), _ptr(sg), _ptr(cs))
        self._check(st, "hgx_attn_forward")

    def forward_from(self, q, k, v, out, pos, wq, wk, cu_seqlens, segs, cu_segs, first_rows, stream=None):
        """hgx_attn_forward_from: recompute rows [first_rows[b], L_b) only (reused prefix)."""
        cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
        _check_path(int(cu[-1]) if cu.size else 0, q, k, v, out, pos, wq, wk)
        fr = _i32(first_rows).reshape(-1)
        st = lib().hgx_attn_forward_from(self._h, _stream_ptr(stream), _dev_ptr(q), _dev_ptr(k), _dev_ptr(v),
                                         _dev_ptr(out), _dev_ptr(pos), _dev_ptr(wq), _dev_ptr(wk), len(cu) - 1,
                                         _ptr(cu), _ptr(sg), _ptr(cs), _ptr(fr))
        self._check(st, "hgx_attn_forward_from")

    def qkv_projection(self, x, w_qkv, q, k, v, pos, wq, wk, stream=None):
        """q', k', v from x: tcgen05 GEMM with RMSNorm + rotation in its epilogue."""
        T = int(x.shape[0])
        if T:
            _expect("x", x, "bf16", (4096,), T)
            _expect("w_qkv", w_qkv, "bf16", (6144, 4096), None)
        _check_path(T, q, k, v, None, pos, wq, wk)
        st = lib().hgx_attn_qkv_projection(self._h, _stream_ptr(stream), _dev_ptr(x), _dev_ptr(w_qkv), _dev_ptr(q),
                                           _dev_ptr(k), _dev_ptr(v), _dev_ptr(pos), _dev_ptr(wq), _dev_ptr(wk),
                                           int(x.shape[0]))
        self._check(st, "hgx_attn_qkv_projection")

    def out_projection(self, attn, w_o, y, stream=None):
        """y = attn W_o^T (attn [T, 32, 128] or [T, 4096], w_o [4096, 4096], y [T, 4096])."""
        T = int(attn.shape[0])
        if T:
            _expect("attn", attn, "bf16", (32, 128) if attn.dim() == 3 else (4096,), T)
            _expect("w_o", w_o, "bf16", (4096, 4096), None)
            _expect("y", y, "bf16", (4096,), T)
        st = lib().hgx_attn_out_projection(self._h, _stream_ptr(stream), _dev_ptr(attn), _dev_ptr(w_o), _dev_ptr(y),
                                           int(attn.shape[0]))
        self._check(st, "hgx_attn_out_projection")

    def layer_forward(self, x, w_qkv, w_o, q, k, v, attn, y, pos, wq, wk, cu_seqlens, segs, cu_segs, stream=None):
        """QKV projection (fused RMSNorm + rotation) -> masked attention -> output projection."""
        cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
        T = int(cu[-1]) if cu.size else 0
        if T:
            _expect("x", x, "bf16", (4096,), T)
            _expect("w_qkv", w_qkv, "bf16", (6144, 4096), None)
            _expect("w_o", w_o, "bf16", (4096, 4096), None)
            _expect("y", y, "bf16", (4096,), T)
        _check_path(T, q, k, v, attn, pos, wq, wk)
        st = lib().hgx_attn_layer_forward(self._h, _stream_ptr(stream), _dev_ptr(x), _dev_ptr(w_qkv), _dev_ptr(w_o),
                                          _dev_ptr(q), _dev_ptr(k), _dev_ptr(v), _dev_ptr(attn), _dev_ptr(y),
                                          _dev_ptr(pos), _dev_ptr(wq), _dev_ptr(wk), len(cu) - 1, _ptr(cu),
                                          _ptr(sg), _ptr(cs))
        self._check(st, "hgx_attn_layer_forward")

    def prologue(self, q, k, pos, wq, wk, total_tokens=None, stream=None):
        T = q.shape[0] if total_tokens is None else total_tokens
        _check_path(int(T), q, k, None, None, pos, wq, wk)
        st = lib().hgx_attn_prologue(self._h, _stream_ptr(stream), _dev_ptr(q), _dev_ptr(k), _dev_ptr(pos),
                                     _dev_ptr(wq), _dev_ptr(wk), int(T))
        self._check(st, "hgx_attn_prologue")

    def attention(self, q, k, v, out, cu_seqlens, segs, cu_segs, stream=None):
        cu, sg, cs = _descriptor(cu_seqlens, segs, cu_segs)
        _check_path(int(cu[-1]) if cu.size else 0, q, k, v, out)
        st = lib().hgx_attn_attention(self._h, _stream_ptr(stream), _dev_ptr(q), _dev_ptr(k), _dev_ptr(v),
                                      _dev_ptr(out), len(cu) - 1, _ptr(cu), _ptr(sg), _ptr(cs))
        self._check(st, "hgx_attn_attention")

    def sync_status(self, stream=None) -> int:
        """Synchronizes the stream; returns the status code (HGX_ERR_TIMEOUT after a wait ran out)."""
        return lib().hgx_attn_sync_status(self._h, _stream_ptr(stream))

    def kernel_clock(self, stream=None):
        """(cycles of the slowest CTA, its span in ns, median effective SM clock in MHz) of the
        last attention launch on this handle; synchronizes the stream."""
        cyc, ns, mhz = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_double()
        self._check(lib().hgx_attn_kernel_clock(self._h, _stream_ptr(stream), ctypes.byref(cyc), ctypes.byref(ns),
                                                ctypes.byref(mhz)), "hgx_attn_kernel_clock")
        return int(cyc.value), int(ns.value), float(mhz.value)

    def set_debug(self, flags: int, wait_limit_ns: int = 0):
        self._check(lib().hgx_attn_set_debug(self._h, flags, wait_limit_ns), "hgx_attn_set_debug")

    def last_error(self) -> str:
        return (lib().hgx_attn_last_error(self._h) or b"").decode(errors="replace")

    # raw access for ABI tests
    @property
    def handle(self):
        return self._h
