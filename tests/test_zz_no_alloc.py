"""hgx_attn_forward_noalloc against hgx_attn_forward (GPU, through the C ABI).

The allocation-free entry point serves callers that may not allocate device memory (a
framework that owns every byte through its own pool, a process whose footprint must not
grow after start-up): it keeps its scratch in a fixed array inside the library. Its output
must match the regular entry point's within the tolerance of the parity tests, on two calls
in a row (the second call finds the first call's leftovers in the shared scratch). This
file is collected last so that a run that stops at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

ATOL_MAX = 2e-2
ATOL_MEAN = 1e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from unified_text_pixel_b200 import binding, build

    build.build()
    L = binding.lib()
    fn = L.hgx_attn_forward_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int32] + [ctypes.c_void_p] * 3 + [ctypes.c_int32]
    return binding


def _inputs(w):
    t = W.tensors(w)
    d = {n: x.cuda() for n, x in t.items()}
    d["pos"] = torch.from_numpy(W.positions(w)).cuda()
    return d


def _desc(w):
    segs, cu_segs = W.flat_segments(w)
    cu = np.ascontiguousarray(W.cu_seqlens(w), dtype=np.int32)
    return cu, np.ascontiguousarray(segs, dtype=np.int32), np.ascontiguousarray(cu_segs, dtype=np.int32)


def _p(x):
    return ctypes.c_void_p(x.data_ptr())


def _h(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _noalloc(B, w):
    d = _inputs(w)
    out = torch.empty_like(d["q"])
    cfg = B.Attention.default_config()
    cu, segs, cu_segs = _desc(w)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = B.lib().hgx_attn_forward_noalloc(ctypes.byref(cfg), stream, _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(out),
                                          _p(d["pos"]), _p(d["wq"]), _p(d["wk"]), len(cu) - 1, _h(cu), _h(segs),
                                          _h(cu_segs), 1)
    assert st == B.HGX_OK
    return out


def _regular(B, w):
    d = _inputs(w)
    out = torch.empty_like(d["q"])
    a = B.Attention()
    a.forward(d["q"], d["k"], d["v"], out, d["pos"], d["wq"], d["wk"], *_desc(w))
    assert a.sync_status() == B.HGX_OK
    a.close()
    return out


def test_noalloc_matches_forward_on_two_calls_in_a_row(lib):
    B = lib
    for w in (W.config(1), W.config(0)):  # the second call reuses the first call's scratch
        got = _noalloc(B, w).float().cpu().numpy()
        ref = _regular(B, w).float().cpu().numpy()
        err = np.abs(got - ref)
        assert np.isfinite(got).all()
        assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (w.name, float(err.max()), float(err.mean()))


def test_noalloc_rejects_sizes_beyond_its_limit(lib):
    B = lib
    cfg = B.Attention.default_config()
    T = 16384 + 1
    cu = np.array([0, T], dtype=np.int32)
    segs = np.array([[0, T, 0]], dtype=np.int32)
    cu_segs = np.array([0, 1], dtype=np.int32)
    z = ctypes.c_void_p(0x10000)
    st = B.lib().hgx_attn_forward_noalloc(ctypes.byref(cfg), None, z, z, z, z, z, z, z, 1, _h(cu), _h(segs),
                                          _h(cu_segs), 1)
    assert st == B.HGX_ERR_UNSUPPORTED
