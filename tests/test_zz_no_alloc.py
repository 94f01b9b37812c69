"""hgx_attn_forward_noalloc against hgx_attn_forward and the fp64 oracle (GPU, through
the C ABI).

The allocation-free entry point serves callers that may not allocate device memory (a
framework that owns every byte through its own pool, a process whose footprint must not
grow after start-up): it keeps its scratch in a fixed array inside the library. Its output
must match the regular entry point's within the tolerance of the parity tests, on calls in
a row (each later call finds the earlier calls' leftovers in the shared scratch), and the
oracle's: element by element on the small workloads, on one row of every 64-token query
block of the Hunyuan GCA workload (full_in_segment rows). This file is collected last so
that a run that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
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
    out = torch.full_like(d["q"], float("nan"))
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
    out = torch.full_like(d["q"], float("nan"))
    a = B.Attention()
    a.forward(d["q"], d["k"], d["v"], out, d["pos"], d["wq"], d["wk"], *_desc(w))
    assert a.sync_status() == B.HGX_OK
    a.close()
    return out


def _within(got, ref, what):
    err = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (what, float(err.max()), float(err.mean()))


def _oracle_rows(w, rows):
    t = W.tensors(w)
    segs, cu_segs = W.flat_segments(w)
    return O.attention_rows(t["q"], t["k"], t["v"], W.positions(w), t["wq"], t["wk"], W.cu_seqlens(w), segs,
                            cu_segs, rows)


def test_noalloc_matches_forward_on_two_calls_in_a_row(lib):
    B = lib
    # the Hunyuan GCA workload (full_in_segment image rows, 9088 tokens), then the 1024^2 CFG
    # pair and the tiny layout: each later call reuses the earlier calls' scratch
    for w in (W.config(4), W.config(1), W.config(0)):
        got = _noalloc(B, w).float().cpu().numpy()
        ref = _regular(B, w).float().cpu().numpy()
        _within(got, ref, w.name + " vs hgx_attn_forward")
        if w.total_tokens <= 2200:
            rows = list(range(w.total_tokens))
        else:
            rng = np.random.default_rng(4)
            rows = sorted({int(rng.integers(r0, min(w.total_tokens, r0 + 64))) for r0 in range(0, w.total_tokens, 64)}
                          | {511, 512, 4607, 4608, 4863, 4864, w.total_tokens - 1})
        _within(got[rows], _oracle_rows(w, rows), w.name + " vs oracle")


def test_noalloc_at_its_size_limit(lib):
    """16 384 packed tokens in 64 batch elements (the most the fixed scratch takes), ragged
    lengths of 257 and 193 tokens (every element ends one token into a query block), causal
    text then a full_in_segment image: against hgx_attn_forward, and against the oracle on one
    row of every 64-token query block plus each element's first and last row."""
    B = lib
    lens = [257] * 63 + [16384 - 63 * 257]
    w = W.custom("noalloc_max", [[(17, 0), (n - 17, 2)] for n in lens], seed=31)
    assert w.total_tokens == 16384 and len(w.batches) == 64
    got = _noalloc(B, w).float().cpu().numpy()
    ref = _regular(B, w).float().cpu().numpy()
    _within(got, ref, "limit vs hgx_attn_forward")
    cu = W.cu_seqlens(w)
    rng = np.random.default_rng(31)
    rows = {int(rng.integers(r0, min(w.total_tokens, r0 + 64))) for r0 in range(0, w.total_tokens, 64)}
    rows |= {int(c) for c in cu[:-1]} | {int(c) - 1 for c in cu[1:]}
    rows = sorted(rows)
    _within(got[rows], _oracle_rows(w, rows), "limit vs oracle")


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


def test_noalloc_refuses_a_capturing_stream(lib):
    """The plan is uploaded from the library's shared static host buffers, which a recorded
    copy would read again at replay; so a call on a stream under capture returns
    HGX_ERR_UNSUPPORTED before any device work, and the next ordinary call still matches."""
    B = lib
    w = W.config(0)
    d = _inputs(w)
    out = torch.full_like(d["q"], float("nan"))
    cfg = B.Attention.default_config()
    cu, segs, cu_segs = _desc(w)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    statuses = []
    with torch.cuda.graph(g, stream=side):  # side is the current (capturing) stream in here
        sp = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        statuses.append(B.lib().hgx_attn_forward_noalloc(
            ctypes.byref(cfg), sp, _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(out), _p(d["pos"]), _p(d["wq"]),
            _p(d["wk"]), len(cu) - 1, _h(cu), _h(segs), _h(cu_segs), 0))
        out.add_(0)  # keeps the capture non-empty; the graph is never replayed
    assert statuses == [B.HGX_ERR_UNSUPPORTED]
    torch.cuda.synchronize()
    assert torch.isnan(out).all()  # nothing ran
    got = _noalloc(B, w).float().cpu().numpy()
    ref = _regular(B, w).float().cpu().numpy()
    _within(got, ref, "after a refused capture")
