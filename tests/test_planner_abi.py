"""Host planner and C ABI, on the CPU (no GPU, no kernel launches).

* per-row key limits and tile classes from the library's planner against the oracle's
  dense mask (built from the segment rules, never through limits): bit-exact;
* descriptor validation: every malformed request returns its documented status before
  any device work;
* the shared library loads and exports every function that include/hgx_attn.h declares.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O
import workloads as W
from unified_text_pixel_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    from unified_text_pixel_b200 import build

    build.build()


def _desc(w):
    segs, cu_segs = W.flat_segments(w)
    return W.cu_seqlens(w), segs, cu_segs


def _check_against_mask(w):
    cu, segs, cu_segs = _desc(w)
    lim = B.row_limits(cu, segs, cu_segs)
    bm, bn, classes = B.classify(cu, segs, cu_segs)
    at, pairs = 0, 0
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        L = t1 - t0
        bsegs = [tuple(int(x) for x in segs[n]) for n in range(cu_segs[b], cu_segs[b + 1])]
        mask = O.dense_mask(bsegs, L)
        pairs += int(mask.sum())
        # every row's visible set lies in [0, lim) and reaches lim - 1 (its own segment or
        # itself is always visible); without gen_image segments it is the whole prefix
        has_gen = any(k == O.GEN_IMAGE for _, _, k in bsegs)
        for i in range(L):
            vis = np.nonzero(mask[i])[0]
            assert vis.max() == lim[t0 + i] - 1
            if not has_gen:
                assert vis.size == lim[t0 + i]
        ref = O.tile_classes(mask, bm, bn)
        got = classes[at : at + ref.size].reshape(ref.shape)
        at += ref.size
        np.testing.assert_array_equal(got, ref)
    assert at == classes.size
    assert B.visible_pairs(cu, segs, cu_segs) == pairs


@pytest.mark.parametrize("cfg", range(5))
def test_limits_and_tile_classes_match_dense_mask(cfg):
    _check_against_mask(W.config(cfg))


@pytest.mark.parametrize("seed", range(40))
def test_limits_and_tile_classes_random_layouts(seed):
    _check_against_mask(W.random_workload(seed, allow_empty=(seed % 5 == 0)))


@pytest.mark.parametrize("seed", range(30))
def test_tile_classes_with_gen_image_holes(seed):
    """Multi-Gen-Image training layouts: holes make FULL, PARTIAL and SKIP blocks
    interleave; classes must still match the dense mask bit for bit."""
    _check_against_mask(W.random_workload(1000 + seed, max_len=1400, kinds=(0, 2, 3, 3)))


def test_multigen_workload_against_dense_mask():
    _check_against_mask(W.CONFIG_BY_NAME["hunyuan_multigen_9088"])


def test_tile_size_is_the_kernels():
    bm, bn, _ = B.classify(*_desc(W.config(0)))
    assert (bm, bn) == (64, 128)


def test_visible_pairs_match_closed_forms():
    from conftest import read_golden

    rows = {ln.split()[0]: int(ln.split()[1]) for ln in read_golden("unmasked_pairs.txt")}
    for w in W.CONFIGS:
        assert int(B.row_limits(*_desc(w)).astype(np.int64).sum()) == rows[w.name]


# ----------------------------------------------------------------------------- validation
def _status_row_limits(cu, segs, cu_segs):
    cu, sg, cs = B._descriptor(cu, segs, cu_segs)
    out = np.zeros(max(1, int(cu[-1]) if cu.size else 1), dtype=np.int32)
    return B.lib().hgx_attn_row_limits(len(cu) - 1, B._ptr(cu), B._ptr(sg), B._ptr(cs), B._ptr(out), out.size)


BAD = {
    "bad_kind": ([0, 5], [[0, 5, 4]], [0, 1]),
    "negative_kind": ([0, 5], [[0, 5, -1]], [0, 1]),
    "gap": ([0, 5], [[0, 2, 0], [3, 2, 1]], [0, 2]),
    "overlap": ([0, 5], [[0, 3, 0], [2, 3, 1]], [0, 2]),
    "zero_len": ([0, 5], [[0, 0, 0], [0, 5, 1]], [0, 2]),
    "short": ([0, 5], [[0, 4, 0]], [0, 1]),
    "long": ([0, 5], [[0, 6, 0]], [0, 1]),
    "cu_decreasing": ([0, 5, 3], [[0, 5, 0]], [0, 1, 1]),
    "cu_nonzero_start": ([1, 5], [[0, 4, 0]], [0, 1]),
    "too_many_tokens": ([0, 1 << 19], [[0, 1 << 19, 1]], [0, 1]),
    "segments_for_empty": ([0, 0], [[0, 1, 0]], [0, 1]),
}


@pytest.mark.parametrize("name", sorted(BAD))
def test_malformed_descriptors_rejected(name):
    assert _status_row_limits(*BAD[name]) == B.HGX_ERR_INVALID_ARG


def test_empty_batch_element_is_valid():
    lim = B.row_limits([0, 0, 3], [[0, 3, 1]], [0, 0, 1])
    assert list(lim) == [3, 3, 3]


def test_create_rejects_bad_configs():
    L = B.lib()
    base = B.Attention.default_config()

    def status(**kw):
        cfg = B.AttnConfig()
        ctypes.pointer(cfg)[0] = base
        for k, v in kw.items():
            if k == "mrope_section":
                cfg.mrope_section[:] = v
            else:
                setattr(cfg, k, v)
        h = ctypes.c_void_p()
        st = L.hgx_attn_create(ctypes.byref(cfg), ctypes.byref(h))
        if h.value:
            L.hgx_attn_destroy(h)
        return st

    assert status() == B.HGX_OK
    assert status(num_q_heads=16) == B.HGX_ERR_UNSUPPORTED
    assert status(head_dim=64) == B.HGX_ERR_UNSUPPORTED
    assert status(num_kv_heads=0) == B.HGX_ERR_INVALID_ARG
    assert status(rope_theta=-1.0) == B.HGX_ERR_INVALID_ARG
    assert status(rms_eps=-1.0) == B.HGX_ERR_INVALID_ARG
    assert status(mrope_section=[24, 20, 21]) == B.HGX_ERR_INVALID_ARG
    assert status(mrope_section=[4, 30, 30]) == B.HGX_ERR_UNSUPPORTED
    assert L.hgx_attn_create(None, ctypes.byref(ctypes.c_void_p())) == B.HGX_ERR_INVALID_ARG
    assert status(rope_layout=3) == B.HGX_ERR_INVALID_ARG
    assert status(rope_layout=-1) == B.HGX_ERR_INVALID_ARG
    # the 2D layouts ignore mrope_section
    assert status(rope_layout=B.HGX_ROPE_2D_ALTERNATING, mrope_section=[4, 30, 30]) == B.HGX_OK
    assert status(rope_layout=B.HGX_ROPE_2D_HALVES, mrope_section=[0, 0, 0]) == B.HGX_OK


def _fake(addr):
    # a non-null host integer posing as a device pointer: these calls must fail before
    # anything dereferences it
    return None if addr is None else ctypes.c_void_p(addr)


def _c_call(a, name, ptrs, cu, segs, cu_segs, *tail):
    """Calls a path entry point of the C ABI directly (below the binding's own tensor
    checks) with raw pointers, raising HgxError like the binding does."""
    c, sg, cs = B._descriptor(cu, segs, cu_segs)
    extra = [B._ptr(B._i32(t).reshape(-1)) for t in tail]
    st = getattr(B.lib(), name)(a.handle, None, *ptrs, len(c) - 1, B._ptr(c), B._ptr(sg), B._ptr(cs), *extra)
    a._check(st, name)


def test_forward_rejects_before_device_work():
    a = B.Attention()
    cu, segs, cu_segs = [0, 8], [[0, 8, 0]], [0, 1]
    good = [_fake(0x10000 * (i + 1)) for i in range(7)]
    # malformed descriptor
    with pytest.raises(B.HgxError) as e:
        _c_call(a, "hgx_attn_forward", good, [0, 8], [[0, 7, 0]], [0, 1])
    assert e.value.status == B.HGX_ERR_INVALID_ARG
    # null pointer
    for i in range(7):
        args = list(good)
        args[i] = None
        with pytest.raises(B.HgxError) as e:
            _c_call(a, "hgx_attn_forward", args, cu, segs, cu_segs)
        assert e.value.status == B.HGX_ERR_INVALID_ARG
    # misaligned pointer
    args = list(good)
    args[2] = _fake(0x30008)
    with pytest.raises(B.HgxError) as e:
        _c_call(a, "hgx_attn_forward", args, cu, segs, cu_segs)
    assert e.value.status == B.HGX_ERR_INVALID_ARG and "aligned" in str(e.value)
    # out overlapping q
    args = list(good)
    args[3] = _fake(0x10000 + 4096)
    with pytest.raises(B.HgxError) as e:
        _c_call(a, "hgx_attn_forward", args, cu, segs, cu_segs)
    assert e.value.status == B.HGX_ERR_INVALID_ARG and "overlap" in str(e.value)
    # an empty batch returns OK without touching the device (works without a GPU)
    _c_call(a, "hgx_attn_forward", [None] * 7, [0, 0], np.zeros((0, 3)), [0, 0])
    a.close()


def test_forward_from_checks_the_reused_prefix_before_device_work():
    """A reused (cached) row must not see a recomputed key: on the 2048^2 edit layout the
    257 causal text rows may be reused, any generation row may not."""
    a = B.Attention()
    w = W.config(3)
    cu, segs, cu_segs = _desc(w)
    good = [_fake(0x40000000 * (i + 1)) for i in range(7)]
    for first, ok in ((0, True), (256, True), (257, True), (258, False), (8449, True), (-1, False), (8450, False)):
        try:
            _c_call(a, "hgx_attn_forward_from", good, cu, segs, cu_segs, [first])
            raised = None
        except B.HgxError as e:
            raised = e
        if ok:  # passes the checks, then fails only because this machine has no GPU
            assert raised is not None and raised.status == B.HGX_ERR_CUDA, (first, raised)
        else:
            assert raised is not None and raised.status == B.HGX_ERR_INVALID_ARG, (first, raised)
    a.close()


def test_set_debug_rejects_unknown_flags():
    a = B.Attention()
    with pytest.raises(B.HgxError):
        a.set_debug(0x80)
    a.set_debug(B.HGX_DEBUG_CHECKED, 10_000_000)
    a.set_debug(B.HGX_DEBUG_FAIL_ALLOC | B.HGX_DEBUG_CHECKED | B.HGX_DEBUG_STALL_TEST | B.HGX_DEBUG_SPLIT_TEST)
    with pytest.raises(B.HgxError):
        a.set_debug(16)
    a.close()


def test_kernel_clock_refuses_before_any_launch():
    """hgx_attn_kernel_clock needs a handle that has launched the attention kernel; the
    refusals come before any CUDA call."""
    L = B.lib()
    c, n, m = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_double()
    assert L.hgx_attn_kernel_clock(None, None, ctypes.byref(c), ctypes.byref(n), ctypes.byref(m)) == B.HGX_ERR_INVALID_ARG
    a = B.Attention()
    assert L.hgx_attn_kernel_clock(a.handle, None, None, ctypes.byref(n), ctypes.byref(m)) == B.HGX_ERR_INVALID_ARG
    with pytest.raises(B.HgxError) as e:
        a.kernel_clock(stream=0)  # the legacy default stream: no torch stream needed here
    assert e.value.status == B.HGX_ERR_INVALID_ARG
    assert "no attention launch" in a.last_error()
    a.close()


def test_library_exports_every_declared_symbol():
    with open(os.path.join(ROOT, "include", "hgx_attn.h")) as f:
        text = f.read()
    declared = sorted(set(re.findall(r"\b(hgx_attn_\w+)\s*\(", text)))
    assert len(declared) >= 11
    L = ctypes.CDLL(B.library_path)
    for name in declared:
        assert hasattr(L, name), name


def test_header_declares_every_exported_symbol():
    """The reverse direction: every hgx_* function the library exports has a prototype in
    include/hgx_attn.h (the dynamic symbol table of the library built here, read with nm)."""
    with open(os.path.join(ROOT, "include", "hgx_attn.h")) as f:
        text = f.read()
    declared = set(re.findall(r"\b(hgx_attn_\w+)\s*\(", text))
    nm = subprocess.run(["nm", "-D", "--defined-only", B.library_path], capture_output=True, text=True, check=True)
    exported = {ln.split()[-1] for ln in nm.stdout.splitlines() if ln.split() and ln.split()[-1].startswith("hgx_")}
    assert exported, nm.stdout[:200]
    assert exported <= declared, sorted(exported - declared)


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "library_path", str(tmp_path / "missing.so"))
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(B.HgxError):
        B.lib()


def _noalloc_status(cfg, cu, segs, cu_segs):
    L = B.lib()
    fn = L.hgx_attn_forward_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int32] + [ctypes.c_void_p] * 3 + [ctypes.c_int32]
    cu, sg, cs = B._descriptor(cu, segs, cu_segs)
    z = [ctypes.c_void_p(0x40000000 * (i + 1)) for i in range(7)]
    return fn(ctypes.byref(cfg), None, *z, len(cu) - 1, B._ptr(cu), B._ptr(sg), B._ptr(cs), 1)


def test_noalloc_rejects_before_device_work():
    """The allocation-free entry point checks its fixed limits and the descriptor on the
    host: too many tokens or a gen_image segment -> UNSUPPORTED, malformed -> INVALID_ARG."""
    cfg = B.Attention.default_config()
    assert _noalloc_status(cfg, [0, 16385], [[0, 16385, 0]], [0, 1]) == B.HGX_ERR_UNSUPPORTED
    assert _noalloc_status(cfg, [0, 10], [[0, 4, 0], [4, 6, 3]], [0, 2]) == B.HGX_ERR_UNSUPPORTED
    assert _noalloc_status(cfg, [0, 10], [[0, 4, 0], [5, 5, 1]], [0, 2]) == B.HGX_ERR_INVALID_ARG
    bad = B.Attention.default_config()
    bad.num_q_heads = 16
    assert _noalloc_status(bad, [0, 10], [[0, 10, 0]], [0, 1]) == B.HGX_ERR_UNSUPPORTED
    bad = B.Attention.default_config()
    bad.rope_layout = 7
    assert _noalloc_status(bad, [0, 10], [[0, 10, 0]], [0, 1]) == B.HGX_ERR_INVALID_ARG
    # an empty batch is done without touching the device
    assert _noalloc_status(cfg, [0], np.zeros((0, 3)), [0]) == B.HGX_OK


def test_binding_rejects_wrong_tensors_before_the_library():
    """Marshalling checks of the binding (no GPU needed: every case is refused before any
    pointer reaches the library): host tensors, wrong dtype, non-contiguous views and
    wrong shapes raise INVALID_ARG."""
    import torch

    bf = torch.bfloat16
    T = 5
    ok = dict(q=torch.zeros(T, 32, 128, dtype=bf), k=torch.zeros(T, 8, 128, dtype=bf))
    cases = [
        ("host tensor", lambda: B._expect("q", ok["q"], "bf16", (32, 128), T)),
        ("not a tensor", lambda: B._expect("q", np.zeros((T, 32, 128)), "bf16", (32, 128), T)),
    ]
    for what, fn in cases:
        with pytest.raises(B.HgxError) as e:
            fn()
        assert e.value.status == B.HGX_ERR_INVALID_ARG, what

    def check(t, dtype, tail, rows):  # CPU tensors that report is_cuda, so the later checks run here
        orig = torch.Tensor.is_cuda
        try:
            torch.Tensor.is_cuda = property(lambda self: True)
            B._expect("x", t, dtype, tail, rows)
        finally:
            torch.Tensor.is_cuda = orig

    for what, t, dt, tail, rows in [
        ("fp32", torch.zeros(T, 32, 128), "bf16", (32, 128), T),
        ("int64 positions", torch.zeros(T, 3, dtype=torch.int64), "i32", (3,), T),
        ("non-contiguous", torch.zeros(T, 128, 32, dtype=bf).transpose(1, 2), "bf16", (32, 128), T),
        ("too few rows", torch.zeros(T - 1, 32, 128, dtype=bf), "bf16", (32, 128), T),
        ("wrong heads", torch.zeros(T, 8, 128, dtype=bf), "bf16", (32, 128), T),
        ("weight shape", torch.zeros(64, dtype=bf), "bf16", (128,), None),
    ]:
        with pytest.raises(B.HgxError) as e:
            check(t, dt, tail, rows)
        assert e.value.status == B.HGX_ERR_INVALID_ARG, what
    check(torch.zeros(T + 2, 32, 128, dtype=bf), "bf16", (32, 128), T)  # more rows than needed is fine
    check(torch.zeros(128, dtype=bf), "bf16", (128,), None)


def _lpt_makespan(costs, ctas):
    import heapq

    h = [(0, c) for c in range(min(ctas, len(costs)))]
    for cost in sorted(costs, reverse=True):
        load, c = heapq.heappop(h)
        heapq.heappush(h, (load + cost, c))
    return max(load for load, _ in h)


@pytest.mark.parametrize("case", ["c1", "c2", "c3", "c4", "multigen", "random_a", "random_b", "holes"])
@pytest.mark.parametrize("split_test", [False, True])
def test_split_schedule_covers_every_key_block_once(case, split_test):
    """The persistent-CTA schedule, with items split by key blocks where that balances the
    CTAs better: for every (query block, KV head) the key-block ranges of its items
    partition the unsplit item's range exactly; the parts of a split item use consecutive
    partial slots and all slots are distinct; list-form (Gen Image hole) items are never
    split; and the schedule's makespan never exceeds the longest-first assignment's. The
    2048^2 CFG pair (1040 equal items on 148 CTAs) must split."""
    mode = 2 if split_test else 1
    w = {"c1": W.config(1), "c2": W.config(2), "c3": W.config(3), "c4": W.config(4),
         "multigen": W.CONFIG_BY_NAME["hunyuan_multigen_9088"],
         "random_a": W.random_workload(31, max_batch=4, max_len=3000),
         "random_b": W.random_workload(32, max_batch=2, max_len=6000),
         "holes": W.random_workload(33, max_batch=3, max_len=4000, kinds=(0, 2, 3, 3))}[case]
    cu, segs, cu_segs = _desc(w)
    base = B.schedule(cu, segs, cu_segs, 1)  # one CTA: nothing to balance, nothing split
    assert (base[:, 5] == -1).all() and (base[:, 3] == 0).all()
    whole = {(int(r[1]), int(r[2])): (int(r[4]), int(r[6]), int(r[7])) for r in base}
    ctas = 148
    s = B.schedule(cu, segs, cu_segs, ctas, mode)
    groups = {}
    for r in s:
        groups.setdefault((int(r[1]), int(r[2])), []).append(r)
    assert set(groups) == set(whole)
    slots = []
    for key, rows in groups.items():
        n, n_full, list_off = whole[key]
        rows = sorted(rows, key=lambda r: r[3])
        assert all(int(r[6]) == n_full for r in rows)
        if len(rows) == 1:
            assert rows[0][5] == -1 and rows[0][3] == 0 and rows[0][4] == n
            continue
        assert list_off < 0, (key, rows)
        at = 0
        for r in rows:  # contiguous, non-empty key-block ranges covering [0, n)
            assert r[3] == at and r[4] >= 1
            at += int(r[4])
        assert at == n
        parts = sorted(int(r[5]) for r in rows)
        assert parts == list(range(parts[0], parts[0] + len(rows)))
        slots += parts
    assert sorted(slots) == list(range(len(slots)))
    # execution order: CTAs in order, every CTA's items contiguous
    assert (np.diff(s[:, 0]) >= 0).all()
    used = int(s[:, 0].max()) + 1

    # the planner's cost model, in tenths of a fully visible key block: 10 per fully visible
    # block, 13 per block that needs the mask compare, + 12 per item, + 30 per part of a split
    # item (prefix-form items: blocks below n_full are fully visible)
    def cost(rows):
        nf = np.clip(rows[:, 6] - rows[:, 3], 0, rows[:, 4])
        return 10 * nf + 13 * (rows[:, 4] - nf) + np.where(rows[:, 5] >= 0, 30, 12)

    has_lists = (base[:, 7] >= 0).any()  # list-form items: their blocks' classes are not in the rows
    lpt = _lpt_makespan([int(x) for x in cost(base)], ctas)
    if case == "c2" and not split_test:
        assert len(slots) > 0
    if split_test:  # the test hook splits every prefix-form item of two or more key blocks
        for key, (n, _, list_off) in whole.items():
            assert len(groups[key]) == (2 if list_off < 0 and n >= 2 else 1), key
    elif not has_lists:
        # a split schedule is taken only when it beats longest-first by more than 3 blocks
        span = np.bincount(s[:, 0], weights=cost(s), minlength=used).max()
        assert (span + 30 < lpt) if slots else (span == lpt)
