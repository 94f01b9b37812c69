"""GPU parity of the sm_100a path against the fp64 oracle, through the C ABI.

Tolerances (bf16 inputs, fp32 accumulation, unit-variance data): attention output
max |err| <= 2e-2 and mean |err| <= 1e-3 against the fp64 oracle; the prologue's bf16
q'/k' within bf16 rounding of the fp64 values (relative 2^-8 plus 1e-5 absolute for the
fp32 arithmetic before rounding).

Small configurations are compared element by element on every output; the full-size
workloads (2048^2 text-to-image and edit, Hunyuan GCA, the multi-Gen-Image training mask)
run in exactly the launch configuration the benchmark times and are compared on sampled
rows that the oracle computes one by one: one random row of every 64-token query block of
every batch element (each block is one work item per KV head, and a row covers all 32
query heads, so every work item is checked), plus segment boundaries, tile edges, first and
last rows. The output buffer is filled with NaN before every call and must come back
finite everywhere, so a work item that is dropped or written to the wrong rows fails.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

ATOL_MAX = 2e-2
ATOL_MEAN = 1e-3


@pytest.fixture(scope="module")
def hgx():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from unified_text_pixel_b200 import build

    build.build()
    import unified_text_pixel_b200 as H

    a = H.Attention()
    yield H, a
    a.close()


def _desc(w):
    segs, cu_segs = W.flat_segments(w)
    return W.cu_seqlens(w), segs, cu_segs


def _device_inputs(w):
    t = W.tensors(w)
    d = {n: x.cuda() for n, x in t.items()}
    d["pos"] = torch.from_numpy(W.positions(w)).cuda()
    return t, d


def _nan_like(x):
    return torch.full_like(x, float("nan"))


def _run(hgx, w, d=None):
    """hgx_attn_forward into an output prefilled with NaN (rows it does not write stay NaN)."""
    H, a = hgx
    if d is None:
        _, d = _device_inputs(w)
    out = _nan_like(d["q"])
    a.forward(d["q"], d["k"], d["v"], out, d["pos"], d["wq"], d["wk"], *_desc(w))
    assert a.sync_status() == H.HGX_OK
    return out, d


def _compare(got, ref, what):
    err = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= ATOL_MAX, (what, float(err.max()))
    assert err.mean() <= ATOL_MEAN, (what, float(err.mean()))
    return float(err.max()), float(err.mean())


def _oracle_full(w, t):
    segs, cu_segs = W.flat_segments(w)
    return O.forward(t["q"], t["k"], t["v"], W.positions(w), t["wq"], t["wk"], W.cu_seqlens(w), segs, cu_segs)


# ------------------------------------------------------------------------------ prologue
@pytest.mark.parametrize("case", ["c0", "c1", "ragged7", "one"])
def test_prologue_matches_oracle(hgx, case):
    H, a = hgx
    w = {"c0": W.config(0), "c1": W.config(1), "ragged7": W.custom("r7", [[(3, 0), (4, 1)]], seed=11),
         "one": W.custom("one", [[(1, 0)]], seed=12)}[case]
    t, d = _device_inputs(w)
    T = w.total_tokens
    # canaries: one token row of padding on each side of q and k
    qpad = torch.full((T + 2, 32, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    kpad = torch.full((T + 2, 8, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    qpad[1:-1] = d["q"]
    kpad[1:-1] = d["k"]
    a.prologue(qpad[1:-1], kpad[1:-1], d["pos"], d["wq"], d["wk"])
    assert a.sync_status() == H.HGX_OK
    qr, kr = O.prologue(t["q"], t["k"], W.positions(w), t["wq"], t["wk"])
    for got, ref in ((qpad[1:-1], qr), (kpad[1:-1], kr)):
        g = got.float().cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(g, ref, rtol=2.0 ** -8, atol=1e-5)
    for pad in (qpad[0], qpad[-1], kpad[0], kpad[-1]):
        assert bool((pad == 7.0).all())


def test_prologue_large_positions(hgx):
    """Positions around and beyond 2^24, positive and negative: below 2^24 the kernel reduces
    the angle in fp32 (position times a two-float split of inv_freq / 2 pi), from 2^24 on it
    takes the fp64 sincos; both must match the fp64 oracle within bf16 rounding. Rows 0-15
    straddle 2^24 by a few units, 16-31 reach 2^30, 32-47 go down to -2^30, and the three
    axes of a row differ."""
    H, a = hgx
    w = W.custom("big_pos", [[(48, 0)]], seed=23)
    t = W.tensors(w)
    d = {n: x.cuda() for n, x in t.items()}
    rng = np.random.default_rng(23)
    pos = np.empty((48, 3), dtype=np.int64)
    pos[:16] = (1 << 24) + rng.integers(-8, 8, size=(16, 3))
    pos[16:32] = rng.integers(1 << 20, 1 << 30, size=(16, 3))
    pos[32:48] = -rng.integers(1 << 20, 1 << 30, size=(16, 3))
    pos = pos.astype(np.int32)
    a.prologue(d["q"], d["k"], torch.from_numpy(pos).cuda(), d["wq"], d["wk"])
    assert a.sync_status() == H.HGX_OK
    qr, kr = O.prologue(t["q"], t["k"], pos, t["wq"], t["wk"])
    np.testing.assert_allclose(d["q"].float().cpu().numpy(), qr, rtol=2.0 ** -8, atol=1e-5)
    np.testing.assert_allclose(d["k"].float().cpu().numpy(), kr, rtol=2.0 ** -8, atol=1e-5)


@pytest.mark.parametrize("layout", [1, 2])
def test_prologue_2d_rope_layouts(hgx, layout):
    """HunyuanImage 3.0 Generalized 2D RoPE, both readings (x = w column, y = h column), on
    the Hunyuan-style positions (text on the diagonal, image tokens on a 2D grid)."""
    H, _ = hgx
    a = H.Attention(rope_layout=layout)
    w = W.Workload("gca_2d", (W._segments([(40, W.CAUSAL, None), (64, W.FULL_IN_SEGMENT, (8, 8)), (9, W.CAUSAL, None)]),),
                   seed=17, style="hunyuan")
    t, d = _device_inputs(w)
    a.prologue(d["q"], d["k"], d["pos"], d["wq"], d["wk"])
    assert a.sync_status() == H.HGX_OK
    qr, kr = O.prologue(t["q"], t["k"], W.positions(w), t["wq"], t["wk"], layout=layout)
    np.testing.assert_allclose(d["q"].float().cpu().numpy(), qr, rtol=2.0 ** -8, atol=1e-5)
    np.testing.assert_allclose(d["k"].float().cpu().numpy(), kr, rtol=2.0 ** -8, atol=1e-5)
    a.close()


# ------------------------------------------------------------------------------ attention
@pytest.mark.parametrize("cfg", [0, 1])
def test_forward_small_configs_elementwise(hgx, cfg):
    w = W.config(cfg)
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    ref, _, _ = _oracle_full(w, t)
    _compare(out.float().cpu().numpy(), ref, w.name)


@pytest.mark.parametrize("seed", range(6))
def test_forward_random_layouts_elementwise(hgx, seed):
    """Ragged lengths, all three kinds, several batch elements, empty elements."""
    w = W.random_workload(100 + seed, max_batch=4, max_len=520, allow_empty=True)
    if w.total_tokens == 0:
        pytest.skip("empty draw")
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    ref, _, _ = _oracle_full(w, t)
    _compare(out.float().cpu().numpy(), ref, w.name)


@pytest.mark.parametrize("seed", range(5))
def test_forward_gen_image_holes_elementwise(hgx, seed):
    """Multi-Gen-Image training layouts (HunyuanImage 3.0, section 3.4): Gen Images are
    hidden from later rows, so key blocks of a row's prefix may be skipped or masked by a
    hole; element by element against the oracle's dense mask."""
    w = W.random_workload(2000 + seed, max_batch=3, max_len=1100, kinds=(0, 2, 3, 3))
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    ref, _, _ = _oracle_full(w, t)
    _compare(out.float().cpu().numpy(), ref, w.name)


@pytest.mark.parametrize("seed", range(8))
def test_forward_larger_mixed_layouts_elementwise(hgx, seed):
    """All four segment kinds (Gen Image holes included) in up to three elements of up to
    1600 tokens, empty elements allowed: several items per CTA of different lengths, so the
    planner's longest-first lists and tail splits (with their combine launch) take part;
    element by element against the oracle's dense mask."""
    w = W.random_workload(300 + seed, max_batch=3, max_len=1600, allow_empty=True, kinds=(0, 1, 2, 3))
    if w.total_tokens == 0:
        pytest.skip("empty draw")
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    ref, _, _ = _oracle_full(w, t)
    _compare(out.float().cpu().numpy(), ref, w.name)


def test_forward_many_tiny_elements_elementwise(hgx):
    """300 packed elements of 1 to 39 tokens in one to three segments of mixed kinds: hundreds
    of short work items, each ending inside a key block, several per CTA; element by element
    against the oracle."""
    rng = np.random.default_rng(77)
    batches = []
    for _ in range(300):
        n_seg = int(rng.integers(1, 4))
        batches.append([(int(rng.integers(1, 14)), int(rng.choice([0, 1, 2, 3]))) for _ in range(n_seg)])
    w = W.custom("tiny300", batches, seed=77)
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    ref, _, _ = _oracle_full(w, t)
    _compare(out.float().cpu().numpy(), ref, w.name)


def test_forward_multigen_full_size_sampled_rows(hgx):
    w = W.CONFIG_BY_NAME["hunyuan_multigen_9088"]
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    _check_sampled(w, t, out, seed=9)


def test_attention_alone_on_kernel_rotated_inputs(hgx):
    """The attention kernel against the oracle's masked softmax applied to the very bf16
    q'/k' the prologue kernel wrote (isolates attention error from prologue rounding)."""
    H, a = hgx
    w = W.config(1)
    t, d = _device_inputs(w)
    a.prologue(d["q"], d["k"], d["pos"], d["wq"], d["wk"])
    out = torch.empty_like(d["q"])
    a.attention(d["q"], d["k"], d["v"], out, *_desc(w))
    assert a.sync_status() == H.HGX_OK
    qp = d["q"].float().cpu().numpy().astype(np.float64)
    kp = d["k"].float().cpu().numpy().astype(np.float64)
    vv = t["v"].float().numpy().astype(np.float64)
    cu, segs, cu_segs = _desc(w)
    got = out.float().cpu().numpy()
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        bsegs = [tuple(int(x) for x in segs[n]) for n in range(cu_segs[b], cu_segs[b + 1])]
        ref = O.masked_gqa_attention(qp[t0:t1], kp[t0:t1], vv[t0:t1], O.dense_mask(bsegs, t1 - t0))
        err = np.abs(got[t0:t1] - ref)
        assert err.max() <= 1e-2 and err.mean() <= 5e-4, (float(err.max()), float(err.mean()))


def test_online_rescale_path_with_divergent_rows(hgx):
    """Key norms that grow along the sequence make the running row maximum jump by far
    more than 2^8 (in exp2 units) from one key block to the next, differently for every
    row, so the kernel's O/row-sum rescaling runs for some rows of a warp and not for
    others. Attention alone on given bf16 q'/k' against the oracle's masked softmax."""
    H, a = hgx
    w = W.custom("ramp", [[(300, W.CAUSAL), (400, W.FULL_SEQUENCE)], [(200, W.FULL_IN_SEGMENT), (333, W.CAUSAL)]],
                 seed=31)
    T = w.total_tokens
    g = torch.Generator().manual_seed(31)
    q = torch.randn(T, 32, 128, generator=g)
    k = torch.randn(T, 8, 128, generator=g)
    v = torch.randn(T, 8, 128, generator=g)
    # per batch element, key norms grow 120-fold from its first to its last token
    ramp = torch.cat([0.1 + 12.0 * torch.linspace(0, 1, L) ** 2 for L in w.lengths])
    k = k * ramp[:, None, None]
    q[:, ::3] *= 0.1  # some heads stay flat: rows of one warp disagree on rescaling
    qb, kb, vb = (x.to(torch.bfloat16) for x in (q, k, v))
    out = torch.empty(T, 32, 128, dtype=torch.bfloat16, device="cuda")
    a.attention(qb.cuda(), kb.cuda(), vb.cuda(), out, *_desc(w))
    assert a.sync_status() == H.HGX_OK
    cu, segs, cu_segs = _desc(w)
    got = out.float().cpu().numpy()
    f64 = lambda x: x.float().numpy().astype(np.float64)
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        bsegs = [tuple(int(x) for x in segs[n]) for n in range(cu_segs[b], cu_segs[b + 1])]
        ref = O.masked_gqa_attention(f64(qb[t0:t1]), f64(kb[t0:t1]), f64(vb[t0:t1]), O.dense_mask(bsegs, t1 - t0))
        err = np.abs(got[t0:t1] - ref)
        assert np.isfinite(got[t0:t1]).all()
        assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (float(err.max()), float(err.mean()))


def test_forward_from_reuses_the_text_prefix(hgx):
    """A denoising step that keeps the text before <|tms|> (causal, so unchanged across
    steps: model card, "What this model is" and "Performance") and recomputes the rest.
    The whole step-1 output is compared element by element with the fp64 oracle on the
    step-1 inputs (the reused rows come from step 0, whose inputs they share); in addition
    the recomputed rows are bit-identical to a full forward on the same inputs, the reused
    output rows are left untouched and the recomputed k rows are rotated like a full
    prologue."""
    H, a = hgx
    w = W.config(1)  # CFG pair: (128 text + <|tms|>, 1024 patches), (16 text + <|tms|>, 1024)
    cu, segs, cu_segs = _desc(w)
    first = [128, 16]
    t0 = W.tensors(w)
    t1 = W.tensors(W.Workload(w.name, w.batches, seed=w.seed + 100, style=w.style))
    pos_h = W.positions(w)
    pos = torch.from_numpy(pos_h).cuda()
    wq, wk = t0["wq"].cuda(), t0["wk"].cuda()
    # step 0: full forward; k is rotated in place
    q0, k0, v0 = t0["q"].cuda(), t0["k"].cuda(), t0["v"].cuda()
    out0 = _nan_like(q0)
    a.forward(q0, k0, v0, out0, pos, wq, wk, cu, segs, cu_segs)
    suffix = torch.zeros(w.total_tokens, dtype=torch.bool)
    for b in range(len(cu) - 1):
        suffix[int(cu[b]) + first[b] : int(cu[b + 1])] = True
    mix = lambda new, old: torch.where(suffix[:, None, None], new, old)  # noqa: E731
    # step 1: new suffix inputs; the prefix keeps its rotated k and its outputs
    q1 = mix(t1["q"], t0["q"]).cuda()
    k1 = torch.where(suffix[:, None, None].cuda(), t1["k"].cuda(), k0)
    v1 = mix(t1["v"], t0["v"]).cuda()
    out1 = out0.clone()
    a.forward_from(q1, k1, v1, out1, pos, wq, wk, cu, segs, cu_segs, first)
    assert a.sync_status() == H.HGX_OK
    # against the oracle on the step-1 inputs (raw q, k, v: prefix from step 0, suffix new)
    ref, _, kp_ref = O.forward(mix(t1["q"], t0["q"]), mix(t1["k"], t0["k"]), mix(t1["v"], t0["v"]), pos_h, t0["wq"],
                               t0["wk"], cu, segs, cu_segs)
    got = out1.float().cpu().numpy()
    _compare(got, ref, "forward_from vs oracle")
    _compare(got[suffix.numpy()], ref[suffix.numpy()], "recomputed rows vs oracle")
    np.testing.assert_allclose(k1.float().cpu().numpy(), kp_ref, rtol=2.0 ** -8, atol=1e-5)
    # the same step computed from scratch by the full path
    qr, kr, vr = mix(t1["q"], t0["q"]).cuda(), mix(t1["k"], t0["k"]).cuda(), mix(t1["v"], t0["v"]).cuda()
    out_r = _nan_like(qr)
    a.forward(qr, kr, vr, out_r, pos, wq, wk, cu, segs, cu_segs)
    assert a.sync_status() == H.HGX_OK
    assert torch.equal(out1, out_r)
    assert torch.equal(out1[~suffix.cuda()], out0[~suffix.cuda()])
    assert torch.equal(k1, kr)  # the recomputed rows were rotated like a full prologue


def test_single_token_returns_its_value(hgx):
    """One causal token sees only itself: out[0, h] == v[0, h // 4] (rounded to bf16)."""
    w = W.custom("one", [[(1, W.CAUSAL)]], seed=5)
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    v = t["v"].float()
    for h in range(32):
        torch.testing.assert_close(out[0, h].float().cpu(), v[0, h // 4], rtol=2 ** -8, atol=1e-6)


def _sample_rows(w, n_random=24, seed=0):
    """Rows for the sampled full-size checks: one random row of every 64-token query block
    of every batch element (so every work item of the kernel is checked on one of its
    rows, for all 32 query heads), the rows around every segment boundary, the edges of
    128-key blocks every 2048 tokens, first and last rows, and n_random rows anywhere."""
    rows = set()
    cu = W.cu_seqlens(w)
    rng = np.random.default_rng(seed)
    for b, batch in enumerate(w.batches):
        base, L = int(cu[b]), w.lengths[b]
        for r0 in range(0, L, 64):
            rows.add(base + int(rng.integers(r0, min(L, r0 + 64))))
        for s in batch:
            for r in (s.start - 1, s.start, s.start + 1, s.start + s.length - 1):
                if 0 <= r < L:
                    rows.add(base + r)
        for edge in range(0, L, 2048):
            for r in (edge - 1, edge, edge + 31, edge + 32, edge + 63, edge + 64, edge + 127, edge + 128):
                if 0 <= r < L:
                    rows.add(base + r)
        rows.update({base, base + L - 1})
    rows.update(int(x) for x in rng.integers(0, w.total_tokens, size=n_random))
    return sorted(rows)


def _check_sampled(w, t, out, seed):
    """Every row written (finite: the buffer was NaN-filled) and the sampled rows within
    the tolerance of the oracle."""
    assert torch.isfinite(out).all(), f"{w.name}: rows left unwritten"
    rows = _sample_rows(w, seed=seed)
    blocks = {(b, (r - int(W.cu_seqlens(w)[b])) // 64) for r in rows
              for b in [int(np.searchsorted(W.cu_seqlens(w), r, side="right") - 1)]}
    assert len(blocks) == sum(-(-L // 64) for L in w.lengths)  # every query block sampled
    segs, cu_segs = W.flat_segments(w)
    ref = O.attention_rows(t["q"], t["k"], t["v"], W.positions(w), t["wq"], t["wk"], W.cu_seqlens(w), segs,
                           cu_segs, rows)
    return _compare(out[rows].float().cpu().numpy(), ref, w.name)


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_forward_full_size_sampled_rows(hgx, cfg):
    w = W.config(cfg)
    t, _ = _device_inputs(w)
    out, _ = _run(hgx, w)
    _check_sampled(w, t, out, seed=cfg)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_forward_is_deterministic(hgx, cfg):
    """Bit-identical outputs from two runs on fresh copies of the inputs (the schedule is
    fixed, and the combine kernel of split items sums its parts in a fixed order)."""
    w = W.config(cfg)
    _, d0 = _device_inputs(w)
    _, d1 = _device_inputs(w)
    o0, _ = _run(hgx, w, d0)
    o1, _ = _run(hgx, w, d1)
    assert torch.equal(o0, o1)


def test_output_canaries_untouched(hgx):
    H, a = hgx
    w = W.random_workload(7, max_batch=3, max_len=300)
    _, d = _device_inputs(w)
    T = w.total_tokens
    pad = torch.full((T + 2, 32, 128), -3.0, dtype=torch.bfloat16, device="cuda")
    a.forward(d["q"], d["k"], d["v"], pad[1:-1], d["pos"], d["wq"], d["wk"], *_desc(w))
    assert a.sync_status() == H.HGX_OK
    assert bool((pad[0] == -3.0).all()) and bool((pad[-1] == -3.0).all())
    assert torch.isfinite(pad[1:-1].float()).all()


def test_maximum_token_count_sampled(hgx):
    """The largest packed size the ABI accepts (2^19 - 1 tokens, 128 batch elements):
    exercises the highest byte offsets. Every element carries the same q, k, v (a
    4096-token draw, the last element its first 4095 tokens) and one of two segment
    layouts, so every element must reproduce, bit for bit, the first element of its layout:
    with the output NaN-filled, a dropped or misplaced work item anywhere fails. The first
    element of each layout and the last element are checked against the oracle on one
    random row of every 64-token query block."""
    H, a = hgx
    n_el, per = 128, 4096
    total = (1 << 19) - 1
    lens = [per] * (n_el - 1) + [total - per * (n_el - 1)]
    layouts = [[(per // 4, W.CAUSAL), (per // 2, kd), (per - per // 4 - per // 2, W.CAUSAL)]
               for kd in (W.FULL_SEQUENCE, W.FULL_IN_SEGMENT)]
    last = [(per // 4, W.CAUSAL), (per // 2, W.FULL_SEQUENCE), (lens[-1] - per // 4 - per // 2, W.CAUSAL)]
    batches = [layouts[i % 2] for i in range(n_el - 1)] + [last]
    w = W.custom("max_tokens", batches, seed=21)
    assert w.total_tokens == total
    one = W.tensors(W.custom("max_el", [layouts[0]], seed=21))
    dev = {n: one[n].cuda() for n in ("q", "k", "v")}
    big = {n: x.repeat(n_el, 1, 1)[:total] for n, x in dev.items()}
    del dev
    big["pos"] = torch.from_numpy(W.positions(w)).cuda()
    big["wq"], big["wk"] = one["wq"].cuda(), one["wk"].cuda()
    out, _ = _run(hgx, w, big)
    del big
    assert torch.isfinite(out).all(), "rows left unwritten"
    for i in range(2, n_el - 1):
        assert torch.equal(out[i * per:(i + 1) * per], out[(i % 2) * per:(i % 2 + 1) * per]), f"element {i}"
    for idx, lay in ((0, layouts[0]), (1, layouts[1]), (n_el - 1, last)):
        sub_w = W.custom(f"max_el_{idx}", [lay], seed=21)
        L = sub_w.total_tokens
        t_el = {n: (one[n][:L] if n in ("q", "k", "v") else one[n]) for n in one}
        _check_sampled(sub_w, t_el, out[idx * per: idx * per + L], seed=idx)


def test_empty_batch_is_a_no_op(hgx):
    H, a = hgx
    z = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    a.forward(z, z, z, z, z, z, z, [0, 0], np.zeros((0, 3)), [0, 0])


def test_injected_allocation_failure_reports_oom_and_handle_recovers(hgx):
    """A one-shot test hook makes the planner's scratch allocation fail: the forward returns
    HGX_ERR_OOM before launching anything (q and k stay untouched), and the next call on the
    same handle allocates and matches the oracle."""
    H, _ = hgx
    w = W.config(0)
    t, d = _device_inputs(w)
    a = H.Attention()  # a fresh handle: its first forward has to allocate
    try:
        out = torch.empty_like(d["q"])
        q0, k0 = d["q"].clone(), d["k"].clone()
        a.set_debug(H.HGX_DEBUG_FAIL_ALLOC, 0)
        with pytest.raises(H.HgxError) as e:
            a.forward(d["q"], d["k"], d["v"], out, d["pos"], d["wq"], d["wk"], *_desc(w))
        assert e.value.status == H.HGX_ERR_OOM
        assert "injected" in a.last_error()
        torch.cuda.synchronize()
        assert torch.equal(d["q"], q0) and torch.equal(d["k"], k0)
        a.forward(d["q"], d["k"], d["v"], out, d["pos"], d["wq"], d["wk"], *_desc(w))
        ref, _, _ = _oracle_full(w, t)
        _compare(out.float().cpu().numpy(), ref, "after-injected-oom")
    finally:
        a.close()


def test_bounded_wait_reports_timeout_and_context_survives(hgx):
    """A softmax warpgroup waits on a barrier that nothing arrives at; its bounded wait
    runs out, the kernel drains and exits, the host sees HGX_ERR_TIMEOUT, and the next
    normal call on the same context is correct."""
    H, a = hgx
    w = W.config(0)
    t, d = _device_inputs(w)
    out = torch.empty_like(d["q"])
    q0, k0 = d["q"].clone(), d["k"].clone()
    a.set_debug(H.HGX_DEBUG_STALL_TEST | H.HGX_DEBUG_CHECKED, 20_000_000)
    with pytest.raises(H.HgxError) as e:
        a.forward(d["q"], d["k"], d["v"], out, d["pos"], d["wq"], d["wk"], *_desc(w))
    assert e.value.status == H.HGX_ERR_TIMEOUT
    a.set_debug(0, 0)
    d["q"].copy_(q0)
    d["k"].copy_(k0)
    out, _ = _run(hgx, w, d)
    ref, _, _ = _oracle_full(w, t)
    _compare(out.float().cpu().numpy(), ref, "after-timeout")


@pytest.mark.parametrize("poison", ["nan_in_element_1", "inf_in_element_2"])
def test_non_finite_v_of_a_later_element_does_not_leak(hgx, poison):
    """A key block that runs past the end of its batch element also covers the next
    element's first keys. Their probabilities are exact zeros, but 0 * NaN = NaN, so the
    kernel must not let those V rows into the earlier element's P V: with NaN (or inf) V in
    a later element, every earlier element still matches the oracle element by element."""
    H, a = hgx
    w = W.custom("poison", [[(200, W.CAUSAL), (100, W.FULL_SEQUENCE)], [(90, W.FULL_IN_SEGMENT), (60, W.CAUSAL)],
                            [(77, W.FULL_SEQUENCE)]], seed=41)
    cu = W.cu_seqlens(w)  # 0, 300, 450, 527: elements 0 and 1 end inside a 128-key block
    t = W.tensors(w)
    v = t["v"].clone()
    if poison == "nan_in_element_1":
        v[int(cu[1]):int(cu[1]) + 84] = float("nan")
        clean = [0]
    else:
        v[int(cu[2]):int(cu[3])] = float("inf")
        clean = [0, 1]
    t["v"] = v
    d = {n: x.cuda() for n, x in t.items()}
    d["pos"] = torch.from_numpy(W.positions(w)).cuda()
    out, _ = _run(hgx, w, d)
    ref, _, _ = _oracle_full(w, t)
    got = out.float().cpu().numpy()
    for b in clean:
        r0, r1 = int(cu[b]), int(cu[b + 1])
        _compare(got[r0:r1], ref[r0:r1], f"{poison}: element {b}")


@pytest.mark.parametrize("case", ["c0", "c1", "random_a", "random_b", "reuse"])
def test_split_items_and_combine_elementwise(hgx, case):
    """Split work items: with HGX_DEBUG_SPLIT_TEST every prefix-form item of two or more key
    blocks runs as two halves by key blocks, whose partial (O, row maximum, row sum) the
    combine kernel merges; element by element against the oracle (the 2048^2 CFG pair and
    the Hunyuan GCA workload take the split schedule on their own, in the sampled tests)."""
    H, _ = hgx
    a = H.Attention()
    try:
        a.set_debug(H.HGX_DEBUG_SPLIT_TEST)
        w = {"c0": W.config(0), "c1": W.config(1), "random_a": W.random_workload(61, max_batch=3, max_len=900),
             "random_b": W.random_workload(62, max_batch=4, max_len=700, allow_empty=True),
             "reuse": W.config(1)}[case]
        if w.total_tokens == 0:
            pytest.skip("empty draw")
        t, d = _device_inputs(w)
        cu, segs, cu_segs = _desc(w)
        assert H.schedule(cu, segs, cu_segs, 148, 2)[:, 5].max() >= 0  # something is split
        out = _nan_like(d["q"])
        if case == "reuse":  # prefix reuse on split items: rows before <|tms|> are kept
            first = [128, 16]
            out.fill_(3.0)
            # the reused rows' k must already hold k': rotate a copy, keep the prefix rows
            qr, kr = d["q"].clone(), d["k"].clone()
            a.prologue(qr, kr, d["pos"], d["wq"], d["wk"])
            prefix = torch.zeros(w.total_tokens, dtype=torch.bool, device="cuda")
            for b in range(2):
                prefix[int(cu[b]):int(cu[b]) + first[b]] = True
            k_in = torch.where(prefix[:, None, None], kr, d["k"])
            a.forward_from(d["q"], k_in, d["v"], out, d["pos"], d["wq"], d["wk"], cu, segs, cu_segs, first)
            assert a.sync_status() == H.HGX_OK
            ref, _, _ = _oracle_full(w, t)
            got = out.float().cpu().numpy()
            for b in range(2):
                r0, r1 = int(cu[b]), int(cu[b + 1])
                assert (got[r0:r0 + first[b]] == 3.0).all()
                _compare(got[r0 + first[b]:r1], ref[r0 + first[b]:r1], f"reuse element {b}")
            return
        a.forward(d["q"], d["k"], d["v"], out, d["pos"], d["wq"], d["wk"], cu, segs, cu_segs)
        assert a.sync_status() == H.HGX_OK
        ref, _, _ = _oracle_full(w, t)
        _compare(out.float().cpu().numpy(), ref, f"split {w.name}")
    finally:
        a.close()


def test_kernel_clock_stamps_of_the_last_attention_launch(hgx):
    """hgx_attn_kernel_clock: refused before any attention launch; afterwards the slowest
    CTA's cycles and span, and an effective SM clock that agrees with them and with the
    event-timed launch."""
    H, _ = hgx
    a = H.Attention()
    try:
        with pytest.raises(H.HgxError):
            a.kernel_clock()
        w = W.CONFIG_BY_NAME["hidream_t2i_1024_cfg"]
        _, d = _device_inputs(w)
        cu, segs, cu_segs = _desc(w)
        a.prologue(d["q"], d["k"], d["pos"], d["wq"], d["wk"])
        out = _nan_like(d["q"])
        stream = torch.cuda.current_stream()
        for _ in range(3):  # the plan is uploaded by the first call
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            a.attention(d["q"], d["k"], d["v"], out, cu, segs, cu_segs)
            e1.record(stream)
        cyc, ns, mhz = a.kernel_clock()
        assert a.sync_status() == H.HGX_OK
        assert bool(torch.isfinite(out).all())
        launch_ms = e0.elapsed_time(e1)
        assert cyc > 0 and ns > 0
        assert 300.0 < mhz < 2500.0, mhz
        assert ns * 1e-6 <= launch_ms * 1.02 + 0.005, (ns, launch_ms)  # inside the launch
        assert abs(cyc / (ns * 1e-3) / mhz - 1.0) < 0.1, (cyc, ns, mhz)
    finally:
        a.close()
