"""Pins of the fp64 oracle to facts the pages and the mathematics fix (no GPU).

Each test states what it pins and which mistake it would catch. None of them re-types the
oracle's own formula: they use hand-written fixtures, closed forms, library routines
(torch scaled_dot_product_attention in fp64), complex arithmetic and 50-digit brute force.
"""
import cmath
import math

import mpmath
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from conftest import parse_segments, read_golden

D = 128


# ------------------------------------------------------------------------------- masks
@pytest.mark.parametrize("fixture", ["mask_hidream_edit_tiny.txt", "mask_gca_tiny.txt", "mask_gca_multigen_tiny.txt"])
def test_dense_mask_matches_hand_written_fixture(fixture):
    """Hand-derived masks from the HiDream and HunyuanImage rules (catches a swapped
    kind, an off-by-one on the diagonal, or a segment rule that looks backwards)."""
    lines = read_golden(fixture)
    segs = parse_segments(lines[0])
    expect = np.array([[c == "1" for c in row] for row in lines[1:]])
    L = expect.shape[0]
    np.testing.assert_array_equal(O.dense_mask(segs, L), expect)


def test_single_gen_image_is_canonical_gca():
    """With one Gen Image and nothing after it the training mask is the canonical
    Generalized Causal Attention mask (section 3.4, "Why this works at inference")."""
    segs_gen = [(0, 7, O.CAUSAL), (7, 9, O.GEN_IMAGE)]
    segs_gca = [(0, 7, O.CAUSAL), (7, 9, O.FULL_IN_SEGMENT)]
    np.testing.assert_array_equal(O.dense_mask(segs_gen, 16), O.dense_mask(segs_gca, 16))
    # a Gen Image followed by text: the text rows lose exactly the image's keys
    g = O.dense_mask([(0, 3, O.CAUSAL), (3, 4, O.GEN_IMAGE), (7, 5, O.CAUSAL)], 12)
    c = O.dense_mask([(0, 3, O.CAUSAL), (3, 4, O.FULL_IN_SEGMENT), (7, 5, O.CAUSAL)], 12)
    diff = c & ~g
    assert not (g & ~c).any()
    assert diff[7:, 3:7].all() and diff.sum() == 5 * 4


def test_rows_after_a_gen_image_ignore_it():
    """Perturbing K and V of a Gen Image leaves every later row bit-identical."""
    segs = [(0, 10, O.CAUSAL), (10, 12, O.GEN_IMAGE), (22, 6, O.CAUSAL), (28, 9, O.GEN_IMAGE), (37, 4, O.CAUSAL)]
    L = 41
    q, k, v = _rand_qkv(L, 12)
    mask = O.dense_mask(segs, L)
    base = O.masked_gqa_attention(q, k, v, mask)
    k2, v2 = k.copy(), v.copy()
    k2[10:22] += 3.0
    v2[10:22] -= 2.0
    got = O.masked_gqa_attention(q, k2, v2, mask)
    np.testing.assert_array_equal(got[22:], base[22:])
    assert not np.array_equal(got[10:22], base[10:22])


def test_unmasked_pairs_closed_forms():
    """Visible-pair counts of the five workloads against closed forms derived by hand."""
    rows = {ln.split()[0]: int(ln.split()[1]) for ln in read_golden("unmasked_pairs.txt")}
    for w in W.CONFIGS:
        total = 0
        for b, batch in enumerate(w.batches):
            segs = [(s.start, s.length, s.kind) for s in batch]
            total += O.unmasked_pairs(segs, w.lengths[b])
        assert total == rows[w.name], w.name


def test_tile_classes_hand_derived_config0():
    lines = read_golden("tiles_hidream_tiny_321.txt")
    bm, bn = int(lines[0].split()[1]), int(lines[0].split()[3])
    expect = np.array([[{"S": 0, "P": 1, "F": 2}[c] for c in row] for row in lines[1:]], dtype=np.uint8)
    w = W.config(0)
    segs = [(s.start, s.length, s.kind) for s in w.batches[0]]
    got = O.tile_classes(O.dense_mask(segs, 321), bm, bn)
    np.testing.assert_array_equal(got, expect)


def _sdpa_gqa(q, k, v, is_causal=False, mask=None):
    # torch fp64 reference: expand KV heads to query heads (h -> h // G)
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(np.repeat(k, G, axis=1)).permute(1, 0, 2)
    vt = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, is_causal=is_causal)
    return o.permute(1, 0, 2).numpy()


def _rand_qkv(L, seed, hq=8, hkv=2, d=16):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((L, hq, d)), rng.standard_normal((L, hkv, d)), rng.standard_normal((L, hkv, d))


def test_all_causal_reduces_to_library_causal_attention():
    """An all-text sequence is plain causal attention (HunyuanImage 3.0 section 3.4:
    text tokens attend only to previous tokens)."""
    q, k, v = _rand_qkv(37, 1)
    segs = [(0, 10, O.CAUSAL), (10, 27, O.CAUSAL)]
    got = O.masked_gqa_attention(q, k, v, O.dense_mask(segs, 37))
    np.testing.assert_allclose(got, _sdpa_gqa(q, k, v, is_causal=True), rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", [O.FULL_SEQUENCE, O.FULL_IN_SEGMENT])
def test_all_generation_reduces_to_full_attention(kind):
    """A sequence of generation tokens only is full (unmasked) attention."""
    q, k, v = _rand_qkv(29, 2)
    got = O.masked_gqa_attention(q, k, v, O.dense_mask([(0, 29, kind)], 29))
    np.testing.assert_allclose(got, _sdpa_gqa(q, k, v), rtol=0, atol=1e-12)


def test_gqa_head_mapping_is_contiguous_groups():
    """With a V that is constant over tokens, each query head returns the V of its KV
    head; query head h must read KV head h // 4 (32 query heads over 8 KV heads)."""
    L = 5
    rng = np.random.default_rng(3)
    q = rng.standard_normal((L, 32, 8))
    k = rng.standard_normal((L, 8, 8))
    v = np.zeros((L, 8, 8))
    for g in range(8):
        v[:, g, :] = g + 1.0
    out = O.masked_gqa_attention(q, k, v, O.dense_mask([(0, L, O.CAUSAL)], L))
    for h in range(32):
        np.testing.assert_allclose(out[:, h, :], h // 4 + 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("wl", [0, 4])
def test_rows_invariant_to_tokens_they_cannot_see(wl):
    """Perturbing K and V of tokens at or beyond a row's last visible key leaves that
    row's output bit-identical (causal text/condition rows; image rows of a segment)."""
    w = W.config(wl) if wl == 0 else W.custom("gca_small", [[(20, 0), (30, 2), (10, 0), (25, 2), (5, 0)]])
    segs = [(s.start, s.length, s.kind) for s in w.batches[0]]
    L = w.lengths[0]
    q, k, v = _rand_qkv(L, 4)
    mask = O.dense_mask(segs, L)
    base = O.masked_gqa_attention(q, k, v, mask)
    rng = np.random.default_rng(5)
    for i in range(0, L, max(1, L // 13)):
        lim = int(np.nonzero(mask[i])[0].max()) + 1
        if lim >= L:
            continue
        k2, v2 = k.copy(), v.copy()
        k2[lim:] += rng.standard_normal(k2[lim:].shape)
        v2[lim:] += rng.standard_normal(v2[lim:].shape)
        got = O.masked_gqa_attention(q, k2, v2, mask)
        np.testing.assert_array_equal(got[i], base[i])


def test_softmax_attention_brute_force_50_digits():
    """Tiny inputs (L = 7, D = 4) recomputed with 50-digit arithmetic."""
    mpmath.mp.dps = 50
    L, d = 7, 4
    q, k, v = _rand_qkv(L, 6, hq=2, hkv=1, d=d)
    segs = [(0, 2, O.CAUSAL), (2, 3, O.FULL_IN_SEGMENT), (5, 2, O.FULL_SEQUENCE)]
    mask = O.dense_mask(segs, L)
    got = O.masked_gqa_attention(q, k, v, mask)
    scale = mpmath.mpf(1) / mpmath.sqrt(d)
    for i in range(L):
        for h in range(2):
            w = []
            for j in range(L):
                if mask[i, j]:
                    s = sum(mpmath.mpf(q[i, h, c]) * mpmath.mpf(k[j, 0, c]) for c in range(d)) * scale
                    w.append((j, mpmath.e ** s))
            z = sum(e for _, e in w)
            for c in range(d):
                ref = sum(e * mpmath.mpf(v[j, 0, c]) for j, e in w) / z
                assert abs(float(ref) - got[i, h, c]) < 1e-12


# ------------------------------------------------------------------------------- RMSNorm
def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 3, D)) * 3.0
    y = O.rms_norm(x, np.ones(D), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(O.rms_norm(17.0 * x, np.ones(D), 0.0), y, rtol=1e-13)


def test_rmsnorm_closed_form_with_eps_and_weight():
    """A constant vector c: output c / sqrt(c^2 + eps) * w (eps inside the root, weight
    multiplies per feature)."""
    c, eps = 0.01, 1e-4
    w = np.linspace(0.5, 1.5, D)
    y = O.rms_norm(np.full((1, D), c), w, eps)
    np.testing.assert_allclose(y[0], c / math.sqrt(c * c + eps) * w, rtol=1e-14)


# ------------------------------------------------------------------------------- mRoPE
def _rope_1d_complex(x, p, theta):
    """1D RoPE written as complex multiplication of the half-split pairs (x_k, x_{k+D/2})."""
    d = x.shape[-1]
    half = d // 2
    out = np.empty_like(x)
    for k in range(half):
        rot = cmath.exp(1j * p * math.exp(-(2.0 * k / d) * math.log(theta)))
        z = (x[..., k] + 1j * x[..., k + half]) * rot
        out[..., k], out[..., k + half] = z.real, z.imag
    return out


def test_mrope_equal_axes_reduces_to_1d_rope():
    """Text on the diagonal (n, n, n) is exactly 1D RoPE ("reduces exactly to 1D RoPE",
    HunyuanImage 3.0 section 3.4 and "Key claims")."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((6, 2, D))
    ps = np.array([0, 1, 7, 250, 4353, 9087])
    pos = np.stack([ps, ps, ps], axis=1)
    got = O.rope_rotate_half(x, O.mrope_angles(pos, 5e6, D, (24, 20, 20)))
    for n, p in enumerate(ps):
        np.testing.assert_allclose(got[n], _rope_1d_complex(x[n], float(p), 5e6), rtol=0, atol=1e-10)


def test_mrope_preserves_pair_norms():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((20, 3, D))
    pos = rng.integers(0, 9000, size=(20, 3))
    y = O.rope_rotate_half(x, O.mrope_angles(pos, 5e6, D, (24, 20, 20)))
    h = D // 2
    np.testing.assert_allclose(y[..., :h] ** 2 + y[..., h:] ** 2, x[..., :h] ** 2 + x[..., h:] ** 2, rtol=1e-12)


def test_mrope_scores_depend_on_relative_position_only():
    """<rope(q, p + d), rope(k, p' + d)> == <rope(q, p), rope(k, p')> for one shift d
    applied to all three axes of both tokens."""
    rng = np.random.default_rng(10)
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, D))
    p, pk = np.array([[300, 12, 40]]), np.array([[250, 3, 61]])
    dlt = np.array([[1234, 77, 5]])
    ang = lambda x: O.mrope_angles(x, 5e6, D, (24, 20, 20))
    a = np.sum(O.rope_rotate_half(q, ang(p)) * O.rope_rotate_half(k, ang(pk)))
    b = np.sum(O.rope_rotate_half(q, ang(p + dlt)) * O.rope_rotate_half(k, ang(pk + dlt)))
    assert abs(a - b) < 1e-9 * max(1.0, abs(a))


def test_mrope_section_sizes_24_20_20():
    """Moving one axis only rotates exactly that axis's share of the 64 pairs: 24 for t,
    20 for h, 20 for w (sections [24, 20, 20])."""
    x = np.ones((1, 1, D))
    for axis, count in ((0, 24), (1, 20), (2, 20)):
        pos = np.zeros((1, 3), dtype=np.int64)
        pos[0, axis] = 5
        y = O.rope_rotate_half(x, O.mrope_angles(pos, 5e6, D, (24, 20, 20)))
        moved = np.abs(y[0, 0, : D // 2] - 1.0) > 1e-15
        assert moved.sum() == count


def test_mrope_frequency_closed_forms():
    inv = O.mrope_inv_freq(5e6, D)
    assert inv[0] == 1.0
    assert abs(inv[32] - 1.0 / math.sqrt(5e6)) < 1e-18
    assert abs(inv[63] - math.exp(-(126.0 / 128.0) * math.log(5e6))) < 1e-20


@pytest.mark.parametrize("name,layout", [("alternating", O.ROPE_2D_ALTERNATING), ("halves", O.ROPE_2D_HALVES)])
def test_2d_rope_layouts_match_the_passage(name, layout):
    """The two readings of the Generalized 2D RoPE, written out by hand from the passage;
    moving x only rotates exactly the x frequencies; text on the diagonal (n, n) is 1D RoPE."""
    row = {ln.split()[0]: ln.split()[1] for ln in read_golden("rope2d_layouts.txt")}[name]
    axis = O.mrope_axis_of_frequency(D, (24, 20, 20), layout)
    assert "".join("x" if a == 2 else "y" if a == 1 else "t" for a in axis) == row
    x = np.ones((1, 1, D))
    pos = np.array([[0, 0, 9]])  # (t, h = y, w = x)
    y = O.rope_rotate_half(x, O.mrope_angles(pos, 5e6, D, (24, 20, 20), layout))
    moved = np.abs(y[0, 0, : D // 2] - 1.0) > 1e-15
    assert "".join("x" if m else "y" for m in moved) == row
    rng = np.random.default_rng(13)
    v = rng.standard_normal((3, 2, D))
    ps = np.array([5, 77, 4000])
    got = O.rope_rotate_half(v, O.mrope_angles(np.stack([ps, ps, ps], 1), 5e6, D, (24, 20, 20), layout))
    for n, p_ in enumerate(ps):
        np.testing.assert_allclose(got[n], _rope_1d_complex(v[n], float(p_), 5e6), rtol=0, atol=1e-10)


def test_prologue_order_norm_then_rotate():
    """RMSNorm before RoPE: the output's RMS per head equals that of rms(x) * w at every
    position (rotation keeps norms), so changing the position never changes it."""
    w = W.config(0)
    t = W.tensors(w)
    pos = W.positions(w)
    qp, kp = O.prologue(t["q"][:8], t["k"][:8], pos[:8], t["wq"], t["wk"])
    qn = O.rms_norm(O.bf16_to_f64(t["q"][:8]), O.bf16_to_f64(t["wq"]), 1e-6)
    np.testing.assert_allclose(np.linalg.norm(qp, axis=-1), np.linalg.norm(qn, axis=-1), rtol=1e-12)


def test_layer_with_selecting_weights_reduces_to_the_core():
    """With projection weights that copy input columns (0/1 matrices) the layer is the
    attention core on those columns, and an identity output projection returns the
    attention output unchanged: pins the q | k | v column order and both transposes."""
    rng = np.random.default_rng(21)
    T, hidden = 12, 4096
    x = rng.standard_normal((T, hidden))
    perm = rng.permutation(hidden)
    w_qkv = np.zeros((6144, hidden))
    cols = np.concatenate([perm, perm[:2048]])  # q from perm[:4096], k and v from perm[:1024], perm[1024:2048]
    w_qkv[np.arange(6144), cols] = 1.0
    w_o = np.eye(4096)
    pos = np.stack([np.arange(T)] * 3, axis=1)
    segs = np.array([[0, 5, O.CAUSAL], [5, 7, O.FULL_SEQUENCE]])
    wq = np.ones(128)
    y, att, qp, kp, v = O.layer_forward(x, w_qkv, w_o, pos, wq, wq, [0, T], segs, [0, 2])
    q_in = x[:, perm[:4096]].reshape(T, 32, 128)
    k_in = x[:, perm[:1024]].reshape(T, 8, 128)
    v_in = x[:, perm[1024:2048]].reshape(T, 8, 128)
    ref, qr, kr = O.forward(q_in, k_in, v_in, pos, wq, wq, [0, T], segs, [0, 2])
    np.testing.assert_allclose(att, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y, att.reshape(T, -1), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(v, v_in)


def test_layer_rows_agrees_with_layer_forward():
    """The sampled-rows layer oracle used at full size equals the whole-layer oracle."""
    w = W.custom("small_layer", [[(9, W.CAUSAL), (14, W.FULL_IN_SEGMENT), (6, W.GEN_IMAGE), (5, W.CAUSAL)]], seed=8)
    lt = W.layer_tensors(w)
    segs, cu_segs = W.flat_segments(w)
    pos, cu = W.positions(w), W.cu_seqlens(w)
    y, att, _, _, _ = O.layer_forward(lt["x"], lt["w_qkv"], lt["w_o"], pos, lt["wq"], lt["wk"], cu, segs, cu_segs)
    rows = [0, 8, 9, 22, 23, 30, 33]
    y_r, att_r = O.layer_rows(lt["x"], lt["w_qkv"], lt["w_o"], pos, lt["wq"], lt["wk"], cu, segs, cu_segs, rows)
    np.testing.assert_allclose(att_r, att[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(y_r, y[rows], rtol=0, atol=1e-11)


@pytest.mark.parametrize("case", ["random_holes", "random_multi", "random_empty", "params"])
def test_attention_rows_agrees_with_forward(case):
    """The sampled-rows oracle that the full-size GPU tests and the CPU baseline use equals
    the whole-sequence oracle (itself pinned to library SDPA and 50-digit brute force) on
    EVERY row of small packed batches: several batch elements (so a row must take the keys
    of its own element), empty elements, all four segment kinds including Gen Image holes,
    and non-default theta / eps / scale (so each is passed through). A wrong head mapping
    (h % Hkv), a dropped scale, a prologue over the wrong key range or a mask row of the
    wrong token each fails here."""
    if case == "random_holes":
        w = W.random_workload(71, max_batch=3, max_len=160, kinds=(0, 1, 2, 3, 3))
        kw = {}
    elif case == "random_multi":
        w = W.random_workload(72, max_batch=4, max_len=150)
        kw = {}
    elif case == "random_empty":
        w = W.custom("with_empty", [[(13, W.CAUSAL), (20, W.FULL_SEQUENCE)], [], [(7, W.FULL_IN_SEGMENT), (9, W.CAUSAL)]],
                     seed=73)
        kw = {}
    else:
        w = W.custom("params", [[(11, W.CAUSAL), (17, W.GEN_IMAGE), (6, W.CAUSAL)], [(21, W.FULL_SEQUENCE)]], seed=74)
        kw = dict(theta=1.0e4, eps=0.25, scale=0.05)
    t = W.tensors(w)
    segs, cu_segs = W.flat_segments(w)
    pos, cu = W.positions(w), W.cu_seqlens(w)
    assert len(cu) - 1 >= 2 or case == "random_holes"
    ref, _, _ = O.forward(t["q"], t["k"], t["v"], pos, t["wq"], t["wk"], cu, segs, cu_segs, **kw)
    rows = list(range(w.total_tokens))
    got = O.attention_rows(t["q"], t["k"], t["v"], pos, t["wq"], t["wk"], cu, segs, cu_segs, rows, **kw)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # an unordered subset with a repeat gives the same rows
    sub = [rows[-1], rows[0], rows[len(rows) // 2], rows[0]]
    got_sub = O.attention_rows(t["q"], t["k"], t["v"], pos, t["wq"], t["wk"], cu, segs, cu_segs, sub, **kw)
    np.testing.assert_allclose(got_sub, ref[sub], rtol=0, atol=1e-12)
