"""GPU parity of the attention layer around the core: the tcgen05 GEMMs of the QKV
projection (with q/k RMSNorm and rotation in the epilogue) and of the output projection,
and the whole layer, against the fp64 oracle, through the C ABI.

Tolerances: the projections accumulate in fp32 and round to bf16, so q', k', v and the
plain GEMM are compared within bf16 rounding (relative 2^-8 + small absolute); the layer
output y and the attention output within max |err| <= 2e-2, mean |err| <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("T", [1, 129, 300, 2194])
def test_out_projection_gemm_against_fp32_matmul(hgx, T):
    """Plain GEMM y = a w^T (ragged row counts: tails of the 128-row tiles)."""
    H, a = hgx
    g = torch.Generator().manual_seed(T)
    att = torch.randn(T, 4096, generator=g).to(torch.bfloat16).cuda()
    w_o = (torch.randn(4096, 4096, generator=g) / 64).to(torch.bfloat16).cuda()
    y = torch.full((T + 1, 4096), 5.0, dtype=torch.bfloat16, device="cuda")
    a.out_projection(att, w_o, y[:T])
    assert a.sync_status() == H.HGX_OK
    ref = att.double() @ w_o.double().T
    err = (y[:T].double() - ref).abs()
    assert (err <= 2.0 ** -8 * ref.abs() + 2e-3).all(), float(err.max())
    assert bool((y[T] == 5.0).all())  # nothing written past the last row


@pytest.mark.parametrize("cfg", [0, 1])
def test_qkv_projection_with_fused_norm_and_rotation(hgx, cfg):
    H, a = hgx
    w = W.config(cfg)
    lt = W.layer_tensors(w)
    d = {n: t.cuda() for n, t in lt.items()}
    T = w.total_tokens
    pos = torch.from_numpy(W.positions(w)).cuda()
    q = torch.empty(T, 32, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(T, 8, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(T, 8, 128, dtype=torch.bfloat16, device="cuda")
    a.qkv_projection(d["x"], d["w_qkv"], q, k, v, pos, d["wq"], d["wk"])
    assert a.sync_status() == H.HGX_OK
    q_r, k_r, v_r = O.qkv_projection(lt["x"], lt["w_qkv"])
    phi = O.mrope_angles(W.positions(w), 5e6, 128, (24, 20, 20))
    qp = O.rope_rotate_half(O.rms_norm(q_r, O.bf16_to_f64(lt["wq"]), 1e-6), phi)
    kp = O.rope_rotate_half(O.rms_norm(k_r, O.bf16_to_f64(lt["wk"]), 1e-6), phi)
    for got, ref in ((q, qp), (k, kp), (v, v_r)):
        np.testing.assert_allclose(got.float().cpu().numpy(), ref, rtol=2.0 ** -8, atol=2e-3)


def test_qkv_projection_at_large_positions(hgx):
    """The projection's (cos, sin) table (fp64 angles per token and frequency) at positions
    around and beyond 2^24 and down to -2^30, against the oracle's rotation."""
    H, a = hgx
    w = W.config(0)
    lt = W.layer_tensors(w)
    d = {n: t.cuda() for n, t in lt.items()}
    T = w.total_tokens
    rng = np.random.default_rng(29)
    pos = np.empty((T, 3), dtype=np.int64)
    pos[: T // 3] = (1 << 24) + rng.integers(-8, 8, size=(T // 3, 3))
    pos[T // 3: 2 * T // 3] = rng.integers(1 << 20, 1 << 30, size=(2 * T // 3 - T // 3, 3))
    pos[2 * T // 3:] = -rng.integers(1 << 20, 1 << 30, size=(T - 2 * T // 3, 3))
    pos = pos.astype(np.int32)
    q = torch.empty(T, 32, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(T, 8, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(T, 8, 128, dtype=torch.bfloat16, device="cuda")
    a.qkv_projection(d["x"], d["w_qkv"], q, k, v, torch.from_numpy(pos).cuda(), d["wq"], d["wk"])
    assert a.sync_status() == H.HGX_OK
    q_r, k_r, _ = O.qkv_projection(lt["x"], lt["w_qkv"])
    phi = O.mrope_angles(pos, 5e6, 128, (24, 20, 20))
    qp = O.rope_rotate_half(O.rms_norm(q_r, O.bf16_to_f64(lt["wq"]), 1e-6), phi)
    kp = O.rope_rotate_half(O.rms_norm(k_r, O.bf16_to_f64(lt["wk"]), 1e-6), phi)
    for got, ref in ((q, qp), (k, kp)):
        np.testing.assert_allclose(got.float().cpu().numpy(), ref, rtol=2.0 ** -8, atol=2e-3)


def _layer(hgx, w):
    H, a = hgx
    lt = W.layer_tensors(w)
    d = {n: t.cuda() for n, t in lt.items()}
    T = w.total_tokens
    pos = torch.from_numpy(W.positions(w)).cuda()
    q = torch.empty(T, 32, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(T, 8, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(T, 8, 128, dtype=torch.bfloat16, device="cuda")
    att = torch.full((T, 32, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.full((T, 4096), float("nan"), dtype=torch.bfloat16, device="cuda")
    a.layer_forward(d["x"], d["w_qkv"], d["w_o"], q, k, v, att, y, pos, d["wq"], d["wk"], *_desc(w))
    assert a.sync_status() == H.HGX_OK
    return lt, y, att


def _check(got, ref, what):
    err = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= 2e-2 and err.mean() <= 1e-3, (what, float(err.max()), float(err.mean()))


@pytest.mark.parametrize("cfg", [0, 1])
def test_layer_forward_elementwise(hgx, cfg):
    w = W.config(cfg)
    lt, y, att = _layer(hgx, w)
    segs, cu_segs = W.flat_segments(w)
    y_r, att_r, _, _, _ = O.layer_forward(lt["x"], lt["w_qkv"], lt["w_o"], W.positions(w), lt["wq"], lt["wk"],
                                          W.cu_seqlens(w), segs, cu_segs)
    _check(att.float().cpu().numpy(), att_r, "attention")
    _check(y.float().cpu().numpy(), y_r, "y")


@pytest.mark.parametrize("seed", range(3))
def test_layer_forward_random_layouts_elementwise(hgx, seed):
    """The whole layer on random packed layouts (all four segment kinds, ragged elements,
    Gen Image holes): row counts that end inside a 128-row GEMM tile, and batch elements
    that start inside one."""
    w = W.random_workload(500 + seed, max_batch=3, max_len=900, kinds=(0, 1, 2, 3))
    lt, y, att = _layer(hgx, w)
    segs, cu_segs = W.flat_segments(w)
    y_r, att_r, _, _, _ = O.layer_forward(lt["x"], lt["w_qkv"], lt["w_o"], W.positions(w), lt["wq"], lt["wk"],
                                          W.cu_seqlens(w), segs, cu_segs)
    _check(att.float().cpu().numpy(), att_r, w.name + " attention")
    _check(y.float().cpu().numpy(), y_r, w.name + " y")


def test_layer_forward_full_size_sampled_rows(hgx):
    """The edit step's layer (8449 tokens): att and y are NaN-filled before the call and
    must come back finite everywhere; one random row of every 64-token query block (every
    attention work item and every 128-row GEMM tile) plus the segment boundaries are
    compared with the oracle."""
    w = W.config(3)
    lt, y, att = _layer(hgx, w)
    assert torch.isfinite(att).all() and torch.isfinite(y).all()
    rng = np.random.default_rng(3)
    T = w.total_tokens
    rows = {0, 256, 257, 4352, 4353, T - 1} | {int(rng.integers(r0, min(T, r0 + 64))) for r0 in range(0, T, 64)}
    rows = sorted(rows)
    segs, cu_segs = W.flat_segments(w)
    y_r, att_r = O.layer_rows(lt["x"], lt["w_qkv"], lt["w_o"], W.positions(w), lt["wq"], lt["wk"], W.cu_seqlens(w),
                              segs, cu_segs, rows)
    _check(att[rows].float().cpu().numpy(), att_r, "attention")
    _check(y[rows].float().cpu().numpy(), y_r, "y")
