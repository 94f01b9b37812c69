"""Plain, slow, fp64 oracle for the hybrid-masked attention core of unified text+pixel
transformers.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py``, never by the product path. It shares no code with the
CUDA path.

What it computes, and where the pages define it (sources are named by page title and
section):

* q/k RMSNorm, per token and head over head_dim -- "hidream-o1-p100a" model card, "What
  this model is" (the language model has "q/k RMSNorm"); "HiDream-O1-Image" summary
  (genai-atlas), "How it works" (RMSNorm in the decoder stack).
* Interleaved 3-axis mRoPE, sections [24, 20, 20], theta 5e6 -- model card, "What this
  model is". Rotation convention: the half-split feature layout
  [cos(n t0), cos(n t1), ..., sin(n t0), sin(n t1), ...] of the 1D RoPE definition in
  "HunyuanImage 3.0 Technical Report" (paper-graph-ui summary), section 3.4, "Generalized
  2D Rotary Position Embedding (RoPE)".
* The mask: HiDream -- model card, "What this model is" (sequence layout; text tokens
  causal, generation tokens see everything) and the genai-atlas summary, "How it works"
  (condition and text tokens causally masked; generation tokens attend to everything,
  including the condition tokens). HunyuanImage 3.0 Generalized Causal Attention --
  paper-graph-ui summary, section 3.4, "The core rule" (text tokens see all previous
  tokens; image tokens see all previous tokens and all tokens of their own image
  segment); bud-325 summary, "Key claims".
* GQA 32 query heads over 8 KV heads, head_dim 128 -- model card, "What this model is".

Readings where the pages are silent (each is a stated choice, not a page fact):
  softmax scale 1/sqrt(head_dim); RMSNorm eps inside the square root and a multiplicative
  weight shared by all heads; RMSNorm before RoPE; query head h uses KV head
  h // (Hq / Hkv); rotation pairs (k, k + D/2); "interleaved [24, 20, 20]" assigns
  frequency k to axis h when k % 3 == 1 and k < 3 * 20, to axis w when k % 3 == 2 and
  k < 3 * 20, and to axis t otherwise (24 slots).
  The exact interleave ORDER is parity-unpinned by the pages: they fix the section
  sizes, the 1D reduction and norm preservation, which every order satisfies.
"""
from __future__ import annotations

from typing import Iterable, List, Sequence, Tuple

import numpy as np

CAUSAL, FULL_SEQUENCE, FULL_IN_SEGMENT, GEN_IMAGE = 0, 1, 2, 3
TILE_SKIP, TILE_PARTIAL, TILE_FULL = 0, 1, 2


def bf16_to_f64(t) -> np.ndarray:
    """Exact widening of a bf16 (torch) or float array to fp64."""
    if hasattr(t, "detach"):
        t = t.detach().to("cpu").float().numpy()
    return np.asarray(t, dtype=np.float64)


# ---------------------------------------------------------------------------------------
# q/k RMSNorm ("hidream-o1-p100a" model card, "What this model is": "q/k RMSNorm")
# ---------------------------------------------------------------------------------------
def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2 over the last axis) + eps) * w, in fp64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


# ---------------------------------------------------------------------------------------
# mRoPE (model card "What this model is": 3-axis interleaved mRoPE [24,20,20], theta 5e6;
# rotation layout from the 1D RoPE definition in HunyuanImage 3.0 section 3.4)
# ---------------------------------------------------------------------------------------
def mrope_inv_freq(theta: float, head_dim: int) -> np.ndarray:
    """Frequency k of the D/2 rotation pairs: theta ** (-2k / D)."""
    k = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * k / head_dim)


ROPE_MROPE_INTERLEAVED, ROPE_2D_ALTERNATING, ROPE_2D_HALVES = 0, 1, 2
AXIS_T, AXIS_H, AXIS_W = 0, 1, 2  # position columns; in 2D layouts y = H (row), x = W (column)


def mrope_axis_of_frequency(head_dim: int, sections: Sequence[int], layout: int = ROPE_MROPE_INTERLEAVED) -> np.ndarray:
    """Axis (0 = t, 1 = h, 2 = w) that drives each of the D/2 frequencies.

    ROPE_MROPE_INTERLEAVED (model card, "3-axis interleaved mRoPE [24,20,20]"): the axes take
      turns t, h, w over the frequency index while h and w still have slots (k < 3 * s_h and
      k < 3 * s_w); all remaining frequencies belong to t.
    The HunyuanImage 3.0 Generalized 2D RoPE (section 3.4) for a 2D position (x, y), x the
    column (w) and y the row (h); its two sentences disagree, so both readings exist:
      ROPE_2D_ALTERNATING: the printed embedding [cos(x t0), cos(y t1), ...] -- frequency k is
        driven by x when k is even and by y when k is odd;
      ROPE_2D_HALVES: "the first half of the frequency spectrum encodes x, the second half y"
        -- frequencies k < D/4 by x, the rest by y.
    """
    half = head_dim // 2
    axis = np.zeros(half, dtype=np.int64)
    if layout == ROPE_2D_ALTERNATING:
        for k in range(half):
            axis[k] = AXIS_W if k % 2 == 0 else AXIS_H
        return axis
    if layout == ROPE_2D_HALVES:
        for k in range(half):
            axis[k] = AXIS_W if k < half // 2 else AXIS_H
        return axis
    s_t, s_h, s_w = (int(s) for s in sections)
    if s_t + s_h + s_w != half:
        raise ValueError("mRoPE sections must sum to head_dim / 2")
    for k in range(half):
        if k % 3 == 1 and k < 3 * s_h:
            axis[k] = AXIS_H
        elif k % 3 == 2 and k < 3 * s_w:
            axis[k] = AXIS_W
    return axis


def mrope_angles(pos: np.ndarray, theta: float, head_dim: int, sections: Sequence[int],
                 layout: int = ROPE_MROPE_INTERLEAVED) -> np.ndarray:
    """phi[n, k] = pos[n, axis(k)] * inv_freq[k], fp64, shape [N, D/2]."""
    pos = np.asarray(pos, dtype=np.float64).reshape(-1, 3)
    axis = mrope_axis_of_frequency(head_dim, sections, layout)
    inv = mrope_inv_freq(theta, head_dim)
    return pos[:, axis] * inv[None, :]


def rope_rotate_half(x: np.ndarray, phi: np.ndarray) -> np.ndarray:
    """Rotate pairs (k, k + D/2) of x [N, H, D] by phi [N, D/2]:
    y_k = x_k cos(phi_k) - x_{k+D/2} sin(phi_k); y_{k+D/2} = x_{k+D/2} cos(phi_k) + x_k sin(phi_k).
    """
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    c = np.cos(phi)[:, None, :]
    s = np.sin(phi)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def prologue(q, k, pos, wq, wk, theta: float = 5.0e6, sections=(24, 20, 20), eps: float = 1e-6,
             layout: int = ROPE_MROPE_INTERLEAVED):
    """q' = rope(rms(q) * wq), k' = rope(rms(k) * wk), fp64. q [N,Hq,D], k [N,Hkv,D]."""
    q = bf16_to_f64(q)
    k = bf16_to_f64(k)
    D = q.shape[-1]
    phi = mrope_angles(pos, theta, D, sections, layout)
    qn = rms_norm(q, bf16_to_f64(wq), eps)
    kn = rms_norm(k, bf16_to_f64(wk), eps)
    return rope_rotate_half(qn, phi), rope_rotate_half(kn, phi)


# ---------------------------------------------------------------------------------------
# The mask, built densely from the segment rules (never through per-row key limits)
# ---------------------------------------------------------------------------------------
def dense_mask(segments: Iterable[Tuple[int, int, int]], length: int) -> np.ndarray:
    """bool [L, L]; M[i, j] is True when query token i may attend to key token j.

    causal row i (HiDream text/condition tokens; Hunyuan text tokens): j <= i.
    full_sequence row i (HiDream generation tokens): every j.
    full_in_segment row i (Hunyuan image tokens): j <= i, or j in the same segment as i.
    gen_image row i (a Hunyuan Gen Image in a multi-Gen-Image training sequence): as
      full_in_segment; in addition no row of a LATER segment may see a key of a gen_image
      segment (the "hole" of "HunyuanImage 3.0 Technical Report", paper-graph-ui summary,
      section 3.4, "The multi-generation training complication", Figure 4(b)).
    """
    seg_id = np.full(length, -1, dtype=np.int64)
    kind = np.full(length, -1, dtype=np.int64)
    for n, (start, seg_len, seg_kind) in enumerate(segments):
        seg_id[start : start + seg_len] = n
        kind[start : start + seg_len] = seg_kind
    if length and (seg_id < 0).any():
        raise ValueError("segments do not cover the sequence")
    i = np.arange(length)[:, None]
    j = np.arange(length)[None, :]
    earlier_or_self = j <= i
    same_segment = seg_id[:, None] == seg_id[None, :]
    row_kind = kind[:, None]
    base = (
        ((row_kind == CAUSAL) & earlier_or_self)
        | (row_kind == FULL_SEQUENCE)
        | (((row_kind == FULL_IN_SEGMENT) | (row_kind == GEN_IMAGE)) & (earlier_or_self | same_segment))
    )
    hole = (kind[None, :] == GEN_IMAGE) & (seg_id[None, :] < seg_id[:, None])
    return base & ~hole


def unmasked_pairs(segments, length: int) -> int:
    """Number of visible (query, key) pairs of one batch element."""
    return int(dense_mask(segments, length).sum())


def tile_classes(mask: np.ndarray, bm: int, bn: int) -> np.ndarray:
    """Class of each (bm-token query block, bn-key block) tile from the dense mask.

    Key positions past the end of the sequence count as masked, so a ragged last key block
    is never FULL. FULL: every (row, key) of the nominal tile is visible; SKIP: none is;
    PARTIAL otherwise. uint8 [ceil(L / bm), ceil(L / bn)].
    """
    L = mask.shape[0]
    nqb, nkb = -(-L // bm), -(-L // bn)
    out = np.zeros((nqb, nkb), dtype=np.uint8)
    for qb in range(nqb):
        r0, r1 = qb * bm, min(L, qb * bm + bm)
        for kb in range(nkb):
            c0, c1 = kb * bn, min(L, kb * bn + bn)
            vis = int(mask[r0:r1, c0:c1].sum())
            if vis == 0:
                out[qb, kb] = TILE_SKIP
            elif vis == (r1 - r0) * bn:
                out[qb, kb] = TILE_FULL
            else:
                out[qb, kb] = TILE_PARTIAL
    return out


# ---------------------------------------------------------------------------------------
# Masked softmax attention with GQA ("What this model is": GQA 32/8, head 128)
# ---------------------------------------------------------------------------------------
def masked_gqa_attention(qp, kp, v, mask, scale=None, row_block: int = 1024) -> np.ndarray:
    """O[i, h] = sum_j softmax_j(q_{i,h} . k_{j,h//G} * scale | mask[i]) v_{j,h//G}, fp64.

    qp [L, Hq, D], kp and v [L, Hkv, D], mask bool [L, L]; G = Hq / Hkv.
    """
    qp = np.asarray(qp, dtype=np.float64)
    kp = np.asarray(kp, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, Hq, D = qp.shape
    Hkv = kp.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((L, Hq, D), dtype=np.float64)
    for h in range(Hq):
        kv = h // G
        kh, vh = kp[:, kv, :], v[:, kv, :]
        for r0 in range(0, L, row_block):
            r1 = min(L, r0 + row_block)
            s = (qp[r0:r1, h, :] @ kh.T) * scale
            s = np.where(mask[r0:r1], s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            out[r0:r1, h, :] = (p @ vh) / p.sum(axis=1, keepdims=True)
    return out


def _batch_segments(segs, cu_segs, b) -> List[Tuple[int, int, int]]:
    return [tuple(int(x) for x in segs[n]) for n in range(int(cu_segs[b]), int(cu_segs[b + 1]))]


def forward(q, k, v, pos, wq, wk, cu_seqlens, segs, cu_segs, theta=5.0e6, sections=(24, 20, 20),
            eps=1e-6, scale=None):
    """Whole path for packed varlen inputs: prologue, then masked GQA attention per batch
    element. Returns (O, q', k'), all fp64, O [T, Hq, D]."""
    qp, kp = prologue(q, k, pos, wq, wk, theta, sections, eps)
    vv = bf16_to_f64(v)
    out = np.zeros_like(qp)
    for b in range(len(cu_seqlens) - 1):
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        if t1 == t0:
            continue
        mask = dense_mask(_batch_segments(segs, cu_segs, b), t1 - t0)
        out[t0:t1] = masked_gqa_attention(qp[t0:t1], kp[t0:t1], vv[t0:t1], mask, scale)
    return out, qp, kp


def attention_rows(q, k, v, pos, wq, wk, cu_seqlens, segs, cu_segs, tokens: Sequence[int],
                   theta=5.0e6, sections=(24, 20, 20), eps=1e-6, scale=None) -> np.ndarray:
    """O for selected packed tokens only (all query heads): fp64 [len(tokens), Hq, D].

    For sampled checks at full size: per batch element it builds the prologue of all keys
    and the dense-mask rows of the selected tokens, then the same masked softmax as
    ``masked_gqa_attention`` one row at a time.
    """
    tokens = [int(t) for t in tokens]
    cu = [int(x) for x in cu_seqlens]
    pos = np.asarray(pos)
    Hq, D = q.shape[1], q.shape[2]
    res = np.zeros((len(tokens), Hq, D))
    for b in range(len(cu) - 1):
        t0, t1 = cu[b], cu[b + 1]
        picked = [(n, t) for n, t in enumerate(tokens) if t0 <= t < t1]
        if not picked:
            continue
        _, kp = prologue(q[t0:t0 + 1], k[t0:t1], pos[t0:t1], wq, wk, theta, sections, eps)
        vv = bf16_to_f64(v[t0:t1])
        mask = dense_mask(_batch_segments(segs, cu_segs, b), t1 - t0)
        G = Hq // kp.shape[1]
        sc = 1.0 / np.sqrt(D) if scale is None else scale
        for n, tok in picked:
            qp, _ = prologue(q[tok:tok + 1], k[tok:tok + 1], pos[tok:tok + 1], wq, wk, theta, sections, eps)
            row = mask[tok - t0]
            for h in range(Hq):
                s = (kp[:, h // G, :] @ qp[0, h, :]) * sc
                s = np.where(row, s, -np.inf)
                p = np.exp(s - s.max())
                res[n, h] = (p @ vv[:, h // G, :]) / p.sum()
    return res


# ---------------------------------------------------------------------------------------
# The attention layer around the core: QKV projection and output projection
# ("hidream-o1-p100a" model card, "What this model is": hidden size 4096, GQA 32/8, head
# 128, so the projection maps 4096 features to 32*128 + 2 * 8*128 = 6144 and back to 4096)
# ---------------------------------------------------------------------------------------
def qkv_projection(x, w_qkv, num_q_heads=32, num_kv_heads=8, head_dim=128):
    """x [T, hidden] @ w_qkv[N, hidden]^T split into q [T,Hq,D], k [T,Hkv,D], v [T,Hkv,D];
    output columns are ordered q heads, then k heads, then v heads."""
    y = bf16_to_f64(x) @ bf16_to_f64(w_qkv).T
    nq, nk = num_q_heads * head_dim, num_kv_heads * head_dim
    T = y.shape[0]
    return (y[:, :nq].reshape(T, num_q_heads, head_dim), y[:, nq:nq + nk].reshape(T, num_kv_heads, head_dim),
            y[:, nq + nk:nq + 2 * nk].reshape(T, num_kv_heads, head_dim))


def layer_forward(x, w_qkv, w_o, pos, wq, wk, cu_seqlens, segs, cu_segs, theta=5.0e6, sections=(24, 20, 20),
                  eps=1e-6, scale=None, layout=ROPE_MROPE_INTERLEAVED):
    """x -> QKV projection -> q/k RMSNorm + RoPE -> masked GQA attention -> output projection,
    fp64. Returns (y [T, hidden], attention output [T, Hq, D], q', k', v)."""
    q, k, v = qkv_projection(x, w_qkv)
    D = q.shape[-1]
    phi = mrope_angles(pos, theta, D, sections, layout)
    qp = rope_rotate_half(rms_norm(q, bf16_to_f64(wq), eps), phi)
    kp = rope_rotate_half(rms_norm(k, bf16_to_f64(wk), eps), phi)
    att = np.zeros_like(qp)
    for b in range(len(cu_seqlens) - 1):
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        if t1 > t0:
            mask = dense_mask(_batch_segments(segs, cu_segs, b), t1 - t0)
            att[t0:t1] = masked_gqa_attention(qp[t0:t1], kp[t0:t1], v[t0:t1], mask, scale)
    T = att.shape[0]
    y = att.reshape(T, -1) @ bf16_to_f64(w_o).T
    return y, att, qp, kp, v


def layer_rows(x, w_qkv, w_o, pos, wq, wk, cu_seqlens, segs, cu_segs, tokens: Sequence[int],
               theta=5.0e6, sections=(24, 20, 20), eps=1e-6, scale=None, layout=ROPE_MROPE_INTERLEAVED):
    """layer_forward for selected packed tokens only: (y rows [n, hidden], attention rows
    [n, Hq, D]). Keys and values of the whole batch element are projected; queries only for
    the selected tokens."""
    tokens = [int(t) for t in tokens]
    xf, wqkv = bf16_to_f64(x), bf16_to_f64(w_qkv)
    pos = np.asarray(pos)
    cu = [int(c) for c in cu_seqlens]
    att = np.zeros((len(tokens), 32, 128))
    for b in range(len(cu) - 1):
        t0, t1 = cu[b], cu[b + 1]
        picked = [(n, t) for n, t in enumerate(tokens) if t0 <= t < t1]
        if not picked:
            continue
        kv = xf[t0:t1] @ wqkv[4096:].T
        k = kv[:, :1024].reshape(-1, 8, 128)
        v = kv[:, 1024:].reshape(-1, 8, 128)
        phi_all = mrope_angles(pos[t0:t1], theta, 128, sections, layout)
        kp = rope_rotate_half(rms_norm(k, bf16_to_f64(wk), eps), phi_all)
        mask = dense_mask(_batch_segments(segs, cu_segs, b), t1 - t0)
        sc = 1.0 / np.sqrt(128) if scale is None else scale
        for n, tok in picked:
            q = (xf[tok] @ wqkv[:4096].T).reshape(1, 32, 128)
            qp = rope_rotate_half(rms_norm(q, bf16_to_f64(wq), eps),
                                  mrope_angles(pos[tok:tok + 1], theta, 128, sections, layout))
            row = mask[tok - t0]
            for h in range(32):
                sv = (kp[:, h // 4, :] @ qp[0, h, :]) * sc
                sv = np.where(row, sv, -np.inf)
                pr = np.exp(sv - sv.max())
                att[n, h] = (pr @ v[:, h // 4, :]) / pr.sum()
    y = att.reshape(len(tokens), -1) @ bf16_to_f64(w_o).T
    return y, att
