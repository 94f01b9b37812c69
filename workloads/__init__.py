"""Seeded synthetic inputs for hybrid-masked attention over mixed text+pixel sequences.

This module is the only code shared by the fp64 oracle side (tests) and the CUDA side
(tests, bench). It holds descriptions of token sequences and seeded random tensors, and
none of the attention method's arithmetic: it never builds a mask, a row limit, a norm,
a rotation or a softmax.

Sequence layouts follow the pages:
  * HiDream-O1 ("hidream-o1-p100a" model card, "What this model is"): one packed
    sequence ``[chat text ... <|boi|><|tms|>] + [target 32x32-px patches] + [reference
    patches]``; text and condition tokens are causal, generation tokens see everything.
  * HunyuanImage 3.0 (paper-graph-ui summary, section 3.4 "Generalized Causal
    Attention"): text segments causal; each image segment sees everything before it and
    all of its own segment.

Positions are 3-axis (t, h, w) integers. They are inputs to both sides, so parity never
depends on how they are chosen; the convention is:
  * HiDream text token at local index i: (i, i, i); a patch segment whose first token sits
    at local index T0: (T0, row, col); the reference (condition) patches of an edit use
    (T0 + 1, row, col).
  * Hunyuan: a running counter n; a text token gets (n, n, n) and n += 1 (text on the
    diagonal, as in the "Generalized 2D RoPE" passage of section 3.4); an image segment
    that starts at counter n gets (n, n + row, n + col) and then n += max(rows, cols).

Random values: Q, K, V ~ N(0, 1) rounded to bf16, q/k norm weights 1 + N(0, 0.1) rounded
to bf16, drawn from ``torch.Generator().manual_seed(seed)`` on the CPU in the order
Q, K, V, wq, wk.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

# Segment kinds, numbered as in include/hgx_attn.h (hgx_seg_kind).
CAUSAL = 0
FULL_SEQUENCE = 1
FULL_IN_SEGMENT = 2
GEN_IMAGE = 3
KIND_NAMES = {CAUSAL: "causal", FULL_SEQUENCE: "full_sequence", FULL_IN_SEGMENT: "full_in_segment",
              GEN_IMAGE: "gen_image"}

NUM_Q_HEADS = 32
NUM_KV_HEADS = 8
HEAD_DIM = 128
ROPE_THETA = 5.0e6
MROPE_SECTION = (24, 20, 20)
RMS_EPS = 1e-6


@dataclasses.dataclass(frozen=True)
class Segment:
    """A run of tokens of one batch element: local start, length, kind, and for image
    segments the patch grid (rows, cols) used to give positions."""

    start: int
    length: int
    kind: int
    grid: Optional[Tuple[int, int]] = None


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batches: Tuple[Tuple[Segment, ...], ...]
    seed: int
    style: str  # "hidream" or "hunyuan": which position convention applies

    @property
    def lengths(self) -> List[int]:
        return [sum(s.length for s in b) for b in self.batches]

    @property
    def total_tokens(self) -> int:
        return sum(self.lengths)


def _segments(spec: Sequence[Tuple[int, int, Optional[Tuple[int, int]]]]) -> Tuple[Segment, ...]:
    out, start = [], 0
    for length, kind, grid in spec:
        out.append(Segment(start, length, kind, grid))
        start += length
    return tuple(out)


def _hidream_t2i(n_text: int, side: int):
    # n_text chat tokens + <|tms|> (causal), then side x side generation patches.
    return _segments([(n_text + 1, CAUSAL, None), (side * side, FULL_SEQUENCE, (side, side))])


CONFIGS: Tuple[Workload, ...] = (
    # 0: tiny HiDream-style mask: 64 text + <|tms|> causal, 256 patches (512^2 at 32 px).
    Workload("hidream_tiny_321", (_hidream_t2i(64, 16),), seed=0, style="hidream"),
    # 1: HiDream 1024^2 text-to-image step, CFG pair packed varlen (128 / 16 text tokens).
    Workload("hidream_t2i_1024_cfg", (_hidream_t2i(128, 32), _hidream_t2i(16, 32)), seed=1, style="hidream"),
    # 2: HiDream 2048^2 text-to-image step, CFG batch of 2 (256 text tokens each).
    Workload("hidream_t2i_2048_cfg", (_hidream_t2i(256, 64), _hidream_t2i(256, 64)), seed=2, style="hidream"),
    # 3: HiDream 2048^2 edit step: 257 causal, 4096 target patches (full sequence),
    #    4096 reference patches (causal).
    Workload(
        "hidream_edit_2048",
        (_segments([(257, CAUSAL, None), (4096, FULL_SEQUENCE, (64, 64)), (4096, CAUSAL, (64, 64))]),),
        seed=3,
        style="hidream",
    ),
    # 4: HunyuanImage-style Generalized Causal mask with two 64x64 image segments.
    Workload(
        "hunyuan_gca_9088",
        (
            _segments(
                [
                    (512, CAUSAL, None),
                    (4096, FULL_IN_SEGMENT, (64, 64)),
                    (256, CAUSAL, None),
                    (4096, FULL_IN_SEGMENT, (64, 64)),
                    (128, CAUSAL, None),
                ]
            ),
        ),
        seed=4,
        style="hunyuan",
    ),
)

# Beyond the five: the HunyuanImage 3.0 multi-Gen-Image TRAINING mask on the same layout as
# hunyuan_gca_9088, both images being Gen Images (each hidden from every later token).
EXTRA: Tuple[Workload, ...] = (
    Workload(
        "hunyuan_multigen_9088",
        (
            _segments(
                [
                    (512, CAUSAL, None),
                    (4096, GEN_IMAGE, (64, 64)),
                    (256, CAUSAL, None),
                    (4096, GEN_IMAGE, (64, 64)),
                    (128, CAUSAL, None),
                ]
            ),
        ),
        seed=5,
        style="hunyuan",
    ),
)

CONFIG_BY_NAME = {w.name: w for w in CONFIGS + EXTRA}


def config(i: int) -> Workload:
    return CONFIGS[i]


def cu_seqlens(w: Workload) -> np.ndarray:
    """int32 [batch + 1]: packed-varlen token offsets."""
    return np.concatenate([[0], np.cumsum(w.lengths)]).astype(np.int32)


def flat_segments(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """(segs int32 [S, 3] rows of (start, len, kind) local to their batch element,
    cu_segs int32 [batch + 1])."""
    rows, cu = [], [0]
    for b in w.batches:
        for s in b:
            rows.append((s.start, s.length, s.kind))
        cu.append(len(rows))
    segs = np.array(rows, dtype=np.int32).reshape(-1, 3)
    return segs, np.array(cu, dtype=np.int32)


def positions(w: Workload) -> np.ndarray:
    """int32 [T, 3] (t, h, w) positions per packed token (convention in the module doc)."""
    out = []
    for batch in w.batches:
        n = 0  # hunyuan running counter
        img_index = 0
        for s in batch:
            if s.grid is None:
                if w.style == "hidream":
                    idx = np.arange(s.start, s.start + s.length)
                    out.append(np.stack([idx, idx, idx], axis=1))
                else:
                    idx = np.arange(n, n + s.length)
                    out.append(np.stack([idx, idx, idx], axis=1))
                    n += s.length
            else:
                rows, cols = s.grid
                assert rows * cols == s.length
                r, c = np.divmod(np.arange(s.length), cols)
                if w.style == "hidream":
                    # target patches at T0 = their first index; reference patches at T0 + 1
                    t0 = s.start if img_index == 0 else _first_image_start(batch) + 1
                    out.append(np.stack([np.full(s.length, t0), r, c], axis=1))
                else:
                    out.append(np.stack([np.full(s.length, n), n + r, n + c], axis=1))
                    n += max(rows, cols)
                img_index += 1
    if not out:
        return np.zeros((0, 3), dtype=np.int32)
    return np.concatenate(out).astype(np.int32)


def _first_image_start(batch: Sequence[Segment]) -> int:
    for s in batch:
        if s.grid is not None:
            return s.start
    raise ValueError("no image segment")


def tensors(w: Workload, device: str = "cpu"):
    """Seeded bf16 inputs: dict(q [T,32,128], k [T,8,128], v [T,8,128], wq [128], wk [128])."""
    g = torch.Generator().manual_seed(w.seed)
    T = w.total_tokens
    q = torch.randn(T, NUM_Q_HEADS, HEAD_DIM, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(T, NUM_KV_HEADS, HEAD_DIM, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(T, NUM_KV_HEADS, HEAD_DIM, generator=g, dtype=torch.float32).to(torch.bfloat16)
    wq = (1.0 + 0.1 * torch.randn(HEAD_DIM, generator=g, dtype=torch.float32)).to(torch.bfloat16)
    wk = (1.0 + 0.1 * torch.randn(HEAD_DIM, generator=g, dtype=torch.float32)).to(torch.bfloat16)
    out = dict(q=q, k=k, v=v, wq=wq, wk=wk)
    if device != "cpu":
        out = {n: t.to(device) for n, t in out.items()}
    return out


def random_workload(seed: int, max_batch: int = 3, max_len: int = 700, allow_empty: bool = False,
                    kinds: Sequence[int] = (CAUSAL, FULL_SEQUENCE, FULL_IN_SEGMENT)) -> Workload:
    """A seeded random segment layout (the given kinds, ragged lengths); every non-causal
    segment gets a (1, len) grid so that positions stay integral."""
    rng = np.random.default_rng(seed)
    batches = []
    for _ in range(int(rng.integers(1, max_batch + 1))):
        n_seg = int(rng.integers(0 if allow_empty else 1, 6))
        spec = []
        for _ in range(n_seg):
            length = int(rng.integers(1, max(2, max_len // max(n_seg, 1))))
            kind = int(kinds[int(rng.integers(0, len(kinds)))])
            grid = None if kind == CAUSAL else (1, length)
            spec.append((length, kind, grid))
        batches.append(_segments(spec))
    return Workload(f"random_{seed}", tuple(batches), seed=seed, style="hunyuan")


def custom(name: str, batches: Sequence[Sequence[Tuple[int, int]]], seed: int = 0) -> Workload:
    """Build a workload from [(length, kind), ...] per batch element (positions: text-style
    diagonal for causal segments, one-row grids for the others)."""
    out = []
    for b in batches:
        out.append(_segments([(n, kd, None if kd == CAUSAL else (1, n)) for n, kd in b]))
    return Workload(name, tuple(out), seed=seed, style="hunyuan")


def layer_tensors(w: Workload, device: str = "cpu"):
    """Seeded bf16 inputs of the whole attention layer: dict(x [T, 4096] ~ N(0, 1),
    w_qkv [6144, 4096] and w_o [4096, 4096] ~ N(0, 1/4096), wq, wk = 1 + N(0, 0.1)), drawn
    from torch.Generator().manual_seed(seed + 1000) in that order."""
    g = torch.Generator().manual_seed(w.seed + 1000)
    T = w.total_tokens
    hidden = NUM_Q_HEADS * HEAD_DIM
    nqkv = hidden + 2 * NUM_KV_HEADS * HEAD_DIM
    x = torch.randn(T, hidden, generator=g, dtype=torch.float32).to(torch.bfloat16)
    w_qkv = (torch.randn(nqkv, hidden, generator=g, dtype=torch.float32) / hidden ** 0.5).to(torch.bfloat16)
    w_o = (torch.randn(hidden, hidden, generator=g, dtype=torch.float32) / hidden ** 0.5).to(torch.bfloat16)
    wq = (1.0 + 0.1 * torch.randn(HEAD_DIM, generator=g, dtype=torch.float32)).to(torch.bfloat16)
    wk = (1.0 + 0.1 * torch.randn(HEAD_DIM, generator=g, dtype=torch.float32)).to(torch.bfloat16)
    out = dict(x=x, w_qkv=w_qkv, w_o=w_o, wq=wq, wk=wk)
    if device != "cpu":
        out = {n: t.to(device) for n, t in out.items()}
    return out
