"""CPU oracle for the VGGT alternating-attention path, in float64.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The product path (the
CUDA library and its Python binding) never calls it and shares no code with it.

What it computes, per head, for bf16 inputs widened exactly to float64:

1. QK prologue: ``x_hat = RoPE2D(LayerNorm(x), pos)`` for every query and key
   head vector (64 dims).
   * LayerNorm over the head's 64 dims, centered, biased variance, eps 1e-5,
     no affine ("Norm: Layer Normalization" slide, ``(x - mu) / sigma``, in the
     VGGT paper-report slides; ``layer_norm_eps 1e-05`` in the VGGT-Omega
     config.json field table; vggt-jax README keeps "centered FP32 LayerNorm"
     and tunes the Q/K LayerNorm shapes).
   * 2D rotary embedding with base 100 (``rope_base: 100.0`` in the VGGT-Omega
     config.json field table). Dims 0-31 rotate by the row position, dims 32-63
     by the column position; within each 32-dim half, dim ``j`` pairs with dim
     ``j + 16`` and turns by ``pos * base**(-2j/32)`` -- the frequency schedule
     of the sinusoidal positional-encoding formula on the "Positional
     Encoding (4/6)" slide, ``pos / 10000^(2i/d)``.
2. Scores ``s_ij = q_hat_i . k_hat_j / sqrt(64)``, softmax over ``j``, and
   ``o_i = sum_j p_ij v_j`` ("Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V"
   and "softmax(x)_i = e^{x_i} / sum_j e^{x_j}" slides, Section V).
3. Which keys a query sees:
   * frame attention: the keys of its own frame ("Frame Attention" panel of the
     "Global + Frame Attention" architecture slide);
   * global attention: all ``S*T`` keys of the scene ("Global Attention" panel);
   * descriptor attention: all frames' compressed descriptors -- each frame's
     five special tokens unchanged plus one average per ``kd x kd`` cell of the
     patch grid (ceil mode), at the cell's mean position (FlashVGGT README,
     Overview: cross-attention between all image tokens and the per-frame
     descriptor set; Key Arguments: ``--kv_downfactor`` 4);
   * streaming descriptor attention: frames arrive in chunks of ``chunk``
     frames; every query of chunk ``c`` sees the descriptors of all frames of
     chunks ``0..c`` -- the cached descriptors of earlier chunks and its own
     chunk's (FlashVGGT README, Overview: a chunk-recursive mechanism that
     reuses cached descriptors from previous chunks; streaming inference with
     ``--chunksize``, default 10).

Options beyond the pages' default reading (both off by default):

* ``layout = (n_front, grid_h, grid_w, n_back)``: a frame of ``n_front``
  special tokens, a rectangular patch grid (vggt-jax README: its two-image
  benchmark feeds 350 x 518 images, a 25 x 37 grid) and ``n_back`` trailing
  tokens (the VGGT-Omega page appends its register tokens after the patches).
  Pooling copies front and trailing tokens and averages the grid's cells.
* ``ln = (q_gamma, q_beta, k_gamma, k_beta)``: a per-dim scale and shift after
  each QK LayerNorm, shared by the heads, applied before the rotation (a
  trained LayerNorm carries them; the pages give no values, so the default is
  the identity).

* several scenes per call (``attn_scenes``): each scene attended on its own
  (the vggt-jax README feeds ``[B, S, 3, H, W]`` image batches);
* token subsets (``attn_subset``): frames whose last ``n_skip_back`` tokens
  take no part in a call, plus ``n_extra`` sequence tokens after the frames
  that take part in global attention only -- the VGGT-Omega page's register
  tokens (after the patches, attending only at register_attention_block_
  indices [2, 6, 9, 14, 20]), storage tokens (4, shared by the sequence) and
  camera token (one for all frames). How the storage and camera tokens attend
  is not on the page; the reading here: as ordinary tokens of the global
  sequence, outside every frame.

Evaluating a subset of query rows is the same definition restricted to those
rows: every output row depends only on its own query and the key set, so
``rows=`` changes nothing about any row that is computed.
"""
from __future__ import annotations

import math

import numpy as np

N_SPECIAL = 5
LN_EPS = 1e-5
ROPE_BASE = 100.0
HEAD_DIM = 64

# --------------------------------------------------------------------------
# bf16 <-> float helpers (exact widening; correctly rounded narrowing)
# --------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of raw bf16 bit patterns (uint16) as float64."""
    b = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact value of raw bf16 bit patterns (uint16) as float32."""
    b = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, round-to-nearest-even, as uint16 bits.

    bf16 keeps the top 16 bits of the float32 pattern. Rounding to nearest
    with ties to even adds ``0x7FFF`` plus the lowest kept bit before
    truncating. NaN stays a quiet NaN with its sign.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    if nan.any():
        sign = ((u >> 16) & 0x8000).astype(np.uint16)
        rounded = np.where(nan, sign | np.uint16(0x7FC0), rounded)
    return rounded


# --------------------------------------------------------------------------
# Softmax, LayerNorm, RoPE
# --------------------------------------------------------------------------


def softmax(x: np.ndarray, axis: int = -1) -> np.ndarray:
    """``e^{x_i} / sum_j e^{x_j}`` along ``axis`` (Section V, softmax slide).

    The row maximum is subtracted first; that leaves every quotient unchanged
    and keeps ``exp`` finite.
    """
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - np.max(x, axis=axis, keepdims=True))
    return e / np.sum(e, axis=axis, keepdims=True)


def layer_norm(x: np.ndarray, eps: float = LN_EPS, gamma=None, beta=None) -> np.ndarray:
    """``(x - mu) / sqrt(var + eps)`` over the last axis; biased variance,
    computed from the centered values. With ``gamma`` / ``beta`` (vectors of
    the last axis' length) the result is then scaled by ``gamma`` and shifted
    by ``beta``, element by element; by default there is no scale or shift."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    c = x - mu
    var = (c * c).mean(axis=-1, keepdims=True)
    y = c / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)
    if beta is not None:
        y = y + np.asarray(beta, dtype=np.float64)
    return y


def rope_frequencies(base: float, d: int) -> np.ndarray:
    """``base ** (-2i / d)`` for ``i = 0 .. d/2 - 1``: the angular frequency of
    pair ``i`` in the sinusoidal formula ``PE(pos, 2i) = sin(pos / base^(2i/d))``
    (Positional Encoding (4/6) slide)."""
    i = np.arange(d // 2, dtype=np.float64)
    return base ** (-2.0 * i / d)


def sinusoidal_pe(pos: float, d: int, base: float) -> np.ndarray:
    """The slide's sinusoidal encoding: sin on even dims, cos on odd dims."""
    f = rope_frequencies(base, d)
    out = np.empty(d, dtype=np.float64)
    out[0::2] = np.sin(pos * f)
    out[1::2] = np.cos(pos * f)
    return out


def rope_2d(x: np.ndarray, pos: np.ndarray, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate head vectors ``x[..., 64]`` by their 2D positions ``pos[..., 2]``.

    Half ``a`` (a=0: dims 0-31, row position; a=1: dims 32-63, column
    position) is split into ``x1 = dims 0-15`` and ``x2 = dims 16-31`` of the
    half; pair ``(x1_j, x2_j)`` turns by ``theta_j = p_a * base**(-2j/32)``:
    ``x1' = x1 cos - x2 sin``, ``x2' = x2 cos + x1 sin``.
    ``pos`` broadcasts against ``x[..., 0]``.
    """
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    quarter = half // 2
    freq = rope_frequencies(base, half)  # quarter entries
    out = np.empty_like(x)
    for a in range(2):
        theta = pos[..., a][..., None] * freq  # [..., quarter]
        c, s = np.cos(theta), np.sin(theta)
        x1 = x[..., a * half: a * half + quarter]
        x2 = x[..., a * half + quarter: (a + 1) * half]
        out[..., a * half: a * half + quarter] = x1 * c - x2 * s
        out[..., a * half + quarter: (a + 1) * half] = x2 * c + x1 * s
    return out


def qk_prologue(x: np.ndarray, pos: np.ndarray, gamma=None, beta=None) -> np.ndarray:
    """LayerNorm (with the optional per-dim ``gamma`` / ``beta``, shared by all
    heads) then 2D RoPE for ``x[N, H, D]`` at ``pos[N, 2]``."""
    return rope_2d(layer_norm(x, gamma=gamma, beta=beta), np.asarray(pos)[:, None, :])


def _ln(ln, which: str):
    """``(gamma, beta)`` of the query (``which == "q"``) or key LayerNorm from
    ``ln = (q_gamma, q_beta, k_gamma, k_beta)`` (entries may be None), or no
    affine when ``ln`` is None."""
    if ln is None:
        return None, None
    return (ln[0], ln[1]) if which == "q" else (ln[2], ln[3])


# --------------------------------------------------------------------------
# Grid geometry and K/V descriptor pooling
# --------------------------------------------------------------------------


def grid_side(T: int) -> int:
    """Side ``g`` of the square patch grid when ``T = 5 + g*g``, else -1."""
    p = T - N_SPECIAL
    if p < 0:
        return -1
    g = math.isqrt(p)
    return g if g * g == p else -1


def frame_layout(T: int, layout=None):
    """The token layout of one frame as ``(n_front, grid_h, grid_w, n_back)``:
    ``n_front`` special tokens, then the ``grid_h x grid_w`` patch grid in
    row-major order, then ``n_back`` trailing tokens (the VGGT-Omega page puts
    its register tokens after each frame's patches). Without ``layout`` the
    frame is VGGT-1B's: 5 special tokens in front of a square grid."""
    if layout is None:
        g = grid_side(T)
        if g < 0:
            raise ValueError(f"T={T} is not 5 + g*g")
        return (N_SPECIAL, g, g, 0)
    nf, gh, gw, nb = (int(x) for x in layout)
    if min(nf, gh, gw, nb) < 0 or nf + gh * gw + nb != T:
        raise ValueError(f"layout {layout} does not describe T={T} tokens")
    return (nf, gh, gw, nb)


def pool_cells_rect(gh: int, gw: int, kd: int):
    """Ceil-mode ``kd x kd`` cells of a ``gh x gw`` grid, row-major.

    Each cell is a list of member patch indices ``r*gw + c`` in row-major
    order; edge cells keep only the members that lie inside the grid.
    """
    nch = -(-gh // kd) if gh > 0 else 0
    ncw = -(-gw // kd) if gw > 0 else 0
    cells = []
    for cr in range(nch):
        for cc in range(ncw):
            rows = range(cr * kd, min(cr * kd + kd, gh))
            cols = range(cc * kd, min(cc * kd + kd, gw))
            cells.append([r * gw + c for r in rows for c in cols])
    return cells


def pool_cells(g: int, kd: int):
    """The cells of a square ``g x g`` grid (``pool_cells_rect(g, g, kd)``)."""
    return pool_cells_rect(g, g, kd)


def pooled_tokens_per_frame(T: int, kd: int, layout=None) -> int:
    nf, gh, gw, nb = frame_layout(T, layout)
    return nf + len(pool_cells_rect(gh, gw, kd)) + nb


def _pooled_sources(T: int, kd: int, layout):
    """For every pooled token of a frame, in order, ``(sources, is_special)``:
    front specials and trailing tokens are their own single source and are
    copied; each cell lists its patches in row-major order."""
    nf, gh, gw, nb = frame_layout(T, layout)
    src = [([t], True) for t in range(nf)]
    src += [([nf + m for m in members], False) for members in pool_cells_rect(gh, gw, kd)]
    src += [([nf + gh * gw + t], True) for t in range(nb)]
    return src


def kv_pool(k: np.ndarray, v: np.ndarray, pos: np.ndarray, S: int, T: int, kd: int, layout=None):
    """Per-frame descriptors in float64: the special (front and trailing)
    tokens unchanged, and the mean of each ceil-mode ``kd x kd`` cell of the
    patch grid (K, V and position alike), ordered front specials, cells
    (row-major), trailing tokens. Inputs are ``[S*T, H, D]`` and ``[S*T, 2]``."""
    src = _pooled_sources(T, kd, layout)
    Tk = len(src)
    k = np.asarray(k, dtype=np.float64).reshape(S, T, *k.shape[1:])
    v = np.asarray(v, dtype=np.float64).reshape(S, T, *v.shape[1:])
    pos = np.asarray(pos, dtype=np.float64).reshape(S, T, 2)
    kp = np.empty((S, Tk) + k.shape[2:])
    vp = np.empty((S, Tk) + v.shape[2:])
    pp = np.empty((S, Tk, 2))
    for i, (members, _) in enumerate(src):
        idx = np.asarray(members)
        kp[:, i] = k[:, idx].mean(axis=1)
        vp[:, i] = v[:, idx].mean(axis=1)
        pp[:, i] = pos[:, idx].mean(axis=1)
    return (kp.reshape(S * Tk, *k.shape[2:]), vp.reshape(S * Tk, *v.shape[2:]),
            pp.reshape(S * Tk, 2))


def kv_pool_bf16_reference(k_bits, v_bits, pos, S: int, T: int, kd: int, layout=None):
    """The stored form of the pooled descriptors, bit for bit.

    For every cell and channel: float32 sum of the members in row-major order
    (each addition rounded to float32), divided in float32 by the member
    count, rounded to bf16 (nearest, ties to even). Positions: the same float32
    sum and division, kept in float32. Special tokens are copied unchanged.
    Returns ``(k_bits, v_bits, pos_f32)``.
    """
    src = _pooled_sources(T, kd, layout)
    Tk = len(src)
    k32 = bf16_bits_to_f32(k_bits).reshape(S, T, -1)
    v32 = bf16_bits_to_f32(v_bits).reshape(S, T, -1)
    p32 = np.asarray(pos, dtype=np.float32).reshape(S, T, 2)
    kb = np.asarray(k_bits).view(np.uint16).reshape(S, T, -1)
    vb = np.asarray(v_bits).view(np.uint16).reshape(S, T, -1)
    ko = np.empty((S, Tk, kb.shape[2]), dtype=np.uint16)
    vo = np.empty((S, Tk, vb.shape[2]), dtype=np.uint16)
    po = np.empty((S, Tk, 2), dtype=np.float32)
    for i, (members, special) in enumerate(src):
        if special:  # copied as it is (a one-member cell is still summed: -0 becomes +0)
            ko[:, i] = kb[:, members[0]]
            vo[:, i] = vb[:, members[0]]
            po[:, i] = p32[:, members[0]]
            continue
        ak = np.zeros((S, k32.shape[2]), dtype=np.float32)
        av = np.zeros((S, v32.shape[2]), dtype=np.float32)
        ap = np.zeros((S, 2), dtype=np.float32)
        for t in members:  # row-major member order
            ak = ak + k32[:, t]
            av = av + v32[:, t]
            ap = ap + p32[:, t]
        n = np.float32(len(members))
        ko[:, i] = f32_to_bf16_bits(ak / n)
        vo[:, i] = f32_to_bf16_bits(av / n)
        po[:, i] = ap / n
    return ko.reshape(S * Tk, -1), vo.reshape(S * Tk, -1), po.reshape(S * Tk, 2)


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

ROW_GROUP = 1024  # rows evaluated together; rows are independent


def _attend(qh: np.ndarray, kh: np.ndarray, v: np.ndarray) -> np.ndarray:
    """``softmax(qh kh^T / sqrt(D)) v`` for one head: qh [n,D], kh [m,D], v [m,Dv]."""
    scores = (qh @ kh.T) / math.sqrt(qh.shape[-1])
    return softmax(scores, axis=-1) @ v


def cross_attention(q_hat, k_hat, v, rows=None) -> np.ndarray:
    """Every selected query row attends to every key, each head on its own.

    ``q_hat [Nq,H,D]``, ``k_hat [Nk,H,D]`` already through the prologue;
    ``v [Nk,H,D]``. Returns ``[len(rows), H, D]``.
    """
    rows = np.arange(q_hat.shape[0]) if rows is None else np.asarray(rows)
    H = q_hat.shape[1]
    out = np.empty((rows.size, H, v.shape[2]))
    for h in range(H):
        kh, vh = k_hat[:, h], v[:, h]
        for s0 in range(0, rows.size, ROW_GROUP):
            r = rows[s0:s0 + ROW_GROUP]
            out[s0:s0 + ROW_GROUP, h] = _attend(q_hat[r, h], kh, vh)
    return out


def _rows(n: int, rows):
    return np.arange(n) if rows is None else np.asarray(rows)


def attn_global(q, k, v, pos, S: int, T: int, rows=None, ln=None) -> np.ndarray:
    """Global attention: all ``S*T`` tokens attend to all ``S*T`` tokens.
    ``ln = (q_gamma, q_beta, k_gamma, k_beta)`` gives the QK LayerNorms an
    affine (any entry may be None); by default they have none."""
    rows = _rows(S * T, rows)
    q_hat = qk_prologue(np.asarray(q)[rows], np.asarray(pos)[rows], *_ln(ln, "q"))
    k_hat = qk_prologue(k, pos, *_ln(ln, "k"))
    return cross_attention(q_hat, k_hat, np.asarray(v, dtype=np.float64))


def attn_frame(q, k, v, pos, S: int, T: int, rows=None, ln=None) -> np.ndarray:
    """Frame attention: each token attends to the ``T`` tokens of its frame
    (``ln`` as for ``attn_global``)."""
    rows = _rows(S * T, rows)
    q, k, pos = np.asarray(q), np.asarray(k), np.asarray(pos)
    v = np.asarray(v, dtype=np.float64)
    out = np.empty((rows.size, q.shape[1], v.shape[2]))
    frames = rows // T
    for s in np.unique(frames):
        sel = np.nonzero(frames == s)[0]
        lo, hi = s * T, (s + 1) * T
        q_hat = qk_prologue(q[rows[sel]], pos[rows[sel]], *_ln(ln, "q"))
        k_hat = qk_prologue(k[lo:hi], pos[lo:hi], *_ln(ln, "k"))
        out[sel] = cross_attention(q_hat, k_hat, v[lo:hi])
    return out


def attn_descriptor(q, k, v, pos, S: int, T: int, kd: int, rows=None, layout=None,
                    ln=None) -> np.ndarray:
    """Descriptor attention: every query attends to all frames' pooled
    descriptors; the pooled keys go through the prologue at their cell-mean
    positions, pooled values are used as they are. ``layout`` is the frame
    layout of ``frame_layout``; ``ln`` as for ``attn_global``."""
    kp, vp, pp = kv_pool(k, v, pos, S, T, kd, layout)
    rows = _rows(S * T, rows)
    q_hat = qk_prologue(np.asarray(q)[rows], np.asarray(pos)[rows], *_ln(ln, "q"))
    k_hat = qk_prologue(kp, pp, *_ln(ln, "k"))
    return cross_attention(q_hat, k_hat, vp)


def attn_descriptor_stream(q, k, v, pos, S: int, T: int, kd: int, chunk: int, rows=None, layout=None,
                           ln=None) -> np.ndarray:
    """Streaming descriptor attention: a query of frame ``f`` sees the
    descriptors of frames ``0 .. min(S, (f // chunk + 1) * chunk) - 1``. The
    descriptors are the per-frame pooled tokens of ``attn_descriptor``; their
    keys go through the prologue at their cell-mean positions."""
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    kp, vp, pp = kv_pool(k, v, pos, S, T, kd, layout)
    k_hat = qk_prologue(kp, pp, *_ln(ln, "k"))
    tk = pooled_tokens_per_frame(T, kd, layout)
    rows = _rows(S * T, rows)
    out = np.empty((rows.size,) + np.asarray(q).shape[1:])
    chunk_of_row = (rows // T) // chunk
    for c in np.unique(chunk_of_row):
        sel = np.nonzero(chunk_of_row == c)[0]
        r = rows[sel]
        n_keys = min(S, (int(c) + 1) * chunk) * tk
        q_hat = qk_prologue(np.asarray(q)[r], np.asarray(pos)[r], *_ln(ln, "q"))
        out[sel] = cross_attention(q_hat, k_hat[:n_keys], vp[:n_keys])
    return out


def attn_scenes(kind: str, q, k, v, pos, B: int, S: int, T: int, kd: int = 1, rows=None, layout=None,
                ln=None) -> np.ndarray:
    """``B`` independent scenes in one batch (the pages' inputs are
    ``[B, S, 3, H, W]``): scene ``b`` is token rows ``[b*S*T, (b+1)*S*T)``, and
    every scene is attended on its own -- ``kind`` "global" or "descriptor"
    as ``attn_global`` / ``attn_descriptor`` of that scene's rows. Returns the
    outputs of the selected rows (all by default), in that order."""
    n_scene = S * T
    rows = _rows(B * n_scene, rows)
    q, k, v, pos = (np.asarray(x) for x in (q, k, v, pos))
    out = np.empty((rows.size,) + q.shape[1:])
    scene = rows // n_scene
    for b in np.unique(scene):
        sel = np.nonzero(scene == b)[0]
        lo, hi = b * n_scene, (b + 1) * n_scene
        local = rows[sel] - lo
        if kind == "global":
            out[sel] = attn_global(q[lo:hi], k[lo:hi], v[lo:hi], pos[lo:hi], S, T, rows=local, ln=ln)
        elif kind == "descriptor":
            out[sel] = attn_descriptor(q[lo:hi], k[lo:hi], v[lo:hi], pos[lo:hi], S, T, kd, rows=local,
                                       layout=layout, ln=ln)
        else:
            raise ValueError("kind must be 'global' or 'descriptor'")
    return out


def subset_rows(S: int, T: int, n_skip_back: int, n_extra: int) -> np.ndarray:
    """The token rows that take part in a subset call, in order: the first
    ``T - n_skip_back`` tokens of each of the ``S`` frames, then the
    ``n_extra`` sequence tokens that follow the frames (rows ``S*T ..``)."""
    keep = T - n_skip_back
    if not (0 <= n_skip_back <= T and n_extra >= 0):
        raise ValueError("need 0 <= n_skip_back <= T and n_extra >= 0")
    rows = [s * T + np.arange(keep) for s in range(S)] + [S * T + np.arange(n_extra)]
    return np.concatenate(rows).astype(np.int64)


def attn_subset(q, k, v, pos, S: int, T: int, n_skip_back: int, n_extra: int, kind: str,
                rows=None, ln=None) -> np.ndarray:
    """Attention over a subset of the tokens -- the VGGT-Omega layout, whose
    register tokens sit after each frame's patches and take part only in some
    blocks, and whose storage and camera tokens belong to the whole sequence
    (VGGT-Omega page: num_register_tokens, register_attention_block_indices,
    num_storage_tokens, camera_token).

    Tokens: ``S`` frames of ``T`` rows, then ``n_extra`` sequence rows. The
    last ``n_skip_back`` rows of every frame take no part (neither query nor
    key). ``kind == "frame"``: every kept row of frame ``s`` attends to the kept
    rows of frame ``s``; the sequence rows take no part. ``kind == "global"``:
    every kept row and every sequence row attends to all of them. Returns the
    outputs of the selected kept rows (``rows``: indices into the original
    token rows, all kept by default), in that order.
    """
    keep_rows = subset_rows(S, T, n_skip_back, n_extra if kind == "global" else 0)
    q, k, pos = np.asarray(q), np.asarray(k), np.asarray(pos)
    v = np.asarray(v, dtype=np.float64)
    if rows is None:
        rows = keep_rows
    rows = np.asarray(rows, dtype=np.int64)
    if not np.isin(rows, keep_rows).all():
        raise ValueError("rows must be rows that take part")
    if kind == "global":
        q_hat = qk_prologue(q[rows], pos[rows], *_ln(ln, "q"))
        k_hat = qk_prologue(k[keep_rows], pos[keep_rows], *_ln(ln, "k"))
        return cross_attention(q_hat, k_hat, v[keep_rows])
    if kind != "frame":
        raise ValueError("kind must be 'frame' or 'global'")
    keep = T - n_skip_back
    out = np.empty((rows.size, q.shape[1], v.shape[2]))
    frames = rows // T
    for s in np.unique(frames):
        sel = np.nonzero(frames == s)[0]
        kr = s * T + np.arange(keep)
        q_hat = qk_prologue(q[rows[sel]], pos[rows[sel]], *_ln(ln, "q"))
        k_hat = qk_prologue(k[kr], pos[kr], *_ln(ln, "k"))
        out[sel] = cross_attention(q_hat, k_hat, v[kr])
    return out
