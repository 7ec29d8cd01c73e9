"""Seeded synthetic inputs for the VGGT attention path.

This module only *draws* inputs; it holds none of the attention arithmetic.
Both the CUDA path and the CPU oracle consume the same tensors built here.

Token layout (VGGT aggregator, one scene, B = 1):

* ``S`` frames, each with ``T = 5 + g*g`` tokens: one camera token and four
  register tokens (the five "special" tokens), then the ``g x g`` patch grid in
  row-major order (vggt-jax README, attention benchmark table: ``[2,930,16,64]``
  is 2 frames of 25*37 patches + 5 specials).
* ``q``, ``k``, ``v`` are ``[S*T, H, D]`` bf16, token-major with heads
  interleaved, as in the ``[B, N, H, D]`` shapes of that table.
* ``pos`` is ``[S*T, 2]`` fp32 ``(row, col)``: special tokens at ``(0, 0)``,
  patch ``(r, c)`` at ``(r + 1, c + 1)``.

Values are i.i.d. N(0, 1) drawn in fp32 from a CPU ``torch.Generator`` and
rounded to bf16 (round-to-nearest-even, torch's own conversion).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

N_SPECIAL = 5
HEADS = 16
HEAD_DIM = 64


@dataclass(frozen=True)
class Workload:
    """One attention workload: kind, frame count, grid side and pooling factor."""

    name: str
    # "global" | "frame" | "descriptor" | "stream" (descriptors, chunk by
    # chunk) | "subset_global" | "subset_frame" (a frame's last `skip` tokens
    # take no part; `n_extra` sequence tokens follow the frames) |
    # "global_f32" | "frame_f32" (the fp32 mode) | "global_batch" (B scenes,
    # each on its own)
    kind: str
    S: int
    g: int
    kv_down: int = 1
    H: int = HEADS
    D: int = HEAD_DIM
    chunk: int = 0  # frames per chunk ("stream")
    n_front: int = N_SPECIAL  # special tokens before the grid
    n_back: int = 0           # tokens after the grid
    skip: int = 0             # trailing tokens per frame left out ("subset_*")
    n_extra: int = 0          # sequence tokens after the frames ("subset_*")
    B: int = 1                # scenes per call ("global_batch")
    terms: int = 2            # bf16 terms per fp32 operand ("*_f32")
    affine: int = -1          # seed of a large QK LayerNorm affine (ln_affine_large), -1: none

    @property
    def T(self) -> int:
        return self.n_front + self.g * self.g + self.n_back

    @property
    def layout(self):
        return (self.n_front, self.g, self.g, self.n_back)

    @property
    def rows(self) -> int:
        """Token rows of the input tensors."""
        return self.B * self.S * self.T + self.n_extra

    @property
    def n_q(self) -> int:
        """Query rows that take part."""
        if self.kind == "subset_global":
            return self.S * (self.T - self.skip) + self.n_extra
        if self.kind == "subset_frame":
            return self.S * (self.T - self.skip)
        return self.B * self.S * self.T

    @property
    def T_k(self) -> int:
        if self.kind in ("subset_global", "subset_frame"):
            return self.T - self.skip
        if self.kind not in ("descriptor", "stream"):
            return self.T
        nc = -(-self.g // self.kv_down) if self.g > 0 else 0
        return N_SPECIAL + nc * nc

    @property
    def n_k(self) -> int:
        if self.kind == "subset_global":
            return self.n_q
        if self.kind == "global_batch":
            return self.S * self.T  # keys per scene
        return self.S * self.T_k

    def flops(self) -> float:
        """Algorithmic attention FLOPs: 4 * H * D per (query, key) pair."""
        if self.kind in ("frame", "frame_f32"):
            pairs = self.S * self.T * self.T
        elif self.kind == "subset_frame":
            pairs = self.S * self.T_k * self.T_k
        elif self.kind == "global_batch":
            pairs = self.B * (self.S * self.T) ** 2
        elif self.kind == "stream":
            # chunk c's queries see the descriptors of chunks 0..c
            pairs = sum(min(self.chunk, self.S - f0) * self.T * min(self.S, f0 + self.chunk) * self.T_k
                        for f0 in range(0, self.S, self.chunk))
        else:
            pairs = self.n_q * self.n_k
        return 4.0 * self.H * self.D * pairs


# The five workloads of the pages' shapes (two 224^2 frames; eight 518^2 frames
# at patch 14; nine 1024^2 frames at patch 16; 200 518^2 frames pooled 4x4).
WORKLOADS = {
    w.name: w
    for w in (
        Workload("global_s2_g16", "global", S=2, g=16),
        Workload("frame_s8_g37", "frame", S=8, g=37),
        Workload("global_s8_g37", "global", S=8, g=37),
        Workload("global_s9_g64", "global", S=9, g=64),
        Workload("descriptor_s200_g37_kd4", "descriptor", S=200, g=37, kv_down=4),
    )
}

# Smaller cases for hardware-counter captures, whose inputs still exceed the
# 126 MB L2: dense global attention over 24 606 tokens (151 MB of q, k, v) for
# the attention kernel and the prologue, and 40 frames of the descriptor
# workload (k and v: 225 MB) for the pooling kernel.
PROFILE_WORKLOADS = {w.name: w for w in (
    Workload("global_s6_g64", "global", S=6, g=64),
    Workload("descriptor_s40_g37_kd4", "descriptor", S=40, g=37, kv_down=4),
    Workload("global_s6_g64_f32", "global_f32", S=6, g=64),
    Workload("global_s6_g64_f32x3", "global_f32", S=6, g=64, terms=3),
)}

# The descriptor workload streamed in chunks of 10 frames (FlashVGGTStream's
# default chunk size), for measurement.
STREAM_WORKLOADS = {w.name: w for w in (
    Workload("stream_s200_g37_kd4_c10", "stream", S=200, g=37, kv_down=4, chunk=10),
)}
# The VGGT-Omega layout at 512 px (patch 16: a 32 x 32 grid, 16 register
# tokens after the patches, 4 storage tokens + 1 camera token for the
# sequence), 32 frames: global and frame attention of a block where the
# registers take no part.
SUBSET_WORKLOADS = {w.name: w for w in (
    Workload("omega_global_s32_g32", "subset_global", S=32, g=32, n_front=0, n_back=16, skip=16, n_extra=5),
    Workload("omega_frame_s32_g32", "subset_frame", S=32, g=32, n_front=0, n_back=16, skip=16, n_extra=5),
)}
# The fp32 mode on the dense global workload (9 frames of 1024^2 at patch 16)
# and on eight 518^2 frames, with two bf16 terms per operand, and with three.
F32_WORKLOADS = {w.name: w for w in (
    Workload("global_s9_g64_f32", "global_f32", S=9, g=64),
    Workload("frame_s8_g37_f32", "frame_f32", S=8, g=37),
    Workload("global_s9_g64_f32x3", "global_f32", S=9, g=64, terms=3),
)}
# Small scenes batched: 32 scenes of the two-frame 224^2 workload in one call.
BATCH_WORKLOADS = {w.name: w for w in (
    Workload("global_b32_s2_g16", "global_batch", S=2, g=16, B=32),
)}
# The dense global workload with a large QK LayerNorm affine (weights up to 8,
# bias norm 4): precise mode (two-term scores, online softmax).
AFFINE_WORKLOADS = {w.name: w for w in (
    Workload("global_s9_g64_affine8", "global", S=9, g=64, affine=0),
)}
ALL_WORKLOADS = {**WORKLOADS, **PROFILE_WORKLOADS, **STREAM_WORKLOADS, **SUBSET_WORKLOADS, **F32_WORKLOADS,
                 **BATCH_WORKLOADS, **AFFINE_WORKLOADS}


def workload_affine(w: Workload):
    """The workload's QK LayerNorm affine ``(q_weight, q_bias, k_weight,
    k_bias)`` as fp32 CPU tensors, or None."""
    return None if w.affine < 0 else ln_affine_large(w.affine)


def grid_side(T: int) -> int:
    """Side of the square patch grid for ``T`` tokens per frame, or -1."""
    p = T - N_SPECIAL
    if p < 0:
        return -1
    g = math.isqrt(p)
    return g if g * g == p else -1


def grid_positions(S: int, g: int) -> torch.Tensor:
    """``[S*T, 2]`` fp32 (row, col): specials at (0,0), patch (r,c) at (r+1,c+1)."""
    T = N_SPECIAL + g * g
    one = torch.zeros(T, 2, dtype=torch.float32)
    if g > 0:
        r = torch.arange(g, dtype=torch.float32).repeat_interleave(g)
        c = torch.arange(g, dtype=torch.float32).repeat(g)
        one[N_SPECIAL:, 0] = r + 1.0
        one[N_SPECIAL:, 1] = c + 1.0
    return one.repeat(S, 1).contiguous()


def normal_bf16(shape, seed: int) -> torch.Tensor:
    """N(0,1) fp32 from a seeded CPU generator, rounded to bf16."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_qkv(S: int, g: int, seed: int, H: int = HEADS, D: int = HEAD_DIM):
    """Return ``(q, k, v, pos)`` CPU tensors for one scene.

    q, k, v are drawn from three generators seeded ``3*seed``, ``3*seed+1``,
    ``3*seed+2`` so each tensor is reproducible on its own.
    """
    T = N_SPECIAL + g * g
    n = S * T
    q = normal_bf16((n, H, D), 3 * seed)
    k = normal_bf16((n, H, D), 3 * seed + 1)
    v = normal_bf16((n, H, D), 3 * seed + 2)
    return q, k, v, grid_positions(S, g)


def layout_positions(S: int, layout) -> torch.Tensor:
    """``[S*T, 2]`` fp32 for frames laid out ``(n_front, grid_h, grid_w,
    n_back)``: front and trailing tokens at (0,0), patch (r,c) at
    (r+1,c+1)."""
    nf, gh, gw, nb = (int(x) for x in layout)
    one = torch.zeros(nf + gh * gw + nb, 2, dtype=torch.float32)
    if gh > 0 and gw > 0:
        one[nf:nf + gh * gw, 0] = torch.arange(gh, dtype=torch.float32).repeat_interleave(gw) + 1.0
        one[nf:nf + gh * gw, 1] = torch.arange(gw, dtype=torch.float32).repeat(gh) + 1.0
    return one.repeat(S, 1).contiguous()


def make_layout_qkv(S: int, layout, seed: int, H: int = HEADS, D: int = HEAD_DIM):
    """``make_qkv`` for frames laid out ``(n_front, grid_h, grid_w, n_back)``."""
    nf, gh, gw, nb = (int(x) for x in layout)
    n = S * (nf + gh * gw + nb)
    q = normal_bf16((n, H, D), 3 * seed)
    k = normal_bf16((n, H, D), 3 * seed + 1)
    v = normal_bf16((n, H, D), 3 * seed + 2)
    return q, k, v, layout_positions(S, layout)


def ln_affine(seed: int, scale: float = 0.5, shift: float = 0.2, D: int = HEAD_DIM):
    """A seeded QK LayerNorm affine ``(q_weight, q_bias, k_weight, k_bias)``:
    weights 1 + U(-scale, scale), biases N(0, shift^2), fp32 CPU tensors."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(20_000 + int(seed))
    w = lambda: 1.0 + scale * (2.0 * torch.rand(D, generator=gen) - 1.0)  # noqa: E731
    b = lambda: shift * torch.randn(D, generator=gen)  # noqa: E731
    return (w(), b(), w(), b())


def ln_affine_large(seed: int, max_weight: float = 8.0, bias_norm: float = 4.0, D: int = HEAD_DIM):
    """A seeded QK LayerNorm affine with large entries ``(q_weight, q_bias,
    k_weight, k_bias)``: weights of random sign and log-uniform magnitude in
    [0.5, max_weight], one of them exactly max_weight; biases N(0, 1) scaled
    to Euclidean norm ``bias_norm``. fp32 CPU tensors."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(30_000 + int(seed))

    def weight():
        mag = torch.exp(math.log(0.5) + (math.log(max_weight) - math.log(0.5)) * torch.rand(D, generator=gen))
        sign = torch.where(torch.rand(D, generator=gen) < 0.5, -1.0, 1.0)
        w = mag * sign
        w[int(torch.randint(D, (1,), generator=gen))] = max_weight
        return w

    def bias():
        b = torch.randn(D, generator=gen)
        return b * (bias_norm / float(b.norm()))

    return (weight(), bias(), weight(), bias())


def make_sequence_qkv(S: int, layout, n_extra: int, seed: int, H: int = HEADS, D: int = HEAD_DIM):
    """``make_layout_qkv`` plus ``n_extra`` sequence tokens after the frames
    (positions (0,0)), drawn from their own generators."""
    q, k, v, pos = make_layout_qkv(S, layout, seed, H, D)
    if n_extra:
        extra = [normal_bf16((n_extra, H, D), 900 + 3 * seed + i) for i in range(3)]
        q, k, v = (torch.cat([a, b]) for a, b in zip((q, k, v), extra))
        pos = torch.cat([pos, torch.zeros(n_extra, 2)])
    return q, k, v, pos


def make_qkv_f32(S: int, layout, seed: int, H: int = HEADS, D: int = HEAD_DIM):
    """fp32 q, k, v (N(0,1), not rounded) and positions for frames laid out
    ``(n_front, grid_h, grid_w, n_back)``: the inputs of the fp32 mode."""
    nf, gh, gw, nb = (int(x) for x in layout)
    n = S * (nf + gh * gw + nb)
    gens = []
    for i in range(3):
        g = torch.Generator(device="cpu")
        g.manual_seed(3 * int(seed) + i + 50_000)
        gens.append(torch.randn(n, H, D, generator=g, dtype=torch.float32))
    return gens[0], gens[1], gens[2], layout_positions(S, layout)


def make_workload(w: Workload, seed: int):
    if w.kind.endswith("_f32"):
        return make_qkv_f32(w.S, w.layout, seed, w.H, w.D)
    if w.kind.startswith("subset"):
        return make_sequence_qkv(w.S, w.layout, w.n_extra, seed, w.H, w.D)
    return make_qkv(w.B * w.S, w.g, seed, w.H, w.D)


def sample_rows(n: int, count: int, seed: int) -> torch.Tensor:
    """Sorted, distinct query-row indices spread over ``[0, n)``, always
    including the first and the last row (the ragged tail)."""
    count = min(count, n)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(10_000 + int(seed))
    idx = torch.randperm(n, generator=gen)[:count]
    return torch.unique(torch.cat([idx, torch.tensor([0, n - 1])]))
