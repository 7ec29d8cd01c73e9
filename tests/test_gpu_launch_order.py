"""Launch order under programmatic dependent launch.

Every kernel of the library may be scheduled while the work before it in the
stream is still finishing, and must not touch global memory before that work
has completed. The hazard this guards against is one call's kernels reading
or overwriting memory that the previous call's kernels still use: consecutive
calls take their q_hat / k_hat scratch from the same stream-ordered pool (so
a call's prologue may write the block the previous call's attention kernel is
reading), and the no-alloc call always uses the same fixed scratch array.

Each test queues several calls back to back with no synchronisation between
them, each on its own seeded inputs and into its own output, then compares
every output with the oracle on that call's inputs at the usual bars
(max-abs 2e-2, relative Frobenius 5e-3). A kernel that started early would
mix one call's data into another's result.
"""
import numpy as np
import pytest
import torch

from oracle import vggt_oracle as O
import synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3
CALLS = 6


@pytest.fixture(scope="module")
def F():
    import feed_forward_view_b200 as F

    return F


def f64(t: torch.Tensor) -> np.ndarray:
    bits = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return O.bf16_bits_to_f64(bits).reshape(t.shape)


def oracle(kind, q, k, v, pos, S, T, kd):
    qn, kn, vn, pn = f64(q), f64(k), f64(v), pos.numpy().astype(np.float64)
    if kind == "frame":
        return O.attn_frame(qn, kn, vn, pn, S, T)
    if kind == "descriptor":
        return O.attn_descriptor(qn, kn, vn, pn, S, T, kd)
    return O.attn_global(qn, kn, vn, pn, S, T)


def call(F, kind, d, out, S, T, kd):
    q, k, v, pos = d
    if kind == "global":
        F.vggt_attn_global(q, k, v, pos, out, S=S, T=T)
    elif kind == "frame":
        F.vggt_attn_frame(q, k, v, pos, out, S=S, T=T)
    elif kind == "descriptor":
        F.vggt_attn_descriptor(q, k, v, pos, out, S=S, T=T, kv_down=kd)
    else:
        F.vggt_attn_global_noalloc(q, k, v, pos, out, S=S, T=T)


@pytest.mark.parametrize("kind,S,g,kd", [
    ("global", 2, 12, 1),      # one-wave grids: the attention kernel signals its dependents first thing
    ("frame", 3, 9, 1),
    ("descriptor", 3, 9, 3),   # three kernels per call: prologue, pooling + key prologue, attention
    ("noalloc", 2, 12, 1),     # every call shares one fixed scratch array
    ("global", 4, 22, 1),      # 1956 tokens: two-tile CTAs
])
def test_back_to_back_calls_each_see_their_own_inputs(F, kind, S, g, kd):
    T = 5 + g * g
    dev = torch.device("cuda:0")
    host = [synth.make_qkv(S, g, seed=300 + i) for i in range(CALLS)]
    dsets = [tuple(t.to(dev) for t in h) for h in host]
    outs = [torch.empty_like(d[0]) for d in dsets]
    call(F, kind, dsets[0], outs[0], S, T, kd)  # set-up outside the chain
    torch.cuda.synchronize()
    for d, o in zip(dsets, outs):
        call(F, kind, d, o, S, T, kd)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    for i, (h, o) in enumerate(zip(host, outs)):
        ref = oracle(kind, *h, S, T, kd)
        got = f64(o)
        d = got - ref
        mx = float(np.abs(d).max())
        rf = float(np.linalg.norm(d) / np.linalg.norm(ref))
        assert np.isfinite(got).all()
        assert mx <= MAX_ABS and rf <= REL_FRO, (kind, i, mx, rf)


def test_prologue_then_core_chain(F):
    # The core call reads the prologue's outputs written by the kernel just
    # before it; each round overwrites the same q_hat / k_hat buffers.
    S, g = 2, 14
    T = 5 + g * g
    n = S * T
    dev = torch.device("cuda:0")
    host = [synth.make_qkv(S, g, seed=400 + i) for i in range(CALLS)]
    dsets = [tuple(t.to(dev) for t in h) for h in host]
    qh = torch.empty((16, n, 64), dtype=torch.bfloat16, device=dev)
    kh = torch.empty_like(qh)
    outs = [torch.empty_like(d[0]) for d in dsets]
    F.vggt_qk_prologue(dsets[0][0], dsets[0][3], qh)
    torch.cuda.synchronize()
    for (q, k, v, pos), o in zip(dsets, outs):
        F.vggt_qk_prologue(q, pos, qh)
        F.vggt_qk_prologue(k, pos, kh)
        F.vggt_attn_core(qh, kh, v, o, 1, n, n)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    for i, (h, o) in enumerate(zip(host, outs)):
        ref = oracle("global", *h, S, T, 1)
        d = f64(o) - ref
        mx = float(np.abs(d).max())
        rf = float(np.linalg.norm(d) / np.linalg.norm(ref))
        assert mx <= MAX_ABS and rf <= REL_FRO, (i, mx, rf)
