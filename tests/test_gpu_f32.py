"""GPU parity of the fp32 mode (fp32 q, k, v in, fp32 out; both attention
products as bf16 MMAs on the operands' bf16 terms) against the fp64 oracle,
with two terms and with three.

Bars (from the arithmetic). Two terms carry an fp32 operand to ~2^-17
relative and the dropped products are ~2^-18 of a product, so a score
q_hat.k_hat/8 (|score| < 8) is off by ~1e-5 at most and p = 2^s (MUFU,
~2^-22) by ~1e-5 relative; an output, a weighted mean of N(0,1) values, is
then off by ~1e-5 of the values' scale at worst -- against ~1e-2 for the bf16
path. The values enter as v_0 + v_1 with p_1 v_1 dropped: with a single key
the output is v to ~1e-5 of |v|. Three terms hold an fp32 value exactly and
drop products of ~2^-27; what is left is fp32 itself: the prologue's fp32
LayerNorm and RoPE angles move a score by ~1e-6, the exponentials are good
to ~2.4e-7, the accumulations round in fp32. The outputs shrink like
1/sqrt(keys) (about 0.04 at 36 909 keys), so the relative Frobenius error of
the same absolute error grows with the key count.
Bars: max-abs <= 2e-5 * max|v| (two terms), 4e-6 * max|v| (three terms);
relative Frobenius <= 2e-4 (two) and 5e-5 (three); two terms at least 50x
below the bf16 path on the same inputs rounded to bf16, three terms at least
10x below two where the value split dominates (a single key)."""
import numpy as np
import pytest
import torch

from oracle import vggt_oracle as O
import synth

pytestmark = pytest.mark.gpu

# terms -> (max-abs per max|v|, relative Frobenius)
BARS = {2: (2e-5, 2e-4), 3: (4e-6, 5e-5)}


@pytest.fixture(scope="module")
def F():
    import feed_forward_view_b200 as F

    return F


def f64(t):
    return t.detach().cpu().double().numpy()


def errs(got, ref):
    d = got - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(ref))


def ln64(ln):
    return None if ln is None else tuple(None if x is None else x.numpy().astype(np.float64) for x in ln)


@pytest.mark.parametrize("terms", [2, 3])
@pytest.mark.parametrize("kind,S,layout,affine", [
    ("global", 2, (5, 16, 16, 0), False),   # 522 tokens: ragged tiles and key blocks
    ("frame", 3, (0, 10, 30, 0), False),    # T = 300
    ("global", 2, (5, 11, 19, 3), True),
    ("frame", 8, (5, 37, 37, 0), False),    # 1374-token frames
    ("global", 1, (0, 1, 1, 0), False),     # a single token
])
def test_f32_mode_matches_oracle(F, kind, S, layout, affine, terms):
    q, k, v, pos = synth.make_qkv_f32(S, layout, seed=71)
    T = q.shape[0] // S
    ln = synth.ln_affine(13) if affine else None
    fn = F.vggt_attn_frame_f32 if kind == "frame" else F.vggt_attn_global_f32
    out = fn(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, ln=ln, terms=terms)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    oracle = O.attn_frame if kind == "frame" else O.attn_global
    ref = oracle(f64(q), f64(k), f64(v), pos.numpy().astype(np.float64), S, T, ln=ln64(ln))
    got = f64(out)
    assert np.isfinite(got).all()
    mx, rf = errs(got, ref)
    bar_abs, bar_fro = BARS[terms]
    assert mx <= bar_abs * float(v.abs().max()) and rf <= bar_fro, (kind, S, layout, terms, mx, rf)


@pytest.mark.parametrize("terms", [2, 3])
@pytest.mark.parametrize("layout", [
    (0, 32, 24, 0),   # 768 keys: 8 blocks, no fold
    (1, 32, 24, 0),   # 769 keys: 9 blocks, the fold lands on the last block
    (1, 32, 48, 0),   # 1537 keys: 17 blocks, a copy fold and an add fold
])
def test_f32_mode_fold_boundaries(F, layout, terms):
    # [O | l] is folded into a second sum every 8 key blocks of 96 keys; key
    # counts around those boundaries, one frame attended globally
    q, k, v, pos = synth.make_qkv_f32(1, layout, seed=75)
    T = q.shape[0]
    out = F.vggt_attn_global_f32(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=1, T=T, terms=terms)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    ref = O.attn_global(f64(q), f64(k), f64(v), pos.numpy().astype(np.float64), 1, T)
    mx, rf = errs(f64(out), ref)
    bar_abs, bar_fro = BARS[terms]
    assert mx <= bar_abs * float(v.abs().max()) and rf <= bar_fro, (layout, terms, mx, rf)


def test_f32_mode_is_far_more_accurate_than_bf16(F):
    S, layout = 2, (5, 16, 16, 0)
    q, k, v, pos = synth.make_qkv_f32(S, layout, seed=72)
    T = q.shape[0] // S
    qb, kb, vb = (t.to(torch.bfloat16) for t in (q, k, v))
    d = [t.cuda() for t in (q, k, v, pos)]
    o32 = F.vggt_attn_global_f32(*d, S=S, T=T)
    o16 = F.vggt_attn_global_ex(qb.cuda(), kb.cuda(), vb.cuda(), d[3], S=S, T=T)
    torch.cuda.synchronize()
    p = pos.numpy().astype(np.float64)
    e32 = errs(f64(o32), O.attn_global(f64(q), f64(k), f64(v), p, S, T))[1]
    e16 = errs(f64(o16.float()), O.attn_global(f64(qb.float()), f64(kb.float()), f64(vb.float()), p, S, T))[1]
    assert e32 * 50 < e16, (e32, e16)


def test_three_terms_carry_the_values(F):
    # one key: the output is v itself; two terms keep v to ~2^-17, three exactly
    q, k, v, pos = synth.make_qkv_f32(1, (0, 1, 1, 0), seed=74)
    d = [t.cuda() for t in (q, k, v, pos)]
    ref = f64(v)
    e = {t: errs(f64(F.vggt_attn_global_f32(*d, S=1, T=1, terms=t)), ref)[0] for t in (2, 3)}
    assert e[3] * 10 < e[2] and e[3] <= 1e-6 * float(v.abs().max()), e


@pytest.mark.parametrize("terms", [2, 3])
def test_f32_mode_full_size_sampled_rows(F, terms):
    # the bench workload's shape (9 frames of 4101 tokens), rows sampled
    S, layout = 9, (5, 64, 64, 0)
    q, k, v, pos = synth.make_qkv_f32(S, layout, seed=73)
    T = q.shape[0] // S
    out = F.vggt_attn_global_f32(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, terms=terms)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    rows = synth.sample_rows(S * T, 256, seed=5).numpy()
    ref = O.attn_global(f64(q), f64(k), f64(v), pos.numpy().astype(np.float64), S, T, rows=rows)
    mx, rf = errs(f64(out)[rows], ref)
    bar_abs, bar_fro = BARS[terms]
    assert mx <= bar_abs * float(v.abs().max()) and rf <= bar_fro, (terms, mx, rf)
