"""GPU parity of the softmax with a running row maximum (online softmax) and of
precise mode, against the fp64 CPU oracle.

* vggt_attn_core_online takes any finite q_hat / k_hat: it is checked against
  the oracle's plain softmax on scores far beyond the maximum-free kernel's
  bound, including rows whose maximum keeps growing from block to block (a
  rescale of [O | l] at every key block).
* QK LayerNorm affines beyond the plain LayerNorm's score scale (weights up
  to 8, bias norm 4) run in precise mode: q_hat in fp32, k_hat in two bf16
  terms, online softmax, bf16 output. Every bf16 entry point that takes an
  affine is checked at the same bars as the plain calls (max-abs 2e-2,
  relative Frobenius 5e-3), small shapes spanning several tiles and ragged
  tails, and the 36 909-token workload on sampled rows.
* The fp32 mode takes the same affines through its own online instance;
  its error grows with the score scale, so its bars are the plain fp32-mode
  bars times r = |q_hat| |k_hat| / 64 (typical norms, sqrt(sum w^2 + sum
  b^2) per side; 1 without an affine)."""
import numpy as np
import pytest
import torch

from oracle import vggt_oracle as O
import synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3


@pytest.fixture(scope="module")
def F():
    import feed_forward_view_b200 as F

    return F


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return O.bf16_bits_to_f64(bits(t)).reshape(t.shape)


def ln64(ln):
    return None if ln is None else tuple(None if x is None else x.numpy().astype(np.float64) for x in ln)


def errors(got: np.ndarray, ref: np.ndarray):
    d = got - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))


def check(got, ref: np.ndarray, what, rows=None):
    g = f64(got) if isinstance(got, torch.Tensor) else got
    if rows is not None:
        g = g[rows]
    assert np.isfinite(g).all(), what
    mx, rf = errors(g, ref)
    assert mx <= MAX_ABS and rf <= REL_FRO, (what, mx, rf)


def status_ok(F):
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0


def head_major(x: torch.Tensor) -> torch.Tensor:
    return x.permute(1, 0, 2).contiguous()


def pos64(pos):
    return pos.numpy().astype(np.float64)


# ------------------------------------------------------------------ the core


def _core_online(F, qh, kh, v, n_seg, q_len, k_len):
    H = qh.shape[1]
    out = torch.empty(qh.shape[0], H, 64, dtype=torch.bfloat16, device="cuda")
    F.vggt_attn_core_online(head_major(qh).cuda(), head_major(kh).cuda(), v.cuda(), out, n_seg, q_len, k_len, H=H)
    status_ok(F)
    return out.cpu()


def _oracle_segments(qh, kh, v, n_seg, q_len, k_len):
    qh, kh, v = f64(qh), f64(kh), f64(v)
    out = np.empty((qh.shape[0], qh.shape[1], 64))
    for s in range(n_seg):
        qs, ks = slice(s * q_len, (s + 1) * q_len), slice(s * k_len, (s + 1) * k_len)
        out[qs] = O.cross_attention(qh[qs], kh[ks], v[ks])
    return out


@pytest.mark.parametrize("n_seg,q_len,k_len,H,scale", [
    (1, 300, 1000, 2, 60.0),    # |q_hat|, |k_hat| ~ 60 * 8: scores up to ~1e4
    (3, 250, 200, 3, 25.0),     # frame-like segments, ragged tails (200 keys = 2 blocks + 8)
    (1, 130, 97, 1, 200.0),     # one key past a block, scores ~1e5
    (2, 5, 7, 2, 10.0),         # tiny segments: every block masked
])
def test_core_online_matches_oracle_on_unbounded_scores(F, n_seg, q_len, k_len, H, scale):
    gen = torch.Generator().manual_seed(500 + q_len)
    qh = (scale * torch.randn(n_seg * q_len, H, 64, generator=gen)).to(torch.bfloat16)
    kh = (scale * torch.randn(n_seg * k_len, H, 64, generator=gen)).to(torch.bfloat16)
    v = torch.randn(n_seg * k_len, H, 64, generator=gen).to(torch.bfloat16)
    out = _core_online(F, qh, kh, v, n_seg, q_len, k_len)
    check(out, _oracle_segments(qh, kh, v, n_seg, q_len, k_len), ("core online", n_seg, q_len, k_len, scale))


def test_core_online_rescales_at_every_block(F):
    # Every query is c * u and key j is t_j * u + (noise orthogonal to u) with
    # t_j rising over the keys: each 96-key block's maximum beats the last by
    # far more than 2^8, so the running reference moves (and [O | l] is
    # rescaled) at every block; the final row is dominated by the last keys.
    gen = torch.Generator().manual_seed(77)
    H, nq, nk = 2, 256, 1100
    u = torch.randn(H, 64, generator=gen, dtype=torch.float64)
    u = u / u.norm(dim=-1, keepdim=True)
    t = torch.linspace(0.0, 40.0, nk, dtype=torch.float64)[:, None, None]
    noise = torch.randn(nk, H, 64, generator=gen, dtype=torch.float64)
    noise = noise - (noise * u).sum(-1, keepdim=True) * u
    qh = (16.0 * u).expand(nq, H, 64).to(torch.bfloat16)
    kh = (t * u + 0.5 * noise).to(torch.bfloat16)
    v = torch.randn(nk, H, 64, generator=gen).to(torch.bfloat16)
    out = _core_online(F, qh, kh, v, 1, nq, nk)
    ref = _oracle_segments(qh, kh, v, 1, nq, nk)
    # the scores span 0 .. 80 (natural units): weights across e^80, 2^115
    s = (f64(qh)[0] * f64(kh)).sum(-1) / 8.0
    assert s.max() - s.min() > 75
    check(out, ref, "rising maxima")


def test_core_online_equals_core_on_prologue_outputs(F):
    # On the prologue's own vectors both softmax forms are valid: each agrees
    # with the oracle, and with the other to within their roundings.
    S, g = 3, 13
    q, k, v, pos = synth.make_qkv(S, g, seed=81)
    T = 5 + g * g
    qd, kd_, vd, pd = (t.cuda() for t in (q, k, v, pos))
    qh = F.vggt_qk_prologue(qd, pd)
    kh = F.vggt_qk_prologue(kd_, pd)
    for kind, n_seg, ql in (("global", 1, S * T), ("frame", S, T)):
        a = torch.empty_like(qd)
        b = torch.empty_like(qd)
        F.vggt_attn_core(qh, kh, vd, a, n_seg, ql, ql)
        F.vggt_attn_core_online(qh, kh, vd, b, n_seg, ql, ql)
        status_ok(F)
        ref = (O.attn_global if kind == "global" else O.attn_frame)(f64(q), f64(k), f64(v), pos64(pos), S, T)
        check(a, ref, (kind, "max-free"))
        check(b, ref, (kind, "online"))
        mx, rf = errors(f64(a), f64(b))
        assert mx <= 2e-2 and rf <= 4e-3, (kind, mx, rf)


# ------------------------------------------------------- precise mode (bf16)

LARGE = [
    dict(max_weight=8.0, bias_norm=4.0),
    dict(max_weight=3.0, bias_norm=0.0),
    dict(max_weight=1.5, bias_norm=1.0),
]


@pytest.mark.parametrize("kind,S,layout", [
    ("global", 2, (5, 16, 16, 0)),
    ("global", 3, (5, 9, 13, 0)),
    ("frame", 3, (5, 14, 14, 0)),
    ("frame", 4, (0, 6, 8, 3)),
])
@pytest.mark.parametrize("aff", range(len(LARGE)))
def test_frame_and_global_large_affine(F, kind, S, layout, aff):
    q, k, v, pos = synth.make_layout_qkv(S, layout, seed=90 + aff)
    T = q.shape[0] // S
    ln = synth.ln_affine_large(aff, **LARGE[aff])
    fn = F.vggt_attn_global_ex if kind == "global" else F.vggt_attn_frame_ex
    out = fn(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, ln=ln)
    status_ok(F)
    oracle = O.attn_global if kind == "global" else O.attn_frame
    ref = oracle(f64(q), f64(k), f64(v), pos64(pos), S, T, ln=ln64(ln))
    check(out, ref, (kind, S, layout, LARGE[aff]))


@pytest.mark.parametrize("layout,kd", [((5, 25, 37, 0), 4), ((0, 12, 12, 4), 3), ((5, 9, 9, 0), 1)])
def test_descriptor_large_affine(F, layout, kd):
    S = 3
    q, k, v, pos = synth.make_layout_qkv(S, layout, seed=95)
    T = q.shape[0] // S
    ln = synth.ln_affine_large(5)
    out = F.vggt_attn_descriptor_ex(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, kv_down=kd, layout=layout,
                                    ln=ln)
    status_ok(F)
    ref = O.attn_descriptor(f64(q), f64(k), f64(v), pos64(pos), S, T, kd, layout=layout, ln=ln64(ln))
    check(out, ref, ("descriptor", layout, kd))


def test_stream_large_affine(F):
    S, layout, kd, chunk = 5, (5, 11, 11, 0), 4, 2
    q, k, v, pos = synth.make_layout_qkv(S, layout, seed=96)
    T = q.shape[0] // S
    ln = synth.ln_affine_large(6)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    qd, kd_, vd, pd = (t.cuda() for t in (q, k, v, pos))
    with F.DescCache(S, T, kv_down=kd, layout=layout, ln=ln) as cache:
        for f0 in range(0, S, chunk):
            c = min(chunk, S - f0)
            r0, r1 = f0 * T, (f0 + c) * T
            cache.attend(qd[r0:r1], kd_[r0:r1], vd[r0:r1], pd[r0:r1], out[r0:r1], C=c)
    status_ok(F)
    ref = O.attn_descriptor_stream(f64(q), f64(k), f64(v), pos64(pos), S, T, kd, chunk, layout=layout, ln=ln64(ln))
    check(out, ref, "stream")


@pytest.mark.parametrize("kind", ["global", "frame"])
def test_subset_large_affine(F, kind):
    S, layout, skip, E = 3, (0, 6, 8, 2), 2, 3
    q, k, v, pos = synth.make_sequence_qkv(S, layout, E, seed=97)
    T = 6 * 8 + 2
    ln = synth.ln_affine_large(7)
    out = torch.full(q.shape, 7.0, dtype=torch.bfloat16, device="cuda")
    F.vggt_attn_subset(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), out, S=S, T=T, n_skip_back=skip, n_extra=E,
                       kind=kind, ln=ln)
    status_ok(F)
    kept = O.subset_rows(S, T, skip, E) if kind == "global" else O.subset_rows(S, T, skip, 0)
    ref = O.attn_subset(f64(q), f64(k), f64(v), pos64(pos), S, T, skip, E, kind, ln=ln64(ln))
    got = f64(out.cpu())
    check(got[kept], ref, ("subset", kind))
    untouched = np.setdiff1d(np.arange(q.shape[0]), kept)
    assert (got[untouched] == 7.0).all()


def test_batch_large_affine(F):
    B, S, g = 3, 2, 7
    T = 5 + g * g
    parts = [synth.make_qkv(S, g, seed=100 + b) for b in range(B)]
    q, k, v, pos = (torch.cat([p[i] for p in parts]) for i in range(4))
    ln = synth.ln_affine_large(8)
    out = F.vggt_attn_global_batch(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), B=B, S=S, T=T, ln=ln)
    outd = F.vggt_attn_descriptor_batch(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), B=B, S=S, T=T, kv_down=2, ln=ln)
    status_ok(F)
    args = (f64(q), f64(k), f64(v), pos64(pos))
    check(out, O.attn_scenes("global", *args, B, S, T, ln=ln64(ln)), "global batch")
    check(outd, O.attn_scenes("descriptor", *args, B, S, T, kd=2, ln=ln64(ln)), "descriptor batch")


@pytest.mark.parametrize("w", [1.09, 1.12])
def test_either_side_of_the_precise_threshold(F, w):
    # uniform weights w on both sides, no bias: at 1.09 the call stays on the
    # bf16 kernel without a row maximum, at 1.12 it runs in precise mode; both
    # meet the bars, with queries equal to the keys (each query's own key
    # scores about w^2 |x_hat|^2 / 8 ~ 10) and with independent keys.
    S, g = 2, 12
    q, _, v, pos = synth.make_qkv(S, g, seed=110)
    T = 5 + g * g
    wt = torch.full((64,), w)
    ln = (wt, None, wt, None)
    for k in (q, synth.make_qkv(S, g, seed=111)[1]):
        out = F.vggt_attn_global_ex(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, ln=ln)
        status_ok(F)
        ref = O.attn_global(f64(q), f64(k), f64(v), pos64(pos), S, T, ln=ln64(ln))
        check(out, ref, ("threshold", w))


def test_large_affine_full_size_sampled_rows(F):
    # the 36 909-token scene (9 frames of 64 x 64 patches + 5 special tokens)
    # with weights up to 8 and bias norm 4; 256 sampled query rows
    S, g = 9, 64
    T = 5 + g * g
    q, k, v, pos = synth.make_qkv(S, g, seed=120)
    ln = synth.ln_affine_large(9)
    out = F.vggt_attn_global_ex(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, ln=ln)
    status_ok(F)
    rows = synth.sample_rows(S * T, 256, seed=4).numpy()
    ref = O.attn_global(f64(q), f64(k), f64(v), pos64(pos), S, T, rows=rows, ln=ln64(ln))
    check(out, ref, "global 36909 large affine", rows=rows)


def test_large_affine_descriptor_many_frames_sampled_rows(F):
    # 40 frames of 1374 tokens, 4 x 4 descriptors (4200 keys), 256 sampled rows
    S, g, kd = 40, 37, 4
    T = 5 + g * g
    q, k, v, pos = synth.make_qkv(S, g, seed=121)
    ln = synth.ln_affine_large(10)
    out = F.vggt_attn_descriptor_ex(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, kv_down=kd, ln=ln)
    status_ok(F)
    rows = synth.sample_rows(S * T, 256, seed=5).numpy()
    ref = O.attn_descriptor(f64(q), f64(k), f64(v), pos64(pos), S, T, kd, rows=rows, ln=ln64(ln))
    check(out, ref, "descriptor 40 frames large affine", rows=rows)


# ------------------------------------------------------------ the fp32 mode


def _typical_ratio(ln):
    def typ(w, b):
        w = np.ones(64) if w is None else w
        b = np.zeros(64) if b is None else b
        return float(np.sqrt((w ** 2).sum() + (b ** 2).sum()))

    return typ(ln[0], ln[1]) * typ(ln[2], ln[3]) / 64.0


@pytest.mark.parametrize("kind", ["global", "frame"])
@pytest.mark.parametrize("terms,bar_abs,bar_rel", [(2, 2e-5, 2e-4), (3, 4e-6, 5e-5)])
def test_f32_mode_large_affine(F, kind, terms, bar_abs, bar_rel):
    S, layout = 3, (5, 10, 10, 0)
    q, k, v, pos = synth.make_qkv_f32(S, layout, seed=130)
    T = 105
    ln = synth.ln_affine_large(11)
    fn = F.vggt_attn_global_f32 if kind == "global" else F.vggt_attn_frame_f32
    out = fn(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, ln=ln, terms=terms)
    status_ok(F)
    oracle = O.attn_global if kind == "global" else O.attn_frame
    ref = oracle(*(t.double().numpy() for t in (q, k, v, pos)), S, T, ln=ln64(ln))
    r = _typical_ratio(ln64(ln))
    mx, rf = errors(out.cpu().double().numpy(), ref)
    vmax = float(v.abs().max())
    assert mx <= bar_abs * r * vmax and rf <= bar_rel * r, (kind, terms, mx, rf, r)
