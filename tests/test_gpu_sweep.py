"""A seeded sweep of random small shapes through every entry point, against the
fp64 oracle: head counts that are not 16 (including odd ones), frames of a
few tokens up to several query tiles, kv_down from 1 to beyond the grid,
rectangular grids with front and trailing tokens, token subsets, chunked
streams and the fp32 mode (two and three terms). Same bars as the other parity tests."""
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


def f64(t):
    t = t.detach().cpu()
    if t.dtype == torch.float32:
        return t.double().numpy()
    return O.bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16)).reshape(t.shape)


def check(got, ref, what, max_abs=MAX_ABS, rel_fro=REL_FRO):
    g = f64(got)
    assert np.isfinite(g).all(), what
    d = g - ref
    mx = float(np.abs(d).max())
    rf = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))
    assert mx <= max_abs and rf <= rel_fro, (what, mx, rf)


def cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        H = int(rng.choice([1, 3, 5, 16, 17]))
        S = int(rng.integers(1, 5))
        nf = int(rng.integers(0, 6))
        gh, gw = int(rng.integers(0, 14)), int(rng.integers(0, 14))
        if gh * gw == 0:
            gh = gw = 0
        nb = int(rng.integers(0, 5))
        if nf + gh * gw + nb == 0:
            nf = 1
        kd = int(rng.integers(1, 7))
        out.append((i, H, S, (nf, gh, gw, nb), kd))
    return out


@pytest.mark.parametrize("i,H,S,layout,kd", cases(80, 2024))
def test_sweep_bf16_entry_points(F, i, H, S, layout, kd):
    q, k, v, pos = (t.cuda() for t in synth.make_layout_qkv(S, layout, seed=100 + i, H=H))
    T = q.shape[0] // S
    qn, kn, vn, pn = f64(q), f64(k), f64(v), pos.cpu().numpy().astype(np.float64)
    ln = synth.ln_affine(200 + i) if i % 3 == 0 else None
    ln64 = None if ln is None else tuple(x.numpy().astype(np.float64) for x in ln)
    what = (i, H, S, layout, kd)
    out = F.vggt_attn_frame_ex(q, k, v, pos, S=S, T=T, H=H, ln=ln)
    check(out, O.attn_frame(qn, kn, vn, pn, S, T, ln=ln64), ("frame",) + what)
    out = F.vggt_attn_global_ex(q, k, v, pos, S=S, T=T, H=H, ln=ln)
    check(out, O.attn_global(qn, kn, vn, pn, S, T, ln=ln64), ("global",) + what)
    if layout[1] * layout[2] > 0 or layout[0] + layout[3] > 0:
        out = F.vggt_attn_descriptor_ex(q, k, v, pos, S=S, T=T, H=H, kv_down=kd, layout=layout, ln=ln)
        check(out, O.attn_descriptor(qn, kn, vn, pn, S, T, kd, layout=layout, ln=ln64), ("descriptor",) + what)
        ko, vo, po = F.vggt_kv_pool_ex(k, v, pos, S=S, T=T, H=H, kv_down=kd, layout=layout)
        rk, rv, rp = O.kv_pool_bf16_reference(
            k.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(S * T, -1),
            v.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(S * T, -1),
            pos.cpu().numpy(), S, T, kd, layout=layout)
        assert np.array_equal(ko.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(rk.shape), rk)
        assert np.array_equal(vo.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(rv.shape), rv)
        assert np.array_equal(po.cpu().numpy(), rp)
    skip = min(layout[3], T - 1)
    E = i % 4
    qs, ks, vs, ps = (t.cuda() for t in synth.make_sequence_qkv(S, layout, E, seed=300 + i, H=H))
    kind = "global" if i % 2 else "frame"
    out = F.vggt_attn_subset(qs, ks, vs, ps, S=S, T=T, n_skip_back=skip, n_extra=E, H=H, kind=kind, ln=ln)
    kept = O.subset_rows(S, T, skip, E if kind == "global" else 0)
    ref = O.attn_subset(f64(qs), f64(ks), f64(vs), ps.cpu().numpy().astype(np.float64), S, T, skip, E, kind,
                        ln=ln64)
    check(out[torch.from_numpy(kept).cuda()], ref, ("subset", kind, skip, E) + what)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0


@pytest.mark.parametrize("i,H,S,layout,kd", cases(32, 77))
def test_sweep_stream_and_fp32(F, i, H, S, layout, kd):
    T = sum(layout[::3]) + layout[1] * layout[2]
    if layout[1] * layout[2] > 0:
        q, k, v, pos = (t.cuda() for t in synth.make_layout_qkv(S, layout, seed=400 + i, H=H))
        out = torch.empty_like(q)
        chunk = 1 + i % 3
        with F.DescCache(S, T, H=H, kv_down=kd, layout=layout) as cache:
            for f0 in range(0, S, chunk):
                c = min(chunk, S - f0)
                r = slice(f0 * T, (f0 + c) * T)
                cache.attend(q[r], k[r], v[r], pos[r], out[r], C=c)
        ref = O.attn_descriptor_stream(f64(q), f64(k), f64(v), pos.cpu().numpy().astype(np.float64), S, T, kd,
                                       chunk, layout=layout)
        check(out, ref, ("stream", i, H, S, layout, kd, chunk))
    q, k, v, pos = (t.cuda() for t in synth.make_qkv_f32(S, layout, seed=500 + i, H=H))
    terms = 2 + i % 2
    bar_abs, bar_fro = {2: (2e-5, 2e-4), 3: (4e-6, 5e-5)}[terms]
    for kind in ("frame", "global"):
        fn = F.vggt_attn_frame_f32 if kind == "frame" else F.vggt_attn_global_f32
        out = fn(q, k, v, pos, S=S, T=T, H=H, terms=terms)
        oracle = O.attn_frame if kind == "frame" else O.attn_global
        ref = oracle(f64(q), f64(k), f64(v), pos.cpu().numpy().astype(np.float64), S, T)
        check(out, ref, ("fp32", kind, terms, i, H, S, layout), max_abs=bar_abs * float(v.abs().max()),
              rel_fro=bar_fro)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
