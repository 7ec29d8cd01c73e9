"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle on
the same seeded inputs.

Bars (fixed by the method's statement of the target):
* attention outputs: max-abs error <= 2e-2 and relative Frobenius error
  <= 5e-3 against the oracle, over every compared row;
* pooled K/V: bit-exact against the oracle's bf16 form of the float32 mean;
  pooled positions: exact;
* prologue: within one bf16 rounding of the exact value (2^-8 relative) plus a
  small absolute allowance for float32 arithmetic.
"""
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


def errors(got: np.ndarray, ref: np.ndarray):
    d = got - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))


def oracle_rows(kind, q, k, v, pos, S, T, kd, rows):
    qn, kn, vn, pn = f64(q), f64(k), f64(v), pos.numpy().astype(np.float64)
    if kind == "global":
        return O.attn_global(qn, kn, vn, pn, S, T, rows=rows)
    if kind == "frame":
        return O.attn_frame(qn, kn, vn, pn, S, T, rows=rows)
    return O.attn_descriptor(qn, kn, vn, pn, S, T, kd, rows=rows)


def run_gpu(F, kind, q, k, v, pos, S, T, kd, stream=None):
    dev = torch.device("cuda:0")
    qd, kd_, vd, pd = (t.to(dev) for t in (q, k, v, pos))
    out = torch.empty_like(qd)
    fn = {"global": F.vggt_attn_global, "frame": F.vggt_attn_frame,
          "descriptor": F.vggt_attn_descriptor}[kind]
    fn(qd, kd_, vd, pd, out, S=S, T=T, kv_down=kd, stream=stream)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    return out.cpu()


def check_attention(F, kind, S, g, kd, seed, rows=None):
    q, k, v, pos = synth.make_qkv(S, g, seed)
    T = 5 + g * g
    out = run_gpu(F, kind, q, k, v, pos, S, T, kd)
    rows = np.arange(S * T) if rows is None else np.asarray(rows)
    ref = oracle_rows(kind, q, k, v, pos, S, T, kd, rows)
    got = f64(out)[rows]
    mx, rf = errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= MAX_ABS and rf <= REL_FRO, (kind, S, g, kd, mx, rf)
    return mx, rf


# ------------------------------------------------------------------ prologue


@pytest.mark.parametrize("S,g,H", [(2, 22, 16), (1, 0, 3), (3, 7, 5)])
def test_prologue_matches_oracle(F, S, g, H):
    x, _, _, pos = synth.make_qkv(S, g, seed=5, H=H)
    xh = F.vggt_qk_prologue(x.cuda(), pos.cuda(), H=H)
    torch.cuda.synchronize()
    ref = O.qk_prologue(f64(x), pos.numpy().astype(np.float64)).transpose(1, 0, 2)
    got = f64(xh.cpu())
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4)


def test_prologue_large_positions(F):
    # 64x64 grid: angles up to 64 rad
    x, _, _, pos = synth.make_qkv(1, 64, seed=6)
    xh = F.vggt_qk_prologue(x.cuda(), pos.cuda())
    torch.cuda.synchronize()
    ref = O.qk_prologue(f64(x), pos.numpy().astype(np.float64)).transpose(1, 0, 2)
    got = f64(xh.cpu())
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4)


# ------------------------------------------------------------------ pooling


@pytest.mark.parametrize("S,g,kd", [(2, 37, 4), (3, 5, 2), (2, 6, 1), (2, 7, 9), (1, 0, 4), (4, 16, 3)])
def test_kv_pool_bit_exact(F, S, g, kd):
    _, k, v, pos = synth.make_qkv(S, g, seed=7)
    T = 5 + g * g
    ko, vo, po = F.vggt_kv_pool(k.cuda(), v.cuda(), pos.cuda(), S=S, T=T, kv_down=kd)
    torch.cuda.synchronize()
    kb, vb, pb = O.kv_pool_bf16_reference(bits(k), bits(v), pos.numpy(), S, T, kd)
    assert np.array_equal(bits(ko).reshape(kb.shape), kb)
    assert np.array_equal(bits(vo).reshape(vb.shape), vb)
    assert np.array_equal(po.cpu().numpy(), pb)


def test_kv_pool_sums_in_row_major_order(F):
    S, g, kd, H = 1, 2, 2, 16
    T = 5 + g * g
    k = torch.zeros(T, H, 64)
    k[5], k[6], k[7], k[8] = 2.0 ** 24, 1.0, -(2.0 ** 24), 1.0
    k = k.to(torch.bfloat16)
    pos = synth.grid_positions(S, g)
    ko, _, _ = F.vggt_kv_pool(k.cuda(), k.cuda(), pos.cuda(), S=S, T=T, kv_down=kd)
    torch.cuda.synchronize()
    assert torch.all(ko[5].float().cpu() == 0.25)


# ------------------------------------------------------------------ attention

SMALL = [
    ("global", 2, 16, 1),      # 522 tokens: 4 full tiles + 10-row tail
    ("frame", 3, 20, 1),       # 405 tokens per frame: 3 tiles + 21-row tail
    ("frame", 2, 11, 1),       # 126 tokens per frame: one partial tile
    ("global", 1, 15, 1),      # 230 tokens: an odd pair with a partial second tile
    ("global", 1, 0, 1),       # 5 special tokens only
    ("global", 2, 1, 1),       # 6 tokens per frame
    ("descriptor", 4, 37, 4),  # 420 pooled keys
    ("descriptor", 3, 9, 3),   # 3x3 cells
    ("descriptor", 2, 10, 1),  # kv_down 1 == dense global
    ("descriptor", 2, 7, 9),   # one cell per frame
]


@pytest.mark.parametrize("kind,S,g,kd", SMALL)
def test_attention_small_full(F, kind, S, g, kd):
    check_attention(F, kind, S, g, kd, seed=11)


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_attention_full_workloads(F, name):
    w = synth.WORKLOADS[name]
    n = w.n_q
    rows = None if n <= 12000 and w.kind == "frame" or n <= 600 else synth.sample_rows(n, 384, seed=3).numpy()
    check_attention(F, w.kind, w.S, w.g, w.kv_down, seed=1, rows=rows)


def test_core_on_prologue_outputs_equals_the_fused_call(F):
    # vggt_attn_core on vggt_qk_prologue outputs runs the same kernels as
    # vggt_attn_global / vggt_attn_frame: the results are identical.
    S, g = 3, 13
    q, k, v, pos = synth.make_qkv(S, g, seed=12)
    T = 5 + g * g
    qd, kd_, vd, pd = (t.cuda() for t in (q, k, v, pos))
    qh = F.vggt_qk_prologue(qd, pd)
    kh = F.vggt_qk_prologue(kd_, pd)
    for kind, n_seg, ql in (("global", 1, S * T), ("frame", S, T)):
        out = torch.empty_like(qd)
        F.vggt_attn_core(qh, kh, vd, out, n_seg, ql, ql)
        torch.cuda.synchronize()
        assert torch.equal(out.cpu(), run_gpu(F, kind, q, k, v, pos, S, T, 1))


def test_descriptor_kd1_equals_global_on_gpu(F):
    q, k, v, pos = synth.make_qkv(2, 12, seed=13)
    T = 5 + 144
    a = run_gpu(F, "descriptor", q, k, v, pos, 2, T, 1)
    b = run_gpu(F, "global", q, k, v, pos, 2, T, 1)
    mx, rf = errors(a.double().numpy(), b.double().numpy())
    assert mx <= 1e-2 and rf <= 2e-3


def test_zero_queries_average_values(F):
    # q = 0 -> every score is 0 -> out = mean of the visible V rows.
    S, g = 2, 12
    q, k, v, pos = synth.make_qkv(S, g, seed=14)
    T = 5 + g * g
    q.zero_()
    out = f64(run_gpu(F, "frame", q, k, v, pos, S, T, 1))
    vv = f64(v)
    for s in range(S):
        want = vv[s * T:(s + 1) * T].mean(axis=0)
        assert np.abs(out[s * T:(s + 1) * T] - want).max() < 4e-3


def test_output_guard_regions_untouched(F):
    S, g = 2, 16
    q, k, v, pos = synth.make_qkv(S, g, seed=15)
    T = 5 + g * g
    n = S * T * 16 * 64
    G = 4096
    buf = torch.full((n + 2 * G,), -7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[G:G + n].view(S * T, 16, 64)
    F.vggt_attn_global(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), out, S=S, T=T)
    torch.cuda.synchronize()
    assert torch.all(buf[:G] == -7.0) and torch.all(buf[G + n:] == -7.0)
    assert torch.isfinite(out).all()


def test_repeatable_and_stream_ordered(F):
    S, g = 3, 20
    q, k, v, pos = synth.make_qkv(S, g, seed=16)
    T = 5 + g * g
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = run_gpu(F, "frame", q, k, v, pos, S, T, 1, stream=s)
        b = run_gpu(F, "frame", q, k, v, pos, S, T, 1, stream=s)
    assert torch.equal(a, b)


def test_empty_problem_is_a_no_op(F):
    q = torch.zeros(0, 16, 64, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(0, 2, device="cuda")
    out = torch.zeros(0, 16, 64, dtype=torch.bfloat16, device="cuda")
    F.vggt_attn_global(q, q, q, pos, out, S=0, T=261)
    assert F.vggt_get_device_status() == 0


def test_bounded_wait_reports_timeout_and_context_survives(F):
    prev = F.vggt_set_wait_limit(200_000)
    try:
        F.vggt_debug_wait_timeout()
        assert F.vggt_get_device_status() == -6
        assert F.vggt_get_device_status() == 0  # cleared by the read
    finally:
        F.vggt_set_wait_limit(prev)
    check_attention(F, "global", 1, 15, 1, seed=17)


def _head_major(x: torch.Tensor) -> torch.Tensor:
    """[N, H, D] token-major -> [H, N, D] head-major, contiguous."""
    return x.permute(1, 0, 2).contiguous()


def test_core_scores_at_the_norm_bound(F):
    # The kernel takes exp(score) with no row maximum subtracted; the LayerNorm
    # caps |q_hat| and |k_hat| at 8, so the scores of prologue outputs lie in
    # [-8, 8]. Sweep the keys across that whole range: every query is 7.99 u
    # (u a unit vector per head) and key j is 7.99 (cos a_j u + sin a_j w_j)
    # with a_j evenly spaced in [0, pi] and w_j orthogonal to u, so the
    # scores run from +7.98 to -7.98 and one row's weights span e^16
    # (about 2^23). The oracle's max-subtracted softmax must agree.
    gen = torch.Generator().manual_seed(31)
    H, nq, nk = 2, 200, 520
    u = torch.randn(H, 64, generator=gen, dtype=torch.float64)
    u = u / u.norm(dim=-1, keepdim=True)
    w = torch.randn(nk, H, 64, generator=gen, dtype=torch.float64)
    w = w - (w * u).sum(-1, keepdim=True) * u
    w = w / w.norm(dim=-1, keepdim=True)
    a = torch.linspace(0.0, np.pi, nk, dtype=torch.float64)[:, None, None]
    qh = (7.99 * u).expand(nq, H, 64).to(torch.bfloat16)
    kh = (7.99 * (torch.cos(a) * u + torch.sin(a) * w)).to(torch.bfloat16)
    v = torch.randn(nk, H, 64, generator=gen).to(torch.bfloat16)
    out = torch.empty(nq, H, 64, dtype=torch.bfloat16, device="cuda")
    F.vggt_attn_core(_head_major(qh).cuda(), _head_major(kh).cuda(), v.cuda(), out, 1, nq, nk, H=H)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    ref = O.cross_attention(f64(qh), f64(kh), f64(v))
    s_max = float((f64(qh)[0] * f64(kh)).sum(-1).max() / 8.0)
    assert s_max > 7.9  # the sweep really reaches the edge
    mx, rf = errors(f64(out.cpu()), ref)
    assert mx <= MAX_ABS and rf <= REL_FRO, (mx, rf)


def test_core_reports_inputs_beyond_the_norm_bound(F):
    # Vectors far outside the core's bound (norm ~1600): the exponentials
    # overflow, the kernel flags it in the status word without faulting, and
    # the next read finds the word clear again.
    S, g = 1, 10
    q, k, v, pos = synth.make_qkv(S, g, seed=32)
    qd, kd_, vd, pd = (t.cuda() for t in (q, k, v, pos))
    qh = F.vggt_qk_prologue(qd, pd)
    kh = F.vggt_qk_prologue(kd_, pd)
    out = torch.empty_like(qd)
    F.vggt_attn_core((qh.float() * 200.0).to(torch.bfloat16), kh, vd, out, 1, qd.shape[0], qd.shape[0])
    assert F.vggt_get_device_status() == -7
    assert F.vggt_get_device_status() == 0
    check_attention(F, "global", 1, 10, 1, seed=32)


def test_scratch_pool_release_and_reuse(F):
    # Scratch comes from the library's pool, which keeps it between calls;
    # vggt_release_scratch hands it back and later calls take it again. The
    # results do not depend on where the scratch came from.
    S, g, kd = 3, 9, 3
    q, k, v, pos = synth.make_qkv(S, g, seed=33)
    T = 5 + g * g
    a = run_gpu(F, "descriptor", q, k, v, pos, S, T, kd)
    b = run_gpu(F, "global", q, k, v, pos, S, T, 1)
    torch.cuda.synchronize()
    F.vggt_release_scratch()
    F.vggt_release_scratch()  # nothing left to release: still fine
    assert torch.equal(run_gpu(F, "descriptor", q, k, v, pos, S, T, kd), a)
    assert torch.equal(run_gpu(F, "global", q, k, v, pos, S, T, 1), b)


# ------------------------------------------------------ streaming descriptors


def _stream_gpu(F, q, k, v, pos, S, T, kd, chunk, H=16):
    """Feed the scene chunk by chunk through one descriptor cache."""
    dev = torch.device("cuda:0")
    qd, kd_, vd, pd = (t.to(dev) for t in (q, k, v, pos))
    out = torch.empty_like(qd)
    with F.DescCache(S, T, H=H, kv_down=kd) as cache:
        for f0 in range(0, S, chunk):
            c = min(chunk, S - f0)
            r0, r1 = f0 * T, (f0 + c) * T
            cache.attend(qd[r0:r1], kd_[r0:r1], vd[r0:r1], pd[r0:r1], out[r0:r1], C=c)
            assert cache.frames == f0 + c
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    return out.cpu()


@pytest.mark.parametrize("S,g,kd,chunk", [(6, 9, 3, 2), (5, 11, 4, 2), (4, 6, 1, 3), (3, 7, 2, 1)])
def test_stream_chunks_match_oracle(F, S, g, kd, chunk):
    q, k, v, pos = synth.make_qkv(S, g, seed=50 + S)
    T = 5 + g * g
    got = f64(_stream_gpu(F, q, k, v, pos, S, T, kd, chunk))
    ref = O.attn_descriptor_stream(f64(q), f64(k), f64(v), pos.numpy().astype(np.float64), S, T, kd, chunk)
    mx, rf = errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= MAX_ABS and rf <= REL_FRO, (S, g, kd, chunk, mx, rf)


def test_stream_single_chunk_equals_descriptor_call(F):
    S, g, kd = 4, 10, 3
    q, k, v, pos = synth.make_qkv(S, g, seed=60)
    T = 5 + g * g
    a = _stream_gpu(F, q, k, v, pos, S, T, kd, S)
    b = run_gpu(F, "descriptor", q, k, v, pos, S, T, kd)
    assert torch.equal(a, b)


def test_stream_cache_capacity_and_reset(F):
    S, g, kd = 3, 6, 2
    q, k, v, pos = (t.cuda() for t in synth.make_qkv(S, g, seed=61))
    T = 5 + g * g
    out1 = torch.empty_like(q)
    out2 = torch.empty_like(q)
    with F.DescCache(2, T, kv_down=kd) as cache:
        cache.attend(q[:2 * T], k[:2 * T], v[:2 * T], pos[:2 * T], out1[:2 * T], C=2)
        with pytest.raises(F.VggtError):
            cache.attend(q[2 * T:], k[2 * T:], v[2 * T:], pos[2 * T:], out1[2 * T:], C=1)  # 3 > 2 frames
        assert cache.frames == 2
        cache.reset()
        assert cache.frames == 0
        cache.attend(q[:2 * T], k[:2 * T], v[:2 * T], pos[:2 * T], out2[:2 * T], C=2)
    torch.cuda.synchronize()
    assert torch.equal(out1[:2 * T], out2[:2 * T])


def test_stream_full_size_sampled_rows(F):
    # The descriptor workload's scene (200 frames of 1374 tokens, 4x4 pooling)
    # streamed in chunks of 10 frames, checked on rows sampled across chunks.
    w = synth.WORKLOADS["descriptor_s200_g37_kd4"]
    q, k, v, pos = synth.make_workload(w, 1)
    got = _stream_gpu(F, q, k, v, pos, w.S, w.T, w.kv_down, 10)
    rows = synth.sample_rows(w.n_q, 160, seed=5).numpy()
    ref = O.attn_descriptor_stream(f64(q), f64(k), f64(v), pos.numpy().astype(np.float64), w.S, w.T,
                                   w.kv_down, 10, rows=rows)
    mx, rf = errors(f64(got)[rows], ref)
    assert mx <= MAX_ABS and rf <= REL_FRO, (mx, rf)


def test_frame_attention_at_the_token_limit(F):
    # the largest call the library accepts: 1526 frames of 1374 tokens =
    # 2 096 724 tokens <= VGGT_MAX_TOKENS (2^21); rows sampled over all frames,
    # the first and the last row included
    S, g = 1526, 37
    T = 5 + g * g
    assert S * T <= 1 << 21 < (S + 1) * T
    q, k, v, pos = synth.make_qkv(S, g, seed=9)
    dev = torch.device("cuda:0")
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    F.vggt_attn_frame(q.to(dev), k.to(dev), v.to(dev), pos.to(dev), out, S=S, T=T)
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    rows = synth.sample_rows(S * T, 256, seed=11).numpy()
    # the oracle needs only the frames the sampled rows live in
    frames = np.unique(rows // T)
    sel = np.concatenate([np.arange(f * T, (f + 1) * T) for f in frames])
    remap = {f: i for i, f in enumerate(frames)}
    local_rows = np.array([remap[r // T] * T + r % T for r in rows])
    ref = O.attn_frame(f64(q[torch.from_numpy(sel)]), f64(k[torch.from_numpy(sel)]),
                       f64(v[torch.from_numpy(sel)]), pos.numpy()[sel].astype(np.float64),
                       frames.size, T, rows=local_rows)
    got = f64(out.cpu()[torch.from_numpy(rows)])
    mx, rf = errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= MAX_ABS and rf <= REL_FRO, (mx, rf)


@pytest.mark.parametrize("kind", ["global", "frame", "descriptor", "noalloc"])
def test_calls_replay_from_a_cuda_graph(F, kind):
    # every call is stream-ordered and allocates from a stream-ordered pool,
    # so it can be captured into a CUDA graph; a replay repeats the call
    S, g = 2, 16
    T = 5 + g * g
    q, k, v, pos = (t.cuda() for t in synth.make_qkv(S, g, seed=21))
    fn = {"global": F.vggt_attn_global, "frame": F.vggt_attn_frame, "descriptor": F.vggt_attn_descriptor,
          "noalloc": F.vggt_attn_global_noalloc}[kind]
    kd = 3 if kind == "descriptor" else 0
    ref = fn(q, k, v, pos, S=S, T=T, kv_down=kd)
    torch.cuda.synchronize()
    out = torch.empty_like(q)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        fn(q, k, v, pos, out, S=S, T=T, kv_down=kd, stream=side)
    for _ in range(3):
        out.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert F.vggt_get_device_status() == 0
    assert torch.equal(out, ref)
