"""Host-side checks of the C ABI that need no GPU: the library loads, exports
exactly what include/vggt_attn.h declares, and rejects invalid arguments
before touching the device."""
import os
import re
import subprocess

import pytest

import feed_forward_view_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vggt_attn.h")

OK, E_NULL, E_UNSUP, E_SHAPE = 0, -1, -2, -3


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"VGGT_API\s+[\w\s\*]+?\b(vggt_\w+)\s*\(", src))


def test_header_declares_the_binding_symbols():
    assert declared_functions() == set(F.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol_and_nothing_else():
    out = subprocess.run(["nm", "-D", "--defined-only", F.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    text_syms = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert declared_functions() <= text_syms
    assert all(s.startswith("vggt_") for s in text_syms), text_syms
    for name in declared_functions():
        assert hasattr(F.lib, name)


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert F.vggt_status_string(code).startswith("VGGT_")
    assert "unknown" in F.vggt_status_string(7)


def test_pool_token_counts():
    assert F.vggt_kv_pool_tokens(1374, 4) == 105
    assert F.vggt_kv_pool_tokens(1374, 1) == 1374
    assert F.vggt_kv_pool_tokens(4101, 4) == 5 + 16 * 16
    assert F.vggt_kv_pool_tokens(261, 3) == 5 + 36
    assert F.vggt_kv_pool_tokens(5, 4) == 5
    assert F.vggt_kv_pool_tokens(930, 4) == E_SHAPE  # 25x37 is not square
    assert F.vggt_kv_pool_tokens(1374, 0) == E_SHAPE
    assert F.vggt_kv_pool_tokens(4, 1) == E_SHAPE


ATTN = ("vggt_attn_frame", "vggt_attn_global", "vggt_attn_descriptor")
FAKE = 0x1000  # never dereferenced: every case below fails validation first


@pytest.mark.parametrize("name", ATTN)
def test_attention_argument_checks(name):
    fn = getattr(F.lib, name)
    kd = 4 if name == "vggt_attn_descriptor" else 1
    p = [FAKE] * 5
    assert fn(*p, 2, 261, 16, 32, kd, None) == E_UNSUP
    assert fn(*p, 2, 262, 16, 64, kd, None) == E_SHAPE      # T - 5 not a square
    assert fn(*p, 2, 4, 16, 64, kd, None) == E_SHAPE        # fewer than 5 tokens
    assert fn(*p, -1, 261, 16, 64, kd, None) == E_SHAPE
    assert fn(*p, 2, 261, -1, 64, kd, None) == E_SHAPE
    assert fn(*p, 1 << 20, 261, 16, 64, kd, None) == E_SHAPE  # beyond VGGT_MAX_TOKENS
    for i in range(5):
        q = list(p)
        q[i] = None
        assert fn(*q, 2, 261, 16, 64, kd, None) == E_NULL
    for i in range(5):
        q = list(p)
        q[i] = FAKE + (4 if i == 3 else 8)  # bf16 arrays need 16 bytes, positions 8
        assert fn(*q, 2, 261, 16, 64, kd, None) == E_UNSUP
    # empty problems succeed without touching any pointer
    assert fn(None, None, None, None, None, 0, 261, 16, 64, kd, None) == OK
    assert fn(None, None, None, None, None, 3, 261, 0, 64, kd, None) == OK


def test_kv_down_rules():
    p = [FAKE] * 5
    assert F.lib.vggt_attn_frame(*p, 2, 261, 16, 64, 2, None) == E_SHAPE
    assert F.lib.vggt_attn_global(*p, 2, 261, 16, 64, 4, None) == E_SHAPE
    assert F.lib.vggt_attn_descriptor(*p, 2, 261, 16, 64, 0, None) == E_SHAPE


def test_pool_and_prologue_argument_checks():
    p6 = [FAKE] * 6
    assert F.lib.vggt_kv_pool(*p6, 2, 261, 16, 32, 4, None) == E_UNSUP
    assert F.lib.vggt_kv_pool(*p6, 2, 262, 16, 64, 4, None) == E_SHAPE
    assert F.lib.vggt_kv_pool(*p6, 2, 261, 16, 64, 0, None) == E_SHAPE
    assert F.lib.vggt_kv_pool(None, *p6[1:], 2, 261, 16, 64, 4, None) == E_NULL
    assert F.lib.vggt_kv_pool(None, None, None, None, None, None, 0, 261, 16, 64, 4, None) == OK
    assert F.lib.vggt_qk_prologue(FAKE, FAKE, FAKE, 10, 16, 48, None) == E_UNSUP
    assert F.lib.vggt_qk_prologue(FAKE, FAKE, FAKE, -1, 16, 64, None) == E_SHAPE
    assert F.lib.vggt_qk_prologue(FAKE, None, FAKE, 10, 16, 64, None) == E_NULL
    assert F.lib.vggt_qk_prologue(None, None, None, 0, 16, 64, None) == OK


def test_core_argument_checks():
    for name in ("vggt_attn_core", "vggt_attn_core_online"):
        _core_checks(getattr(F.lib, name))


def _core_checks(fn):
    p = [FAKE] * 4
    assert fn(*p, 1, 100, 100, 16, 32, None) == E_UNSUP
    assert fn(*p, -1, 100, 100, 16, 64, None) == E_SHAPE
    assert fn(*p, 1, 1 << 22, 100, 16, 64, None) == E_SHAPE
    assert fn(None, *p[1:], 1, 100, 100, 16, 64, None) == E_NULL
    assert fn(FAKE + 4, *p[1:], 1, 100, 100, 16, 64, None) == E_UNSUP
    assert fn(None, None, None, None, 1, 0, 100, 16, 64, None) == OK


def test_binding_rejects_host_tensors():
    import torch

    q = torch.zeros(261 * 2, 16, 64, dtype=torch.bfloat16)
    pos = torch.zeros(261 * 2, 2)
    with pytest.raises(ValueError):
        F.vggt_attn_global(q, q, q, pos, q.clone(), S=2, T=261)


def test_descriptor_cache_argument_checks():
    import ctypes

    h = ctypes.c_void_p()
    create = F.lib.vggt_desc_cache_create
    assert create(None, 4, 41, 16, 64, 4) == E_NULL
    assert create(ctypes.byref(h), 0, 41, 16, 64, 4) == E_SHAPE and not h.value
    assert create(ctypes.byref(h), 4, 40, 16, 64, 4) == E_SHAPE  # 40 - 5 is not a square
    assert create(ctypes.byref(h), 4, 41, 16, 64, 0) == E_SHAPE
    assert create(ctypes.byref(h), 4, 41, 16, 32, 4) == E_UNSUP
    assert create(ctypes.byref(h), 1 << 20, 1374, 16, 64, 4) == E_SHAPE  # beyond VGGT_MAX_TOKENS
    assert F.lib.vggt_desc_cache_frames(None) == E_NULL
    assert F.lib.vggt_desc_cache_reset(None) == E_NULL
    assert F.lib.vggt_desc_cache_destroy(None) == OK
    fake = ctypes.c_void_p(0x1000)
    assert F.lib.vggt_attn_descriptor_chunk(None, fake, fake, fake, fake, fake, 1, None) == E_NULL


# ----------------------------------------------------------------- _ex calls (layouts, LN affine)


def test_pool_token_counts_for_layouts():
    assert F.vggt_kv_pool_tokens_ex(5 + 25 * 37, 4, (5, 25, 37, 0)) == 5 + 7 * 10
    assert F.vggt_kv_pool_tokens_ex(32 * 32 + 16, 4, (0, 32, 32, 16)) == 64 + 16
    assert F.vggt_kv_pool_tokens_ex(1374, 4, None) == 105
    assert F.vggt_kv_pool_tokens_ex(1374, 4, (5, 37, 37, 0)) == 105
    assert F.vggt_kv_pool_tokens_ex(2 + 3 * 5 + 3, 2, (2, 3, 5, 3)) == 2 + 6 + 3
    assert F.vggt_kv_pool_tokens_ex(5 + 25 * 37, 4, (5, 37, 25, 1)) == E_SHAPE  # does not add up to T
    assert F.vggt_kv_pool_tokens_ex(10, 4, (-1, 3, 3, 2)) == E_SHAPE
    assert F.vggt_kv_pool_tokens_ex(10, 0, (1, 3, 3, 0)) == E_SHAPE


def _ex_call(fn, T, ln=None, layout=None, kd=None, S=0):
    """An empty problem (S = 0): validation runs, nothing is launched."""
    norm, keep = F._norm(ln)
    if fn is F.lib.vggt_attn_descriptor_ex:
        return fn(FAKE, FAKE, FAKE, FAKE, FAKE, S, T, 16, 64, 4 if kd is None else kd, F._layout(layout), norm, None)
    return fn(FAKE, FAKE, FAKE, FAKE, FAKE, S, T, 16, 64, norm, None)


def test_ex_frame_and_global_take_any_frame_length():
    for plain, ex in ((F.lib.vggt_attn_frame, F.lib.vggt_attn_frame_ex),
                      (F.lib.vggt_attn_global, F.lib.vggt_attn_global_ex)):
        assert plain(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 100, 16, 64, 0, None) == E_SHAPE
        assert _ex_call(ex, 100) == OK
        assert _ex_call(ex, 0) == E_SHAPE
        assert ex(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 100, 16, 32, None, None) == E_UNSUP


def test_ex_descriptor_layout_checks():
    d = F.lib.vggt_attn_descriptor_ex
    assert _ex_call(d, 5 + 25 * 37, layout=(5, 25, 37, 0)) == OK
    assert _ex_call(d, 5 + 25 * 37) == E_SHAPE              # default layout wants a square grid
    assert _ex_call(d, 5 + 25 * 37, layout=(5, 25, 36, 0)) == E_SHAPE
    assert _ex_call(d, 1374, kd=0) == E_SHAPE


def test_ln_affine_any_finite_values():
    # Any finite affine is accepted (large ones run the online softmax); only
    # non-finite weights or biases are refused.
    g = F.lib.vggt_attn_global_ex
    w = lambda c: [c] * 64  # noqa: E731
    assert _ex_call(g, 100, ln=(w(2.0), None, w(2.0), None)) == OK
    assert _ex_call(g, 100, ln=(w(2.4), None, w(2.4), None)) == OK
    assert _ex_call(g, 100, ln=(w(-60.0), w(8.0), w(40.0), w(-3.0))) == OK
    assert _ex_call(g, 100, ln=(w(1e30), None, None, None)) == OK
    assert _ex_call(g, 100, ln=(w(float("nan")), None, None, None)) == E_UNSUP
    assert _ex_call(g, 100, ln=(None, None, None, w(float("inf")))) == E_UNSUP
    assert _ex_call(g, 100, ln=(None, w(float("-inf")), None, None)) == E_UNSUP
    one_nan = w(1.0)
    one_nan[37] = float("nan")
    assert _ex_call(g, 100, ln=(None, None, one_nan, None)) == E_UNSUP
    # the prologue alone has no score bound, only finiteness
    wp, keep = F._host_f32(w(50.0), "w")
    assert F.lib.vggt_qk_prologue_ex(FAKE, FAKE, FAKE, 0, 16, 64, wp, None, None) == OK
    nanp, keep2 = F._host_f32(w(float("nan")), "w")
    assert F.lib.vggt_qk_prologue_ex(FAKE, FAKE, FAKE, 0, 16, 64, nanp, None, None) == E_UNSUP


def test_descriptor_keys_and_pool_ex_argument_checks():
    lay = F._layout((5, 25, 37, 0))
    T = 5 + 25 * 37
    k = F.lib.vggt_descriptor_keys
    assert k(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, T, 16, 64, 4, lay, None, None, None) == OK
    assert k(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, T, 16, 64, 4, None, None, None, None) == E_SHAPE
    assert k(FAKE, FAKE, FAKE, None, FAKE, FAKE, 1, T, 16, 64, 4, lay, None, None, None) == E_NULL
    assert k(FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, 1, T, 16, 64, 4, lay, None, None, None) == E_UNSUP
    p = F.lib.vggt_kv_pool_ex
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, T, 16, 64, 4, lay, None) == OK
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, T, 16, 64, 4, None, None) == E_SHAPE
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, T, 16, 64, 0, lay, None) == E_SHAPE


def test_descriptor_cache_ex_checks_before_allocating():
    import ctypes
    h = ctypes.c_void_p()
    c = F.lib.vggt_desc_cache_create_ex
    assert c(ctypes.byref(h), 10, 5 + 25 * 37, 16, 64, 4, None, None) == E_SHAPE
    assert not h.value
    norm, keep = F._norm(([3.0] * 64, None, [float("nan")] * 64, None))
    assert c(ctypes.byref(h), 10, 5 + 25 * 37, 16, 64, 4, F._layout((5, 25, 37, 0)), norm) == E_UNSUP
    assert not h.value


def test_subset_argument_checks():
    s = F.lib.vggt_attn_subset
    args = lambda S, T, skip, E, H=16, D=64, g=1: (FAKE, FAKE, FAKE, FAKE, FAKE, S, T, skip, E, H, D, g, None, None)  # noqa: E731
    assert s(*args(0, 1040, 16, 5, g=0)) == OK         # frame attention of no frames (the sequence
                                                       # tokens take no part in frame attention)
    assert s(*args(2, 10, 10, 0)) == OK                # every frame token left out, no sequence tokens
    assert s(*args(2, 10, 11, 0)) == E_SHAPE
    assert s(*args(2, 10, -1, 0)) == E_SHAPE
    assert s(*args(2, 10, 0, -1)) == E_SHAPE
    assert s(*args(2, 0, 0, 0)) == E_SHAPE
    assert s(*args(2, 10, 0, 0, g=2)) == E_SHAPE
    assert s(*args(2, 10, 0, 0, D=32)) == E_UNSUP
    assert s(*args(2, 10, 0, 0, H=0)) == OK
    assert s(FAKE, None, FAKE, FAKE, FAKE, 2, 10, 0, 0, 16, 64, 1, None, None) == E_NULL
    assert s(FAKE, FAKE, FAKE + 8, FAKE, FAKE, 2, 10, 0, 0, 16, 64, 1, None, None) == E_UNSUP
    norm, keep = F._norm(([3.0] * 64, None, [float("inf")] * 64, None))
    assert s(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 10, 0, 0, 16, 64, 1, norm, None) == E_UNSUP


def test_f32_mode_argument_checks():
    for name in ("vggt_attn_frame_f32", "vggt_attn_global_f32"):
        fn = getattr(F.lib, name)
        for terms in (2, 3):
            assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 100, 16, 64, None, terms, None) == OK
            assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 0, 16, 64, None, terms, None) == E_SHAPE
            assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 10, 16, 32, None, terms, None) == E_UNSUP
            assert fn(FAKE, None, FAKE, FAKE, FAKE, 2, 10, 16, 64, None, terms, None) == E_NULL
            assert fn(FAKE, FAKE, FAKE + 8, FAKE, FAKE, 2, 10, 16, 64, None, terms, None) == E_UNSUP
            norm, keep = F._norm(([3.0] * 64, [float("nan")] * 64, None, None))
            assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 10, 16, 64, norm, terms, None) == E_UNSUP
        for terms in (0, 1, 4, -1):  # only two or three bf16 terms
            assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 10, 16, 64, None, terms, None) == E_UNSUP
            assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 10, 16, 64, None, terms, None) == E_UNSUP


def test_batch_argument_checks():
    g, d = F.lib.vggt_attn_global_batch, F.lib.vggt_attn_descriptor_batch
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 261, 16, 64, None, None) == OK
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 3, 0, 261, 16, 64, None, None) == OK
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 261, 16, 64, None, None) == E_SHAPE
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 12, 1 << 10, 261, 16, 64, None, None) == E_SHAPE  # too many tokens
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 2, 261, 16, 32, None, None) == E_UNSUP
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 261, 16, 64, 4, None, None, None) == OK
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 260, 16, 64, 4, None, None, None) == E_SHAPE  # not 5 + g*g
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 261, 16, 64, 0, None, None, None) == E_SHAPE


def test_noalloc_argument_checks():
    na = F.lib.vggt_attn_global_noalloc
    p = [FAKE] * 5
    assert na(*p, 1, 4101, 16, 64, 0, None) == E_SHAPE       # 16.8 MB of scratch > the 16 MiB array
    assert na(*p, 2, 261, 16, 32, 0, None) == E_UNSUP
    assert na(*p, 2, 262, 16, 64, 0, None) == E_SHAPE        # T - 5 not a square
    assert na(*p, 2, 261, 16, 64, 2, None) == E_SHAPE        # kv_down
    assert na(None, None, None, None, None, 0, 261, 16, 64, 0, None) == OK
    # token counts beyond the library's limit are rejected before the byte
    # count is formed (which could wrap for sizes near 2^31)
    big = 2 ** 31 - 1
    assert na(*p, big, 5 + 215 * 215, 1, 64, 0, None) == E_SHAPE
    assert na(*p, big, 5 + 46340 * 46340, 65535, 64, 0, None) == E_SHAPE


def test_scratch_pool_info_needs_its_pointers():
    import ctypes
    e, r = ctypes.c_int(7), ctypes.c_ulonglong(7)
    assert F.lib.vggt_scratch_pool_info(None, ctypes.byref(r)) == E_NULL
    assert F.lib.vggt_scratch_pool_info(ctypes.byref(e), None) == E_NULL
