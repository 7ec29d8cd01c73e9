"""vggt_attn_global_noalloc: global attention whose scratch comes from the
library's fixed device array instead of an allocation, for callers that may
not allocate device memory while they run (fixed start-up memory budgets, no
stream-ordered allocator). Called through the C ABI with raw pointers and
checked against vggt_attn_global, the allocating entry point, on two calls in
a row with different inputs -- the second call must not see anything left in
the shared array by the first -- and against the fp64 oracle on the same
inputs."""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import synth
from oracle import vggt_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3
E_SHAPE = -3


def _c_call(lib, fn_name, q, k, v, pos, out, S, T, H=16, D=64):
    fn = getattr(lib, fn_name)
    stream = torch.cuda.current_stream().cuda_stream
    return fn(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
              ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(out.data_ptr()), S, T, H, D, 0,
              ctypes.c_void_p(stream))


def _errors(a: torch.Tensor, b: torch.Tensor):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    d = a - b
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(b), 1e-30))


def _f64(t: torch.Tensor) -> np.ndarray:
    b = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return O.bf16_bits_to_f64(b).reshape(t.shape)


def test_noalloc_matches_allocating_entry_point_on_two_calls():
    import feed_forward_view_b200 as F

    cases = [(2, 16, 21), (3, 20, 22)]  # 522 and 1215 tokens; different inputs per call
    for S, g, seed in cases:
        q, k, v, pos = (t.cuda() for t in synth.make_qkv(S, g, seed))
        T = 5 + g * g
        out_na = torch.full_like(q, float("nan"))
        out_ref = torch.empty_like(q)
        assert _c_call(F.lib, "vggt_attn_global_noalloc", q, k, v, pos, out_na, S, T) == 0
        assert _c_call(F.lib, "vggt_attn_global", q, k, v, pos, out_ref, S, T) == 0
        torch.cuda.synchronize()
        assert F.vggt_get_device_status() == 0
        assert torch.isfinite(out_na.float()).all()
        mx, rf = _errors(out_na, out_ref)
        assert mx <= MAX_ABS and rf <= REL_FRO, (S, g, mx, rf)
        # and against the oracle, like every other entry point
        ref = O.attn_global(_f64(q), _f64(k), _f64(v), pos.cpu().numpy().astype(np.float64), S, T)
        got = _f64(out_na)
        d = got - ref
        mx, rf = float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(ref))
        assert mx <= MAX_ABS and rf <= REL_FRO, ("oracle", S, g, mx, rf)


def test_noalloc_rejects_sizes_beyond_its_array():
    import feed_forward_view_b200 as F

    limit = F.lib.vggt_attn_global_noalloc
    fake = ctypes.c_void_p(0x1000)
    # 4101 tokens x 16 heads x 64 dims x 2 B, for q and k: 16.8 MB > 16 MiB.
    # Rejected before any launch (the fake pointers are never touched).
    assert limit(fake, fake, fake, fake, fake, 1, 4101, 16, 64, 0, None) == E_SHAPE
    # S*T beyond the library's token limit, whose byte count would wrap a
    # 64-bit product if it were formed first: rejected as well.
    big = 2 ** 31 - 1
    assert limit(fake, fake, fake, fake, fake, big, 5 + 215 * 215, 1, 64, 0, None) == E_SHAPE
    assert limit(fake, fake, fake, fake, fake, big, 5 + 46340 * 46340, 65535, 64, 0, None) == E_SHAPE


_FRESH_FIRST_CALL = r"""
import ctypes, sys
import torch
sys.path.insert(0, sys.argv[1])
import feed_forward_view_b200 as F
import synth
q, k, v, pos = (t.cuda() for t in synth.make_qkv(2, 16, 5))
out = torch.empty_like(q)
s = torch.cuda.current_stream().cuda_stream
rc = F.lib.vggt_attn_global_noalloc(*(ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, pos, out)),
                                    2, 261, 16, 64, 0, ctypes.c_void_p(s))
torch.cuda.synchronize()
exists, reserved = F.vggt_scratch_pool_info()
print(rc, F.vggt_get_device_status(), int(exists), reserved, bool(torch.isfinite(out.float()).all()))
"""


def test_noalloc_first_call_in_a_fresh_process_creates_no_pool():
    # The no-alloc call as the first library call of a process: it succeeds
    # and leaves the library's scratch pool uncreated (it needs only the status
    # word's address and its own array's).
    res = subprocess.run([sys.executable, "-c", _FRESH_FIRST_CALL, ROOT], capture_output=True, text=True,
                         timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    rc, status, exists, reserved, finite = res.stdout.split()[-5:]
    assert (rc, status, exists, reserved, finite) == ("0", "0", "0", "0", "True"), res.stdout
