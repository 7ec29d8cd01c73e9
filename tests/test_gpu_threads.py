"""Host threads calling the library at once, from a fresh process so that the
per-device set-up (status word, scratch pool, kernel attributes) happens
inside the race: every thread's result must equal a single-threaded call."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import threading
import torch
import feed_forward_view_b200 as F
import synth

n = 4
q, k, v, pos = (t.cuda() for t in synth.make_qkv(S=2, g=16, seed=0))
T = q.shape[0] // 2
torch.cuda.synchronize()
streams = [torch.cuda.Stream() for _ in range(n)]
outs = [torch.zeros_like(q) for _ in range(n)]
outs32 = [None] * n
q32, k32, v32 = (t.float() for t in (q, k, v))
torch.cuda.synchronize()
start = threading.Barrier(n)
errors = []


def run(i):
    try:
        start.wait()
        with torch.cuda.stream(streams[i]):
            F.vggt_attn_global(q, k, v, pos, out=outs[i], S=2, T=T)
            outs32[i] = F.vggt_attn_frame_f32(q32, k32, v32, pos, S=2, T=T, terms=2 + i % 2)
    except Exception as e:  # reported below
        errors.append(repr(e))


threads = [threading.Thread(target=run, args=(i,)) for i in range(n)]
for t in threads:
    t.start()
for t in threads:
    t.join()
torch.cuda.synchronize()
assert not errors, errors
ref = F.vggt_attn_global(q, k, v, pos, S=2, T=T)
ref32 = {t: F.vggt_attn_frame_f32(q32, k32, v32, pos, S=2, T=T, terms=t) for t in (2, 3)}
torch.cuda.synchronize()
for i in range(n):
    assert torch.equal(outs[i], ref), i
    assert torch.equal(outs32[i], ref32[2 + i % 2]), i
assert F.vggt_get_device_status() == 0
print("threads ok")
"""


def test_first_calls_from_several_threads():
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "threads ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
