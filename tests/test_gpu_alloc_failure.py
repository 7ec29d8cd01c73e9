"""The scratch-allocation failure path (VGGT_ERR_ALLOC), forced on the host:
a fresh process caps the library's scratch pool with
VGGT_SCRATCH_POOL_MAX_BYTES, so that calls needing more scratch than the cap
fail to allocate. Such a call must return VGGT_ERR_ALLOC, launch nothing
(the output keeps its sentinel, the status word stays clear) and leave the
library usable: a call that fits under the cap still succeeds."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CAP = 32 << 20

_SCRIPT = r"""
import json, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import feed_forward_view_b200 as F
import synth
from oracle import vggt_oracle as O

E_ALLOC = -4
cap = int(sys.argv[2])

def f64(t):
    b = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return O.bf16_bits_to_f64(b).reshape(t.shape)

results = []
# global attention over 9 frames of 4101 tokens: 151 MB of scratch > cap
q, k, v, pos = (t.cuda() for t in synth.make_qkv(9, 64, 0))
out = torch.full_like(q, 7.0)
rc = F.lib.vggt_attn_global(*(t.data_ptr() for t in (q, k, v, pos, out)), 9, 4101, 16, 64, 1, F._stream(None))
torch.cuda.synchronize()
results.append(["global", rc, F.vggt_get_device_status(), bool((out.float() == 7.0).all())])
# descriptor attention: 40 frames of 1374 tokens, kd 4 (about 200 MB of scratch)
del q, k, v, pos, out
q, k, v, pos = (t.cuda() for t in synth.make_qkv(40, 37, 1))
out = torch.full_like(q, 7.0)
rc = F.lib.vggt_attn_descriptor(*(t.data_ptr() for t in (q, k, v, pos, out)), 40, 1374, 16, 64, 4, F._stream(None))
torch.cuda.synchronize()
results.append(["descriptor", rc, F.vggt_get_device_status(), bool((out.float() == 7.0).all())])
exists, reserved = F.vggt_scratch_pool_info()
# a call that fits under the cap still works, and matches the oracle
q, k, v, pos = (t.cuda() for t in synth.make_qkv(2, 16, 2))
out = torch.empty_like(q)
rc = F.lib.vggt_attn_global(*(t.data_ptr() for t in (q, k, v, pos, out)), 2, 261, 16, 64, 1, F._stream(None))
torch.cuda.synchronize()
ref = O.attn_global(f64(q), f64(k), f64(v), pos.cpu().numpy().astype(np.float64), 2, 261)
err = float(np.abs(f64(out) - ref).max())
results.append(["small", rc, F.vggt_get_device_status(), err <= 2e-2])
exists2, reserved2 = F.vggt_scratch_pool_info()
print("RESULT " + json.dumps({"results": results, "pool": [exists, reserved, exists2, reserved2]}))
"""


def test_calls_beyond_the_pool_cap_return_alloc_and_launch_nothing():
    env = dict(os.environ, VGGT_SCRATCH_POOL_MAX_BYTES=str(CAP))
    res = subprocess.run([sys.executable, "-c", _SCRIPT, ROOT, str(CAP)], capture_output=True, text=True,
                         timeout=600, env=env)
    assert res.returncode == 0, res.stderr[-3000:]
    line = [ln for ln in res.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    got = json.loads(line[len("RESULT "):])
    results = got["results"]
    exists, reserved, exists2, reserved2 = got["pool"]
    assert results[0] == ["global", -4, 0, True], results
    assert results[1] == ["descriptor", -4, 0, True], results
    assert results[2] == ["small", 0, 0, True], results
    assert exists and exists2
    assert reserved <= CAP and reserved2 <= CAP, (reserved, reserved2)
