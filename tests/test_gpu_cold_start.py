"""The first decode call of a fresh process, where the CTAs' start times are
spread out: a 8192x8192 projection at one token is cut into K slices, so
each CTA's fixed range ends after a few boxes and the rest of the items are
handed out through the work counter.  A CTA whose fixed range had filled
the box ring before it waited for the preceding grid (the quantizer) must
still load that range's activations before it takes a shared item; the
test runs the call in a new interpreter, compares every output with an exact
product of the generator's ternary matrix and the oracle's int8 codes, and
checks that no device-side wait ran out.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
import numpy as np
import torch
sys.path.insert(0, {root!r})
import oracle
from i2_mpgemm_b200 import i2s, inputs
n, k, seed = {n}, {k}, {seed}
w, t, _ = inputs.ternary_weights(n, k, seed)
x = inputs.activations(1, k, seed)
d_packed = i2s.bitnet_i2s_pack(w.cuda())
y, acc = i2s.bitnet_i2s_quant_gemv(d_packed, n, k, x.cuda(), want_acc=True)
xq, xs = oracle.act_quant(x.numpy())
want = (xq.astype(np.float64) @ t.numpy().astype(np.float64).T).astype(np.int64)
bad = int(np.count_nonzero(acc.cpu().numpy() != want.astype(np.int32)))
i2s.bitnet_device_status()
print("bad", bad)
sys.exit(1 if bad else 0)
"""


@pytest.mark.parametrize("n,k,seed", [(8192, 8192, 31), (2560, 6912, 32), (640, 2560, 33)])
def test_first_call_in_a_fresh_process(n, k, seed):
    code = SCRIPT.format(root=ROOT, n=n, k=k, seed=seed)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
