"""First calls from several host threads at once.

The library keeps per-device caches (SM count, kernel attributes, cluster
occupancy, symbol addresses) as atomics filled on first use.  In a fresh
process, eight host threads start together (a barrier releases them) and
each makes its first hbl_forward on its own stream, with its own inputs, on
paths that fill different caches (the decode-sized kernel, the split-K,
1-SM and 2-SM GEMMs, INT4 and INT8).  Every result must equal the oracle's
GEMM and dequantisation of the library's own codes, and the codes must be
the oracle's quantizer applied to the library's own transform output.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import sys, threading
sys.path.insert(0, ROOT)
import numpy as np
import torch
import ternary_gemm_b200 as H
import oracle
from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x
oracle.build()
torch.cuda.init()
cases = [(1, 4096, 4096, 4), (16, 4096, 4096, 4), (128, 2048, 1024, 8), (300, 2048, 528, 4),
         (512, 4096, 1024, 4), (2, 1024, 256, 8), (1024, 1024, 512, 8), (64, 8192, 256, 4)]
inputs = []
for i, (M, K, N, bits) in enumerate(cases):
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    inputs.append((make_x(wl), make_w(wl)))
dev = []
for (M, K, N, bits), (x, W) in zip(cases, inputs):
    xd = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).cuda()
    Wd = torch.from_numpy(W.view(np.int16).copy()).view(torch.bfloat16).cuda() if W.dtype == np.uint16 \
        else torch.from_numpy(W).cuda()
    dev.append((xd, Wd))
torch.cuda.synchronize()
start = threading.Barrier(len(cases))
out = [None] * len(cases)
err = []
def run(i):
    try:
        M, K, N, bits = cases[i]
        xd, Wd = dev[i]
        s = torch.cuda.Stream()
        start.wait()
        with torch.cuda.stream(s):
            packed, alpha = H.hbl_pack_ternary(Wd, stream=s)
            y = H.hbl_forward(xd, packed, alpha, N, bits, stream=s)
            codes, scales = H.hbl_fht_quant_i8(xd, bits, stream=s)
            t = H.hbl_debug_ln_fht(xd, stream=s)
        s.synchronize()
        out[i] = (y.view(torch.int16).cpu().numpy().view(np.uint16), codes.cpu().numpy(), scales.cpu().numpy(),
                  t.cpu().numpy(), float(alpha.cpu()[0]))
    except Exception as e:
        err.append((i, repr(e)))
th = [threading.Thread(target=run, args=(i,)) for i in range(len(cases))]
for t_ in th: t_.start()
for t_ in th: t_.join()
assert not err, err
for i, (M, K, N, bits) in enumerate(cases):
    y, codes, scales, t, alpha = out[i]
    x, W = inputs[i]
    w, a = oracle.ternary(W)
    assert alpha == float(a), (i, alpha, a)
    qo, so = oracle.quant(t, bits)
    assert np.array_equal(codes, qo) and np.array_equal(scales, so), i
    y_exact = oracle.dequant(oracle.gemm_i32(codes, w), scales, a)
    assert np.array_equal(y, oracle.round_to_bf16(y_exact)), i
assert H.hbl_last_device_error() == H.HBL_OK
print("concurrent first calls ok:", len(cases))
'''


def test_concurrent_first_calls_fresh_process():
    code = "ROOT = %r\n" % ROOT + SCRIPT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "concurrent first calls ok" in r.stdout
