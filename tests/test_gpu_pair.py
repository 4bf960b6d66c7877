"""GPU parity of the CTA-pair GEMM (cta_group::2 MMAs over 256-row tiles,
each CTA staging its own A rows and half of W), an opt-in instantiation of
the dual-path linear selected by SHARQ_GEMM_PAIR=1 (read once per process,
so the check runs in a child process): outputs within 1e-3 sum|a||w| of the
oracle, with even and odd numbers of 128-row tiles (a pair whose second
block is padding), both formats, and a bias."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys
import numpy as np
import torch
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import oracle
import sparsity_gemm_b200 as sq
import synth
from gpu_common import assert_linear_close, cuda16
for (M, N, K, fmt, with_bias) in [(256, 256, 512, 0, False), (300, 544, 1024, 0, True), (512, 1024, 2048, 1, False),
                                   (1000, 4096, 4096, 0, False)]:
    x = synth.activations_student(11 + M, M, K)
    w = synth.weights(12 + N, N, K)
    p = sq.prepare(cuda16(x), None, None, 1e-5, 2, 4, fmt)
    qw = sq.quantize_weight(cuda16(w), fmt)
    b = synth.activations_gaussian(3, 1, N, 0, 1.0)[0] if with_bias else None
    out = sq.linear(p, qw, bias=None if b is None else cuda16(b)).cpu().numpy()
    assert sq.get_last_error() == sq.OK
    rows = sorted(set(list(range(min(M, 48))) + [M - 1, M // 2]))
    op = oracle.prepare(x[rows], None, None, 1e-5, 2, 4, fmt, s_t=np.float32(sq.prep_export(p)["s_t"]))
    ow = oracle.quantize_weight(w, fmt)
    if b is None:
        want, bound = oracle.linear_prepared(op, ow)
    else:
        want, bound = oracle.linear_fused(op, [ow], bias=b)
    assert_linear_close(out[rows], want, bound)
print("pair ok")
'''.replace("ROOT", repr(ROOT))


def test_pair_gemm_within_tolerance():
    env = dict(os.environ, SHARQ_GEMM_PAIR="1")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "pair ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
