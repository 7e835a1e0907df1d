"""The attention kernel computes part of its exponentials with a polynomial on the FMA
pipe (range reduction + minimax degree-3 fit for 2^f on [-1/2, 1/2]). This re-fits the
polynomial, checks the constants compiled into the kernel, and bounds the float32
evaluation error against exp2 (no GPU)."""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_tcgen05_b200", "csrc")
sys.path.insert(0, CSRC)

import gen_exp2_poly  # noqa: E402


def _kernel_constants():
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    vals = {}
    for i in range(4):
        m = re.search(rf"kExpC{i}\s*=\s*([-+0-9.eE]+)f", text)
        vals[i] = np.float32(float(m.group(1)))
    return [vals[i] for i in range(4)]


def test_constants_match_the_fit():
    c, err = gen_exp2_poly.fit()
    assert err < 8e-5
    kc = _kernel_constants()
    for a, b in zip(kc, np.float32(c)):
        assert abs(float(a) - float(b)) <= 2e-7 * abs(float(b)), (a, b)


def test_float32_evaluation_error_bound():
    kc = _kernel_constants()
    xs = np.linspace(-120.0, 8.0, 400001, dtype=np.float32)
    got = gen_exp2_poly.emulate_float32(xs, kc).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
    # far below the range the kernel clamps: tiny, never negative
    low = gen_exp2_poly.emulate_float32(np.array([-200.0, -127.0, -126.0], np.float32), kc)
    assert (low >= 0).all() and (low < 1e-37).all()
