"""How precise a tensor-core form of the chunked backward could be.

The forward's tensor-core kernels take every derived fp32 operand as a pair of bf16
values, X = hi + lo, and form each product from three bf16 products,
hi*hi + lo*hi + hi*lo, accumulated in fp32.  This test runs the chunkwise gradient
algebra (tests/chunked_fp64.py) with every matrix product replaced by that model,
on the draws of the B1 H16 T4096 workload (here two heads, 256 tokens, d = 128),
and compares the gradients with the oracle's: the model's max-abs error lands at
2e-5 to 6e-5 of each gradient's rms, inside the 1e-4 bar of the fp32 backward but
with little to spare (up to 8e-5 at 1024 tokens).  With the bf16 inputs exact and only
the derived operands split, that is the precision a three-term tcgen05 backward
would start from.
"""
import math

import numpy as np
import torch

import oracle
from gated_delta_rule_109_b200 import inputs as I
from tests.chunked_fp64 import chunked_backward

NAMES = ("q", "k", "v", "log_alpha", "beta")


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def split3(a, b):
    """fp32 operands split into bf16 hi + lo; hi*hi + lo*hi + hi*lo, rounded to fp32."""
    a32, b32 = np.asarray(a, dtype=np.float32), np.asarray(b, dtype=np.float32)
    ah, bh = _bf16(a32), _bf16(b32)
    al, bl = _bf16(a32 - ah), _bf16(b32 - bh)
    return (ah @ bh + al @ bh + ah @ bl).astype(np.float32).astype(np.float64)


def test_split_bf16_product_model_of_the_chunked_gradient():
    w = I.scaled(I.PREFILL_H16_T4K, H=2, T=256, seed=8300)
    x = {n: t.float().numpy() for n, t in I.make_inputs(w).items() if t is not None}
    rng = np.random.default_rng(8301)
    d_out = rng.standard_normal((w.B, w.T, w.H, w.dv))
    d_fin = rng.standard_normal((w.B, w.H, w.dk, w.dv)) / math.sqrt(w.dk)
    ref = oracle.backward(*(x[n] for n in NAMES), d_out, None, d_fin)
    exact = chunked_backward(*(x[n] for n in NAMES), d_out, None, d_fin)
    model = chunked_backward(*(x[n] for n in NAMES), d_out, None, d_fin, mm=split3)
    for n in ref:
        assert oracle.parity_error(exact[n], ref[n]) < 1e-12, n
        err = oracle.parity_error(model[n], ref[n])
        assert 1e-7 < err < 1e-4, (n, err)
