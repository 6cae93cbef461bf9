"""CPU pins of the LM-head step's oracle contraction and of the synthetic
LM-head inputs (no GPU).

The oracle's logits are numpy's float64 product of the decoded bf16 inputs;
here they are checked against exact integer arithmetic (Python integers on
the inputs' codes), which the recipe makes equal: every input is a code over
8, so every logit is an integer over 64.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402
from synth import lmhead as LM  # noqa: E402


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def test_oracle_logits_equal_exact_integer_dot_products():
    V, d, B, L = 96, 64, 1, 12
    wc = LM.weight_codes(V, d, seed=5)
    hc = LM.hidden_codes(wc, B, L, s=7, num_steps=8, seed=5)
    z = O.lmhead_logits(_bits(LM.to_bf16(hc)), _bits(LM.to_bf16(wc)))
    wi, hi = wc.numpy().astype(int).tolist(), hc.numpy().astype(int).tolist()
    for r in range(B * L):
        for v in range(V):
            exact = sum(a * b for a, b in zip(hi[r], wi[v]))  # over 64
            assert z[r, v] * 64.0 == exact


def test_codes_decode_exactly_and_logits_stay_in_fp32_exact_range():
    V, d = 300, 2560
    wc = LM.weight_codes(V, d, seed=1)
    assert wc.min() >= LM.CODE_LO and wc.max() <= LM.CODE_HI
    w = LM.to_bf16(wc)
    assert torch.equal(w.to(torch.float32) * 8, wc.to(torch.float32))
    # |z| <= d * 4 / 64: an integer over 64 below 2^24 / 64, exact in fp32
    bound = d * LM.CODE_HI * LM.CODE_HI
    assert bound < 2 ** 24


def test_confident_rows_carry_their_target_and_grow_with_the_step():
    V, d, B, L, N = 512, 2560, 1, 64, 48
    wc = LM.weight_codes(V, d, seed=3)
    t = LM.targets(B * L, V, seed=3)
    w = _bits(LM.to_bf16(wc))
    conf = []
    for s in (0, N - 1):
        z = O.lmhead_logits(_bits(LM.to_bf16(LM.hidden_codes(wc, B, L, s, N, seed=3))), w)
        top = z.argmax(axis=1)
        conf.append(float(np.mean(top == t.numpy())))
    assert conf[0] < 0.5 and conf[1] > 0.95  # 5 % -> 100 % confident rows
