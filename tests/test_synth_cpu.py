"""The seeded input generator (CPU side): shapes, recipe properties, bf16
rounding, determinism.  The generator holds no sampler arithmetic; these
tests check that it produces the workloads the benchmark and parity tests
describe."""
import math

import numpy as np
import pytest

import synth

pytestmark = []


def test_log_matches_libm():
    for x in [2.0 ** -40, 1e-7, 0.3, 0.7071, 1.0, 1.4142, 2.0, 7.7, 1234.5, 262144.0]:
        assert synth.log(x) == pytest.approx(math.log(x), abs=2e-6, rel=2e-7)


def test_tiny_workload_shape_and_targets():
    w = synth.WORKLOADS["tiny"]
    x = synth.generate_host(w, 0)
    assert x.shape == (1, 16, 1024) and x.dtype == np.float32
    assert abs(float(x.mean())) < 0.05 and abs(float(x.std()) - 1.0) < 0.05
    for l in range(16):
        t = synth.target(w, 0, l)
        assert 0 <= t < w.V
    # the confident fraction ramps to 100% at the last step: every target is boosted >= 12
    last = synth.generate_host(w, w.num_steps - 1)
    for l in range(16):
        t = synth.target(w, 0, l)
        assert last[0, l, t] > 8.0 and int(np.argmax(last[0, l])) == t


def test_confident_fraction_rises_over_steps():
    w = synth.WORKLOADS["canvas"].replace(L=256, V=2048)
    frac = []
    for s in (0, 12, 24, 36, 47):
        x = synth.generate_host(w, s)
        tg = np.array([synth.target(w, 0, l) for l in range(w.L)])
        boost = x[0, np.arange(w.L), tg].astype(np.uint32)
        zt = (boost << 16).view(np.float32)
        frac.append(float((zt > 9.0).mean()))
    assert frac[0] < 0.2 and frac[-1] > 0.95
    assert all(a <= b + 0.05 for a, b in zip(frac, frac[1:]))


def test_bf16_output_is_round_to_nearest_of_fp32():
    w32 = synth.WORKLOADS["canvas"].replace(L=4, V=3000, dtype=synth.F32)
    w16 = w32.replace(dtype=synth.BF16)
    a = synth.generate_host(w32, 5)
    b = synth.generate_host(w16, 5)
    u = a.view(np.uint32).astype(np.uint64)
    rne = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    assert np.array_equal(rne, b)


def test_zipf_workload_ranks_are_a_permutation():
    w = synth.WORKLOADS["stress"].replace(L=2, V=4096, zipf_noise_sd=0.0, boost_hi=0.0)
    x = synth.generate_host(w, 0)
    ranks = np.rint(np.exp(-x[0, 0].astype(np.float64) / 2.75)).astype(np.int64)
    assert sorted(ranks.tolist()) == list(range(1, 4097))


def test_generator_is_deterministic_and_keyed():
    w = synth.WORKLOADS["canvas"].replace(L=3, V=500)
    a = synth.generate_host(w, 7)
    b = synth.generate_host(w, 7)
    c = synth.generate_host(w, 8)
    d = synth.generate_host(w.replace(seed=99), 7)
    assert np.array_equal(a, b) and not np.array_equal(a, c) and not np.array_equal(a, d)
    # rows and canvases can be generated piecewise
    w2 = w.replace(B=3)
    full = synth.generate_host(w2, 2)
    part = synth.generate_host(w2, 2, b0=1, nb=2, l0=1, nl=2)
    assert np.array_equal(full[1:3, 1:3], part)


def test_serve_ramps_are_staggered():
    w = synth.WORKLOADS["serve"].replace(L=64, V=1024)
    s = 25
    x = synth.generate_host(w, s)
    fr = []
    for b in range(w.B):
        tg = np.array([synth.target(w, b, l) for l in range(w.L)])
        fr.append(float((x[b, np.arange(w.L), tg].astype(np.uint32) << 16).view(np.float32).__gt__(9.0).mean()))
    assert fr[0] > fr[-1]
