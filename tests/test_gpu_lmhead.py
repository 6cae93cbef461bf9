"""GPU parity of the sampler fused into the LM-head contraction
(eb_lmhead_logits / eb_lmhead_step, through the C ABI).

The synthetic inputs (synth/lmhead.py) make the fp32 contraction exact under
any summation order, so the logits the tensor cores form equal the oracle's
float64 logits bit for bit; the step is then compared with the oracle exactly
as the logits-input step is (integer outputs bit-exact outside the near-tie
windows, entropies within the fp32 tolerance).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
from parity import Stats, compare_canvas, compare_rows, oracle_config
from synth import lmhead as LM

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def E():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from entropy_bound_canvas_b200 import build as B
    B.build()
    import entropy_bound_canvas_b200 as E
    return E


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("rows,V,d", [(128, 256, 64), (300, 1024, 256), (256, 4096, 2560),
                                      (1, 512, 128)])
def test_lmhead_logits_equal_the_oracle_bit_for_bit(E, rows, V, d):
    wc = LM.weight_codes(V, d, seed=11)
    hc = torch.randint(LM.CODE_LO, LM.CODE_HI + 1, (rows, d), dtype=torch.int8,
                       generator=torch.Generator().manual_seed(rows + d))
    h, w = LM.to_bf16(hc), LM.to_bf16(wc)
    z = E.lmhead_logits(h.to(DEV), w.to(DEV))
    torch.cuda.synchronize()
    ref = O.lmhead_logits(bits(h), bits(w))
    assert np.array_equal(z.cpu().numpy().astype(np.float64), ref)


def test_lmhead_logits_of_random_bf16_within_the_fp32_summation_bound(E):
    """General bf16 inputs: |z - z_exact| <= gamma_d sum_k |h_k w_k|, the
    bound of any order of d fp32 additions of exact products."""
    g = torch.Generator().manual_seed(3)
    rows, V, d = 384, 2048, 768
    h = torch.randn((rows, d), generator=g).to(torch.bfloat16)
    w = torch.randn((V, d), generator=g).to(torch.bfloat16)
    z = E.lmhead_logits(h.to(DEV), w.to(DEV)).cpu().numpy().astype(np.float64)
    hd, wd = O.decode_bf16(bits(h)), O.decode_bf16(bits(w))
    exact = hd @ wd.T
    u = 2.0 ** -24
    gamma = d * u / (1 - d * u)
    bound = gamma * (np.abs(hd) @ np.abs(wd).T)
    assert np.all(np.abs(z - exact) <= bound)


def test_lmhead_rejects_unsupported_sizes(E):
    h = torch.zeros((128, 96), dtype=torch.bfloat16, device=DEV)  # d not a multiple of 64
    w = torch.zeros((256, 96), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(E.EBError):
        E.lmhead_logits(h, w)
    h = torch.zeros((128, 64), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((320, 64), dtype=torch.bfloat16, device=DEV)  # V not a multiple of 256
    with pytest.raises(E.EBError):
        E.lmhead_logits(h, w)


def run_lmhead(E, w, d, steps=None):
    """A trajectory of LM-head steps, every position of every canvas compared
    with the oracle run on the float64 logits of the same inputs."""
    eb = E.EBSampler(w.B, w.L, w.V, device=DEV, **w.sampler_config())
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    st = O.State(oracle_config(w)).init()
    wc = LM.weight_codes(w.V, d, seed=w.seed)
    wb = LM.to_bf16(wc)
    Wd = wb.to(DEV)
    w64 = O.decode_bf16(bits(wb))
    stats = Stats()
    prev_H = None
    n = w.num_steps if steps is None else steps
    for s in range(n):
        hb = LM.to_bf16(LM.hidden_codes(wc, w.B, w.L, s, w.num_steps, seed=w.seed))
        eb.lmhead_step(hb.to(DEV), Wd, s, canvas, committed, H, amax, stop)
        smp, pm = eb.draws()
        torch.cuda.synchronize()
        z = (O.decode_bf16(bits(hb)) @ w64.T).astype(np.float32).reshape(w.B, w.L, w.V)
        Hg, amg, cvg, cmg, spg = (H.cpu().numpy(), amax.cpu().numpy(), canvas.cpu().numpy(),
                                  committed.cpu().numpy(), stop.cpu().numpy())
        smg, pmg = smp.cpu().numpy(), pm.cpu().numpy()
        for i in range(w.B):
            if st.stop[i]:
                assert spg[i] == st.stop[i]
                assert np.array_equal(cvg[i], st.canvas[i]) and cmg[i].all()
                assert np.array_equal(Hg[i], prev_H[i])
                continue
            cv_before = st.canvas[i].copy()
            out = O.step_canvas(st, i, z[i], s)
            compare_rows(stats, i, s, Hg[i], amg[i], pmg[i], smg[i], out, range(w.L), True,
                         out["open_before"])
            excused = (np.asarray(smg[i]) != out["sample"]) & out["open_before"]
            compare_canvas(stats, st, i, s, (cvg[i], cmg[i], spg[i]), out["margins"],
                           dict(H=out["H"], pmax=out["pmax"], amax=out["amax"],
                                open_before=out["open_before"], canvas_before=cv_before,
                                excused=excused))
        prev_H = Hg.copy()
        if st.stop.all():
            break
    assert stats.resyncs == 0, stats
    assert eb.status() == 0
    eb.close()
    return stats


LMW = synth.WORKLOADS["canvas"].replace(name="lm", B=2, L=128, V=8192, num_steps=16, seed=21)


@pytest.mark.parametrize("name,w,d", [
    ("eb", LMW, 256),
    ("eb_ragged_rows", LMW.replace(B=1, L=200, seed=22), 192),
    ("br_greedy", synth.WORKLOADS["br"].replace(B=2, L=128, V=4096, num_steps=12, seed=23), 128),
    ("eb_mi", LMW.replace(rule=O.RULE_EB_MI, seed=24), 256),
])
def test_lmhead_trajectory_matches_the_oracle(E, name, w, d):
    stats = run_lmhead(E, w, d)
    print(name, stats)


def test_lmhead_full_size_first_steps_match_the_oracle(E):
    """The canvas shape of the model card (1 x 256 x 262144) at hidden size
    2560, the first three steps, every position."""
    w = synth.WORKLOADS["canvas"].replace(name="lm_full", seed=25)
    stats = run_lmhead(E, w, 2560, steps=3)
    print(stats)
