"""GPU parity: the CUDA sampler (through the C ABI) against the CPU oracle.

Full element-by-element comparison over whole trajectories for configurations
the oracle finishes in seconds (several tiles per row and a ragged last
group), and sampled comparison at the full workload sizes the benchmark uses.
"""
from __future__ import annotations

import os

import numpy as np
import pytest

import oracle as O
import synth
from parity import (Stats, compare_canvas, compare_rows, h_tol, oracle_config)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from entropy_bound_canvas_b200 import build as B
    B.build()
    import entropy_bound_canvas_b200 as E
    return E


DEV = "cuda:0"


def tdtype(w):
    return torch.float32 if w.dtype == synth.F32 else torch.bfloat16


def host_logits(t):
    """Device logits -> numpy (float32, or uint16 bf16 bits)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def alloc_logits(w, nb=None, byte_offset=0):
    nb = w.B if nb is None else nb
    n = nb * w.L * w.V
    if byte_offset == 0:
        return torch.empty((nb, w.L, w.V), dtype=tdtype(w), device=DEV)
    raw = torch.empty(n * w.elt + 64, dtype=torch.uint8, device=DEV)
    return raw[byte_offset:byte_offset + n * w.elt].view(tdtype(w)).view(nb, w.L, w.V)


def decided_by_oracle(out, canvas_before, smp_gpu):
    """What the oracle decided a canvas with, for compare_canvas: its own
    per-position values, the state before the step, and the draws that
    differed from the GPU's within the N1 window."""
    excused = (np.asarray(smp_gpu) != out["sample"]) & out["open_before"]
    return dict(H=out["H"], pmax=out["pmax"], amax=out["amax"], open_before=out["open_before"],
                canvas_before=canvas_before, excused=excused)


def make_sampler(E, w, **over):
    cfg = w.sampler_config()
    cfg.update(over)
    return E.EBSampler(w.B, w.L, w.V, device=DEV, **cfg)


def run_full(E, w, byte_offset=0, canvas_offset=0, max_resyncs=0, mask=None, eb=None):
    """Whole trajectory, every canvas, every position compared with the oracle.
    `mask(logits, s)` may edit the generated logits in place (e.g. -inf).
    `eb`: an existing handle to continue with (it is restarted here)."""
    if eb is None:
        eb = make_sampler(E, w, canvas_offset=canvas_offset)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    st = O.State(oracle_config(w, canvas_offset=canvas_offset)).init()
    torch.cuda.synchronize()
    assert np.array_equal(canvas.cpu().numpy(), st.canvas)
    assert not committed.cpu().numpy().any() and not stop.cpu().numpy().any()
    logits = alloc_logits(w, byte_offset=byte_offset)
    f32 = w.dtype == synth.F32
    stats = Stats()
    prev_H = None
    for s in range(w.num_steps):
        synth.generate_device(w, s, logits, b0=canvas_offset)
        if mask is not None:
            mask(logits, s)
        eb.step(logits, s, canvas, committed, H, amax, stop)
        smp, pm = eb.draws()
        torch.cuda.synchronize()
        lg = host_logits(logits)
        Hg, amg, cvg, cmg, spg = (H.cpu().numpy(), amax.cpu().numpy(), canvas.cpu().numpy(),
                                  committed.cpu().numpy(), stop.cpu().numpy())
        smg, pmg = smp.cpu().numpy(), pm.cpu().numpy()
        for i in range(w.B):
            if st.stop[i]:
                assert spg[i] == st.stop[i]
                assert np.array_equal(cvg[i], st.canvas[i]) and cmg[i].all()
                assert np.array_equal(Hg[i], prev_H[i])  # untouched once stopped
                continue
            cv_before = st.canvas[i].copy()
            out = O.step_canvas(st, i, lg[i], s)
            compare_rows(stats, i, s, Hg[i], amg[i], pmg[i], smg[i], out, range(w.L), f32,
                         out["open_before"])
            stats.edits += int(out["margins"]["n_edit"])
            compare_canvas(stats, st, i, s, (cvg[i], cmg[i], spg[i]), out["margins"],
                           decided_by_oracle(out, cv_before, smg[i]))
            if st.stop[i]:
                stats.stop_steps[i] = s
        prev_H = Hg.copy()
        if st.stop.all():
            assert eb.done(stop)
            break
    assert st.stop.all(), "every canvas stops by the last step"
    assert stats.resyncs <= max_resyncs, stats
    eb.close()
    return stats


# ----------------------------------------------------------------------------- full parity

MID = synth.WORKLOADS["canvas"].replace(name="mid", B=3, L=64, V=8232, num_steps=24)


@pytest.mark.parametrize("name,w", [
    ("tiny", synth.WORKLOADS["tiny"]),
    ("mid_bf16_eb", MID),
    ("mid_f32_eb", MID.replace(dtype=synth.F32, seed=7)),
    ("mid_bf16_mi", MID.replace(rule=O.RULE_EB_MI, seed=8)),
    ("mid_bf16_br_greedy", MID.replace(rule=O.RULE_BR, greedy=1, quota=3, seed=9)),
    ("mid_bf16_br_editing", MID.replace(rule=O.RULE_BR, greedy=1, quota=3, seed=14,
                                        editing_threshold=0.5)),
    ("mid_f32_br_sampled_editing", MID.replace(dtype=synth.F32, rule=O.RULE_BR, quota=2,
                                               seed=15, t_max=1.0, t_min=1.0,
                                               editing_threshold=0.3)),
    ("mid_f32_br_sampled", MID.replace(dtype=synth.F32, rule=O.RULE_BR, quota=2, seed=10,
                                       t_max=1.0, t_min=1.0)),
    ("mid_zipf_f32", MID.replace(kind=synth.ZIPF, dtype=synth.F32, seed=11, B=2)),
    ("mid_stop_disabled", MID.replace(stop_entropy=-1.0, seed=12, B=2, num_steps=10)),
    ("mid_small_V", MID.replace(V=40, L=100, B=2, seed=13)),
])
def test_full_parity(E, name, w):
    stats = run_full(E, w)
    print(name, stats, "edits", stats.edits)
    if w.editing_threshold >= 0.0:
        assert stats.edits > 0, "the editing configuration re-edits some committed token"


@pytest.mark.parametrize("name,w", [
    # one-token vocabulary: every entropy is 0, every canvas commits at step 0
    ("V1_eb", MID.replace(V=1, L=16, B=2, num_steps=6, seed=41)),
    ("V1_br_greedy", MID.replace(V=1, L=16, B=2, num_steps=6, seed=45, rule=O.RULE_BR,
                                 greedy=1, quota=3)),
    # one position per canvas: the commit rule's minimum of one commits it
    ("L1", MID.replace(L=1, B=3, V=1000, num_steps=5, seed=42)),
    # a one-step trajectory: temperature t_max, and the step is the last one
    ("N1", MID.replace(num_steps=1, B=2, seed=43)),
    # long canvases: 4 and then 2 finish lanes per position
    ("L512", MID.replace(L=512, B=1, V=200, num_steps=6, seed=46)),
    ("L1024_max", MID.replace(L=1024, B=1, V=200, num_steps=6, seed=44)),
])
def test_degenerate_shapes(E, name, w):
    stats = run_full(E, w)
    print(name, stats)


def test_many_canvases_stopping_at_different_steps(E):
    """64 canvases: more finish clusters than fit on the GPU at once, so some
    start after others have run their epilogue and set their stop flags in
    the same step.  Canvases stop (all committed) between steps 12 and 15."""
    w = synth.WORKLOADS["serve"].replace(name="many", B=64, L=16, V=1000, seed=48)
    stats = run_full(E, w)
    print("many", stats)
    assert len(set(stats.stop_steps.values())) > 1, "canvases stop at different steps"


def test_all_canvases_stopped_is_a_no_op(E):
    w = MID.replace(B=2, seed=47)
    eb = make_sampler(E, w)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    H.fill_(-7.0)
    amax.fill_(-9)
    stop.fill_(1)
    before = (canvas.clone(), committed.clone())
    logits = alloc_logits(w)
    for s in range(3):
        synth.generate_device(w, s, logits)
        eb.step(logits, s, canvas, committed, H, amax, stop)
    torch.cuda.synchronize()
    assert torch.equal(canvas, before[0]) and torch.equal(committed, before[1])
    assert (H == -7.0).all() and (amax == -9).all() and (stop == 1).all()
    assert eb.status() == 0
    eb.close()


def _mask_neg_inf(V):
    """-inf logits, as a vocabulary mask would leave them: a random tenth of the
    vocabulary (new each step), one whole 64-logit group, and the last logit."""
    def apply(logits, s):
        g = torch.Generator(device="cpu").manual_seed(1000 + s)
        m = torch.rand(V, generator=g) < 0.1
        m[3 * 64:4 * 64] = True
        m[V - 1] = True
        logits[:, :, m.to(logits.device)] = float("-inf")
    return apply


@pytest.mark.parametrize("name,w", [
    ("masked_bf16", MID.replace(B=2, num_steps=12, seed=21)),
    ("masked_f32", MID.replace(B=2, num_steps=12, seed=22, dtype=synth.F32)),
    ("masked_unaligned_bf16", MID.replace(B=2, num_steps=8, seed=23, V=5001)),
])
def test_full_parity_neg_inf_logits(E, name, w):
    """Masked (-inf) logits contribute nothing to the entropy, never win a
    draw, and never become the argmax, exactly as in the oracle."""
    stats = run_full(E, w, mask=_mask_neg_inf(w.V))
    print(name, stats)


def run_split(E, w, bounds, max_resyncs=0):
    """Vocabulary-sharded logits emulated on one device: one handle per slice
    (bounds on 64-logit group boundaries), the records stacked in slice order
    as an all-gather would, slice 0's handle combining; compared with the
    oracle over the full vocabulary."""
    handles = []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        cfg = w.sampler_config()
        handles.append(E.EBSampler(w.B, w.L, hi - lo, device=DEV, vocab_offset=lo,
                                   vocab_total=w.V, **cfg))
    h0 = handles[0]
    canvas, committed, stop = h0.new_canvas()
    H, amax = h0.outputs()
    st = O.State(oracle_config(w)).init()
    torch.cuda.synchronize()
    assert np.array_equal(canvas.cpu().numpy(), st.canvas)
    logits = alloc_logits(w)
    f32 = w.dtype == synth.F32
    stats = Stats()
    for s in range(w.num_steps):
        synth.generate_device(w, s, logits)
        recs = []
        for h, (lo, hi) in zip(handles, zip(bounds[:-1], bounds[1:])):
            r = h.slice_records()
            h.step_slice(logits[:, :, lo:hi].contiguous(), s, committed, stop, r)
            recs.append(r)
        h0.combine(torch.stack(recs), s, canvas, committed, H, amax, stop)
        smp, pm = h0.draws()
        torch.cuda.synchronize()
        lg = host_logits(logits)
        Hg, amg, cvg, cmg, spg = (H.cpu().numpy(), amax.cpu().numpy(), canvas.cpu().numpy(),
                                  committed.cpu().numpy(), stop.cpu().numpy())
        smg, pmg = smp.cpu().numpy(), pm.cpu().numpy()
        for i in range(w.B):
            if st.stop[i]:
                assert spg[i] == st.stop[i] and cmg[i].all()
                continue
            cv_before = st.canvas[i].copy()
            out = O.step_canvas(st, i, lg[i], s)
            compare_rows(stats, i, s, Hg[i], amg[i], pmg[i], smg[i], out, range(w.L), f32,
                         out["open_before"])
            compare_canvas(stats, st, i, s, (cvg[i], cmg[i], spg[i]), out["margins"],
                           decided_by_oracle(out, cv_before, smg[i]))
        if st.stop.all():
            break
    assert st.stop.all()
    assert stats.resyncs <= max_resyncs, stats
    for h in handles:
        assert h.status() == 0
        h.close()
    return stats


@pytest.mark.parametrize("name,w,bounds", [
    ("split3_bf16", MID.replace(B=2, num_steps=16, seed=31), [0, 2560, 5120, 8232]),
    ("split2_f32", MID.replace(B=2, num_steps=12, seed=32, dtype=synth.F32), [0, 4096, 8232]),
    ("split2_br_greedy", MID.replace(B=2, num_steps=12, seed=33, rule=O.RULE_BR, greedy=1,
                                     quota=3), [0, 64, 8232]),
])
def test_vocabulary_sharded_step_matches_oracle(E, name, w, bounds):
    stats = run_split(E, w, bounds)
    print(name, stats)


def test_slice_handle_refuses_the_plain_step(E):
    w = MID.replace(B=1)
    h = E.EBSampler(w.B, w.L, 4096, device=DEV, vocab_offset=4096, vocab_total=w.V,
                    **w.sampler_config())
    canvas, committed, stop = h.new_canvas()
    H, amax = h.outputs()
    z = torch.zeros((w.B, w.L, 4096), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(E.EBError):
        h.step(z, 0, canvas, committed, H, amax, stop)
    assert int(canvas.max()) < w.V  # the initial canvas covers the whole vocabulary
    h.close()


def test_split_event_is_recorded_after_the_step_kernel(E):
    w = MID.replace(B=1, num_steps=4)
    eb = make_sampler(E, w)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    logits = alloc_logits(w)
    synth.generate_device(w, 0, logits)
    H0 = None
    for use in (False, True):
        eb.init_canvas(canvas, committed, stop)
        a, m, b = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        eb.set_split_event(m if use else None)
        a.record()
        eb.step(logits, 0, canvas, committed, H, amax, stop)
        b.record()
        torch.cuda.synchronize()
        if use:
            assert a.elapsed_time(m) > 0 and m.elapsed_time(b) >= 0
            assert torch.equal(H, H0)  # recording the event changes no result
        H0 = H.clone()
    eb.set_split_event(None)
    eb.close()


def test_full_parity_unaligned_rows(E):
    """Odd V (rows not 16-byte aligned): the element-load path."""
    stats = run_full(E, MID.replace(V=5001, B=2, seed=14))
    print(stats)


def test_full_parity_offset_base_pointer(E):
    """Logits base 2 bytes off a 16-byte boundary: the element-load path."""
    stats = run_full(E, MID.replace(B=2, seed=15), byte_offset=2)
    print(stats)


def test_full_parity_canvas_offset(E):
    stats = run_full(E, MID.replace(B=2, seed=16), canvas_offset=5)
    print(stats)


# ----------------------------------------------------------------------------- full size

_POOL = None


def _pool():
    """Threads for the oracle: its C calls release the GIL, so rows of a
    step run on every host core."""
    global _POOL
    if _POOL is None:
        from concurrent.futures import ThreadPoolExecutor
        _POOL = ThreadPoolExecutor(max(1, os.cpu_count() or 1))
    return _POOL


def oracle_rows(cfg, rows, T, b, s, open_before, greedy):
    """The oracle's per-position outputs of one canvas at step s, every row:
    entropy, max probability, argmax, and the draw of every open row."""
    L = rows.shape[0]

    def one(l):
        Hh, pmh, amh, _ = O.row_stats(rows[l], 1.0 / T)
        if not open_before[l]:
            return Hh, pmh, amh, -1, np.inf, -1
        if greedy:
            return Hh, pmh, amh, amh, np.inf, -1
        x, mgn, grp = O.sample(cfg, rows[l], 1.0 / T, b, l, s)
        return Hh, pmh, amh, x, mgn, grp

    res = list(_pool().map(one, range(L)))
    out = {"H": np.array([r[0] for r in res]), "pmax": np.array([r[1] for r in res]),
           "amax": np.array([r[2] for r in res], np.int64),
           "sample": np.array([r[3] for r in res], np.int64),
           "sample_margin": np.array([r[4] for r in res]),
           "sample_group": np.array([r[5] for r in res], np.int64)}
    return out


def run_full_size(E, w, canvases):
    """Full-size trajectory, every step: every position of the tracked
    canvases is compared with the oracle element by element (entropy, max
    probability, argmax, draw), and every canvas decision is re-derived by
    the oracle from the GPU's per-position outputs.  The logits of each step
    are generated in place, so only one step's logits are held at a time."""
    eb = make_sampler(E, w)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    st = O.State(oracle_config(w), canvases=canvases).init()
    torch.cuda.synchronize()
    assert np.array_equal(canvas.cpu().numpy()[canvases], st.canvas)
    logits = alloc_logits(w)
    f32 = w.dtype == synth.F32
    stats = Stats()
    for s in range(w.num_steps):
        synth.generate_device(w, s, logits)
        cm_before = committed.cpu().numpy()
        eb.step(logits, s, canvas, committed, H, amax, stop)
        smp, pm = eb.draws()
        torch.cuda.synchronize()
        Hg, amg, cvg, cmg, spg = (H.cpu().numpy(), amax.cpu().numpy(), canvas.cpu().numpy(),
                                  committed.cpu().numpy(), stop.cpu().numpy())
        smg, pmg = smp.cpu().numpy(), pm.cpu().numpy()
        T = O.temperature(st.cfg, s)
        for i, b in enumerate(canvases):
            if st.stop[i]:
                assert spg[b] == st.stop[i]
                continue
            open_before = cm_before[b] == 0
            out = oracle_rows(st.cfg, host_logits(logits[b]), T, b, s, open_before, w.greedy)
            compare_rows(stats, b, s, Hg[b], amg[b], pmg[b], smg[b], out, range(w.L), f32,
                         open_before)
            cv_before = st.canvas[i].copy()
            mg = O.canvas_decide(st, i, s, Hg[b].astype(np.float64), amg[b],
                                 pmg[b].astype(np.float64), smg[b])
            compare_canvas(stats, st, i, s, (cvg[b], cmg[b], spg[b]), mg,
                           dict(H=Hg[b], pmax=pmg[b], amax=amg[b], open_before=open_before,
                                canvas_before=cv_before, excused=np.zeros(w.L, bool)))
            if st.stop[i]:
                stats.stop_steps[b] = s
        if spg.all():
            assert eb.done(stop)
            break
    assert eb.status() == 0
    eb.close()
    return stats, stop.cpu().numpy()


@pytest.mark.parametrize("name,canvases", [
    ("canvas", [0]),
    ("serve", [0, 3, 7]),
    ("br", [0, 3]),
    ("stress", [0, 31]),
])
def test_full_size_every_step(E, name, canvases):
    """The workloads at their full sizes over all their steps (48 unless the
    adaptive stop ends a canvas earlier)."""
    w = synth.WORKLOADS[name]
    stats, stop = run_full_size(E, w, canvases)
    print(name, stats)
    assert stats.resyncs == 0, stats
    assert stop.all(), "every canvas stops by the last step"


# ----------------------------------------------------------------------------- edge cases

def test_init_canvas_matches_oracle(E):
    w = MID.replace(B=5)
    eb = make_sampler(E, w, canvas_offset=11)
    canvas, committed, stop = eb.new_canvas()
    st = O.State(oracle_config(w, canvas_offset=11)).init()
    torch.cuda.synchronize()
    assert np.array_equal(canvas.cpu().numpy(), st.canvas)
    assert (canvas.cpu().numpy() < w.V).all()


def test_step_order_and_arguments(E):
    w = MID.replace(B=1)
    eb = make_sampler(E, w)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    logits = alloc_logits(w)
    synth.generate_device(w, 0, logits)
    with pytest.raises(E.EBError) as ei:
        eb.step(logits, 3, canvas, committed, H, amax, stop)
    assert ei.value.code == 4
    with pytest.raises(E.EBError) as ei:
        eb.step(logits, w.num_steps, canvas, committed, H, amax, stop)
    assert ei.value.code == 1
    assert eb.step_ptr(0, 1, 0, canvas.data_ptr(), committed.data_ptr(), H.data_ptr(),
                       amax.data_ptr(), stop.data_ptr()) == 1
    assert eb.step_ptr(logits.data_ptr(), 7, 0, canvas.data_ptr(), committed.data_ptr(),
                       H.data_ptr(), amax.data_ptr(), stop.data_ptr()) == 5
    eb.step(logits, 0, canvas, committed, H, amax, stop)
    eb.step(logits, 1, canvas, committed, H, amax, stop)
    with pytest.raises(E.EBError):
        eb.step(logits, 1, canvas, committed, H, amax, stop)
    eb.step(logits, 0, canvas, committed, H, amax, stop)  # restart is allowed
    assert eb.status() == 0


def test_bad_config_rejected(E):
    with pytest.raises(E.EBError):
        E.EBSampler(1, 0, 100, device=DEV)
    with pytest.raises(E.EBError):
        E.EBSampler(1, 2000, 100, device=DEV)
    with pytest.raises(E.EBError):
        E.EBSampler(1, 16, 100, device=DEV, t_max=-1.0)


def test_stopped_canvas_is_skipped(E):
    w = MID.replace(B=3, seed=21)
    eb = make_sampler(E, w)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    H.fill_(-7.0)
    amax.fill_(-9)
    stop[1] = 2
    before = (canvas[1].clone(), committed[1].clone())
    logits = alloc_logits(w)
    for s in range(4):
        synth.generate_device(w, s, logits)
        eb.step(logits, s, canvas, committed, H, amax, stop)
    torch.cuda.synchronize()
    assert torch.equal(canvas[1], before[0]) and torch.equal(committed[1], before[1])
    assert (H[1] == -7.0).all() and (amax[1] == -9).all() and int(stop[1]) == 2
    assert (H[0] >= 0).all() and (H[2] >= 0).all()


def test_bad_committed_token_sets_status(E):
    w = MID.replace(B=1, seed=22)
    eb = make_sampler(E, w)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    committed[0, 3] = 1
    canvas[0, 3] = w.V + 5
    logits = alloc_logits(w)
    synth.generate_device(w, 0, logits)
    eb.step(logits, 0, canvas, committed, H, amax, stop)
    assert eb.status(clear=True) & E.STATUS_BAD_TOKEN
    assert eb.status() == 0
    assert int(canvas[0, 3]) == w.V + 5  # committed tokens are never rewritten


def test_stop_fires_on_predicted_step(E):
    L, V = 16, 512
    eb = E.EBSampler(1, L, V, device=DEV, num_steps=30, seed=5, entropy_bound=0.0)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    tgt = torch.arange(L, device=DEV) * 31 % V
    fired = None
    for s in range(30):
        z = torch.zeros((1, L, V), dtype=torch.float32, device=DEV)
        t = tgt if s >= 6 else (tgt + s) % V
        z[0, torch.arange(L, device=DEV), t] = 40.0 if s >= 6 else 0.5
        eb.step(z, s, canvas, committed, H, amax, stop)
        if int(stop[0]):
            fired = (s, int(stop[0]))
            break
    assert fired == (7, E.STOP_ADAPTIVE)
    assert bool(committed.all())


def test_sharded_canvases_equal_one_handle(E):
    """Canvases split over two handles with canvas offsets give the same bits."""
    w = MID.replace(B=4, seed=23, num_steps=8)
    logits = alloc_logits(w)
    one = make_sampler(E, w)
    c1, m1, s1 = one.new_canvas()
    H1, a1 = one.outputs()
    parts = []
    for r in range(2):
        off, cnt = E.shard_canvases(w.B, 2, r)
        wp = w.replace(B=cnt)
        e = make_sampler(E, wp, canvas_offset=off)
        c, m, s = e.new_canvas()
        h, a = e.outputs()
        parts.append((e, off, cnt, c, m, s, h, a))
    for st in range(w.num_steps):
        synth.generate_device(w, st, logits)
        one.step(logits, st, c1, m1, H1, a1, s1)
        for e, off, cnt, c, m, s, h, a in parts:
            e.step(logits[off:off + cnt].contiguous(), st, c, m, h, a, s)
    torch.cuda.synchronize()
    for e, off, cnt, c, m, s, h, a in parts:
        assert torch.equal(c, c1[off:off + cnt]) and torch.equal(m, m1[off:off + cnt])
        assert torch.equal(s, s1[off:off + cnt]) and torch.equal(a, a1[off:off + cnt])
        assert torch.allclose(h, H1[off:off + cnt], atol=1e-6, rtol=0)


def test_deterministic_and_graph_capture(E):
    w = MID.replace(B=2, seed=24, num_steps=12)
    logits = torch.empty((w.num_steps, w.B, w.L, w.V), dtype=tdtype(w), device=DEV)
    for s in range(w.num_steps):
        synth.generate_device(w, s, logits[s])

    def eager():
        eb = make_sampler(E, w)
        c, m, st = eb.new_canvas()
        h, a = eb.outputs()
        for s in range(w.num_steps):
            eb.step(logits[s], s, c, m, h, a, st)
        torch.cuda.synchronize()
        return c, m, st, h, a

    r1, r2 = eager(), eager()
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)

    eb = make_sampler(E, w)
    c, m, st = eb.new_canvas()
    h, a = eb.outputs()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        eb.init_canvas(c, m, st)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            eb.init_canvas(c, m, st)
            for s in range(w.num_steps):
                eb.step(logits[s], s, c, m, h, a, st)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        for x, y in zip((c, m, st, h, a), r1):
            assert torch.equal(x, y)
    del g


# ----------------------------------------------------------------------------- failure paths

def test_timed_out_wait_reports_status_and_the_next_trajectory_matches(E):
    """A stream-kernel pipeline wait that runs out (limit shortened to 1 ns
    through the diagnostic hook) sets STATUS_TIMEOUT and returns instead of
    hanging; after the normal limit is restored and the canvases are started
    again, a trajectory matches the oracle."""
    w = MID.replace(B=1, L=16, V=262144, num_steps=3, seed=61)
    eb = make_sampler(E, w)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    logits = alloc_logits(w)
    synth.generate_device(w, 0, logits)
    eb.set_wait_limit(1)
    eb.step(logits, 0, canvas, committed, H, amax, stop)
    torch.cuda.synchronize()
    st = eb.status(clear=True)
    assert st & E.STATUS_TIMEOUT, st
    assert eb.status() == 0
    eb.set_wait_limit(0)
    stats = run_full(E, w, eb=eb)  # the same handle, started again
    print(stats)


def test_handles_with_different_batch_sizes_coexist(E):
    """A handle for many canvases keeps working after a handle for one canvas
    is created on the same device (kernel attributes are per device and are
    never lowered)."""
    wb = MID.replace(B=128, L=8, V=300, num_steps=3, seed=62)
    big = make_sampler(E, wb)
    small = make_sampler(E, wb.replace(B=1))
    small.close()
    canvas, committed, stop = big.new_canvas()
    H, amax = big.outputs()
    st = O.State(oracle_config(wb)).init()
    logits = alloc_logits(wb)
    for s in range(wb.num_steps):
        synth.generate_device(wb, s, logits)
        big.step(logits, s, canvas, committed, H, amax, stop)
        torch.cuda.synchronize()
        lg = host_logits(logits)
        Hg, cvg = H.cpu().numpy(), canvas.cpu().numpy()
        for i in range(wb.B):
            out = O.step_canvas(st, i, lg[i], s)
            if out is None:
                continue
            assert np.abs(Hg[i] - out["H"]).max() <= h_tol(False)
            assert np.array_equal(cvg[i], st.canvas[i])
    assert big.status() == 0
    big.close()
