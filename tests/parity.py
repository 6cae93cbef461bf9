"""Step-by-step comparison of the CUDA sampler with the CPU oracle.

Tolerances and near-tie windows (the integer outputs must match bit for bit
except where the oracle's own margins say the decision hinges on rounding):

  entropies        |H_gpu - H_oracle| <= 1e-4 (fp32 logits), 2e-3 (bf16 logits)
  draw (N1)        excused when the oracle's top-2 perturbed scores are within
                   1e-6 of each other relative to max(1, |score|)
  EB prefix (N2)   excused when a cumulative entropy at the cut is within 1e-6
                   of entropy_bound
  EB cut (N3)      excused when the last committed and first left-out entropies
                   differ by <= CUT_WINDOW
  stop (N4)        excused when the canvas mean entropy is within STOP_WINDOW of
                   the stop threshold
  BR (N5)          excused when a pmax is within 1e-6 of the threshold or the
                   two pmax values at the quota cut differ by <= 1e-5 relative
  BR edit (N6)     excused when a moved committed position's pmax is within
                   1e-6 of editing_threshold

CUT_WINDOW and STOP_WINDOW bound the GPU's entropy error on low-entropy rows:
fp32 accumulation of 64-term groups with the group that holds the maximum
recomputed in float64 gives |dH| <~ 2.4e-7 (ex2.approx relative error) times
H plus ~1e-7; 1e-6 leaves a factor of ~5.

After an excused divergence -- every differing position is one a raised flag
names -- the oracle takes over the GPU's canvas state and continues (resync);
the number of resyncs is reported so a test can bound it.
"""
from __future__ import annotations

import math

import numpy as np

import oracle as O

CUT_WINDOW = 1e-6
STOP_WINDOW = 1e-6
N1_WINDOW = 1e-6
N2_WINDOW = 1e-6
BR_WINDOW = 1e-6
QUOTA_WINDOW = 1e-5


def h_tol(dtype_is_f32: bool) -> float:
    return 1e-4 if dtype_is_f32 else 2e-3


def oracle_config(w, **over) -> O.Config:
    kw = dict(B=w.B, L=w.L, V=w.V, group_size=64)
    kw.update(w.sampler_config())
    kw.update(over)
    return O.Config(**kw)


class Stats:
    def __init__(self):
        self.max_dH = 0.0
        self.max_dH_low = 0.0  # positions with H < 0.2 (the ones decisions use)
        self.max_rel_dpmax = 0.0
        self.edits = 0  # committed positions the oracle re-edited (block refinement)
        self.rows = 0
        self.draws = 0
        self.excused_draws = 0
        self.resyncs = 0
        self.flags = []
        self.stop_steps = {}

    def __repr__(self):
        return (f"Stats(rows={self.rows}, draws={self.draws}, max_dH={self.max_dH:.3g}, "
                f"max_dH_low={self.max_dH_low:.3g}, max_rel_dpmax={self.max_rel_dpmax:.3g}, "
                f"excused_draws={self.excused_draws}, resyncs={self.resyncs}, "
                f"stop_steps={self.stop_steps}, flags={self.flags[:10]})")


def compare_rows(stats, i, s, H_g, am_g, pm_g, smp_g, out, rows, f32, open_before):
    """Per-position outputs of canvas i at `rows` against the oracle's `out`."""
    tol = h_tol(f32)
    for l in rows:
        stats.rows += 1
        dH = abs(float(H_g[l]) - out["H"][l])
        stats.max_dH = max(stats.max_dH, dH)
        if out["H"][l] < 0.2:
            stats.max_dH_low = max(stats.max_dH_low, dH)
        assert dH <= tol, f"canvas {i} step {s} pos {l}: H {H_g[l]} vs {out['H'][l]}"
        assert int(am_g[l]) == int(out["amax"][l]), f"canvas {i} step {s} pos {l}: argmax"
        rel = abs(float(pm_g[l]) - out["pmax"][l]) / out["pmax"][l]
        stats.max_rel_dpmax = max(stats.max_rel_dpmax, rel)
        assert rel <= 1e-4, f"canvas {i} step {s} pos {l}: pmax {pm_g[l]} vs {out['pmax'][l]}"
        if open_before[l]:
            stats.draws += 1
            if int(smp_g[l]) != int(out["sample"][l]):
                if out["sample_margin"][l] <= N1_WINDOW:
                    stats.excused_draws += 1
                else:
                    raise AssertionError(
                        f"canvas {i} step {s} pos {l}: draw {smp_g[l]} vs {out['sample'][l]} "
                        f"(margin {out['sample_margin'][l]:.3g}, group {out['sample_group'][l]})")


def flagged_positions(cfg, s, mg, H, pmax, amax, open_before, canvas_before, committed_after,
                      excused):
    """Positions whose canvas outcome a raised near-tie flag leaves open, from
    the per-position values the oracle decided with: (bool mask [L], whole)
    where `whole` means the flag decides the whole canvas (the stop test).

      N1  an excused draw: that position's committed token
      N2  cumulative entropy at the EB cut within the window of gamma, and
      N3  the entropies at the cut within the window of each other: the open
          positions whose entropy lies between the last committed and the
          first left-out entropy, widened by the window
      N4  the stop test: the whole canvas
      N5  pmax within the window of the threshold, or the pmax values at the
          quota cut within the relative window: those positions
      N6  a committed position whose pmax is within the window of
          editing_threshold and whose argmax moved
    """
    H = np.asarray(H, np.float64)
    pmax = np.asarray(pmax, np.float64)
    open_before = np.asarray(open_before, bool)
    L = H.shape[0]
    flag = np.zeros(L, bool)
    flag |= np.asarray(excused, bool)
    if mg["stop_margin"] <= STOP_WINDOW:
        return flag, True
    final = bool(mg["fired"]) or s == cfg.num_steps - 1
    if not final and cfg.rule in (O.RULE_EB, O.RULE_EB_MI):
        if mg["cum_margin"] <= N2_WINDOW or mg["cut_gap"] <= CUT_WINDOW:
            w = max(N2_WINDOW, CUT_WINDOW)
            newc = open_before & (np.asarray(committed_after) != 0)
            left = open_before & ~newc
            h_in = H[newc].max() if newc.any() else None
            h_out = H[left].min() if left.any() else None
            lo = (h_in if h_in is not None else h_out) - w
            hi = (h_out if h_out is not None else h_in) + w
            flag |= open_before & (H >= lo) & (H <= hi)
    if not final and cfg.rule == O.RULE_BR:
        if mg["br_margin"] <= BR_WINDOW:
            flag |= open_before & (np.abs(pmax - cfg.threshold) <= BR_WINDOW)
        if mg["quota_gap"] <= QUOTA_WINDOW:
            below = np.nonzero(open_before & ~(pmax >= cfg.threshold))[0]
            order = below[np.lexsort((below, -pmax[below]))]
            q = min(cfg.quota, order.size)
            if 0 < q < order.size:
                p_in, p_out = pmax[order[q - 1]], pmax[order[q]]
                flag |= (open_before & ~(pmax >= cfg.threshold)
                         & (pmax >= p_out * (1 - QUOTA_WINDOW)) & (pmax <= p_in * (1 + QUOTA_WINDOW)))
    if not bool(mg["fired"]) and cfg.editing_threshold >= 0.0 and mg["edit_margin"] <= BR_WINDOW:
        moved = ~open_before & (np.asarray(amax) != np.asarray(canvas_before))
        flag |= moved & (np.abs(pmax - cfg.editing_threshold) <= BR_WINDOW)
    return flag, False


def compare_canvas(stats, st, i, s, gpu_state, mg, decided):
    """Canvas-level state after the step.  A difference from the oracle is
    excused (and the oracle takes over the GPU's state: a resync) only when
    every differing position is one a raised near-tie flag names; anything
    else fails.  `decided` holds the per-position values the oracle decided
    with (H, pmax, amax), the state before the step (open_before,
    canvas_before) and the positions whose draw differed within the N1
    window (excused)."""
    cv, cm, sp = gpu_state
    diff = (st.canvas[i] != cv) | (st.committed[i] != cm)
    stop_differs = int(st.stop[i]) != int(sp)
    if not diff.any() and not stop_differs:
        return
    flag, whole = flagged_positions(
        st.cfg, s, mg, decided["H"], decided["pmax"], decided["amax"], decided["open_before"],
        decided["canvas_before"], st.committed[i], decided["excused"])
    ok = whole or not (diff & ~flag).any()
    if stop_differs and not whole:
        # a flipped commit may leave nothing open on one side only
        ok = ok and diff.any() and {int(st.stop[i]), int(sp)} == {0, O.STOP_ALL_COMMITTED}
    if not ok:
        where = np.nonzero(diff & ~flag)[0]
        raise AssertionError(
            f"canvas {i} step {s}: state differs at unflagged positions {where[:8]} "
            f"(stop oracle {st.stop[i]} gpu {sp}); margins {mg}")
    stats.resyncs += 1
    stats.flags.append((i, s, "whole" if whole else np.nonzero(flag)[0][:8].tolist()))
    st.canvas[i] = cv
    st.committed[i] = cm
    st.stop[i] = sp
