"""CPU reference ("oracle") of the entropy-bound canvas sampler.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library (``entropy_bound_canvas_b200``) never imports, loads or calls it.

The arithmetic lives in ``eb_oracle.c`` (plain C, float64, single thread);
this module only compiles it with gcc on first use and marshals numpy arrays
through ctypes.  Logits are numpy arrays: ``float32`` for fp32 logits and
``uint16`` raw bit patterns for bf16 logits.

Parity of the functions pinned by the CPU tests (``tests/test_oracle_pins.py``):
Philox4x32-10, the temperature schedule, the entropy/argmax statistics, the
two-level Gumbel-max draw, the commit rules, the adaptive stop and renoise.
Full multi-step trajectories at the large synthetic configurations are
pinned only through these parts (the pages print no worked trajectory).
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eb_oracle.c")
_HDR = os.path.join(_HERE, "eb_oracle.h")
_LIB_PATH = os.path.join(_HERE, "_build", "libeb_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1
RULE_EB, RULE_BR, RULE_EB_MI = 0, 1, 2
STOP_ACTIVE, STOP_ADAPTIVE, STOP_ALL_COMMITTED, STOP_LAST_STEP = 0, 1, 2, 3
STREAM_GUMBEL, STREAM_RENOISE, STREAM_INIT, STREAM_GROUP = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile eb_oracle.c into oracle/_build/libeb_oracle.so (IEEE, no FMA contraction)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB_PATH) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Config(C.Structure):
    _fields_ = [
        ("B", C.c_int32), ("L", C.c_int32), ("V", C.c_int32), ("num_steps", C.c_int32),
        ("t_max", C.c_double), ("t_min", C.c_double),
        ("entropy_bound", C.c_double), ("stop_entropy", C.c_double),
        ("stability_steps", C.c_int32), ("rule", C.c_int32),
        ("threshold", C.c_double), ("quota", C.c_int32), ("greedy", C.c_int32),
        ("group_size", C.c_int32), ("canvas_offset", C.c_int32),
        ("seed", C.c_uint64), ("editing_threshold", C.c_double),
    ]


class Margins(C.Structure):
    _fields_ = [
        ("cum_margin", C.c_double), ("cut_gap", C.c_double), ("stop_margin", C.c_double),
        ("br_margin", C.c_double), ("quota_gap", C.c_double), ("mean_H", C.c_double),
        ("n_commit", C.c_int32), ("fired", C.c_int32),
        ("edit_margin", C.c_double), ("n_edit", C.c_int32), ("pad", C.c_int32),
    ]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


@dataclasses.dataclass
class Config:
    """Sampler configuration (same meaning as the library's eb_config_t)."""
    B: int = 1
    L: int = 256
    V: int = 262144
    num_steps: int = 48
    t_max: float = 0.8
    t_min: float = 0.4
    entropy_bound: float = 0.1
    stop_entropy: float = 0.005
    stability_steps: int = 1
    rule: int = RULE_EB
    threshold: float = 0.9
    quota: int = 6
    greedy: int = 0
    group_size: int = 64
    canvas_offset: int = 0
    seed: int = 0
    editing_threshold: float = -1.0

    def c(self) -> _Config:
        return _Config(**{f.name: getattr(self, f.name) for f in dataclasses.fields(self)})


def _p(a, ct):
    return a.ctypes.data_as(C.POINTER(ct))


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            u32p, i32p, u8p, f64p = (C.POINTER(C.c_uint32), C.POINTER(C.c_int32),
                                     C.POINTER(C.c_uint8), C.POINTER(C.c_double))
            cfgp = C.POINTER(_Config)
            L.ebo_philox4x32_10.argtypes = [u32p, u32p, u32p]
            L.ebo_philox4x32_10.restype = None
            L.ebo_draw_word.argtypes = [C.c_uint64] + [C.c_uint32] * 4 + [C.c_int]
            L.ebo_draw_word.restype = C.c_uint32
            L.ebo_uniform.argtypes = [C.c_uint32]
            L.ebo_uniform.restype = C.c_double
            L.ebo_gumbel.argtypes = [C.c_uint32]
            L.ebo_gumbel.restype = C.c_double
            L.ebo_uniform_token.argtypes = [C.c_uint32, C.c_uint32]
            L.ebo_uniform_token.restype = C.c_uint32
            L.ebo_temperature.argtypes = [cfgp, C.c_int]
            L.ebo_temperature.restype = C.c_double
            L.ebo_row_stats.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_double,
                                        f64p, f64p, i32p, f64p]
            L.ebo_row_stats.restype = None
            L.ebo_slice_record.argtypes = [cfgp, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_double,
                                           C.c_int, C.c_int, C.c_int, C.POINTER(Slice)]
            L.ebo_slice_record.restype = None
            L.ebo_combine_slices.argtypes = [C.POINTER(Slice), C.c_int, C.c_double, f64p, f64p,
                                             i32p, i32p]
            L.ebo_combine_slices.restype = None
            L.ebo_sample.argtypes = [cfgp, C.c_void_p, C.c_int, C.c_double, C.c_int, C.c_int,
                                     C.c_int, f64p, i32p]
            L.ebo_sample.restype = C.c_int32
            L.ebo_sample_flat.argtypes = [cfgp, C.c_void_p, C.c_int, C.c_double, C.c_int,
                                          C.c_int, C.c_int, f64p]
            L.ebo_sample_flat.restype = C.c_int32
            L.ebo_init_canvas.argtypes = [cfgp, C.c_int, i32p, u8p, u8p, i32p]
            L.ebo_init_canvas.restype = None
            L.ebo_canvas_decide.argtypes = [cfgp, C.c_int, C.c_int, f64p, i32p, f64p, i32p,
                                            i32p, u8p, u8p, i32p, i32p, C.POINTER(Margins)]
            L.ebo_canvas_decide.restype = None
            L.ebo_step_canvas.argtypes = [cfgp, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                          i32p, u8p, u8p, i32p, i32p,
                                          f64p, i32p, f64p, i32p, f64p, i32p,
                                          C.POINTER(Margins)]
            L.ebo_step_canvas.restype = C.c_int
            _lib = L
    return _lib


# --------------------------------------------------------------------------- draws

def philox4x32_10(ctr, key):
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    lib().ebo_philox4x32_10(_p(c, C.c_uint32), _p(k, C.c_uint32), _p(o, C.c_uint32))
    return o


def draw_word(seed, c0, c1, c2, c3, word):
    return int(lib().ebo_draw_word(seed, c0, c1, c2, c3, word))


def uniform(x):
    return float(lib().ebo_uniform(x))


def gumbel(x):
    return float(lib().ebo_gumbel(x))


def uniform_token(x, V):
    return int(lib().ebo_uniform_token(x, V))


def temperature(cfg: Config, s: int) -> float:
    c = cfg.c()
    return float(lib().ebo_temperature(C.byref(c), s))


# --------------------------------------------------------------------------- per position

def _row(row):
    row = np.ascontiguousarray(row)
    if row.dtype == np.float32:
        return row, F32
    if row.dtype == np.uint16:
        return row, BF16
    raise TypeError("logits rows must be float32 or uint16 (bf16 bits)")


def row_stats(row, inv_T: float):
    """(H, pmax, amax, H_direct) of one logits row."""
    r, dt = _row(row)
    H, pm, Hd = C.c_double(), C.c_double(), C.c_double()
    am = C.c_int32()
    lib().ebo_row_stats(r.ctypes.data, dt, r.size, inv_T, C.byref(H), C.byref(pm),
                        C.byref(am), C.byref(Hd))
    return H.value, pm.value, am.value, Hd.value


def sample(cfg: Config, row, inv_T: float, b: int, l: int, s: int):
    """Two-level Gumbel-max draw: (token, margin, group)."""
    r, dt = _row(row)
    c = cfg.c()
    mg, gr = C.c_double(), C.c_int32()
    x = lib().ebo_sample(C.byref(c), r.ctypes.data, dt, inv_T, b, l, s, C.byref(mg), C.byref(gr))
    return int(x), mg.value, gr.value


class Slice(C.Structure):
    _fields_ = [("S", C.c_double), ("W", C.c_double), ("zmax", C.c_double),
                ("gscore", C.c_double), ("amax", C.c_int32), ("sample", C.c_int32)]


def slice_record(cfg: Config, row_slice, v_off: int, inv_T: float, b: int, l: int, s: int):
    """A vocabulary slice's contribution (ebo_slice_t) for one position."""
    r, dt = _row(row_slice)
    c = cfg.c()
    out = Slice()
    lib().ebo_slice_record(C.byref(c), r.ctypes.data, dt, r.size, v_off, inv_T, b, l, s,
                           C.byref(out))
    return out


def combine_slices(slices, inv_T: float):
    """(H, pmax, amax, sample) of a row from its slices in increasing v_off."""
    arr = (Slice * len(slices))(*slices)
    H, pm = C.c_double(), C.c_double()
    am, x = C.c_int32(), C.c_int32()
    lib().ebo_combine_slices(arr, len(slices), inv_T, C.byref(H), C.byref(pm), C.byref(am),
                             C.byref(x))
    return H.value, pm.value, am.value, x.value


def sample_flat(cfg: Config, row, inv_T: float, b: int, l: int, s: int):
    r, dt = _row(row)
    c = cfg.c()
    mg = C.c_double()
    x = lib().ebo_sample_flat(C.byref(c), r.ctypes.data, dt, inv_T, b, l, s, C.byref(mg))
    return int(x), mg.value


# --------------------------------------------------------------------------- canvas state

def lmhead_logits(hidden_bits, weight_bits):
    """The decoder's logits from its last hidden states and the LM head:
    z[row, v] = sum_k h[row, k] W[v, k], in float64 (diffusers "DiffusionGemma"
    page, `__call__` parameters: the pipeline's logits are the decoder's
    [batch, canvas_length, vocab_size] output; model card, summary table:
    a vocabulary of about 262K).  Inputs are bf16 bit patterns (uint16
    [rows, d] and [V, d]); the product is numpy's float64 matrix product,
    which is exact for inputs whose products and sums are exactly
    representable (the synthetic recipe's multiples of 1/64)."""
    return decode_bf16(hidden_bits) @ decode_bf16(weight_bits).T


def decode_bf16(bits):
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


class State:
    """Per-canvas sampler state the oracle carries between steps."""

    def __init__(self, cfg: Config, canvases=None):
        self.cfg = cfg
        self.canvases = list(range(cfg.B)) if canvases is None else list(canvases)
        n, L = len(self.canvases), cfg.L
        self.canvas = np.zeros((n, L), np.int32)
        self.committed = np.zeros((n, L), np.uint8)
        self.stop = np.zeros(n, np.uint8)
        self.prev = np.zeros((n, L), np.int32)
        self.stable = np.zeros(n, np.int32)

    def init(self):
        c = self.cfg.c()
        for i, b in enumerate(self.canvases):
            st, sb = np.zeros(1, np.uint8), np.zeros(1, np.int32)
            cv, cm = self.canvas[i], self.committed[i]
            lib().ebo_init_canvas(C.byref(c), b, _p(cv, C.c_int32), _p(cm, C.c_uint8),
                                  _p(st, C.c_uint8), _p(sb, C.c_int32))
            self.stop[i], self.stable[i] = st[0], sb[0]
        return self

    def copy(self):
        o = State(self.cfg, self.canvases)
        for k in ("canvas", "committed", "stop", "prev", "stable"):
            setattr(o, k, getattr(self, k).copy())
        return o


def _scalar_views(st: State, i: int):
    stop = st.stop[i:i + 1]
    stable = st.stable[i:i + 1]
    return stop, stable


def step_canvas(st: State, i: int, logits_canvas, s: int):
    """One full step of canvas st.canvases[i]; logits_canvas is its [L, V] block.

    Returns None if the canvas was already stopped, else a dict of the
    per-position outputs and the decision margins."""
    cfg = st.cfg
    lg = np.ascontiguousarray(logits_canvas)
    dt = F32 if lg.dtype == np.float32 else BF16
    assert lg.shape == (cfg.L, cfg.V), lg.shape
    L = cfg.L
    H = np.zeros(L, np.float64)
    amax = np.zeros(L, np.int32)
    pmax = np.zeros(L, np.float64)
    smp = np.zeros(L, np.int32)
    smg = np.zeros(L, np.float64)
    sgr = np.zeros(L, np.int32)
    mg = Margins()
    c = cfg.c()
    cv, cm, pv = st.canvas[i], st.committed[i], st.prev[i]
    stop, stable = _scalar_views(st, i)
    open_before = (cm == 0).copy()
    ran = lib().ebo_step_canvas(
        C.byref(c), lg.ctypes.data, dt, st.canvases[i], s,
        _p(cv, C.c_int32), _p(cm, C.c_uint8), _p(stop, C.c_uint8), _p(pv, C.c_int32),
        _p(stable, C.c_int32), _p(H, C.c_double), _p(amax, C.c_int32), _p(pmax, C.c_double),
        _p(smp, C.c_int32), _p(smg, C.c_double), _p(sgr, C.c_int32), C.byref(mg))
    if not ran:
        return None
    return dict(H=H, amax=amax, pmax=pmax, sample=smp, sample_margin=smg, sample_group=sgr,
                open_before=open_before, margins=mg.as_dict())


def canvas_decide(st: State, i: int, s: int, H, amax, pmax, sample_tok):
    """Canvas-level decisions of one step from given per-position quantities."""
    cfg = st.cfg
    c = cfg.c()
    H = np.ascontiguousarray(H, np.float64)
    amax = np.ascontiguousarray(amax, np.int32)
    pmax = np.ascontiguousarray(pmax, np.float64)
    sample_tok = np.ascontiguousarray(sample_tok, np.int32)
    cv, cm, pv = st.canvas[i], st.committed[i], st.prev[i]
    stop, stable = _scalar_views(st, i)
    mg = Margins()
    lib().ebo_canvas_decide(C.byref(c), st.canvases[i], s, _p(H, C.c_double),
                            _p(amax, C.c_int32), _p(pmax, C.c_double), _p(sample_tok, C.c_int32),
                            _p(cv, C.c_int32), _p(cm, C.c_uint8), _p(stop, C.c_uint8),
                            _p(pv, C.c_int32), _p(stable, C.c_int32), C.byref(mg))
    return mg.as_dict()
