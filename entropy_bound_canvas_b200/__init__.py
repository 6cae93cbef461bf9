"""Python binding of the B200 entropy-bound canvas sampler (libebsampler.so).

Argument marshalling only: every step of the sampler runs in the CUDA
kernels behind the C ABI of ``include/eb_sampler.h``.  PyTorch supplies device
buffers and the current stream; nothing here computes on the data, and there
is no CPU fallback -- importing fails loudly when the library is missing.

    from entropy_bound_canvas_b200 import EBSampler
    s = EBSampler(B=1, L=256, V=262144, seed=1)
    canvas, committed, stop = s.new_canvas()
    H, amax = s.outputs()
    for step in range(48):
        s.step(logits[step], step, canvas, committed, H, amax, stop)
        if s.done(stop):
            break
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libebsampler.so")

F32, BF16 = 0, 1
RULE_ENTROPY_BOUND, RULE_BLOCK_REFINEMENT, RULE_ENTROPY_BOUND_MI = 0, 1, 2
STOP_ACTIVE, STOP_ADAPTIVE, STOP_ALL_COMMITTED, STOP_LAST_STEP = 0, 1, 2, 3
STATUS_BAD_TOKEN, STATUS_NONFINITE, STATUS_TIMEOUT = 1, 2, 4
GUMBEL_GROUP = 64

EB_OK = 0
ERRORS = {
    1: "EB_ERR_INVALID_ARG", 2: "EB_ERR_CUDA", 3: "EB_ERR_OUT_OF_MEMORY",
    4: "EB_ERR_STEP_ORDER", 5: "EB_ERR_UNSUPPORTED", 6: "EB_ERR_OVERFLOW",
    7: "EB_ERR_DEVICE_STATUS",
}


class EBError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({_lib().eb_strerror(code).decode()})")


class Config(C.Structure):
    """eb_config_t (same field order and types as include/eb_sampler.h)."""
    _fields_ = [
        ("B", C.c_int32), ("L", C.c_int32), ("V", C.c_int32), ("num_steps", C.c_int32),
        ("t_max", C.c_double), ("t_min", C.c_double),
        ("entropy_bound", C.c_double), ("stop_entropy", C.c_double),
        ("stability_steps", C.c_int32), ("rule", C.c_int32),
        ("threshold", C.c_double), ("quota", C.c_int32), ("greedy", C.c_int32),
        ("canvas_offset", C.c_int32), ("seed", C.c_uint64),
        ("editing_threshold", C.c_double), ("vocab_offset", C.c_int32), ("vocab_total", C.c_int32),
    ]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m entropy_bound_canvas_b200.build` "
                "(nvcc, sm_100a). There is no CPU fallback.")
        L = C.CDLL(LIB_PATH)
        vp, i32, u32p = C.c_void_p, C.c_int, C.POINTER(C.c_uint32)
        L.eb_config_default.argtypes = [C.POINTER(Config), C.c_int32, C.c_int32, C.c_int32]
        L.eb_config_default.restype = None
        L.eb_sampler_init.argtypes = [C.POINTER(vp), C.POINTER(Config), i32]
        L.eb_sampler_init.restype = i32
        L.eb_sampler_init_canvas.argtypes = [vp, vp, vp, vp, vp]
        L.eb_sampler_init_canvas.restype = i32
        L.eb_sampler_step.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp, vp, vp]
        L.eb_sampler_step.restype = i32
        L.eb_canvas_done.argtypes = [vp, vp, i32, C.POINTER(C.c_int), vp]
        L.eb_canvas_done.restype = i32
        L.eb_sampler_status.argtypes = [vp, u32p, i32, vp]
        L.eb_sampler_status.restype = i32
        L.eb_sampler_draws.argtypes = [vp, vp, vp, vp]
        L.eb_sampler_draws.restype = i32
        L.eb_sampler_set_state.argtypes = [vp, vp, vp, i32, vp]
        L.eb_sampler_set_state.restype = i32
        L.eb_sampler_step_slice.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp]
        L.eb_sampler_step_slice.restype = i32
        L.eb_sampler_combine.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp, vp, vp]
        L.eb_sampler_combine.restype = i32
        L.eb_slice_record_bytes.argtypes = []
        L.eb_slice_record_bytes.restype = C.c_size_t
        L.eb_sampler_set_split_event.argtypes = [vp, vp]
        L.eb_sampler_set_split_event.restype = i32
        L.eb_sampler_set_wait_limit.argtypes = [vp, C.c_uint64]
        L.eb_sampler_set_wait_limit.restype = i32
        L.eb_sampler_workspace_bytes.argtypes = [vp]
        L.eb_sampler_workspace_bytes.restype = C.c_size_t
        L.eb_sampler_destroy.argtypes = [vp]
        L.eb_sampler_destroy.restype = None
        L.eb_strerror.argtypes = [i32]
        L.eb_strerror.restype = C.c_char_p
        L.eb_version.argtypes = []
        L.eb_version.restype = i32
        L.eb_lmhead_logits.argtypes = [vp, vp, i32, i32, i32, vp, vp]
        L.eb_lmhead_logits.restype = i32
        L.eb_lmhead_reserve.argtypes = [vp, i32]
        L.eb_lmhead_reserve.restype = i32
        L.eb_lmhead_step.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp]
        L.eb_lmhead_step.restype = i32
        _LIB = L
    return _LIB


def library():
    """The loaded ctypes library (raises ImportError if it was not built)."""
    return _lib()


def default_config(B: int, L: int, V: int) -> Config:
    c = Config()
    _lib().eb_config_default(C.byref(c), B, L, V)
    return c


def make_config(B, L, V, **kw) -> Config:
    c = default_config(B, L, V)
    for k, v in kw.items():
        if not hasattr(c, k):
            raise TypeError(f"unknown config field {k!r}")
        setattr(c, k, v)
    return c


def _check(rc: int, what: str):
    if rc != EB_OK:
        raise EBError(rc, what)


def _torch():
    import torch
    return torch


def lmhead_logits(hidden, weight, out=None):
    """The LM head's logits hidden @ weight^T (bf16 [rows, d] and [V, d] on
    one device) formed by the fused LM-head kernel's tensor-core contraction,
    written as fp32 [rows, V]: the diagnostic form of eb_lmhead_step."""
    torch = _torch()
    for t, n in ((hidden, "hidden"), (weight, "weight")):
        if t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous 2-D bf16 tensor")
    rows, d = hidden.shape
    V = weight.shape[0]
    if weight.shape[1] != d:
        raise ValueError("hidden and weight disagree on the hidden size")
    if out is None:
        out = torch.empty((rows, V), dtype=torch.float32, device=hidden.device)
    stream = torch.cuda.current_stream(hidden.device).cuda_stream
    _check(_lib().eb_lmhead_logits(C.c_void_p(hidden.data_ptr()), C.c_void_p(weight.data_ptr()),
                                   int(rows), int(V), int(d), C.c_void_p(out.data_ptr()),
                                   C.c_void_p(stream)), "eb_lmhead_logits")
    return out


def shard_canvases(B: int, world: int, rank: int):
    """Contiguous split of B canvases over `world` ranks: (canvas_offset, count)."""
    base, extra = divmod(B, world)
    count = base + (1 if rank < extra else 0)
    offset = rank * base + min(rank, extra)
    return offset, count


class EBSampler:
    """One sampler handle on one CUDA device (see include/eb_sampler.h)."""

    def __init__(self, B: int, L: int, V: int, device=None, **config):
        torch = _torch()
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None
                                   else torch.device(device).index or 0)
        self.cfg = make_config(B, L, V, **config)
        self.B, self.L, self.V = B, L, V
        h = C.c_void_p()
        _check(_lib().eb_sampler_init(C.byref(h), C.byref(self.cfg), self.device.index),
               "eb_sampler_init")
        self._h = h

    # -- helpers --------------------------------------------------------------
    def _stream(self):
        return C.c_void_p(_torch().cuda.current_stream(self.device).cuda_stream)

    def _ptr(self, t, dtype, shape, name):
        torch = _torch()
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch tensor")
        if t.device != self.device:
            raise ValueError(f"{name} is on {t.device}, sampler is on {self.device}")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return C.c_void_p(t.data_ptr())

    # -- buffers --------------------------------------------------------------
    def new_canvas(self):
        """Allocate (canvas, committed, stop_flags) and start fresh canvases."""
        torch = _torch()
        canvas = torch.empty((self.B, self.L), dtype=torch.int32, device=self.device)
        committed = torch.empty((self.B, self.L), dtype=torch.uint8, device=self.device)
        stop = torch.empty((self.B,), dtype=torch.uint8, device=self.device)
        self.init_canvas(canvas, committed, stop)
        return canvas, committed, stop

    def outputs(self):
        """Allocate (entropies, argmax) output buffers."""
        torch = _torch()
        return (torch.empty((self.B, self.L), dtype=torch.float32, device=self.device),
                torch.empty((self.B, self.L), dtype=torch.int32, device=self.device))

    # -- ABI calls ------------------------------------------------------------
    def init_canvas(self, canvas, committed, stop_flags):
        torch = _torch()
        _check(_lib().eb_sampler_init_canvas(
            self._h, self._ptr(canvas, torch.int32, (self.B, self.L), "canvas"),
            self._ptr(committed, torch.uint8, (self.B, self.L), "committed"),
            self._ptr(stop_flags, torch.uint8, (self.B,), "stop_flags"), self._stream()),
            "eb_sampler_init_canvas")

    def step(self, logits, step: int, canvas, committed, entropies, argmax, stop_flags):
        torch = _torch()
        if logits.dtype == torch.float32:
            dt = F32
        elif logits.dtype == torch.bfloat16:
            dt = BF16
        else:
            raise TypeError("logits must be float32 or bfloat16")
        if logits.device != self.device or tuple(logits.shape) != (self.B, self.L, self.V):
            raise ValueError(f"logits must be [{self.B}, {self.L}, {self.V}] on {self.device}")
        if not logits.is_contiguous():
            raise ValueError("logits must be contiguous")
        _check(_lib().eb_sampler_step(
            self._h, C.c_void_p(logits.data_ptr()), dt, int(step),
            self._ptr(canvas, torch.int32, (self.B, self.L), "canvas"),
            self._ptr(committed, torch.uint8, (self.B, self.L), "committed"),
            self._ptr(entropies, torch.float32, (self.B, self.L), "entropies"),
            self._ptr(argmax, torch.int32, (self.B, self.L), "argmax"),
            self._ptr(stop_flags, torch.uint8, (self.B,), "stop_flags"), self._stream()),
            "eb_sampler_step")

    # -- the sampler fused into the LM head --------------------------------------
    def lmhead_step(self, hidden, weight, step: int, canvas, committed, entropies, argmax,
                    stop_flags):
        """A step from the decoder's hidden states: hidden [B, L, d] (or
        [B*L, d]) and the LM head weight [V, d], both bf16; the logits are
        formed on the tensor cores and reduced on chip (never written)."""
        torch = _torch()
        for t, n in ((hidden, "hidden"), (weight, "weight")):
            if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != self.device:
                raise ValueError(f"{n} must be a contiguous bf16 tensor on {self.device}")
        d = int(hidden.shape[-1])
        if hidden.numel() != self.B * self.L * d or tuple(weight.shape) != (self.V, d):
            raise ValueError(f"hidden must hold [{self.B}*{self.L}, d], weight [{self.V}, d]")
        if not getattr(self, "_lm_reserved", False):
            _check(_lib().eb_lmhead_reserve(self._h, d), "eb_lmhead_reserve")
            self._lm_reserved = True
        _check(_lib().eb_lmhead_step(
            self._h, C.c_void_p(hidden.data_ptr()), C.c_void_p(weight.data_ptr()), d, int(step),
            self._ptr(canvas, torch.int32, (self.B, self.L), "canvas"),
            self._ptr(committed, torch.uint8, (self.B, self.L), "committed"),
            self._ptr(entropies, torch.float32, (self.B, self.L), "entropies"),
            self._ptr(argmax, torch.int32, (self.B, self.L), "argmax"),
            self._ptr(stop_flags, torch.uint8, (self.B,), "stop_flags"), self._stream()),
            "eb_lmhead_step")

    # -- vocabulary-sharded logits ---------------------------------------------
    def slice_records(self):
        """A records buffer for one slice: [B, L, record bytes] uint8."""
        torch = _torch()
        n = int(_lib().eb_slice_record_bytes())
        return torch.empty((self.B, self.L, n), dtype=torch.uint8, device=self.device)

    def step_slice(self, logits, step: int, committed, stop_flags, records):
        """This device's vocabulary slice of a step: per-position records."""
        torch = _torch()
        dt = self._dtype(logits)
        n = int(_lib().eb_slice_record_bytes())
        _check(_lib().eb_sampler_step_slice(
            self._h, C.c_void_p(logits.data_ptr()), dt, int(step),
            self._ptr(committed, torch.uint8, (self.B, self.L), "committed"),
            self._ptr(stop_flags, torch.uint8, (self.B,), "stop_flags"),
            self._ptr(records, torch.uint8, (self.B, self.L, n), "records"), self._stream()),
            "eb_sampler_step_slice")

    def combine(self, all_records, step: int, canvas, committed, entropies, argmax, stop_flags):
        """Every slice's records ([n_slices, B, L, record bytes], slice order) ->
        the step's results and canvas decisions, as step() gives them."""
        torch = _torch()
        n = int(_lib().eb_slice_record_bytes())
        if all_records.dim() != 4 or tuple(all_records.shape[1:]) != (self.B, self.L, n):
            raise ValueError(f"records must be [n_slices, {self.B}, {self.L}, {n}]")
        _check(_lib().eb_sampler_combine(
            self._h, self._ptr(all_records, torch.uint8, None, "records"),
            int(all_records.shape[0]), int(step),
            self._ptr(canvas, torch.int32, (self.B, self.L), "canvas"),
            self._ptr(committed, torch.uint8, (self.B, self.L), "committed"),
            self._ptr(entropies, torch.float32, (self.B, self.L), "entropies"),
            self._ptr(argmax, torch.int32, (self.B, self.L), "argmax"),
            self._ptr(stop_flags, torch.uint8, (self.B,), "stop_flags"), self._stream()),
            "eb_sampler_combine")

    def step_split(self, logits, step: int, canvas, committed, entropies, argmax, stop_flags,
                   group=None):
        """A step over vocabulary-sharded logits: this rank's slice, one
        all-gather of the records over `group` (ranks ordered by slice), then
        the combine.  Without a process group the handle is the only slice."""
        torch = _torch()
        rec = self.slice_records()
        self.step_slice(logits, step, committed, stop_flags, rec)
        world = 1
        if group is not None or (torch.distributed.is_available()
                                 and torch.distributed.is_initialized()):
            world = torch.distributed.get_world_size(group)
        if world == 1:
            allr = rec.unsqueeze(0)
        else:
            allr = torch.empty((world,) + tuple(rec.shape), dtype=rec.dtype, device=rec.device)
            torch.distributed.all_gather_into_tensor(allr, rec, group=group)
        self.combine(allr, step, canvas, committed, entropies, argmax, stop_flags)

    def _dtype(self, logits):
        torch = _torch()
        if logits.dtype == torch.float32:
            dt = F32
        elif logits.dtype == torch.bfloat16:
            dt = BF16
        else:
            raise TypeError("logits must be float32 or bfloat16")
        if logits.device != self.device or tuple(logits.shape) != (self.B, self.L, self.V):
            raise ValueError(f"logits must be [{self.B}, {self.L}, {self.V}] on {self.device}")
        if not logits.is_contiguous():
            raise ValueError("logits must be contiguous")
        return dt

    def step_ptr(self, logits_ptr: int, dtype: int, step: int, canvas_ptr: int,
                 committed_ptr: int, entropies_ptr: int, argmax_ptr: int, stop_ptr: int,
                 stream_ptr: int = 0) -> int:
        """Raw pointer form of eb_sampler_step (returns the status code)."""
        return _lib().eb_sampler_step(self._h, C.c_void_p(logits_ptr), dtype, step,
                                      C.c_void_p(canvas_ptr), C.c_void_p(committed_ptr),
                                      C.c_void_p(entropies_ptr), C.c_void_p(argmax_ptr),
                                      C.c_void_p(stop_ptr), C.c_void_p(stream_ptr))

    def done(self, stop_flags, b: int = -1, check_status: bool = True) -> bool:
        torch = _torch()
        d = C.c_int(0)
        rc = _lib().eb_canvas_done(self._h, self._ptr(stop_flags, torch.uint8, (self.B,),
                                                      "stop_flags"), b, C.byref(d), self._stream())
        if rc != EB_OK and (check_status or rc != 7):
            raise EBError(rc, "eb_canvas_done")
        return bool(d.value)

    def status(self, clear: bool = False) -> int:
        s = C.c_uint32(0)
        _check(_lib().eb_sampler_status(self._h, C.byref(s), int(clear), self._stream()),
               "eb_sampler_status")
        return int(s.value)

    def draws(self):
        """(sample [B, L] int32, pmax [B, L] float32) of the last step."""
        torch = _torch()
        smp = torch.empty((self.B, self.L), dtype=torch.int32, device=self.device)
        pm = torch.empty((self.B, self.L), dtype=torch.float32, device=self.device)
        _check(_lib().eb_sampler_draws(self._h, C.c_void_p(smp.data_ptr()),
                                       C.c_void_p(pm.data_ptr()), self._stream()),
               "eb_sampler_draws")
        return smp, pm

    def set_state(self, prev_argmax, stable=None, next_step: int = 0):
        torch = _torch()
        sp = self._ptr(stable, torch.int32, (self.B,), "stable") if stable is not None else None
        _check(_lib().eb_sampler_set_state(
            self._h, self._ptr(prev_argmax, torch.int32, (self.B, self.L), "prev_argmax"),
            sp, next_step, self._stream()), "eb_sampler_set_state")

    def set_split_event(self, event=None):
        """Record `event` (a torch.cuda.Event, or None to stop) between the two
        kernels of every following step, for timing them apart."""
        ptr = None
        if event is not None:
            if not event.cuda_event:  # torch creates the CUDA event on first record
                event.record(_torch().cuda.current_stream(self.device))
            ptr = C.c_void_p(event.cuda_event)
        _check(_lib().eb_sampler_set_split_event(self._h, ptr), "eb_sampler_set_split_event")

    def set_wait_limit(self, limit_ns: int = 0):
        """Limit (ns) of the stream kernel's pipeline waits; 0 = the default
        2 s.  A diagnostic hook: a tiny limit makes a wait run out, which sets
        STATUS_TIMEOUT instead of hanging (see include/eb_sampler.h)."""
        _check(_lib().eb_sampler_set_wait_limit(self._h, int(limit_ns)),
               "eb_sampler_set_wait_limit")

    def workspace_bytes(self) -> int:
        return int(_lib().eb_sampler_workspace_bytes(self._h))

    def close(self):
        if getattr(self, "_h", None):
            _lib().eb_sampler_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
