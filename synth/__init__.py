"""Seeded synthetic decoder logits and the five sampler workloads.

Input generator shared by the tests, the benchmark and the smoke check.  It
holds none of the sampler's arithmetic: it only produces [B, L, V] logits
(see eb_synth.h for the recipe) and names the sampler settings each workload
is run with.  The same element function runs on the GPU (for full-size
inputs) and on the host (for CPU tests); both give identical bits.

Workloads (shapes of the model card: canvas 256, vocabulary ~262K; the
decoder itself needs trained weights and is out of scope):
  tiny   B=1,  L=16,  V=1024,   fp32, seed 0, N(0,1) + target boost
         U(12,20) for a confident fraction 10% -> 100%, else U(0,4)
  canvas B=1,  L=256, V=262144, bf16, seed 1, confident fraction 5% -> 100%
  serve  B=8,  L=256, V=262144, bf16, seed 2, staggered ramps
         f_b(s) = min(1, 0.05 + 0.95 s / (22 + 3 b))
  br     B=4,  L=256, V=262144, bf16, seed 3, canvas generator, block
         refinement (threshold 0.9, quota ceil(256/48) = 6), greedy
  stress B=32, L=256, V=262144, fp32, seed 4, -2.75 ln(rank) over a keyed
         permutation + N(0, 0.5^2) + U(0, 20) target boost
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eb_synth.cu")
_HDR = os.path.join(_HERE, "eb_synth.h")
LIB_PATH = os.path.join(_HERE, "_build", "libebsynth.so")
_lock = threading.Lock()
_lib = None

TARGET_BOOST, ZIPF = 0, 1
F32, BF16 = 0, 1


class Params(C.Structure):
    _fields_ = [
        ("kind", C.c_int32), ("dtype", C.c_int32),
        ("B", C.c_int32), ("L", C.c_int32), ("V", C.c_int32), ("num_steps", C.c_int32),
        ("seed", C.c_uint64),
        ("f0", C.c_float), ("f1", C.c_float), ("ramp_base", C.c_float),
        ("ramp_per_canvas", C.c_float),
        ("conf_lo", C.c_float), ("conf_hi", C.c_float), ("unc_lo", C.c_float),
        ("unc_hi", C.c_float), ("noise_sd", C.c_float),
        ("zipf_scale", C.c_float), ("zipf_noise_sd", C.c_float), ("boost_lo", C.c_float),
        ("boost_hi", C.c_float),
    ]


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    L: int
    V: int
    dtype: int
    seed: int
    kind: int = TARGET_BOOST
    num_steps: int = 48
    f0: float = 0.05
    f1: float = 1.0
    ramp_base: float = 47.0
    ramp_per_canvas: float = 0.0
    conf_lo: float = 12.0
    conf_hi: float = 20.0
    unc_lo: float = 0.0
    unc_hi: float = 4.0
    noise_sd: float = 1.0
    zipf_scale: float = 2.75
    zipf_noise_sd: float = 0.5
    boost_lo: float = 0.0
    boost_hi: float = 20.0
    # sampler settings the workload is run with
    rule: int = 0
    greedy: int = 0
    quota: int = 6
    threshold: float = 0.9
    entropy_bound: float = 0.1
    stop_entropy: float = 0.005
    stability_steps: int = 1
    t_max: float = 0.8
    t_min: float = 0.4
    editing_threshold: float = -1.0

    @property
    def elt(self) -> int:
        return 4 if self.dtype == F32 else 2

    @property
    def step_bytes(self) -> int:
        return self.B * self.L * self.V * self.elt

    def params(self) -> Params:
        p = Params()
        for f, _ in Params._fields_:
            setattr(p, f, getattr(self, f))
        return p

    def sampler_config(self) -> dict:
        """Keyword arguments of the sampler config (library and oracle alike)."""
        return dict(num_steps=self.num_steps, t_max=self.t_max, t_min=self.t_min,
                    entropy_bound=self.entropy_bound, stop_entropy=self.stop_entropy,
                    stability_steps=self.stability_steps, rule=self.rule,
                    threshold=self.threshold, quota=self.quota, greedy=self.greedy,
                    seed=self.seed, editing_threshold=self.editing_threshold)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, L=16, V=1024, dtype=F32, seed=0, f0=0.10),
    "canvas": Workload("canvas", B=1, L=256, V=262144, dtype=BF16, seed=1),
    "serve": Workload("serve", B=8, L=256, V=262144, dtype=BF16, seed=2, ramp_base=22.0,
                      ramp_per_canvas=3.0),
    "br": Workload("br", B=4, L=256, V=262144, dtype=BF16, seed=3, rule=1, greedy=1, quota=6),
    "stress": Workload("stress", B=32, L=256, V=262144, dtype=F32, seed=4, kind=ZIPF),
}


def build(force: bool = False) -> str:
    os.makedirs(os.path.dirname(LIB_PATH), exist_ok=True)
    stale = not os.path.exists(LIB_PATH) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB_PATH) for p in (_SRC, _HDR))
    if force or stale:
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
        subprocess.check_call([
            nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-fmad=false",
            "-prec-div=true", "-prec-sqrt=true", "-Xcompiler", "-fPIC,-ffp-contract=off",
            "-shared", "-o", tmp, _SRC])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            L.ebs_generate_device.argtypes = [C.POINTER(Params), C.c_int, C.c_int, C.c_int,
                                              C.c_void_p, C.c_void_p]
            L.ebs_generate_device.restype = C.c_int
            L.ebs_generate_host.argtypes = [C.POINTER(Params), C.c_int, C.c_int, C.c_int,
                                            C.c_int, C.c_int, C.c_void_p]
            L.ebs_generate_host.restype = C.c_int
            L.ebs_log.argtypes = [C.c_float]
            L.ebs_log.restype = C.c_float
            L.ebs_target.argtypes = [C.POINTER(Params), C.c_int, C.c_int]
            L.ebs_target.restype = C.c_uint32
            _lib = L
    return _lib


def generate_host(w: Workload, s: int, b0: int = 0, nb: int | None = None, l0: int = 0,
                  nl: int | None = None) -> np.ndarray:
    """Logits of canvases b0.. and rows l0.. at step s as numpy (float32, or
    uint16 bf16 bits), shape [nb, nl, V]."""
    nb = w.B - b0 if nb is None else nb
    nl = w.L - l0 if nl is None else nl
    out = np.empty((nb, nl, w.V), np.float32 if w.dtype == F32 else np.uint16)
    p = w.params()
    lib().ebs_generate_host(C.byref(p), b0, nb, s, l0, nl, out.ctypes.data)
    return out


def generate_device(w: Workload, s: int, out, b0: int = 0, stream=None):
    """Fill torch tensor `out` ([nb, L, V], float32 or bfloat16, CUDA) with the
    logits of canvases b0 .. b0 + nb - 1 at step s."""
    import torch
    nb = out.shape[0]
    assert tuple(out.shape) == (nb, w.L, w.V) and out.is_contiguous()
    assert out.dtype == (torch.float32 if w.dtype == F32 else torch.bfloat16)
    st = torch.cuda.current_stream(out.device) if stream is None else stream
    p = w.params()
    rc = lib().ebs_generate_device(C.byref(p), b0, nb, s, C.c_void_p(out.data_ptr()),
                                   C.c_void_p(st.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"ebs_generate_device failed: {rc}")


def target(w: Workload, b: int, l: int) -> int:
    p = w.params()
    return int(lib().ebs_target(C.byref(p), b, l))


def log(x: float) -> float:
    return float(lib().ebs_log(x))
