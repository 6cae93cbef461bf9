"""The C-ABI library loads and exports every symbol include/eb_sampler.h
declares; host-side validation works without a GPU (no compute calls)."""
import ctypes as C
import os
import re
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eb_sampler.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(eb_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def E():
    if shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"):
        pytest.skip("nvcc not available")
    from entropy_bound_canvas_b200 import build as B
    B.build()
    import entropy_bound_canvas_b200 as E
    return E


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("eb_sampler_init", "eb_sampler_step", "eb_canvas_done", "eb_sampler_init_canvas",
              "eb_sampler_destroy", "eb_strerror"):
        assert f in names


def test_every_declared_symbol_is_exported(E):
    lib = C.CDLL(E.LIB_PATH)
    missing = [f for f in declared_functions() if not hasattr(lib, f)]
    assert not missing, missing


def test_default_config_matches_model_card(E):
    c = E.default_config(1, 256, 262144)
    assert (c.B, c.L, c.V, c.num_steps) == (1, 256, 262144, 48)
    assert (c.t_max, c.t_min, c.entropy_bound, c.stop_entropy) == (0.8, 0.4, 0.1, 0.005)
    assert c.stability_steps == 1 and c.rule == E.RULE_ENTROPY_BOUND and c.quota == 6
    assert c.threshold == 0.9 and c.greedy == 0
    assert c.editing_threshold == -1.0  # block refinement editing off


def test_strerror_and_version(E):
    lib = E.library()
    assert lib.eb_version() >= 100
    for code in range(0, 8):
        assert lib.eb_strerror(code)
    assert lib.eb_strerror(999) == b"unknown status"


@pytest.mark.parametrize("field,value,code", [
    ("L", 0, 1), ("B", 0, 1), ("V", 0, 1), ("num_steps", 0, 1), ("L", 5000, 6),
    ("B", 5000, 6), ("rule", 7, 1), ("greedy", 2, 1), ("t_max", -0.5, 1),
    ("entropy_bound", -1.0, 1), ("stability_steps", -1, 1), ("quota", -2, 1),
    ("canvas_offset", (1 << 24), 6), ("editing_threshold", float("nan"), 1),
])
def test_init_validates_config_on_host(E, field, value, code):
    lib = E.library()
    c = E.default_config(1, 256, 262144)
    setattr(c, field, value)
    h = C.c_void_p()
    assert lib.eb_sampler_init(C.byref(h), C.byref(c), 0) == code
    assert not h.value


def test_null_arguments_are_rejected(E):
    lib = E.library()
    c = E.default_config(1, 16, 1024)
    assert lib.eb_sampler_init(None, C.byref(c), 0) == 1
    h = C.c_void_p()
    assert lib.eb_sampler_init(C.byref(h), None, 0) == 1
    assert lib.eb_sampler_step(None, None, 0, 0, None, None, None, None, None, None) == 1
    assert lib.eb_canvas_done(None, None, 0, None, None) == 1
    assert lib.eb_sampler_workspace_bytes(None) == 0
    lib.eb_sampler_destroy(None)


def test_shard_canvases_partition(E):
    for B in (1, 5, 8, 33):
        for world in (1, 2, 3, 8):
            parts = [E.shard_canvases(B, world, r) for r in range(world)]
            assert sum(c for _, c in parts) == B
            off = 0
            for o, c in parts:
                assert o == off
                off += c
