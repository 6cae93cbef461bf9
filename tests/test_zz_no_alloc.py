"""eb_row_stats_noalloc, the allocation-free per-row statistics call.

Its scratch is a static device array inside the library, so this file is
collected last and checks that the call gives the same results alone and
after every other test has used the device.  Both entry points are called
through the C ABI.
"""
import ctypes as C
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

EB_OK, EB_ERR_INVALID_ARG, EB_ERR_OVERFLOW = 0, 1, 6
EB_BF16 = 1


def _lib():
    import entropy_bound_canvas_b200 as E
    lib = E.library()
    lib.eb_row_stats_noalloc.argtypes = [C.c_void_p, C.c_int, C.c_int32, C.c_int32, C.c_double,
                                         C.c_void_p, C.c_void_p, C.c_void_p]
    lib.eb_row_stats_noalloc.restype = C.c_int
    return E, lib


def _logits(L, V, seed, dev):
    g = torch.Generator(device="cpu").manual_seed(seed)
    z = torch.randn((L, V), generator=g) * 2.0
    # a confident half: one boosted token per row
    tgt = torch.randint(0, V, (L,), generator=g)
    boost = torch.where(torch.arange(L) % 2 == 0, 14.0, 1.5)
    z[torch.arange(L), tgt] += boost
    return z.to(torch.bfloat16).to(dev)


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a GPU")
def test_noalloc_matches_sampler_step_on_two_calls_in_a_row():
    E, lib = _lib()
    dev = torch.device("cuda", 0)
    L, V, N = 256, 8232, 24  # V % 64 != 0: every row ends in a partial group
    t_max, t_min = 0.8, 0.4
    eb = E.EBSampler(1, L, V, device=dev, num_steps=N, t_max=t_max, t_min=t_min)
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    eb.init_canvas(canvas, committed, stop)
    stream = torch.cuda.current_stream(dev)
    for s in (0, 1):
        z = _logits(L, V, 11 + s, dev)
        eb.step(z.view(1, L, V), s, canvas, committed, H, amax, stop)
        T = t_max + (t_min - t_max) * s / (N - 1)
        Hn = torch.full((L,), float("nan"), dtype=torch.float32, device=dev)
        An = torch.full((L,), -7, dtype=torch.int32, device=dev)
        rc = lib.eb_row_stats_noalloc(C.c_void_p(z.data_ptr()), EB_BF16, L, V, T,
                                      C.c_void_p(Hn.data_ptr()), C.c_void_p(An.data_ptr()),
                                      C.c_void_p(stream.cuda_stream))
        assert rc == EB_OK
        torch.cuda.synchronize()
        assert torch.equal(An, amax[0]), f"step {s}: argmax differs"
        assert torch.equal(Hn, H[0]), f"step {s}: entropies differ (max {(Hn - H[0]).abs().max()})"
        # the argmax is the row's maximum logit, lowest index first
        ref = torch.argmax(z.float(), dim=1).to(torch.int32)
        assert torch.equal(An, ref)
    assert eb.status() == 0
    eb.close()


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a GPU")
def test_noalloc_matches_the_oracle_on_more_rows_than_a_canvas_holds():
    """3000 rows (more than the sampler's 1024 positions per canvas) of a
    ragged vocabulary, bf16 and fp32: every row's entropy and argmax against
    the CPU oracle, on two calls in a row."""
    import numpy as np

    import oracle as O
    _, lib = _lib()
    dev = torch.device("cuda", 0)
    rows, V, T = 3000, 1000, 0.7
    stream = torch.cuda.current_stream(dev)
    for dt_code, dt in ((EB_BF16, torch.bfloat16), (0, torch.float32)):
        z = _logits(rows, V, 5 + dt_code, dev).to(dt)
        host = (z.view(torch.int16).cpu().numpy().view(np.uint16) if dt == torch.bfloat16
                else z.cpu().numpy())
        ref = [O.row_stats(host[i], 1.0 / T) for i in range(rows)]
        for _ in range(2):
            Hn = torch.full((rows,), float("nan"), dtype=torch.float32, device=dev)
            An = torch.full((rows,), -7, dtype=torch.int32, device=dev)
            rc = lib.eb_row_stats_noalloc(C.c_void_p(z.data_ptr()), dt_code, rows, V, T,
                                          C.c_void_p(Hn.data_ptr()), C.c_void_p(An.data_ptr()),
                                          C.c_void_p(stream.cuda_stream))
            assert rc == EB_OK
            torch.cuda.synchronize()
            Hh, Ah = Hn.cpu().numpy(), An.cpu().numpy()
            tol = 2e-3 if dt == torch.bfloat16 else 1e-4
            for i in range(rows):
                assert abs(float(Hh[i]) - ref[i][0]) <= tol, (i, Hh[i], ref[i][0])
                assert int(Ah[i]) == ref[i][2], (i, Ah[i], ref[i][2])


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a GPU")
def test_noalloc_rejects_sizes_beyond_the_scratch_and_bad_arguments():
    _, lib = _lib()
    dev = torch.device("cuda", 0)
    z = torch.zeros((4, 64), dtype=torch.bfloat16, device=dev)
    Hn = torch.zeros((4,), dtype=torch.float32, device=dev)
    An = torch.zeros((4,), dtype=torch.int32, device=dev)
    p = lambda t: C.c_void_p(t.data_ptr())
    stream = C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    # 1 M rows of 262144 logits need ~0.8 GB of records: refused before any launch
    assert lib.eb_row_stats_noalloc(p(z), EB_BF16, 1 << 20, 262144, 1.0, p(Hn), p(An),
                                    stream) == EB_ERR_OVERFLOW
    assert lib.eb_row_stats_noalloc(p(z), EB_BF16, 4, 64, 0.0, p(Hn), p(An),
                                    stream) == EB_ERR_INVALID_ARG
    assert lib.eb_row_stats_noalloc(None, EB_BF16, 4, 64, 1.0, p(Hn), p(An),
                                    stream) == EB_ERR_INVALID_ARG
    assert lib.eb_row_stats_noalloc(p(z), EB_BF16, 0, 64, 1.0, p(Hn), p(An),
                                    stream) == EB_ERR_INVALID_ARG
    # a valid small call still works after the refusals
    assert lib.eb_row_stats_noalloc(p(z), EB_BF16, 4, 64, 1.0, p(Hn), p(An), stream) == EB_OK
    torch.cuda.synchronize()
    # all-zero logits: uniform over 64 tokens
    assert torch.allclose(Hn, torch.full_like(Hn, float(torch.log(torch.tensor(64.0)))),
                          atol=1e-6)
    assert torch.equal(An, torch.zeros_like(An))
