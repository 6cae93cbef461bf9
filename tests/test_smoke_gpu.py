"""The build-and-smoke entry point, run as a test.

`__graft_entry__.smoke()` builds what is stale and runs one tiny sampler
trajectory on cuda:0 through the C ABI, checking entropies and argmaxes
against the CPU oracle at every step.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a GPU")
def test_smoke_entry_point():
    import __graft_entry__ as G
    G.smoke()
