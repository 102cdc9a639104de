"""Debug mode on the GPU: the guard regions and index-list checks leave results unchanged,
and a guard overwritten from the host right after a stage (the library's test hook; no
device fault involved) is reported as Q1M_ERR_CHECK, after which the library runs clean."""
import pytest
import torch

from long_context_prefill_dca_b200 import q1m
from long_context_prefill_dca_b200.layer import Layer
from synth import configs as C
from synth import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture
def debug():
    q1m.set_debug(True)
    try:
        yield
    finally:
        q1m.debug_inject(-1)
        q1m.set_debug(False)


@pytest.mark.parametrize("w", [C.SMALL_SPARSE, C.SMALL_DENSE_D128, C.SMALL_SPARSE.with_(equal_cost_chunks=3)],
                         ids=["sparse", "dense", "equal-cost"])
def test_debug_mode_results_unchanged(w, debug, deterministic):
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    got = Layer(w)(g["q"], g["k"], g["v"])
    torch.cuda.synchronize()
    assert q1m.status_poll() == 0
    q1m.set_debug(False)
    ref = Layer(w)(g["q"], g["k"], g["v"])
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("stage", ["keys", "select", "attn", "merge"])
def test_injected_guard_write_is_reported(stage, debug):
    w = C.SMALL_SPARSE
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    layer = Layer(w)
    q1m.debug_inject(stage)
    layer(g["q"], g["k"], g["v"])
    assert q1m.status_poll() == -7
    assert "guard region 0" in q1m.last_error()
    layer(g["q"], g["k"], g["v"])            # the injection fires once; the guards are refilled
    assert q1m.status_poll() == 0
