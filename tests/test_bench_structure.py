"""The bench's step structure, on CPU (no kernel runs): what each segment
calls, which calls the per-kernel table times, and the launch counts the
JSON line reports.  The dispatch segment is one moe_dispatch call; the
per-kernel table times the layout and the permute as separate calls; the
stand-in expert is never a timed method kernel."""
import dataclasses
import os
import sys

import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


@pytest.fixture(scope="module")
def bench():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    import bench as b
    return b


@pytest.mark.parametrize("name", ["qwen3", "tiny", "mixtral"])
def test_segments_and_kernel_calls(bench, name):
    from combine_moe_dispatch_03_b200.inputs import CONFIGS, make_inputs
    cfg = dataclasses.replace(CONFIGS[name], T=min(CONFIGS[name].T, 64))   # small host buffers
    inp = make_inputs(cfg, with_grad=cfg.backward)
    path = bench.Path(inp, cfg, torch.device("cpu"))
    segs = path.segments()
    assert segs[0] == ("dispatch", ("dispatch",), True)
    timed = [n for n, _, t in segs if t]
    untimed = [c for _, calls, t in segs if not t for c in calls]
    assert all(c in bench.STAND_IN for c in untimed)
    kc = path.kernel_calls()
    assert kc[:2] == ["layout", "permute"] and "dispatch" not in kc
    assert set(path.method_launches()) <= set(bench.METHOD)
    assert not set(path.method_launches()) & set(bench.STAND_IN)
    if cfg.backward:
        assert timed == ["dispatch", "combine", "dispatch_backward"]
        assert path.method_launches() == ["layout", "permute", "combine", "combine_backward",
                                          "dispatch_backward"]
    else:
        assert timed == ["dispatch", "combine"]
        assert path.method_launches() == ["layout", "permute", "combine"]
    # Kernels per step: the same whether the dispatch is one call or two.
    per_call = lambda calls: sum(bench.KERNELS_PER_CALL.get(n, 1) for n in calls)
    assert per_call(path.launches()) == per_call(kc)
    assert per_call(path.launches()) == (8 if cfg.backward else 5)
