"""CPU checks of the parity harness itself (tests/_pipeline.py): the oracle
leg runs end to end, an exact copy of the oracle's results passes the
comparison, and planted mistakes in a copy are caught."""
import numpy as np
import pytest

from _pipeline import compare, run_oracle
from combine_moe_dispatch_03_b200.inputs import CONFIGS, capacity_rows, make_inputs


def _as_gpu(ref):
    g = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in ref.items()}
    g["out"] = ref["out_seq"].copy()
    g["grad_x"] = ref["grad_x_seq"].copy()
    g["grad_w"] = ref["grad_w_ref"].astype(np.float32)
    return g


@pytest.fixture(scope="module")
def ref():
    c = CONFIGS["tiny"]
    inp = make_inputs("tiny", with_grad=True)
    return run_oracle(inp, c.E, c.R, c.align, capacity_rows(c.T, c.K, c.E, c.align))


def test_exact_copy_passes(ref):
    compare(_as_gpu(ref), ref)


@pytest.mark.parametrize("key,mutate", [
    ("x_perm", lambda a: a.__setitem__((3, 5), a[3, 5] ^ 1)),
    ("flat_to_row", lambda a: a.__setitem__((0, 0), a[0, 1])),
    ("counts", lambda a: a.__setitem__((0, 0, 0), a[0, 0, 0] + 1)),
    ("out", lambda a: a.__setitem__((1, 1), a[1, 1] ^ 0x40)),
    ("grad_rows", lambda a: a.__setitem__((0, 0), a[0, 0] ^ 1)),
    ("grad_w", lambda a: a.__setitem__((2, 1), a[2, 1] * 1.1 + 1e-3)),
    ("grad_x", lambda a: a.__setitem__((4, 7), a[4, 7] ^ 0x80)),
])
def test_planted_mistakes_are_caught(ref, key, mutate):
    g = _as_gpu(ref)
    mutate(g[key])
    with pytest.raises(AssertionError):
        compare(g, ref)


def test_nonzero_status_fails(ref):
    g = _as_gpu(ref)
    g["status"] = 4
    with pytest.raises(AssertionError):
        compare(g, ref)
