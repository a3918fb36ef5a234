"""Randomised problems through the whole CUDA path against the oracle.

Hypothesis draws the shape and the routing of each problem over the ranges
the C ABI accepts (logical ranks R, experts per rank, tokens per rank, top_k
up to the maximum of 32, row widths that end in a partial 4 KB piece, group
alignments, a buffer larger than the worst case, zero-padded or not, FP32 or
bf16 router weights, routing by softmax top-k or by independent draws with
repeated experts, the layout and the permute as two calls or as one), then
runs every call of the path forward and backward and
compares every output with the oracle: bit-exact for the layout, the row
maps and every row buffer, the stated tolerance (and the oracle's FP32
slot-order chain, bit-exact) for the combine outputs and gradients.  The
draws are derandomised, so a run is reproducible; both permute kernels (the
ring at fan-out <= 2, the register kernel above it) and every combine path
(slot-major up to K = 8, any-K above) are reached.
"""
import numpy as np
import pytest
import torch

from _pipeline import compare, run_gpu, run_oracle
from combine_moe_dispatch_03_b200.inputs import capacity_rows, custom_inputs

pytestmark = pytest.mark.gpu

# Keep the oracle's share of a case to well under a second: T * K * H bound.
_MAX_ELEMS = 3_000_000


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_random_problems_match_oracle():
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    ran = []
    @settings(max_examples=300, deadline=None, derandomize=True,
              suppress_health_check=list(HealthCheck))
    @given(R=st.sampled_from([1, 1, 2, 3, 4, 8]), El=st.integers(1, 24), Tb=st.integers(0, 500),
           K=st.sampled_from([1, 2, 2, 2, 3, 4, 6, 8, 8, 9, 16, 32]),
           hv=st.integers(1, 700), align=st.sampled_from([1, 2, 3, 8, 16, 17, 64, 128, 160]),
           extra=st.sampled_from([0, 0, 1, 37]), zero_pad=st.booleans(), bf16_w=st.booleans(),
           repeats=st.booleans(), fused=st.booleans(), seed=st.integers(0, 2 ** 31 - 1))
    def case(R, El, Tb, K, hv, align, extra, zero_pad, bf16_w, repeats, fused, seed):
        ran.append(1)
        E, T = R * El, R * Tb
        if K > E:
            repeats = True                          # softmax top-k needs K <= E
        H = 8 * max(1, min(hv, _MAX_ELEMS // (8 * max(1, T * K))))
        if repeats:
            g = torch.Generator().manual_seed(seed)
            topk = torch.randint(0, E, (T, K), generator=g)
            inp = custom_inputs(T, H, E, K, seed=seed, topk_idx=topk)
        else:
            inp = custom_inputs(T, H, E, K, seed=seed)
        N_cap = capacity_rows(T, K, E, align) + extra
        w = inp["weights"].to(torch.bfloat16) if bf16_w else None
        gpu = run_gpu(inp, E, R, align, N_cap, zero_pad=zero_pad, weights=w, fused=fused)
        ref = run_oracle(inp, E, R, align, N_cap, zero_pad=zero_pad, weights=w)
        compare(gpu, ref, bf16_weights=bf16_w)
        assert np.all(gpu["row_to_flat"][int(gpu["expert_offsets"][-1]):] == -1)

    case()
    assert len(ran) >= 50, len(ran)      # the draws really ran
