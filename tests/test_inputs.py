"""The seeded input recipe (CPU): every workload draws what its description
says, the same way every time.  The generator holds none of the method's
arithmetic; these checks keep the workloads the tests and the benchmark run
on what the design notes state."""
import numpy as np
import pytest
import torch

from combine_moe_dispatch_03_b200.inputs import CONFIGS, custom_inputs, make_inputs

SMALL_H = 8      # the routing does not depend on H; keep the draws cheap


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_shapes_ranges_and_distinct_experts(name):
    cfg = CONFIGS[name]
    inp = make_inputs(name, H=SMALL_H, T=min(cfg.T, 8192))
    T = inp["topk_idx"].shape[0]
    assert inp["x"].shape == (T, SMALL_H) and inp["x"].dtype == torch.bfloat16
    assert inp["topk_idx"].shape == (T, cfg.K) and inp["topk_idx"].dtype == torch.int64
    assert inp["weights"].shape == (T, cfg.K) and inp["weights"].dtype == torch.float32
    tk = inp["topk_idx"]
    assert int(tk.min()) >= 0 and int(tk.max()) < cfg.E
    srt = torch.sort(tk, dim=1).values
    assert bool((srt[:, 1:] != srt[:, :-1]).all()), "top-k experts of a token are distinct"
    s = inp["scales"]
    assert s.shape == (cfg.E,) and bool(((s >= 0.5) & (s < 1.5)).all())
    assert cfg.T % cfg.R == 0 and cfg.E % cfg.R == 0


@pytest.mark.parametrize("name", ["tiny", "qwen3", "dsv3_skew"])
def test_draws_are_deterministic(name):
    a = make_inputs(name, H=SMALL_H, T=1024)
    b = make_inputs(name, H=SMALL_H, T=1024)
    for k in ("x", "topk_idx", "weights", "scales"):
        assert torch.equal(a[k].view(torch.int16) if a[k].dtype == torch.bfloat16 else a[k],
                           b[k].view(torch.int16) if b[k].dtype == torch.bfloat16 else b[k]), k


def test_routers():
    """softmax routers keep the selected probabilities (not renormalised: the
    K weights sum to less than 1); the sigmoid router normalises sigma over
    the selected experts (the weights sum to 1).  Top-k by the logits, so the
    weights of a token are non-increasing along its slots."""
    for name in ("qwen3", "mixtral", "tiny"):
        w = make_inputs(name, H=SMALL_H)["weights"]
        assert bool((w > 0).all()) and bool((w.sum(dim=1) < 1).all()), name
        assert bool((w[:, 1:] <= w[:, :-1]).all()), name
    for name in ("dsv3", "page_k8"):
        w = make_inputs(name, H=SMALL_H, T=4096)["weights"]
        np.testing.assert_allclose(w.sum(dim=1).numpy(), 1.0, rtol=1e-6)
        assert bool((w[:, 1:] <= w[:, :-1]).all()), name


def test_severe_skew_puts_half_the_assignments_on_eight_experts():
    """Zipf(1.2) bias, scale found by bisection: 50% +- 2% of all
    assignments land on the 8 most favoured experts (balanced: ~8/256)."""
    inp = make_inputs("dsv3_skew", H=SMALL_H)
    assert abs(inp["info"]["hot_share"] - 0.50) <= 0.02
    counts = np.bincount(inp["topk_idx"].numpy().reshape(-1), minlength=256)
    top8 = np.sort(counts)[-8:].sum() / counts.sum()
    assert 0.48 <= top8 <= 0.55
    bal = np.bincount(make_inputs("dsv3", H=SMALL_H)["topk_idx"].numpy().reshape(-1),
                      minlength=256)
    assert np.sort(bal)[-8:].sum() / bal.sum() < 0.05


def test_mild_skew_is_mild():
    """A per-expert bias of standard deviation 0.5: busier experts than
    balanced routing, far from the severe case."""
    c = np.bincount(make_inputs("qwen3", H=SMALL_H)["topk_idx"].numpy().reshape(-1),
                    minlength=128).astype(np.float64)
    cv = c.std() / c.mean()
    assert 0.2 < cv < 1.5


def test_custom_inputs_impose_routing():
    tk = torch.zeros(16, 3, dtype=torch.int64)
    inp = custom_inputs(16, 8, 4, 3, seed=1, topk_idx=tk)
    assert torch.equal(inp["topk_idx"], tk)
    assert inp["weights"].shape == (16, 3)
