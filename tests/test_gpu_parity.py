"""Parity of the CUDA path (through the C ABI) with the CPU oracle, element by
element, on the seeded workloads and on edge cases.

Bar: bit-exact for layout, offsets, row maps, permuted rows, stand-in rows and
row gradients; |gpu - oracle| <= 2^-7 |oracle| + 1e-6 for the combine output,
the weight gradient and the dispatch-backward output (the FP32 slot-order
value is additionally expected bit-exact).
"""
import numpy as np
import pytest
import torch

from _pipeline import SENTINEL, compare, run_gpu, run_oracle
from combine_moe_dispatch_03_b200.inputs import (CONFIGS, bf16_bits, capacity_rows, custom_inputs,
                                                 make_inputs)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check(inp, E, R, align, N_cap=None, **kw):
    T, K = inp["topk_idx"].shape
    if N_cap is None:
        N_cap = capacity_rows(T, K, E, align)
    gpu = run_gpu(inp, E, R, align, N_cap, **kw)
    ref = run_oracle(inp, E, R, align, N_cap, zero_pad=kw.get("zero_pad", True),
                     weights=kw.get("weights"), backward=kw.get("backward", True))
    compare(gpu, ref, backward=kw.get("backward", True),
            bf16_weights=kw.get("weights") is not None and kw["weights"].dtype == torch.bfloat16)
    return gpu, ref


# ------------------------------------------------------- seeded workloads ---

@pytest.mark.parametrize("name", ["tiny", "mixtral", "dsv3", "dsv3_skew", "qwen3", "page_k4",
                                  "page_k8"])
def test_config_full_size(name):
    """Every output of every call at the workload's full size, forward and
    backward, with the capacity and launch configuration the bench uses."""
    cfg = CONFIGS[name]
    inp = make_inputs(name, with_grad=True)
    _check(inp, cfg.E, cfg.R, cfg.align)


@pytest.mark.parametrize("name", ["tiny", "mixtral", "qwen3"])
def test_fused_dispatch_full_size(name):
    """moe_dispatch (layout and permute in one call): every output against
    the oracle, and bit-identical to the two separate calls."""
    cfg = CONFIGS[name]
    inp = make_inputs(name, with_grad=True)
    gpu, _ = _check(inp, cfg.E, cfg.R, cfg.align, fused=True)
    N = capacity_rows(cfg.T, cfg.K, cfg.E, cfg.align)
    sep = run_gpu(inp, cfg.E, cfg.R, cfg.align, N)
    for k in ("x_perm", "row_to_flat", "flat_to_row", "expert_offsets", "counts", "splits",
              "tokens_per_rank", "is_token_in_rank", "out", "grad_x", "grad_w"):
        np.testing.assert_array_equal(gpu[k], sep[k], err_msg=k)


@pytest.mark.parametrize("T,H,E,K,R,align", [
    (0, 64, 4, 2, 2, 8), (1, 8, 1, 1, 1, 1), (100, 2048, 8, 2, 1, 16), (777, 24, 5, 1, 1, 3),
    (4000, 2056, 8, 2, 2, 16), (3008, 4104, 1024, 2, 64, 1), (160000, 8, 16, 2, 2, 8),
    (997, 264, 13, 5, 1, 8),
])
def test_fused_dispatch_edge_shapes(T, H, E, K, R, align):
    inp = custom_inputs(T, H, E, K, seed=T * 5 + K + 1)
    N_cap = 16 if T == 0 else None
    _check(inp, E, R, align, N_cap=N_cap, fused=True)


def test_tiny_twice_deterministic():
    cfg = CONFIGS["tiny"]
    inp = make_inputs("tiny", with_grad=True)
    N = capacity_rows(cfg.T, cfg.K, cfg.E, cfg.align)
    a = run_gpu(inp, cfg.E, cfg.R, cfg.align, N)
    b = run_gpu(inp, cfg.E, cfg.R, cfg.align, N)
    for k in ("x_perm", "flat_to_row", "out", "grad_rows", "grad_w", "grad_x"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


# ------------------------------------------------------------ edge cases ---

@pytest.mark.parametrize("T,H,E,K,R,align", [
    (1, 8, 1, 1, 1, 1),          # smallest everything
    (3, 16, 3, 2, 1, 2),         # hand-example sizes
    (1000, 136, 7, 3, 1, 4),     # ragged T, H not a multiple of 32 vectors, odd K
    (997, 264, 13, 5, 1, 8),     # prime T, K=5
    (640, 64, 16, 6, 8, 16),     # K=6, 8 logical ranks
    (512, 72, 32, 7, 4, 3),      # K=7, align 3
    (300, 40, 40, 9, 4, 1),      # K=9 (generic paths)
    (64, 32, 64, 32, 2, 2),      # K=32 (maximum)
    (256, 16, 1024, 4, 64, 1),   # E=1024 and R=64 (maxima)
    (130, 8192, 8, 2, 2, 16),    # wide rows
    (66, 8200, 4, 2, 2, 8),      # long rows
    (20000, 8, 64, 8, 1, 4),     # 148 layout tiles, one per SM
    (40000, 8, 64, 8, 1, 4),     # 157 tiles: more tiles than SMs
    (9728, 8, 1024, 32, 8, 1),   # 152 tiles x 1032 rows of per-tile counts
    (120000, 8, 16, 8, 2, 8),    # 470 tiles: rows longer than 32 x 8 tiles (several loads per lane)
    # The ring permute (K <= 2): one CTA per SM, each a balanced range of
    # 4 KB token pieces.
    (100, 2048, 8, 2, 1, 16),    # fewer pieces than CTAs: idle CTAs
    (777, 24, 5, 1, 1, 3),       # K = 1
    (4000, 2056, 8, 2, 2, 16),   # 2 pieces per row, the last 16 bytes: ranges start mid-token
    (3008, 4104, 1024, 2, 64, 1),  # E = 1024 (largest shared-memory footprint), 3 pieces per row
    (160000, 8, 16, 2, 2, 8),    # more tokens than 148 CTAs' row tables hold: 157 CTAs
    (160000, 8, 16, 1, 1, 8),    # the same at K = 1
])
def test_edge_shapes(T, H, E, K, R, align):
    inp = custom_inputs(T, H, E, K, seed=T * 7 + K)
    _check(inp, E, R, align)


def test_empty_input():
    inp = custom_inputs(0, 64, 4, 2, seed=1)
    gpu, ref = _check(inp, 4, 2, 8, N_cap=16)
    assert np.all(gpu["row_to_flat"] == -1)


def test_all_tokens_on_one_expert():
    T, K, E = 776, 4, 16
    topk = torch.zeros(T, K, dtype=torch.int64)
    topk[:, 1] = 5                         # a repeated expert within a token
    topk[:, 3] = 15
    inp = custom_inputs(T, 128, E, K, seed=5, topk_idx=topk)
    _check(inp, E, 4, 16)
    topk[:] = 2                            # every slot of every token on one expert
    inp = custom_inputs(T, 128, E, K, seed=6, topk_idx=topk)
    _check(inp, E, 1, 128)


def test_repeated_experts_and_skew():
    g = torch.Generator().manual_seed(3)
    T, K, E = 2048, 8, 64
    topk = torch.randint(0, 4, (T, K), generator=g)        # heavy repeats on 4 experts
    topk[::3] = torch.randint(0, E, (len(range(0, T, 3)), K), generator=g)
    inp = custom_inputs(T, 256, E, K, seed=9, topk_idx=topk)
    _check(inp, E, 8, 16)


def test_no_zero_pad_leaves_pad_rows():
    cfg = CONFIGS["tiny"]
    inp = make_inputs("tiny", with_grad=True)
    gpu, ref = _check(inp, cfg.E, cfg.R, cfg.align, zero_pad=False)
    r2f = gpu["row_to_flat"]
    N_pad = gpu["expert_offsets"][-1]
    pads = np.nonzero(r2f[:N_pad] < 0)[0]
    assert len(pads) > 0
    assert np.all(gpu["x_perm"][pads] == SENTINEL)


def test_bf16_router_weights():
    cfg = CONFIGS["tiny"]
    inp = make_inputs("tiny", with_grad=True)
    _check(inp, cfg.E, cfg.R, cfg.align, weights=inp["weights"].to(torch.bfloat16))


def test_logical_ranks_do_not_change_rows():
    """R only regroups the counts: rows, maps and outputs are identical for
    R = 1 and R = 8 on the same routing (partitioned == unpartitioned)."""
    cfg = CONFIGS["qwen3"]
    inp = make_inputs("qwen3", T=2048, with_grad=True)
    N = capacity_rows(2048, cfg.K, cfg.E, cfg.align)
    a = run_gpu(inp, cfg.E, 1, cfg.align, N)
    b = run_gpu(inp, cfg.E, 8, cfg.align, N)
    for k in ("x_perm", "row_to_flat", "flat_to_row", "y", "out", "grad_rows", "grad_w", "grad_x",
              "expert_offsets", "tokens_per_expert"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_combine_token_chunks_concatenate():
    """Combining two halves of the tokens gives the same bytes as all at once."""
    from combine_moe_dispatch_03_b200 import api
    cfg = CONFIGS["tiny"]
    inp = make_inputs("tiny", T=512)
    dev = torch.device("cuda:0")
    lay = api.dispatch_layout(inp["topk_idx"].to(dev), cfg.E, cfg.R, cfg.align)
    xp, r2f, f2r = api.permute(inp["x"].to(dev), inp["topk_idx"].to(dev), lay)
    w = inp["weights"].to(dev)
    full = api.combine_weighted(xp, f2r, w)
    h = 256
    a = api.combine_weighted(xp, f2r[:h].contiguous(), w[:h].contiguous())
    b = api.combine_weighted(xp, f2r[h:].contiguous(), w[h:].contiguous())
    assert torch.equal(full.view(torch.int16), torch.cat([a, b]).view(torch.int16))


def test_layout_workspace_reused_across_calls():
    """One workspace, never initialised by the caller, serves several layouts
    in a row: each call's counts, offsets and rows match the oracle, whatever
    the previous call (or garbage) left in it."""
    import oracle as orc
    from combine_moe_dispatch_03_b200 import api
    dev = torch.device("cuda:0")
    T, H, E, K, R, align = 2048, 64, 128, 8, 8, 16
    lay = api.alloc_layout(T, K, E, R, align, dev)
    lay.workspace.fill_(0xA5)                               # garbage, as from a caching allocator
    N = capacity_rows(T, K, E, align)
    g = torch.Generator().manual_seed(77)
    routings = [torch.randint(0, E, (T, K), generator=g),
                torch.randint(0, 5, (T, K), generator=g),     # heavy skew, repeats in a token
                None]
    routings[2] = routings[0]
    for topk in routings:
        inp = custom_inputs(T, H, E, K, seed=3, topk_idx=topk)
        st = api.new_status(dev)
        api.dispatch_layout(inp["topk_idx"].to(dev), E, R, align, status=st, out=lay)
        xp, r2f, f2r = api.permute(inp["x"].to(dev), inp["topk_idx"].to(dev), lay, capacity=N,
                                   status=st)
        api.check_status(st)
        ref = orc.layout(inp["topk_idx"].numpy(), E, R, align)
        for key in ("tokens_per_expert", "counts", "splits", "tokens_per_rank", "is_token_in_rank",
                    "expert_offsets"):
            np.testing.assert_array_equal(getattr(lay, key).cpu().numpy(), ref[key], err_msg=key)
        pm = orc.permute(bf16_bits(inp["x"]), inp["topk_idx"].numpy(), E, ref["expert_offsets"], N)
        np.testing.assert_array_equal(f2r.cpu().numpy(), pm["flat_to_row"])
        np.testing.assert_array_equal(r2f.cpu().numpy(), pm["row_to_flat"])
        n_pad = int(ref["expert_offsets"][-1])                # rows past it are left untouched
        np.testing.assert_array_equal(bf16_bits(xp[:n_pad].cpu()), pm["x_perm"][:n_pad])


def test_side_stream_matches_default_stream():
    """Every call enqueues on the caller's current stream: the whole chain
    run on a side stream (kernels back to back, no host sync in between)
    gives the same bytes as on the default stream."""
    cfg = CONFIGS["qwen3"]
    inp = make_inputs("qwen3", T=2048, with_grad=True)
    N = capacity_rows(2048, cfg.K, cfg.E, cfg.align)
    a = run_gpu(inp, cfg.E, cfg.R, cfg.align, N)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        b = run_gpu(inp, cfg.E, cfg.R, cfg.align, N)
    for k in ("expert_offsets", "counts", "x_perm", "row_to_flat", "flat_to_row", "y", "out",
              "grad_rows", "grad_w", "grad_x"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)
