"""The folded restore (DeepSpeed PR "AutoEP: support
combine_impl=fused_weighted_sum with AutoEP+AutoTP folding", Change and
Tests): tensor-parallel peers each hold part of the expert-output rows; the
rows are gathered together with one flat index (token * top_k + slot) per
row, the flat indices are scattered into [tokens, top_k], and the fused
restore runs on the gathered rows.

Checked here on one GPU, the gather being a concatenation of the peers'
slices:
  * moe_scatter_flat_index is bit-exact against the oracle's scatter, and
    its coverage check flags a missing, duplicated or out-of-range index;
  * with 2 peers of different row counts (one of them in shuffled order), the
    output is bitwise equal to the unpartitioned restore;
  * each peer back-propagates a different gradient; the row and score
    gradients, summed over the peers, match the gradients of the summed
    gradient (fp64, within the bf16 / fp32 rounding of each peer's term),
    and each peer's own gradients are bitwise those of the unpartitioned
    backward for the same incoming gradient.
"""
import types

import numpy as np
import pytest
import torch

import oracle as orc
from _pipeline import f32, to_bits
from combine_moe_dispatch_03_b200.inputs import bf16_bits, custom_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _api():
    from combine_moe_dispatch_03_b200 import api
    return api


def _forward(T, H, E, K, align, seed, wdtype=torch.float32):
    api = _api()
    dev = torch.device("cuda:0")
    inp = custom_inputs(T, H, E, K, seed=seed)
    st = api.new_status(dev)
    x, topk = inp["x"].to(dev), inp["topk_idx"].to(dev)
    w = inp["weights"].to(wdtype).to(dev)
    lay = api.dispatch_layout(topk, E, 1, align, status=st)
    xp, r2f, f2r = api.permute(x, topk, lay, status=st)
    y = api.expert_scale(xp, lay, inp["scales"].to(dev), status=st)
    out = api.combine_weighted(y, f2r, w, row_to_flat=r2f, validate=True, status=st)
    api.check_status(st)
    return dict(inp=inp, lay=lay, y=y, r2f=r2f, f2r=f2r, w=w, out=out, dev=dev)


def _peers(fw, seed):
    """Two peers: experts [0, E/2) and [E/2, E) with their pad rows; the second
    peer's rows in a shuffled order.  Returns the gathered rows, flat indices
    and, per gathered row, the row it came from."""
    off = fw["lay"].expert_offsets.cpu().numpy()
    E = off.shape[0] - 1
    cut, end = int(off[E // 2]), int(off[E])
    g = torch.Generator().manual_seed(seed)
    src1 = cut + torch.randperm(end - cut, generator=g)
    src = torch.cat([torch.arange(cut), src1]).to(fw["dev"])
    rows_g = fw["y"].index_select(0, src).contiguous()
    flat_g = fw["r2f"].index_select(0, src).contiguous()
    return rows_g, flat_g, src, cut


@pytest.mark.parametrize("T,H,E,K,align,seed", [
    (1024, 2048, 64, 8, 16, 501),       # pad rows among the gathered rows
    (333, 264, 10, 3, 1, 502),          # ragged sizes, no padding
    (8192, 256, 256, 8, 128, 503),      # DeepSeek-V3 routing, heavy padding
])
def test_scatter_matches_oracle_and_inverts_permute(T, H, E, K, align, seed):
    api = _api()
    fw = _forward(T, H, E, K, align, seed)
    rows_g, flat_g, src, _ = _peers(fw, seed)
    st = api.new_status(fw["dev"])
    f2r_g = api.scatter_flat_index(flat_g, T, K, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = orc.scatter_flat_index(flat_g.cpu().numpy(), T, K)
    assert ref["status"] == 0
    np.testing.assert_array_equal(f2r_g.cpu().numpy(), ref["flat_to_row"])
    # the gathered row of each slot came from the slot's unpartitioned row
    np.testing.assert_array_equal(src.cpu().numpy()[f2r_g.cpu().numpy()], fw["f2r"].cpu().numpy())


@pytest.mark.parametrize("wdtype", [torch.float32, torch.bfloat16])
def test_two_peers_forward_bitwise_and_gradients_sum(wdtype):
    api = _api()
    T, H, E, K = 1024, 2048, 64, 8
    fw = _forward(T, H, E, K, 16, 511, wdtype)
    dev = fw["dev"]
    rows_g, flat_g, src, cut = _peers(fw, 511)
    assert cut != rows_g.shape[0] - cut            # different row counts
    st = api.new_status(dev)
    f2r_g = api.scatter_flat_index(flat_g, T, K, status=st)
    out_g = api.combine_weighted(rows_g, f2r_g, fw["w"], row_to_flat=flat_g, validate=True,
                                 status=st)
    api.check_status(st)
    assert torch.equal(out_g.view(torch.int16), fw["out"].view(torch.int16))

    # each peer back-propagates its own gradient through the replicated output
    gen = torch.Generator().manual_seed(512)
    gs = [torch.randn(T, H, generator=gen).to(torch.bfloat16) for _ in range(2)]
    n_g = rows_g.shape[0]
    gathered = types.SimpleNamespace(expert_offsets=torch.tensor([0, n_g], dtype=torch.int32,
                                                                 device=dev), E=1)
    per_peer = []
    for g in gs:
        gr, gw = api.combine_backward(g.to(dev), rows_g, flat_g, f2r_g, fw["w"], gathered,
                                      status=st)
        gr_u, gw_u = api.combine_backward(g.to(dev), fw["y"], fw["r2f"], fw["f2r"], fw["w"],
                                          fw["lay"], status=st)
        api.check_status(st)
        # same values as the unpartitioned backward, row for row
        assert torch.equal(gr.view(torch.int16), gr_u.index_select(0, src).view(torch.int16))
        assert torch.equal(gw.view(-1).view(torch.int16 if wdtype == torch.bfloat16 else torch.int32),
                           gw_u.view(-1).view(torch.int16 if wdtype == torch.bfloat16 else torch.int32))
        per_peer.append((f32(to_bits(gr)).astype(np.float64), gw.float().cpu().numpy().astype(np.float64)))

    # summed over the peers vs the gradient of the summed incoming gradient (fp64)
    g_sum = sum(f32(bf16_bits(g)).astype(np.float64) for g in gs)
    g_abs = sum(np.abs(f32(bf16_bits(g)).astype(np.float64)) for g in gs)
    w64 = fw["w"].float().cpu().numpy().astype(np.float64).reshape(-1)
    f2r = f2r_g.cpu().numpy().reshape(-1)
    y64 = f32(to_bits(rows_g)).astype(np.float64)
    gr_sum = per_peer[0][0] + per_peer[1][0]
    tok = np.arange(T * K) // K
    ref_rows = w64[:, None] * g_sum[tok]
    lim_rows = 1.01 * 2.0 ** -8 * np.abs(w64)[:, None] * g_abs[tok] + 1e-30
    assert (np.abs(gr_sum[f2r] - ref_rows) <= lim_rows).all()
    pad = flat_g.cpu().numpy() < 0
    assert (gr_sum[pad] == 0).all()
    gw_sum = (per_peer[0][1] + per_peer[1][1]).reshape(-1)
    ref_w = np.einsum("ah,ah->a", g_sum[tok], y64[f2r])
    u = 2.0 ** -8 if wdtype == torch.bfloat16 else 2.0 ** -24
    lim_w = u * (np.abs(per_peer[0][1]) + np.abs(per_peer[1][1])).reshape(-1) + 1e-12 * (
        np.einsum("ah,ah->a", g_abs[tok], np.abs(y64[f2r])))
    assert (np.abs(gw_sum - ref_w) <= lim_w).all()


def _coverage_status(flat: np.ndarray, T: int, K: int) -> int:
    api = _api()
    dev = torch.device("cuda:0")
    st = api.new_status(dev)
    api.scatter_flat_index(torch.from_numpy(flat).to(dev), T, K, status=st)
    torch.cuda.synchronize()
    return int(st.item())


def test_missing_duplicate_and_out_of_range_flagged():
    api = _api()
    T, K = 300, 4
    rng = np.random.default_rng(7)
    flat = np.concatenate([rng.permutation(T * K), np.full(50, -1)]).astype(np.int32)
    rng.shuffle(flat)
    assert _coverage_status(flat, T, K) == 0
    cases = {
        "missing": np.delete(flat, int(np.flatnonzero(flat == 17)[0])),
        "duplicate": np.where(flat == 17, 18, flat).astype(np.int32),
        "out_of_range": np.where(flat == 17, T * K, flat).astype(np.int32),
        "negative": np.where(flat == 17, -2, flat).astype(np.int32),
    }
    for name, bad in cases.items():
        got = _coverage_status(bad, T, K)
        want = orc.scatter_flat_index(bad, T, K)["status"]
        assert want == orc.COVERAGE, name
        assert got == api._lib.ST_COVERAGE, name
    # the user-facing error: a clear RuntimeError naming the coverage bit
    st = api.new_status(torch.device("cuda:0"))
    api.scatter_flat_index(torch.from_numpy(cases["missing"]).cuda(), T, K, status=st)
    with pytest.raises(RuntimeError, match="cover every"):
        api.check_status(st)


def test_empty_and_degenerate():
    # no tokens: nothing to cover; rows holding only pads are fine
    assert _coverage_status(np.full(5, -1, np.int32), 0, 4) == 0
    assert _coverage_status(np.zeros(0, np.int32), 0, 2) == 0
    # tokens but no rows: every slot is missing
    from combine_moe_dispatch_03_b200 import _lib
    assert _coverage_status(np.zeros(0, np.int32), 3, 2) == _lib.ST_COVERAGE
