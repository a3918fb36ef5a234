"""Dispatch and combine across R ranks, emulated in one process on one GPU.

Every rank's send and receive steps run in the library's kernels (layout,
permute, segment labels, combine); the exchanges between ranks are plain
tensor copies of exactly what all_to_all_single would deliver, so no kernel
waits on another.  Against the single-device path with the ranks as logical
groups: every rank's plan equals the single-device count matrix and splits,
the expert-grouped rows of every local expert are bit-identical to that
expert's rows there (pads zero), and the combined output of every rank's
tokens is bit-identical to the single-device output."""
import numpy as np
import pytest
import torch

from combine_moe_dispatch_03_b200.inputs import CONFIGS, custom_inputs, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _i16(t):
    return t.contiguous().view(torch.int16)


@pytest.mark.parametrize("R,E,K,Tb,H,align,skew", [
    (4, 32, 4, 512, 256, 8, 0.0),
    (8, 64, 8, 256, 136, 16, 3.0),      # ragged rows (17 vectors), severe skew
    (2, 8, 2, 300, 64, 1, 0.0),         # no padding
])
def test_ep_dispatch_combine_emulated(R, E, K, Tb, H, align, skew):
    T = R * Tb
    g = torch.Generator().manual_seed(R * 1000 + E + K)
    logits = torch.randn(T, E, generator=g)
    if skew:
        rank = torch.randperm(E, generator=g).double() + 1.0
        logits += (skew * torch.log(rank ** -1.2 / (rank ** -1.2).sum())).float()
    topk = torch.topk(logits, K, dim=1).indices
    _run_emulated(custom_inputs(T, H, E, K, seed=R + E, topk_idx=topk), R, E, align)


@pytest.mark.parametrize("name", ["dsv3", "dsv3_skew"])
def test_ep_dispatch_combine_emulated_full_size(name):
    """The DeepSeek-V3-shaped workloads at full size (8 ranks x 1024 tokens,
    256 experts, top-8, H 7168, align 128), their seeded routing."""
    cfg = CONFIGS[name]
    _run_emulated(make_inputs(name), cfg.R, cfg.E, cfg.align)


def _run_emulated(inp, R, E, align):
    from combine_moe_dispatch_03_b200 import api, ep
    dev = torch.device("cuda:0")
    T, K = inp["topk_idx"].shape
    H = inp["x"].shape[1]
    Tb, El = T // R, E // R
    x, w, tk = inp["x"].to(dev), inp["weights"].to(dev), inp["topk_idx"].to(dev)
    st = api.new_status(dev)

    # single device, ranks as logical groups
    lay = api.dispatch_layout(tk, E, R, align, status=st)
    xp, _, f2r = api.permute(x, tk, lay, status=st)
    out_ref = api.combine_weighted(xp * 2, f2r, w, status=st)
    off = lay.expert_offsets.cpu().tolist()
    cnt = lay.tokens_per_expert.cpu().tolist()
    counts_all = lay.counts.cpu()
    splits_all = lay.splits.cpu()

    # send side of every rank
    sends = [ep.dispatch_send(x[r * Tb:(r + 1) * Tb].contiguous(),
                              tk[r * Tb:(r + 1) * Tb].contiguous(), E, R, st) for r in range(R)]
    # count exchange: rank r receives row r of every rank's count matrix
    plans = []
    for r in range(R):
        received = torch.stack([sends[s][4][r] for s in range(R)]).to(torch.int32).contiguous()
        plans.append(ep.plan_from_counts(sends[r][4].to(torch.int32), received))
        assert torch.equal(plans[r].received_counts.cpu(), counts_all[:, r, :])
        assert plans[r].input_splits == splits_all[r, :].tolist()
        assert plans[r].output_splits == splits_all[:, r].tolist()
    # row exchange: rank r receives, source by source, the rows each sends to r
    starts = [np.concatenate([[0], np.cumsum(p.input_splits)]) for p in plans]
    handles, grouped = [], []
    for r in range(R):
        parts = [sends[s][0][starts[s][r]:starts[s][r + 1]] for s in range(R)]
        recv = torch.cat(parts).contiguous()
        assert recv.shape[0] == sum(plans[r].output_splits)
        gr, rlay, rr2f, rf2r = ep.dispatch_recv(recv, plans[r], align, st)
        handles.append(ep.EPHandle(sends[r][1], sends[r][2], sends[r][3], plans[r], rlay, rr2f,
                                   rf2r, st))
        grouped.append(gr)
        roff = rlay.expert_offsets.cpu().tolist()
        for el in range(El):
            e, c = r * El + el, cnt[r * El + el]
            assert roff[el + 1] - roff[el] == off[e + 1] - off[e]
            assert torch.equal(_i16(gr[roff[el]:roff[el] + c]), _i16(xp[off[e]:off[e] + c])), e
            assert not _i16(gr[roff[el] + c:roff[el + 1]]).any()
    # experts, then the reverse exchange and the restore on every source rank
    backs = [ep.combine_send(grouped[r] * 2, handles[r]) for r in range(R)]
    rstarts = [np.concatenate([[0], np.cumsum(p.output_splits)]) for p in plans]
    for s in range(R):
        returned = torch.empty(Tb * K, H, dtype=torch.bfloat16, device=dev)
        parts = torch.cat([backs[r][rstarts[r][s]:rstarts[r][s + 1]] for r in range(R)])
        returned[:parts.shape[0]] = parts
        out_s = ep.combine_recv(returned, handles[s], w[s * Tb:(s + 1) * Tb].contiguous(),
                                validate=True)
        assert torch.equal(_i16(out_s), _i16(out_ref[s * Tb:(s + 1) * Tb])), s
    api.check_status(st)


# ----------------------------------------------- direct, no send buffer ---

@pytest.mark.parametrize("R,E,K,Tb,H,align,skew", [
    (4, 32, 4, 512, 256, 8, 0.0),
    (8, 64, 8, 256, 136, 16, 3.0),
    (2, 8, 2, 300, 64, 1, 0.0),
])
def test_ep_direct_emulated(R, E, K, Tb, H, align, skew):
    T = R * Tb
    g = torch.Generator().manual_seed(R * 1000 + E + K + 1)
    logits = torch.randn(T, E, generator=g)
    if skew:
        rank = torch.randperm(E, generator=g).double() + 1.0
        logits += (skew * torch.log(rank ** -1.2 / (rank ** -1.2).sum())).float()
    topk = torch.topk(logits, K, dim=1).indices
    _run_direct(custom_inputs(T, H, E, K, seed=R + E + 1, topk_idx=topk), R, E, align)


def test_ep_direct_emulated_full_size():
    cfg = CONFIGS["dsv3_skew"]
    _run_direct(make_inputs("dsv3_skew"), cfg.R, cfg.E, cfg.align)


def _run_direct(inp, R, E, align):
    """Every rank stores its rows straight into the R receive buffers (a
    table of addresses: separate buffers on this one GPU, peer addresses
    across GPUs) and gathers the expert outputs straight from them."""
    from combine_moe_dispatch_03_b200 import api, ep
    dev = torch.device("cuda:0")
    T, K = inp["topk_idx"].shape
    H = inp["x"].shape[1]
    Tb, El = T // R, E // R
    x, w, tk = inp["x"].to(dev), inp["weights"].to(dev), inp["topk_idx"].to(dev)
    st = api.new_status(dev)
    lay = api.dispatch_layout(tk, E, R, align, status=st)
    xp, _, f2r = api.permute(x, tk, lay, status=st)
    out_ref = api.combine_weighted(xp * 2, f2r, w, status=st)
    off = lay.expert_offsets.cpu().tolist()
    cnt = lay.tokens_per_expert.cpu().tolist()

    blk = lambda t, s: t[s * Tb:(s + 1) * Tb].contiguous()
    lays = [api.dispatch_layout(blk(tk, s), E, 1, 1, status=st) for s in range(R)]
    all_counts = torch.stack([l.tokens_per_expert for l in lays])      # the all-gather
    cap = ep.direct_receive_rows(all_counts, align)
    recv = [torch.full((cap, H), 0x3F80, dtype=torch.int16, device=dev).view(torch.bfloat16)
            for _ in range(R)]
    table = torch.tensor([b.data_ptr() for b in recv], dtype=torch.int64, device=dev)
    f2rs = []
    for s in range(R):
        dest_base, own_off, own_cnt = ep.rank_bases(all_counts, s, align)
        f2rs.append(api.permute_to_ranks(blk(x, s), blk(tk, s), lays[s], dest_base, table, cap, s,
                                         own_off, own_cnt, status=st))
    for r in range(R):
        _, own_off, own_cnt = ep.rank_bases(all_counts, r, align)
        roff = own_off.cpu().tolist()
        for el in range(El):
            e, c = r * El + el, cnt[r * El + el]
            assert roff[el + 1] - roff[el] == off[e + 1] - off[e]
            assert torch.equal(_i16(recv[r][roff[el]:roff[el] + c]), _i16(xp[off[e]:off[e] + c])), e
            assert not _i16(recv[r][roff[el] + c:roff[el + 1]]).any()
    ys = [b * 2 for b in recv]
    ytab = torch.tensor([y.data_ptr() for y in ys], dtype=torch.int64, device=dev)
    for s in range(R):
        out_s = api.combine_from_ranks(ytab, cap, H, f2rs[s], blk(tk, s), E, blk(w, s), status=st)
        assert torch.equal(_i16(out_s), _i16(out_ref[s * Tb:(s + 1) * Tb])), s
    api.check_status(st)
