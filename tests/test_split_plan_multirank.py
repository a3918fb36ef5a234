"""The split plan of expert parallelism across real processes (gloo ranks on
CPU, 127.0.0.1), after the Tests section of the DeepSpeed PR "Derive AutoEP
rank splits from the per-expert count exchange":

  * for every rank and three token distributions (balanced, mild skew,
    severe skew), the derived output_splits equal the per-rank totals, and
    received_counts.sum(dim=1) == output_splits element-wise;
  * against a local restatement of the old planner (a separate all-to-all of
    the per-rank totals, then the count matrix), the new plan issues one
    collective instead of two and all four fields are identical;
  * every field equals what the single-device layout computes for the same
    routing with the ranks as logical groups (the oracle's count matrix
    [R, R, E_local] and splits [R, R]), and the per-rank totals also match
    an independent direct count.

The direct (send-buffer-free) dispatch's metadata runs the same way: one
all-gather of the per-expert counts, then each rank's row bases, checked
against the oracle's single-device rows.

Each rank's own counts come from the oracle here (no GPU); on a GPU they
come from the library's layout kernel (tests/test_gpu_split_plan.py)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, K, TB = 32, 4, 256               # experts, top_k, tokens per rank


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _routing(kind: str, ws: int) -> np.ndarray:
    """All ranks' routing [ws*TB, K] (the same on every rank: seeded)."""
    g = torch.Generator().manual_seed({"balanced": 11, "mild": 12, "severe": 13}[kind] + 100 * ws)
    logits = torch.randn(ws * TB, E, generator=g)
    if kind == "mild":
        logits += 0.5 * torch.randn(E, generator=g)
    elif kind == "severe":
        rank = torch.randperm(E, generator=g).double() + 1.0
        logits += (3.0 * torch.log(rank ** -1.2 / (rank ** -1.2).sum())).float()
    return torch.topk(logits, K, dim=1).indices.numpy().astype(np.int64)


def _old_plan(cm, dist):
    """The old planner as the page describes it: the per-rank totals
    exchanged on their own (one all-to-all and one copy to the host), then
    the count matrix (a second all-to-all), then the input splits (a second
    copy to the host)."""
    totals = cm.sum(dim=1).to(torch.int32)
    remote = torch.empty_like(totals)
    dist.all_to_all_single(remote, totals)
    output_splits = remote.cpu().tolist()
    received = torch.empty_like(cm)
    dist.all_to_all_single(received.view(-1), cm.contiguous().view(-1))
    input_splits = cm.sum(dim=1).cpu().tolist()
    return input_splits, output_splits, received, received.sum(dim=0)


def _worker(rank, ws, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as orc
    from combine_moe_dispatch_03_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    real = dist.all_to_all_single
    calls = [0]

    def counting(*a, **kw):
        calls[0] += 1
        return real(*a, **kw)

    try:
        out = {}
        for kind in ("balanced", "mild", "severe"):
            topk = _routing(kind, ws)
            mine = topk[rank * TB:(rank + 1) * TB]
            cm = ep.count_matrix(torch.from_numpy(orc.layout(mine, E, 1, 1)["tokens_per_expert"]),
                                 ws)
            dist.all_to_all_single = counting
            calls[0] = 0
            plan = ep.split_plan(cm)
            n_new = calls[0]
            calls[0] = 0
            old = _old_plan(cm.to(torch.int32), dist)
            n_old = calls[0]
            dist.all_to_all_single = real
            full = orc.layout(topk, E, ws, 1)
            direct = orc.output_splits(topk, E, ws)          # [dest, src]
            out[kind] = dict(
                plan=(plan.input_splits, plan.output_splits, plan.received_counts.numpy(),
                      plan.tokens_per_local_expert.numpy()),
                old=(old[0], old[1], old[2].numpy(), old[3].numpy()),
                counts_to_me=full["counts"][:, rank, :], splits=full["splits"],
                direct_to_me=direct[rank], n_new=n_new, n_old=n_old,
                skew=float(np.bincount(topk.reshape(-1), minlength=E).max()) / (topk.size / E))
        q.put((rank, out))
    finally:
        dist.all_to_all_single = real
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 4])
def test_split_plan_across_processes(ws):
    import oracle as orc
    orc.build()
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in range(ws))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert res[0]["severe"]["skew"] > 3 * res[0]["balanced"]["skew"] / 2   # the skew is real
    for rank in range(ws):
        for kind, r in res[rank].items():
            inp, outp, received, per_expert = r["plan"]
            np.testing.assert_array_equal(received, r["counts_to_me"], err_msg=kind)
            assert outp == r["splits"][:, rank].tolist() == r["direct_to_me"].tolist(), kind
            assert inp == r["splits"][rank, :].tolist(), kind
            assert received.sum(axis=1).tolist() == outp, kind       # the page's invariant
            np.testing.assert_array_equal(per_expert, r["counts_to_me"].sum(axis=0))
            o_in, o_out, o_recv, o_pe = r["old"]
            assert (o_in, o_out) == (inp, outp), kind
            np.testing.assert_array_equal(o_recv, received)
            np.testing.assert_array_equal(o_pe, per_expert)
            assert (r["n_new"], r["n_old"]) == (1, 2), kind


def _direct_worker(rank, ws, port, align, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as orc
    from combine_moe_dispatch_03_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        topk = _routing("severe", ws)
        mine = topk[rank * TB:(rank + 1) * TB]
        tpe = torch.from_numpy(orc.layout(mine, E, 1, 1)["tokens_per_expert"])
        all_counts = ep.gather_counts(tpe)          # the one exchange of the direct dispatch
        rb = orc.rank_bases(all_counts.numpy(), rank, align)
        q.put((rank, all_counts.numpy(), rb["dest_base"], rb["own_offsets"], rb["own_counts"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,align", [(2, 8), (4, 1)])
def test_direct_plan_across_processes(ws, align):
    """The direct dispatch's metadata over real processes: one all-gather of
    the per-expert counts (ep.gather_counts), then each rank's row bases from
    what it received (the oracle's definition here; the device kernel is
    pinned to it on the GPU), which must put every assignment at the
    oracle's single-device row minus the start of its owner rank's block
    (the owner's padded groups and real rows likewise)."""
    import oracle as orc
    orc.build()
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_direct_worker, args=(r, ws, port, align, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = dict((r[0], r[1:]) for r in (q.get(timeout=240) for _ in range(ws)))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    topk = _routing("severe", ws)
    El = E // ws
    lay = orc.layout(topk, E, ws, align)
    off = lay["expert_offsets"]
    pm = orc.permute(np.zeros((topk.shape[0], 8), np.uint16), topk, E, off, int(off[-1]))
    for rank in range(ws):
        all_counts, dest_base, own_off, own_cnt = res[rank]
        for s in range(ws):
            np.testing.assert_array_equal(
                all_counts[s], orc.layout(topk[s * TB:(s + 1) * TB], E, 1, 1)["tokens_per_expert"])
        np.testing.assert_array_equal(own_off, off[rank * El:(rank + 1) * El + 1] - off[rank * El])
        np.testing.assert_array_equal(own_cnt, lay["tokens_per_expert"][rank * El:(rank + 1) * El])
        seen = np.zeros(E, np.int64)
        for t in range(rank * TB, (rank + 1) * TB):
            for k in range(K):
                e = int(topk[t, k])
                want = int(pm["flat_to_row"][t, k]) - int(off[(e // El) * El])
                assert dest_base[e] + seen[e] == want, (rank, t, k)
                seen[e] += 1
