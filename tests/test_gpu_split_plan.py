"""split_plan_from_expert_indices on a GPU: the count matrix comes from the
library's layout kernel, the exchange runs over NCCL (one rank here: every
GPU run has one GPU; the multi-rank exchange is tested over gloo in
tests/test_split_plan_multirank.py).  Against the oracle, and with one
device-to-host copy."""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle as orc
from combine_moe_dispatch_03_b200.inputs import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_split_plan_from_expert_indices_nccl_one_rank():
    import torch.distributed as dist
    from combine_moe_dispatch_03_b200 import api, ep
    cfg = CONFIGS["dsv3_skew"]
    inp = make_inputs("dsv3_skew", H=8)
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        topk = inp["topk_idx"].to(dev)
        st = api.new_status(dev)
        plan = ep.split_plan_from_expert_indices(topk, cfg.E, status=st)
        api.check_status(st)
        ref = orc.layout(inp["topk_idx"].numpy(), cfg.E, 1, 1)
        A = cfg.T * cfg.K
        assert plan.input_splits == [A] and plan.output_splits == [A]
        np.testing.assert_array_equal(plan.received_counts.cpu().numpy(),
                                      ref["tokens_per_expert"].reshape(1, cfg.E))
        np.testing.assert_array_equal(plan.tokens_per_local_expert.cpu().numpy(),
                                      ref["tokens_per_expert"])
        assert plan.received_counts.sum(dim=1).tolist() == plan.output_splits
    finally:
        dist.destroy_process_group()


def test_ep_dispatch_combine_nccl_one_rank():
    """ep_dispatch / ep_combine through NCCL with one rank: equal, bit for
    bit, to the single-device layout, permute and restore."""
    import torch.distributed as dist
    from combine_moe_dispatch_03_b200 import api, ep
    cfg = CONFIGS["qwen3"]
    inp = make_inputs("qwen3", T=2048)
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x, tk, w = inp["x"].to(dev), inp["topk_idx"].to(dev), inp["weights"].to(dev)
        st = api.new_status(dev)
        lay = api.dispatch_layout(tk, cfg.E, 1, cfg.align, status=st)
        xp, _, f2r = api.permute(x, tk, lay, status=st)
        out_ref = api.combine_weighted(xp * 2, f2r, w, status=st)
        grouped, h = ep.ep_dispatch(x, tk, cfg.E, cfg.align, status=st)
        n_pad = int(lay.expert_offsets[-1])
        assert torch.equal(grouped[:n_pad].view(torch.int16), xp[:n_pad].view(torch.int16))
        out = ep.ep_combine(grouped * 2, h, w, validate=True)
        assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
        api.check_status(st)
    finally:
        dist.destroy_process_group()


def test_ep_direct_nccl_one_rank():
    """ep_dispatch_direct / ep_combine_direct through NCCL with one rank (the
    table holds this GPU's own buffer): equal, bit for bit, to the
    single-device permute and restore."""
    import torch.distributed as dist
    from combine_moe_dispatch_03_b200 import api, ep
    cfg = CONFIGS["qwen3"]
    inp = make_inputs("qwen3", T=2048)
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x, tk, w = inp["x"].to(dev), inp["topk_idx"].to(dev), inp["weights"].to(dev)
        st = api.new_status(dev)
        lay = api.dispatch_layout(tk, cfg.E, 1, cfg.align, status=st)
        xp, _, f2r = api.permute(x, tk, lay, status=st)
        out_ref = api.combine_weighted(xp * 2, f2r, w, status=st)
        cap = api.worst_case_rows(2048, cfg.K, cfg.E, cfg.align)
        buf = torch.empty(cap, x.shape[1], dtype=torch.bfloat16, device=dev)
        table = torch.tensor([buf.data_ptr()], dtype=torch.int64, device=dev)
        h = ep.ep_dispatch_direct(x, tk, cfg.E, table, cap, cfg.align, status=st)
        n_pad = int(lay.expert_offsets[-1])
        assert torch.equal(buf[:n_pad].view(torch.int16), xp[:n_pad].view(torch.int16))
        y = buf * 2
        ytab = torch.tensor([y.data_ptr()], dtype=torch.int64, device=dev)
        out = ep.ep_combine_direct(ytab, cap, x.shape[1], h, tk, w)
        assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
        api.check_status(st)
    finally:
        dist.destroy_process_group()
