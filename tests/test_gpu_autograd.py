"""The autograd chain (forward: dispatch -> stand-in experts -> combine;
backward: combine backward -> stand-in backward -> unit-weight combine) on
the Qwen3-MoE-shaped fwd+bwd workload, against the oracle's gradients."""
import numpy as np
import pytest
import torch

import oracle as orc
from _pipeline import assert_within_tol, f32, to_bits
from combine_moe_dispatch_03_b200.inputs import CONFIGS, bf16_bits, capacity_rows, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_autograd_qwen3_fwd_bwd():
    from combine_moe_dispatch_03_b200 import api
    from combine_moe_dispatch_03_b200.autograd import moe_dispatch_combine
    cfg = CONFIGS["qwen3"]
    inp = make_inputs("qwen3")
    dev = torch.device("cuda:0")
    x = inp["x"].to(dev).requires_grad_(True)
    w = inp["weights"].to(dev).requires_grad_(True)
    topk = inp["topk_idx"].to(dev)
    s = inp["scales"].to(dev)
    out, status = moe_dispatch_combine(x, topk, w, s, cfg.E, cfg.R, cfg.align, True)
    out.backward(inp["grad_out"].to(dev))
    api.check_status(status)

    # oracle chain
    xb = bf16_bits(inp["x"])
    tk = inp["topk_idx"].numpy()
    w32 = inp["weights"].numpy()
    lay = orc.layout(tk, cfg.E, cfg.R, cfg.align)
    N = capacity_rows(cfg.T, cfg.K, cfg.E, cfg.align)
    pm = orc.permute(xb, tk, cfg.E, lay["expert_offsets"], N)
    y = orc.expert_scale(pm["x_perm"], lay["expert_offsets"], lay["tokens_per_expert"],
                         inp["scales"].numpy())
    cb = orc.combine(y, pm["flat_to_row"], w32)
    bw = orc.combine_backward(bf16_bits(inp["grad_out"]), y, pm["row_to_flat"], pm["flat_to_row"],
                              w32, lay["expert_offsets"])
    gxp = orc.expert_scale(bw["grad_rows"], lay["expert_offsets"], lay["tokens_per_expert"],
                           inp["scales"].numpy())
    gx = orc.combine(gxp, pm["flat_to_row"], None)

    assert_within_tol(f32(to_bits(out)), cb["ref"].astype(np.float32), "out")
    assert_within_tol(f32(to_bits(x.grad)), gx["ref"].astype(np.float32), "x.grad")
    assert_within_tol(w.grad.cpu().numpy(), bw["grad_w"].astype(np.float32), "weights.grad")
    np.testing.assert_array_equal(to_bits(out), cb["seq"])
    np.testing.assert_array_equal(to_bits(x.grad), gx["seq"])


def test_forward_makes_no_host_sync():
    """The forward issues no synchronising torch operation (the hot path of
    the XTuner PR "Integrate MoonEP dispatcher": no host sync; histc rather
    than bincount)."""
    from combine_moe_dispatch_03_b200.autograd import moe_dispatch_combine
    cfg = CONFIGS["tiny"]
    inp = make_inputs("tiny")
    dev = torch.device("cuda:0")
    args = [inp["x"].to(dev), inp["topk_idx"].to(dev), inp["weights"].to(dev),
            inp["scales"].to(dev)]
    moe_dispatch_combine(*args, cfg.E, cfg.R, cfg.align)   # warm-up (library load)
    torch.cuda.synchronize()
    torch.cuda.set_sync_debug_mode("error")
    try:
        out, status = moe_dispatch_combine(*args, cfg.E, cfg.R, cfg.align)
    finally:
        torch.cuda.set_sync_debug_mode("default")
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_split_dispatch_combine_with_a_torch_expert():
    """dispatch / combine as separate autograd Functions with the caller's
    own expert in between (here y = 2 * x_perm in torch, exact in bf16):
    output and both gradients equal, bit for bit, the chain with the
    stand-in expert at s_e = 2, whose gradients the oracle pins above."""
    from combine_moe_dispatch_03_b200 import api
    from combine_moe_dispatch_03_b200.autograd import combine, dispatch, moe_dispatch_combine
    cfg = CONFIGS["qwen3"]
    inp = make_inputs("qwen3", T=2048, with_grad=True)
    dev = torch.device("cuda:0")
    topk = inp["topk_idx"].to(dev)
    g = inp["grad_out"].to(dev)
    two = torch.full((cfg.E,), 2.0, dtype=torch.float32, device=dev)

    x1 = inp["x"].to(dev).requires_grad_(True)
    w1 = inp["weights"].to(dev).requires_grad_(True)
    out1, st1 = moe_dispatch_combine(x1, topk, w1, two, cfg.E, cfg.R, cfg.align)
    out1.backward(g)

    x2 = inp["x"].to(dev).requires_grad_(True)
    w2 = inp["weights"].to(dev).requires_grad_(True)
    x_perm, handle = dispatch(x2, topk, cfg.E, cfg.R, cfg.align)
    out2 = combine(x_perm * 2, handle, w2, validate=True)
    out2.backward(g)
    api.check_status(st1)
    api.check_status(handle.status)

    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(x1.grad.view(torch.int16), x2.grad.view(torch.int16))
    assert torch.equal(w1.grad, w2.grad)
    off = handle.layout.expert_offsets
    assert int(off[-1]) <= handle.num_rows
