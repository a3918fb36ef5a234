"""Test helpers: run one seeded problem through the CUDA path (via the C ABI
binding) and through the CPU oracle, and compare.  Not collected by pytest."""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from combine_moe_dispatch_03_b200.inputs import bf16_bits

SENTINEL = 0x4B4B          # a finite bf16 bit pattern pre-filled in untouched rows
TOL_REL = 2.0 ** -7        # |gpu - oracle| <= 2^-7 |oracle| + 1e-6
TOL_ABS = 1e-6


def fill_bits(shape, bits, device):
    return torch.full(shape, bits if bits < 0x8000 else bits - 0x10000, dtype=torch.int16,
                      device=device).view(torch.bfloat16)


def to_bits(t: torch.Tensor) -> np.ndarray:
    return bf16_bits(t.detach().cpu())


def assert_within_tol(got: np.ndarray, ref: np.ndarray, what: str):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    lim = TOL_REL * np.abs(ref) + TOL_ABS
    bad = err > lim
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at "
                             f"{tuple(i)} got {got[tuple(i)]!r} want {ref[tuple(i)]!r}")


def f32(bits: np.ndarray) -> np.ndarray:
    return orc.f32_from_bf16(bits)


def run_gpu(inp: dict, E: int, R: int, align: int, N_cap: int, *, zero_pad=True, validate=True,
            weights=None, backward=True, fused=False, device="cuda:0"):
    """All calls of the path through the binding; returns numpy copies.  With
    fused, the layout and the permute are one call (moe_dispatch)."""
    from combine_moe_dispatch_03_b200 import api
    dev = torch.device(device)
    x = inp["x"].to(dev)
    topk = inp["topk_idx"].to(dev)
    w = (inp["weights"] if weights is None else weights).to(dev)
    s = inp["scales"].to(dev)
    T, H = x.shape
    K = topk.shape[1]
    st = api.new_status(dev)
    xp = fill_bits((N_cap, H), SENTINEL, dev)
    r2f = torch.empty(N_cap, dtype=torch.int32, device=dev)
    f2r = torch.empty(T, K, dtype=torch.int32, device=dev)
    if fused:
        lay, _, _, _ = api.dispatch(x, topk, E, R, align, capacity=N_cap, zero_pad=zero_pad,
                                    status=st, out=(xp, r2f, f2r))
    else:
        lay = api.dispatch_layout(topk, E, R, align, status=st)
        api.permute(x, topk, lay, capacity=N_cap, zero_pad=zero_pad, status=st,
                    out=(xp, r2f, f2r))
    y = fill_bits((N_cap, H), SENTINEL, dev)
    api.expert_scale(xp, lay, s, status=st, out=y)
    out = api.combine_weighted(y, f2r, w, row_to_flat=r2f, validate=validate, status=st)
    res = dict(layout=lay, status_fwd=None)
    torch.cuda.synchronize()
    res["status_fwd"] = int(st.item())
    if backward:
        g = inp["grad_out"].to(dev)
        grad_rows = fill_bits((N_cap, H), SENTINEL, dev)
        _, grad_w = api.combine_backward(g, y, r2f, f2r, w, lay, zero_pad=zero_pad, status=st,
                                         out=(grad_rows, torch.empty(T, K, dtype=w.dtype,
                                                                     device=dev)))
        grad_xp = fill_bits((N_cap, H), SENTINEL, dev)
        api.expert_scale(grad_rows, lay, s, status=st, out=grad_xp)
        grad_x = api.combine_weighted(grad_xp, f2r, None, status=st)
        torch.cuda.synchronize()
        res.update(grad_rows=to_bits(grad_rows), grad_w=grad_w.float().cpu().numpy(),
                   grad_xp=to_bits(grad_xp), grad_x=to_bits(grad_x))
    res.update(
        status=int(st.item()),
        tokens_per_expert=lay.tokens_per_expert.cpu().numpy(),
        counts=lay.counts.cpu().numpy(), splits=lay.splits.cpu().numpy(),
        tokens_per_rank=lay.tokens_per_rank.cpu().numpy(),
        is_token_in_rank=lay.is_token_in_rank.cpu().numpy(),
        expert_offsets=lay.expert_offsets.cpu().numpy(),
        x_perm=to_bits(xp), row_to_flat=r2f.cpu().numpy(), flat_to_row=f2r.cpu().numpy(),
        y=to_bits(y), out=to_bits(out))
    return res


def run_oracle(inp: dict, E: int, R: int, align: int, N_cap: int, *, zero_pad=True, weights=None,
               backward=True):
    x = bf16_bits(inp["x"])
    topk = inp["topk_idx"].numpy()
    wt = inp["weights"] if weights is None else weights
    w32 = wt.float().numpy()
    s = inp["scales"].numpy()
    T, H = x.shape
    lay = orc.layout(topk, E, R, align)
    init = np.full((N_cap, H), SENTINEL, np.uint16)
    pm = orc.permute(x, topk, E, lay["expert_offsets"], N_cap, zero_pad=zero_pad, x_perm_init=init)
    y = orc.expert_scale(pm["x_perm"], lay["expert_offsets"], lay["tokens_per_expert"], s,
                         out_init=init)
    cb = orc.combine(y, pm["flat_to_row"], w32)
    res = dict(lay)
    res.update(pm)
    res.update(y=y, out_ref=cb["ref"], out_seq=cb["seq"],
               status=lay["status"] | pm["status"] | cb["status"])
    if backward:
        g = bf16_bits(inp["grad_out"])
        bw = orc.combine_backward(g, y, pm["row_to_flat"], pm["flat_to_row"], w32,
                                  lay["expert_offsets"], zero_pad=zero_pad, grad_rows_init=init)
        gxp = orc.expert_scale(bw["grad_rows"], lay["expert_offsets"], lay["tokens_per_expert"], s,
                               out_init=init)
        gx = orc.combine(gxp, pm["flat_to_row"], None)
        res.update(grad_rows=bw["grad_rows"], grad_w_ref=bw["grad_w"], grad_xp=gxp,
                   grad_x_ref=gx["ref"], grad_x_seq=gx["seq"])
    return res


def compare(gpu: dict, ref: dict, backward=True, bf16_weights=False):
    """Bit-exact for the integer and copy outputs; tolerance for combine
    outputs and gradients (plus the FP32 slot-order reading, bit-exact)."""
    assert gpu["status"] == 0, gpu["status"]
    for key in ("tokens_per_expert", "counts", "splits", "tokens_per_rank", "is_token_in_rank",
                "expert_offsets", "flat_to_row", "row_to_flat"):
        np.testing.assert_array_equal(gpu[key], ref[key], err_msg=key)
    for key in ("x_perm", "y"):
        if not np.array_equal(gpu[key], ref[key]):
            bad = np.argwhere(gpu[key] != ref[key])
            raise AssertionError(f"{key}: {len(bad)} elements differ, first at {tuple(bad[0])}")
    assert_within_tol(f32(gpu["out"]), ref["out_ref"].astype(np.float32), "out")
    np.testing.assert_array_equal(gpu["out"], ref["out_seq"], err_msg="out vs fmaf chain")
    if backward:
        for key in ("grad_rows", "grad_xp"):
            if not np.array_equal(gpu[key], ref[key]):
                bad = np.argwhere(gpu[key] != ref[key])
                raise AssertionError(f"{key}: {len(bad)} elements differ, first at {tuple(bad[0])}")
        gw_ref = ref["grad_w_ref"].astype(np.float32)
        if bf16_weights:
            gw_ref = f32(orc.bf16_from_f32(gw_ref))
        assert_within_tol(gpu["grad_w"], gw_ref, "grad_w")
        assert_within_tol(f32(gpu["grad_x"]), ref["grad_x_ref"].astype(np.float32), "grad_x")
        np.testing.assert_array_equal(gpu["grad_x"], ref["grad_x_seq"], err_msg="grad_x vs chain")
