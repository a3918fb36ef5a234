"""The OpenMP build of the oracle (the multi-core CPU baseline) gives the
same bits as the plain single-threaded checker on every routine it
parallelises: the pragmas only split independent loop iterations."""
import numpy as np
import pytest

from combine_moe_dispatch_03_b200.inputs import CONFIGS, bf16_bits, capacity_rows, make_inputs


def _path(orc, inp, cfg, T):
    tk = inp["topk_idx"].numpy()
    lay = orc.layout(tk, cfg.E, cfg.R, cfg.align)
    N = capacity_rows(T, cfg.K, cfg.E, cfg.align)
    pm = orc.permute(bf16_bits(inp["x"]), tk, cfg.E, lay["expert_offsets"], N)
    s = inp["scales"].numpy()
    y = orc.expert_scale(pm["x_perm"], lay["expert_offsets"], lay["tokens_per_expert"], s)
    w = inp["weights"].numpy()
    cb = orc.combine(y, pm["flat_to_row"], w)
    bw = orc.combine_backward(bf16_bits(inp["grad_out"]), y, pm["row_to_flat"], pm["flat_to_row"],
                              w, lay["expert_offsets"])
    gx = orc.combine(bw["grad_rows"], pm["flat_to_row"], None)
    yf = orc.f32_from_bf16(y)
    cf = orc.combine_f32(yf, pm["flat_to_row"], w)
    bf = orc.combine_backward_f32(orc.f32_from_bf16(bf16_bits(inp["grad_out"])), yf,
                                  pm["row_to_flat"], pm["flat_to_row"], w, lay["expert_offsets"])
    dr = orc.restore_activation_dtype(y, pm["flat_to_row"], w, bf16_bits(inp["grad_out"]))
    return [lay["expert_offsets"], lay["counts"], pm["x_perm"], pm["row_to_flat"],
            pm["flat_to_row"], y, cb["ref"], cb["seq"], bw["grad_rows"], bw["grad_w"], gx["ref"],
            gx["seq"], cf["ref"], cf["seq"], bf["grad_rows"], bf["grad_w"], dr["out"], dr["grad_w"]]


@pytest.mark.parametrize("name", ["qwen3", "tiny"])
def test_openmp_build_equals_plain(orc, name):
    cfg = CONFIGS[name]
    T = min(cfg.T, 256)
    inp = make_inputs(name, T=T, with_grad=True)
    plain = _path(orc, inp, cfg, T)
    orc.use_openmp(True)
    try:
        assert orc.threads() >= 1
        par = _path(orc, inp, cfg, T)
    finally:
        orc.use_openmp(False)
    assert orc.threads() == 1
    for i, (a, b) in enumerate(zip(plain, par)):
        assert np.array_equal(a, b), f"output {i} differs between the plain and OpenMP builds"
