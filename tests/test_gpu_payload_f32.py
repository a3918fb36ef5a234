"""Dispatch of an FP8 (data, scales) payload and of fp32 rows, and the fused
restore / backward on fp32 rows, against the CPU oracle.

Sources: the DeepEP issue "Does Deepep's Dispatch/Combine Support Autograd
Like PyTorch's all_to_all?" (dispatch takes x as bf16 or as an FP8 tuple);
the DeepSpeed PR "AutoEP: support combine_impl=fused_weighted_sum with
AutoEP+AutoTP folding", Tests ("fp32 and bf16 rows").

Bars: rows, maps and both payloads bit-exact; the fp32 restore bit-exact
against the oracle's FP32 fmaf chain; fp32 row gradients bit-exact; weight
gradients within one rounding of the fp64 reference."""
import numpy as np
import pytest
import torch

import oracle as orc
from combine_moe_dispatch_03_b200.inputs import capacity_rows, custom_inputs

pytestmark = pytest.mark.gpu
SENT8 = 0x5A


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _api():
    from combine_moe_dispatch_03_b200 import api
    return api


def _fp8_tuple(x: torch.Tensor, block: int = 128):
    """Per-(token, 128-column block) e4m3 quantisation (input preparation)."""
    T, H = x.shape
    xb = x.float().view(T, H // block, block)
    scales = (xb.abs().amax(-1) / 448.0).clamp_min(1e-12)
    data = (xb / scales[..., None]).to(torch.float8_e4m3fn).view(T, H)
    return data, scales.contiguous()


def _layout(topk, E, align, dev, st):
    api = _api()
    return api.dispatch_layout(topk.to(dev), E, 1, align, status=st)


@pytest.mark.parametrize("T,H,E,K,align,seed,zero_pad", [
    (8192, 7168, 256, 8, 128, 601, True),     # DeepSeek-V3 shape, full size
    (1000, 384, 24, 3, 8, 602, False),        # ragged: 3 scales per row, pads untouched
    (0, 256, 8, 2, 4, 603, True),             # no tokens
])
def test_fp8_tuple_dispatch_bit_exact(T, H, E, K, align, seed, zero_pad):
    api = _api()
    dev = torch.device("cuda:0")
    if T:
        inp = custom_inputs(T, H, E, K, seed=seed, with_grad=False)
        x, topk = inp["x"], inp["topk_idx"]
    else:
        x, topk = torch.zeros(0, H, dtype=torch.bfloat16), torch.zeros(0, K, dtype=torch.int64)
    data, scales = _fp8_tuple(x) if T else (torch.zeros(0, H, dtype=torch.float8_e4m3fn),
                                            torch.zeros(0, H // 128 if H >= 128 else 1))
    N_cap = capacity_rows(T, K, E, align)
    st = api.new_status(dev)
    lay = _layout(topk, E, align, dev, st)
    S = scales.shape[1]
    xp = torch.full((N_cap, H), SENT8, dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
    ap = torch.full((N_cap, S), 7.0, dtype=torch.float32, device=dev)
    r2f = torch.empty(N_cap, dtype=torch.int32, device=dev)
    f2r = torch.empty(T, K, dtype=torch.int32, device=dev)
    api.permute_payload(data.to(dev), topk.to(dev), lay, aux=scales.to(dev), capacity=N_cap,
                        zero_pad=zero_pad, status=st, out=(xp, ap, r2f, f2r))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = orc.permute_payload(data.view(torch.uint8).numpy(), topk.numpy(), E,
                              lay.expert_offsets.cpu().numpy(), N_cap,
                              aux=scales.numpy().astype(np.float32), zero_pad=zero_pad,
                              x_perm_init=np.full((N_cap, H), SENT8, np.uint8),
                              aux_perm_init=np.full((N_cap, S), 7.0, np.float32))
    assert ref["status"] == 0
    np.testing.assert_array_equal(r2f.cpu().numpy(), ref["row_to_flat"])
    np.testing.assert_array_equal(f2r.cpu().numpy(), ref["flat_to_row"])
    np.testing.assert_array_equal(ap.cpu().numpy().view(np.uint32), ref["aux_perm"].view(np.uint32))
    assert np.array_equal(xp.view(torch.uint8).cpu().numpy(), ref["x_perm"])


def test_bf16_rows_through_payload_equal_permute():
    """moe_permute_payload on bf16 rows (row_bytes = 2H) is moe_permute."""
    api = _api()
    dev = torch.device("cuda:0")
    T, H, E, K, align = 3000, 1032, 40, 4, 16
    inp = custom_inputs(T, H, E, K, seed=611, with_grad=False)
    st = api.new_status(dev)
    lay = _layout(inp["topk_idx"], E, align, dev, st)
    x, topk = inp["x"].to(dev), inp["topk_idx"].to(dev)
    a = api.permute(x, topk, lay, status=st)
    b = api.permute_payload(x, topk, lay, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert b[1] is None
    n_pad = int(lay.expert_offsets[-1].item())      # rows past the padded total stay untouched
    assert torch.equal(a[0][:n_pad].view(torch.int16), b[0][:n_pad].view(torch.int16))
    assert torch.equal(a[1], b[2]) and torch.equal(a[2], b[3])


def _grad_w_ok(got, ref, mag, what):
    got = np.asarray(got, np.float64)
    lim = 2.0 ** -23 * np.abs(ref) + 1e-12 * mag + 1e-30
    bad = np.abs(got - ref) > lim
    assert not bad.any(), f"{what}: {int(bad.sum())} outside; first {np.argwhere(bad)[0]}"


@pytest.mark.parametrize("T,H,E,K,align,wdtype,seed", [
    (4096, 2048, 128, 8, 16, torch.float32, 621),     # Qwen3 routing, fp32 activations
    (777, 264, 10, 3, 4, torch.bfloat16, 622),        # ragged, bf16 router weights
    (200, 128, 64, 12, 1, torch.float32, 623),        # top-12: the any-K kernels
])
def test_fp32_rows_dispatch_restore_backward(T, H, E, K, align, wdtype, seed):
    _check_fp32(T, H, E, K, align, wdtype, seed)


def _check_fp32(T, H, E, K, align, wdtype, seed, topk=None):
    api = _api()
    dev = torch.device("cuda:0")
    inp = custom_inputs(T, H, E, K, seed=seed, topk_idx=topk)
    g = torch.Generator().manual_seed(seed + 1)
    x = torch.randn(T, H, generator=g)
    grad = torch.randn(T, H, generator=g)
    w = inp["weights"].to(wdtype)
    st = api.new_status(dev)
    lay = _layout(inp["topk_idx"], E, align, dev, st)
    xp, _, r2f, f2r = api.permute_payload(x.to(dev), inp["topk_idx"].to(dev), lay, status=st)
    # fp32 rows straight into the restore (an identity expert)
    out = api.combine_weighted(xp, f2r, w.to(dev), row_to_flat=r2f, validate=True, status=st)
    gr, gw = api.combine_backward(grad.to(dev), xp, r2f, f2r, w.to(dev), lay, status=st)
    unit = api.combine_weighted(gr, f2r, None, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert out.dtype == torch.float32 and gr.dtype == torch.float32 and gw.dtype == wdtype

    off = lay.expert_offsets.cpu().numpy()
    N_cap = capacity_rows(T, K, E, align)
    pm = orc.permute_payload(x.numpy(), inp["topk_idx"].numpy(), E, off, N_cap)
    np.testing.assert_array_equal(f2r.cpu().numpy(), pm["flat_to_row"])
    rows = pm["x_perm"]
    real = pm["row_to_flat"] >= 0
    np.testing.assert_array_equal(xp.cpu().numpy()[real], rows[real])
    wf = w.float().numpy()
    c = orc.combine_f32(rows, pm["flat_to_row"], wf)
    np.testing.assert_array_equal(out.cpu().numpy(), c["seq"])          # same fmaf chain
    bw = orc.combine_backward_f32(grad.numpy(), rows, pm["row_to_flat"], pm["flat_to_row"], wf, off)
    grc = gr.cpu().numpy()
    np.testing.assert_array_equal(grc[: off[-1]], bw["grad_rows"][: off[-1]])
    mag = np.abs(np.einsum("th,tkh->tk", np.abs(grad.numpy()).astype(np.float64),
                           np.abs(rows[pm["flat_to_row"]]).astype(np.float64)))
    if wdtype == torch.float32:
        _grad_w_ok(gw.cpu().numpy(), bw["grad_w"], mag, "grad_w")
    else:   # one rounding to bf16
        lim = 2.0 ** -8 * np.abs(bw["grad_w"]) + 1e-12 * mag
        assert (np.abs(gw.float().cpu().numpy() - bw["grad_w"]) <= lim).all()
    u = orc.combine_f32(bw["grad_rows"], pm["flat_to_row"], None)
    np.testing.assert_array_equal(unit.cpu().numpy(), u["seq"])


def test_random_payloads_match_oracle():
    """Hypothesis (derandomised): opaque payload rows of random byte widths
    (16-byte units, rows ending in a partial 4 KB piece), with or without a
    per-token aux payload of a few 4-byte words, any fan-out up to 32 with
    repeated experts, padded or not: rows, aux rows and both maps bit-exact
    against the oracle, and rows past the padded total untouched."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st
    api = _api()
    dev = torch.device("cuda:0")

    ran = []
    @settings(max_examples=150, deadline=None, derandomize=True,
              suppress_health_check=list(HealthCheck))
    @given(E=st.integers(1, 64), T=st.integers(0, 700), K=st.sampled_from([1, 2, 3, 4, 8, 9, 32]),
           m=st.integers(1, 400), aux_words=st.sampled_from([0, 0, 1, 2, 3, 7]),
           align=st.sampled_from([1, 2, 16, 33, 128]), zero_pad=st.booleans(),
           seed=st.integers(0, 2 ** 31 - 1))
    def case(E, T, K, m, aux_words, align, zero_pad, seed):
        ran.append(1)
        m = max(1, min(m, 2_000_000 // (16 * max(1, T * K))))
        g = torch.Generator().manual_seed(seed)
        x = torch.randint(0, 256, (T, 16 * m), dtype=torch.uint8, generator=g)
        topk = torch.randint(0, E, (T, K), generator=g)
        aux = torch.randn(T, aux_words, generator=g) if aux_words else None
        N_cap = capacity_rows(T, K, E, align) + 3
        st_ = api.new_status(dev)
        lay = _layout(topk, E, align, dev, st_)
        xp = torch.full((N_cap, 16 * m), SENT8, dtype=torch.uint8, device=dev)
        ap = torch.full((N_cap, aux_words), 7.0, device=dev) if aux_words else None
        r2f = torch.empty(N_cap, dtype=torch.int32, device=dev)
        f2r = torch.empty(T, K, dtype=torch.int32, device=dev)
        api.permute_payload(x.to(dev), topk.to(dev), lay,
                            aux=aux.to(dev) if aux_words else None, capacity=N_cap,
                            zero_pad=zero_pad, status=st_, out=(xp, ap, r2f, f2r))
        torch.cuda.synchronize()
        assert int(st_.item()) == 0
        ref = orc.permute_payload(x.numpy(), topk.numpy(), E, lay.expert_offsets.cpu().numpy(),
                                  N_cap, aux=aux.numpy() if aux_words else None,
                                  zero_pad=zero_pad,
                                  x_perm_init=np.full((N_cap, 16 * m), SENT8, np.uint8),
                                  aux_perm_init=(np.full((N_cap, aux_words), 7.0, np.float32)
                                                 if aux_words else None))
        assert ref["status"] == 0
        np.testing.assert_array_equal(r2f.cpu().numpy(), ref["row_to_flat"])
        np.testing.assert_array_equal(f2r.cpu().numpy(), ref["flat_to_row"])
        assert np.array_equal(xp.cpu().numpy(), ref["x_perm"])
        if aux_words:
            np.testing.assert_array_equal(ap.cpu().numpy().view(np.uint32),
                                          ref["aux_perm"].view(np.uint32))

    case()
    assert len(ran) >= 50, len(ran)      # the draws really ran


def test_random_fp32_rows_match_oracle():
    """Hypothesis (derandomised): fp32 rows through dispatch, the restore,
    its backward and the unit-weight restore, at random shapes, fan-outs
    (the slot-major kernels up to K = 8, the any-K ones above), router
    dtypes and routings with repeated experts; the bars of the fixed cases
    above."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    ran = []
    @settings(max_examples=60, deadline=None, derandomize=True,
              suppress_health_check=list(HealthCheck))
    @given(E=st.integers(1, 48), T=st.integers(1, 500), K=st.sampled_from([1, 2, 3, 5, 8, 9, 13]),
           m=st.integers(1, 300), align=st.sampled_from([1, 4, 16, 17]), bf16_w=st.booleans(),
           seed=st.integers(0, 2 ** 31 - 1))
    def case(E, T, K, m, align, bf16_w, seed):
        ran.append(1)
        m = max(1, min(m, 400_000 // (4 * T * K)))
        topk = torch.randint(0, E, (T, K), generator=torch.Generator().manual_seed(seed))
        _check_fp32(T, 4 * m, E, K, align, torch.bfloat16 if bf16_w else torch.float32, seed,
                    topk=topk)

    case()
    assert len(ran) >= 50, len(ran)      # the draws really ran


def test_payload_argument_errors():
    api = _api()
    from combine_moe_dispatch_03_b200 import _lib
    dev = torch.device("cuda:0")
    T, H, E, K = 64, 256, 8, 2
    inp = custom_inputs(T, H, E, K, seed=631, with_grad=False)
    st = api.new_status(dev)
    lay = _layout(inp["topk_idx"], E, 1, dev, st)
    topk = inp["topk_idx"].to(dev)
    N = capacity_rows(T, K, E, 1)
    lib = _lib.lib()
    x = torch.zeros(T, 24, dtype=torch.uint8, device=dev)        # 24-byte rows: not 16-byte units
    xp = torch.zeros(N, 24, dtype=torch.uint8, device=dev)
    r2f = torch.empty(N, dtype=torch.int32, device=dev)
    f2r = torch.empty(T, K, dtype=torch.int32, device=dev)
    args = lambda rb, aux, ab, auxp: (x.data_ptr(), rb, aux, ab, topk.data_ptr(), T, K, E,
                                      lay.expert_offsets.data_ptr(), lay.workspace.data_ptr(), 1, N,
                                      xp.data_ptr(), auxp, r2f.data_ptr(), f2r.data_ptr(),
                                      st.data_ptr(), None)
    assert lib.moe_permute_payload(*args(24, None, 0, None)) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_payload(*args(0, None, 0, None)) == _lib.MOE_ERR_INVALID_ARG
    a = torch.zeros(T, 2, dtype=torch.float32, device=dev)
    ap = torch.zeros(N, 2, dtype=torch.float32, device=dev)
    assert lib.moe_permute_payload(*args(16, a.data_ptr(), 8, None)) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_payload(*args(16, a.data_ptr(), 6, ap.data_ptr())) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_payload(*args(16, None, 8, ap.data_ptr())) == _lib.MOE_ERR_INVALID_ARG
    rows = torch.zeros(N, 6, dtype=torch.float32, device=dev)           # H % 4 != 0
    out = torch.zeros(T, 6, dtype=torch.float32, device=dev)
    assert lib.moe_combine_weighted_f32(rows.data_ptr(), N, None, f2r.data_ptr(), None, 0, T, K, 6,
                                        0, out.data_ptr(), st.data_ptr(), None) == _lib.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(st.item()) == 0
