"""Error paths of the CUDA path, injected on the host as bad data or bad
arguments (no GPU fault, trap or hang is provoked).  Each case expects the
documented status bit or return code, and canary guard zones around the
output buffers show that nothing was written out of bounds."""
import numpy as np
import pytest
import torch

from combine_moe_dispatch_03_b200.inputs import capacity_rows, custom_inputs

pytestmark = pytest.mark.gpu

GUARD = 64          # guard elements on each side of an output buffer
CANARY = 0x5A5A


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def guarded(n, dtype, dev):
    """A buffer of n elements between two CANARY-filled guard zones; returns
    (inner view, whole buffer)."""
    G = GUARD * 8
    if dtype == torch.bfloat16:
        full = torch.full((n + 2 * G,), CANARY, dtype=torch.int16, device=dev)
        return full[G:G + n].view(torch.bfloat16), full
    full = torch.full((n + 2 * G,), CANARY, dtype=dtype, device=dev)
    return full[G:G + n], full


def guards_intact(full):
    G = GUARD * 8
    return bool((full[:G] == CANARY).all() and (full[-G:] == CANARY).all())


def _api():
    from combine_moe_dispatch_03_b200 import api
    return api


def _setup(T=128, H=64, E=8, K=2, R=2, align=4, topk=None):
    api = _api()
    dev = torch.device("cuda:0")
    inp = custom_inputs(T, H, E, K, seed=17, topk_idx=topk)
    return api, dev, inp


# K = 2 runs the ring permute, K = 4 the register permute.
@pytest.mark.parametrize("K", [2, 4])
def test_expert_out_of_range_is_flagged_and_contained(K):
    T, H, E = 128, 64, 8
    topk = torch.randint(0, E, (T, K), generator=torch.Generator().manual_seed(1))
    topk[5, 1] = -1
    topk[77, 0] = E
    api, dev, inp = _setup(T, H, E, K, topk=topk)
    st = api.new_status(dev)
    lay = api.dispatch_layout(inp["topk_idx"].to(dev), E, 2, 4, status=st)
    torch.cuda.synchronize()
    assert st.item() & api._lib.ST_EXPERT_OOR
    assert int(lay.tokens_per_expert.sum()) == T * K - 2
    N = capacity_rows(T, K, E, 4)
    xp, xpf = guarded(N * H, torch.bfloat16, dev)
    r2f, r2ff = guarded(N, torch.int32, dev)
    f2r, f2rf = guarded(T * K, torch.int32, dev)
    st2 = api.new_status(dev)
    api.permute(inp["x"].to(dev), inp["topk_idx"].to(dev), lay, capacity=N, status=st2,
                out=(xp.view(N, H), r2f, f2r.view(T, K)))
    torch.cuda.synchronize()
    assert st2.item() & api._lib.ST_EXPERT_OOR
    assert guards_intact(xpf) and guards_intact(r2ff) and guards_intact(f2rf)
    f2r_h = f2r.view(T, K).cpu()
    assert f2r_h[5, 1] == -1 and f2r_h[77, 0] == -1
    with pytest.raises(RuntimeError, match="outside"):
        api.check_status(st2)


@pytest.mark.parametrize("K", [2, 4])
def test_capacity_overflow_is_flagged_and_contained(K):
    T, H, E, align = 64, 32, 8, 16
    api, dev, inp = _setup(T, H, E, K)
    lay = api.dispatch_layout(inp["topk_idx"].to(dev), E, 1, align)
    n_pad = int(lay.expert_offsets[-1])
    N = T * K                         # >= A (host check) but < padded total
    assert n_pad > N
    xp, xpf = guarded(N * H, torch.bfloat16, dev)
    r2f, r2ff = guarded(N, torch.int32, dev)
    f2r, f2rf = guarded(T * K, torch.int32, dev)
    st = api.new_status(dev)
    api.permute(inp["x"].to(dev), inp["topk_idx"].to(dev), lay, capacity=N, status=st,
                out=(xp.view(N, H), r2f, f2r.view(T, K)))
    y, yf = guarded(N * H, torch.bfloat16, dev)
    api.expert_scale(xp.view(N, H), lay, inp["scales"].to(dev), status=st, out=y.view(N, H))
    torch.cuda.synchronize()
    assert st.item() & api._lib.ST_CAPACITY
    assert all(guards_intact(b) for b in (xpf, r2ff, f2rf, yf))
    assert int((f2r >= N).sum()) == 0


def _pipeline(api, dev, inp, E, R, align):
    lay = api.dispatch_layout(inp["topk_idx"].to(dev), E, R, align)
    xp, r2f, f2r = api.permute(inp["x"].to(dev), inp["topk_idx"].to(dev), lay)
    return lay, xp, r2f, f2r


def test_coverage_validation():
    T, H, E, K = 128, 64, 8, 2
    api, dev, inp = _setup(T, H, E, K)
    lay, xp, r2f, f2r = _pipeline(api, dev, inp, E, 2, 4)
    w = inp["weights"].to(dev)
    st = api.new_status(dev)
    api.combine_weighted(xp, f2r, w, row_to_flat=r2f, validate=True, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    # a (token, slot) whose row was never set: its row claims no flat index
    bad = r2f.clone()
    bad[int(f2r[3, 1])] = -1
    st = api.new_status(dev)
    api.combine_weighted(xp, f2r, w, row_to_flat=bad, validate=True, status=st)
    torch.cuda.synchronize()
    assert st.item() & api._lib.ST_COVERAGE
    # two slots pointing at the same row
    bad_f = f2r.clone()
    bad_f[4, 0] = f2r[9, 1]
    st = api.new_status(dev)
    api.combine_weighted(xp, bad_f, w, row_to_flat=r2f, validate=True, status=st)
    torch.cuda.synchronize()
    assert st.item() & api._lib.ST_COVERAGE
    # a stray row claiming a flat index
    bad = r2f.clone()
    pad = int(torch.nonzero(r2f < 0)[0])
    bad[pad] = 0
    st = api.new_status(dev)
    api.combine_weighted(xp, f2r, w, row_to_flat=bad, validate=True, status=st)
    torch.cuda.synchronize()
    assert st.item() & api._lib.ST_COVERAGE
    with pytest.raises(RuntimeError, match="cover every"):
        api.check_status(st)


def test_row_out_of_range_is_flagged_and_skipped():
    T, H, E, K = 64, 64, 4, 2
    api, dev, inp = _setup(T, H, E, K)
    lay, xp, r2f, f2r = _pipeline(api, dev, inp, E, 1, 4)
    bad_f = f2r.clone()
    bad_f[2, 1] = xp.shape[0] + 5
    bad_f[7, 0] = -3
    w = inp["weights"].to(dev)
    st = api.new_status(dev)
    out = api.combine_weighted(xp, bad_f, w, status=st)
    g = inp["grad_out"].to(dev)
    gr, gw = api.combine_backward(g, xp, r2f, bad_f, w, lay, status=st)
    torch.cuda.synchronize()
    assert st.item() & api._lib.ST_ROW_OOR
    assert float(gw[2, 1]) == 0.0 and float(gw[7, 0]) == 0.0
    want = (w[2, 0] * xp[f2r[2, 0]].float()).to(torch.bfloat16)
    assert torch.equal(out[2].view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("K", [2, 4])
def test_workspace_mismatch_writes_nothing(K):
    api, dev, inp = _setup(64, 32, 8, K)
    lay = api.dispatch_layout(inp["topk_idx"].to(dev), 8, 2, 4)
    inp2 = custom_inputs(32, 32, 8, K, seed=3)
    N = capacity_rows(32, K, 8, 4)
    xp = torch.full((N, 32), 7, dtype=torch.int16, device=dev).view(torch.bfloat16)
    r2f = torch.full((N,), 7, dtype=torch.int32, device=dev)
    f2r = torch.full((32, K), 7, dtype=torch.int32, device=dev)
    st = api.new_status(dev)
    # Through the C ABI: the Python layer would refuse this on the host (see
    # test_python_layer_refuses_mismatched_shapes); the device check is what
    # guards a C caller.
    from combine_moe_dispatch_03_b200._lib import lib
    x2, t2 = inp2["x"].to(dev), inp2["topk_idx"].to(dev)
    rc = lib().moe_permute(x2.data_ptr(), t2.data_ptr(), 32, K, 8, 32,
                           lay.expert_offsets.data_ptr(), lay.workspace.data_ptr(), 1, N,
                           xp.data_ptr(), r2f.data_ptr(), f2r.data_ptr(), st.data_ptr(),
                           torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert st.item() & api._lib.ST_LAYOUT_MISMATCH
    assert bool((r2f == 7).all()) and bool((f2r == 7).all())


def test_python_layer_refuses_mismatched_shapes():
    """Tensors whose sizes disagree with each other or with the layout are
    refused by the binding before anything is enqueued."""
    api, dev, inp = _setup(64, 32, 8, 2)
    topk = inp["topk_idx"].to(dev)
    x = inp["x"].to(dev)
    st = api.new_status(dev)
    lay = api.dispatch_layout(topk, 8, 2, 4, status=st)
    xp, r2f, f2r = api.permute(x, topk, lay, status=st)
    w = inp["weights"].to(dev)
    torch.cuda.synchronize()
    with pytest.raises(ValueError):                     # topk_idx rows != x rows
        api.permute(x[:32].contiguous(), topk, lay)
    with pytest.raises(ValueError):                     # layout built for other T
        api.permute(x[:32].contiguous(), topk[:32].contiguous(), lay)
    with pytest.raises(ValueError):                     # undersized output
        api.combine_weighted(xp, f2r, w, out=torch.empty(63, 32, dtype=torch.bfloat16,
                                                         device=dev))
    with pytest.raises(ValueError):                     # grad_out of the wrong size
        api.combine_backward(torch.zeros(64, 16, dtype=torch.bfloat16, device=dev), xp, r2f,
                             f2r, w, lay)
    with pytest.raises(ValueError):                     # scales of the wrong length
        api.expert_scale(xp, lay, torch.ones(7, device=dev))
    with pytest.raises(ValueError):                     # reused layout of other sizes
        api.dispatch_layout(topk[:32].contiguous(), 8, 2, 4, out=lay)
    with pytest.raises(ValueError):                     # one-call dispatch: topk rows != x rows
        api.dispatch(x[:32].contiguous(), topk, 8, 2, 4)
    with pytest.raises(ValueError):                     # ... a layout of other sizes
        api.dispatch(x[:32].contiguous(), topk[:32].contiguous(), 8, 2, 4, layout_out=lay)
    with pytest.raises(ValueError):                     # ... an undersized row map
        api.dispatch(x, topk, 8, 2, 4, out=(xp, r2f[:10], f2r))
    torch.cuda.synchronize()
    assert st.item() == 0


@pytest.mark.parametrize("case", ["H%8", "misaligned", "ncap<A", "E%R", "T%R", "K>32", "E>1024"])
def test_host_checks_launch_nothing(case):
    from combine_moe_dispatch_03_b200._lib import lib
    api = _api()
    dev = torch.device("cuda:0")
    T, H, E, K = 64, 64, 8, 2
    inp = custom_inputs(T, H, E, K, seed=2)
    topk = inp["topk_idx"].to(dev)
    st = api.new_status(dev)
    lay = api.dispatch_layout(topk, E, 2, 4)
    N = capacity_rows(T, K, E, 4)
    x = inp["x"].to(dev)
    xp = torch.zeros(N + 8, H, dtype=torch.bfloat16, device=dev)
    r2f = torch.zeros(N, dtype=torch.int32, device=dev)
    f2r = torch.zeros(T, K, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()
    args = dict(x=P(x), topk=P(topk), T=T, K=K, E=E, H=H, N=N, xp=P(xp))
    if case == "H%8":
        args["H"] = 60
    elif case == "misaligned":
        args["xp"] = P(xp) + 2
    elif case == "ncap<A":
        args["N"] = T * K - 1
    elif case == "K>32":
        args["K"] = 33
    elif case == "E>1024":
        args["E"] = 1025
    if case in ("E%R", "T%R"):
        ws = torch.zeros(1 << 20, dtype=torch.uint8, device=dev)
        rc = lib().moe_dispatch_layout(
            P(topk), T if case == "E%R" else T - 1, K, E if case == "T%R" else E - 1, 2, 4,
            P(lay.tokens_per_expert), P(lay.counts), P(lay.splits), P(lay.tokens_per_rank),
            P(lay.is_token_in_rank), P(lay.expert_offsets), P(ws), P(st), s)
    else:
        rc = lib().moe_permute(args["x"], args["topk"], T, args["K"], args["E"], args["H"],
                               P(lay.expert_offsets), P(lay.workspace), 1, args["N"], args["xp"],
                               P(r2f), P(f2r), P(st), s)
    assert rc == -1
    torch.cuda.synchronize()
    assert st.item() == 0
    assert not xp.view(torch.int16).any() and not r2f.any() and not f2r.any()
