"""moe_dispatch_layout_noalloc -- the layout for callers that cannot allocate
device memory (a plugin inside a server or framework that owns the device's
memory pool, or a path where cudaMalloc/cudaFree must not run because they can
synchronise the device).  Its workspace is a static device array inside the
library, so the call itself allocates nothing.

Checked through the C ABI against moe_dispatch_layout (caller workspace) on
two calls in a row with different sizes, so that a stale result left in the
shared array by the first call would show up in the second.  The outputs are
integers, so they must match exactly.  This file is collected last."""
import pytest
import torch

from combine_moe_dispatch_03_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _outputs(T, E, R, dev):
    i32 = dict(dtype=torch.int32, device=dev)
    return dict(tokens_per_expert=torch.full((E,), -7, **i32),
                counts=torch.full((R, R, E // R), -7, **i32),
                splits=torch.full((R, R), -7, **i32),
                tokens_per_rank=torch.full((R, R), -7, **i32),
                is_token_in_rank=torch.full((T, R), 9, dtype=torch.uint8, device=dev),
                expert_offsets=torch.full((E + 1,), -7, **i32))


def _call_noalloc(L, topk, T, K, E, R, align, out, status, stream):
    P = lambda t: t.data_ptr()
    return L.moe_dispatch_layout_noalloc(
        P(topk), T, K, E, R, align, P(out["tokens_per_expert"]), P(out["counts"]),
        P(out["splits"]), P(out["tokens_per_rank"]), P(out["is_token_in_rank"]),
        P(out["expert_offsets"]), P(status), stream)


def test_noalloc_layout_matches_layout_with_workspace():
    from combine_moe_dispatch_03_b200 import api
    from combine_moe_dispatch_03_b200._lib import lib
    L = lib()
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev).cuda_stream
    for name in ("qwen3", "dsv3_skew"):                    # two calls, different sizes
        inp = make_inputs(name, H=8)
        cfg = inp["cfg"]
        topk = inp["topk_idx"].to(dev)
        ref = api.dispatch_layout(topk, cfg.E, cfg.R, cfg.align)
        out = _outputs(cfg.T, cfg.E, cfg.R, dev)
        status = api.new_status(dev)
        rc = _call_noalloc(L, topk, cfg.T, cfg.K, cfg.E, cfg.R, cfg.align, out, status, stream)
        assert rc == 0, L.moe_strerror(rc)
        torch.cuda.synchronize(dev)
        assert int(status.item()) == 0
        for key, t in out.items():
            assert torch.equal(t, getattr(ref, key)), f"{name}: {key} differs"


def test_noalloc_rejects_sizes_beyond_the_scratch():
    from combine_moe_dispatch_03_b200 import api
    from combine_moe_dispatch_03_b200._lib import MOE_ERR_SCRATCH, NOALLOC_SCRATCH_BYTES, lib
    L = lib()
    T, K, E, R = 1 << 20, 32, 1024, 1                       # workspace far above 4 MiB
    assert L.moe_layout_workspace_bytes(T, K, E, R) > NOALLOC_SCRATCH_BYTES
    dev = torch.device("cuda:0")
    status = api.new_status(dev)
    dummy = torch.zeros(16, dtype=torch.int64, device=dev)
    p = dummy.data_ptr()
    rc = L.moe_dispatch_layout_noalloc(p, T, K, E, R, 1, p, p, p, p, p, p, status.data_ptr(),
                                       torch.cuda.current_stream(dev).cuda_stream)
    assert rc == MOE_ERR_SCRATCH
    assert b"static scratch" in L.moe_strerror(rc)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0 and not dummy.any()
