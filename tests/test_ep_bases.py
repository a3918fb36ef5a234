"""The row bases of the direct (send-buffer-free) expert-parallel dispatch.

On CPU, the oracle's definition (oracle_rank_bases) is pinned to the
oracle's single-device rows: with the ranks as logical groups, the
single-device layout puts assignment f = (t, k) of expert e at row(f); the
buffer of e's owner rank r holds rows [off[r*E_local], off[(r+1)*E_local])
of it.  So rank s's assignment of e must land at row(f) - off[r*E_local] in
r's buffer, which is dest_base[e] + (its stable rank among s's own
assignments of e); the owner's padded group starts and real rows must be
that slice's offsets and counts.  A property test over random count
matrices checks the tiling.  On the GPU, the library's moe_rank_bases must
equal the oracle bit for bit."""
import numpy as np
import pytest
import torch

import oracle as orc


@pytest.mark.parametrize("R,E,K,Tb,align,seed", [(4, 32, 4, 200, 8, 1), (8, 64, 8, 64, 16, 2),
                                                 (2, 6, 3, 50, 1, 3), (3, 9, 2, 31, 5, 4)])
def test_rank_bases_match_single_device_rows(R, E, K, Tb, align, seed):
    orc.build()
    rng = np.random.default_rng(seed)
    T, El = R * Tb, E // R
    topk = rng.integers(0, E, size=(T, K)).astype(np.int64)
    topk[: T // 3] = rng.integers(0, max(1, E // 4), size=(T // 3, K))     # skew, repeats
    lay = orc.layout(topk, E, R, align)
    off = lay["expert_offsets"]
    pm = orc.permute(np.zeros((T, 8), np.uint16), topk, E, off, int(off[-1]))
    all_counts = np.stack([orc.layout(topk[s * Tb:(s + 1) * Tb], E, 1, 1)["tokens_per_expert"]
                           for s in range(R)])
    for s in range(R):
        rb = orc.rank_bases(all_counts, s, align)
        assert rb["status"] == 0
        assert rb["max_rows"] == max(int(off[(r + 1) * El] - off[r * El]) for r in range(R))
        dest_base, own_off, own_cnt = rb["dest_base"], rb["own_offsets"], rb["own_counts"]
        np.testing.assert_array_equal(own_off, off[s * El:(s + 1) * El + 1] - off[s * El])
        np.testing.assert_array_equal(own_cnt, lay["tokens_per_expert"][s * El:(s + 1) * El])
        seen = np.zeros(E, np.int64)
        for t in range(s * Tb, (s + 1) * Tb):
            for k in range(K):
                e = int(topk[t, k])
                r = e // El
                want = int(pm["flat_to_row"][t, k]) - int(off[r * El])
                assert dest_base[e] + seen[e] == want, (s, t, k)
                seen[e] += 1


def test_rank_bases_tile_every_group_exactly():
    """Random count matrices (hypothesis): for every expert e, the ranks'
    row ranges [dest_base_s[e], dest_base_s[e] + counts[s][e]) tile the real
    rows of e's group in its owner's buffer exactly, in rank order; the
    groups are aligned, contiguous, padded by less than the alignment and
    do not overlap; the buffer size is the largest owner's padded total."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=200, deadline=None)
    @given(R=st.integers(1, 6), El=st.integers(1, 5), align=st.integers(1, 9),
           data=st.data())
    def check(R, El, align, data):
        E = R * El
        c = np.array(data.draw(st.lists(st.integers(0, 40), min_size=R * E, max_size=R * E)),
                     np.int32).reshape(R, E)
        total = c.sum(axis=0)
        cap = orc.rank_bases(c, 0, align)["max_rows"]
        owner_sizes = []
        for s in range(R):
            rb = orc.rank_bases(c, s, align)
            base, own_off, own_cnt = rb["dest_base"], rb["own_offsets"], rb["own_counts"]
            assert rb["max_rows"] == cap
            assert own_off[0] == 0 and np.all(np.diff(own_off) >= own_cnt)
            assert np.all(own_off[:-1] % align == 0)
            assert np.all(np.diff(own_off) - own_cnt < align)
            np.testing.assert_array_equal(own_cnt, total[s * El:(s + 1) * El])
            owner_sizes.append(int(own_off[-1]))
            for e in range(E):
                r, el = divmod(e, El)
                r_off = orc.rank_bases(c, r, align)["own_offsets"]
                assert base[e] == int(r_off[el]) + int(c[:s, e].sum())
        assert cap == max(owner_sizes)

    check()


@pytest.mark.parametrize("R,E,K,Tb,H,align,seed", [(4, 16, 3, 40, 8, 4, 5), (3, 9, 2, 25, 16, 1, 6),
                                                   (2, 8, 4, 33, 8, 8, 7)])
def test_receive_buffers_by_definition(R, E, K, Tb, H, align, seed):
    """Brute force from the definition of expert parallelism: rank r's
    receive buffer holds, for each of its experts e in order, the rows
    x[t] of every assignment (t, k) with topk[t, k] == e, source ranks in
    order, each source's tokens then slots in order, padded with zeros to the
    alignment.  That buffer is exactly rows [off[r*E_local], off[(r+1)*E_local])
    of the oracle's single-device grouped buffer, and rank s's align-1
    permute of its own tokens is its send buffer: destination rank, local
    expert, token, slot."""
    orc.build()
    rng = np.random.default_rng(seed)
    T, El = R * Tb, E // R
    topk = rng.integers(0, E, size=(T, K)).astype(np.int64)
    x = rng.integers(1, 0x7F00, size=(T, H)).astype(np.uint16)       # distinct-ish, nonzero rows
    lay = orc.layout(topk, E, R, align)
    off = lay["expert_offsets"]
    single = orc.permute(x, topk, E, off, int(off[-1]))["x_perm"]
    for r in range(R):
        rows = []
        for e in range(r * El, (r + 1) * El):
            n = 0
            for s in range(R):
                for t in range(s * Tb, (s + 1) * Tb):
                    for k in range(K):
                        if topk[t, k] == e:
                            rows.append(x[t])
                            n += 1
            rows.extend([np.zeros(H, np.uint16)] * ((-n) % align))
        recv = np.array(rows, np.uint16).reshape(-1, H)
        np.testing.assert_array_equal(recv, single[off[r * El]:off[(r + 1) * El]])
    for s in range(R):
        mine = topk[s * Tb:(s + 1) * Tb]
        lay_s = orc.layout(mine, E, 1, 1)
        send = orc.permute(x[s * Tb:(s + 1) * Tb], mine, E, lay_s["expert_offsets"], Tb * K)["x_perm"]
        want = [x[s * Tb + t] for e in range(E) for t in range(Tb) for k in range(K)
                if mine[t, k] == e]
        np.testing.assert_array_equal(send, np.array(want, np.uint16).reshape(-1, H))


def test_oracle_rank_bases_negative_count():
    """A negative count is an error (counted as 0), as the library reports."""
    c = np.array([[1, -2], [3, 4]], np.int32)
    rb = orc.rank_bases(c, 1, 1)
    assert rb["status"] == orc.COVERAGE
    np.testing.assert_array_equal(rb["dest_base"], [1, 0])


@pytest.mark.gpu
def test_rank_bases_device_equals_oracle():
    """moe_rank_bases through the C ABI, bit for bit against the oracle, on
    random count matrices (hypothesis; up to the limits: E = 1024 experts,
    R = 64 ranks), on the DeepSeek-V3 shape's seeded routing, and with a
    negative count (MOE_ST_COVERAGE)."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    from combine_moe_dispatch_03_b200 import api, build
    from combine_moe_dispatch_03_b200.inputs import make_inputs
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")

    def check(c, rank, align):
        want = orc.rank_bases(c, rank, align)
        stt = api.new_status(dev)
        got = api.rank_bases(torch.from_numpy(c).to(dev), rank, align, status=stt)
        assert int(stt.item()) == want["status"]
        for name, g in zip(("dest_base", "own_offsets", "own_counts"), got[:3]):
            np.testing.assert_array_equal(g.cpu().numpy(), want[name], err_msg=name)
        assert int(got[3].item()) == want["max_rows"]

    @settings(max_examples=150, deadline=None)
    @given(R=st.sampled_from([1, 2, 3, 4, 8, 64]), El=st.integers(1, 16), align=st.integers(1, 130),
           data=st.data())
    def random_matrices(R, El, align, data):
        E = R * El
        seed = data.draw(st.integers(0, 2 ** 31 - 1))
        hi = data.draw(st.sampled_from([0, 3, 40, 5000]))
        c = np.random.default_rng(seed).integers(0, hi + 1, size=(R, E)).astype(np.int32)
        rank = data.draw(st.integers(0, R - 1))
        check(c, rank, align)

    random_matrices()
    rng = np.random.default_rng(11)
    check(rng.integers(0, 300, size=(64, 1024)).astype(np.int32), 37, 128)     # the limits
    tk = make_inputs("dsv3_skew")["topk_idx"].numpy()
    c = np.stack([orc.layout(tk[s * 1024:(s + 1) * 1024], 256, 1, 1)["tokens_per_expert"]
                  for s in range(8)])
    for rank in range(8):
        check(c, rank, 128)
    bad = c.copy()
    bad[3, 17] = -5
    check(bad, 2, 128)
