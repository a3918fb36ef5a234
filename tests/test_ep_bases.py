"""The row bases of the direct (send-buffer-free) expert-parallel dispatch,
on CPU against the oracle: with the ranks as logical groups, the oracle's
single-device layout puts assignment f = (t, k) of expert e at row(f); the
buffer of e's owner rank r holds rows [off[r*E_local], off[(r+1)*E_local])
of it.  So rank s's assignment of e must land at row(f) - off[r*E_local] in
r's buffer, which is dest_base[e] + (its stable rank among s's own
assignments of e); the owner's padded group starts and real rows must be
that slice's offsets and counts."""
import numpy as np
import pytest
import torch

import oracle as orc
from combine_moe_dispatch_03_b200 import ep


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
    all_counts = torch.stack([
        torch.from_numpy(orc.layout(topk[s * Tb:(s + 1) * Tb], E, 1, 1)["tokens_per_expert"])
        for s in range(R)])
    assert ep.direct_receive_rows(all_counts, align) == max(
        int(off[(r + 1) * El] - off[r * El]) for r in range(R))
    for s in range(R):
        dest_base, own_off, own_cnt = ep.rank_bases(all_counts, s, align)
        dest_base = dest_base.numpy()
        np.testing.assert_array_equal(own_off.numpy(), off[s * El:(s + 1) * El + 1] - off[s * El])
        np.testing.assert_array_equal(own_cnt.numpy(), lay["tokens_per_expert"][s * El:(s + 1) * El])
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
        all_counts = torch.from_numpy(c)
        total = c.sum(axis=0)
        cap = ep.direct_receive_rows(all_counts, align)
        owner_sizes = []
        for s in range(R):
            base, own_off, own_cnt = (t.numpy() for t in ep.rank_bases(all_counts, s, align))
            assert own_off[0] == 0 and np.all(np.diff(own_off) >= own_cnt)
            assert np.all(own_off[:-1] % align == 0)
            assert np.all(np.diff(own_off) - own_cnt < align)
            np.testing.assert_array_equal(own_cnt, total[s * El:(s + 1) * El])
            owner_sizes.append(int(own_off[-1]))
            for e in range(E):
                r, el = divmod(e, El)
                _, r_off, _ = ep.rank_bases(all_counts, r, align)
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
