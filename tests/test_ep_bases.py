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
