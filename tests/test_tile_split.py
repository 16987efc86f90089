"""The split of a layer's row tiles over the fused kernel's CTAs (host logic,
no GPU), as sqz_create_layer computes it: the even split for uniform
outliers, and for outliers skewed over the rows a split of consecutive runs
(1 to twice the even count of tiles each) whose heaviest run is as light as
possible, where a tile weighs w x its 256-column units + its nonzeros
(w = 100 at 3 bits, 150 at 4), used only when it lowers the heaviest CTA's
weight by more than 5 %.  Checked against an exhaustive dynamic program on
small random layers and on the workloads' layers."""
import numpy as np
import pytest

import synth
from lut_dequant_gemv_b200 import binding as B


def tile_weights(rowptr, n_out, k_in, bits):
    ntiles = (n_out + 15) // 16
    nsteps = -(-k_in // 16)
    nsg = -(-nsteps // 16)
    unit = 100 if bits == 3 else 150
    return [nsg * unit + int(rowptr[min(n_out, 16 * t + 16)] - rowptr[16 * t]) for t in range(ntiles)]


def even_split(ntiles, grid):
    q, r = divmod(ntiles, grid)
    return [c * q + min(c, r) for c in range(grid + 1)]


def heaviest(first, w):
    pre = np.concatenate([[0], np.cumsum(w)])
    return max(int(pre[first[c + 1]] - pre[first[c]]) for c in range(len(first) - 1))


def best_heaviest(w, grid, cap):
    """Least possible heaviest run over all splits of the tiles into exactly
    `grid` consecutive runs of 1..cap tiles (exhaustive dynamic program)."""
    n = len(w)
    pre = np.concatenate([[0], np.cumsum(w)])
    inf = float("inf")
    dp = [[inf] * (n + 1) for _ in range(grid + 1)]
    dp[0][0] = 0
    for c in range(1, grid + 1):
        for t in range(1, n + 1):
            for k in range(1, min(cap, t) + 1):
                if dp[c - 1][t - k] < inf:
                    dp[c][t] = min(dp[c][t], max(dp[c - 1][t - k], int(pre[t] - pre[t - k])))
    return dp[grid][n]


def skewed_rowptr(rng, n_out, k_in, total):
    """Row counts drawn with Zipf weights 1/r over a random row order, capped at K."""
    p = 1.0 / np.arange(1, n_out + 1)
    p = p[rng.permutation(n_out)]
    counts = np.minimum(rng.multinomial(total, p / p.sum()), k_in)
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def check_split(rowptr, n_out, k_in, bits, sms):
    ntiles = (n_out + 15) // 16
    grid = min(sms, ntiles)
    first, weighted = B.sqz_tile_split_query(rowptr, n_out, k_in, bits, sm_count=sms)
    first = [int(v) for v in first]
    w = tile_weights(rowptr, n_out, k_in, bits)
    even = even_split(ntiles, grid)
    assert len(first) == grid + 1 and first[0] == 0 and first[-1] == ntiles
    cap = 2 * (-(-ntiles // grid))
    assert all(1 <= first[c + 1] - first[c] <= cap for c in range(grid)), first
    if int(rowptr[-1]) == 0 or grid == 1:
        assert not weighted and first == even
        return weighted
    opt = best_heaviest(w, grid, cap)
    if weighted:
        assert heaviest(first, w) == opt, (first, opt)
        assert opt * 100 < heaviest(even, w) * 95
    else:
        assert first == even
        assert opt * 100 >= heaviest(even, w) * 95
    return weighted


@pytest.mark.parametrize("seed", range(40))
def test_split_by_weight_is_the_lightest_on_small_layers(seed):
    rng = np.random.default_rng(1000 + seed)
    ntiles = int(rng.integers(2, 41))
    n_out = 16 * ntiles - int(rng.integers(0, 16))
    sms = int(rng.integers(2, 9))
    bits = int(rng.choice([3, 4]))
    k_in = 256 * int(rng.integers(1, 5)) - (int(rng.integers(0, 8)) * 32 if bits == 3 else 0)
    k_in = max(k_in, 32)
    # from uniform to a few rows holding most outliers
    total = int(rng.integers(0, 40 * n_out))
    if seed % 3 == 0:
        counts = rng.multinomial(total, np.full(n_out, 1.0 / n_out))
        rowptr = np.concatenate([[0], np.cumsum(np.minimum(counts, k_in))]).astype(np.int32)
    else:
        rowptr = skewed_rowptr(rng, n_out, k_in, total)
    check_split(rowptr, n_out, k_in, bits, sms)


def test_splits_of_the_workload_layers():
    seen = set()
    for name, shapes in synth.workloads().items():
        for s in shapes:
            if s.key in seen or s.density == 0 or s.n_out * s.k_in > 5120 * 13824:
                continue
            seen.add(s.key)
            L = synth.layer_for(s)
            first, weighted = B.sqz_tile_split_query(L.rowptr, L.n_out, L.k_in, L.bits)
            assert weighted == (s.dist == "skew"), s.key
            w = tile_weights(L.rowptr, L.n_out, L.k_in, L.bits)
            ntiles, grid = len(w), len(first) - 1
            if weighted:
                # the skewed layers: heaviest CTA well below the even split's
                assert heaviest(list(first), w) * 100 < heaviest(even_split(ntiles, grid), w) * 95
            else:
                assert list(first) == even_split(ntiles, grid)


def test_a_layer_without_outliers_keeps_the_even_split():
    first, weighted = B.sqz_tile_split_query(np.zeros(1001, np.int32), 1000, 4096, 3, sm_count=8)
    assert not weighted and list(first) == even_split(63, 8)


def test_tile_split_query_rejects_bad_arguments():
    rp = np.zeros(65, np.int32)
    for args in ((rp, 64, 4096, 5), (rp, 64, 0, 3)):
        with pytest.raises(B.SqzError) as e:
            B.sqz_tile_split_query(*args)
        assert e.value.status == B.SQZ_ERR_INVALID_ARG
    with pytest.raises(B.SqzError):
        B.sqz_tile_split_query(rp, 64, 4096, 3, sm_count=0)
    bad = rp.copy()
    bad[10] = 5  # rowptr decreases after row 10
    with pytest.raises(B.SqzError):
        B.sqz_tile_split_query(bad, 64, 4096, 3)
    bad = rp + 1  # does not start at 0
    with pytest.raises(B.SqzError):
        B.sqz_tile_split_query(bad, 64, 4096, 3)
    with pytest.raises(ValueError):
        B.sqz_tile_split_query(rp[:-1], 64, 4096, 3)
