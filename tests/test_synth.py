"""The synthetic input generator emits well-formed storage (no GPU needed):
CSR with rowptr[0] = 0, rowptr[N] = nnz, non-decreasing rowptr, columns in
[0, K), strictly ascending within a row; the skewed outlier distribution
concentrates the outliers on few rows."""
import numpy as np
import pytest

import synth


@pytest.mark.parametrize("dist", ["uniform", "t3", "skew"])
def test_outliers_are_well_formed_csr(dist):
    n, k = 700, 512
    L = synth.make_layer(n, k, 3, 0.01, key=f"csr-{dist}", dist=dist)
    rp, col = L.rowptr.astype(np.int64), L.col.astype(np.int64)
    assert rp[0] == 0 and rp[-1] == L.nnz and np.all(np.diff(rp) >= 0)
    assert np.all((col >= 0) & (col < k))
    for i in range(n):
        assert np.all(np.diff(col[rp[i]:rp[i + 1]]) > 0)
    if dist != "skew":
        assert L.nnz == synth.nnz_for(n, k, 0.01)


def test_skewed_outliers_concentrate_on_few_rows():
    n, k = 2000, 1024
    L = synth.make_layer(n, k, 3, 0.0045, key="skew-shape", dist="skew")
    counts = np.diff(L.rowptr)
    assert counts.max() == k                      # the heaviest rows are entirely outliers
    assert np.sort(counts)[-n // 100:].sum() > 0.15 * L.nnz   # 1 % of the rows hold > 15 %
    assert 0.8 * synth.nnz_for(n, k, 0.0045) <= L.nnz <= synth.nnz_for(n, k, 0.0045)
    u = synth.make_layer(n, k, 3, 0.0045, key="skew-shape")
    assert np.diff(u.rowptr).max() < k // 8
