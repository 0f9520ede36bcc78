"""The selector study's machinery on a reduced clustered workload (CPU):
the true block mass is a causal distribution, densities are matched, the
retention grows with density, and the per-block upper bound (best pairs by
true mass at the same per-head kept counts) dominates the variant it is
matched to.  The full study is ``python -m tests.selector_study``."""
import math

import numpy as np

from sparse_attention_aware_b200 import workloads as W
from tests import selector_study as S
from tests.helpers import dense_kv


def test_true_block_mass_is_a_causal_distribution():
    wl = W.clustered_prefill(7, T=300, Hq=2, Hkv=1, d=128, block=64, n_clusters=8)
    K, _ = dense_kv(wl.cache, 0, 0, 300)
    M = S.true_block_mass(wl.q, K, 1 / math.sqrt(128), 32)
    assert M.shape == (2, 300, 10)
    np.testing.assert_allclose(M.sum(axis=2), 1.0, atol=1e-12)
    blk = np.arange(300) // 32
    for j in range(10):
        assert np.all(M[:, blk < j, j] == 0)        # no mass on future blocks
    assert np.all(M[:, 0, 0] == 1.0)                # the first token sees only itself


def test_study_matches_density_and_orders_sensibly():
    rows = S.run_study(T=2048, Hq=2, block_sizes=(32,), densities=(0.15, 0.3), deltas=(0.02,))
    assert len(rows) == 2
    for r in rows:
        for key in ("centroid", "rescue", "or_0.02", "upper"):
            mean, low, dens = r[key]
            assert abs(dens - r["density"]) <= 0.0025 + 1e-9 and 0.0 <= mean <= 1.0 and 0.0 <= low <= 1.0
        assert r["upper"][0] >= r["or_0.02"][0] - 1e-12
    for key in ("centroid", "rescue", "or_0.02", "upper"):
        assert rows[1][key][0] > rows[0][key][0]
