"""GPU selector study (the library's selector, not the oracle's).

1. On the study's small clustered case, the GPU selector and the oracle give
   the same mask bit for bit for each variant the study compares: centroid
   branch only, rescue branch only, and their OR (thresholds placed in >= 1e-3
   gaps of the fp64 scores; a switched-off branch gets +inf).
2. A reduced run of the study at the 32768-token workload shape: densities are
   matched, retention is a fraction, and the per-row upper bound is never
   below the OR variant it takes its budgets from.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import workloads as W
from tests import selector_study_gpu as S
from tests.helpers import csr_to_mask, tau_in_gap

pytestmark = pytest.mark.gpu


def test_gpu_selector_matches_oracle_for_each_study_variant(cuda_dev):
    wl = W.clustered_prefill(2001, T=4096, Hq=8, Hkv=2, d=128, block=64, n_clusters=32)
    T, Hq, d = wl.q.shape
    nB = T // 64
    scale = 1 / math.sqrt(d)
    c, r = oracle.block_stats(wl.cache, 64)
    qbar, qn = oracle.pool_q(wl.q, 64)
    Sc, Sr = oracle.pair_scores(qbar, qn, c, r, scale)
    tc = [tau_in_gap(Sc[h], 0.9)[0] for h in range(Hq)]
    tr = [tau_in_gap(Sr[h], 0.93)[0] for h in range(Hq)]
    inf = [math.inf] * Hq
    gc, gq = wl.cache.to(cuda_dev), wl.q.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    for name, a, b in [("centroid", tc, inf), ("rescue", inf, tr), ("or", tc, tr)]:
        want = oracle.rbs_mask(Sc, Sr, a, b, True, True)
        csr = sa.select_blocks_rbs(gc, gq, 64, scale, tau_c=torch.tensor(a), tau_r=torch.tensor(b), ws=ws)
        ws.raise_on_fault(name)
        got = csr_to_mask(csr.row_ptr.cpu().numpy(), csr.cols.cpu().numpy(), Hq, nB)
        np.testing.assert_array_equal(got, want, err_msg=name)


def test_reduced_gpu_study_at_workload_shape(cuda_dev):
    rows = S.run(32768, densities=(0.10,), deltas=(0.02,), heads=(0, 17), n_rows=24, dev=cuda_dev)
    assert len(rows) == 1
    r = rows[0]
    for key in ("centroid", "rescue", "or_0.02", "row_upper"):
        mean, low, dens = r[key][:3]
        assert abs(dens - 0.10) <= 0.0025 + 1e-9, (key, dens)
        assert 0.0 <= mean <= 1.0 and 0.0 <= low <= 1.0
    assert r["row_upper"][0] >= r["or_0.02"][0] - 1e-12
