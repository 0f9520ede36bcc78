"""GPU parity: RBS two-branch block selection (CSR masks bit-exact).

Thresholds are placed inside >= 1e-3 gaps of the oracle's fp64 pair scores so
that the fp32 GPU scores provably fall on the same side; quantile mode is
checked bit-exact on tiny inputs with every sorted gap >= 1e-3, and at full
size through exact kept counts of one branch.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import csr_to_mask, tau_in_gap

pytestmark = pytest.mark.gpu


def _oracle_scores(wl, scale):
    c, r = oracle.block_stats(wl.cache, wl.block)
    qbar, qn = oracle.pool_q(wl.q, wl.block)
    return oracle.pair_scores(qbar, qn, c, r, scale)


def _score_error_bound(wl, scale):
    """Per head: 4 * 2^-18 * scale * max over pairs of sum_k |qbar_ik c_jk|."""
    c, _ = oracle.block_stats(wl.cache, wl.block)
    qbar, _ = oracle.pool_q(wl.q, wl.block)
    Hq, Hkv = qbar.shape[0], c.shape[0]
    return np.array([4 * 2.0 ** -18 * scale * (np.abs(qbar[h]) @ np.abs(c[h // (Hq // Hkv)]).T).max()
                     for h in range(Hq)])


def _gpu_mask(cuda_dev, wl, csr):
    nB = (wl.T + 63) // 64
    rp = csr.row_ptr.cpu().numpy()
    return csr_to_mask(rp, csr.cols.cpu().numpy()[: rp[-1]], wl.q.shape[1], nB)


@pytest.mark.parametrize("T,Hq,Hkv,P,pc,pr", [
    (1000, 8, 2, 64, 0.9, 0.95),
    (4096, 8, 1, 16, 0.95, 0.97),
    (2000, 4, 4, 64, 0.5, 0.8),
    (20000, 4, 2, 64, 0.9, 0.95),     # 313 blocks: three 128-block row tiles, ragged tail
])
def test_rbs_explicit_thresholds_bit_exact(cuda_dev, T, Hq, Hkv, P, pc, pr):
    wl = W.clustered_prefill(50 + T, T=T, Hq=Hq, Hkv=Hkv, d=128, block=64, n_clusters=16)
    if P != 64:   # re-page the same keys with a different page size
        wl = W.PrefillWorkload(_repage(wl.cache, P), wl.q, wl.T, wl.block)
    scale = 1 / math.sqrt(128)
    Sc, Sr = _oracle_scores(wl, scale)
    tc = [tau_in_gap(Sc[h], pc)[0] for h in range(Hq)]
    tr = [tau_in_gap(Sr[h], pr)[0] for h in range(Hq)]
    want = oracle.rbs_mask(Sc, Sr, tc, tr, True, True)
    ws = sa.Workspace(cuda_dev)
    csr = sa.select_blocks_rbs(wl.cache.to(cuda_dev), wl.q.to(cuda_dev), 64, scale,
                               tau_c=torch.tensor(tc), tau_r=torch.tensor(tr), ws=ws)
    ws.raise_on_fault()
    np.testing.assert_array_equal(_gpu_mask(cuda_dev, wl, csr), want)
    np.testing.assert_array_equal(csr.tau.cpu().numpy(), np.array([tc, tr], dtype=np.float32))


def _repage(cache, P):
    """Same logical keys/values laid out with page size P (identity order)."""
    Hkv, P0, d = cache.k.shape[1:]
    L = int(cache.seq_lens[0])
    pt = cache.page_table[0].long()
    t = torch.arange(cache.max_pages * P0)
    k = cache.k[pt[t // P0], :, t % P0]          # [Lpad][Hkv][d]
    v = cache.v[pt[t // P0], :, t % P0]
    k_log = k.permute(1, 0, 2)[None]
    v_log = v.permute(1, 0, 2)[None]
    return W.make_cache(k_log.contiguous(), v_log.contiguous(), [L], P, seed=9, shuffle=True, extra_pages=1)


def test_rbs_quantile_tiny_bit_exact(cuda_dev):
    """Quantile thresholds on tiny inputs whose sorted scores are all >= 1e-3 apart."""
    scale = 1 / math.sqrt(128)
    for seed in range(60, 200):
        wl = W.clustered_prefill(seed, T=8 * 64 - 13, Hq=4, Hkv=2, d=128, block=64, n_clusters=8)
        Sc, Sr = _oracle_scores(wl, scale)
        if all(np.diff(np.sort(x)).min() >= 1e-3 for x in list(Sc) + list(Sr)):
            break
    else:
        pytest.skip("no well-separated seed")
    pc, pr = np.float32(0.6), np.float32(0.85)
    tc = [oracle.quantile(Sc[h], float(pc)) for h in range(4)]
    tr = [oracle.quantile(Sr[h], float(pr)) for h in range(4)]
    want = oracle.rbs_mask(Sc, Sr, tc, tr, True, True)
    ws = sa.Workspace(cuda_dev)
    csr = sa.select_blocks_rbs(wl.cache.to(cuda_dev), wl.q.to(cuda_dev), 64, scale, p_c=float(pc),
                               p_r=float(pr), ws=ws)
    ws.raise_on_fault()
    np.testing.assert_array_equal(_gpu_mask(cuda_dev, wl, csr), want)
    # the quantile thresholds are GPU scores: within the error bound of the
    # split-bf16 tensor-core product, 3 * 2^-18 * scale * sum_k |qbar_k c_k|
    # (taken as 4 * 2^-18 to cover the fp32 accumulation), of the oracle's
    bound = _score_error_bound(wl, scale)
    err = np.abs(csr.tau.cpu().numpy().astype(np.float64) - np.array([tc, tr]))
    assert np.all(err <= bound[None, :]), (err, bound)


def test_rbs_block_sparse_config_full_size(cuda_dev):
    """32768 tokens, 32/4 heads, d=128, 64x64 blocks, clustered keys with 0.5%
    outliers; thresholds at quantiles 0.95 / 0.97 moved into >= 1e-3 gaps."""
    wl = W.clustered_prefill(1004)
    scale = 1 / math.sqrt(128)
    Sc, Sr = _oracle_scores(wl, scale)
    Hq = 32
    tc = [tau_in_gap(Sc[h], 0.95)[0] for h in range(Hq)]
    tr = [tau_in_gap(Sr[h], 0.97)[0] for h in range(Hq)]
    want = oracle.rbs_mask(Sc, Sr, tc, tr, True, True)
    gc = wl.cache.to(cuda_dev)
    q = wl.q.to(cuda_dev)
    ws = sa.Workspace(cuda_dev)
    csr = sa.select_blocks_rbs(gc, q, 64, scale, tau_c=torch.tensor(tc), tau_r=torch.tensor(tr), ws=ws)
    ws.raise_on_fault()
    got = _gpu_mask(cuda_dev, wl, csr)
    np.testing.assert_array_equal(got, want)
    density = want.mean()
    assert 0.04 < density < 0.12, density
    # quantile mode at scale: centroid branch alone keeps exactly n-1-floor(p(n-1))
    pc = np.float32(0.95)
    csr_q = sa.select_blocks_rbs(gc, q, 64, scale, p_c=float(pc), p_r=1.0, force_diag=False,
                                 force_first=False, ws=ws)
    ws.raise_on_fault()
    nB = 512
    nP = nB * (nB + 1) // 2
    rp = csr_q.row_ptr.cpu().numpy().reshape(-1)
    kept = np.array([rp[(h + 1) * nB] - rp[h * nB] for h in range(Hq)])
    assert np.all(kept == nP - 1 - math.floor(float(pc) * (nP - 1)))
    got_q = _gpu_mask(cuda_dev, wl, csr_q)
    want_q = oracle.rbs_mask(Sc, Sr, [oracle.quantile(Sc[h], float(pc)) for h in range(Hq)], [np.inf] * Hq,
                             False, False)
    assert (got_q != want_q).sum() <= 1e-4 * got_q.size


def test_rbs_capacity_overflow_recorded(cuda_dev):
    wl = W.random_prefill(3, 640, 4, 2, 128, 64)
    ws = sa.Workspace(cuda_dev)
    csr = sa.select_blocks_rbs(wl.cache.to(cuda_dev), wl.q.to(cuda_dev), 64, 0.1, tau_c=-1e9, tau_r=-1e9,
                               nnz_capacity=50, ws=ws)
    st, det = ws.status()
    assert st == 7
    assert int(csr.row_ptr[-1]) == 4 * 55
