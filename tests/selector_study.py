"""Selector study at matched density on clustered keys with outliers -- TEST
INFRASTRUCTURE (runs on the CPU oracle).

Question ("RBS-Attention: Radius-Bounded Sparse Prefill…", sections
"关键技术点" items 1-2 and "我的技术点评"): at the same fraction of kept
(query block, key block) pairs, how much of the true causal attention mass do
the centroid branch alone, the radius-rescue branch alone, and their OR keep?
The generator's 0.5% outlier keys (6x a draw from another cluster) are the
mean-dilution case: one outlier barely moves its block's centroid but can
dominate the attention of queries from its cluster.

Per block size bs (16, 32, 64), per head h, with scale 1/sqrt(d):
* true mass  M[t][j] = sum over keys t' <= t in block j of softmax_t'(scale q_t.k_t')
  (dense fp64, causal);
* selection  the oracle's block statistics, pooled queries and pair scores
  (S_c = scale qbar.c, S_r = scale (qbar.c + |qbar| r)), thresholds at the
  lower quantile levels of each branch, diagonal and first block forced;
  matched density: the quantile level of the variant is bisected until the
  kept fraction of causal pairs is within 0.25% of the target (OR: p_r =
  p_c + delta, bisection on p_c);
* retention  for query row t in block i: sum of M[t][j] over the kept j of
  row (h, i); reported as the mean over rows and heads, and the share of rows
  that keep less than half of their mass;
* upper bound  per head, the kept count of pairs chosen by the true mean mass
  of the pair (its rows' mass summed), forced pairs included.

Run ``python -m tests.selector_study`` for the full table (T=4096, 4 heads).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import dense_kv


def true_block_mass(q, K, scale, bs):
    """M [Hq][T][nB] fp64: causal softmax mass of each key block per query row."""
    T, Hq, d = q.shape
    nB = (T + bs - 1) // bs
    Kd = K.numpy()
    causal = np.tril(np.ones((T, T), dtype=bool))
    out = np.empty((Hq, T, nB))
    for h in range(Hq):
        s = (q[:, h].double().numpy() @ Kd.T) * scale
        s = np.where(causal, s, -np.inf)
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        pad = nB * bs - T
        if pad:
            p = np.concatenate([p, np.zeros((T, pad))], axis=1)
        out[h] = p.reshape(T, nB, bs).sum(axis=2)
    return out


def pair_index(nB):
    """(i, j) of every causal pair in the oracle's order i(i+1)/2 + j."""
    ii, jj = [], []
    for i in range(nB):
        ii.extend([i] * (i + 1))
        jj.extend(range(i + 1))
    return np.array(ii), np.array(jj)


def retention(mask, M, bs, T):
    """mean retained mass over rows, share of rows below 0.5."""
    Hq, nP = mask.shape
    nB = M.shape[2]
    ii, jj = pair_index(nB)
    kept = np.zeros((Hq, nB, nB), dtype=bool)
    for h in range(Hq):
        kept[h, ii[mask[h] != 0], jj[mask[h] != 0]] = True
    rows_blk = np.arange(T) // bs
    r = np.stack([(M[h] * kept[h, rows_blk]).sum(axis=1) for h in range(Hq)])
    return float(r.mean()), float((r < 0.5).mean())


def density(mask):
    return float(mask.mean())


def match(make_mask, target, lo=0.0, hi=1.0, iters=40):
    """Bisection on a quantile level until the kept fraction is within 0.25%."""
    best = None
    for _ in range(iters):
        p = 0.5 * (lo + hi)
        m = make_mask(p)
        dens = density(m)
        best = (p, m, dens)
        if abs(dens - target) <= 0.0025:
            break
        if dens > target:
            lo = p
        else:
            hi = p
    return best


def upper_bound_mask(M, bs, kept_counts, forced):
    """Per head, forced pairs plus the remaining count by summed true mass."""
    Hq, T, nB = M.shape
    ii, jj = pair_index(nB)
    rows_blk = np.arange(T) // bs
    out = np.zeros((Hq, len(ii)), dtype=np.uint8)
    for h in range(Hq):
        pm = np.zeros((nB, nB))
        np.add.at(pm, rows_blk, M[h])            # [query block][key block] mass
        score = pm[ii, jj].copy()
        score[forced[h] != 0] = np.inf
        order = np.argsort(-score, kind="stable")
        out[h, order[:kept_counts[h]]] = 1
    return out


def run_study(T=4096, Hq=4, seed=2001, block_sizes=(16, 32, 64), densities=(0.05, 0.10, 0.20),
              deltas=(0.0, 0.02, 0.05), n_clusters=32):
    d = 128
    scale = 1 / math.sqrt(d)
    wl = W.clustered_prefill(seed, T=T, Hq=Hq, Hkv=1, d=d, block=64, n_clusters=n_clusters)
    K, _ = dense_kv(wl.cache, 0, 0, T)
    rows = []
    for bs in block_sizes:
        M = true_block_mass(wl.q, K, scale, bs)
        c, r = oracle.block_stats(wl.cache, bs)
        qbar, qn = oracle.pool_q(wl.q, bs)
        Sc, Sr = oracle.pair_scores(qbar, qn, c, r, scale)
        forced = oracle.rbs_mask(Sc, Sr, np.inf, np.inf)
        q_c = lambda p: [oracle.quantile(Sc[h], p) for h in range(Hq)]
        q_r = lambda p: [oracle.quantile(Sr[h], p) for h in range(Hq)]
        for target in densities:
            row = {"bs": bs, "density": target}
            p, m, dens = match(lambda p: oracle.rbs_mask(Sc, Sr, q_c(p), np.inf), target)
            row["centroid"] = retention(m, M, bs, T) + (dens,)
            p, m, dens = match(lambda p: oracle.rbs_mask(Sc, Sr, np.inf, q_r(p)), target)
            row["rescue"] = retention(m, M, bs, T) + (dens,)
            for delta in deltas:
                p, m, dens = match(lambda p: oracle.rbs_mask(Sc, Sr, q_c(p), q_r(min(p + delta, 1.0))), target)
                row["or_%.2f" % delta] = retention(m, M, bs, T) + (dens,)
            ub = upper_bound_mask(M, bs, m.sum(axis=1), forced)
            row["upper"] = retention(ub, M, bs, T) + (density(ub),)
            rows.append(row)
    return rows


def table(rows, deltas=(0.0, 0.02, 0.05)):
    cols = ["centroid", "rescue"] + ["or_%.2f" % d for d in deltas] + ["upper"]
    head = "| block | density | " + " | ".join(cols) + " |"
    sep = "|---|---|" + "---|" * len(cols)
    lines = [head, sep]
    for r in rows:
        cells = ["%.3f (%.2f)" % (r[c][0], r[c][1]) for c in cols]
        lines.append("| %d | %.0f%% | %s |" % (r["bs"], 100 * r["density"], " | ".join(cells)))
    return "\n".join(lines)


if __name__ == "__main__":
    torch.set_num_threads(max(1, oracle.threads()))
    res = run_study()
    print("mean retained attention mass (share of rows keeping < 0.5 of their mass)")
    print(table(res))
