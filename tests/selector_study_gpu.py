"""Selector study on the library's own GPU selector, at the prefill workload's
shapes -- TEST INFRASTRUCTURE.

Question ("RBS-Attention: Radius-Bounded Sparse Prefill…", section
"关键技术点" items 1-2, and the mean-dilution argument of "我的技术点评"): at
the same fraction of kept (query block, key block) pairs, how much of the
true causal attention mass does each branch of the selector keep on its own,
and how much does their OR keep?

* workload: the clustered prefill generator (clusters of keys, 0.5% outlier
  keys at 6x norm from another cluster -- the mean-dilution case), 32 query
  heads on 4 kv heads, d = 128, 64-token blocks, T = 32768 and 131072;
* selection: ``select_blocks_rbs`` on the GPU in quantile mode; a branch is
  switched off with quantile level 1.0 (its threshold is then the largest
  score, and the comparison is strict, so it keeps nothing); centroid only =
  (p, 1), rescue only = (1, p), OR = (p, p + delta); p is bisected on the GPU
  until the kept fraction of causal pairs (forced diagonal and first block
  included) is within 0.25% of the target;
* scoring: for sampled query rows t of a few heads, the true causal softmax
  mass of every key block, in fp64 on the CPU from the cache's bf16 keys and
  the bf16 queries; the retention of a variant is the mass of the blocks its
  CSR row (h, t // 64) keeps, averaged over the sampled rows (with the share
  of rows keeping less than half);
* row upper bound: per sampled row, the same number of blocks as the OR
  variant keeps in that row, chosen by true mass (what any block selector
  with that row's budget could keep at best).

Run ``python -m tests.selector_study_gpu`` on a B200 for the table.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import workloads as W


def gpu_mask_density(csr) -> float:
    n = csr.num_q_heads * csr.num_q_blocks * (csr.num_q_blocks + 1) // 2
    return int(csr.row_ptr[-1]) / n


def select(wl, pc, pr, ws):
    d = wl.q.shape[-1]
    return sa.select_blocks_rbs(wl.cache, wl.q, 64, 1 / math.sqrt(d), p_c=pc, p_r=pr, ws=ws)


def match(wl, variant, target, ws, delta=0.0, iters=30):
    """Bisect the quantile level of ``variant`` (centroid / rescue / or) until
    the kept fraction is within 0.25% of ``target``; returns (p, csr, density)."""
    lo, hi = 0.0, 1.0
    best = None
    for _ in range(iters):
        p = 0.5 * (lo + hi)
        if variant == "centroid":
            pc, pr = p, 1.0
        elif variant == "rescue":
            pc, pr = 1.0, p
        else:
            pc, pr = p, min(p + delta, 1.0)
        csr = select(wl, pc, pr, ws)
        dens = gpu_mask_density(csr)
        best = (p, csr, dens)
        if abs(dens - target) <= 0.0025:
            break
        if dens > target:
            lo = p
        else:
            hi = p
    return best


def sample_rows(T, heads, n_rows, seed):
    """(head, token) pairs: uniform tokens past the first block, plus the last one."""
    rng = np.random.default_rng(seed)
    out = []
    for h in heads:
        ts = np.concatenate([rng.integers(64, T, n_rows - 1), [T - 1]])
        out.extend((int(h), int(t)) for t in ts)
    return out


def true_row_mass(wl, rows):
    """fp64 causal softmax mass per key block for each sampled (head, token):
    list of arrays [t // 64 + 1]."""
    T, Hq, d = wl.q.shape
    Hkv = wl.cache.k.shape[1]
    G = Hq // Hkv
    scale = 1 / math.sqrt(d)
    pt = wl.cache.page_table[0].cpu().long()
    kc = wl.cache.k.cpu()
    by_g = {}
    for h, t in rows:
        by_g.setdefault(h // G, []).append((h, t))
    out = {}
    for g, lst in by_g.items():
        tok = torch.arange(T)
        K = kc[pt[tok // 64], g, tok % 64].double().numpy()          # [T][d] keys of kv head g
        for h, t in lst:
            q = wl.q[t, h].double().cpu().numpy()
            s = (K[: t + 1] @ q) * scale
            p = np.exp(s - s.max())
            p /= p.sum()
            nb = t // 64 + 1
            pad = np.zeros(nb * 64)
            pad[: t + 1] = p
            out[(h, t)] = pad.reshape(nb, 64).sum(axis=1)
    return out


class HostCSR:
    """The CSR read back once: row (h, i) -> its key blocks."""

    def __init__(self, csr):
        self.nB = csr.num_q_blocks
        self.rp = csr.row_ptr.cpu().numpy()
        self.cols = csr.cols[: int(self.rp[-1])].cpu().numpy()

    def row(self, h, i):
        r = h * self.nB + i
        return self.cols[self.rp[r]:self.rp[r + 1]]


def retention(csr, mass):
    hc = HostCSR(csr)
    r = []
    for (h, t), m in mass.items():
        r.append(float(m[hc.row(h, t // 64)].sum()))
    r = np.array(r)
    return float(r.mean()), float((r < 0.5).mean())


def row_upper(csr_ref, mass):
    hc = HostCSR(csr_ref)
    r = []
    for (h, t), m in mass.items():
        n = len(hc.row(h, t // 64))
        r.append(float(np.sort(m)[::-1][:n].sum()))
    r = np.array(r)
    return float(r.mean()), float((r < 0.5).mean())


def run(T, densities=(0.05, 0.10), deltas=(0.0, 0.02), heads=(0, 9, 18, 27), n_rows=96, seed=1004, dev="cuda"):
    wl = W.clustered_prefill(seed, device=dev, T=T, Hq=32, Hkv=4, d=128, block=64)
    ws = sa.Workspace(dev)
    rows = sample_rows(T, heads, n_rows, seed)
    mass = true_row_mass(wl, rows)
    out = []
    for target in densities:
        row = {"T": T, "density": target}
        for variant in ["centroid", "rescue"] + ["or_%.2f" % x for x in deltas]:
            delta = float(variant[3:]) if variant.startswith("or") else 0.0
            p, csr, dens = match(wl, variant.split("_")[0], target, ws, delta)
            row[variant] = retention(csr, mass) + (dens, p)
            if variant == "or_%.2f" % deltas[-1]:
                row["row_upper"] = row_upper(csr, mass) + (dens, None)
        ws.raise_on_fault("selector study")
        out.append(row)
    return out


def table(rows, deltas=(0.0, 0.02)):
    keys = ["centroid", "rescue"] + ["or_%.2f" % x for x in deltas] + ["row_upper"]
    lines = ["| T | density | " + " | ".join(keys) + " |", "|" + "---|" * (2 + len(keys))]
    for r in rows:
        cells = ["%.3f (%.2f)" % (r[k][0], r[k][1]) for k in keys]
        lines.append("| %d | %d%% | %s |" % (r["T"], round(100 * r["density"]), " | ".join(cells)))
    return "\n".join(lines)


if __name__ == "__main__":
    allrows = []
    for T in (32768, 131072):
        allrows += run(T)
    print(table(allrows))
    for r in allrows:
        print({k: (tuple(round(x, 5) if isinstance(x, float) else x for x in v) if isinstance(v, tuple) else v)
               for k, v in r.items()})
