"""Test-side helpers: dense gathers written independently of both sides."""
import numpy as np
import torch


def dense_kv(cache, b: int, g: int, L: int, v=None):
    """fp64 K, V rows [L][d] of sequence b, kv head g (logical order)."""
    P = cache.k.shape[2]
    t = torch.arange(L)
    pages = cache.page_table[b].cpu().long()[t // P]
    slots = t % P
    K = cache.k.cpu()[pages, g, slots].double()
    V = (cache.v if v is None else v).cpu()[pages, g, slots].double()
    return K, V


def sdpa64(q, K, V, scale, mask=None):
    """torch scaled_dot_product_attention in fp64 (library reference).
    q [n][d], K/V [L][d], mask bool [n][L] (True = attend)."""
    out = torch.nn.functional.scaled_dot_product_attention(
        q[None, None], K[None, None], V[None, None], attn_mask=None if mask is None else mask[None, None],
        scale=scale)
    return out[0, 0]


def lse64(q, K, scale, mask=None):
    s = scale * (q @ K.T)
    if mask is not None:
        s = s.masked_fill(~mask, float("-inf"))
    return torch.logsumexp(s, dim=-1)


# ---------------------------------------------------------------------------
# top-k score-gap enforcement (the k-th / (k+1)-th fp64 scores must differ by
# >= 1e-3 and by more than twice the fp32 dot-product error bound, so the
# GPU's fp32 ranking provably matches the oracle's set)
# ---------------------------------------------------------------------------
U32 = 2.0 ** -24


def _boundary(r, k):
    """(k-th, (k+1)-th) largest positions of r, ties to the lower position."""
    cand = np.argpartition(-r, k)[: k + 1]
    order = cand[np.lexsort((cand, -r[cand]))]
    return order[k - 1], order[k]


def head_gap_ok(Kn, Ka, qh, k, min_gap=1e-3):
    """Kn/Ka: fp64 keys and |keys| [L][d]; qh fp64 [d]."""
    d = qh.shape[0]
    gam = (d + 1) * U32 / (1 - (d + 1) * U32)
    r = Kn @ qh
    if len(r) <= k:
        return True
    a, c = _boundary(r, k)
    gap = r[a] - r[c]
    err = gam * (Ka[a] @ np.abs(qh) + Ka[c] @ np.abs(qh))
    return gap >= min_gap and gap > 2 * err


def enforce_gap(cache, q, k, seed, max_tries=1000, min_gap=1e-3):
    """Redraw (b, h) query rows until the top-k boundary gap holds: the k-th
    and (k+1)-th fp64 scores differ by >= min_gap and by more than twice the
    fp32 dot-product error bound gamma_{d+1} (|q|.|k_kth| + |q|.|k_next|).
    Returns (new q on q's device, number of redraws)."""
    from sparse_attention_aware_b200 import workloads as W
    dev, dt = q.device, q.dtype
    q = q.detach().cpu().clone()
    B, Hq, d = q.shape
    Hkv = cache.k.shape[1]
    grp = Hq // Hkv
    redraws = 0
    for b in range(B):
        L = int(cache.seq_lens[b])
        if L <= k:
            continue
        for g in range(Hkv):
            K, _ = dense_kv(cache, b, g, L)
            Kn, Ka = K.numpy(), K.abs().numpy()
            for h in range(g * grp, (g + 1) * grp):
                for attempt in range(max_tries):
                    if head_gap_ok(Kn, Ka, q[b, h].double().numpy(), k, min_gap):
                        break
                    q[b, h] = W.randn((d,), seed, W.S_REDRAW, (b << 40) | (h << 20) | (attempt + 1), "cpu",
                                      torch.float32).to(dt)
                    redraws += 1
                else:
                    raise RuntimeError("could not enforce the top-k gap")
    return q.to(dev), redraws


def assert_close_attn(out_gpu, out_ref, max_abs=2e-2, mean_abs=1e-2):
    """The stated tolerance for bf16-in / fp32-accumulate attention outputs."""
    g = np.asarray(out_gpu, dtype=np.float64)
    r = np.asarray(out_ref, dtype=np.float64)
    assert g.shape == r.shape
    err = np.abs(g - r)
    assert np.all(np.isfinite(g))
    assert err.max() <= max_abs, "max-abs %.3g > %.3g" % (err.max(), max_abs)
    assert err.mean() <= mean_abs, "mean-abs %.3g > %.3g" % (err.mean(), mean_abs)
    return float(err.max()), float(err.mean())


# ---------------------------------------------------------------------------
# RBS helpers
# ---------------------------------------------------------------------------
def tau_in_gap(scores, p, min_gap=1e-3):
    """An fp32 threshold inside the gap (>= min_gap) between consecutive sorted
    fp64 scores that lies nearest to the lower-quantile rank floor(p*(n-1));
    returns (tau as float32-representable float, kept count)."""
    s = np.sort(np.asarray(scores, dtype=np.float64).ravel())
    n = len(s)
    r = int(np.floor(p * (n - 1)))
    gaps = np.diff(s)
    ok = np.nonzero(gaps >= min_gap)[0]
    if len(ok) == 0:
        raise RuntimeError("no gap")
    m = ok[np.argmin(np.abs(ok - r))]
    tau = float(np.float32((s[m] + s[m + 1]) / 2))
    assert s[m] < tau < s[m + 1]
    return tau, int(n - 1 - m)


def csr_to_mask(row_ptr, cols, Hq, nB):
    """CSR rows (h*nB + i) -> u8 [Hq][nB(nB+1)/2] over causal pairs."""
    row_ptr = np.asarray(row_ptr)
    cols = np.asarray(cols)
    nP = nB * (nB + 1) // 2
    m = np.zeros((Hq, nP), dtype=np.uint8)
    for h in range(Hq):
        for i in range(nB):
            r = h * nB + i
            c = cols[row_ptr[r]:row_ptr[r + 1]]
            assert np.all(np.diff(c) > 0) and (len(c) == 0 or (c[0] >= 0 and c[-1] <= i))
            m[h, i * (i + 1) // 2 + c] = 1
    return m
