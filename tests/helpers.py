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
