"""Bounded device waits end by themselves (GPU): a wait that nothing
satisfies gives up after its limit, the kernel records SA_ERR_TIMEOUT in the
workspace status word, and the context stays usable for the next work."""
import math
import time

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import workloads as W
from tests.helpers import assert_close_attn

pytestmark = pytest.mark.gpu


def test_unsatisfied_wait_times_out_and_the_context_stays_usable(cuda_dev):
    ws = sa.Workspace(cuda_dev)
    assert ws.status()[0] == 0
    t0 = time.perf_counter()
    sa.check_bounded_wait(0.02, device=cuda_dev, ws=ws)
    st, det = ws.status()                       # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert st == 6 and det[1] == 11             # SA_ERR_TIMEOUT, check id CHK_WAIT
    assert 0.015 <= elapsed < 5.0               # the wait lasted about its limit and ended
    assert ws.status()[0] == 0                  # cleared after reading
    # the same context decodes correctly afterwards
    lens = [300, 1029]
    cache, q = W.random_decode(5, len(lens), 8, 2, 128, lens, 16)
    rng = np.random.default_rng(1)
    idx = np.full((2, 8, 64), -1, dtype=np.int32)
    cnt = np.full((2, 8), 64, dtype=np.int32)
    for b, L in enumerate(lens):
        for h in range(8):
            idx[b, h] = np.sort(rng.choice(L, 64, replace=False))
    scale = 1 / math.sqrt(128)
    ref, _ = oracle.decode_tokens(cache, q, idx, cnt, scale)
    sel = sa.TokenSelection(torch.from_numpy(idx).to(cuda_dev), torch.from_numpy(cnt).to(cuda_dev))
    out, _ = sa.sparse_decode_attn(cache.to(cuda_dev), q.to(cuda_dev), sel, scale, 2, ws=ws)
    ws.raise_on_fault()
    assert_close_attn(out.float().cpu().numpy().reshape(-1, 128), ref)


def test_bounded_wait_rejects_bad_limits(cuda_dev):
    with pytest.raises(sa.SAError):
        sa.check_bounded_wait(0.0, device=cuda_dev)
    with pytest.raises(sa.SAError):
        sa.check_bounded_wait(11.0, device=cuda_dev)
