"""The library inside a CUDA graph (GPU): a captured sequence of calls --
masked-decode steps (span selection + block-list decode + combine) and a
Kascade group (top-k + decode layers) -- replays to the same bits as the
same calls run eagerly, and the replay reads fresh inputs written into the
captured buffers (the programmatic-launch edges become graph edges)."""
import math

import pytest
import torch

import sparse_attention_aware_b200 as sa
from sparse_attention_aware_b200 import spans as SP
from sparse_attention_aware_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _masked_setup(dev, steps):
    L, P = 8192, 16
    msk = W.masked_decode(1003, device=dev, B=2, Hq=16, Hkv=2, d=128, L=L, P=P, chunk=1024, steps=steps)
    packs = []
    for s in range(steps):
        lists = [SP.spans_for(SP.MODE_IDS[int(msk.modes[s, b])], L, msk.chunk, msk.origin,
                              msk.focus_chunks[s, b].tolist()) for b in range(2)]
        packs.append(SP.pack(lists, dev, max_spans=2))
    return msk, packs


def test_masked_steps_replay_bitwise(cuda_dev):
    steps = 6
    msk, packs = _masked_setup(cuda_dev, steps)
    ws = sa.Workspace(cuda_dev)
    blk = sa.BlockSelection(torch.empty((2, 8192 // 16 + 8, 4), dtype=torch.int32, device=cuda_dev),
                            torch.empty((2,), dtype=torch.int32, device=cuda_dev))
    outs = [torch.empty((2, 16, 128), dtype=torch.bfloat16, device=cuda_dev) for _ in range(steps)]
    lses = [torch.empty((2, 16), dtype=torch.float32, device=cuda_dev) for _ in range(steps)]
    q = msk.q_steps.clone()

    def run():
        for s in range(steps):
            spans, cnt, rnd = packs[s]
            b = sa.select_blocks_spans(msk.cache, spans, cnt, rnd, out=blk, ws=ws)
            sa.sparse_decode_attn(msk.cache, q[s], b, 1 / math.sqrt(128), 8, out=outs[s], lse=lses[s], ws=ws)

    stream = torch.cuda.Stream(cuda_dev)
    stream.wait_stream(torch.cuda.current_stream(cuda_dev))
    with torch.cuda.stream(stream):
        run()                                   # eager; sizes every buffer
    torch.cuda.synchronize(cuda_dev)
    eager = [(o.clone(), l.clone()) for o, l in zip(outs, lses)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    for o in outs:
        o.zero_()
    g.replay()
    torch.cuda.synchronize(cuda_dev)
    ws.raise_on_fault("graph replay")
    for (eo, el), o, l in zip(eager, outs, lses):
        assert torch.equal(o, eo) and torch.equal(l, el)
    # new queries written into the captured buffer are what the replay reads
    q.copy_(torch.roll(msk.q_steps, 1, dims=0))
    g.replay()
    torch.cuda.synchronize(cuda_dev)
    replayed = [(o.clone(), l.clone()) for o, l in zip(outs, lses)]
    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize(cuda_dev)
    assert not torch.equal(replayed[0][0], eager[0][0])
    for (ro, rl), o, l in zip(replayed, outs, lses):
        assert torch.equal(ro, o) and torch.equal(rl, l)
    del g


def test_kascade_group_replays_bitwise(cuda_dev):
    dec = W.gqa_decode(1005, device=cuda_dev, B=4, Hq=16, Hkv=4, d=128, L=8192, P=16, k=512, layers=3,
                       num_splits=4)
    caches = [dec.cache.with_v(v) for v in dec.v_layers]
    ws = sa.Workspace(cuda_dev)
    idx = torch.empty((4, 16, 512), dtype=torch.int32, device=cuda_dev)
    cnt = torch.empty((4, 16), dtype=torch.int32, device=cuda_dev)
    outs = [torch.empty((4, 16, 128), dtype=torch.bfloat16, device=cuda_dev) for _ in range(3)]
    lses = [torch.empty((4, 16), dtype=torch.float32, device=cuda_dev) for _ in range(3)]

    def run():
        sel = sa.select_topk(caches[0], dec.q_layers[0], 512, idx=idx, count=cnt, ws=ws)
        for li in range(3):
            sa.sparse_decode_attn(caches[li], dec.q_layers[li], sel, 1 / math.sqrt(128), 4, out=outs[li],
                                  lse=lses[li], ws=ws)

    stream = torch.cuda.Stream(cuda_dev)
    stream.wait_stream(torch.cuda.current_stream(cuda_dev))
    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize(cuda_dev)
    eager = (idx.clone(), [o.clone() for o in outs], [l.clone() for l in lses])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    idx.fill_(-7)
    for o in outs:
        o.zero_()
    g.replay()
    torch.cuda.synchronize(cuda_dev)
    ws.raise_on_fault("graph replay")
    assert torch.equal(idx, eager[0])
    for o, l, eo, el in zip(outs, lses, eager[1], eager[2]):
        assert torch.equal(o, eo) and torch.equal(l, el)
    del g
