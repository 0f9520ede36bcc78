"""Host DA state machine (CPU): scripted tag streams -> span lists per step.

Expected spans are written out by hand from the readings stated in the
module's docstring (mode change on the step after the completing token, focus
chunks [origin + c*chunk, origin + (c+1)*chunk) rounded out, local = last 512
tokens, global = [0, L); fallbacks as parameters)."""
import pytest
import torch

from sparse_attention_aware_b200 import da_state as DA
from sparse_attention_aware_b200 import spans as SP

V = DA.DAVocab()
G, LOC, FO, FC = V.global_tag, V.local_tag, V.focus_open, V.focus_close


def C(c):
    return V.chunk_base + c


def run(machine, tokens, start_len, confidences=None):
    out = []
    for i, t in enumerate(tokens):
        machine.observe(t)
        conf = 1.0 if confidences is None else confidences[i]
        out.append(machine.next_spans(start_len + i + 1, conf))
    return out


def test_declarations_take_effect_on_the_next_step():
    m = DA.DAStateMachine(10000)
    got = run(m, [5, FO, C(1), C(3), FC, 7, LOC, 9, G, 11], 10000)
    want = [
        [(0, 10001, True)],                      # before any declaration: global
        [(0, 10002, True)],                      # focus declaration open: previous mode
        [(0, 10003, True)],
        [(0, 10004, True)],
        [(2048, 4096, True), (6144, 8192, True)],  # closed: chunks 1 and 3
        [(2048, 4096, True), (6144, 8192, True)],  # text keeps the mode
        [(10007 - 512, 10007, True)],            # local
        [(10008 - 512, 10008, True)],
        [(0, 10009, True)],                      # global
        [(0, 10010, True)],
    ]
    assert got == want


def test_invalid_or_empty_focus_reads_globally_and_duplicates_merge():
    m = DA.DAStateMachine(10000)
    got = run(m, [LOC, FO, C(99), FC], 10000)        # chunk 99 starts past the prompt
    assert got[0] == [(10001 - 512, 10001, True)]
    assert got[3] == [(0, 10004, True)]
    got = run(m, [FO, FC], 20000)                     # no chunk at all
    assert got[1] == [(0, 20002, True)]
    got = run(m, [FO, C(2), C(2), C(0), FC], 20000)   # declaration order, each once
    assert got[-1] == [(4096, 6144, True), (0, 2048, True)]


def test_open_focus_interrupted_by_another_tag():
    m = DA.DAStateMachine(9000)
    got = run(m, [FO, C(1), LOC, 3, C(2), FC], 9000)
    assert got[2] == [(9003 - 512, 9003, True)]       # LOCAL closes the open declaration
    assert got[4] == [(9005 - 512, 9005, True)]       # a stray chunk token is text
    assert got[5] == [(9006 - 512, 9006, True)]       # a stray close tag is text


def test_chunk_grid_origin():
    m = DA.DAStateMachine(5000, origin=-500)
    got = run(m, [FO, C(0), C(1), C(3), FC], 5000)
    # chunk c covers [c*2048 - 500, (c+1)*2048 - 500); chunk 3 starts at 5644 > prompt
    assert got[-1] == [(-500, 1548, True), (1548, 3596, True)]


def test_periodic_and_forced_global():
    m = DA.DAStateMachine(8000, fallbacks=DA.DAFallbacks(periodic_global=3))
    got = run(m, [LOC, 1, 2, 3, 4, 5, 6], 8000)
    glob = [i for i, s in enumerate(got) if s == [(0, 8001 + i, True)]]
    assert glob == [2, 5]                             # steps 3 and 6
    m = DA.DAStateMachine(8000, fallbacks=DA.DAFallbacks(force_global=True))
    got = run(m, [LOC, FO, C(1), FC], 8000)
    assert all(s == [(0, 8001 + i, True)] for i, s in enumerate(got))


def test_focus_margin_is_a_minimum_neighbourhood():
    m = DA.DAStateMachine(10000, fallbacks=DA.DAFallbacks(focus_margin=100))
    got = run(m, [FO, C(1), FC], 10000)
    assert got[-1] == [(1948, 4196, True)]


def test_low_confidence_reads_globally_or_widens():
    m = DA.DAStateMachine(10000, fallbacks=DA.DAFallbacks(low_conf_threshold=0.5))
    got = run(m, [FO, C(2), FC, 1], 10000, confidences=[1, 1, 0.9, 0.2])
    assert got[2] == [(4096, 6144, True)]
    assert got[3] == [(0, 10004, True)]
    m = DA.DAStateMachine(10000, fallbacks=DA.DAFallbacks(low_conf_threshold=0.5, low_conf_action="widen"))
    got = run(m, [FO, C(2), FC, 1, LOC, 1], 10000, confidences=[1, 1, 1, 0.1, 1, 0.1])
    assert got[3] == [(2048, 4096, True), (4096, 6144, True), (6144, 8192, True)]   # chunks 1, 2, 3
    assert got[5] == [(10006 - 2048, 10006, True)]                                  # local window x4
    m = DA.DAStateMachine(10000, fallbacks=DA.DAFallbacks(low_conf_threshold=0.5, low_conf_action="widen"))
    got = run(m, [FO, C(0), C(4), FC], 10000, confidences=[1, 1, 1, 0.0])
    # chunk 0 has no left neighbour, chunk 5 starts past the prompt
    assert got[3] == [(0, 2048, True), (2048, 4096, True), (6144, 8192, True), (8192, 10240, True)]


def test_spans_agree_with_the_mode_builder():
    m = DA.DAStateMachine(70000)
    got = run(m, [FO, C(3), C(7), FC, LOC, G], 70000)
    assert got[3] == SP.spans_for(SP.FOCUS, 70004, 2048, 0, [3, 7])
    assert got[4] == SP.spans_for(SP.LOCAL, 70005)
    assert got[5] == SP.spans_for(SP.GLOBAL, 70006)


def test_batch_packs_one_list_per_sequence():
    b = DA.DABatch([5000, 9000, 300])
    spans, cnt, rnd = b.step([FO, LOC, 7], [5001, 9001, 301], device="cpu", max_spans=2)
    assert cnt.tolist() == [1, 1, 1] and spans.shape == (3, 2, 2)
    assert spans[1, 0].tolist() == [9001 - 512, 9001]
    b.step([C(1), 1, 1], [5002, 9002, 302], device="cpu")
    spans, cnt, rnd = b.step([FC, G, 1], [5003, 9003, 303], device="cpu")
    assert spans[0, 0].tolist() == [2048, 4096] and spans[1, 0].tolist() == [0, 9003]
    assert rnd.dtype == torch.uint8 and int(rnd[0, 0]) == 1
    with pytest.raises(ValueError):
        b.step([1, 2], [1, 2, 3], device="cpu")
