"""Host logic of the sequence-length sweep (no GPU): the shapes it times."""
import math

from attn_inputs import SWEEP_D, SWEEP_N, SWEEP_TOKENS, SWEEP_WIDTH, sweep_workloads


def test_sweep_covers_every_length_head_size_and_mask_once():
    ws = sweep_workloads()
    keys = {(w.N, w.d, w.causal) for w in ws}
    assert len(ws) == len(keys) == len(SWEEP_N) * len(SWEEP_D) * 2
    assert len({w.name for w in ws}) == len(ws)
    assert len({w.seed for w in ws}) == len(ws)


def test_sweep_holds_tokens_and_width_fixed():
    for w in sweep_workloads():
        assert w.Hq * w.d == SWEEP_WIDTH and w.Hkv == w.Hq
        # B*N is the token budget, except where one sequence is already longer
        assert w.B * w.N == max(SWEEP_TOKENS, w.N)
        assert "bwd" in w.passes and w.scale == 1.0 / math.sqrt(w.d)


def test_sweep_inputs_exceed_l2():
    # each timed call reads at least Q, K, V: more than the 126 MB L2, so no flush is needed
    for w in sweep_workloads():
        assert 3 * w.B * w.Hq * w.N * w.d * 2 > 126e6
