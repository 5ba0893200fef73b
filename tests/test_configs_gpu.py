"""Parity at the full sizes of the five benchmark workloads, in the launch configuration
bench.py times (same entry points, same shapes, same input recipe).

The oracle cannot afford every output at these sizes, so each workload checks
sampled outputs it can compute one by one: whole heads for the small workloads,
and for the large ones a fixed set of rows (tile edges, the ragged end, random
rows) of the first, a middle and the last head.  dQ rows come from
``grad_q_rows``; dK/dV rows of sampled keys from ``grad_kv_rows`` (one full
forward per q-head of the group).
"""
import numpy as np
import pytest
import torch

from attn_inputs import WORKLOADS, to_f64, workload_inputs
from oracle import reference as ref
from tests.parity import check_grad, check_lse, check_o, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


def sample_rows(N, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 2, 127, 128, 129, N // 2, N - 129, N - 128, N - 2, N - 1]
    rnd = rng.choice(N, size=min(N, 21), replace=False).tolist()
    return np.array(sorted({r for r in fixed + rnd if 0 <= r < N}))


def heads_to_check(w):
    return sorted({(0, 0), (w.B // 2, w.Hq // 2), (w.B - 1, w.Hq - 1)})


def run(attn, w):
    x = workload_inputs(w, device="cpu")
    dev = {k: v.cuda() for k, v in x.items()}
    o, lse = attn.attn_fwd(dev["q"], dev["k"], dev["v"], scale=w.scale, causal=w.causal)
    grads = None
    if "bwd" in w.passes:
        grads = attn.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    return x, o, lse, grads


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_forward(attn, name):
    w = WORKLOADS[name]
    x, o, lse, _ = run(attn, w)
    G = w.Hq // w.Hkv
    for b, h in heads_to_check(w):
        qh = to_f64(x["q"][b, h])
        kh, vh = to_f64(x["k"][b, h // G]), to_f64(x["v"][b, h // G])
        rows = np.arange(w.N) if w.N <= 1024 else sample_rows(w.N, 100 * b + h)
        o_ref, lse_ref = ref.attend_head(qh, kh, vh, w.scale, w.causal, rows=rows)
        check_o(f64(o[b, h])[rows], o_ref, what=f"{name} O[b={b},h={h}]")
        check_lse(f64(lse[b, h])[rows], lse_ref, what=f"{name} LSE[b={b},h={h}]")


@pytest.mark.parametrize("name", [n for n, w in WORKLOADS.items() if "bwd" in w.passes])
def test_workload_backward(attn, name):
    w = WORKLOADS[name]
    x, o, lse, (dq, dk, dv) = run(attn, w)
    G = w.Hq // w.Hkv
    for b, h in heads_to_check(w)[:2]:
        g = h // G
        qh, doh = to_f64(x["q"][b, h]), to_f64(x["do"][b, h])
        kh, vh = to_f64(x["k"][b, g]), to_f64(x["v"][b, g])
        rows = np.arange(w.N) if w.N <= 1024 else sample_rows(w.N, 7 + b + h)
        dq_ref = ref.grad_q_rows(qh, kh, vh, doh, w.scale, w.causal, rows)
        check_grad(f64(dq[b, h])[rows], dq_ref, f"{name} dQ[b={b},h={h}]")
        keys = rows
        hs = range(g * G, (g + 1) * G)
        dk_ref, dv_ref = ref.grad_kv_rows([to_f64(x["q"][b, hh]) for hh in hs], kh, vh,
                                          [to_f64(x["do"][b, hh]) for hh in hs], w.scale, w.causal, keys)
        check_grad(f64(dk[b, g])[keys], dk_ref, f"{name} dK[b={b},g={g}]")
        check_grad(f64(dv[b, g])[keys], dv_ref, f"{name} dV[b={b},g={g}]")
