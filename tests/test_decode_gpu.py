"""Split-KV decoding on the CUDA path vs the fp64 oracle.

Nq query rows against Nk keys (page "attention 的显存线性化", reading list:
FlashDecoding), with the partials of the key splits merged by their log-sum-exp
(page "attn-efficient", online-softmax section).  Cases cover Nq in {1, 16, 128},
Nk in {1, 1000, 32768}, group sizes 1 to 128 (including a group size that does not
divide 128), both head sizes, causal (queries at the last Nq positions) and not,
one split (written directly) and many (merged), and causal query blocks whose
later splits see no key at all.
"""
import numpy as np
import pytest
import torch

from attn_inputs import make_inputs, to_f64
from oracle import reference as ref
from tests.parity import check_lse, check_o, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


def decode_inputs(B, Hq, Hkv, Nq, Nk, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Nq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Nk, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Nk, d, generator=g).to(torch.bfloat16)
    return q, k, v


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 1, 1, 1, 1, 128, False),
    (2, 4, 1, 1, 1000, 128, True),
    (1, 8, 8, 16, 1000, 64, True),
    (2, 32, 8, 1, 32768, 128, True),
    (1, 4, 4, 128, 1000, 128, False),
    (1, 8, 2, 128, 32768, 128, True),
    (1, 2, 2, 16, 1, 64, False),
    (3, 6, 2, 7, 300, 128, True),
    (1, 128, 1, 1, 5000, 64, True),
    (1, 2, 2, 1000, 1000, 128, True),
    (2, 16, 16, 3, 777, 64, False),
]


def _ids(c):
    return f"B{c[0]}-Hq{c[1]}-Hkv{c[2]}-Nq{c[3]}-Nk{c[4]}-d{c[5]}-{'causal' if c[6] else 'full'}"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_decode_matches_oracle(attn, case):
    B, Hq, Hkv, Nq, Nk, d, causal = case
    q, k, v = decode_inputs(B, Hq, Hkv, Nq, Nk, d, seed=Nq * 31 + Nk + d)
    o, lse = attn.attn_decode(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    o_ref, lse_ref = ref.ref_decode(to_f64(q), to_f64(k), to_f64(v), d ** -0.5, causal)
    tag = f"decode {_ids(case)} splits={attn.attn_decode_splits(B, Hq, Hkv, Nq, Nk, d, causal)}"
    check_o(f64(o), o_ref, f"{tag} O")
    check_lse(f64(lse), lse_ref, f"{tag} LSE")


def test_decode_uses_several_splits_and_a_caller_workspace(attn):
    B, Hq, Hkv, Nq, Nk, d = 1, 8, 2, 4, 32768, 128
    S = attn.attn_decode_splits(B, Hq, Hkv, Nq, Nk, d, True)
    size = attn.attn_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, True)
    assert S > 1 and size >= B * Hq * Nq * S * (d + 1) * 4
    q, k, v = decode_inputs(B, Hq, Hkv, Nq, Nk, d, seed=9)
    ws = torch.full((size,), 255, dtype=torch.uint8, device="cuda")     # stale contents must not matter
    o1, l1 = attn.attn_decode(q.cuda(), k.cuda(), v.cuda(), causal=True, workspace=ws)
    o2, l2 = attn.attn_decode(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o_ref, lse_ref = ref.ref_decode(to_f64(q), to_f64(k), to_f64(v), d ** -0.5, True)
    check_o(f64(o1), o_ref, "decode caller workspace O")
    check_lse(f64(l1), lse_ref, "decode caller workspace LSE")


def test_decode_of_the_last_rows_matches_the_causal_forward(attn):
    """Nq = Nk causal decoding is square causal attention; both paths agree with the oracle
    and with each other within two bf16 roundings."""
    B, H, N, d = 1, 4, 640, 128
    x = make_inputs(B, H, H, N, d, seed=21, with_grad=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = attn.attn_decode(q, k, v, causal=True)
    o2, l2 = attn.attn_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert np.abs(f64(l1) - f64(l2)).max() < 1e-3
    assert np.abs(f64(o1) - f64(o2)).max() < 2e-2


def test_decode_is_bitwise_deterministic(attn):
    """The split plan and the merge order are fixed, so repeated calls give the same bits."""
    q, k, v = decode_inputs(2, 16, 4, 3, 20000, 128, seed=33)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = attn.attn_decode(q, k, v, causal=True)
    o2, l2 = attn.attn_decode(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert attn.attn_decode_splits(2, 16, 4, 3, 20000, 128, True) > 1
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
