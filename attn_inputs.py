"""Seeded synthetic inputs for exact attention, shared by the oracle tests and the CUDA path.

This module holds no attention arithmetic: it only draws random tensors with the
shapes and value distributions of the workloads the attention pages discuss
(GPT-2-medium shape B=64, H=16, n=1024, d=64 from the cost table on the
"attn-efficient" page; long-context and grouped-query shapes), so that both sides
of every parity check see the same bf16 bits.

Conventions
-----------
* Layout is [B, H, N, d], contiguous, bf16 (each head is a dense N x d matrix).
* Q has Hq heads; K and V have Hkv heads; dO has Hq heads.
* Values are drawn as fp32 normals from a ``torch.Generator`` seeded with the given
  seed, scaled, then rounded to bf16 (round-to-nearest-even, torch's cast).
* ``boost_rows``: per (b, h_kv), exactly floor(frac * N) distinct K rows, chosen by a
  seeded permutation, are multiplied by ``boost`` (a power of two, so exact in bf16).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, mask, scale and input distribution."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    passes: str = "fwd+bwd"  # "fwd" or "fwd+bwd"
    qk_std: float = 1.0
    vo_std: float = 1.0
    boost_frac: float = 0.0
    boost: float = 1.0
    seed: int = 1000

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


# The five problems the measurements are quoted on, in order; seeds 1000+k.
WORKLOADS = {
    "single_head_n256_d64": Workload("single_head_n256_d64", 1, 1, 1, 256, 64, False, "fwd", seed=1000),
    "gpt2_medium_b64_h16_n1024_d64": Workload(
        "gpt2_medium_b64_h16_n1024_d64", 64, 16, 16, 1024, 64, False, "fwd+bwd", seed=1001),
    "causal_b8_h16_n4096_d128": Workload("causal_b8_h16_n4096_d128", 8, 16, 16, 4096, 128, True, "fwd", seed=1002),
    "long_causal_b1_h32_n32768_d128": Workload(
        "long_causal_b1_h32_n32768_d128", 1, 32, 32, 32768, 128, True, "fwd+bwd", seed=1003),
    "gqa_causal_b4_hq32_hkv8_n8192_d128": Workload(
        "gqa_causal_b4_hq32_hkv8_n8192_d128", 4, 32, 8, 8192, 128, True, "fwd+bwd",
        qk_std=3.0, boost_frac=0.01, boost=8.0, seed=1004),
}

# Decoding problems (split-KV path): Nq new query rows against an Nk-key cache.  Shapes
# of a grouped-query model at long context (32 query heads, 8 KV heads, d = 128);
# inputs N(0, 1).
@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int = 3000

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


DECODE_WORKLOADS = {
    "decode_b16_hq32_hkv8_nq1_nk32768_d128": DecodeWorkload(
        "decode_b16_hq32_hkv8_nq1_nk32768_d128", 16, 32, 8, 1, 32768, 128, True, seed=3000),
    "decode_b4_hq32_hkv8_nq16_nk131072_d128": DecodeWorkload(
        "decode_b4_hq32_hkv8_nq16_nk131072_d128", 4, 32, 8, 16, 131072, 128, True, seed=3001),
    "decode_b64_hq16_hkv16_nq1_nk4096_d64": DecodeWorkload(
        "decode_b64_hq16_hkv16_nq1_nk4096_d64", 64, 16, 16, 1, 4096, 64, True, seed=3002),
}


# Local (sliding-window) attention problems: a causal window of 4096 keys at 32K
# context (Mistral-style), a 1024-key causal window at 8K, and a symmetric band.
WINDOW_WORKLOADS = {
    "window_causal_w4096_b1_h32_n32768_d128": (Workload("window_causal_w4096_b1_h32_n32768_d128", 1, 32, 32, 32768,
                                                        128, False, "fwd+bwd", seed=4000), (4095, 0)),
    "window_causal_w1024_b4_hq32_hkv8_n8192_d128": (Workload("window_causal_w1024_b4_hq32_hkv8_n8192_d128", 4, 32, 8,
                                                             8192, 128, False, "fwd+bwd", seed=4001), (1023, 0)),
    "window_sym_w512_b2_h16_n16384_d64": (Workload("window_sym_w512_b2_h16_n16384_d64", 2, 16, 16, 16384, 64, False,
                                                   "fwd+bwd", seed=4002), (256, 256)),
}


def make_decode_inputs(w: DecodeWorkload, device="cpu"):
    """q [B,Hq,Nq,d], k and v [B,Hkv,Nk,d]: bf16 N(0,1) draws from one seeded generator."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    q = _normal_bf16((w.B, w.Hq, w.Nq, w.d), 1.0, gen, dev)
    k = _normal_bf16((w.B, w.Hkv, w.Nk, w.d), 1.0, gen, dev)
    v = _normal_bf16((w.B, w.Hkv, w.Nk, w.d), 1.0, gen, dev)
    return {"q": q, "k": k, "v": v}


# Sequence-length sweep: a fixed number of tokens B*N and a fixed model width Hq*d,
# so the work per token grows with N and the FLOP/byte of each head is ~N/4.  At
# N = 32768 one sequence already exceeds the token budget, so B stays 1 there.
SWEEP_TOKENS = 16384
SWEEP_WIDTH = 2048
SWEEP_N = (1024, 2048, 4096, 8192, 16384, 32768)
SWEEP_D = (64, 128)


def sweep_workloads():
    """Workloads of the sequence-length sweep, non-causal and causal, both head sizes; seeds 2000+k."""
    out = []
    for d in SWEEP_D:
        for causal in (False, True):
            for n in SWEEP_N:
                B = max(1, SWEEP_TOKENS // n)
                H = SWEEP_WIDTH // d
                name = f"sweep_{'causal' if causal else 'full'}_b{B}_h{H}_n{n}_d{d}"
                out.append(Workload(name, B, H, H, n, d, causal, "fwd+bwd", seed=2000 + len(out)))
    return out


def _normal_bf16(shape, std, gen, device):
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def make_inputs(B, Hq, Hkv, N, d, *, seed=0, qk_std=1.0, vo_std=1.0, boost_frac=0.0,
                boost=1.0, device="cpu", with_grad=True):
    """Return dict q, k, v (and dO) as contiguous bf16 tensors on ``device``.

    Draw order is fixed (q, k, v, dO, then the boosted-row permutations), so the
    same seed gives the same bits for a given device type.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    q = _normal_bf16((B, Hq, N, d), qk_std, gen, dev)
    k = _normal_bf16((B, Hkv, N, d), qk_std, gen, dev)
    v = _normal_bf16((B, Hkv, N, d), vo_std, gen, dev)
    out = {"q": q, "k": k, "v": v}
    if with_grad:
        out["do"] = _normal_bf16((B, Hq, N, d), vo_std, gen, dev)
    nboost = int(math.floor(boost_frac * N))
    if nboost > 0:
        pgen = torch.Generator(device="cpu")
        pgen.manual_seed(seed + 7919)
        for b in range(B):
            for h in range(Hkv):
                rows = torch.randperm(N, generator=pgen)[:nboost].to(dev)
                k[b, h, rows] = (k[b, h, rows].float() * boost).to(torch.bfloat16)
    return out


def make_fp8_inputs(B, Hq, Hkv, N, d, *, seed=0, qk_std=1.0, vo_std=1.0, device="cpu"):
    """e4m3 q, k, v (torch.float8_e4m3fn) and their per-tensor descales.

    Values are drawn as fp32 normals (q, k, v in that order from one seeded
    generator), each tensor's descale is its largest magnitude over 448 (the largest
    finite e4m3), and the codes are the values divided by the descale, cast by torch
    (round to nearest even).  Returns {"q", "k", "v", "q_descale", "k_descale", "v_descale"}.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    out = {}
    for name, shape, std in (("q", (B, Hq, N, d), qk_std), ("k", (B, Hkv, N, d), qk_std),
                             ("v", (B, Hkv, N, d), vo_std)):
        x = torch.randn(shape, generator=gen, dtype=torch.float32, device=dev) * std
        descale = float(x.abs().max()) / 448.0
        out[name] = (x / descale).to(torch.float8_e4m3fn)
        out[name + "_descale"] = descale
    return out


def workload_inputs(w: Workload, device="cpu", with_grad=None):
    if with_grad is None:
        with_grad = "bwd" in w.passes
    return make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, qk_std=w.qk_std,
                       vo_std=w.vo_std, boost_frac=w.boost_frac, boost=w.boost,
                       device=device, with_grad=with_grad)


def to_f64(t: torch.Tensor):
    """Exact upcast of bf16 bits to a float64 numpy array (bf16 -> fp64 is exact)."""
    return t.detach().to("cpu", torch.float64).numpy()
