"""Seeded synthetic inputs for the attention workloads.

This module is shared by the float64 oracle's tests, the GPU parity tests and
the benchmark. It holds shapes and random-number recipes only: none of the
attention arithmetic lives here, so neither side of a parity comparison can
inherit a mistake from the other through it.

Workload shapes follow the benchmark family the FlashAttention README summary
describes (hysenlabs.com "Leistungs- und Speicherangaben im README": head
dimension 64 and 128, sequence lengths 512 to 16k) and the five configurations
the build is measured on. Values are iid standard normal, drawn in float32 on
the CPU from a fixed seed and rounded once to bfloat16; the GPU and the oracle
see the same bits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: [B, H, N, d] tensors, Hq query heads, Hkv KV heads."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    q_mult: float = 1.0          # stress variant: Q scaled before the bf16 cast
    backward: bool = False       # whether the workload includes dQ, dK, dV
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4*B*Hq*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    def bwd_flops(self) -> float:
        """Backward is five N*N*d contractions against the forward's two: 2.5x."""
        return 2.5 * self.fwd_flops()


# The five configurations (c3 has three variants). Seeds are 1000 + index.
C1 = Workload("c1_B1_H1_N128_d64", 1, 1, 1, 128, 64, causal=False, seed=1000)
C2 = Workload("c2_B2_H8_N1024_d64_causal", 2, 8, 8, 1024, 64, causal=True, seed=1001)
C3_CAUSAL = Workload("c3_B4_H16_N4096_d128_causal", 4, 16, 16, 4096, 128, causal=True, seed=1002)
C3_FULL = Workload("c3_B4_H16_N4096_d128_noncausal", 4, 16, 16, 4096, 128, causal=False, seed=1002)
C3_STRESS = Workload("c3_B4_H16_N4096_d128_causal_q4", 4, 16, 16, 4096, 128, causal=True,
                     q_mult=4.0, seed=1002)
C4 = Workload("c4_B1_Hq32_Hkv8_N16384_d128_causal_gqa", 1, 32, 8, 16384, 128, causal=True,
              seed=1003)
C5 = Workload("c5_B8_H16_N2048_d128_causal_fwdbwd", 8, 16, 16, 2048, 128, causal=True,
              backward=True, seed=1004)

ALL = [C1, C2, C3_CAUSAL, C3_FULL, C3_STRESS, C4, C5]


def make_inputs(w: Workload, with_grad_out: bool | None = None):
    """Return (q, k, v[, dO]) as CPU bfloat16 tensors of shape [B, H, N, d].

    Draw order is Q, K, V, dO from one generator seeded with ``w.seed``;
    float32 standard normal, Q multiplied by ``w.q_mult`` (a power of two, so
    exact) and every tensor rounded once to bfloat16.
    """
    if with_grad_out is None:
        with_grad_out = w.backward
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    q = torch.randn((w.B, w.Hq, w.N, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.Hkv, w.N, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.Hkv, w.N, w.d), generator=g, dtype=torch.float32)
    q = (q * w.q_mult).to(torch.bfloat16)
    k = k.to(torch.bfloat16)
    v = v.to(torch.bfloat16)
    if not with_grad_out:
        return q, k, v
    do = torch.randn((w.B, w.Hq, w.N, w.d), generator=g, dtype=torch.float32)
    return q, k, v, do.to(torch.bfloat16)


def small(name: str, B: int, Hq: int, Hkv: int, N: int, d: int, causal: bool,
          seed: int = 7, q_mult: float = 1.0, backward: bool = True) -> Workload:
    """An edge-case shape for parity tests (ragged N, tiny heads, GQA...)."""
    return Workload(name, B, Hq, Hkv, N, d, causal, q_mult=q_mult, backward=backward, seed=seed)


def make_inputs_qk(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, seed: int,
                   q_mult: float = 1.0, with_grad_out: bool = True):
    """(q, k, v[, dO]) with Nq query rows and Nk key rows, CPU bfloat16.

    Same recipe as ``make_inputs``: one generator seeded with ``seed``, draw
    order Q [B,Hq,Nq,d], K and V [B,Hkv,Nk,d], dO [B,Hq,Nq,d], float32 standard
    normal rounded once to bfloat16.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((B, Hq, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    out = [(q * q_mult).to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)]
    if with_grad_out:
        out.append(torch.randn((B, Hq, Nq, d), generator=g, dtype=torch.float32).to(torch.bfloat16))
    return tuple(out)


def make_packed_inputs(lens_q, lens_k, Hq: int, Hkv: int, d: int, seed: int,
                       q_mult: float = 1.0, with_grad_out: bool = True):
    """A packed (varlen) batch: (q, k, v[, dO], cu_q, cu_k) on the CPU.

    q/dO are [sum(lens_q), Hq, d] and k/v [sum(lens_k), Hkv, d], bfloat16,
    drawn like ``make_inputs`` (one generator seeded with ``seed``, order
    Q, K, V, dO, float32 normal rounded once). cu_q/cu_k are int32 offsets of
    length B + 1 starting at 0.
    """
    if len(lens_q) != len(lens_k):
        raise ValueError("lens_q and lens_k must have the same length")
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((tq, Hq, d), generator=g, dtype=torch.float32)
    k = torch.randn((tk, Hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((tk, Hkv, d), generator=g, dtype=torch.float32)
    out = [(q * q_mult).to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)]
    if with_grad_out:
        out.append(torch.randn((tq, Hq, d), generator=g, dtype=torch.float32).to(torch.bfloat16))
    cu = lambda lens: torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0).tolist()),
                                   dtype=torch.int32)
    out += [cu(lens_q), cu(lens_k)]
    return tuple(out)
