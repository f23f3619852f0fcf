"""Seeded synthetic inputs for GLA workloads (shared by the tests and the benchmark).

This module only draws random numbers; it holds none of the method's arithmetic.
Recipe (one torch CPU generator, seeded, tensors drawn in this fixed order):
  q ~ N(0,1), k ~ N(0,1)/sqrt(d_k), v ~ N(0,1), z ~ N(z_mean,1), do ~ N(0,1),
  then (only when asked for) h0 ~ N(0,1)/sqrt(d_k), dh_final ~ N(0,1) and, for
  the general gate, z_beta ~ N(z_mean,1) per (token, value channel) with
  log_beta = logsigmoid(z_beta)/16 (fp32).
  Gate: alpha = sigmoid(z)^(1/16), passed as log_alpha = logsigmoid(z)/16,
  evaluated in float64 and rounded to float32.  Vector gates draw z per
  (token, key channel); scalar gates draw one z per token; "none" has no gate.
q, k, v, do are rounded to the requested dtype; log_alpha and states are fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    log_alpha: Optional[torch.Tensor]
    do: torch.Tensor
    h0: Optional[torch.Tensor]
    dh_final: Optional[torch.Tensor]
    gate: str
    log_beta: Optional[torch.Tensor] = None


def make_inputs(B, H, T, K, V, *, dtype=torch.bfloat16, gate="vector", seed=0, z_mean=0.0,
                with_h0=False, with_dh_final=False, gate_scale=None, log_alpha_const=None, with_log_beta=False):
    """Draw one seeded workload on the CPU.

    gate_scale: if given, log_alpha is multiplied by it (stress tests of strong gates).
    log_alpha_const: if given, log_alpha is this constant everywhere (edge cases)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn(B, H, T, K, generator=g, dtype=torch.float64)
    k = torch.randn(B, H, T, K, generator=g, dtype=torch.float64) / math.sqrt(K)
    v = torch.randn(B, H, T, V, generator=g, dtype=torch.float64)
    if gate == "vector":
        z = torch.randn(B, H, T, K, generator=g, dtype=torch.float64) + z_mean
    elif gate == "scalar":
        z = torch.randn(B, H, T, generator=g, dtype=torch.float64) + z_mean
    elif gate == "none":
        z = None
    else:
        raise ValueError(f"unknown gate mode {gate!r}")
    do = torch.randn(B, H, T, V, generator=g, dtype=torch.float64)
    h0 = torch.randn(B, H, K, V, generator=g, dtype=torch.float64) / math.sqrt(K) if with_h0 else None
    dhT = torch.randn(B, H, K, V, generator=g, dtype=torch.float64) if with_dh_final else None
    lb = None
    if with_log_beta:
        zb = torch.randn(B, H, T, V, generator=g, dtype=torch.float64) + z_mean
        lb = (torch.nn.functional.logsigmoid(zb) / 16.0).to(torch.float32)
    la = None
    if z is not None:
        la = torch.nn.functional.logsigmoid(z) / 16.0
        if gate_scale is not None:
            la = la * float(gate_scale)
        if log_alpha_const is not None:
            la = torch.full_like(la, float(log_alpha_const))
        la = la.to(torch.float32)
    return Inputs(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), log_alpha=la, do=do.to(dtype),
                  h0=None if h0 is None else h0.to(torch.float32),
                  dh_final=None if dhT is None else dhT.to(torch.float32), gate=gate, log_beta=lb)
