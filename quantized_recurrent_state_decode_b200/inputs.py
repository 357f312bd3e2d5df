"""Seeded synthetic workloads for the decode step.

This module only draws inputs: random numbers shaped like the workloads the
method is evaluated on (GLA, Gated DeltaNet and Mamba2-SSD decode). It holds
none of the decode step's arithmetic, and it is the one module that both the
CUDA path's callers and the CPU oracle's callers use.

All draws come from ``torch.Generator`` streams seeded per (workload, tensor,
step), so any step's inputs can be regenerated on their own. Draws are made on
the device the caller names (CPU by default); a CUDA generator gives other
numbers than a CPU one, so a comparison takes both of its sides from one
device's draws. Tensors are float32 and C-contiguous:

  q, k   [B][H][d_k]       v   [B][H][d_v]
  gates  [B][H][d_k] (per-key decay) or [B][H] (scalar decay), already the
         multiplicative decay in (0, 1)
  beta   [B][H] (delta rule) or None
"""
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

ROUND_RTN, ROUND_SR, ROUND_BDR = 0, 1, 2
UPDATE_GATED, UPDATE_DELTA = 0, 1
GATE_SCALAR, GATE_PER_KEY = 0, 1

_T_Q, _T_K, _T_V, _T_G, _T_BETA, _T_S0, _T_HEAD = range(7)


@dataclass(frozen=True)
class Workload:
    name: str
    family: str            # "gla", "gdn" or "mamba2"
    batch: int
    heads: int
    d_k: int
    d_v: int
    group: int
    steps: int
    mode: int
    precision: str         # "int8", "int4" or "mixed"
    int8_fraction: float = 1.0
    s0_std: float = 0.0
    gate_mu: float = 0.0   # location of the normal draw behind the decay
    seed_id: int = 0
    description: str = ""
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def update_kind(self):
        return UPDATE_DELTA if self.family == "gdn" else UPDATE_GATED

    @property
    def gate_kind(self):
        return GATE_PER_KEY if self.family == "gla" else GATE_SCALAR

    @property
    def tiles(self):
        return self.batch * self.heads

    def with_batch(self, batch):
        return replace(self, batch=batch)


WORKLOADS = {
    # GLA, per-key decay exp(-softplus(N(-3,1))), int8 RTN, one scale per value
    # column over all 64 key rows.
    "gla_rtn_int8_b2h2_64": Workload(
        "gla_rtn_int8_b2h2_64", "gla", 2, 2, 64, 64, 64, 16, ROUND_RTN, "int8",
        gate_mu=-3.0, seed_id=1,
        description="GLA decode, int8 RTN, B=2 H=2 64x64, group 64, 16 steps"),
    # Gated DeltaNet, scalar decay sigmoid(N(4,1)), beta sigmoid(N(0,1)),
    # S0 ~ N(0, 0.02^2), int8 with hash stochastic rounding, group 32.
    "gdn_sr_int8_b64h16_128": Workload(
        "gdn_sr_int8_b64h16_128", "gdn", 64, 16, 128, 128, 32, 256, ROUND_SR, "int8",
        s0_std=0.02, gate_mu=4.0, seed_id=2,
        description="Gated DeltaNet decode, int8 SR, B=64 H=16 128x128, group 32, 256 steps"),
    # Mamba2-SSD: key axis = state N=128, value axis = headdim P=64,
    # decay exp(dt*A_h), dt = softplus(N(-2,0.5)), A_h = -exp(U(0,2));
    # top 25% of heads by mean decay int8, the rest int4; SR.
    "mamba2_mixed_sr_b128h64": Workload(
        "mamba2_mixed_sr_b128h64", "mamba2", 128, 64, 128, 64, 32, 512, ROUND_SR, "mixed",
        int8_fraction=0.25, gate_mu=-2.0, seed_id=3,
        description="Mamba2-SSD decode, mixed int8/int4 by mean decay (25% int8), SR, "
                    "B=128 H=64 N=128 P=64, group 32, 512 steps"),
    # GLA, per-key decay exp(-softplus(N(-4,1))), int4, BDR (and RTN), 1024 steps.
    "gla_bdr_int4_b256h32_128": Workload(
        "gla_bdr_int4_b256h32_128", "gla", 256, 32, 128, 128, 32, 1024, ROUND_BDR, "int4",
        gate_mu=-4.0, seed_id=4,
        description="GLA decode, int4 BDR vs RTN, B=256 H=32 128x128, group 32, 1024 steps"),
    # Gated DeltaNet mixed int8/int4 (50/50 by decay rank), SR; batch sweep.
    "gdn_mixed_sr_h32_128": Workload(
        "gdn_mixed_sr_h32_128", "gdn", 256, 32, 128, 128, 32, 72, ROUND_SR, "mixed",
        int8_fraction=0.5, s0_std=0.02, gate_mu=4.0, seed_id=5,
        description="Gated DeltaNet mixed int8/int4 (50/50 by decay rank), SR, H=32 128x128, "
                    "group 32, batch 64/256/1024, 8 warm-up + 64 timed steps"),
    # Throughput workload: B=256, 32 heads, 128x128 int8 state, group 32, RTN,
    # GLA with the distributions of the int4 workload, S0 ~ N(0, 0.02^2).
    "gla_rtn_int8_b256h32_128": Workload(
        "gla_rtn_int8_b256h32_128", "gla", 256, 32, 128, 128, 32, 72, ROUND_RTN, "int8",
        s0_std=0.02, gate_mu=-4.0, seed_id=6,
        description="GLA decode, int8 RTN, B=256 H=32 128x128, group 32"),
}


def _gen(w: Workload, tensor: int, t: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 * w.seed_id + 10_007 * tensor + t)
    return g


def _normal(shape, gen, mean=0.0, std=1.0):
    return torch.randn(shape, generator=gen, dtype=torch.float32, device=gen.device) * std + mean


def _unit_rows(x):
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def head_log_decay_rates(w: Workload, device="cpu") -> torch.Tensor:
    """Mamba2 per-head A_h = -exp(U(0, 2)); empty for other families."""
    if w.family != "mamba2":
        return torch.empty(0, device=device)
    g = _gen(w, _T_HEAD, 0, device)
    return -torch.exp(torch.rand(w.heads, generator=g, dtype=torch.float32, device=device) * 2.0)


def step_inputs(w: Workload, t: int, batch_offset: int = 0, batch: Optional[int] = None,
                device="cpu"):
    """Inputs of decode step t (0-based) for batch rows [batch_offset, +batch).

    Rows are drawn for the whole batch and sliced, so a batch shard sees the
    same numbers as the unsharded run.
    """
    B, H, dk, dv = w.batch, w.heads, w.d_k, w.d_v
    if batch is None:
        batch = B - batch_offset
    sl = slice(batch_offset, batch_offset + batch)
    q = _normal((B, H, dk), _gen(w, _T_Q, t, device))
    k = _normal((B, H, dk), _gen(w, _T_K, t, device))
    v = _normal((B, H, dv), _gen(w, _T_V, t, device))
    beta = None
    if w.family == "gla":
        k = _unit_rows(k)
        z = _normal((B, H, dk), _gen(w, _T_G, t, device), mean=w.gate_mu)
        gates = torch.exp(-torch.nn.functional.softplus(z))
    elif w.family == "gdn":
        k = _unit_rows(k)
        gates = torch.sigmoid(_normal((B, H), _gen(w, _T_G, t, device), mean=w.gate_mu))
        beta = torch.sigmoid(_normal((B, H), _gen(w, _T_BETA, t, device)))
    elif w.family == "mamba2":
        # B_t plays k, C_t plays q, x_t scaled by dt plays v; decay exp(dt*A_h).
        dt = torch.nn.functional.softplus(_normal((B, H), _gen(w, _T_G, t, device),
                                                  mean=w.gate_mu, std=0.5))
        A = head_log_decay_rates(w, device)
        gates = torch.exp(dt * A[None, :])
        v = v * dt[:, :, None]
    else:
        raise ValueError(w.family)
    out = dict(q=q[sl], k=k[sl], v=v[sl], gates=gates[sl],
               beta=None if beta is None else beta[sl])
    return {n: (None if x is None else x.contiguous()) for n, x in out.items()}


def chunk_inputs(w: Workload, t0: int, T: int, batch_offset: int = 0,
                 batch: Optional[int] = None, device="cpu"):
    """The inputs of steps t0 .. t0 + T - 1 stacked on a leading token axis:
    q, k [T][B][H][d_k], v [T][B][H][d_v], gates [T][B][H][d_k] or [T][B][H],
    beta [T][B][H] or None (a chunk of T tokens)."""
    xs = [step_inputs(w, t, batch_offset, batch, device=device) for t in range(t0, t0 + T)]
    return {n: (None if xs[0][n] is None else torch.stack([x[n] for x in xs]).contiguous())
            for n in xs[0]}


def initial_state(w: Workload, batch_offset: int = 0, batch: Optional[int] = None,
                  device="cpu"):
    """S0 [B][H][d_k][d_v]: zeros, or N(0, s0_std^2)."""
    if batch is None:
        batch = w.batch - batch_offset
    shape = (batch, w.heads, w.d_k, w.d_v)
    if w.s0_std == 0.0:
        return torch.zeros(shape, dtype=torch.float32, device=device)
    full = _normal((w.batch, w.heads, w.d_k, w.d_v), _gen(w, _T_S0, 0, device), std=w.s0_std)
    return full[batch_offset:batch_offset + batch].contiguous()


def decay_tensor(w: Workload, steps: Optional[int] = None, device="cpu"):
    """All decay values of the run, [steps*B][H][inner] (inner = d_k or 1),
    the input of the decay-based precision map."""
    steps = w.steps if steps is None else steps
    parts = []
    for t in range(steps):
        g = step_inputs(w, t, device=device)["gates"]
        parts.append(g.reshape(w.batch, w.heads, -1))
    return torch.cat(parts, 0).contiguous()


def n_int8_heads(w: Workload) -> int:
    """Number of heads kept at 8 bits."""
    if w.precision == "int8":
        return w.heads
    if w.precision == "int4":
        return 0
    return int(round(w.int8_fraction * w.heads))


def uniform_prec_map(w: Workload):
    """Precision map for the single-precision workloads (None for mixed)."""
    if w.precision == "int8":
        return torch.full((w.heads,), 8, dtype=torch.uint8)
    if w.precision == "int4":
        return torch.full((w.heads,), 4, dtype=torch.uint8)
    return None


def sr_seed(w: Workload) -> int:
    return 0x5EED + w.seed_id
