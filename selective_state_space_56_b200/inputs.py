"""Seeded synthetic inputs for the selective scan and its decode step.

This module only draws numbers; it holds none of the method's arithmetic, and it
is the one module both the CUDA path's callers and the CPU oracle's tests use.

Workloads (layer shapes of the Mamba family; the distributions stand in for
real activations, no dataset is read):

=========  =====  =====  =====  ==========  ===========================
name       batch  dim    N      seqlen      dtypes (u, delta, z, B, C / y)
=========  =====  =====  =====  ==========  ===========================
tiny_fp32  1      16     4      64          fp32 / fp32
m130m      8      1536   16     2048        bf16 / bf16
m2p8b      4      5120   16     4096        bf16 / bf16
million    1      2048   16     1048576     bf16 / bf16
decode     256    5120   16     1 token x 1000 steps, fp32 state
=========  =====  =====  =====  ==========  ===========================

The causal conv1d producer (conv_inputs) draws, from its own seed, x ~ N(0, 1) with shape
(batch, dim, L) in the storage dtype, then weight (dim, K) and bias (dim) ~ U(-1/sqrt(K),
1/sqrt(K)) in fp32, then (when asked) an initial state (batch, dim, K - 1) ~ N(0, 1); the
bench uses the m2p8b layer's shape (4, 5120, 4096), K = 4, bf16, seed 56010, and decode
tokens of (256, 5120) from seed 56011.

Recipe: u, delta_raw, z ~ N(0, 1) with shape (batch, dim, L); B, C ~ N(0, 1)
with shape (batch, N, L), shared by all channels of a batch; A[d, n] = -(n + 1);
D ~ N(0, 1) per channel; delta_bias = log(expm1(v)) with v ~ U[0.001, 0.1] per
channel (so the biased step size starts in [0.001, 0.1]).  Values are drawn in
fp32 and rounded to the storage dtype (round-to-nearest-even for bf16).  The
draw order is u, delta_raw, z, B, C, D, v from one ``torch.Generator`` seeded
with 56000 + the workload's index (1..4).  The decode workload draws D, v and
the initial state ~ N(0, 0.1^2) (standard deviation 0.1) from seed 56005, and
step k's u, delta_raw, z, B, C from seed 56006 + k.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class ScanWorkload:
    name: str
    index: int
    batch: int
    dim: int
    dstate: int
    seqlen: int
    in_dtype: torch.dtype
    out_dtype: torch.dtype

    @property
    def seed(self) -> int:
        return 56000 + self.index

    @property
    def elements(self) -> int:
        return self.batch * self.dim * self.seqlen


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    index: int
    batch: int
    dim: int
    dstate: int
    steps: int
    io_dtype: torch.dtype

    @property
    def seed(self) -> int:
        return 56000 + self.index


SCAN_WORKLOADS = {
    "tiny_fp32": ScanWorkload("tiny_fp32", 1, 1, 16, 4, 64, torch.float32, torch.float32),
    "m130m": ScanWorkload("m130m", 2, 8, 1536, 16, 2048, torch.bfloat16, torch.bfloat16),
    "m2p8b": ScanWorkload("m2p8b", 3, 4, 5120, 16, 4096, torch.bfloat16, torch.bfloat16),
    "million": ScanWorkload("million", 4, 1, 2048, 16, 1 << 20, torch.bfloat16, torch.bfloat16),
}
DECODE_WORKLOAD = DecodeWorkload("decode", 5, 256, 5120, 16, 1000, torch.bfloat16)


def a_matrix(dim: int, dstate: int, device="cpu") -> torch.Tensor:
    """A[d, n] = -(n + 1), fp32, shape (dim, dstate)."""
    row = -torch.arange(1, dstate + 1, dtype=torch.float32, device=device)
    return row.expand(dim, dstate).contiguous()


def _bias_from_uniform(v: torch.Tensor) -> torch.Tensor:
    # inverse of log(1 + e^x) at v, evaluated in fp64 and stored as fp32
    return torch.log(torch.expm1(v.double())).float()


def scan_inputs(batch, dim, dstate, seqlen, in_dtype=torch.bfloat16, seed=0, device="cpu",
                with_z=True, with_d=True, with_bias=True):
    """One seeded set of scan inputs with the workload recipe above."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))

    def normal(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32, device=device)

    u = normal(batch, dim, seqlen).to(in_dtype)
    delta = normal(batch, dim, seqlen).to(in_dtype)
    z = normal(batch, dim, seqlen).to(in_dtype)
    B = normal(batch, dstate, seqlen).to(in_dtype)
    C = normal(batch, dstate, seqlen).to(in_dtype)
    D = normal(dim)
    v = 0.001 + 0.099 * torch.rand(dim, generator=g, dtype=torch.float32, device=device)
    return dict(
        u=u, delta=delta, A=a_matrix(dim, dstate, device), B=B, C=C,
        D=D if with_d else None,
        z=z if with_z else None,
        delta_bias=_bias_from_uniform(v) if with_bias else None,
    )


def workload_inputs(w: ScanWorkload, device="cpu"):
    return scan_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed, device)


def decode_params(w: DecodeWorkload = DECODE_WORKLOAD, device="cpu"):
    """A, D, delta_bias and the initial state for the decode workload."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    D = torch.randn(w.dim, generator=g, dtype=torch.float32, device=device)
    v = 0.001 + 0.099 * torch.rand(w.dim, generator=g, dtype=torch.float32, device=device)
    state0 = 0.1 * torch.randn(w.batch, w.dim, w.dstate, generator=g, dtype=torch.float32,
                               device=device)
    return dict(A=a_matrix(w.dim, w.dstate, device), D=D, delta_bias=_bias_from_uniform(v),
                state0=state0)


def decode_step_inputs(step: int, w: DecodeWorkload = DECODE_WORKLOAD, device="cpu",
                       batch=None, dim=None):
    """Fresh per-token inputs u, delta, z (batch, dim) and B, C (batch, N) for one step."""
    b = w.batch if batch is None else batch
    d = w.dim if dim is None else dim
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 1 + int(step))

    def normal(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32, device=device)

    u = normal(b, d).to(w.io_dtype)
    delta = normal(b, d).to(w.io_dtype)
    z = normal(b, d).to(w.io_dtype)
    B = normal(b, w.dstate).to(w.io_dtype)
    C = normal(b, w.dstate).to(w.io_dtype)
    return dict(u=u, delta=delta, z=z, B=B, C=C)


def decode_tokens_batched(steps: int, w: DecodeWorkload = DECODE_WORKLOAD, device="cpu"):
    """u, delta, z (steps, batch, dim) and B, C (steps, batch, N) for `steps` tokens at once,
    drawn in that order from one generator seeded with the workload seed + 1_000_000
    (used where per-token seeding is not needed and fewer, larger draws are wanted)."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 1_000_000)

    def normal(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32, device=device).to(w.io_dtype)

    return dict(u=normal(steps, w.batch, w.dim), delta=normal(steps, w.batch, w.dim),
                z=normal(steps, w.batch, w.dim), B=normal(steps, w.batch, w.dstate),
                C=normal(steps, w.batch, w.dstate))


def inverse_softplus_range():
    """The bias range the recipe produces: [log(expm1(0.001)), log(expm1(0.1))]."""
    return math.log(math.expm1(0.001)), math.log(math.expm1(0.1))


CONV_WIDTH = 4
CONV_SEED = 56010


def conv_inputs(batch, dim, seqlen, width=CONV_WIDTH, dtype=torch.bfloat16, seed=CONV_SEED,
                device="cpu", with_bias=True, with_initial_state=False):
    """x (batch, dim, L), weight (dim, K), bias (dim) [, initial_state (batch, dim, K-1)]."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(batch, dim, seqlen, generator=g, dtype=torch.float32, device=device).to(dtype)
    bound = 1.0 / math.sqrt(width)
    w = (torch.rand(dim, width, generator=g, dtype=torch.float32, device=device) * 2 - 1) * bound
    bias = (torch.rand(dim, generator=g, dtype=torch.float32, device=device) * 2 - 1) * bound
    init = None
    if with_initial_state:
        init = torch.randn(batch, dim, width - 1, generator=g, dtype=torch.float32,
                           device=device).to(dtype)
    return dict(x=x, weight=w, bias=bias if with_bias else None, initial_state=init)
