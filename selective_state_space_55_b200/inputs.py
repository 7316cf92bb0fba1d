"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and lays them out; it holds none of the
scan's arithmetic.  Both the CUDA path and the float64 oracle consume what it
produces (the oracle through an exact conversion to float64), so the two sides
always see bit-identical values.

Workloads (sizes from the pages' model shapes; all values synthetic):

  tiny_fp32         batch 1, 16 channels, N 16, L 256, fp32.  u, delta, z, B, C,
                    D ~ N(0,1); delta_bias ~ U(-4,-2); softplus on.
  mamba_1p4b_layer  batch 8, d_inner 4096, N 16, L 2048, bf16 in/out, fp32 state.
  mamba_2p8b_layer  batch 16, d_inner 5120, N 16, L 2048, bf16, returns last_state.
                    Both layer shapes: u, delta, z ~ N(0,1); B, C ~ N(0,1)/4;
                    delta_bias = log(expm1(v)), v ~ U(1e-3, 0.1) (so softplus of
                    the bias alone is v); D = 1.
  long_dna_1m       batch 1, d_inner 1536, N 16, L 1,048,576, bf16.  u_t is one of
                    4 symbols (i.i.d. uniform) embedded by a fixed seeded 4 x 1536
                    N(0,1) matrix, standing in for the pages' DNA sequences (no
                    dataset is used); the rest as the layer shapes.
  decode_b128       selective_state_update over 48 layers: batch 128, d_inner
                    4096, N 16, fp32 state per layer; x, dt, z ~ N(0,1) bf16;
                    B, C ~ N(0,1)/4 bf16; dt_bias as the layer shapes; D = 1.

A is the S4D-real initialisation A_d,n = -(n+1), i.e. -1 ... -16 for N = 16
("Mamba 与状态空间模型", section 每一步都一样).

Mamba-2 layer workloads (scalar A per head, head dim 64, state 128 per
channel as in "Mamba 与状态空间模型", section "Mamba-2：两种算法"; layout
(batch, L, heads, headdim)):

  ssd_small          batch 2, L 300 (three chunks of 128, the last ragged),
                     4 heads in 2 groups, with a start state.
  mamba2_2p7b_layer  batch 16, L 2048, 80 heads x 64 (d_inner 5120), 1 group.
                     Both: x, z, dt ~ N(0,1) bf16; dt_bias as the layer shapes;
                     A_h = -U(1, 16); B, C ~ N(0,1)/4 bf16; D = 1; start state
                     ~ N(0,1)/4 fp32 where used.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class ScanConfig:
    name: str
    batch: int
    dim: int
    dstate: int
    seqlen: int
    io_dtype: torch.dtype
    bc_dtype: torch.dtype
    recipe: str                 # "tiny" | "layer" | "dna"
    has_z: bool = True
    has_D: bool = True
    has_bias: bool = True
    softplus: bool = True
    last_state: bool = False

    @property
    def elements(self) -> int:
        return self.batch * self.dim * self.seqlen

    def resized(self, **kw) -> "ScanConfig":
        return replace(self, **kw)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    dim: int
    dstate: int
    layers: int
    steps: int
    io_dtype: torch.dtype = torch.bfloat16
    bc_dtype: torch.dtype = torch.bfloat16


SCAN_CONFIGS = {
    "tiny_fp32": ScanConfig("tiny_fp32", 1, 16, 16, 256, torch.float32, torch.float32,
                            "tiny", last_state=True),
    "mamba_1p4b_layer": ScanConfig("mamba_1p4b_layer", 8, 4096, 16, 2048, torch.bfloat16,
                                   torch.bfloat16, "layer"),
    "mamba_2p8b_layer": ScanConfig("mamba_2p8b_layer", 16, 5120, 16, 2048, torch.bfloat16,
                                   torch.bfloat16, "layer", last_state=True),
    "long_dna_1m": ScanConfig("long_dna_1m", 1, 1536, 16, 1 << 20, torch.bfloat16,
                              torch.bfloat16, "dna", last_state=True),
}

@dataclass(frozen=True)
class SsdConfig:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int = 64
    ngroups: int = 1
    dstate: int = 128
    has_z: bool = True
    has_D: bool = True
    has_bias: bool = True
    initial_state: bool = False

    @property
    def elements(self) -> int:
        return self.batch * self.seqlen * self.nheads * self.headdim

    def resized(self, **kw) -> "SsdConfig":
        return replace(self, **kw)


SSD_CONFIGS = {
    "ssd_small": SsdConfig("ssd_small", batch=2, seqlen=300, nheads=4, ngroups=2,
                           initial_state=True),
    "mamba2_2p7b_layer": SsdConfig("mamba2_2p7b_layer", batch=16, seqlen=2048, nheads=80),
}


def make_ssd_inputs(cfg: SsdConfig, device="cpu", seed: int = 0) -> dict:
    """All Mamba-2 layer inputs for ``cfg`` as contiguous tensors on ``device``.

    Keys: x, dt, A, B, C, D, z, dt_bias, initial_state (None where absent).
    """
    g = _gen(device, seed)
    bsz, L, H, P, G, N = cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim, cfg.ngroups, cfg.dstate
    bf = torch.bfloat16
    x = _normal((bsz, L, H, P), g, device, dtype=bf)
    z = _normal((bsz, L, H, P), g, device, dtype=bf)
    dt = _normal((bsz, L, H), g, device, dtype=bf)
    bias = layer_delta_bias(H, g, device)
    A = (-_uniform((H,), 1.0, 16.0, g, device)).to(torch.float32)
    B = _normal((bsz, L, G, N), g, device, scale=0.25, dtype=bf)
    C = _normal((bsz, L, G, N), g, device, scale=0.25, dtype=bf)
    h0 = _normal((bsz, H, P, N), g, device, scale=0.25)
    return dict(
        x=x.contiguous(), dt=dt.contiguous(), A=A.contiguous(), B=B.contiguous(),
        C=C.contiguous(),
        D=torch.ones(H, dtype=torch.float32, device=device) if cfg.has_D else None,
        z=z.contiguous() if cfg.has_z else None,
        dt_bias=bias.contiguous() if cfg.has_bias else None,
        initial_state=h0.contiguous() if cfg.initial_state else None,
    )


DECODE_CONFIG = DecodeConfig("decode_b128", batch=128, dim=4096, dstate=16, layers=48, steps=128)


def s4d_real_A(dim: int, dstate: int, device="cpu") -> torch.Tensor:
    """A_d,n = -(n+1) for every channel, fp32 (dim, dstate)."""
    row = -torch.arange(1, dstate + 1, dtype=torch.float32, device=device)
    return row.repeat(dim, 1).contiguous()


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, g, device, scale=1.0, dtype=torch.float32):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def _uniform(shape, lo, hi, g, device):
    x = torch.rand(shape, generator=g, device=device, dtype=torch.float64)
    return x * (hi - lo) + lo


def layer_delta_bias(dim: int, g, device) -> torch.Tensor:
    """delta_bias = log(expm1(v)), v ~ U(1e-3, 0.1); drawn in float64, stored fp32."""
    v = _uniform((dim,), 1e-3, 0.1, g, device)
    return torch.log(torch.expm1(v)).to(torch.float32)


def make_scan_inputs(cfg: ScanConfig, device="cpu", seed: int = 0) -> dict:
    """All scan inputs for ``cfg`` as contiguous tensors on ``device``.

    Keys: u, delta, z (or None), A, B, C, D (or None), delta_bias (or None).
    """
    g = _gen(device, seed)
    bsz, dim, N, L = cfg.batch, cfg.dim, cfg.dstate, cfg.seqlen
    io, bc = cfg.io_dtype, cfg.bc_dtype
    if cfg.recipe == "tiny":
        u = _normal((bsz, dim, L), g, device, dtype=io)
        delta = _normal((bsz, dim, L), g, device, dtype=io)
        z = _normal((bsz, dim, L), g, device, dtype=io)
        bias = _uniform((dim,), -4.0, -2.0, g, device).to(torch.float32)
        B = _normal((bsz, N, L), g, device, dtype=bc)
        C = _normal((bsz, N, L), g, device, dtype=bc)
        D = _normal((dim,), g, device)
    elif cfg.recipe in ("layer", "dna"):
        if cfg.recipe == "layer":
            u = _normal((bsz, dim, L), g, device, dtype=io)
        else:
            W = _normal((4, dim), _gen("cpu", 1234), "cpu").to(device)
            sym = torch.randint(0, 4, (bsz, L), generator=g, device=device)
            u = W.t()[:, sym].permute(1, 0, 2).to(io).contiguous()   # (bsz, dim, L)
        delta = _normal((bsz, dim, L), g, device, dtype=io)
        z = _normal((bsz, dim, L), g, device, dtype=io)
        bias = layer_delta_bias(dim, g, device)
        B = _normal((bsz, N, L), g, device, scale=0.25, dtype=bc)
        C = _normal((bsz, N, L), g, device, scale=0.25, dtype=bc)
        D = torch.ones(dim, dtype=torch.float32, device=device)
    else:
        raise ValueError(f"unknown recipe {cfg.recipe!r}")
    return dict(
        u=u.contiguous(), delta=delta.contiguous(),
        z=z.contiguous() if cfg.has_z else None,
        A=s4d_real_A(dim, N, device),
        B=B.contiguous(), C=C.contiguous(),
        D=D.contiguous() if cfg.has_D else None,
        delta_bias=bias.contiguous() if cfg.has_bias else None,
    )


def make_decode_layer(cfg: DecodeConfig, device="cpu", seed: int = 0,
                      state_scale: float = 1.0) -> dict:
    """One layer's parameters and initial state: state, A, D, dt_bias."""
    g = _gen(device, seed)
    dim, N = cfg.dim, cfg.dstate
    if state_scale == 0.0:
        state = torch.zeros((cfg.batch, dim, N), dtype=torch.float32, device=device)
    else:
        state = _normal((cfg.batch, dim, N), g, device, scale=state_scale)
    return dict(
        state=state.contiguous(),
        A=s4d_real_A(dim, N, device),
        D=torch.ones(dim, dtype=torch.float32, device=device),
        dt_bias=layer_delta_bias(dim, g, device),
    )


def make_decode_token(cfg: DecodeConfig, device="cpu", seed: int = 0) -> dict:
    """One token's per-layer inputs: x, dt, z (batch, dim); B, C (batch, N)."""
    g = _gen(device, seed)
    shape = (cfg.batch, cfg.dim)
    return dict(
        x=_normal(shape, g, device, dtype=cfg.io_dtype).contiguous(),
        dt=_normal(shape, g, device, dtype=cfg.io_dtype).contiguous(),
        z=_normal(shape, g, device, dtype=cfg.io_dtype).contiguous(),
        B=_normal((cfg.batch, cfg.dstate), g, device, scale=0.25, dtype=cfg.bc_dtype).contiguous(),
        C=_normal((cfg.batch, cfg.dstate), g, device, scale=0.25, dtype=cfg.bc_dtype).contiguous(),
    )


def sample_chains(batch: int, dim: int, count: int, seed: int = 0) -> list[tuple[int, int]]:
    """``count`` distinct (b, d) chains, always including the first and last channel."""
    g = torch.Generator().manual_seed(seed)
    total = batch * dim
    count = min(count, total)
    picks = {0, total - 1}
    perm = torch.randperm(total, generator=g).tolist()
    for p in perm:
        if len(picks) >= count:
            break
        picks.add(p)
    return sorted((p // dim, p % dim) for p in picks)


def gather_chains(inputs: dict, chains: list[tuple[int, int]]) -> dict:
    """CPU copies of the inputs of each chain in ``chains``, one dict per chain.

    Each dict is a batch-1, one-channel problem: u, delta, z (1, 1, L);
    B, C (1, N, L) of that chain's batch row; A (1, N); D, delta_bias (1,).
    """
    rows = []
    for b, d in chains:
        sl = lambda t: None if t is None else t[b:b + 1, d:d + 1].cpu()  # noqa: E731
        rows.append(dict(
            b=b, d=d,
            u=sl(inputs["u"]), delta=sl(inputs["delta"]), z=sl(inputs["z"]),
            B=inputs["B"][b:b + 1].cpu(), C=inputs["C"][b:b + 1].cpu(),
            A=inputs["A"][d:d + 1].cpu(),
            D=None if inputs["D"] is None else inputs["D"][d:d + 1].cpu(),
            delta_bias=None if inputs["delta_bias"] is None else inputs["delta_bias"][d:d + 1].cpu(),
        ))
    return rows


__all__ = [
    "ScanConfig", "DecodeConfig", "SCAN_CONFIGS", "DECODE_CONFIG", "s4d_real_A",
    "make_scan_inputs", "make_decode_layer", "make_decode_token", "sample_chains",
    "gather_chains", "layer_delta_bias", "SsdConfig", "SSD_CONFIGS", "make_ssd_inputs",
]
