"""Seeded synthetic inputs for the CSA / HCA hot path.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic, so both the CUDA path and the CPU oracle can be fed
from it.  Values are ~N(0, 1) (weights scaled by 1/sqrt(fan_in)), cast to
bf16 (round to nearest even); pooling logits stay fp32.

Small cases are drawn on the host with a seeded ``torch.Generator('cpu')``;
the 1M-token workloads are drawn on the device with a seeded CUDA generator
(same distribution, different stream) so that gigabytes of raw cache need not
cross PCIe.  Each workload records which one it uses.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic workload of the hot path, named by what it is."""
    name: str
    kind: str            # "csa_decode" | "hca_decode" | "csa_prefill"
    B: int               # sequences
    L: int               # raw context length (max over sequences)
    m: int               # compression factor (m' for HCA)
    H: int = 64          # attention heads x 128
    W: int = 128         # raw sliding window
    D: int = 4096        # d_model of the indexer input h
    r: int = 512         # indexer query rank
    Hi: int = 8          # indexer heads x 64
    k: int = 512         # top-k
    L_min: int = 0       # ragged lengths: U[L_min, L] per sequence (0 = all L)
    T_new: int = 0       # prefill: new query tokens appended after L - T_new
    seed: int = 0
    device_rng: bool = False
    notes: str = ""

    @property
    def max_blocks(self) -> int:
        return self.L // self.m


# The five workloads of the method's long-context regime.
CSA_DECODE_4K = Workload("csa_decode_b1_ctx4096_m4_k64", "csa_decode", B=1, L=4096, m=4, H=16,
                         D=1024, r=256, Hi=4, k=64, seed=1001)
CSA_DECODE_64K_RAGGED = Workload("csa_decode_b32_ctx32k-64k_m4_k512", "csa_decode", B=32, L=65536,
                                 L_min=32768, m=4, k=512, seed=1002, device_rng=True)
CSA_DECODE_1M = Workload("csa_decode_b8_ctx1m_m4_k1024", "csa_decode", B=8, L=1 << 20, m=4, k=1024,
                         seed=1003, device_rng=True)
HCA_DECODE_1M = Workload("hca_decode_b16_ctx1m_m128", "hca_decode", B=16, L=1 << 20, m=128, k=0,
                         seed=1004, device_rng=True)
CSA_PREFILL_8K = Workload("csa_prefill_8192_after_131072_m4_k512", "csa_prefill", B=1,
                          L=131072 + 8192, T_new=8192, m=4, k=512, seed=1005, device_rng=True)

ALL = [CSA_DECODE_4K, CSA_DECODE_64K_RAGGED, CSA_DECODE_1M, HCA_DECODE_1M, CSA_PREFILL_8K]


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller test sizes)."""
    d = {f: getattr(w, f) for f in w.__dataclass_fields__}
    d.update(kw)
    return Workload(**d)


def _gen(device: str, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, g: torch.Generator, device: str, scale: float = 1.0) -> torch.Tensor:
    """~N(0, scale^2) rounded to bf16; drawn in row chunks to bound memory."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1, shape[-1]) if len(shape) > 1 else out.view(1, -1)
    rows = flat.shape[0]
    step = max(1, (1 << 26) // flat.shape[1])
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = torch.randn((r1 - r0, flat.shape[1]), generator=g, device=device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        flat[r0:r1].copy_(x)
    return out


def lengths(w: Workload, g: torch.Generator, device: str) -> torch.Tensor:
    if w.L_min and w.L_min < w.L:
        return torch.randint(w.L_min, w.L + 1, (w.B,), generator=g, device=device, dtype=torch.int32)
    return torch.full((w.B,), w.L, dtype=torch.int32, device=device)


@dataclass
class Inputs:
    """Host- or device-resident tensors of one workload (bf16 unless noted)."""
    w: Workload
    lens: torch.Tensor          # int32 [B]
    raw_kv: torch.Tensor        # [B][Lcap][128]
    raw_ki: torch.Tensor        # [B][Lcap][64]   raw indexer keys
    z_kv: torch.Tensor          # fp32 [m][128]   pooling logits (latent)
    z_ki: torch.Tensor          # fp32 [m][64]    pooling logits (indexer keys)
    q_seq: torch.Tensor         # int32 [T]
    q_pos: torch.Tensor         # int32 [T]
    h: torch.Tensor             # [T][D]
    W_dq: torch.Tensor          # [r][D]
    W_uq: torch.Tensor          # [Hi*64][r]
    W_w: torch.Tensor           # [Hi][D]
    q: torch.Tensor             # [T][H][128]  attention queries
    extra: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.q_seq.shape[0])


def make_inputs(w: Workload, device: str | None = None, Lcap: int | None = None) -> Inputs:
    """Draw every input of ``w`` in a fixed order from its seed.

    Queries: decode has one query per sequence at position len-1; prefill
    has T_new queries at positions L-T_new .. L-1 of sequence 0."""
    if device is None:
        device = "cuda" if w.device_rng else "cpu"
    g = _gen(device, w.seed)
    lens = lengths(w, g, device)
    Lc = Lcap if Lcap is not None else w.L
    z_kv = torch.randn((w.m, 128), generator=g, device=device, dtype=torch.float32)
    z_ki = torch.randn((w.m, 64), generator=g, device=device, dtype=torch.float32)
    raw_kv = randn_bf16((w.B, Lc, 128), g, device)
    raw_ki = randn_bf16((w.B, Lc, 64), g, device)
    if w.kind == "csa_prefill":
        T = w.T_new
        q_seq = torch.zeros(T, dtype=torch.int32, device=device)
        q_pos = torch.arange(w.L - w.T_new, w.L, dtype=torch.int32, device=device)
    else:
        T = w.B
        q_seq = torch.arange(w.B, dtype=torch.int32, device=device)
        q_pos = (lens - 1).to(torch.int32)
    h = randn_bf16((T, w.D), g, device)
    W_dq = randn_bf16((w.r, w.D), g, device, 1.0 / w.D ** 0.5)
    W_uq = randn_bf16((w.Hi * 64, w.r), g, device, 1.0 / w.r ** 0.5)
    W_w = randn_bf16((w.Hi, w.D), g, device, 1.0 / w.D ** 0.5)
    q = randn_bf16((T, w.H, 128), g, device)
    return Inputs(w, lens, raw_kv, raw_ki, z_kv, z_ki, q_seq, q_pos, h, W_dq, W_uq, W_w, q)


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def from_bits(a, device="cpu") -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
