"""Seeded synthetic inputs for the gated delta-net scan.

This module is the one piece shared by the CUDA library's tests/bench and the
FP64 oracle: it draws random tensors and holds none of the method's
arithmetic.  Every tensor is drawn on the CPU from `torch.Generator`
seeded with the workload's seed, in the fixed order q, k, v, alpha-noise,
beta-noise, normalised in fp32 and then cast to the workload's dtype, so the
same seed gives the same numbers on every machine.

Workloads (shapes follow the latent grids of the video models on the pages:
21 latent frames of 30x52 tokens at 480p, 45x80 at 720p, 1,560 tokens per
frame for the streaming rollout):

  tiny       B=1, H=2,  T=256,    d=64,  fp32  (parity-only size)
  stream480  B=1, H=12, T=32,760, d=128, bf16  causal
  bidir720   B=1, H=20, T=75,600, d=128, bf16  bidirectional
  rollout    B=1, H=16, 168 calls x 1,560 tokens, d=128, bf16, state carried
  skewed     B=4, H=32, T=16,384, d=128, bf16, fast-forgetting gates
  vda480     B=1, H=12, T=32,760 = 21 frames x 1,560 tokens, d=128, bf16,
             frame-wise delta operator, bidirectional (the per-frame decay is
             the alpha drawn for the frame's first token)

Distributions: q, k ~ N(0,1) then L2-normalised over the head dimension per
token and head; v ~ N(0,1).  "default" gates: alpha = exp(-softplus(n)*0.05),
beta = sigmoid(n') with n, n' ~ N(0,1).  "skewed" gates: log alpha ~ U[-2,0],
beta ~ U[0.9, 1.0].
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str          # "f32" or "bf16": dtype of q, k, v and o
    seed: int
    gates: str = "default"
    mode: str = "causal"  # "causal", "bidir", "rollout" or "vda" (frame-wise, bidirectional)
    calls: int = 1        # rollout: number of successive calls of T tokens
    frame: int = 0        # vda: tokens per frame

    @property
    def total_T(self) -> int:
        return self.T * self.calls

    @property
    def token_heads(self) -> int:
        return self.B * self.H * self.total_T


WORKLOADS = {
    "tiny": Workload("tiny", 1, 256, 2, 64, 64, "f32", 0),
    "stream480": Workload("stream480", 1, 32760, 12, 128, 128, "bf16", 1),
    "bidir720": Workload("bidir720", 1, 75600, 20, 128, 128, "bf16", 2, mode="bidir"),
    "rollout": Workload("rollout", 1, 1560, 16, 128, 128, "bf16", 3, mode="rollout", calls=168),
    "skewed": Workload("skewed", 4, 16384, 32, 128, 128, "bf16", 4, gates="skewed"),
    "vda480": Workload("vda480", 1, 32760, 12, 128, 128, "bf16", 5, mode="vda", frame=1560),
}


def frame_alpha(alpha: torch.Tensor, U: int) -> torch.Tensor:
    """Per-frame decays [B, F, H] for frames of U tokens: the alpha drawn for
    each frame's first token."""
    return alpha[:, ::U].contiguous()

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def generate(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
             seed: int = 0, gates: str = "default", device="cpu") -> dict:
    """Draw one set of inputs.  Returns q, k [B,T,H,dk] and v [B,T,H,dv] in
    `dtype`, alpha and beta [B,T,H] in fp32, on `device` (drawn on the CPU)."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = _unit(torch.randn(B, T, H, dk, generator=g))
    k = _unit(torch.randn(B, T, H, dk, generator=g))
    v = torch.randn(B, T, H, dv, generator=g)
    if gates == "default":
        alpha = torch.exp(-torch.nn.functional.softplus(torch.randn(B, T, H, generator=g)) * 0.05)
        beta = torch.sigmoid(torch.randn(B, T, H, generator=g))
    elif gates == "skewed":
        alpha = torch.exp(-2.0 * torch.rand(B, T, H, generator=g))
        beta = 0.9 + 0.1 * torch.rand(B, T, H, generator=g)
    else:
        raise ValueError("unknown gate recipe %r" % gates)
    td = TORCH_DTYPE[dtype]
    out = dict(q=q.to(td), k=k.to(td), v=v.to(td),
               alpha=alpha.float().contiguous(), beta=beta.float().contiguous())
    if device != "cpu":
        out = {n: t.to(device) for n, t in out.items()}
    return out


def workload_inputs(w: Workload | str, device="cpu") -> dict:
    """Inputs of a named workload (a rollout is one tensor of calls*T tokens,
    sliced per call by the caller)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    return generate(w.B, w.total_T, w.H, w.dk, w.dv, w.dtype, w.seed, w.gates, device)
