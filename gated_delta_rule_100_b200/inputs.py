"""Seeded synthetic inputs for KDA prefill and decode.

This module holds no part of the method's arithmetic: it only draws random
tensors and brings them to the value ranges the workloads use.  Both the
CUDA path and the fp64 oracle consume the same tensors it returns (the
oracle receives host copies, upcast to float64).

Recipe (all draws from one ``torch.Generator`` seeded with ``seed``, in this
order, each ``torch.randn`` in fp32, drawn in blocks of ``BLOCK_T`` tokens
along T so the fp32 temporaries stay small on long sequences):

* q, k : randn, divided by their L2 norm over the key dimension
         (floored at 1e-12), then rounded to bf16.
* v    : randn rounded to bf16.
* g    : log-decay, ``-decay * softplus(randn)`` in fp32 (so g <= 0).
* beta : ``sigmoid(randn)`` in fp32.
* h0   : ``h0_std * randn`` in fp32 when ``h0_std > 0``, else absent.

Decode draws the fp32 state first (``state_std * randn``), then for every
step the same five tensors as above with T = 1.

The shapes and decay scales are those of the workloads in ``CONFIGS``; two more
shapes measure paths of their own: a few-heads long sequence
(``TWO_LEVEL_CONFIG``) and a packed batch of sequences of mixed lengths
(``VARLEN_CONFIG``, lengths from ``varlen_lengths``).
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass

import torch

BLOCK_T = 65536


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    decay: float
    h0_std: float
    seed: int

    @property
    def scale(self) -> float:
        return self.dk ** -0.5


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    decay: float
    state_std: float
    steps: int
    seed: int

    @property
    def scale(self) -> float:
        return self.dk ** -0.5


CONFIGS = {
    "oracle_scale_B1_H1_T256_d64": PrefillConfig("oracle_scale_B1_H1_T256_d64", 1, 1, 256, 64, 64, 0.1, 0.0, 0),
    "prefill_B1_H4_T2048_d128": PrefillConfig("prefill_B1_H4_T2048_d128", 1, 4, 2048, 128, 128, 0.05, 0.02, 1),
    "training_B8_H32_T4096_d128": PrefillConfig("training_B8_H32_T4096_d128", 8, 32, 4096, 128, 128, 0.05, 0.0, 2),
    "long_context_B1_H32_T1M_d128": PrefillConfig("long_context_B1_H32_T1M_d128", 1, 32, 1 << 20, 128, 128, 0.01, 0.0, 3),
    # the training shape at a quarter of the batch: inputs (0.34 GB) above L2, small enough for
    # multi-pass counter captures
    "profile_B2_H32_T4096_d128": PrefillConfig("profile_B2_H32_T4096_d128", 2, 32, 4096, 128, 128, 0.05, 0.0, 4),
    # the long-context recipe on its first 65,536 tokens: 3.2 GB of inputs and records beyond the
    # 2 GiB workspace cap, so it runs the long-context code path (segments on two streams)
    "long_context_slice_B1_H32_T65536_d128": PrefillConfig("long_context_slice_B1_H32_T65536_d128", 1, 32, 65536,
                                                           128, 128, 0.01, 0.0, 3),
}
DECODE_CONFIG = DecodeConfig("decode_B256_H32_d128_64steps", 256, 32, 128, 128, 0.05, 0.02, 64, 4)

# Few heads, long sequence: the shape the two-level pass is for (4 heads leave most
# SMs idle under one chain CTA per head).
TWO_LEVEL_CONFIG = PrefillConfig("two_level_B1_H4_T262144_d128", 1, 4, 1 << 18, 128, 128, 0.01, 0.02, 5)


@dataclass(frozen=True)
class VarlenConfig:
    """A packed batch: N sequences whose lengths are drawn log-uniformly in
    [min_len, max_len] (a serving mix of short and long prompts), back to back
    along the token axis, each with its own initial state."""
    name: str
    N: int
    H: int
    dk: int
    dv: int
    min_len: int
    max_len: int
    decay: float
    h0_std: float
    seed: int

    @property
    def scale(self) -> float:
        return self.dk ** -0.5


VARLEN_CONFIG = VarlenConfig("varlen_N64_H32_d128_len128-16384", 64, 32, 128, 128, 128, 16384, 0.05, 0.02, 6)


def varlen_lengths(cfg: VarlenConfig):
    """The N sequence lengths of a packed-batch workload (a CPU generator seeded with
    ``seed``: log-uniform draws, rounded down, at least min_len)."""
    gen = torch.Generator().manual_seed(int(cfg.seed))
    u = torch.rand(cfg.N, generator=gen, dtype=torch.float64)
    lo, hi = torch.log(torch.tensor(float(cfg.min_len))), torch.log(torch.tensor(float(cfg.max_len)))
    return [max(cfg.min_len, int(x)) for x in torch.exp(lo + u * (hi - lo)).tolist()]


def make_varlen(cfg: VarlenConfig, device="cpu"):
    """Packed-batch inputs: dict(q, k, v, g, beta [T_total, ...], h0 [N, H, dk, dv] or
    None, cu_seqlens int32 [N + 1]) drawn with the prefill recipe on one row of
    T_total = sum of the lengths tokens (seed + 1 for h0 after the row's draws)."""
    lengths = varlen_lengths(cfg)
    T = sum(lengths)
    d = make_prefill(1, T, cfg.H, cfg.dk, cfg.dv, decay=cfg.decay, h0_std=0.0, seed=cfg.seed, device=device)
    d = {k: (v[0] if v is not None else None) for k, v in d.items()}
    if cfg.h0_std > 0:
        gen = torch.Generator(device=device)
        gen.manual_seed(int(cfg.seed) + 1)
        d["h0"] = cfg.h0_std * _randn((cfg.N, cfg.H, cfg.dk, cfg.dv), gen, device)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    d["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    return d


def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _unit_bf16(x):
    n = x.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    return (x / n).to(torch.bfloat16)


def _blocked(B, T, H, d, gen, device, fn, dtype):
    out = torch.empty((B, T, H, d), device=device, dtype=dtype)
    for t0 in range(0, T, BLOCK_T):
        t1 = min(T, t0 + BLOCK_T)
        out[:, t0:t1] = fn(_randn((B, t1 - t0, H, d), gen, device))
    return out


def make_prefill(B, T, H, dk, dv, *, decay, h0_std=0.0, seed=0, device="cpu"):
    """Return dict(q, k, v, g, beta, h0) on ``device`` (h0 is None when h0_std == 0)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    q = _blocked(B, T, H, dk, gen, device, _unit_bf16, torch.bfloat16)
    k = _blocked(B, T, H, dk, gen, device, _unit_bf16, torch.bfloat16)
    v = _blocked(B, T, H, dv, gen, device, lambda x: x.to(torch.bfloat16), torch.bfloat16)
    g = _blocked(B, T, H, dk, gen, device,
                 lambda x: -decay * torch.nn.functional.softplus(x), torch.float32)
    beta = _blocked(B, T, H, 1, gen, device, torch.sigmoid, torch.float32)[..., 0].contiguous()
    h0 = None
    if h0_std > 0:
        h0 = h0_std * _randn((B, H, dk, dv), gen, device)
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)


def make_config(cfg: PrefillConfig, device="cpu"):
    return make_prefill(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, decay=cfg.decay,
                        h0_std=cfg.h0_std, seed=cfg.seed, device=device)


def make_decode(B, H, dk, dv, *, decay, state_std, steps, seed=0, device="cpu"):
    """Return dict(state [B,H,dk,dv] fp32, and per-step stacks q,k,v [S,B,H,d] bf16,
    g [S,B,H,dk] fp32, beta [S,B,H] fp32)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    state = state_std * _randn((B, H, dk, dv), gen, device)
    qs, ks, vs, gs, bs = [], [], [], [], []
    for _ in range(steps):
        qs.append(_unit_bf16(_randn((B, H, dk), gen, device)))
        ks.append(_unit_bf16(_randn((B, H, dk), gen, device)))
        vs.append(_randn((B, H, dv), gen, device).to(torch.bfloat16))
        gs.append(-decay * torch.nn.functional.softplus(_randn((B, H, dk), gen, device)))
        bs.append(torch.sigmoid(_randn((B, H), gen, device)))
    return dict(state=state, q=torch.stack(qs), k=torch.stack(ks), v=torch.stack(vs),
                g=torch.stack(gs), beta=torch.stack(bs))


def make_decode_config(cfg: DecodeConfig = DECODE_CONFIG, device="cpu", steps=None):
    return make_decode(cfg.B, cfg.H, cfg.dk, cfg.dv, decay=cfg.decay, state_std=cfg.state_std,
                       steps=cfg.steps if steps is None else steps, seed=cfg.seed, device=device)


def digest(*tensors) -> str:
    """SHA-256 over the raw bytes of host copies of ``tensors`` (None skipped)."""
    h = hashlib.sha256()
    for t in tensors:
        if t is None:
            continue
        t = t.detach().contiguous().cpu()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        h.update(t.numpy().tobytes())
    return h.hexdigest()
