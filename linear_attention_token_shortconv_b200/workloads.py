"""Seeded synthetic inputs for the GDN token mixer.

This module only draws random numbers; it holds none of the method's
arithmetic.  The CUDA path and the fp64 oracle both consume the tensors it
returns (the oracle through their exact stored bits), so the two sides always
see identical inputs.

Distributions (the workload descriptions name N(mu, var), read as variances):
q, k, v, z pre-activations N(0, 1); conv weights N(0, 0.25) (std 0.5); alpha
and beta logits N(0, 1); A = log U[1, 16] per head; b_alpha = 0; RMSNorm
weight 0; initial state 0 or N(0, 0.02) (std sqrt(0.02)).  Values are drawn in
fp32 and rounded once to the input dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    lengths: tuple            # tokens per sequence
    H: int
    dk: int
    dv: int
    conv_k: int = 4
    in_dtype: torch.dtype = torch.bfloat16
    s0_var: float = 0.0       # 0 -> no initial state (zeros)
    seed: int = 0
    long_memory: bool = False  # alpha close to 1 (A = log U[0.01, 0.1], a ~ N(-2, 1))
    varlen: bool = False      # pass cu_seqlens even when lengths are equal

    @property
    def num_seqs(self) -> int:
        return len(self.lengths)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    conv_k: int = 4
    in_dtype: torch.dtype = torch.bfloat16
    s_var: float = 0.02
    seed: int = 4
    steps: int = 1000
    pool: int = 8             # distinct per-step input sets, used cyclically
    random_ring_pos: bool = False
    long_memory: bool = False  # alpha close to 1 (A = log U[0.01, 0.1], a ~ N(-2, 1))


def varlen_lengths(total: int = 262144, n: int = 8, lo: int = 4096, hi: int = 131072,
                   seed: int = 3) -> tuple:
    """n lengths drawn log-uniform on [lo, hi], rescaled to sum exactly to total.

    Rescaling clips to [lo, hi] and hands the excess (or deficit) to the
    unclipped lengths in proportion; integer rounding is settled on the longest
    unclipped length.
    """
    rng = np.random.default_rng(seed)
    raw = np.exp(rng.uniform(math.log(lo), math.log(hi), n))
    L = raw * (total / raw.sum())
    for _ in range(100):
        C = np.clip(L, lo, hi)
        free = (C > lo) & (C < hi)
        rem = total - C.sum()
        if abs(rem) < 1e-9 or not free.any():
            L = C
            break
        C[free] += rem * C[free] / C[free].sum()
        L = C
    Li = np.floor(L).astype(np.int64)
    free = (Li > lo) & (Li < hi)
    idx = int(np.argmax(np.where(free, Li, -1))) if free.any() else int(np.argmax(Li))
    Li[idx] += total - int(Li.sum())
    assert int(Li.sum()) == total and Li.min() >= lo and Li.max() <= hi
    return tuple(int(x) for x in Li)


# The five workloads of the GDN mixer (prefill 0-3, decode 4).
TINY_F32 = PrefillConfig("tiny-fp32 B=1 T=256 H=2 d=64", (256,), 2, 64, 64,
                         in_dtype=torch.float32, seed=0)
PRETRAIN = PrefillConfig("pretrain B=4 T=4096 H=16 d=128", (4096,) * 4, 16, 128, 128, seed=1)
LONG = PrefillConfig("long B=1 T=32768 H=32 d=128 S0~N(0,0.02)", (32768,), 32, 128, 128,
                     s0_var=0.02, seed=2)
VARLEN = PrefillConfig("varlen 256K tokens / 8 seqs H=16 d=128", varlen_lengths(), 16, 128, 128,
                       seed=3, varlen=True)
DECODE = DecodeConfig("decode B=256 H=32 d=128 x1000 steps", 256, 32, 128, 128, seed=4)

PREFILL_CONFIGS = {0: TINY_F32, 1: PRETRAIN, 2: LONG, 3: VARLEN}


def scaled(cfg: PrefillConfig, lengths=None, H=None, **kw) -> PrefillConfig:
    """A smaller (or otherwise modified) copy of a workload, same distributions."""
    return replace(cfg, lengths=tuple(lengths) if lengths is not None else cfg.lengths,
                   H=H if H is not None else cfg.H, **kw)


def _normal(shape, gen, device, std=1.0, mean=0.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def _uniform(shape, gen, device, lo, hi):
    return torch.rand(shape, generator=gen, device=device, dtype=torch.float32) * (hi - lo) + lo


def make_prefill_inputs(cfg: PrefillConfig, device="cpu", seed=None) -> dict:
    """All inputs of one prefill call as torch tensors on `device`."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed if seed is None else seed)
    N, H, dk, dv, K = cfg.total_tokens, cfg.H, cfg.dk, cfg.dv, cfg.conv_k
    dt = cfg.in_dtype
    C = H * (2 * dk + dv)
    d = {}
    d["q"] = _normal((N, H, dk), gen, device).to(dt)
    d["k"] = _normal((N, H, dk), gen, device).to(dt)
    d["v"] = _normal((N, H, dv), gen, device).to(dt)
    d["z"] = _normal((N, H, dv), gen, device).to(dt)
    d["conv_w"] = _normal((C, K), gen, device, std=0.5)
    if cfg.long_memory:
        d["a_logit"] = _normal((N, H), gen, device, mean=-2.0).to(dt)
        d["A"] = torch.log(_uniform((H,), gen, device, 0.01, 0.1))
    else:
        d["a_logit"] = _normal((N, H), gen, device).to(dt)
        d["A"] = torch.log(_uniform((H,), gen, device, 1.0, 16.0))
    d["b_logit"] = _normal((N, H), gen, device).to(dt)
    d["b_alpha"] = torch.zeros(H, device=device)
    d["norm_w"] = torch.zeros(dv, device=device)
    if cfg.s0_var > 0:
        d["S0"] = _normal((cfg.num_seqs, H, dk, dv), gen, device, std=math.sqrt(cfg.s0_var))
    else:
        d["S0"] = None
    if cfg.varlen or len(set(cfg.lengths)) > 1:
        cu = np.concatenate([[0], np.cumsum(cfg.lengths)]).astype(np.int32)
        d["cu_seqlens"] = torch.from_numpy(cu).to(device)
    else:
        d["cu_seqlens"] = None
    return d


def make_decode_inputs(cfg: DecodeConfig, device="cpu", seed=None) -> dict:
    """Initial decode state plus a pool of per-step token inputs.

    Returns tensors: S [B,H,dk,dv] fp32, ring [B,K-1,C] (input dtype),
    ring_pos [B] int32, conv_w, A, b_alpha, norm_w, and per-step stacks
    q,k [P,B,H,dk], v,z [P,B,H,dv], a_logit,b_logit [P,B,H] (P = pool size).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed if seed is None else seed)
    B, H, dk, dv, K, P = cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.conv_k, cfg.pool
    dt = cfg.in_dtype
    C = H * (2 * dk + dv)
    d = {}
    d["S"] = _normal((B, H, dk, dv), gen, device, std=math.sqrt(cfg.s_var))
    d["ring"] = _normal((B, K - 1, C), gen, device).to(dt)
    if cfg.random_ring_pos:
        d["ring_pos"] = torch.randint(0, K - 1, (B,), generator=gen, device=device,
                                      dtype=torch.int32)
    else:
        d["ring_pos"] = torch.zeros(B, dtype=torch.int32, device=device)
    d["conv_w"] = _normal((C, K), gen, device, std=0.5)
    if cfg.long_memory:
        d["A"] = torch.log(_uniform((H,), gen, device, 0.01, 0.1))
    else:
        d["A"] = torch.log(_uniform((H,), gen, device, 1.0, 16.0))
    d["b_alpha"] = torch.zeros(H, device=device)
    d["norm_w"] = torch.zeros(dv, device=device)
    d["q"] = _normal((P, B, H, dk), gen, device).to(dt)
    d["k"] = _normal((P, B, H, dk), gen, device).to(dt)
    d["v"] = _normal((P, B, H, dv), gen, device).to(dt)
    d["z"] = _normal((P, B, H, dv), gen, device).to(dt)
    d["a_logit"] = _normal((P, B, H), gen, device, mean=-2.0 if cfg.long_memory else 0.0).to(dt)
    d["b_logit"] = _normal((P, B, H), gen, device).to(dt)
    return d


def to_oracle_bits(t: torch.Tensor) -> np.ndarray:
    """A CPU numpy view of a tensor's exact stored bits: bf16 -> uint16, fp32 -> float32."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.int32:
        return t.numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")


@dataclass(frozen=True)
class QsaConfig:
    """QSA compressed indexer workload: `B` sequences of `n` tokens, 4 indexer
    heads of 128 dims, blocks of 4 tokens, a token budget of `budget`."""
    name: str
    B: int
    n: int
    budget: int = 2048
    seed: int = 5


QSA = QsaConfig("qsa indexer n=32768 B=1 K=2048 r=4 H=4 d=128", 1, 32768)


def make_qsa_inputs(cfg: QsaConfig, device="cpu", seed=None) -> dict:
    """Projected indexer queries [B, n, 4, 128] and shared keys [B, n, 128] ~ N(0, 1)
    in bf16; RMSNorm weights 1 + N(0, 0.01) (std 0.1) in fp32."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed if seed is None else seed)
    d = {"q": _normal((cfg.B, cfg.n, 4, 128), gen, device).to(torch.bfloat16),
         "k": _normal((cfg.B, cfg.n, 128), gen, device).to(torch.bfloat16),
         "w_q": _normal((128,), gen, device, std=0.1, mean=1.0),
         "w_k": _normal((128,), gen, device, std=0.1, mean=1.0)}
    return d


def make_layer_inputs(cfg: PrefillConfig, d_model: int, device="cpu", seed=None) -> dict:
    """Inputs of the layer from the hidden states: x [N_tok, d_model] ~ N(0, 1),
    W_in [d_model, H(2dk + 2dv) + 2H] ~ N(0, 1 / d_model) (so the projections are
    about N(0, 1), like the mixer's inputs), W_o [H dv, d_model] ~ N(0, 1 / (H dv)),
    all bf16; the mixer's parameters (conv_w, A, b_alpha, norm_w, S0, cu_seqlens)
    drawn as for the prefill of `cfg`."""
    device = torch.device(device)
    base = make_prefill_inputs(cfg, device, seed)
    gen = torch.Generator(device=device)
    gen.manual_seed((cfg.seed if seed is None else seed) + 7919)
    H, dk, dv, N = cfg.H, cfg.dk, cfg.dv, cfg.total_tokens
    c_in = H * (2 * dk + 2 * dv) + 2 * H
    d = {key: base[key] for key in ("conv_w", "A", "b_alpha", "norm_w", "S0", "cu_seqlens")}
    d["x"] = _normal((N, d_model), gen, device).to(torch.bfloat16)
    d["w_in"] = _normal((d_model, c_in), gen, device, std=d_model ** -0.5).to(torch.bfloat16)
    d["w_o"] = _normal((H * dv, d_model), gen, device, std=(H * dv) ** -0.5).to(torch.bfloat16)
    return d
