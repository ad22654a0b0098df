"""Seeded synthetic inputs for the FP8-AMAX linear layer (shared by tests, the
benchmark and the CPU oracle checks).

This module draws random tensors and nothing else: it holds none of the
method's arithmetic (no amax, no bias, no cast, no matmul), so the CUDA path and
the oracle can both read the bytes it makes without sharing any computation.

Workloads (layer shapes of the models the review page "Training and inference
of large language models using 8-bit floating point" trains and runs —
GPT 111M up to Llama 2 70B, "Abstract" and "Main findings"):
  c0  one forward linear 256->256, 128 tokens, FP32 output
  c1  GPT-111M shapes, d_model 768, d_ff 3072, 8192 tokens (4 x 2048)
  c2  Llama-2-7B SwiGLU MLP, d 4096, ffn 11008, 4096 tokens, outlier channels
  c3  Llama-2-70B projections, d 8192, ffn 28672, GQA QKV 8192->10240, 8192 tokens,
      Student-t(3) activations, gradient scales 1e-7 .. 1e-2
  c4  amax + bias + cast sweep, 2^16 .. 2^30 elements, BF16 and FP32

Seeds are ``1000 * config + 10 * linear + tensor (+ 100000 * step)`` with a
torch Generator on the requested device; the same call always returns the same
bytes on the same device type.
"""
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

X_ID, W_ID, DY_ID = 0, 1, 2


@dataclass(frozen=True)
class Linear:
    name: str
    in_features: int
    out_features: int
    sigma_dy: float


@dataclass(frozen=True)
class LayerConfig:
    cid: int
    name: str
    tokens: int
    linears: Tuple[Linear, ...]
    x_kind: str                      # "normal" | "outlier" | "student_t"
    sigma_w: float = 0.02
    margins: Tuple[int, ...] = (0,)
    out_dtype: torch.dtype = torch.bfloat16
    passes: Tuple[str, ...] = ("fwd", "dgrad", "wgrad")

    def flops_per_step(self) -> int:
        return sum(2 * self.tokens * l.in_features * l.out_features * len(self.passes)
                   for l in self.linears)


C0 = LayerConfig(0, "single-linear-256x256-t128", 128,
                 (Linear("proj", 256, 256, 0.0),), "normal",
                 out_dtype=torch.float32, passes=("fwd",))
C1 = LayerConfig(1, "gpt-111m-d768-ff3072-t8192", 8192,
                 (Linear("qkv_out", 768, 768, 1e-4),
                  Linear("mlp_up", 768, 3072, 1e-4),
                  Linear("mlp_down", 3072, 768, 1e-4)), "normal")
C2 = LayerConfig(2, "llama2-7b-mlp-d4096-ffn11008-t4096", 4096,
                 (Linear("gate", 4096, 11008, 1e-5),
                  Linear("up", 4096, 11008, 1e-5),
                  Linear("down", 11008, 4096, 1e-5)), "outlier", margins=(0, 1))
C3 = LayerConfig(3, "llama2-70b-proj-d8192-ffn28672-t8192", 8192,
                 (Linear("qkv_gqa", 8192, 10240, 1e-7),
                  Linear("gate", 8192, 28672, 1e-5),
                  Linear("up", 8192, 28672, 1e-3),
                  Linear("down", 28672, 8192, 1e-2)), "student_t")
CONFIGS = {0: C0, 1: C1, 2: C2, 3: C3}

SWEEP_SIZES = [1 << k for k in range(16, 31, 2)]          # 2^16 .. 2^30
SWEEP_SIGMAS = (1e-6, 1.0, 1e3)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device).type)
    g.manual_seed(int(seed))
    return g


def seed_for(cid: int, linear: int, tensor: int, step: int = 0) -> int:
    return 1000 * cid + 10 * linear + tensor + 100000 * step


def _x(cfg: LayerConfig, n_in: int, seed: int, device, dtype) -> torch.Tensor:
    g = _gen(seed, device)
    shape = (cfg.tokens, n_in)
    if cfg.x_kind == "normal":
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    elif cfg.x_kind == "outlier":
        # N(0,1) with 8 channels, chosen by a seeded permutation, scaled x50
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        ch = torch.randperm(n_in, generator=g, device=device)[:8]
        x[:, ch] *= 50.0
    elif cfg.x_kind == "student_t":
        # Student-t with 3 degrees of freedom: Z / sqrt(chi2_3 / 3)
        z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        c = torch.zeros(shape, device=device, dtype=torch.float32)
        for _ in range(3):
            c += torch.randn(shape, generator=g, device=device, dtype=torch.float32).square_()
        x = z.div_(c.div_(3.0).sqrt_())
        del c
    else:
        raise ValueError(cfg.x_kind)
    return x.to(dtype)


def linear_inputs(cid: int, li: int, step: int = 0, device="cpu",
                  dtype: torch.dtype = torch.bfloat16):
    """(X [T,in], W [out,in], dY [T,out] or None) for linear ``li`` of config ``cid``."""
    cfg = CONFIGS[cid]
    lin = cfg.linears[li]
    x = _x(cfg, lin.in_features, seed_for(cid, li, X_ID, step), device, dtype)
    g = _gen(seed_for(cid, li, W_ID, step), device)
    w = (torch.randn((lin.out_features, lin.in_features), generator=g, device=device,
                     dtype=torch.float32) * cfg.sigma_w).to(dtype)
    dy = None
    if "dgrad" in cfg.passes or "wgrad" in cfg.passes:
        g = _gen(seed_for(cid, li, DY_ID, step), device)
        dy = (torch.randn((cfg.tokens, lin.out_features), generator=g, device=device,
                          dtype=torch.float32) * lin.sigma_dy).to(dtype)
    return x, w, dy


SWEEP_KINDS = ("normal", "zeros", "spike_zeros", "spike_normal", "exact_pow2")


def sweep_tensor(n: int, dtype: torch.dtype, kind: str = "normal", sigma: float = 1.0,
                 seed: int = 4000, device="cpu", fmt_max: Optional[float] = None) -> torch.Tensor:
    """One tensor of the memory-bound amax + bias + cast sweep.

    kinds: "normal" N(0, sigma); "zeros"; "spike_zeros" zeros plus one 1e4 at a
    seeded index; "spike_normal" N(0,1) plus one 1e4 spike; "exact_pow2"
    values +-fmt_max * 2^-k with k seeded in [0, 20] (``fmt_max`` is passed in
    by the caller: 448 or 57344, the formats' largest finite values)."""
    g = _gen(seed, device)
    if kind == "normal":
        return (torch.randn(n, generator=g, device=device, dtype=torch.float32) * sigma).to(dtype)
    if kind == "zeros":
        return torch.zeros(n, device=device, dtype=dtype)
    if kind in ("spike_zeros", "spike_normal"):
        if kind == "spike_zeros":
            x = torch.zeros(n, device=device, dtype=torch.float32)
        else:
            x = torch.randn(n, generator=g, device=device, dtype=torch.float32)
        idx = int(torch.randint(0, n, (1,), generator=g, device=device).item())
        x[idx] = 1e4
        return x.to(dtype)
    if kind == "exact_pow2":
        assert fmt_max is not None
        k = torch.randint(0, 21, (n,), generator=g, device=device, dtype=torch.int32)
        s = torch.randint(0, 2, (n,), generator=g, device=device, dtype=torch.int32)
        # 2^-k built from its bit pattern (exact), times +-fmt_max (exact)
        p = ((127 - k) << 23).view(torch.float32)
        return (p * fmt_max * (1 - 2 * s).to(torch.float32)).to(dtype)
    raise ValueError(kind)
