"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module draws random numbers and shapes them into the workloads; it holds
none of the loss or log-probability arithmetic.  Every tensor is produced by a
seeded ``torch.Generator`` (fp32 master values, then rounded to nearest-even
into the working dtype).  Parity tests generate on the CPU, so the GPU path and
the oracle see the same bits; the benchmark may generate the same recipes
directly on the GPU (``device="cuda"``), which is faster for the 1 GB weights.

Recipes (N(mu, sigma): sigma is the standard deviation; "uniform in [a, b]" on
integers includes both ends):

* loss-only: policy = -2|N(0,1)|, old = policy + N(0,0.1), ref = policy + N(0,0.05),
  advantages N(0,1) per sequence (fp32), int8 prefix mask with lengths uniform in
  the given range;
* fused linear: X ~ N(0,1) [N,H], W ~ N(0,0.02) [V,H], Xref = X + N(0,0.01),
  Wref = W + N(0,0.002), optional bias ~ N(0,0.01), targets uniform in [0,V),
  advantages N(0,1) per sequence, prefix mask, and the N(0,0.1) noise that is
  added to the policy log-prob to make the behaviour log-probs (old_lp);
* reverse KL: student logits N(0,1) [bs, seq, V]; teacher logits independent
  N(0,1), or (``teacher_std`` given) student + N(0, teacher_std) for a teacher
  close to the student; mask = uniform(0,1) > 0.2 per token (as the model card's
  reverse-KL example draws it).

Seeds are ``0x5EED0000 + 16*workload + variant``.
"""
from __future__ import annotations

import torch

SEED_BASE = 0x5EED0000


def seed_for(workload: int, variant: int = 0) -> int:
    return SEED_BASE + 16 * workload + variant


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, seed: int, std: float = 1.0, mean: float = 0.0, device="cpu") -> torch.Tensor:
    x = torch.randn(tuple(shape), generator=_gen(seed, device), dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def randint(shape, lo: int, hi_inclusive: int, seed: int, device="cpu") -> torch.Tensor:
    return torch.randint(lo, hi_inclusive + 1, tuple(shape), generator=_gen(seed, device),
                         dtype=torch.int64, device=device)


def prefix_mask(lengths: torch.Tensor, T: int) -> torch.Tensor:
    """int8 [bs, T] mask whose row b has its first lengths[b] entries set."""
    pos = torch.arange(T, dtype=torch.int64, device=lengths.device).unsqueeze(0)
    return (pos < lengths.to(torch.int64).unsqueeze(1)).to(torch.int8)


def loss_inputs(bs: int, seq: int, dtype: torch.dtype, seed: int,
                len_lo: int = 64, len_hi: int = 1024, device="cpu") -> dict:
    """Log-prob inputs for the loss-only kernel."""
    s = int(seed)
    pol = normal((bs, seq), s + 1, device=device).abs_().mul_(-2.0)
    old = pol + normal((bs, seq), s + 2, std=0.1, device=device)
    ref = pol + normal((bs, seq), s + 3, std=0.05, device=device)
    adv = normal((bs,), s + 4, device=device)
    lens = randint((bs,), min(len_lo, seq), min(len_hi, seq), s + 5, device=device)
    return {
        "policy_lp": pol.to(dtype), "old_lp": old.to(dtype), "ref_lp": ref.to(dtype),
        "adv": adv, "mask": prefix_mask(lens, seq), "lengths": lens,
    }


def fused_inputs(bs: int, T: int, H: int, V: int, dtype: torch.dtype, seed: int, *,
                 bias: bool = False, len_lo: int = 1, len_hi: int | None = None,
                 fully_masked_last: bool = False, need_ref: bool = True, device="cpu") -> dict:
    """Inputs of the fused linear path.  ``old_noise`` is the N(0,0.1) term the
    caller adds to the policy log-prob to form old_lp."""
    s = int(seed)
    N = bs * T
    len_hi = T if len_hi is None else len_hi
    X32 = normal((N, H), s + 1, device=device)
    out = {"X": X32.to(dtype)}
    if need_ref:
        out["Xref"] = (X32 + normal((N, H), s + 3, std=0.01, device=device)).to(dtype)
    del X32
    W32 = normal((V, H), s + 2, std=0.02, device=device)
    out["W"] = W32.to(dtype, copy=True)  # a copy even for fp32: W32 becomes Wref below
    if need_ref:
        W32.add_(normal((V, H), s + 4, std=0.002, device=device))
        out["Wref"] = W32.to(dtype)
    else:
        out["Xref"] = None
        out["Wref"] = None
    del W32
    out["bias"] = normal((V,), s + 5, std=0.01, device=device).to(dtype) if bias else None
    out["targets"] = randint((N,), 0, V - 1, s + 6, device=device)
    out["adv"] = normal((bs,), s + 7, device=device)
    lens = randint((bs,), min(len_lo, T), min(len_hi, T), s + 8, device=device)
    if fully_masked_last and bs > 0:
        lens[bs - 1] = 0
    out["lengths"] = lens
    out["mask"] = prefix_mask(lens, T)
    out["old_noise"] = normal((N,), s + 9, std=0.1, device=device)
    return out


def reverse_kl_inputs(bs: int, seq: int, V: int, dtype: torch.dtype, seed: int, *,
                      teacher_std: float | None = None, device="cpu") -> dict:
    s = int(seed)
    student = normal((bs, seq, V), s + 1, device=device)
    if teacher_std is None:
        teacher = normal((bs, seq, V), s + 2, device=device)
    else:
        teacher = student + normal((bs, seq, V), s + 2, std=teacher_std, device=device)
    u = torch.rand((bs, seq), generator=_gen(s + 3, device), device=device)
    return {"student": student.to(dtype), "teacher": teacher.to(dtype), "mask": (u > 0.2).to(torch.uint8)}


# Reverse-KL workloads: the model card's example shape (bs=4, seq=256,
# V=248320) and the fused path's vocabulary at a loss-only-sized batch.
RKL_WORKLOADS = {
    0: dict(bs=2, seq=8, V=1000, dtype=torch.bfloat16),
    1: dict(bs=4, seq=256, V=248320, dtype=torch.bfloat16),
    2: dict(bs=16, seq=128, V=128256, dtype=torch.bfloat16),
}


# The workloads, by number, as (kind, shape) records.
WORKLOADS = {
    0: dict(kind="fused", bs=2, T=16, H=64, V=512, dtype=torch.bfloat16, len_lo=1, len_hi=16,
            eps_lo=0.2, eps_hi=0.28, beta=0.04),
    1: dict(kind="loss", bs=16, seq=1024, len_lo=64, len_hi=1024, eps_lo=0.2, eps_hi=0.28,
            beta=0.04),
    2: dict(kind="fused", bs=1, T=1024, H=4096, V=128256, dtype=torch.bfloat16, len_lo=256,
            len_hi=1024, eps_lo=0.2, eps_hi=0.28, beta=0.04),
    3: dict(kind="fused", bs=4, T=1024, H=4096, V=128256, dtype=torch.float16, bias=True,
            len_lo=256, len_hi=1024, eps_lo=0.2, eps_hi=0.28, beta=0.04),
    4: dict(kind="fused", bs=8, T=1024, H=4096, V=128256, dtype=torch.bfloat16, len_lo=1,
            len_hi=1024, fully_masked_last=True, eps_lo=0.2, eps_hi=0.28, beta=0.04),
    5: dict(kind="fused", bs=8, T=1024, H=4000, V=152064, dtype=torch.bfloat16, len_lo=1,
            len_hi=1024, fully_masked_last=True, eps_lo=0.2, eps_hi=0.28, beta=0.04),
}
