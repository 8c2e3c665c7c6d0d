"""Data-parallel GRPO / BNPO across torch.distributed ranks: the fused linear
step (``dp_fused_linear_grpo``) and the loss-only step (``dp_policy_loss``).

The path shards by sequences: each rank holds its own rows (X, Xref, targets,
old_lp, adv, mask) and a replica of the policy weight W (and Wref, bias).  One
step of ``dp_fused_linear_grpo``:

1. the rank's fused forward + backward (``pl_fused_linear_grpo``) on its shard,
   normalised by the shard's own count: the valid-token count n_l for BNPO, the
   sequence count bs_l for GRPO ("Geometric-AI Kernels" card, sections "BNPO
   Loss" and "GRPO Loss");
2. one all-reduce (sum) of that count, an int64 device scalar;
3. the rank's share f_l = max(count_l, 1) / max(count, 1) (``pl_count_ratio``,
   on the device).  loss_l * f_l is the rank's exact part of the global loss:
   for BNPO, the sum of its terms over max(n, 1); for GRPO, its sequences'
   means over the global bs.  The same factor scales its dX, dW and dbias
   (``pl_scale``);
4. an all-reduce (sum) of the loss, dW and dbias.  dX stays with its rows.

Step 4 is the gradient all-reduce of data-parallel training, on NCCL over
NVLink; it is the path's only exchange.  The host never waits: every count,
factor and scale stays on the device.

``dp_policy_loss`` is the same sequence for the loss-only kernel on per-token
log-probs: the rank's ``pl_loss_ex`` normalised by its own count, the count
all-reduce, the share f_l applied to the rank's loss and gradient, and an
all-reduce of the loss alone.  The gradient rows stay with their rank, so the
loss-only step exchanges two scalars.

Argument marshalling and collectives only; the arithmetic runs in libpl.so.  The
per-rank operations are grouped in ``LibraryOps`` so the host-side sequence can
be exercised on CPU ranks with other implementations of the three operations.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as pl


class LibraryOps:
    """The three per-rank operations, run by libpl.so on the rank's GPU."""

    def __init__(self):
        self._ws = {}

    def _workspace(self, kind, nbytes, device):
        # one zero-filled workspace per entry point, device and size (calls that
        # share one are stream-ordered)
        key = (kind, torch.device(device).index, nbytes)
        if key not in self._ws:
            self._ws[key] = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        return self._ws[key]

    def local_step(self, X, W, bias, targets, Xref, Wref, old_lp, adv, mask, eps_lo, eps_hi, beta,
                   reduction, temperature=1.0, chunk_rows=None, want=("dX", "dW", "dbias")):
        bs, T = mask.shape
        N, H = X.shape
        V = W.shape[0]
        dev = X.device
        mode = pl.dtype_mode(X.dtype) | reduction | (pl.PL_CHUNK_ROWS(chunk_rows) if chunk_rows else 0)
        dX = torch.empty_like(X) if "dX" in want else None
        dW = torch.empty_like(W) if "dW" in want else None
        db = torch.empty_like(bias) if (bias is not None and "dbias" in want) else None
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        nv = torch.empty(1, dtype=torch.int64, device=dev)
        wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, int(dW is not None), int(db is not None))
        ws = self._workspace("fused", wsb, dev)
        pl.check(pl.pl_fused_linear_grpo_temp(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, bs, T, H, V,
                                              eps_lo, eps_hi, beta, temperature, mode, loss, dX, dW, db, None,
                                              None, nv, ws, wsb), "pl_fused_linear_grpo_temp")
        return {"loss": loss, "dX": dX, "dW": dW, "dbias": db, "n_valid": nv}

    def local_loss(self, policy_lp, old_lp, ref_lp, adv, mask, eps_lo, eps_hi, beta, reduction, two_sided=False,
                   want_grad=True):
        bs, seq = mask.shape
        dev = policy_lp.device
        mode = (pl.dtype_mode(policy_lp.dtype) | reduction | (pl.PL_CLIP_TWO_SIDED if two_sided else 0) |
                (pl.PL_ADV_LP_DTYPE if adv.dtype == policy_lp.dtype and adv.dtype != torch.float32 else 0))
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        grad = torch.empty_like(policy_lp) if want_grad else None
        nv = torch.empty(1, dtype=torch.int64, device=dev)
        wsb = pl.pl_loss_workspace_bytes(bs, seq)
        ws = self._workspace("loss", wsb, dev)
        pl.check(pl.pl_loss_ex(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode, loss,
                               grad, nv, None, ws, wsb), "pl_loss_ex")
        return {"loss": loss, "grad": grad, "n_valid": nv}

    def ratio(self, local, total):
        f = torch.empty(1, dtype=torch.float32, device=local.device)
        pl.check(pl.pl_count_ratio(local, total, f), "pl_count_ratio")
        return f

    def scale(self, t, factor):
        pl.check(pl.pl_scale(t, t.numel(), pl.dtype_mode(t.dtype), factor), "pl_scale")


def dp_fused_linear_grpo(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, *, eps_lo=0.2, eps_hi=0.2,
                         beta=0.0, reduction=pl.PL_GRPO, temperature=1.0, chunk_rows=None,
                         want=("dX", "dW", "dbias"), group=None, ops=None) -> dict:
    """One data-parallel step over the ranks of ``group`` (every rank calls it with
    its own rows).  Returns the global loss (device fp32 [1], identical on every
    rank), the rank's dX rows, the global dW / dbias (identical on every rank), and
    the global count (valid tokens for BNPO, sequences for GRPO)."""
    ops = ops or _default_ops()
    bs_l = mask.shape[0]
    out = ops.local_step(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, eps_lo, eps_hi, beta, reduction,
                         temperature=temperature, chunk_rows=chunk_rows, want=want)
    dev = out["loss"].device
    if reduction == pl.PL_BNPO:
        count = out["n_valid"].reshape(1).to(torch.int64)
    else:
        count = torch.full((1,), bs_l, dtype=torch.int64, device=dev)
    total = count.clone()
    dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    f = ops.ratio(count, total)
    for k in ("loss", "dX", "dW", "dbias"):
        if out.get(k) is not None:
            ops.scale(out[k], f)
    for k in ("loss", "dW", "dbias"):
        if out.get(k) is not None:
            dist.all_reduce(out[k], op=dist.ReduceOp.SUM, group=group)
    return {"loss": out["loss"], "dX": out["dX"], "dW": out["dW"], "dbias": out["dbias"], "count": total}


def dp_policy_loss(policy_lp, old_lp, ref_lp, adv, mask, *, eps_lo=0.2, eps_hi=0.2, beta=0.0,
                   reduction=pl.PL_GRPO, two_sided=False, want_grad=True, group=None, ops=None) -> dict:
    """One data-parallel loss-only step over the ranks of ``group``; every rank
    passes its own sequences (policy_lp, old_lp, ref_lp [bs_l, seq], adv [bs_l],
    mask [bs_l, seq]).  Returns the global loss (device fp32 [1], identical on
    every rank), the rank's gradient rows d loss / d policy_lp, and the global
    count (valid tokens for BNPO, sequences for GRPO)."""
    ops = ops or _default_ops()
    bs_l = mask.shape[0]
    out = ops.local_loss(policy_lp, old_lp, ref_lp, adv, mask, eps_lo, eps_hi, beta, reduction,
                         two_sided=two_sided, want_grad=want_grad)
    dev = out["loss"].device
    if reduction == pl.PL_BNPO:
        count = out["n_valid"].reshape(1).to(torch.int64)
    else:
        count = torch.full((1,), bs_l, dtype=torch.int64, device=dev)
    total = count.clone()
    dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    f = ops.ratio(count, total)
    ops.scale(out["loss"], f)
    if out.get("grad") is not None:
        ops.scale(out["grad"], f)
    dist.all_reduce(out["loss"], op=dist.ReduceOp.SUM, group=group)
    return {"loss": out["loss"], "grad": out["grad"], "count": total}


_ops = None


def _default_ops():
    global _ops
    if _ops is None:
        _ops = LibraryOps()
    return _ops
