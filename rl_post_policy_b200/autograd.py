"""Autograd-aware wrappers of the library's entry points.

* ``bnpo_loss_autograd`` / ``grpo_loss_autograd`` -- the "autograd-aware" entry
  points of the "Geometric-AI Kernels" model card ("Entry points"): the same
  fused forward+backward kernel (pl_loss_ex) registered with autograd, so
  ``loss.backward()`` works.  The forward keeps dLoss/dlp; the backward scales
  it by the incoming gradient with pl_scale (a device scalar, no host sync).
* ``reverse_kl_autograd`` -- the card's autograd-aware reverse-KL entry point:
  pl_reverse_kl's fused forward + student-logit gradient, scaled by the
  incoming gradient in the backward (pl_scale).
* ``fused_linear_grpo_loss`` -- the fused linear GRPO / BNPO loss of "Add
  SM100 CuTe DSL GRPO fast path" ("Summary"): the forward is one
  pl_fused_linear_grpo_temp call that also produces dX, dW and dbias (the
  chunked path computes them with the loss); the backward scales them by the
  incoming gradient (pl_scale).
* ``fused_selective_logprob`` -- the fused-linear selective log-prob autograd
  path of "Add SM100 CuTe DSL GRPO fast path" (Liger-Kernel PR #1363,
  "Summary"): forward = pl_fused_selective_logprob (log-probs), backward = the
  same entry point with the incoming dL/dlogp (dX, dW, dbias).

Argument marshalling only: every arithmetic step runs in libpl.so's kernels.
Workspaces are cached per (entry point, device, size) and zero-filled once, as
the C ABI requires; calls that share one must be ordered on one stream.
"""
from __future__ import annotations

import torch

from . import binding as pl

_ws_cache: dict = {}


def _workspace(kind: str, nbytes: int, device) -> torch.Tensor:
    """A zero-filled workspace per entry point (`kind`), device and size: entry
    points lay their workspaces out differently, so they never share one."""
    key = (kind, torch.device(device).index, nbytes)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


class _PolicyLoss(torch.autograd.Function):
    @staticmethod
    def forward(ctx, policy_lp, old_lp, ref_lp, adv, mask, eps_lo, eps_hi, beta, reduction, two_sided):
        bs, seq = policy_lp.shape
        dtype = policy_lp.dtype
        mode = pl.dtype_mode(dtype) | reduction | (pl.PL_CLIP_TWO_SIDED if two_sided else 0)
        lp = policy_lp.detach().contiguous()
        grad = torch.empty_like(lp)
        loss = torch.empty(1, dtype=torch.float32, device=lp.device)
        wsb = pl.pl_loss_workspace_bytes(bs, seq)
        ws = _workspace("loss", wsb, lp.device)
        adv_c = adv.detach().to(torch.float32).contiguous()
        pl.check(pl.pl_loss_ex(lp, old_lp.detach().contiguous(), None if beta == 0 else ref_lp.detach().contiguous(),
                               adv_c, mask.detach().contiguous(), bs, seq, eps_lo, eps_hi, beta, mode, loss,
                               grad, None, None, ws, wsb), "pl_loss_ex")
        ctx.save_for_backward(grad)
        ctx.mode = pl.dtype_mode(dtype)
        return loss[0]

    @staticmethod
    def backward(ctx, grad_out):
        (grad,) = ctx.saved_tensors
        g = grad.clone()
        scale = grad_out.detach().to(torch.float32).reshape(1).contiguous()
        pl.check(pl.pl_scale(g, g.numel(), ctx.mode, scale), "pl_scale")
        return g, None, None, None, None, None, None, None, None, None


def bnpo_loss_autograd(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0,
                       two_sided=False):
    """BNPO loss (global token mean) with autograd support."""
    return _PolicyLoss.apply(policy_lp, old_lp, ref_lp, adv, mask, float(epsilon), float(epsilon_high),
                             float(beta), pl.PL_BNPO, bool(two_sided))


def grpo_loss_autograd(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0,
                       two_sided=False):
    """GRPO loss (per-sequence mean, then batch mean) with autograd support."""
    return _PolicyLoss.apply(policy_lp, old_lp, ref_lp, adv, mask, float(epsilon), float(epsilon_high),
                             float(beta), pl.PL_GRPO, bool(two_sided))


class _ReverseKL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, student, teacher, mask):
        V = student.shape[-1]
        N = student.numel() // V if V else 0
        s = student.detach().contiguous()
        t = teacher.detach().to(s.dtype).contiguous()
        m = mask.detach().to(torch.uint8).contiguous() if mask is not None else None
        grad = torch.empty_like(s)
        loss = torch.empty(1, dtype=torch.float32, device=s.device)
        pl.check(pl.pl_reverse_kl(s, t, m, N, V, pl.dtype_mode(s.dtype), loss, grad, None, None, None, 0),
                 "pl_reverse_kl")
        ctx.save_for_backward(grad)
        ctx.mode = pl.dtype_mode(s.dtype)
        return loss[0]

    @staticmethod
    def backward(ctx, grad_out):
        (grad,) = ctx.saved_tensors
        g = grad.clone()
        scale = grad_out.detach().to(torch.float32).reshape(1).contiguous()
        pl.check(pl.pl_scale(g, g.numel(), ctx.mode, scale), "pl_scale")
        return g, None, None


def reverse_kl_autograd(student_logits, teacher_logits, completions_mask=None):
    """Masked mean over rows of KL(softmax(student) || softmax(teacher)), differentiable
    in the student logits (shape (..., V); mask of the leading shape, or None)."""
    return _ReverseKL.apply(student_logits, teacher_logits, completions_mask)


class _FusedLinearGRPO(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, bias, targets, Xref, Wref, old_lp, adv, mask, eps_lo, eps_hi, beta, reduction,
                two_sided, temperature, chunk_rows):
        bs, T = mask.shape
        N, H = X.shape
        V = W.shape[0]
        mode = (pl.dtype_mode(X.dtype) | reduction | (pl.PL_CLIP_TWO_SIDED if two_sided else 0) |
                (pl.PL_CHUNK_ROWS(chunk_rows) if chunk_rows else 0))
        Xc, Wc = X.detach().contiguous(), W.detach().contiguous()
        bc = bias.detach().contiguous() if bias is not None else None
        need_x, need_w, need_b = ctx.needs_input_grad[0], ctx.needs_input_grad[1], ctx.needs_input_grad[2]
        dX = torch.empty_like(Xc) if need_x else None
        dW = torch.empty_like(Wc) if need_w else None
        db = torch.empty_like(bc) if (need_b and bc is not None) else None
        loss = torch.empty(1, dtype=torch.float32, device=X.device)
        ref_x = Xref.detach().contiguous() if beta != 0 else None
        ref_w = Wref.detach().contiguous() if beta != 0 else None
        wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, int(dW is not None), int(db is not None))
        ws = _workspace("fused", wsb, X.device)
        pl.check(pl.pl_fused_linear_grpo_temp(Xc, Wc, bc, targets.detach().to(torch.int64).contiguous(), ref_x,
                                              ref_w, old_lp.detach().to(torch.float32).contiguous(),
                                              adv.detach().to(torch.float32).contiguous(),
                                              mask.detach().contiguous(), bs, T, H, V, eps_lo, eps_hi, beta,
                                              temperature, mode, loss, dX, dW, db, None, None, None, ws, wsb),
                 "pl_fused_linear_grpo_temp")
        ctx.save_for_backward(dX, dW, db)
        return loss[0]

    @staticmethod
    def backward(ctx, grad_out):
        dX, dW, db = ctx.saved_tensors
        scale = grad_out.detach().to(torch.float32).reshape(1).contiguous()
        out = []
        for g in (dX, dW, db):
            if g is None:
                out.append(None)
                continue
            g = g.clone()
            pl.check(pl.pl_scale(g, g.numel(), pl.dtype_mode(g.dtype), scale), "pl_scale")
            out.append(g)
        return (*out, None, None, None, None, None, None, None, None, None, None, None, None, None)


def fused_linear_grpo_loss(X, W, targets, old_lp, adv, mask, bias=None, Xref=None, Wref=None, epsilon=0.2,
                           epsilon_high=0.2, beta=0.0, reduction="grpo", two_sided=False, temperature=1.0,
                           chunk_rows=None):
    """GRPO (or BNPO) loss of the sampled tokens' log-probs under log_softmax((X W^T + bias) / temperature),
    with the reference model's (Xref Wref^T / temperature) in the KL term when beta != 0; differentiable
    in X, W and bias.  X [N, H], W [V, H], targets [N], old_lp [N] (or [bs, T]), adv [bs], mask [bs, T]."""
    red = {"grpo": pl.PL_GRPO, "bnpo": pl.PL_BNPO}[reduction] if isinstance(reduction, str) else int(reduction)
    return _FusedLinearGRPO.apply(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, float(epsilon),
                                  float(epsilon_high), float(beta), red, bool(two_sided), float(temperature),
                                  chunk_rows)


class _SelectiveLogprob(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, bias, targets, chunk_rows):
        N, H = X.shape
        V = W.shape[0]
        mode = pl.dtype_mode(X.dtype) | (pl.PL_CHUNK_ROWS(chunk_rows) if chunk_rows else 0)
        Xc, Wc = X.detach().contiguous(), W.detach().contiguous()
        bc = bias.detach().contiguous() if bias is not None else None
        tg = targets.detach().to(torch.int64).contiguous()
        logp = torch.empty(N, dtype=torch.float32, device=X.device)
        wsb = pl.pl_fused_selective_logprob_workspace_bytes(N, H, V, mode, 1, int(bc is not None))
        ws = _workspace("selective", wsb, X.device)
        pl.check(pl.pl_fused_selective_logprob(Xc, Wc, bc, tg, N, H, V, mode, None, logp, None, None, None,
                                               ws, wsb), "pl_fused_selective_logprob")
        ctx.save_for_backward(Xc, Wc, bc, tg)
        ctx.mode, ctx.has_bias = mode, bc is not None
        return logp

    @staticmethod
    def backward(ctx, grad_logp):
        Xc, Wc, bc, tg = ctx.saved_tensors
        N, H = Xc.shape
        V = Wc.shape[0]
        need_x, need_w, need_b = ctx.needs_input_grad[0], ctx.needs_input_grad[1], ctx.needs_input_grad[2]
        dX = torch.empty_like(Xc) if need_x else None
        dW = torch.empty_like(Wc) if need_w else None
        db = torch.empty_like(bc) if (need_b and bc is not None) else None
        if dX is None and dW is None and db is None:
            return None, None, None, None, None
        g = grad_logp.detach().to(torch.float32).contiguous()
        wsb = pl.pl_fused_selective_logprob_workspace_bytes(N, H, V, ctx.mode, int(dW is not None),
                                                            int(db is not None))
        ws = _workspace("selective", wsb, Xc.device)
        pl.check(pl.pl_fused_selective_logprob(Xc, Wc, bc, tg, N, H, V, ctx.mode, g, None, dX, dW, db, ws,
                                               wsb), "pl_fused_selective_logprob")
        return dX, dW, db, None, None


def fused_selective_logprob(X, W, targets, bias=None, chunk_rows=None):
    """log_softmax(X W^T + bias)[targets] per row (fp32), differentiable in X, W and bias."""
    return _SelectiveLogprob.apply(X, W, bias, targets, chunk_rows)
