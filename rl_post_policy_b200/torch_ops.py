"""The library's entry points as PyTorch custom operators (``torch.library``).

Registered under ``torch.ops.rl_post_policy_b200``:

* ``policy_loss(policy_lp, old_lp, ref_lp?, adv, mask, eps_lo, eps_hi, beta,
  reduction, two_sided) -> (loss, dloss_dlp)`` -- pl_loss_ex, the fused
  forward+backward loss kernel;
* ``reverse_kl(student, teacher, mask?) -> (loss, dloss_dstudent)`` --
  pl_reverse_kl with the student gradient;
* ``selective_logprob(X, W, bias?, targets, chunk_rows) -> logp`` and
  ``selective_logprob_backward(X, W, bias?, targets, grad_logp, chunk_rows,
  need_x, need_w, need_b) -> (dX, dW, dbias)`` -- pl_fused_selective_logprob;
* ``fused_linear_grpo(X, W, bias?, targets, Xref?, Wref?, old_lp, adv, mask,
  ..., need_x, need_w, need_b) -> (loss, dX, dW, dbias)`` --
  pl_fused_linear_grpo_temp, loss and gradients in one call;
* ``scale(x, factor) -> x * factor`` -- pl_scale, for the backward passes.

Each operator has a shape function (so tracing with FakeTensors, as
``torch.compile`` does, needs no GPU work) and the autograd formulas of the
"Entry points" section of the "Geometric-AI Kernels" model card: the loss
kernels return dLoss/dinput with the loss, and the backward scales it by the
incoming gradient.  The functions at the bottom (``bnpo_loss``, ``grpo_loss``,
``reverse_kl_loss``, ``selective_logprob``, ``fused_linear_grpo_loss``) are the
user-facing forms.

Argument marshalling only: every arithmetic step runs in libpl.so.  Gradients
that are not needed come back from ``selective_logprob_backward`` and
``fused_linear_grpo`` as empty tensors (an operator cannot return None).
"""
from __future__ import annotations

from typing import Optional

import torch
from torch import Tensor

from . import binding as pl
from .autograd import _workspace

_NS = "rl_post_policy_b200"


# ------------------------------------------------------------------ scale
@torch.library.custom_op(f"{_NS}::scale", mutates_args=())
def scale(x: Tensor, factor: Tensor) -> Tensor:
    y = x.detach().contiguous().clone()
    f = factor.detach().to(torch.float32).reshape(1).contiguous()
    pl.check(pl.pl_scale(y, y.numel(), pl.dtype_mode(y.dtype), f), "pl_scale")
    return y


@scale.register_fake
def _(x, factor):
    return torch.empty_like(x, memory_format=torch.contiguous_format)


# ------------------------------------------------------------------ policy loss
@torch.library.custom_op(f"{_NS}::policy_loss", mutates_args=())
def policy_loss(policy_lp: Tensor, old_lp: Tensor, ref_lp: Optional[Tensor], adv: Tensor, mask: Tensor,
                eps_lo: float, eps_hi: float, beta: float, reduction: int,
                two_sided: bool) -> tuple[Tensor, Tensor]:
    bs, seq = policy_lp.shape
    lp = policy_lp.detach().contiguous()
    mode = pl.dtype_mode(lp.dtype) | int(reduction) | (pl.PL_CLIP_TWO_SIDED if two_sided else 0)
    grad = torch.empty_like(lp)
    loss = torch.empty((), dtype=torch.float32, device=lp.device)
    wsb = pl.pl_loss_workspace_bytes(bs, seq)
    ws = _workspace("loss", wsb, lp.device)
    ref = None if beta == 0.0 or ref_lp is None else ref_lp.detach().contiguous()
    pl.check(pl.pl_loss_ex(lp, old_lp.detach().contiguous(), ref, adv.detach().to(torch.float32).contiguous(),
                           mask.detach().contiguous(), bs, seq, eps_lo, eps_hi, beta, mode, loss, grad, None,
                           None, ws, wsb), "pl_loss_ex")
    return loss, grad


@policy_loss.register_fake
def _(policy_lp, old_lp, ref_lp, adv, mask, eps_lo, eps_hi, beta, reduction, two_sided):
    return (policy_lp.new_empty((), dtype=torch.float32),
            torch.empty_like(policy_lp, memory_format=torch.contiguous_format))


def _policy_loss_setup(ctx, inputs, output):
    ctx.save_for_backward(output[1])


def _policy_loss_backward(ctx, grad_loss, grad_grad):
    (g,) = ctx.saved_tensors
    return scale(g, grad_loss), None, None, None, None, None, None, None, None, None


policy_loss.register_autograd(_policy_loss_backward, setup_context=_policy_loss_setup)


# ------------------------------------------------------------------ reverse KL
@torch.library.custom_op(f"{_NS}::reverse_kl", mutates_args=())
def reverse_kl(student: Tensor, teacher: Tensor, mask: Optional[Tensor]) -> tuple[Tensor, Tensor]:
    V = student.shape[-1]
    N = student.numel() // V if V else 0
    s = student.detach().contiguous()
    t = teacher.detach().to(s.dtype).contiguous()
    m = mask.detach().to(torch.uint8).contiguous() if mask is not None else None
    grad = torch.empty_like(s)
    loss = torch.empty((), dtype=torch.float32, device=s.device)
    pl.check(pl.pl_reverse_kl(s, t, m, N, V, pl.dtype_mode(s.dtype), loss, grad, None, None, None, 0),
             "pl_reverse_kl")
    return loss, grad


@reverse_kl.register_fake
def _(student, teacher, mask):
    return (student.new_empty((), dtype=torch.float32),
            torch.empty_like(student, memory_format=torch.contiguous_format))


def _reverse_kl_setup(ctx, inputs, output):
    ctx.save_for_backward(output[1])


def _reverse_kl_backward(ctx, grad_loss, grad_grad):
    (g,) = ctx.saved_tensors
    return scale(g, grad_loss), None, None


reverse_kl.register_autograd(_reverse_kl_backward, setup_context=_reverse_kl_setup)


# ------------------------------------------------------------------ selective log-prob
def _sl_mode(X: Tensor, chunk_rows: int) -> int:
    return pl.dtype_mode(X.dtype) | (pl.PL_CHUNK_ROWS(chunk_rows) if chunk_rows else 0)


@torch.library.custom_op(f"{_NS}::selective_logprob", mutates_args=())
def selective_logprob_op(X: Tensor, W: Tensor, bias: Optional[Tensor], targets: Tensor, chunk_rows: int) -> Tensor:
    N, H = X.shape
    V = W.shape[0]
    mode = _sl_mode(X, chunk_rows)
    Xc, Wc = X.detach().contiguous(), W.detach().contiguous()
    bc = bias.detach().contiguous() if bias is not None else None
    logp = torch.empty(N, dtype=torch.float32, device=X.device)
    wsb = pl.pl_fused_selective_logprob_workspace_bytes(N, H, V, mode, 1, int(bc is not None))
    ws = _workspace("selective", wsb, X.device)
    pl.check(pl.pl_fused_selective_logprob(Xc, Wc, bc, targets.detach().to(torch.int64).contiguous(), N, H, V,
                                           mode, None, logp, None, None, None, ws, wsb),
             "pl_fused_selective_logprob")
    return logp


@selective_logprob_op.register_fake
def _(X, W, bias, targets, chunk_rows):
    return X.new_empty((X.shape[0],), dtype=torch.float32)


@torch.library.custom_op(f"{_NS}::selective_logprob_backward", mutates_args=())
def selective_logprob_backward(X: Tensor, W: Tensor, bias: Optional[Tensor], targets: Tensor, grad_logp: Tensor,
                               chunk_rows: int, need_x: bool, need_w: bool,
                               need_b: bool) -> tuple[Tensor, Tensor, Tensor]:
    N, H = X.shape
    V = W.shape[0]
    mode = _sl_mode(X, chunk_rows)
    Xc, Wc = X.detach().contiguous(), W.detach().contiguous()
    bc = bias.detach().contiguous() if bias is not None else None
    dX = torch.empty_like(Xc) if need_x else Xc.new_empty((0,))
    dW = torch.empty_like(Wc) if need_w else Wc.new_empty((0,))
    db = torch.empty_like(bc) if (need_b and bc is not None) else Xc.new_empty((0,))
    if need_x or need_w or (need_b and bc is not None):
        g = grad_logp.detach().to(torch.float32).contiguous()
        wsb = pl.pl_fused_selective_logprob_workspace_bytes(N, H, V, mode, int(need_w),
                                                            int(need_b and bc is not None))
        ws = _workspace("selective", wsb, X.device)
        pl.check(pl.pl_fused_selective_logprob(Xc, Wc, bc, targets.detach().to(torch.int64).contiguous(), N, H,
                                               V, mode, g, None, dX if need_x else None,
                                               dW if need_w else None,
                                               db if (need_b and bc is not None) else None, ws, wsb),
                 "pl_fused_selective_logprob")
    return dX, dW, db


@selective_logprob_backward.register_fake
def _(X, W, bias, targets, grad_logp, chunk_rows, need_x, need_w, need_b):
    dX = torch.empty_like(X, memory_format=torch.contiguous_format) if need_x else X.new_empty((0,))
    dW = torch.empty_like(W, memory_format=torch.contiguous_format) if need_w else W.new_empty((0,))
    db = (torch.empty_like(bias, memory_format=torch.contiguous_format) if (need_b and bias is not None)
          else X.new_empty((0,)))
    return dX, dW, db


def _sl_setup(ctx, inputs, output):
    X, W, bias, targets, chunk_rows = inputs
    ctx.save_for_backward(X, W, bias, targets)
    ctx.chunk_rows = chunk_rows
    ctx.has_bias = bias is not None


def _sl_backward(ctx, grad_logp):
    X, W, bias, targets = ctx.saved_tensors
    nx, nw, nb = ctx.needs_input_grad[0], ctx.needs_input_grad[1], ctx.needs_input_grad[2] and ctx.has_bias
    dX, dW, db = selective_logprob_backward(X, W, bias, targets, grad_logp, ctx.chunk_rows, nx, nw, nb)
    return (dX if nx else None), (dW if nw else None), (db if nb else None), None, None


selective_logprob_op.register_autograd(_sl_backward, setup_context=_sl_setup)


# ------------------------------------------------------------------ fused linear GRPO / BNPO
@torch.library.custom_op(f"{_NS}::fused_linear_grpo", mutates_args=())
def fused_linear_grpo(X: Tensor, W: Tensor, bias: Optional[Tensor], targets: Tensor, Xref: Optional[Tensor],
                      Wref: Optional[Tensor], old_lp: Tensor, adv: Tensor, mask: Tensor, eps_lo: float,
                      eps_hi: float, beta: float, reduction: int, two_sided: bool, temperature: float,
                      chunk_rows: int, need_x: bool, need_w: bool,
                      need_b: bool) -> tuple[Tensor, Tensor, Tensor, Tensor]:
    bs, T = mask.shape
    N, H = X.shape
    V = W.shape[0]
    mode = (pl.dtype_mode(X.dtype) | int(reduction) | (pl.PL_CLIP_TWO_SIDED if two_sided else 0) |
            (pl.PL_CHUNK_ROWS(chunk_rows) if chunk_rows else 0))
    Xc, Wc = X.detach().contiguous(), W.detach().contiguous()
    bc = bias.detach().contiguous() if bias is not None else None
    nb = need_b and bc is not None
    dX = torch.empty_like(Xc) if need_x else Xc.new_empty((0,))
    dW = torch.empty_like(Wc) if need_w else Wc.new_empty((0,))
    db = torch.empty_like(bc) if nb else Xc.new_empty((0,))
    loss = torch.empty((), dtype=torch.float32, device=X.device)
    ref_x = Xref.detach().contiguous() if (beta != 0.0 and Xref is not None) else None
    ref_w = Wref.detach().contiguous() if (beta != 0.0 and Wref is not None) else None
    wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, int(need_w), int(nb))
    ws = _workspace("fused", wsb, X.device)
    pl.check(pl.pl_fused_linear_grpo_temp(Xc, Wc, bc, targets.detach().to(torch.int64).contiguous(), ref_x, ref_w,
                                          old_lp.detach().to(torch.float32).contiguous(),
                                          adv.detach().to(torch.float32).contiguous(), mask.detach().contiguous(),
                                          bs, T, H, V, eps_lo, eps_hi, beta, temperature, mode, loss,
                                          dX if need_x else None, dW if need_w else None, db if nb else None,
                                          None, None, None, ws, wsb), "pl_fused_linear_grpo_temp")
    return loss, dX, dW, db


@fused_linear_grpo.register_fake
def _(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, eps_lo, eps_hi, beta, reduction, two_sided,
      temperature, chunk_rows, need_x, need_w, need_b):
    dX = torch.empty_like(X, memory_format=torch.contiguous_format) if need_x else X.new_empty((0,))
    dW = torch.empty_like(W, memory_format=torch.contiguous_format) if need_w else W.new_empty((0,))
    db = (torch.empty_like(bias, memory_format=torch.contiguous_format) if (need_b and bias is not None)
          else X.new_empty((0,)))
    return X.new_empty((), dtype=torch.float32), dX, dW, db


def _flg_setup(ctx, inputs, output):
    _, dX, dW, db = output
    ctx.save_for_backward(dX, dW, db)
    ctx.need = (inputs[16], inputs[17], inputs[18] and inputs[2] is not None)


def _flg_backward(ctx, grad_loss, g_dx, g_dw, g_db):
    dX, dW, db = ctx.saved_tensors
    out = [scale(g, grad_loss) if need else None for g, need in zip((dX, dW, db), ctx.need)]
    return (out[0], out[1], out[2]) + (None,) * 16


fused_linear_grpo.register_autograd(_flg_backward, setup_context=_flg_setup)


# ------------------------------------------------------------------ user-facing forms
def fused_linear_grpo_loss(X, W, targets, old_lp, adv, mask, bias=None, Xref=None, Wref=None, epsilon=0.2,
                           epsilon_high=0.2, beta=0.0, reduction="grpo", two_sided=False, temperature=1.0,
                           chunk_rows=0):
    """The fused linear GRPO / BNPO loss through the custom operator; differentiable in X, W and bias
    (see ``rl_post_policy_b200.autograd.fused_linear_grpo_loss`` for the arguments)."""
    red = {"grpo": pl.PL_GRPO, "bnpo": pl.PL_BNPO}[reduction] if isinstance(reduction, str) else int(reduction)
    grad_on = torch.is_grad_enabled()
    loss, _, _, _ = fused_linear_grpo(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, float(epsilon),
                                      float(epsilon_high), float(beta), red, bool(two_sided), float(temperature),
                                      int(chunk_rows or 0), grad_on and X.requires_grad,
                                      grad_on and W.requires_grad,
                                      grad_on and bias is not None and bias.requires_grad)
    return loss


def bnpo_loss(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0, two_sided=False):
    """BNPO loss (global token mean) through the custom operator; differentiable in policy_lp."""
    return policy_lp_loss(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, pl.PL_BNPO, two_sided)


def grpo_loss(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0, two_sided=False):
    """GRPO loss (per-sequence mean, then batch mean) through the custom operator."""
    return policy_lp_loss(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, pl.PL_GRPO, two_sided)


def policy_lp_loss(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, reduction, two_sided=False):
    loss, _ = policy_loss(policy_lp, old_lp, ref_lp, adv, mask, float(epsilon), float(epsilon_high), float(beta),
                          int(reduction), bool(two_sided))
    return loss


def reverse_kl_loss(student_logits, teacher_logits, completions_mask=None):
    """Masked mean over rows of KL(softmax(student) || softmax(teacher)); differentiable in the student."""
    loss, _ = reverse_kl(student_logits, teacher_logits, completions_mask)
    return loss


def selective_logprob(X, W, targets, bias=None, chunk_rows=0):
    """log_softmax(X W^T + bias)[targets] per row (fp32); differentiable in X, W and bias."""
    return selective_logprob_op(X, W, bias, targets, int(chunk_rows or 0))
