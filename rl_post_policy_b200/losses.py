"""Direct and forward-only entry points of the loss kernels, in the shape of the
"Geometric-AI Kernels" model card's "Kernels" table:

  ==========  ==============================  ====================
  family      direct (loss, grad)             forward only (loss)
  ==========  ==============================  ====================
  BNPO        ``bnpo_loss``                   ``bnpo_loss_fwd``
  GRPO        ``grpo_loss``                   ``grpo_loss_fwd``
  Reverse KL  ``reverse_kl``                  ``reverse_kl_fwd``
  ==========  ==============================  ====================

(the autograd-aware variants are in ``autograd``).  The direct form returns the
gradient the caller chains upstream, e.g. ``policy_logprobs.backward(grad)``.

Argument marshalling only: each call is one launch of libpl.so's kernel with
the library-owned workspace of the current stream (pl_loss / pl_reverse_kl with
a NULL workspace), so the host never waits.  The loss is a 0-dim fp32 tensor on
the device; gradients have the input's dtype and shape.
"""
from __future__ import annotations

import torch

from . import binding as pl


def _policy(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, reduction, two_sided, want_grad):
    bs, seq = policy_lp.shape
    lp = policy_lp.detach().contiguous()
    mode = pl.dtype_mode(lp.dtype) | reduction | (pl.PL_CLIP_TWO_SIDED if two_sided else 0)
    loss = torch.empty(1, dtype=torch.float32, device=lp.device)
    grad = torch.empty_like(lp) if want_grad else None
    ref = None if beta == 0 else ref_lp.detach().to(lp.dtype).contiguous()
    pl.check(pl.pl_loss(lp, old_lp.detach().to(lp.dtype).contiguous(), ref,
                        adv.detach().to(torch.float32).contiguous(),
                        mask.detach().to(torch.uint8).contiguous(), bs, seq, float(epsilon),
                        float(epsilon_high), float(beta), mode, loss, grad), "pl_loss")
    return (loss[0], grad) if want_grad else loss[0]


def bnpo_loss(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0, two_sided=False):
    """(loss, dloss/dpolicy_lp): BNPO, one fused forward+backward launch."""
    return _policy(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, pl.PL_BNPO, two_sided, True)


def bnpo_loss_fwd(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0, two_sided=False):
    """BNPO loss only (no gradient buffer)."""
    return _policy(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, pl.PL_BNPO, two_sided, False)


def grpo_loss(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0, two_sided=False):
    """(loss, dloss/dpolicy_lp): GRPO, one fused forward+backward launch."""
    return _policy(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, pl.PL_GRPO, two_sided, True)


def grpo_loss_fwd(policy_lp, old_lp, ref_lp, adv, mask, epsilon=0.2, epsilon_high=0.2, beta=0.0, two_sided=False):
    """GRPO loss only (no gradient buffer)."""
    return _policy(policy_lp, old_lp, ref_lp, adv, mask, epsilon, epsilon_high, beta, pl.PL_GRPO, two_sided, False)


def _rkl(student, teacher, mask, want_grad):
    V = student.shape[-1]
    N = student.numel() // V if V else 0
    s = student.detach().contiguous()
    t = teacher.detach().to(s.dtype).contiguous()
    m = mask.detach().to(torch.uint8).contiguous() if mask is not None else None
    loss = torch.empty(1, dtype=torch.float32, device=s.device)
    grad = torch.empty_like(s) if want_grad else None
    pl.check(pl.pl_reverse_kl(s, t, m, N, V, pl.dtype_mode(s.dtype), loss, grad, None, None, None, 0),
             "pl_reverse_kl")
    return (loss[0], grad) if want_grad else loss[0]


def reverse_kl(student_logits, teacher_logits, completions_mask=None):
    """(loss, dloss/dstudent_logits) of the masked mean of KL(softmax(student) || softmax(teacher))."""
    return _rkl(student_logits, teacher_logits, completions_mask, True)


def reverse_kl_fwd(student_logits, teacher_logits, completions_mask=None):
    """Reverse-KL loss only: one read of each logit row, no gradient buffer."""
    return _rkl(student_logits, teacher_logits, completions_mask, False)
