"""The custom-operator registrations (rl_post_policy_b200.torch_ops) without a
GPU: every operator is registered under torch.ops.rl_post_policy_b200 and its
shape function gives the outputs' shapes, dtypes and devices for FakeTensor
inputs, as torch.compile's tracing needs."""
import torch
from torch._subclasses.fake_tensor import FakeTensorMode

from rl_post_policy_b200 import torch_ops  # noqa: F401  (registers the operators)

OPS = torch.ops.rl_post_policy_b200


def test_operators_are_registered():
    for name in ("policy_loss", "reverse_kl", "selective_logprob", "selective_logprob_backward", "scale",
                 "fused_linear_grpo"):
        assert hasattr(OPS, name), name


def test_shapes_under_fake_tensors():
    with FakeTensorMode():
        lp = torch.empty(3, 5, dtype=torch.bfloat16, device="cuda")
        adv = torch.empty(3, device="cuda")
        mask = torch.empty(3, 5, dtype=torch.uint8, device="cuda")
        loss, g = OPS.policy_loss(lp, lp, lp, adv, mask, 0.2, 0.28, 0.04, 1, False)
        assert loss.shape == () and loss.dtype == torch.float32
        assert g.shape == lp.shape and g.dtype == lp.dtype and g.device == lp.device

        s = torch.empty(2, 7, 96, dtype=torch.float16, device="cuda")
        loss, g = OPS.reverse_kl(s, s, None)
        assert loss.shape == () and g.shape == s.shape and g.dtype == s.dtype

        X = torch.empty(10, 64, dtype=torch.bfloat16, device="cuda")
        W = torch.empty(300, 64, dtype=torch.bfloat16, device="cuda")
        b = torch.empty(300, dtype=torch.bfloat16, device="cuda")
        t = torch.empty(10, dtype=torch.int64, device="cuda")
        logp = OPS.selective_logprob(X, W, b, t, 0)
        assert logp.shape == (10,) and logp.dtype == torch.float32
        dX, dW, db = OPS.selective_logprob_backward(X, W, b, t, logp, 0, True, False, True)
        assert dX.shape == X.shape and dW.numel() == 0 and db.shape == b.shape

        old = torch.empty(10, device="cuda")
        loss, dX, dW, db = OPS.fused_linear_grpo(X, W, b, t, X, W, old, adv[:2], torch.empty(2, 5, dtype=torch.uint8, device="cuda"),
                                                 0.2, 0.28, 0.04, 1, False, 1.0, 0, True, True, False)
        assert loss.shape == () and dX.shape == X.shape and dW.shape == W.shape and db.numel() == 0

        y = OPS.scale(lp, adv[:1])
        assert y.shape == lp.shape and y.dtype == lp.dtype
