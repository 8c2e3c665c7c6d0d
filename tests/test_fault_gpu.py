"""Failure detection without a GPU fault: bounded device waits that are made to
run out on purpose must come back as PL_ERR_DEVICE_TIMEOUT, release what they
hold, and leave the context usable.

The loss kernel's grid barrier is told to wait for one arrival more than there
are blocks; the GEMM's pipeline stages and the register-resident reverse-KL
kernel's slots are told to expect 16 bytes more than their TMA loads deliver.
The waits are bounded to 50 ms for the test.
"""
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gemm_tile")]


@pytest.fixture
def pl():
    import rl_post_policy_b200 as m
    yield m
    m.pl_debug_set_wait(0, 0, 0)


def _loss_call(m, inp, ws, wsb, loss, g):
    bs, seq = inp["policy_lp"].shape
    d = {k: inp[k].cuda() for k in ("policy_lp", "old_lp", "ref_lp", "adv", "mask")}
    return m.pl_loss_ex(d["policy_lp"], d["old_lp"], d["ref_lp"], d["adv"], d["mask"], bs, seq, 0.2,
                        0.28, 0.04, m.PL_BF16 | m.PL_GRPO, loss, g, None, None, ws, wsb)


def test_loss_barrier_timeout_is_reported(pl):
    inp = synth.loss_inputs(16, 1024, torch.bfloat16, 31)
    wsb = pl.pl_loss_workspace_bytes(16, 1024)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    loss = torch.zeros(1, device="cuda")
    g = torch.empty(16, 1024, dtype=torch.bfloat16, device="cuda")
    pl.pl_debug_set_wait(50_000_000, 1, 0)
    pl.check(_loss_call(pl, inp, ws, wsb, loss, g))
    assert pl.pl_device_status(ws) == pl.PL_ERR_DEVICE_TIMEOUT
    assert pl.pl_device_status(ws) == pl.PL_OK  # the flag was cleared by the read
    # normal operation afterwards, on the same workspace
    pl.pl_debug_set_wait(0, 0, 0)
    pl.check(_loss_call(pl, inp, ws, wsb, loss, g))
    assert pl.pl_device_status(ws) == pl.PL_OK
    want = oracle.policy_loss(inp["policy_lp"], inp["old_lp"], inp["ref_lp"], inp["adv"], inp["mask"],
                              eps_lo=0.2, eps_hi=0.28, beta=0.04, reduction=oracle.GRPO)
    assert abs(loss.item() - want["loss"]) <= 1e-3 * abs(want["loss"])


def test_gemm_pipeline_timeout_is_reported(pl):
    A = torch.randn(256, 128, device="cuda").to(torch.bfloat16)
    B = torch.randn(512, 128, device="cuda").to(torch.bfloat16)
    D = torch.zeros(256, 512, device="cuda")
    pl.pl_debug_set_wait(50_000_000, 0, 16)
    pl.check(pl.pl_debug_gemm(A, 0, 128, B, 0, 128, D, 256, 512, 128, pl.PL_BF16))
    assert pl.pl_device_status(None) == pl.PL_ERR_DEVICE_TIMEOUT
    pl.pl_debug_set_wait(0, 0, 0)
    pl.check(pl.pl_debug_gemm(A, 0, 128, B, 0, 128, D, 256, 512, 128, pl.PL_BF16))
    assert pl.pl_device_status(None) == pl.PL_OK
    ref = A.double() @ B.double().t()
    assert torch.allclose(D.double(), ref, rtol=1e-4, atol=1e-3)


def test_reverse_kl_slot_timeout_is_reported(pl):
    # the register-resident reverse-KL kernel's slots expect 16 bytes more than their
    # bulk copies deliver: the bounded waits run out, the cluster still finishes
    # together, and the next normal call on the same workspace is correct
    inp = synth.reverse_kl_inputs(2, 12, 5000, torch.bfloat16, synth.seed_for(51))
    s, t, mk = inp["student"].cuda(), inp["teacher"].cuda(), inp["mask"].cuda()
    N, V = 24, 5000
    g = torch.empty(N, V, dtype=torch.bfloat16, device="cuda")
    loss = torch.zeros(1, device="cuda")
    wsb = pl.pl_reverse_kl_workspace_bytes(N, V)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    assert pl.pl_debug_set_rkl_path(2) == 0
    pl.pl_debug_set_wait(50_000_000, 0, 16)
    try:
        pl.check(pl.pl_reverse_kl(s, t, mk, N, V, pl.PL_BF16, loss, g, None, None, ws, wsb))
        assert pl.pl_device_status(ws) == pl.PL_ERR_DEVICE_TIMEOUT
    finally:
        pl.pl_debug_set_wait(0, 0, 0)
        pl.pl_debug_set_rkl_path(0)
    pl.check(pl.pl_reverse_kl(s, t, mk, N, V, pl.PL_BF16, loss, g, None, None, ws, wsb))
    assert pl.pl_device_status(ws) == pl.PL_OK
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"])
    assert abs(loss.item() - want["loss"]) <= 1e-4 * abs(want["loss"])


def test_merged_chunk_launch_timeout_is_reported(pl):
    # several chunks: the merged backward + forward launch (dynamic tile queue)
    # times out like any other, and its queue counters are back at zero for the
    # next call on the same workspace
    import numpy as np
    bs, T, H, V = 2, 192, 128, 1000
    inp = synth.fused_inputs(bs, T, H, V, torch.bfloat16, 6161, bias=False, need_ref=True)
    _, lp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], None, inp["targets"])
    inp["old_lp"] = (torch.from_numpy(lp) + inp["old_noise"].double()).float()
    g = {k: inp[k].cuda() for k in ("X", "W", "Xref", "Wref", "targets", "old_lp", "adv", "mask")}
    mode = pl.PL_BF16 | pl.PL_GRPO | pl.PL_CHUNK_ROWS(128)
    wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, 1, 0)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    loss = torch.zeros(1, device="cuda")
    dX = torch.empty(bs * T, H, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(V, H, dtype=torch.bfloat16, device="cuda")

    def call():
        return pl.pl_fused_linear_grpo(g["X"], g["W"], None, g["targets"], g["Xref"], g["Wref"], g["old_lp"],
                                       g["adv"], g["mask"], bs, T, H, V, 0.2, 0.28, 0.04, mode, loss, dX, dW,
                                       None, None, None, None, ws, wsb)

    pl.pl_debug_set_wait(50_000_000, 0, 16)
    pl.check(call())
    assert pl.pl_device_status(ws) == pl.PL_ERR_DEVICE_TIMEOUT
    pl.pl_debug_set_wait(0, 0, 0)
    # a workspace that saw a device error is zeroed again before reuse
    ws.zero_()
    pl.check(call())
    assert pl.pl_device_status(ws) == pl.PL_OK
    want = oracle.fused_grpo(inp["X"], inp["W"], None, inp["targets"], inp["Xref"], inp["Wref"],
                             inp["old_lp"].reshape(bs, T), inp["adv"], inp["mask"], eps_lo=0.2, eps_hi=0.28,
                             beta=0.04, reduction=oracle.GRPO)
    assert abs(loss.item() - want["loss"]) <= 1e-3 * abs(want["loss"])
    rel = np.linalg.norm(dW.cpu().double().numpy() - want["dW"]) / np.linalg.norm(want["dW"])
    assert rel <= 1e-2
