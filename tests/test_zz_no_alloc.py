"""pl_loss_static, the allocation-free loss entry point, against pl_loss_ex.

Some callers cannot allocate device memory on this path (a process that handed
its free memory to its own pool at start-up, or code that must not risk the
device-wide synchronisation of an allocation).  pl_loss_static keeps the loss
kernel's scratch in a fixed array of the library instead.  This test calls it
through the C ABI twice in a row, with different inputs, reductions and dtypes
(so the second call runs on the first call's leftover scratch), and checks each
result against the workspace entry point within the loss tests' tolerances.
It lives in its own file, collected last, and passes alone or after the others.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _args(inp, dtype):
    return [inp[k].to(dtype).cuda() for k in ("policy_lp", "old_lp", "ref_lp")] + [
        inp["adv"].cuda(), inp["mask"].cuda()]


def _run(pl, fn, inp, dtype, red, use_ws):
    bs, seq = inp["policy_lp"].shape
    lp, old, ref, adv, mask = _args(inp, dtype)
    loss = torch.full((1,), float("nan"), device="cuda")
    g = torch.full((bs, seq), float("nan"), dtype=dtype, device="cuda")
    nv = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    rv = torch.full((bs,), -1, dtype=torch.int64, device="cuda")
    mode = pl.dtype_mode(dtype) | red
    if use_ws:
        wsb = pl.pl_loss_workspace_bytes(bs, seq)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        rc = pl.pl_loss_ex(lp, old, ref, adv, mask, bs, seq, 0.2, 0.28, 0.04, mode, loss, g, nv, rv, ws, wsb)
        status = None
    else:
        st = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
        rc = pl.pl_loss_static(lp, old, ref, adv, mask, bs, seq, 0.2, 0.28, 0.04, mode, loss, g, nv, rv, st)
        status = st
    pl.check(rc, fn)
    torch.cuda.synchronize()
    return {"loss": loss.item(), "grad": g.float().cpu(), "n_valid": int(nv.item()),
            "row_valid": rv.cpu(), "status": None if status is None else int(status.item())}


def _ulp(x: np.ndarray, dtype) -> np.ndarray:
    mant, emin = {torch.bfloat16: (7, -126), torch.float16: (10, -14)}[dtype]
    ax = np.abs(x)
    e = np.maximum(np.floor(np.log2(np.where(ax > 0, ax, 1.0))), emin)
    return np.exp2(e - mant)


def _close(a, b, dtype):
    assert a["n_valid"] == b["n_valid"]
    assert torch.equal(a["row_valid"], b["row_valid"])
    tol = 1e-5 if dtype == torch.float32 else 1e-3
    assert abs(a["loss"] - b["loss"]) <= tol * abs(b["loss"])
    ga, gb = a["grad"].double().numpy(), b["grad"].double().numpy()
    if dtype == torch.float32:
        assert np.max(np.abs(ga - gb)) <= 1e-6
    else:
        assert np.all(np.abs(ga - gb) <= _ulp(gb, dtype))


def test_static_scratch_matches_workspace_entry_point_twice():
    import rl_post_policy_b200 as pl
    cases = [
        (synth.loss_inputs(16, 1024, torch.float32, synth.seed_for(1, 3)), torch.bfloat16, pl.PL_GRPO),
        (synth.loss_inputs(7, 333, torch.float32, synth.seed_for(1, 4), len_lo=0, len_hi=333),
         torch.float32, pl.PL_BNPO),
    ]
    for inp, dtype, red in cases:
        got = _run(pl, "pl_loss_static", inp, dtype, red, use_ws=False)
        want = _run(pl, "pl_loss_ex", inp, dtype, red, use_ws=True)
        assert got["status"] == 0
        _close(got, want, dtype)


def test_static_scratch_rejects_batch_beyond_limit():
    import rl_post_policy_b200 as pl
    bs, seq = 4097, 2
    x = torch.zeros(bs, seq, dtype=torch.bfloat16, device="cuda")
    adv = torch.zeros(bs, device="cuda")
    mask = torch.ones(bs, seq, dtype=torch.int8, device="cuda")
    loss = torch.zeros(1, device="cuda")
    rc = pl.pl_loss_static(x, x, x, adv, mask, bs, seq, 0.2, 0.28, 0.04, pl.PL_BF16, loss, None, None, None,
                           None)
    assert rc == pl.PL_ERR_WORKSPACE
