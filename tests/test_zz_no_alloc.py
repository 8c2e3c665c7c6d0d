"""pl_loss_static, the allocation-free loss entry point, against the oracle and
pl_loss_ex.

Some callers cannot allocate device memory on this path (a process that handed
its free memory to its own pool at start-up, or code that must not risk the
device-wide synchronisation of an allocation).  pl_loss_static keeps the loss
kernel's scratch in a fixed array of the library instead.  These tests call it
through the C ABI several times in a row with different inputs, reductions,
dtypes and kernels -- the small-batch kernel, then the cooperative one (more
than 65536 tokens), which starts on the first call's leftover scratch -- and
check each result against the oracle and against the workspace entry point
within the loss tests' tolerances.  They also check that a call changes the
device's free memory by nothing.  The file is collected last and passes alone
or after the others.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

EPS_LO, EPS_HI, BETA = 0.2, 0.28, 0.04


def _device_args(inp, dtype):
    bs, seq = inp["policy_lp"].shape
    a = {k: inp[k].to(dtype).cuda() for k in ("policy_lp", "old_lp", "ref_lp")}
    a["adv"], a["mask"] = inp["adv"].cuda(), inp["mask"].cuda()
    a["loss"] = torch.full((1,), float("nan"), device="cuda")
    a["grad"] = torch.full((bs, seq), float("nan"), dtype=dtype, device="cuda")
    a["nv"] = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    a["rv"] = torch.full((bs,), -1, dtype=torch.int64, device="cuda")
    a["status"] = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
    return a


def _call_static(pl, a, bs, seq, mode):
    return pl.pl_loss_static(a["policy_lp"], a["old_lp"], a["ref_lp"], a["adv"], a["mask"], bs, seq, EPS_LO,
                             EPS_HI, BETA, mode, a["loss"], a["grad"], a["nv"], a["rv"], a["status"])


def _result(a):
    return {"loss": a["loss"].item(), "grad": a["grad"].float().cpu(), "n_valid": int(a["nv"].item()),
            "row_valid": a["rv"].cpu().numpy()}


def _run(pl, inp, dtype, red, use_ws):
    bs, seq = inp["policy_lp"].shape
    a = _device_args(inp, dtype)
    mode = pl.dtype_mode(dtype) | red
    if use_ws:
        wsb = pl.pl_loss_workspace_bytes(bs, seq)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        pl.check(pl.pl_loss_ex(a["policy_lp"], a["old_lp"], a["ref_lp"], a["adv"], a["mask"], bs, seq, EPS_LO,
                               EPS_HI, BETA, mode, a["loss"], a["grad"], a["nv"], a["rv"], ws, wsb), "pl_loss_ex")
        torch.cuda.synchronize()
        return _result(a)
    pl.check(_call_static(pl, a, bs, seq, mode), "pl_loss_static")
    torch.cuda.synchronize()
    out = _result(a)
    out["status"] = int(a["status"].item())
    return out


def _ulp(x: np.ndarray, dtype) -> np.ndarray:
    mant, emin = {torch.bfloat16: (7, -126), torch.float16: (10, -14)}[dtype]
    ax = np.abs(x)
    e = np.maximum(np.floor(np.log2(np.where(ax > 0, ax, 1.0))), emin)
    return np.exp2(e - mant)


def _kink(inp, dtype):
    # a ratio within 8 fp32 ulps of 1 + eps_hi may take either side of the min() in fp32
    lp, old = oracle.decode(inp["policy_lp"].to(dtype)), oracle.decode(inp["old_lp"].to(dtype))
    hi = np.float32(1.0) + np.float32(EPS_HI)
    return np.abs(np.exp(lp - old) - float(hi)) <= 8 * float(np.spacing(hi))


def _check_vs_oracle(got, inp, dtype, red):
    want = oracle.policy_loss(inp["policy_lp"].to(dtype), inp["old_lp"].to(dtype), inp["ref_lp"].to(dtype),
                              inp["adv"], inp["mask"], eps_lo=EPS_LO, eps_hi=EPS_HI, beta=BETA, reduction=red)
    assert got["n_valid"] == want["n_valid"]
    assert np.array_equal(got["row_valid"], want["row_valid"])
    tol = 1e-5 if dtype == torch.float32 else 1e-3
    assert abs(want["loss"]) > 0.05 * want["abs_sum"]  # no +/-A cancellation in these inputs
    assert abs(got["loss"] - want["loss"]) <= tol * abs(want["loss"]), (got["loss"], want["loss"])
    g, w = got["grad"].double().numpy(), want["grad"]
    if dtype == torch.float32:
        err, bound = np.abs(g - w), 1e-6
    else:
        wr = torch.from_numpy(w).to(dtype).double().numpy()
        err, bound = np.abs(g - wr) / _ulp(wr, dtype), 1.0
    bad = (err > bound) & ~_kink(inp, dtype)
    assert not bad.any(), int(bad.sum())


def _check_vs_workspace_call(a, b, dtype):
    assert a["n_valid"] == b["n_valid"]
    assert np.array_equal(a["row_valid"], b["row_valid"])
    tol = 1e-5 if dtype == torch.float32 else 1e-3
    assert abs(a["loss"] - b["loss"]) <= tol * abs(b["loss"])
    ga, gb = a["grad"].double().numpy(), b["grad"].double().numpy()
    if dtype == torch.float32:
        assert np.max(np.abs(ga - gb)) <= 1e-6
    else:
        assert np.all(np.abs(ga - gb) <= _ulp(gb, dtype))


def _same_sign(inp):
    # large batches of N(0,1) advantages sum to a loss near zero, where a relative
    # error says nothing: same-sign advantages keep it away from zero
    inp["adv"] = inp["adv"].abs() + 0.1
    return inp


def _cases(pl):
    return [
        # small-batch kernel (16 x 1024 tokens)
        (synth.loss_inputs(16, 1024, torch.float32, synth.seed_for(1, 3)), torch.bfloat16, pl.PL_GRPO),
        # small-batch kernel, a ragged batch with an empty sequence, fp32
        (synth.loss_inputs(7, 333, torch.float32, synth.seed_for(1, 4), len_lo=0, len_hi=333),
         torch.float32, pl.PL_BNPO),
        # cooperative kernel (131072 tokens), right after a small call
        (_same_sign(synth.loss_inputs(128, 1024, torch.float32, synth.seed_for(1, 5))), torch.bfloat16, pl.PL_GRPO),
        # cooperative kernel, more sequences than the small kernel takes (bs = 2048), fp16
        (_same_sign(synth.loss_inputs(2048, 40, torch.float32, synth.seed_for(1, 6), len_lo=0, len_hi=40)),
         torch.float16, pl.PL_BNPO),
    ]


def test_static_scratch_matches_oracle_and_workspace_entry_point():
    import rl_post_policy_b200 as pl
    for inp, dtype, red in _cases(pl):
        got = _run(pl, inp, dtype, red, use_ws=False)
        assert got["status"] == 0
        _check_vs_oracle(got, inp, dtype, red)
        _check_vs_workspace_call(got, _run(pl, inp, dtype, red, use_ws=True), dtype)


def test_static_scratch_calls_allocate_nothing():
    import rl_post_policy_b200 as pl
    cases = _cases(pl)
    staged = []
    for inp, dtype, red in (cases[0], cases[2]):  # one call on each kernel
        bs, seq = inp["policy_lp"].shape
        a = _device_args(inp, dtype)
        mode = pl.dtype_mode(dtype) | red
        pl.check(_call_static(pl, a, bs, seq, mode), "pl_loss_static")  # warm-up: kernels loaded
        staged.append((a, bs, seq, mode))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for a, bs, seq, mode in staged:
        pl.check(_call_static(pl, a, bs, seq, mode), "pl_loss_static")
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    for (inp, dtype, red), (a, _, _, _) in zip((cases[0], cases[2]), staged):
        assert int(a["status"].item()) == 0
        _check_vs_oracle(_result(a), inp, dtype, red)


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
