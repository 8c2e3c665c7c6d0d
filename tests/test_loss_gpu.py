"""Parity of the loss-only CUDA kernels (pl_loss / pl_loss_ex) with the CPU oracle.
Every test runs twice through the loss_path fixture: with the small-batch kernel
(taken whenever the batch has at most 65536 tokens and 1024 sequences) and with
the cooperative kernel.

Tolerances: loss relative error <= 1e-5 (fp32 inputs) and <= 1e-3 (bf16/fp16);
fp32 grad max abs error <= 1e-6; bf16/fp16 grad within one unit in the last
place of the dtype of the rounded oracle value; valid-token counts bit-exact.
A token whose oracle ratio lies within 8 fp32 ulps of the clip bound 1+eps_hi may
take either side of the min() in fp32 (both sides are correct), so its gradient
is left out of the element-wise comparison.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("loss_path")]

EPS_LO, EPS_HI = 0.2, 0.28
DTYPES = [torch.bfloat16, torch.float16, torch.float32]


def pl():
    import rl_post_policy_b200 as m
    return m


def run_gpu(inp, dtype, red, beta, grad=True, two_sided=False, adv_lp=False, stream=None,
            offset=0):
    m = pl()
    dev = torch.device("cuda")
    bs, seq = inp["policy_lp"].shape

    def up(t, dt=None):
        t = t.to(dt) if dt is not None else t
        if offset:  # deliberately misaligned device copies
            buf = torch.empty(t.numel() + offset, dtype=t.dtype, device=dev)
            v = buf[offset:].view(t.shape)
            v.copy_(t)
            return v
        return t.to(dev).contiguous()

    lp, old = up(inp["policy_lp"], dtype), up(inp["old_lp"], dtype)
    ref = up(inp["ref_lp"], dtype) if beta != 0.0 else None
    adv = up(inp["adv"], dtype if adv_lp else torch.float32)
    mask = up(inp["mask"].to(torch.int8))
    loss = torch.full((1,), float("nan"), dtype=torch.float32, device=dev)
    g = torch.full((bs, seq), float("nan"), dtype=dtype, device=dev) if grad else None
    nv = torch.full((1,), -1, dtype=torch.int64, device=dev)
    rv = torch.full((max(bs, 1),), -1, dtype=torch.int64, device=dev)
    wsb = m.pl_loss_workspace_bytes(bs, seq)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    mode = m.dtype_mode(dtype) | red | (m.PL_CLIP_TWO_SIDED if two_sided else 0) | (
        m.PL_ADV_LP_DTYPE if adv_lp else 0)
    rc = m.pl_loss_ex(lp, old, ref, adv, mask, bs, seq, EPS_LO, EPS_HI, beta, mode, loss, g, nv, rv,
                      ws, wsb, stream=stream)
    m.check(rc, "pl_loss_ex")
    torch.cuda.synchronize()
    m.check(m.pl_device_status(ws, stream), "device status")
    return {"loss": float(loss.item()), "grad": None if g is None else g.float().cpu(),
            "n_valid": int(nv.item()), "row_valid": rv[:bs].cpu().numpy(), "ws": ws}


def ulp(x: np.ndarray, dtype) -> np.ndarray:
    mant, emin = {torch.bfloat16: (7, -126), torch.float16: (10, -14)}[dtype]
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, emin)
    return np.exp2(e - mant)


def kink_tokens(inp, dtype):
    lp = oracle.decode(inp["policy_lp"].to(dtype))
    old = oracle.decode(inp["old_lp"].to(dtype))
    hi = np.float32(1.0) + np.float32(EPS_HI)
    r = np.exp(lp - old)
    return np.abs(r - float(hi)) <= 8 * float(np.spacing(hi))


def oracle_ref(inp, dtype, red, beta, two_sided=False, adv_lp=False):
    adv = inp["adv"].to(dtype) if adv_lp else inp["adv"]
    return oracle.policy_loss(inp["policy_lp"].to(dtype), inp["old_lp"].to(dtype),
                              inp["ref_lp"].to(dtype) if beta != 0 else None, adv, inp["mask"],
                              eps_lo=EPS_LO, eps_hi=EPS_HI, beta=beta, reduction=red,
                              two_sided=two_sided)


def compare(inp, dtype, red, beta, got, two_sided=False, adv_lp=False):
    want = oracle_ref(inp, dtype, red, beta, two_sided, adv_lp)
    assert got["n_valid"] == want["n_valid"]
    assert np.array_equal(got["row_valid"], want["row_valid"])
    tol = 1e-5 if dtype == torch.float32 else 1e-3
    denom = max(abs(want["loss"]), 1e-30)
    if want["loss"] == 0.0:
        assert got["loss"] == 0.0
    else:
        assert abs(got["loss"] - want["loss"]) / denom <= tol, (got["loss"], want["loss"])
    if got["grad"] is None:
        return want
    g = got["grad"].double().numpy()
    w = want["grad"]
    kink = kink_tokens(inp, dtype)
    if dtype == torch.float32:
        err = np.abs(g - w)
    else:
        wr = torch.from_numpy(w).to(dtype).double().numpy()
        err = np.abs(g - wr) / ulp(wr, dtype)
    bound = 1e-6 if dtype == torch.float32 else 1.0
    bad = (err > bound) & ~kink
    assert not bad.any(), f"{bad.sum()} tokens off (max {err[~kink].max()})"
    return want


@pytest.fixture(scope="module")
def w1():
    return {dt: synth.loss_inputs(16, 1024, torch.float32, synth.seed_for(1)) for dt in [0]}[0]


@pytest.mark.parametrize("dtype", DTYPES, ids=["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("red", [0, 1], ids=["bnpo", "grpo"])
@pytest.mark.parametrize("beta", [0.04, 0.0], ids=["beta0.04", "beta0"])
@pytest.mark.parametrize("grad", [True, False], ids=["fwdbwd", "fwd"])
def test_workload_loss_only(w1, dtype, red, beta, grad):
    got = run_gpu(w1, dtype, red, beta, grad=grad)
    compare(w1, dtype, red, beta, got)


@pytest.mark.parametrize("dtype", DTYPES, ids=["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("bs,seq", [(1, 1), (3, 7), (2, 1023), (5, 17), (3000, 5), (1, 70001),
                                    (7, 4096)])
def test_ragged_shapes(dtype, bs, seq):
    inp = synth.loss_inputs(bs, seq, torch.float32, 1234 + bs * 31 + seq, len_lo=0, len_hi=seq)
    for red in (0, 1):
        got = run_gpu(inp, dtype, red, 0.04)
        compare(inp, dtype, red, 0.04, got)


@pytest.mark.parametrize("dtype", DTYPES, ids=["bf16", "fp16", "fp32"])
def test_misaligned_pointers_take_scalar_path(dtype):
    inp = synth.loss_inputs(4, 333, torch.float32, 77, len_lo=0, len_hi=333)
    for red in (0, 1):
        got = run_gpu(inp, dtype, red, 0.04, offset=1)
        compare(inp, dtype, red, 0.04, got)


@pytest.mark.parametrize("dtype", DTYPES, ids=["bf16", "fp16", "fp32"])
def test_two_sided_clip_and_adv_in_lp_dtype(w1, dtype):
    for red in (0, 1):
        got = run_gpu(w1, dtype, red, 0.04, two_sided=True, adv_lp=True)
        compare(w1, dtype, red, 0.04, got, two_sided=True, adv_lp=True)


@pytest.mark.parametrize("red", [0, 1])
def test_all_masked_and_empty(red):
    inp = synth.loss_inputs(4, 64, torch.float32, 5)
    inp["mask"] = torch.zeros_like(inp["mask"])
    got = run_gpu(inp, torch.bfloat16, red, 0.04)
    assert got["loss"] == 0.0 and got["n_valid"] == 0
    assert torch.all(got["grad"] == 0)
    for bs, seq in [(0, 16), (3, 0), (0, 0)]:
        e = synth.loss_inputs(bs, seq, torch.float32, 6)
        got = run_gpu(e, torch.bfloat16, red, 0.04)
        assert got["loss"] == 0.0 and got["n_valid"] == 0


def test_deterministic_and_reusable_workspace(w1):
    a = run_gpu(w1, torch.bfloat16, 1, 0.04)
    b = run_gpu(w1, torch.bfloat16, 1, 0.04)
    assert a["loss"] == b["loss"] and torch.equal(a["grad"], b["grad"])
    # the kernel returns its counters to zero: the header words after the flag are 0
    hdr = a["ws"][:32].cpu().numpy()
    assert np.all(hdr == 0)


def test_runs_on_callers_stream(w1):
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        got = run_gpu(w1, torch.bfloat16, 0, 0.04, stream=s)
    compare(w1, torch.bfloat16, 0, 0.04, got)


def test_library_owned_scratch_entry_point(w1):
    m = pl()
    dev = torch.device("cuda")
    dt = torch.bfloat16
    lp, old, ref = (w1[k].to(dt).to(dev) for k in ("policy_lp", "old_lp", "ref_lp"))
    adv = w1["adv"].to(dev)
    mask = w1["mask"].to(dev)
    loss = torch.empty(1, device=dev)
    g = torch.empty_like(lp)
    for _ in range(2):
        m.check(m.pl_loss(lp, old, ref, adv, mask, 16, 1024, EPS_LO, EPS_HI, 0.04,
                          m.PL_BF16 | m.PL_GRPO, loss, g))
    torch.cuda.synchronize()
    assert m.pl_device_status(None) == m.PL_OK
    want = oracle_ref(w1, dt, 1, 0.04)
    assert abs(loss.item() - want["loss"]) <= 1e-3 * abs(want["loss"])


@pytest.mark.parametrize("log2n", [22, 26])
def test_large_sweep_point(log2n):
    """A bandwidth-sweep size (bs=16); every token is compared."""
    n = 1 << log2n
    inp = synth.loss_inputs(16, n // 16, torch.float32, synth.seed_for(1, 8), len_lo=1,
                            len_hi=n // 16)
    got = run_gpu(inp, torch.bfloat16, 0, 0.04)
    compare(inp, torch.bfloat16, 0, 0.04, got)
