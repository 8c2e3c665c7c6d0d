"""Parity of the fused linear path (pl_fused_linear_grpo) with the CPU oracle.

Tolerances: selected log-probs abs <= 2e-3; loss relative <= 1e-3; dX, dW and
dbias relative Frobenius <= 1e-2; the valid-token count bit-exact.  Inputs are
seeded; the behaviour log-probs are moved at least 2e-4 (in log space) off the
clip bounds, where fp32 and fp64 may legitimately choose different sides of the
min(), and a test asserts that none is left within 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gemm_tile", "gemm_variant")]

EPS_LO, EPS_HI = 0.2, 0.28


def pl():
    import rl_post_policy_b200 as m
    return m


def build_inputs(bs, T, H, V, dtype, seed, bias=False, beta=0.04, len_lo=1, len_hi=None,
                 fully_masked_last=False):
    inp = synth.fused_inputs(bs, T, H, V, dtype, seed, bias=bias, len_lo=len_lo, len_hi=len_hi,
                             fully_masked_last=fully_masked_last, need_ref=True)
    _, logp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"])
    old = torch.from_numpy(logp) + inp["old_noise"].double()
    for bound in (np.log(float(np.float32(1) + np.float32(EPS_HI))),
                  np.log(float(np.float32(1) - np.float32(EPS_LO)))):
        d = torch.from_numpy(logp) - old - bound
        near = d.abs() < 2e-4
        old[near] -= torch.where(d[near] >= 0, 2e-4, -2e-4).double()
    inp["old_lp"] = old.float()
    return inp


def run_fused(inp, dtype, red, beta, chunk=None, want=("dX", "dW", "dbias"), two_sided=False,
              targets=None, out_offset=0):
    m = pl()
    dev = "cuda"
    bs, T = inp["mask"].shape
    N, H = inp["X"].shape
    V = inp["W"].shape[0]
    X, W = inp["X"].to(dev), inp["W"].to(dev)
    b = inp["bias"].to(dev) if inp["bias"] is not None else None
    Xr = inp["Xref"].to(dev) if beta != 0 else None
    Wr = inp["Wref"].to(dev) if beta != 0 else None
    tg = (targets if targets is not None else inp["targets"]).to(dev)
    old = inp["old_lp"].to(dev)
    adv = inp["adv"].float().to(dev)
    mask = inp["mask"].to(dev)
    loss = torch.full((1,), float("nan"), device=dev)
    bufs = []

    def out(shape):
        # a NaN-filled view `out_offset` elements into a buffer 8 elements longer
        n = int(np.prod(shape))
        buf = torch.full((n + out_offset + 8,), float("nan"), dtype=dtype, device=dev)
        bufs.append((buf, n))
        return buf[out_offset:out_offset + n].view(shape)

    dX = out((N, H)) if "dX" in want else None
    dW = out((V, H)) if "dW" in want else None
    db = out((V,)) if ("dbias" in want and b is not None) else None
    lp = torch.full((N,), float("nan"), device=dev)
    rlp = torch.full((N,), float("nan"), device=dev)
    nv = torch.full((1,), -1, dtype=torch.int64, device=dev)
    mode = m.dtype_mode(dtype) | red | (m.PL_CLIP_TWO_SIDED if two_sided else 0)
    if chunk:
        mode |= m.PL_CHUNK_ROWS(chunk)
    wsb = m.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, dW is not None, db is not None)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    rc = m.pl_fused_linear_grpo(X, W, b, tg, Xr, Wr, old, adv, mask, bs, T, H, V, EPS_LO, EPS_HI,
                                beta, mode, loss, dX, dW, db, lp, rlp, nv, ws, wsb)
    m.check(rc, "pl_fused_linear_grpo")
    torch.cuda.synchronize()
    status = m.pl_device_status(ws)
    res = {"loss": loss.item(), "logp": lp.cpu().double().numpy(), "ref_logp": rlp.cpu().double().numpy(),
           "n_valid": int(nv.item()), "status": status}
    for buf, n in bufs:   # nothing written outside the outputs
        assert torch.isnan(buf[:out_offset]).all() and torch.isnan(buf[out_offset + n:]).all()
    for k, t in (("dX", dX), ("dW", dW), ("dbias", db)):
        res[k] = None if t is None else t.cpu().double().numpy()
    return res


def rel_fro(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def check(inp, got, red, beta, two_sided=False, check_grads=True):
    want = oracle.fused_grpo(inp["X"], inp["W"], inp["bias"], inp["targets"], inp["Xref"],
                             inp["Wref"], inp["old_lp"].reshape(inp["mask"].shape), inp["adv"],
                             inp["mask"], eps_lo=EPS_LO, eps_hi=EPS_HI, beta=beta, reduction=red,
                             two_sided=two_sided)
    old = inp["old_lp"].double().numpy()
    d = want["logp"] - old
    assert np.all(np.abs(d - np.log(float(np.float32(1) + np.float32(EPS_HI)))) > 1e-4)
    assert got["status"] == 0
    assert got["n_valid"] == want["n_valid"]
    assert np.max(np.abs(got["logp"] - want["logp"])) <= 2e-3
    if beta != 0:
        assert np.max(np.abs(got["ref_logp"] - want["ref_logp"])) <= 2e-3
    assert abs(got["loss"] - want["loss"]) <= 1e-3 * abs(want["loss"]), (got["loss"], want["loss"])
    if check_grads:
        for k in ("dX", "dW", "dbias"):
            if got.get(k) is not None:
                e = rel_fro(got[k], want[k])
                assert e <= 1e-2, (k, e)
    return want


@pytest.mark.parametrize("red", [0, 1], ids=["bnpo", "grpo"])
def test_tiny_workload(red):
    w = synth.WORKLOADS[0]
    inp = build_inputs(w["bs"], w["T"], w["H"], w["V"], w["dtype"], synth.seed_for(0),
                       len_lo=w["len_lo"], len_hi=w["len_hi"])
    got = run_fused(inp, w["dtype"], red, w["beta"])
    check(inp, got, red, w["beta"])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("chunk", [None, 128], ids=["one_chunk", "chunks128"])
@pytest.mark.parametrize("beta", [0.04, 0.0], ids=["beta0.04", "beta0"])
def test_ragged_multi_tile(dtype, chunk, beta):
    # N=300 rows (3 row tiles, ragged), H=200 (K tail), V=1000 (4 vocab tiles, ragged), bias
    inp = build_inputs(3, 100, 200, 1000, dtype, 4242, bias=True, len_lo=0, len_hi=100,
                       fully_masked_last=True)
    for red in (0, 1):
        got = run_fused(inp, dtype, red, beta, chunk=chunk)
        check(inp, got, red, beta)


@pytest.mark.parametrize("nchunks", [2, 3, 4, 5])
def test_paired_weight_gradient(nchunks):
    # bf16 with several chunks: chunks 2i and 2i+1 contribute to dW through one GEMM
    # job whose K runs over both chunks' rows (two tensor-map segments), with the
    # dlogits of every chunk unscaled; the last chunk of an odd count contributes
    # alone, and two chunks make a single contribution stored straight in bf16.
    # The last chunk is ragged.  Both ways, and one dW job per chunk, match the
    # oracle, and dX and the log-probs do not depend on the pairing beyond
    # rounding (a launch's epilogue warp count, and with it the grouping of the
    # logsumexp partials, can differ between the two ways under some variants).
    m = pl()
    T = 128 * nchunks - 37
    inp = build_inputs(1, T, 192, 900, torch.bfloat16, 5150 + nchunks, bias=True, len_lo=T - 40, len_hi=T)
    got = {}
    try:
        for mode in (2, 1):
            assert m.pl_debug_set_dw_pair(mode) == 0
            got[mode] = run_fused(inp, torch.bfloat16, 1, 0.04, chunk=128)
            check(inp, got[mode], 1, 0.04)
    finally:
        m.pl_debug_set_dw_pair(0)
    assert np.max(np.abs(got[2]["logp"] - got[1]["logp"])) <= 1e-5
    assert rel_fro(got[2]["dX"], got[1]["dX"]) <= 1e-3
    assert m.pl_debug_set_dw_pair(3) != 0


def test_two_sided_clip():
    inp = build_inputs(2, 64, 128, 640, torch.bfloat16, 99, bias=False)
    got = run_fused(inp, torch.bfloat16, 1, 0.04, two_sided=True)
    check(inp, got, 1, 0.04, two_sided=True)


@pytest.mark.parametrize("want", [("dX",), ("dW",), ("dbias",), ()])
def test_partial_gradients(want):
    inp = build_inputs(2, 96, 128, 700, torch.bfloat16, 7, bias=True)
    got = run_fused(inp, torch.bfloat16, 1, 0.04, want=want, chunk=128)
    check(inp, got, 1, 0.04)


def test_bad_target_is_flagged_and_masked():
    m = pl()
    inp = build_inputs(2, 32, 64, 512, torch.bfloat16, 11)
    bad = inp["targets"].clone()
    bad[0] = 512  # == V: out of range (position 0 is always inside the valid prefix)
    got = run_fused(inp, torch.bfloat16, 0, 0.04, targets=bad)
    assert got["status"] == m.PL_ERR_BAD_TARGET
    assert np.isnan(got["logp"][0])
    # the row counts as masked: compare against the oracle with that token masked out
    masked = dict(inp)
    mk = inp["mask"].clone().reshape(-1)
    mk[0] = 0
    masked["mask"] = mk.reshape(inp["mask"].shape)
    want = oracle.fused_grpo(inp["X"], inp["W"], None, inp["targets"], inp["Xref"], inp["Wref"],
                             inp["old_lp"].reshape(2, 32), inp["adv"], masked["mask"], eps_lo=EPS_LO,
                             eps_hi=EPS_HI, beta=0.04, reduction=0)
    # the token contributes nothing, but the BNPO denominator is the mask's own count
    n_orig = int(inp["mask"].sum())
    expect = want["loss"] * (n_orig - 1) / n_orig
    assert got["n_valid"] == n_orig
    assert abs(got["loss"] - expect) <= 1e-3 * abs(expect)
    assert np.all(got["dX"][0] == 0.0)


@pytest.mark.parametrize("chunk", [4096, 8192])
def test_large_chunk_small_model(chunk):
    # many rows in one chunk (the per-row buffers grow with the chunk), fp16 with bias
    inp = build_inputs(36, 128, 64, 512, torch.float16, 77 + chunk, bias=True, len_lo=0, len_hi=128)
    got = run_fused(inp, torch.float16, 1, 0.04, chunk=chunk)
    check(inp, got, 1, 0.04)


@pytest.mark.parametrize("offset", [0, 1, 4], ids=["aligned", "odd", "8byte"])
@pytest.mark.parametrize("chunk", [None, 256], ids=["one_chunk", "chunks256"])
def test_gradient_output_alignment(offset, chunk):
    # dX, dW and dbias views 0, 2 or 8 bytes into their buffers: 16-byte aligned
    # outputs take the TMA stores, the others per-thread stores; nothing is
    # written before or after an output
    inp = build_inputs(2, 300, 136, 1000, torch.bfloat16, 4242 + offset, bias=True, len_lo=0, len_hi=300)
    got = run_fused(inp, torch.bfloat16, 0, 0.04, chunk=chunk, out_offset=offset)
    check(inp, got, 0, 0.04)


@pytest.mark.parametrize("tau", [0.7, 1.5])
@pytest.mark.parametrize("chunk", [None, 128], ids=["one_chunk", "chunks128"])
def test_temperature(tau, chunk):
    # logits (X W^T + b) / tau for both models; gradients with respect to the raw weights
    m = pl()
    dev = "cuda"
    inp = synth.fused_inputs(3, 100, 200, 1000, torch.bfloat16, 4343, bias=True, need_ref=True)
    _, logp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"], temperature=tau)
    old = torch.from_numpy(logp) + inp["old_noise"].double()
    d = torch.from_numpy(logp) - old - np.log(float(np.float32(1) + np.float32(EPS_HI)))
    old[d.abs() < 2e-4] -= 4e-4
    inp["old_lp"] = old.float()
    want = oracle.fused_grpo(inp["X"], inp["W"], inp["bias"], inp["targets"], inp["Xref"], inp["Wref"],
                             inp["old_lp"].reshape(3, 100), inp["adv"], inp["mask"], eps_lo=EPS_LO,
                             eps_hi=EPS_HI, beta=0.04, reduction=1, temperature=tau)
    bs, T, H, V, N = 3, 100, 200, 1000, 300
    g = {k: inp[k].to(dev) for k in ("X", "W", "bias", "targets", "Xref", "Wref", "old_lp", "adv", "mask")}
    loss = torch.zeros(1, device=dev)
    dX = torch.empty(N, H, dtype=torch.bfloat16, device=dev)
    dW = torch.empty(V, H, dtype=torch.bfloat16, device=dev)
    db = torch.empty(V, dtype=torch.bfloat16, device=dev)
    lp, rlp = torch.empty(N, device=dev), torch.empty(N, device=dev)
    nv = torch.zeros(1, dtype=torch.int64, device=dev)
    mode = m.PL_BF16 | m.PL_GRPO | (m.PL_CHUNK_ROWS(chunk) if chunk else 0)
    wsb = m.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, 1, 1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    m.check(m.pl_fused_linear_grpo_temp(g["X"], g["W"], g["bias"], g["targets"], g["Xref"], g["Wref"],
                                        g["old_lp"], g["adv"], g["mask"], bs, T, H, V, EPS_LO, EPS_HI, 0.04,
                                        tau, mode, loss, dX, dW, db, lp, rlp, nv, ws, wsb))
    torch.cuda.synchronize()
    assert m.pl_device_status(ws) == 0
    assert int(nv.item()) == want["n_valid"]
    assert np.max(np.abs(lp.cpu().double().numpy() - want["logp"])) <= 2e-3
    assert np.max(np.abs(rlp.cpu().double().numpy() - want["ref_logp"])) <= 2e-3
    assert abs(loss.item() - want["loss"]) <= 1e-3 * abs(want["loss"])
    for k, t in (("dX", dX), ("dW", dW), ("dbias", db)):
        assert rel_fro(t.cpu().double().numpy(), want[k]) <= 1e-2, k


def test_empty_batch_gives_zero_loss_and_zero_weight_gradients():
    # no rows: loss 0, n_valid 0, dW and dbias written as zeros (nothing to accumulate)
    m = pl()
    H, V = 128, 700
    W = synth.normal((V, H), 11, std=0.02).to(torch.bfloat16).cuda()
    b = synth.normal((V,), 12, std=0.01).to(torch.bfloat16).cuda()
    dW = torch.full((V, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    db = torch.full((V,), float("nan"), dtype=torch.bfloat16, device="cuda")
    loss = torch.full((1,), float("nan"), device="cuda")
    nv = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    empty16 = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    mode = m.PL_BF16 | m.PL_GRPO
    wsb = m.pl_fused_linear_grpo_workspace_bytes(0, 64, H, V, mode, 1, 1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    m.check(m.pl_fused_linear_grpo(empty16, W, b, torch.empty(0, dtype=torch.int64, device="cuda"), empty16, W,
                                   torch.empty(0, device="cuda"), torch.empty(0, device="cuda"),
                                   torch.empty(0, 64, dtype=torch.uint8, device="cuda"), 0, 64, H, V, EPS_LO,
                                   EPS_HI, 0.04, mode, loss, None, dW, db, None, None, nv, ws, wsb))
    torch.cuda.synchronize()
    assert m.pl_device_status(ws) == 0
    assert loss.item() == 0.0 and int(nv.item()) == 0
    assert torch.all(dW == 0) and torch.all(db == 0)


@pytest.mark.parametrize("red", [0, 1], ids=["bnpo", "grpo"])
def test_all_masked_batch(red):
    # every token masked: loss 0 through max(n, 1), every gradient exactly zero
    inp = build_inputs(2, 64, 128, 640, torch.bfloat16, 4444, bias=True)
    inp["mask"] = torch.zeros_like(inp["mask"])
    got = run_fused(inp, torch.bfloat16, red, 0.04)
    assert got["status"] == 0 and got["n_valid"] == 0
    assert got["loss"] == 0.0
    for k in ("dX", "dW", "dbias"):
        assert np.all(got[k] == 0.0), k
    want = oracle.fused_grpo(inp["X"], inp["W"], inp["bias"], inp["targets"], inp["Xref"], inp["Wref"],
                             inp["old_lp"].reshape(2, 64), inp["adv"], inp["mask"], eps_lo=EPS_LO, eps_hi=EPS_HI,
                             beta=0.04, reduction=red)
    assert want["loss"] == 0.0
    assert np.max(np.abs(got["logp"] - want["logp"])) <= 2e-3   # log-probs are still produced


def test_repeat_calls_are_bit_identical():
    inp = build_inputs(3, 100, 200, 1000, torch.bfloat16, 4545, bias=True)
    a = run_fused(inp, torch.bfloat16, 1, 0.04, chunk=128)
    b = run_fused(inp, torch.bfloat16, 1, 0.04, chunk=128)
    assert a["loss"] == b["loss"]
    for k in ("logp", "ref_logp", "dX", "dW", "dbias"):
        assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("beta", [0.04, 0.0], ids=["beta0.04", "beta0"])
def test_forward_last_wave_in_half_tiles(beta):
    # 256 rows x V = 40900 (80 vocabulary tiles of 512, the last one ragged) per model:
    # 160 forward tiles (80 at beta = 0) on 74 pairs leave a last wave of 12 (6) tiles,
    # which run as 256-wide halves with the tile512 fixture; the logsumexp partials
    # and the stored logits of those halves must be those of whole tiles
    m = pl()
    inp = build_inputs(2, 128, 128, 40900, torch.bfloat16, 5252, bias=True, len_lo=0, len_hi=128)
    try:
        for no_tail in (0, 1):
            assert m.pl_debug_set_gemm_tail(no_tail) == 0
            for red in (0, 1):
                got = run_fused(inp, torch.bfloat16, red, beta)
                check(inp, got, red, beta)
    finally:
        m.pl_debug_set_gemm_tail(0)
