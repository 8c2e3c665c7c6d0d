"""Parity of pl_reverse_kl (reverse-KL self-distillation, forward and student
gradient) with the CPU oracle.

Tolerances, from the kernel's arithmetic (fp32 statistics of exactly decoded
inputs; ex2.approx has a relative error of a few 2^-23; a CTA's slice sums at
most a few hundred terms per thread before fixed-order tree merges):
  * per-row kl: |gpu - oracle| <= 1e-5 + 1e-4 |oracle|;  loss: relative 1e-4;
  * gradient: relative Frobenius <= 1e-2 in bf16/fp16 (the output rounding,
    about 2^-9 RMS, dominates) and <= 1e-4 in fp32;
  * n_valid exact; masked rows' gradient and kl exactly zero.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("rkl_path")]


def pl():
    import rl_post_policy_b200 as m
    return m


def run(s, t, mask, grad=True, kl_rows=True, views=None, fetch_grad=True):
    m = pl()
    dev = "cuda"
    V = s.shape[-1]
    N = s.numel() // V
    if views is None:
        S, T = s.to(dev).contiguous(), t.to(dev).contiguous()
        G = torch.full_like(S, float("nan")) if grad else None
    else:
        S, T, G = views
    M = mask.to(dev).contiguous() if mask is not None else None
    loss = torch.full((1,), float("nan"), device=dev)
    kl = torch.full((N,), float("nan"), device=dev) if kl_rows else None
    nv = torch.full((1,), -1, dtype=torch.int64, device=dev)
    wsb = m.pl_reverse_kl_workspace_bytes(N, V)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    m.check(m.pl_reverse_kl(S, T, M, N, V, m.dtype_mode(s.dtype), loss, G, kl, nv, ws, wsb), "pl_reverse_kl")
    torch.cuda.synchronize()
    return {"loss": loss.item(), "n_valid": int(nv.item()),
            "kl": None if kl is None else kl.cpu().double().numpy(),
            "grad": None if (G is None or not fetch_grad) else G.float().cpu().double().numpy().reshape(N, V),
            "G": G}


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def check(got, want, mask, dtype, N, V):
    assert got["n_valid"] == want["n_valid"]
    assert abs(got["loss"] - want["loss"]) <= 1e-4 * abs(want["loss"]) + 1e-7, (got["loss"], want["loss"])
    valid = np.ones(N, bool) if mask is None else mask.reshape(-1).numpy() != 0
    if got["kl"] is not None:
        wk = want["kl_rows"].reshape(-1)
        err = np.abs(got["kl"] - wk)
        assert np.all(err[valid] <= 1e-5 + 1e-4 * np.abs(wk[valid])), err[valid].max()
        assert np.all(got["kl"][~valid] == 0.0)
    if got["grad"] is not None:
        wg = want["grad"].reshape(N, V)
        assert rel(got["grad"], wg) <= (1e-4 if dtype == torch.float32 else 1e-2)
        assert np.all(got["grad"][~valid] == 0.0)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32], ids=["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("grad", [True, False], ids=["fwd_bwd", "fwd"])
def test_small_ragged(dtype, grad):
    # V = 1001: rows start at every offset mod 16, so each row has a scalar head and tail
    inp = synth.reverse_kl_inputs(3, 37, 1001, dtype, synth.seed_for(40))
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"], want_grad=grad)
    got = run(inp["student"], inp["teacher"], inp["mask"], grad=grad)
    check(got, want, inp["mask"], dtype, 111, 1001)


@pytest.mark.parametrize("cl", [1, 2, 4, 8])
def test_every_cluster_split(cl):
    m = pl()
    inp = synth.reverse_kl_inputs(2, 20, 5000, torch.bfloat16, synth.seed_for(41, cl))
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"])
    assert m.pl_debug_set_rkl_cluster(cl) == 0
    try:
        got = run(inp["student"], inp["teacher"], inp["mask"])
    finally:
        m.pl_debug_set_rkl_cluster(0)
    check(got, want, inp["mask"], torch.bfloat16, 40, 5000)


@pytest.mark.parametrize("cl", [1, 8])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_many_rows_per_cluster_with_masked_runs(cl, dtype):
    # Several rows per cluster, so a row's gradient pass runs inside the next
    # valid row's statistics pass: masked rows first, in runs between valid
    # rows, and last; one valid row alone at the end of a cluster's rows.
    m = pl()
    bs, seq, V = 3, 400, 2048
    inp = synth.reverse_kl_inputs(bs, seq, V, dtype, synth.seed_for(47, cl))
    mask = inp["mask"].reshape(-1).clone()
    mask[:5] = 0
    mask[100:160] = 0
    mask[300:302] = 0
    mask[-7:] = 0
    mask[-9] = 1
    mask = mask.reshape(bs, seq)
    want = oracle.reverse_kl(inp["student"], inp["teacher"], mask)
    assert m.pl_debug_set_rkl_cluster(cl) == 0
    try:
        got = run(inp["student"], inp["teacher"], mask)
    finally:
        m.pl_debug_set_rkl_cluster(0)
    check(got, want, mask, dtype, bs * seq, V)


@pytest.mark.parametrize("cl", [1, 2, 4])
def test_rows_dealt_by_kind_across_row_blocks(cl):
    # Valid rows are dealt to the clusters by their rank among valid rows and
    # masked rows by theirs, in blocks of 512 rows: here the masked rows all
    # come first (a plain round-robin would give every cluster the same share
    # of them), the run of valid rows crosses two block boundaries, and the
    # last block is partial; without a mask every row is valid.
    m = pl()
    bs, seq, V = 3, 500, 1544
    inp = synth.reverse_kl_inputs(bs, seq, V, torch.bfloat16, synth.seed_for(48, cl))
    mask = torch.ones(bs * seq, dtype=torch.uint8)
    mask[:700] = 0
    mask[1100] = 0
    mask = mask.reshape(bs, seq)
    assert m.pl_debug_set_rkl_cluster(cl) == 0
    try:
        for mk in (mask, None):
            want = oracle.reverse_kl(inp["student"], inp["teacher"], mk)
            got = run(inp["student"], inp["teacher"], mk)
            check(got, want, mk, torch.bfloat16, bs * seq, V)
    finally:
        m.pl_debug_set_rkl_cluster(0)


def test_close_teacher_small_kl():
    # teacher = student + N(0, 0.05): kl ~ 1e-3, the cancellation-prone regime
    inp = synth.reverse_kl_inputs(4, 16, 32000, torch.bfloat16, synth.seed_for(42), teacher_std=0.05)
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"])
    got = run(inp["student"], inp["teacher"], inp["mask"])
    check(got, want, inp["mask"], torch.bfloat16, 64, 32000)


def test_no_mask_identical_teacher_and_all_masked():
    inp = synth.reverse_kl_inputs(2, 8, 700, torch.bfloat16, synth.seed_for(43))
    s = inp["student"]
    got = run(s, s.clone(), None)
    assert got["n_valid"] == 16 and got["loss"] == 0.0 and np.all(got["kl"] == 0.0)
    assert np.all(got["grad"] == 0.0)
    want = oracle.reverse_kl(s, inp["teacher"], None)
    check(run(s, inp["teacher"], None), want, None, torch.bfloat16, 16, 700)
    none = run(s, inp["teacher"], torch.zeros(2, 8, dtype=torch.uint8))
    assert none["loss"] == 0.0 and none["n_valid"] == 0 and np.all(none["grad"] == 0.0)


def test_empty_batch():
    s = torch.zeros(0, 64, dtype=torch.bfloat16)
    got = run(s, s.clone(), torch.zeros(0, dtype=torch.uint8), kl_rows=False)
    assert got["loss"] == 0.0 and got["n_valid"] == 0


@pytest.mark.parametrize("shift", [(1, 1, 1), (1, 1, 0), (0, 3, 0)], ids=["same_offset", "grad_offset", "teacher_offset"])
def test_misaligned_views(shift):
    # element-aligned views at different offsets mod 16: the vector path needs a shared
    # offset (same_offset: vectors after a scalar head), otherwise every element is scalar
    inp = synth.reverse_kl_inputs(2, 9, 777, torch.bfloat16, synth.seed_for(44))
    N, V = 18, 777
    views = []
    for src, k in zip((inp["student"], inp["teacher"], None), shift):
        buf = torch.zeros(N * V + 8, dtype=torch.bfloat16, device="cuda")
        v = buf[k:k + N * V].view(N, V)
        if src is not None:
            v.copy_(src.reshape(N, V))
        else:
            v.fill_(float("nan"))
        views.append(v)
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"])
    got = run(inp["student"], inp["teacher"], inp["mask"], views=tuple(views))
    check(got, want, inp["mask"], torch.bfloat16, N, V)


def test_deterministic():
    inp = synth.reverse_kl_inputs(4, 32, 20000, torch.bfloat16, synth.seed_for(45))
    a = run(inp["student"], inp["teacher"], inp["mask"])
    b = run(inp["student"], inp["teacher"], inp["mask"])
    assert a["loss"] == b["loss"] and np.array_equal(a["kl"], b["kl"]) and np.array_equal(a["grad"], b["grad"])


@pytest.mark.slow
@pytest.mark.parametrize("workload", [1, 2])
def test_full_size_sampled_rows(workload):
    # the benchmarked shapes; the oracle's gradient on sampled rows (a row's gradient
    # is its own softmax quantity times mask_r / n_valid, so the sample is rescaled)
    w = synth.RKL_WORKLOADS[workload]
    bs, seq, V = w["bs"], w["seq"], w["V"]
    N = bs * seq
    inp = synth.reverse_kl_inputs(bs, seq, V, w["dtype"], synth.seed_for(46, workload))
    got = run(inp["student"], inp["teacher"], inp["mask"], fetch_grad=False)
    full = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"], want_grad=False)
    check(got, full, inp["mask"], w["dtype"], N, V)
    mask = inp["mask"].reshape(-1)
    rng = np.random.default_rng(workload)
    valid_rows = np.nonzero(mask.numpy())[0]
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(valid_rows, 6, replace=False)]))
    s = inp["student"].reshape(N, V)[torch.from_numpy(rows)]
    t = inp["teacher"].reshape(N, V)[torch.from_numpy(rows)]
    sub = oracle.reverse_kl(s, t, mask[torch.from_numpy(rows)])
    wg = sub["grad"] * (max(sub["n_valid"], 1) / max(full["n_valid"], 1))
    g_rows = got["G"].reshape(N, V)[torch.from_numpy(rows).cuda()].float().cpu().double().numpy()
    assert rel(g_rows, wg) <= 1e-2
    for i, r in enumerate(rows):
        if mask[r] == 0:
            assert np.all(g_rows[i] == 0.0)
    # every row of the gradient sums to zero (softmax Jacobian): a full-size property
    G = got["G"].reshape(N, V).float()
    assert torch.all(G.sum(dim=1).abs() <= 1e-3 * G.abs().sum(dim=1) + 1e-30)


def test_python_entry_points():
    from rl_post_policy_b200 import autograd as ag
    from rl_post_policy_b200 import losses
    inp = synth.reverse_kl_inputs(2, 16, 3000, torch.bfloat16, synth.seed_for(47))
    s = inp["student"].cuda()
    t = inp["teacher"].cuda()
    m = inp["mask"].cuda()
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"])
    loss, grad = losses.reverse_kl(s, t, m)
    assert abs(loss.item() - want["loss"]) <= 1e-4 * abs(want["loss"])
    assert abs(losses.reverse_kl_fwd(s, t, m).item() - loss.item()) <= 1e-6 * abs(loss.item())
    x = s.clone().requires_grad_(True)
    l2 = ag.reverse_kl_autograd(x, t, m)
    (3.0 * l2).backward()
    assert torch.equal(x.grad, (grad.float() * 3.0).to(torch.bfloat16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32], ids=["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("grad", [True, False], ids=["fwd_bwd", "fwd"])
def test_aligned_rows(dtype, grad):
    # V = 3000: every row starts on a 16-byte boundary in every dtype (no scalar head or tail)
    inp = synth.reverse_kl_inputs(2, 24, 3000, dtype, synth.seed_for(49))
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"], want_grad=grad)
    got = run(inp["student"], inp["teacher"], inp["mask"], grad=grad)
    check(got, want, inp["mask"], dtype, 48, 3000)


@pytest.mark.parametrize("V,cl", [(40008, 0), (16, 8), (8, 2)], ids=["five_slots_last_partial", "empty_slices",
                                                                  "one_vector"])
def test_resident_slices(V, cl):
    # The register-resident kernel's edges: a slice of several 8 KB slots whose last
    # slot is partial (V = 40008 takes two CTAs of 20008 columns), and clusters whose
    # last CTAs own no columns at all; many rows per cluster with masked rows between.
    m = pl()
    inp = synth.reverse_kl_inputs(3, 70, V, torch.bfloat16, synth.seed_for(50, V))
    mask = inp["mask"].reshape(-1).clone()
    mask[:3] = 0
    mask[50:90] = 0
    mask = mask.reshape(3, 70)
    want = oracle.reverse_kl(inp["student"], inp["teacher"], mask)
    assert m.pl_debug_set_rkl_cluster(cl) == 0
    try:
        got = run(inp["student"], inp["teacher"], mask)
    finally:
        m.pl_debug_set_rkl_cluster(0)
    check(got, want, mask, torch.bfloat16, 210, V)
