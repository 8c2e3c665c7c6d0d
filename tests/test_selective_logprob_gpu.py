"""pl_fused_selective_logprob (the fused linear path without the loss step)
against the CPU oracle's selective log-prob and its backward with an external
dL/dlogp.  Tolerances as for the fused loss path: logp abs <= 2e-3, dX / dW /
dbias relative Frobenius <= 1e-2."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gemm_tile", "gemm_variant")]


def run(inp, dtype, grad_logp=None, chunk=None, want=("dX", "dW", "dbias"), targets=None):
    import rl_post_policy_b200 as pl
    dev = "cuda"
    N, H = inp["X"].shape
    V = inp["W"].shape[0]
    X, W = inp["X"].to(dev), inp["W"].to(dev)
    b = inp["bias"].to(dev) if inp["bias"] is not None else None
    tg = (targets if targets is not None else inp["targets"]).to(dev)
    g = grad_logp.to(dev) if grad_logp is not None else None
    lp = torch.full((N,), float("nan"), device=dev)
    dX = torch.full((N, H), float("nan"), dtype=dtype, device=dev) if (g is not None and "dX" in want) else None
    dW = torch.full((V, H), float("nan"), dtype=dtype, device=dev) if (g is not None and "dW" in want) else None
    db = (torch.full((V,), float("nan"), dtype=dtype, device=dev)
          if (g is not None and b is not None and "dbias" in want) else None)
    mode = pl.dtype_mode(dtype) | (pl.PL_CHUNK_ROWS(chunk) if chunk else 0)
    wsb = pl.pl_fused_selective_logprob_workspace_bytes(N, H, V, mode, dW is not None, db is not None)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    pl.check(pl.pl_fused_selective_logprob(X, W, b, tg, N, H, V, mode, g, lp, dX, dW, db, ws, wsb))
    torch.cuda.synchronize()
    status = pl.pl_device_status(ws)
    out = {"logp": lp.cpu().double().numpy(), "status": status}
    for k, t in (("dX", dX), ("dW", dW), ("dbias", db)):
        out[k] = None if t is None else t.cpu().double().numpy()
    return out


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("chunk", [None, 128], ids=["one_chunk", "chunks128"])
def test_forward_and_backward(dtype, chunk):
    inp = synth.fused_inputs(3, 100, 200, 1000, dtype, 515, bias=True, need_ref=False)
    N = 300
    g = synth.normal((N,), 516, std=1e-3)
    g[7] = 0.0  # a row with no upstream gradient
    lse, logp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"])
    fwd = run(inp, dtype, chunk=chunk)
    assert fwd["status"] == 0
    assert np.max(np.abs(fwd["logp"] - logp)) <= 2e-3
    got = run(inp, dtype, grad_logp=g, chunk=chunk)
    assert np.max(np.abs(got["logp"] - logp)) <= 2e-3
    wX, wW, wb = oracle.lm_head_backward(inp["X"], inp["W"], inp["bias"], inp["targets"], lse,
                                         g.double().numpy(), np.arange(N), np.arange(1000))
    assert rel(got["dX"], wX) <= 1e-2
    assert rel(got["dW"], wW) <= 1e-2
    assert rel(got["dbias"], wb) <= 1e-2
    assert np.all(got["dX"][7] == 0.0)


def test_partial_outputs_and_bad_target():
    import rl_post_policy_b200 as pl
    inp = synth.fused_inputs(1, 64, 64, 512, torch.bfloat16, 517, bias=False, need_ref=False)
    g = synth.normal((64,), 518, std=1e-2)
    bad = inp["targets"].clone()
    bad[3] = -1
    got = run(inp, torch.bfloat16, grad_logp=g, want=("dW",), targets=bad)
    assert got["status"] == pl.PL_ERR_BAD_TARGET
    assert np.isnan(got["logp"][3])
    lse, _, _ = oracle.lm_head_logprob(inp["X"], inp["W"], None, inp["targets"])
    gz = g.double().numpy().copy()
    gz[3] = 0.0
    _, wW, _ = oracle.lm_head_backward(inp["X"], inp["W"], None, inp["targets"], lse, gz, [], np.arange(512))
    assert rel(got["dW"], wW) <= 1e-2
