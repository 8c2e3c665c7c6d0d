"""The seeded input recipes (synth/) against their stated distributions and
structure: the parity tests and the benchmark rely on these shapes, value
ranges and masks, so a change to a recipe should fail here first.  Statistics
are checked with tolerances several standard errors wide."""
import math

import pytest
import torch

import synth


def test_seed_formula():
    assert synth.seed_for(0) == 0x5EED0000
    assert synth.seed_for(4, 3) == 0x5EED0000 + 16 * 4 + 3


def test_same_seed_same_bits_other_seed_other_bits():
    a = synth.loss_inputs(4, 300, torch.bfloat16, 11)
    b = synth.loss_inputs(4, 300, torch.bfloat16, 11)
    c = synth.loss_inputs(4, 300, torch.bfloat16, 12)
    for k in ("policy_lp", "old_lp", "ref_lp", "adv", "mask"):
        assert torch.equal(a[k], b[k]), k
    assert not torch.equal(a["policy_lp"], c["policy_lp"])


def test_loss_recipe():
    bs, seq = 64, 4096
    d = synth.loss_inputs(bs, seq, torch.float32, 5, len_lo=64, len_hi=1024)
    pol, old, ref = d["policy_lp"], d["old_lp"], d["ref_lp"]
    assert pol.dtype == torch.float32 and pol.shape == (bs, seq)
    assert bool((pol <= 0).all())                                   # -2|N(0,1)|
    assert abs(pol.mean().item() + 2 * math.sqrt(2 / math.pi)) < 0.02
    assert abs((old - pol).std().item() - 0.1) < 0.002
    assert abs((ref - pol).std().item() - 0.05) < 0.001
    assert d["adv"].shape == (bs,) and d["adv"].dtype == torch.float32
    lens = d["lengths"]
    assert int(lens.min()) >= 64 and int(lens.max()) <= 1024
    m = d["mask"]
    assert m.dtype == torch.int8 and torch.equal(m.sum(1).to(torch.int64), lens)
    # a prefix: no valid token after an invalid one
    assert bool((m[:, 1:] <= m[:, :-1]).all())


def test_loss_recipe_rounds_each_dtype_from_the_same_master():
    a = synth.loss_inputs(2, 512, torch.float32, 9)
    b = synth.loss_inputs(2, 512, torch.bfloat16, 9)
    assert torch.equal(a["policy_lp"].to(torch.bfloat16), b["policy_lp"])
    assert torch.equal(a["mask"], b["mask"])


@pytest.mark.parametrize("fully_masked_last", [False, True])
def test_fused_recipe(fully_masked_last):
    bs, T, H, V = 4, 256, 128, 3000
    d = synth.fused_inputs(bs, T, H, V, torch.float32, 21, bias=True, len_lo=1, len_hi=T,
                           fully_masked_last=fully_masked_last, need_ref=True)
    N = bs * T
    assert d["X"].shape == (N, H) and d["W"].shape == (V, H) and d["bias"].shape == (V,)
    assert abs(d["X"].std().item() - 1.0) < 0.01
    assert abs(d["W"].std().item() - 0.02) < 0.0005
    assert abs((d["Xref"] - d["X"]).std().item() - 0.01) < 0.0003
    assert abs((d["Wref"] - d["W"]).std().item() - 0.002) < 0.00005
    assert abs(d["bias"].std().item() - 0.01) < 0.001
    t = d["targets"]
    assert t.dtype == torch.int64 and int(t.min()) >= 0 and int(t.max()) < V
    assert abs(d["old_noise"].std().item() - 0.1) < 0.005
    lens = d["lengths"]
    assert torch.equal(d["mask"].sum(1).to(torch.int64), lens)
    if fully_masked_last:
        assert int(lens[-1]) == 0
    else:
        assert int(lens.min()) >= 1


def test_fused_recipe_without_reference():
    d = synth.fused_inputs(1, 8, 16, 40, torch.bfloat16, 3, need_ref=False)
    assert d["Xref"] is None and d["Wref"] is None and d["bias"] is None


def test_reverse_kl_recipe():
    d = synth.reverse_kl_inputs(8, 64, 2000, torch.float32, 7)
    assert d["student"].shape == (8, 64, 2000)
    assert abs(d["student"].std().item() - 1.0) < 0.01
    assert abs(torch.corrcoef(torch.stack([d["student"].flatten(), d["teacher"].flatten()]))[0, 1].item()) < 0.01
    keep = d["mask"].float().mean().item()                      # uniform(0,1) > 0.2
    assert abs(keep - 0.8) < 0.06
    close = synth.reverse_kl_inputs(2, 4, 5000, torch.float32, 7, teacher_std=0.05)
    assert abs((close["teacher"] - close["student"]).std().item() - 0.05) < 0.001


def test_workload_table_matches_the_published_shapes():
    w = synth.WORKLOADS
    assert (w[2]["bs"] * w[2]["T"], w[2]["H"], w[2]["V"]) == (1024, 4096, 128256)
    assert w[2]["dtype"] == torch.bfloat16
    assert synth.RKL_WORKLOADS[1]["V"] == 248320
