"""CPU-side checks of the C ABI: the library loads, exports every declared entry
point, and rejects invalid arguments before touching the device."""
import re
from pathlib import Path

import pytest
import torch

import rl_post_policy_b200 as pl

INCLUDE = Path(__file__).resolve().parent.parent / "include"
FAKE = 0x10000  # never dereferenced: validation fails before any device call


def declared_symbols():
    names = set()
    for h in INCLUDE.glob("*.h"):
        text = h.read_text()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(pl_[a-z0-9_]+)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert {"pl_loss", "pl_loss_ex", "pl_fused_linear_grpo"} <= names
    for n in names:
        assert hasattr(pl._lib, n), f"{n} declared in include/ but not exported by libpl.so"


def test_binding_names_match_header():
    for n in declared_symbols():
        assert callable(getattr(pl, n)), f"binding lacks {n}"


def test_status_strings():
    for s in range(0, 9):
        assert pl.pl_status_string(s).startswith("PL_")
    assert pl.pl_version() >= 100


def _loss(**over):
    args = dict(policy_lp=FAKE, old_lp=FAKE, ref_lp=FAKE, adv=FAKE, mask=FAKE, bs=4, seq=8,
                eps_lo=0.2, eps_hi=0.28, beta=0.04, mode=pl.PL_BF16 | pl.PL_BNPO, loss_out=FAKE,
                grad_out=FAKE)
    args.update(over)
    return pl.pl_loss(**args, stream=0)


@pytest.mark.parametrize("over,code", [
    (dict(bs=-1), pl.PL_ERR_ARG),
    (dict(seq=-3), pl.PL_ERR_ARG),
    (dict(loss_out=None), pl.PL_ERR_ARG),
    (dict(policy_lp=None), pl.PL_ERR_ARG),
    (dict(old_lp=None), pl.PL_ERR_ARG),
    (dict(adv=None), pl.PL_ERR_ARG),
    (dict(mask=None), pl.PL_ERR_ARG),
    (dict(ref_lp=None), pl.PL_ERR_ARG),          # beta != 0 needs ref
    (dict(eps_lo=-0.1), pl.PL_ERR_ARG),
    (dict(eps_hi=float("nan")), pl.PL_ERR_ARG),
    (dict(beta=-1.0), pl.PL_ERR_ARG),
    (dict(mode=3 << 4), pl.PL_ERR_DTYPE),
    (dict(mode=2), pl.PL_ERR_ARG),                # reduction code 2 is not defined
    (dict(mode=pl.PL_BF16 | (1 << 12)), pl.PL_ERR_ARG),  # unknown bit
])
def test_loss_rejects_invalid_arguments(over, code):
    assert _loss(**over) == code


def test_loss_ex_rejects_small_workspace():
    need = pl.pl_loss_workspace_bytes(4, 8)
    rc = pl.pl_loss_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 0.2, 0.28, 0.04, pl.PL_BF16, FAKE, FAKE,
                       None, None, FAKE, need - 1, stream=0)
    assert rc == pl.PL_ERR_WORKSPACE
    rc = pl.pl_loss_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 0.2, 0.28, 0.04, pl.PL_BF16, FAKE, FAKE,
                       None, None, None, need, stream=0)
    assert rc == pl.PL_ERR_WORKSPACE


def test_workspace_sizes_grow_with_batch():
    assert pl.pl_loss_workspace_bytes(1, 10) <= pl.pl_loss_workspace_bytes(1000, 10)
    assert pl.pl_loss_workspace_bytes(16, 1024) >= 256 + 16 * 8


def test_fused_workspace_logits_slots():
    # The fused path's logits region holds one chunk-sized slot for one chunk, two
    # with several (a chunk's backward shares a launch with the next chunk's
    # forward), and three with several bf16 chunks and a weight gradient from three
    # chunks on (chunks 2i and 2i+1 make one dW contribution, so chunk 2i's dlogits
    # wait one launch).  A slot is C x ceil(V/64)*64 16-bit values.
    H, V, C = 256, 1000, 128
    slot = C * 1024 * 2

    def ws(bs, dtype, dW):
        mode = dtype | pl.PL_CHUNK_ROWS(C)
        return pl.pl_fused_linear_grpo_workspace_bytes(bs, C, H, V, mode, dW, 0)

    for dtype in (pl.PL_BF16, pl.PL_F16):
        # one chunk -> two chunks: one more slot, plus the fp32 dW accumulator with dW
        assert ws(2, dtype, 0) - ws(1, dtype, 0) >= slot
    # three chunks: bf16 with dW has a third slot, fp16 and bf16 without dW do not
    assert ws(3, pl.PL_BF16, 1) - ws(3, pl.PL_F16, 1) == slot
    assert ws(3, pl.PL_BF16, 0) == ws(3, pl.PL_F16, 0)
    # two chunks: the pair needs no third slot
    assert ws(2, pl.PL_BF16, 1) == ws(2, pl.PL_F16, 1)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_device_reports_cuda_error():
    assert _loss() in (pl.PL_ERR_CUDA, pl.PL_ERR_ARCH)


@pytest.mark.skipif(torch.cuda.is_available(), reason="would launch on fake pointers")
def test_beta_zero_allows_null_ref_validation():
    # beta == 0 and ref NULL passes validation (it then fails only for lack of a device)
    rc = _loss(ref_lp=None, beta=0.0)
    assert rc != pl.PL_ERR_ARG


@pytest.mark.parametrize("over,code", [
    (dict(N=-1), pl.PL_ERR_ARG),
    (dict(X=None), pl.PL_ERR_ARG),
    (dict(targets=None), pl.PL_ERR_ARG),
    (dict(grad_logp=None), pl.PL_ERR_ARG),          # gradients requested without dL/dlogp
    (dict(logp_out=None, dX=None, dW=None, dbias=None), pl.PL_ERR_ARG),  # nothing requested
    (dict(mode=pl.PL_F32), pl.PL_ERR_DTYPE),
    (dict(H=100), pl.PL_ERR_ALIGN),                  # 200-byte row pitch is not a multiple of 16
    (dict(mode=pl.PL_BF16 | 1), pl.PL_ERR_ARG),      # reduction bits are not part of this entry
    (dict(ws_bytes=16), pl.PL_ERR_WORKSPACE),
])
def test_selective_logprob_rejects_invalid_arguments(over, code):
    args = dict(X=FAKE, W=FAKE, bias=None, targets=FAKE, N=64, H=128, V=512, mode=pl.PL_BF16,
                grad_logp=FAKE, logp_out=FAKE, dX=FAKE, dW=FAKE, dbias=None, workspace=FAKE,
                ws_bytes=1 << 40)
    args.update(over)
    assert pl.pl_fused_selective_logprob(**args, stream=0) == code


def test_fused_rejects_invalid_arguments():
    base = dict(X=FAKE, W=FAKE, bias=None, targets=FAKE, Xref=FAKE, Wref=FAKE, old_lp=FAKE, adv=FAKE,
                mask=FAKE, bs=2, T=8, H=64, V=512, eps_lo=0.2, eps_hi=0.28, beta=0.04,
                mode=pl.PL_BF16 | pl.PL_GRPO, loss=FAKE, dX=None, dW=None, dbias=None, logp_out=None,
                ref_logp_out=None, n_valid_out=None, workspace=FAKE, ws_bytes=1 << 40)
    for over, code in [(dict(loss=None), pl.PL_ERR_ARG), (dict(Wref=None), pl.PL_ERR_ARG),
                       (dict(mode=pl.PL_F32), pl.PL_ERR_DTYPE), (dict(H=60), pl.PL_ERR_ALIGN),
                       (dict(X=FAKE + 8), pl.PL_ERR_ALIGN), (dict(ws_bytes=1), pl.PL_ERR_WORKSPACE),
                       (dict(eps_hi=-1.0), pl.PL_ERR_ARG), (dict(mode=pl.PL_BF16 | (1 << 10)), pl.PL_ERR_ARG)]:
        args = dict(base)
        args.update(over)
        assert pl.pl_fused_linear_grpo(**args, stream=0) == code, over
        assert pl.pl_fused_linear_grpo_temp(**args, temperature=1.0, stream=0) == code, over
    for tau in (0.0, -1.0, float("inf"), float("nan")):
        assert pl.pl_fused_linear_grpo_temp(**base, temperature=tau, stream=0) == pl.PL_ERR_ARG, tau


def test_scale_rejects_invalid_arguments():
    assert pl.pl_scale(FAKE, -1, pl.PL_BF16, FAKE, stream=0) == pl.PL_ERR_ARG
    assert pl.pl_scale(None, 10, pl.PL_BF16, FAKE, stream=0) == pl.PL_ERR_ARG
    assert pl.pl_scale(FAKE, 10, pl.PL_BF16, None, stream=0) == pl.PL_ERR_ARG
    assert pl.pl_scale(FAKE, 10, 3 << 4, FAKE, stream=0) == pl.PL_ERR_DTYPE
    assert pl.pl_scale(FAKE, 10, pl.PL_BF16 | pl.PL_GRPO, FAKE, stream=0) == pl.PL_ERR_ARG
    assert pl.pl_scale(None, 0, pl.PL_BF16, None, stream=0) == pl.PL_OK   # nothing to do


def _rkl(**over):
    args = dict(student=FAKE, teacher=FAKE, mask=None, N=8, V=512, mode=pl.PL_BF16, loss_out=FAKE,
                grad_out=FAKE, kl_rows_out=None, n_valid_out=None, workspace=FAKE * 16,
                ws_bytes=pl.pl_reverse_kl_workspace_bytes(8, 512))
    args.update(over)
    return pl.pl_reverse_kl(**args, stream=0)


@pytest.mark.parametrize("over,code", [
    (dict(student=None), pl.PL_ERR_ARG), (dict(teacher=None), pl.PL_ERR_ARG),
    (dict(loss_out=None), pl.PL_ERR_ARG), (dict(N=-1), pl.PL_ERR_ARG), (dict(V=0), pl.PL_ERR_ARG),
    (dict(mode=pl.PL_BF16 | pl.PL_GRPO), pl.PL_ERR_ARG), (dict(mode=3 << 4), pl.PL_ERR_DTYPE),
    (dict(student=FAKE + 1), pl.PL_ERR_ALIGN), (dict(grad_out=FAKE + 1), pl.PL_ERR_ALIGN),
    (dict(mode=pl.PL_F32, teacher=FAKE + 2), pl.PL_ERR_ALIGN), (dict(workspace=FAKE + 16), pl.PL_ERR_ALIGN),
    (dict(ws_bytes=100), pl.PL_ERR_WORKSPACE),
])
def test_reverse_kl_rejects_invalid_arguments(over, code):
    assert _rkl(**over) == code


@pytest.mark.skipif(torch.cuda.is_available(), reason="would launch on fake pointers")
def test_reverse_kl_valid_call_without_device():
    # element-aligned (not 16-byte aligned) pointers and a NULL workspace pass validation
    assert _rkl(student=FAKE + 2, workspace=None, ws_bytes=0) in (pl.PL_ERR_CUDA, pl.PL_ERR_ARCH)


def test_init_rejects_negative_batch():
    assert pl.pl_init(-1, stream=0) == pl.PL_ERR_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_init_without_device():
    assert pl.pl_init(16, stream=0) in (pl.PL_ERR_CUDA, pl.PL_ERR_ARCH)


def test_debug_gemm_out_rejects_invalid_arguments():
    base = dict(A=FAKE, a_mn=0, lda=64, B=FAKE, b_mn=0, ldb=64, D=FAKE, ldd=256, out_path=2, M=128, N=256,
                K=64, mode=pl.PL_BF16)
    for over, code in [(dict(out_path=3), pl.PL_ERR_ARG), (dict(out_path=-1), pl.PL_ERR_ARG),
                       (dict(ldd=255), pl.PL_ERR_ARG),           # ldd < N
                       (dict(ldd=258), pl.PL_ERR_ALIGN),         # TMA rows must be 16-byte pitched
                       (dict(N=254), pl.PL_ERR_ALIGN),           # and end on a 16-byte boundary
                       (dict(N=254, out_path=0), pl.PL_ERR_CUDA),  # row stores take any N (no device here)
                       (dict(D=FAKE + 4), pl.PL_ERR_ALIGN), (dict(mode=pl.PL_F32), pl.PL_ERR_DTYPE),
                       (dict(D=None), pl.PL_ERR_ARG)]:
        args = dict(base)
        args.update(over)
        assert pl.pl_debug_gemm_out(**args, stream=0) == code, over


def test_loss_path_knob_rejects_invalid_values():
    assert pl.pl_debug_set_loss_path(3) == pl.PL_ERR_ARG
    assert pl.pl_debug_set_loss_path(-1) == pl.PL_ERR_ARG
    assert pl.pl_debug_set_loss_path(0) == pl.PL_OK
