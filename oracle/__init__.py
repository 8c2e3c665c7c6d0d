"""Plain fp64 CPU oracle for the fused GRPO/BNPO policy loss -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it: the
GPU path and this oracle share no code, headers, tables or helpers.  The
arithmetic lives in ``pl_oracle.cpp`` (plain C++, fp64, std::thread); this
module only marshals arrays and composes the three steps the pages describe:

1. selective log-probability of the sampled token through the lm_head
   ("Add SM100 CuTe DSL GRPO fast path", Liger-Kernel PR #1363, "Summary"),
2. the PPO-clipped loss with the k3 KL penalty, reduced BNPO- or GRPO-style
   ("Geometric-AI Kernels" model card, "BNPO Loss" and "GRPO Loss"),
3. the backward pass to dX, dW and dbias (chain rule through log-softmax and
   the linear layer);

with the logits divided by a sampling temperature where one is given, and,
separately, the reverse-KL self-distillation loss and its student gradient
("Geometric-AI Kernels" model card, "Reverse KL").  Every function is pinned
by tests/test_oracle_pins.py and tests/test_oracle_reverse_kl.py against
closed forms, invariants, brute force, library routines and finite
differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np
import torch

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "pl_oracle.cpp"
_LIB_PATH = _HERE / "liborc.so"
_lib = None

BNPO, GRPO = 0, 1

_DT = {torch.float64: 0, torch.float32: 1, torch.float16: 2, torch.bfloat16: 3}


def build_library(force: bool = False) -> Path:
    """Compile pl_oracle.cpp into liborc.so (plain g++, no CUDA)."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["g++", "-O3", "-march=x86-64-v3", "-std=c++17", "-fPIC", "-shared",
               "-pthread", str(_SRC), "-o", str(tmp)]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build_library()
        lib = ctypes.CDLL(str(_LIB_PATH))
        P, I64, I32, D, F = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                             ctypes.c_double, ctypes.c_float)
        lib.orc_threads.argtypes = [I32]
        lib.orc_threads.restype = I32
        lib.orc_decode.argtypes = [I32, P, I64, P]
        lib.orc_decode.restype = I32
        lib.orc_policy_loss.argtypes = [P, P, P, P, P, I64, I64, F, F, D, I32, I32,
                                        P, P, P, P, P]
        lib.orc_policy_loss.restype = I32
        lib.orc_lm_head_logprob.argtypes = [P, I32, P, I32, P, I32, P, P, I64, I64, I64,
                                            I64, I32, D, P, P, P]
        lib.orc_lm_head_logprob.restype = I32
        lib.orc_lm_head_backward.argtypes = [P, I32, P, I32, P, I32, P, P, P, I64, I64,
                                             I64, I32, D, P, I64, P, P, I64, P, P]
        lib.orc_lm_head_backward.restype = I32
        lib.orc_reverse_kl.argtypes = [P, P, I32, P, I64, I64, I32, P, P, P, P]
        lib.orc_reverse_kl.restype = I32
        _lib = lib
    return _lib


def threads(requested: int = 0) -> int:
    """Worker threads the oracle uses (the process's CPU affinity count)."""
    return int(_load().orc_threads(requested))


def _t(x, floating: bool = True) -> torch.Tensor:
    t = x if isinstance(x, torch.Tensor) else torch.as_tensor(np.asarray(x))
    t = t.detach().to("cpu").contiguous()
    if floating and t.dtype not in _DT:
        raise TypeError(f"oracle: unsupported dtype {t.dtype}")
    return t


def _p(a):
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return ctypes.c_void_p(a.data_ptr())
    return a.ctypes.data_as(ctypes.c_void_p)


def decode(x) -> np.ndarray:
    """Exact fp64 value of every element of a f64/f32/f16/bf16 tensor."""
    t = _t(x)
    out = np.empty(t.numel(), dtype=np.float64)
    rc = _load().orc_decode(_DT[t.dtype], _p(t), t.numel(), _p(out))
    if rc:
        raise ValueError("oracle: decode failed")
    return out.reshape(tuple(t.shape))


def policy_loss(lp, old_lp, ref_lp, adv, mask, *, eps_lo: float, eps_hi: float,
                beta: float, reduction: int, two_sided: bool = False) -> dict:
    """PPO-clipped BNPO/GRPO loss and dLoss/dlp, all in fp64.

    ``lp``, ``old_lp``, ``ref_lp``: (bs, seq) of any float dtype (decoded exactly);
    ``adv``: (bs,); ``mask``: (bs, seq) bool/int8 (nonzero = valid).
    """
    lp64 = decode(lp)
    bs, seq = lp64.shape
    old64 = decode(old_lp).reshape(bs, seq)
    ref64 = decode(ref_lp).reshape(bs, seq) if ref_lp is not None else None
    adv64 = decode(adv).reshape(bs)
    m = _t(mask, False).to(torch.bool).to(torch.uint8).reshape(bs, seq).contiguous()
    loss = np.zeros(1)
    grad = np.zeros((bs, seq))
    nv = np.zeros(1, dtype=np.int64)
    rv = np.zeros(max(bs, 1), dtype=np.int64)
    ab = np.zeros(1)
    rc = _load().orc_policy_loss(_p(lp64), _p(old64), _p(ref64), _p(adv64), _p(m), bs, seq,
                                 float(eps_lo), float(eps_hi), float(beta), int(reduction),
                                 int(bool(two_sided)), _p(loss), _p(grad), _p(nv), _p(rv),
                                 _p(ab))
    if rc:
        raise ValueError(f"oracle: policy_loss rejected its arguments (rc={rc})")
    return {"loss": float(loss[0]), "grad": grad, "n_valid": int(nv[0]),
            "row_valid": rv[:bs].copy(), "abs_sum": float(ab[0])}


def lm_head_logprob(X, W, bias, targets, rows=None, nthreads: int = 0, temperature: float = 1.0):
    """(lse, logp, target_logit) for the selected rows (all rows if ``rows`` is None);
    logits are (X W^T + bias) / temperature."""
    Xt, Wt = _t(X), _t(W)
    N, H = Xt.shape
    V = Wt.shape[0]
    bt = _t(bias) if bias is not None else None
    tg = _t(targets, False).to(torch.int64).contiguous()
    ri = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = N if ri is None else len(ri)
    lse = np.zeros(n)
    logp = np.zeros(n)
    zt = np.zeros(n)
    rc = _load().orc_lm_head_logprob(_p(Xt), _DT[Xt.dtype], _p(Wt), _DT[Wt.dtype], _p(bt),
                                     _DT[bt.dtype] if bt is not None else 0, _p(tg), _p(ri),
                                     n, N, H, V, nthreads, float(temperature), _p(lse), _p(logp),
                                     _p(zt))
    if rc:
        raise ValueError(f"oracle: lm_head_logprob failed (rc={rc})")
    return lse, logp, zt


def lm_head_backward(X, W, bias, targets, lse, g, dx_rows, dw_rows, nthreads: int = 0,
                     temperature: float = 1.0):
    """(dX[dx_rows], dW[dw_rows], dbias[dw_rows]) in fp64 given per-row lse and g."""
    Xt, Wt = _t(X), _t(W)
    N, H = Xt.shape
    V = Wt.shape[0]
    bt = _t(bias) if bias is not None else None
    tg = _t(targets, False).to(torch.int64).contiguous()
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    g = np.ascontiguousarray(g, dtype=np.float64)
    dxr = np.ascontiguousarray(np.asarray(dx_rows, dtype=np.int64))
    dwr = np.ascontiguousarray(np.asarray(dw_rows, dtype=np.int64))
    dX = np.zeros((len(dxr), H))
    dW = np.zeros((len(dwr), H))
    db = np.zeros(len(dwr))
    rc = _load().orc_lm_head_backward(_p(Xt), _DT[Xt.dtype], _p(Wt), _DT[Wt.dtype], _p(bt),
                                      _DT[bt.dtype] if bt is not None else 0, _p(tg),
                                      _p(lse), _p(g), N, H, V, nthreads, float(temperature),
                                      _p(dxr), len(dxr),
                                      _p(dX), _p(dwr), len(dwr), _p(dW), _p(db))
    if rc:
        raise ValueError(f"oracle: lm_head_backward failed (rc={rc})")
    return dX, dW, db


def fused_grpo(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, *, eps_lo: float,
               eps_hi: float, beta: float, reduction: int, two_sided: bool = False,
               dx_rows="all", dw_rows="all", nthreads: int = 0, temperature: float = 1.0) -> dict:
    """Fused linear GRPO/BNPO forward + backward, composed from the three steps.

    ``mask`` is (bs, T); the N = bs*T rows of X are sequence-major.  The
    reference model has no bias.  ``dx_rows`` / ``dw_rows`` select which rows of
    dX and dW (and dbias) to evaluate ("all" or an index list).
    """
    m = _t(mask, False)
    bs, T = m.shape
    Xt = _t(X)
    N, H = Xt.shape
    V = _t(W).shape[0]
    if N != bs * T:
        raise ValueError("oracle: X rows must equal bs*T")
    lse, logp, _ = lm_head_logprob(X, W, bias, targets, None, nthreads, temperature)
    if beta != 0.0:
        _, ref_logp, _ = lm_head_logprob(Xref, Wref, None, targets, None, nthreads, temperature)
    else:
        ref_logp = None
    lo = policy_loss(logp.reshape(bs, T), old_lp, None if ref_logp is None else ref_logp.reshape(bs, T),
                     adv, m, eps_lo=eps_lo, eps_hi=eps_hi, beta=beta, reduction=reduction,
                     two_sided=two_sided)
    g = lo["grad"].reshape(N)
    dxr = np.arange(N) if isinstance(dx_rows, str) else np.asarray(dx_rows, dtype=np.int64)
    dwr = np.arange(V) if isinstance(dw_rows, str) else np.asarray(dw_rows, dtype=np.int64)
    dX, dW, db = lm_head_backward(X, W, bias, targets, lse, g, dxr, dwr, nthreads, temperature)
    return {"loss": lo["loss"], "abs_sum": lo["abs_sum"], "n_valid": lo["n_valid"],
            "row_valid": lo["row_valid"], "logp": logp, "ref_logp": ref_logp, "lse": lse,
            "g": g, "dX": dX, "dW": dW, "dbias": db, "dx_rows": dxr, "dw_rows": dwr}


def reverse_kl(student, teacher, mask=None, *, want_grad: bool = True, nthreads: int = 0) -> dict:
    """Reverse-KL self-distillation KL(softmax(student) || softmax(teacher)) per row,
    masked mean over rows (denominator max(n_valid, 1)), and its gradient with
    respect to the student logits, all in fp64.

    ``student``, ``teacher``: (..., V) of one float dtype (decoded exactly);
    ``mask``: shape of the leading dims, nonzero = valid, or None (all valid).
    Returns loss, grad (same shape as student, or None), kl_rows (leading
    shape; every row) and n_valid.
    """
    s = _t(student)
    t = _t(teacher)
    if s.shape != t.shape or s.dtype != t.dtype:
        raise ValueError("oracle: student and teacher must share shape and dtype")
    lead = tuple(s.shape[:-1])
    V = int(s.shape[-1])
    N = int(np.prod(lead)) if lead else 1
    m = None
    if mask is not None:
        m = _t(mask, False).to(torch.bool).to(torch.uint8).reshape(N).contiguous()
    loss = np.zeros(1)
    grad = np.zeros((N, V)) if want_grad else None
    kl = np.zeros(max(N, 1))
    nv = np.zeros(1, dtype=np.int64)
    rc = _load().orc_reverse_kl(_p(s), _p(t), _DT[s.dtype], _p(m), N, V, nthreads, _p(loss),
                                _p(grad), _p(kl), _p(nv))
    if rc:
        raise ValueError(f"oracle: reverse_kl rejected its arguments (rc={rc})")
    return {"loss": float(loss[0]), "grad": None if grad is None else grad.reshape(lead + (V,)),
            "kl_rows": kl[:N].reshape(lead), "n_valid": int(nv[0])}
