"""Thin Python binding of libpl.so (the C ABI declared in include/pl.h).

Every function here has the name of the C entry point it calls and does
argument marshalling only: torch tensors become device pointers, torch streams
become cudaStream_t handles.  All arithmetic runs in the library's CUDA
kernels.  If libpl.so has not been built, importing this package raises
ImportError: there is no fallback path.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

_PKG = Path(__file__).resolve().parent  # the package directory
LIB_PATH = _PKG / "libpl.so"

if not LIB_PATH.exists():
    raise ImportError(
        f"{LIB_PATH} is missing; build it with `python -m rl_post_policy_b200.build` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(str(LIB_PATH))

# ---- constants mirrored from include/pl.h --------------------------------------
PL_OK, PL_ERR_ARG, PL_ERR_DTYPE, PL_ERR_ALIGN, PL_ERR_WORKSPACE = 0, 1, 2, 3, 4
PL_ERR_ARCH, PL_ERR_CUDA, PL_ERR_DEVICE_TIMEOUT, PL_ERR_BAD_TARGET = 5, 6, 7, 8
PL_BNPO, PL_GRPO = 0, 1
PL_F32, PL_F16, PL_BF16 = 0 << 4, 1 << 4, 2 << 4
PL_ADV_LP_DTYPE = 1 << 8
PL_CLIP_TWO_SIDED = 1 << 9
PL_CHUNK_SHIFT = 16


def PL_CHUNK_ROWS(n: int) -> int:
    return ((n // 128) & 0xFF) << PL_CHUNK_SHIFT


_P, _I64, _U32, _F, _SZ, _I = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float,
                               ctypes.c_size_t, ctypes.c_int)

_lib.pl_loss.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _F, _F, _F, _U32, _P, _P, _P]
_lib.pl_loss.restype = _I
_lib.pl_loss_ex.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _F, _F, _F, _U32, _P, _P, _P, _P, _P,
                            _SZ, _P]
_lib.pl_loss_ex.restype = _I
_lib.pl_loss_static.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _F, _F, _F, _U32, _P, _P, _P, _P, _P,
                                _P]
_lib.pl_loss_static.restype = _I
_lib.pl_loss_workspace_bytes.argtypes = [_I64, _I64]
_lib.pl_loss_workspace_bytes.restype = _SZ
_lib.pl_fused_linear_grpo.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64,
                                      _F, _F, _F, _U32, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.pl_fused_linear_grpo.restype = _I
_lib.pl_fused_linear_grpo_temp.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64,
                                           _F, _F, _F, _F, _U32, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                                           _P]
_lib.pl_fused_linear_grpo_temp.restype = _I
_lib.pl_fused_linear_grpo_workspace_bytes.argtypes = [_I64, _I64, _I64, _I64, _U32, _I, _I]
_lib.pl_fused_linear_grpo_workspace_bytes.restype = _SZ
_lib.pl_fused_selective_logprob.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _U32, _P, _P, _P, _P, _P,
                                            _P, _SZ, _P]
_lib.pl_fused_selective_logprob.restype = _I
_lib.pl_fused_selective_logprob_workspace_bytes.argtypes = [_I64, _I64, _I64, _U32, _I, _I]
_lib.pl_fused_selective_logprob_workspace_bytes.restype = _SZ
_lib.pl_reverse_kl.argtypes = [_P, _P, _P, _I64, _I64, _U32, _P, _P, _P, _P, _P, _SZ, _P]
_lib.pl_reverse_kl.restype = _I
_lib.pl_reverse_kl_workspace_bytes.argtypes = [_I64, _I64]
_lib.pl_reverse_kl_workspace_bytes.restype = _SZ
_lib.pl_count_ratio.argtypes = [_P, _P, _P, _P]
_lib.pl_count_ratio.restype = _I
_lib.pl_init.argtypes = [_I64, _P]
_lib.pl_init.restype = _I
_lib.pl_scale.argtypes = [_P, _I64, _U32, _P, _P]
_lib.pl_scale.restype = _I
_lib.pl_device_status.argtypes = [_P, _P]
_lib.pl_device_status.restype = _I
_lib.pl_status_string.argtypes = [_I]
_lib.pl_status_string.restype = ctypes.c_char_p
_lib.pl_version.argtypes = []
_lib.pl_version.restype = _I
_lib.pl_debug_gemm.argtypes = [_P, _I, _I64, _P, _I, _I64, _P, _I64, _I64, _I64, _U32, _P]
_lib.pl_debug_gemm.restype = _I
_lib.pl_debug_gemm_out.argtypes = [_P, _I, _I64, _P, _I, _I64, _P, _I64, _I, _I64, _I64, _I64, _U32, _P]
_lib.pl_debug_gemm_out.restype = _I
_lib.pl_debug_timing.argtypes = [_I]
_lib.pl_debug_timing.restype = None
_lib.pl_debug_timing_read.argtypes = [_P, _P]
_lib.pl_debug_timing_read.restype = _I
_lib.pl_debug_set_wait.argtypes = [ctypes.c_ulonglong, ctypes.c_uint, ctypes.c_uint]
_lib.pl_debug_set_wait.restype = None
_lib.pl_debug_pair_tiles.argtypes = [_I, _I, _I, _I, _I, _P]
_lib.pl_debug_pair_tiles.restype = _I
_lib.pl_debug_set_loss_path.argtypes = [_I]
_lib.pl_debug_set_loss_path.restype = _I
_lib.pl_debug_pick_tile.argtypes = [_I, _P, _I]
_lib.pl_debug_pick_tile.restype = _I
_lib.pl_debug_set_gemm_tile.argtypes = [_I]
_lib.pl_debug_set_gemm_tile.restype = _I
_lib.pl_debug_set_rkl_cluster.argtypes = [_I]
_lib.pl_debug_set_rkl_cluster.restype = _I
_lib.pl_debug_set_gemm_tail.argtypes = [_I]
_lib.pl_debug_set_gemm_tail.restype = _I
_lib.pl_debug_tail_halves.argtypes = [_I, _I]
_lib.pl_debug_tail_halves.restype = _I
_lib.pl_debug_set_dw_finish.argtypes = [_I]
_lib.pl_debug_set_dw_finish.restype = _I
_lib.pl_debug_set_dw_pair.argtypes = [_I]
_lib.pl_debug_set_dw_pair.restype = _I
_lib.pl_debug_set_gemm_merge.argtypes = [_I]
_lib.pl_debug_set_gemm_merge.restype = _I
_lib.pl_debug_queue_tiles.argtypes = [_I, _P, _I, _I, _P]
_lib.pl_debug_queue_tiles.restype = _I
_lib.pl_debug_set_rkl_path.argtypes = [_I]
_lib.pl_debug_set_rkl_path.restype = _I
_lib.pl_debug_pick_split.argtypes = [_P, _I, _P]
_lib.pl_debug_pick_split.restype = _I
_lib.pl_debug_set_gemm_split.argtypes = [_I]
_lib.pl_debug_set_gemm_split.restype = _I
_lib.pl_debug_launch_count.argtypes = []
_lib.pl_debug_launch_count.restype = _I64

EXPORTED = ("pl_init", "pl_loss", "pl_loss_ex", "pl_loss_static", "pl_fused_linear_grpo_temp", "pl_fused_selective_logprob",
            "pl_fused_selective_logprob_workspace_bytes", "pl_reverse_kl", "pl_reverse_kl_workspace_bytes", "pl_scale", "pl_count_ratio", "pl_loss_workspace_bytes", "pl_fused_linear_grpo",
            "pl_fused_linear_grpo_workspace_bytes", "pl_device_status", "pl_status_string",
            "pl_version", "pl_debug_gemm", "pl_debug_gemm_out", "pl_debug_timing", "pl_debug_timing_read",
            "pl_debug_launch_count", "pl_debug_set_wait", "pl_debug_set_rkl_cluster", "pl_debug_set_gemm_tile", "pl_debug_pair_tiles",
            "pl_debug_pick_tile", "pl_debug_set_loss_path", "pl_debug_pick_split", "pl_debug_set_gemm_split",
            "pl_debug_set_rkl_path", "pl_debug_set_gemm_merge", "pl_debug_queue_tiles",
            "pl_debug_set_dw_finish", "pl_debug_set_gemm_tail", "pl_debug_tail_halves", "pl_debug_set_dw_pair")


class PLError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {pl_status_string(status)}")
        self.status = status


def _ptr(x):
    """Device pointer of a tensor, an int address, or NULL for None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def dtype_mode(dtype) -> int:
    import torch
    return {torch.float32: PL_F32, torch.float16: PL_F16, torch.bfloat16: PL_BF16}[dtype]


def check(status: int, where: str = "libpl") -> None:
    if status != PL_OK:
        raise PLError(status, where)


# ---- C entry points ---------------------------------------------------------------
def pl_init(max_bs, stream=None) -> int:
    return _lib.pl_init(max_bs, _stream(stream))


def pl_loss(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode, loss_out,
            grad_out, stream=None) -> int:
    return _lib.pl_loss(_ptr(policy_lp), _ptr(old_lp), _ptr(ref_lp), _ptr(adv), _ptr(mask), bs, seq,
                        eps_lo, eps_hi, beta, mode, _ptr(loss_out), _ptr(grad_out), _stream(stream))


def pl_loss_ex(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode, loss_out,
               grad_out, n_valid_out, row_valid_out, workspace, ws_bytes, stream=None) -> int:
    return _lib.pl_loss_ex(_ptr(policy_lp), _ptr(old_lp), _ptr(ref_lp), _ptr(adv), _ptr(mask), bs,
                           seq, eps_lo, eps_hi, beta, mode, _ptr(loss_out), _ptr(grad_out),
                           _ptr(n_valid_out), _ptr(row_valid_out), _ptr(workspace), ws_bytes,
                           _stream(stream))


def pl_loss_static(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode,
                   loss_out, grad_out, n_valid_out, row_valid_out, status_out, stream=None) -> int:
    """Allocation-free pl_loss_ex: scratch in a fixed array of libpl.so (bs <= 4096)."""
    return _lib.pl_loss_static(_ptr(policy_lp), _ptr(old_lp), _ptr(ref_lp), _ptr(adv), _ptr(mask), bs,
                               seq, eps_lo, eps_hi, beta, mode, _ptr(loss_out), _ptr(grad_out),
                               _ptr(n_valid_out), _ptr(row_valid_out), _ptr(status_out),
                               _stream(stream))


def pl_loss_workspace_bytes(bs, seq) -> int:
    return int(_lib.pl_loss_workspace_bytes(bs, seq))


def pl_fused_linear_grpo(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, bs, T, H, V, eps_lo,
                         eps_hi, beta, mode, loss, dX, dW, dbias, logp_out, ref_logp_out,
                         n_valid_out, workspace, ws_bytes, stream=None) -> int:
    return _lib.pl_fused_linear_grpo(
        _ptr(X), _ptr(W), _ptr(bias), _ptr(targets), _ptr(Xref), _ptr(Wref), _ptr(old_lp),
        _ptr(adv), _ptr(mask), bs, T, H, V, eps_lo, eps_hi, beta, mode, _ptr(loss), _ptr(dX),
        _ptr(dW), _ptr(dbias), _ptr(logp_out), _ptr(ref_logp_out), _ptr(n_valid_out),
        _ptr(workspace), ws_bytes, _stream(stream))


def pl_fused_linear_grpo_temp(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, bs, T, H, V, eps_lo,
                              eps_hi, beta, temperature, mode, loss, dX, dW, dbias, logp_out, ref_logp_out,
                              n_valid_out, workspace, ws_bytes, stream=None) -> int:
    return _lib.pl_fused_linear_grpo_temp(
        _ptr(X), _ptr(W), _ptr(bias), _ptr(targets), _ptr(Xref), _ptr(Wref), _ptr(old_lp),
        _ptr(adv), _ptr(mask), bs, T, H, V, eps_lo, eps_hi, beta, temperature, mode, _ptr(loss),
        _ptr(dX), _ptr(dW), _ptr(dbias), _ptr(logp_out), _ptr(ref_logp_out), _ptr(n_valid_out),
        _ptr(workspace), ws_bytes, _stream(stream))


def pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, need_dW, need_dbias) -> int:
    return int(_lib.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, int(need_dW),
                                                         int(need_dbias)))


def pl_fused_selective_logprob(X, W, bias, targets, N, H, V, mode, grad_logp, logp_out, dX, dW, dbias,
                               workspace, ws_bytes, stream=None) -> int:
    return _lib.pl_fused_selective_logprob(_ptr(X), _ptr(W), _ptr(bias), _ptr(targets), N, H, V, mode,
                                           _ptr(grad_logp), _ptr(logp_out), _ptr(dX), _ptr(dW),
                                           _ptr(dbias), _ptr(workspace), ws_bytes, _stream(stream))


def pl_fused_selective_logprob_workspace_bytes(N, H, V, mode, need_dW, need_dbias) -> int:
    return int(_lib.pl_fused_selective_logprob_workspace_bytes(N, H, V, mode, int(need_dW),
                                                               int(need_dbias)))


def pl_reverse_kl(student, teacher, mask, N, V, mode, loss_out, grad_out, kl_rows_out, n_valid_out, workspace,
                  ws_bytes, stream=None) -> int:
    return _lib.pl_reverse_kl(_ptr(student), _ptr(teacher), _ptr(mask), N, V, mode, _ptr(loss_out),
                              _ptr(grad_out), _ptr(kl_rows_out), _ptr(n_valid_out), _ptr(workspace), ws_bytes,
                              _stream(stream))


def pl_reverse_kl_workspace_bytes(N, V) -> int:
    return _lib.pl_reverse_kl_workspace_bytes(N, V)


def pl_scale(x, n, mode, scale, stream=None) -> int:
    return _lib.pl_scale(_ptr(x), n, mode, _ptr(scale), _stream(stream))


def pl_count_ratio(local, global_, factor_out, stream=None) -> int:
    return _lib.pl_count_ratio(_ptr(local), _ptr(global_), _ptr(factor_out), _stream(stream))


def pl_device_status(workspace=None, stream=None) -> int:
    return _lib.pl_device_status(_ptr(workspace), _stream(stream))


def pl_status_string(status: int) -> str:
    return _lib.pl_status_string(status).decode()


def pl_version() -> int:
    return int(_lib.pl_version())


def pl_debug_gemm(A, a_mn, lda, B, b_mn, ldb, D, M, N, K, mode, stream=None) -> int:
    """Test hook (include/pl_debug.h): plain GEMM through the tcgen05 kernel."""
    return _lib.pl_debug_gemm(_ptr(A), int(a_mn), lda, _ptr(B), int(b_mn), ldb, _ptr(D), M, N, K,
                              mode, _stream(stream))


def pl_debug_gemm_out(A, a_mn, lda, B, b_mn, ldb, D, ldd, out_path, M, N, K, mode, stream=None) -> int:
    """Test hook (include/pl_debug.h): the same GEMM through a chosen fp32 output path
    (0 row stores, 1 TMA store, 2 TMA add into D)."""
    return _lib.pl_debug_gemm_out(_ptr(A), int(a_mn), lda, _ptr(B), int(b_mn), ldb, _ptr(D), ldd, int(out_path),
                                  M, N, K, mode, _stream(stream))


def pl_debug_timing(enable: bool) -> None:
    _lib.pl_debug_timing(int(bool(enable)))


def pl_debug_timing_read():
    """((gemm_ms, loss_ms, other_ms), (gemm_launches, loss_launches, other_launches))."""
    ms = (ctypes.c_double * 3)()
    n = (ctypes.c_int64 * 3)()
    check(_lib.pl_debug_timing_read(ms, n), "pl_debug_timing_read")
    return tuple(ms), tuple(n)


def pl_debug_launch_count() -> int:
    return int(_lib.pl_debug_launch_count())


def pl_debug_set_wait(wait_ns: int, extra_arrivals: int = 0, extra_tx: int = 0) -> None:
    """Test knob (include/pl_debug.h): wait bound and wait-run-out injection."""
    _lib.pl_debug_set_wait(int(wait_ns), int(extra_arrivals), int(extra_tx))


def pl_debug_set_gemm_tile(nh: int) -> int:
    return _lib.pl_debug_set_gemm_tile(nh)


def pl_debug_set_rkl_cluster(cl: int) -> int:
    return _lib.pl_debug_set_rkl_cluster(cl)


def pl_debug_pair_tiles(t0: int, t1: int, c0: int, c1: int, pairs: int):
    """Test hook: (status, [pair running tile t for each t]) of the GEMM tile schedule."""
    out = (ctypes.c_int32 * max(t0 + t1, 1))()
    rc = _lib.pl_debug_pair_tiles(t0, t1, c0, c1, pairs, out)
    return int(rc), list(out)[: t0 + t1]


def pl_debug_pick_tile(problems, pairs: int) -> int:
    """Test hook: the GEMM launcher's tile width (1 or 2) for one or two (M, N, K) problems."""
    flat = [int(x) for mnk in problems for x in mnk]
    arr = (ctypes.c_int64 * max(len(flat), 1))(*flat)
    return int(_lib.pl_debug_pick_tile(len(problems), arr, pairs))


def pl_debug_pick_split(problems, pairs: int):
    """Test hook: the backward launch's K split of its dX problem (1 or 2) and the
    tile width that goes with it, for the (M, N, K) of dX and dW."""
    flat = [int(x) for mnk in problems for x in mnk]
    if len(flat) != 6:
        return -1, 0
    arr = (ctypes.c_int64 * 6)(*flat)
    nh = ctypes.c_int(0)
    split = int(_lib.pl_debug_pick_split(arr, pairs, ctypes.byref(nh)))
    return split, int(nh.value)


def pl_debug_set_rkl_path(path: int) -> int:
    """Test hook: reverse KL with a gradient -- 0 the default (the streaming kernel), 1 the
    streaming kernel, 2 the register-resident kernel where it applies."""
    return int(_lib.pl_debug_set_rkl_path(int(path)))


def pl_debug_set_gemm_tail(mode: int) -> int:
    """Test hook: 512-wide round-robin launches -- 0 the last partial wave in 256-wide halves
    where that helps (default), 1 never."""
    return int(_lib.pl_debug_set_gemm_tail(int(mode)))


def pl_debug_tail_halves(tiles: int, pairs: int) -> int:
    """Test hook: tiles of the last partial wave that run in halves (0: none)."""
    return int(_lib.pl_debug_tail_halves(int(tiles), int(pairs)))


def pl_debug_set_dw_pair(mode: int) -> int:
    """Test hook: several bf16 chunks -- 1 one dW job per chunk, 2 one per pair of chunks
    (K over both chunks' rows; the default, 0)."""
    return int(_lib.pl_debug_set_dw_pair(int(mode)))


def pl_debug_set_dw_finish(mode: int) -> int:
    """Test hook: several-chunk dW -- 1 fp32 add then a separate rounding kernel (the default, 0),
    2 the last chunk's epilogue adds the accumulator and stores the model dtype."""
    return int(_lib.pl_debug_set_dw_finish(int(mode)))


def pl_debug_set_gemm_merge(mode: int) -> int:
    """Test hook: several-chunk fused calls -- 0 merged backward/forward launches (default),
    1 separate launches, 2 merged launches with 4 epilogue warps."""
    return int(_lib.pl_debug_set_gemm_merge(int(mode)))


def pl_debug_queue_tiles(tiles, q_f0: int, q_w: int):
    """Test hook: the GEMM's dynamic tile-queue order for jobs of the given tile counts."""
    n = int(sum(tiles))
    arr = (ctypes.c_int32 * max(len(tiles), 1))(*[int(t) for t in tiles])
    out = (ctypes.c_int32 * max(n, 1))()
    rc = int(_lib.pl_debug_queue_tiles(len(tiles), arr, int(q_f0), int(q_w), out))
    return rc, list(out)[:n]


def pl_debug_set_gemm_split(mode: int) -> int:
    """Test hook: K split of the backward dX problem -- 0 the host's choice, 1 never, 2 always."""
    return int(_lib.pl_debug_set_gemm_split(int(mode)))


def pl_debug_set_loss_path(path: int) -> int:
    """Test hook: 0 default, 1 small-batch loss kernel when eligible, 2 cooperative kernel."""
    return int(_lib.pl_debug_set_loss_path(int(path)))
