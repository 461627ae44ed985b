"""Thin Python binding of libsk.so (the sketched linear layer's C ABI).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  Importing
this module fails loudly when the library has not been built; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsk.so")

SK_OK = 0
SK_OP_FWD, SK_OP_BWD_INPUT, SK_OP_BWD_LUT = 0, 1, 2
SK_CHECK_TASK_RANGE = 1
SK_CHECK_INDEX_RANGE = 2
SK_CHECK_TIMEOUT = 4
SK_CHECK_NOT_SPD = 8
SK_CHECK_LUT_ORDER = 16

EXPORTED = (
    "sk_abi_version", "sk_status_string", "sk_last_error", "sk_packed_row_bytes", "sk_packed_bytes",
    "sk_pack", "sk_unpack", "sk_dequant", "sk_workspace_bytes", "sk_linear_fwd", "sk_linear_fwd_group",
    "sk_linear_bwd_input",
    "sk_linear_bwd_lut", "sk_linear_bwd_lut_noalloc", "sk_bin_counts", "sk_lut_adamw", "sk_lut_sgd",
    "sk_device_check", "sk_inverse_factor_workspace_bytes", "sk_sketch_round_workspace_bytes", "sk_gram",
    "sk_inverse_factor", "sk_lloyd", "sk_sketch_round",
)


SK_MAX_GROUP_LAYERS = 8


class _Layer(ctypes.Structure):
    """sk_layer of sk.h: one layer of a grouped forward."""
    _fields_ = [("packed", ctypes.c_void_p), ("lut", ctypes.c_void_p), ("gpr", ctypes.c_int),
                ("n", ctypes.c_int64), ("d", ctypes.c_int64), ("X", ctypes.c_void_p), ("Y", ctypes.c_void_p)]


class SketchError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m compressive_fine_tuning_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    f64 = ctypes.c_double
    sigs = {
        "sk_abi_version": ([], i32),
        "sk_status_string": ([i32], ctypes.c_char_p),
        "sk_last_error": ([], ctypes.c_char_p),
        "sk_packed_row_bytes": ([i64, i32], sz),
        "sk_packed_bytes": ([i64, i64, i32], sz),
        "sk_pack": ([vp, i64, i64, i32, vp, sz, vp], i32),
        "sk_unpack": ([vp, i64, i64, i32, vp, vp], i32),
        "sk_dequant": ([vp, vp, i32, i32, i64, i64, i32, i32, vp, vp], i32),
        "sk_workspace_bytes": ([i32, i64, i64, i32, i32, i64, i32], sz),
        "sk_linear_fwd": ([vp, vp, i32, i32, i64, i64, vp, i64, vp, i32, vp, vp, sz, vp], i32),
        "sk_linear_fwd_group": ([ctypes.POINTER(_Layer), i32, i32, i64, vp, i32, vp], i32),
        "sk_linear_bwd_input": ([vp, vp, i32, i32, i64, i64, vp, i64, vp, i32, vp, vp, sz, vp], i32),
        "sk_linear_bwd_lut": ([vp, i32, i32, i64, i64, vp, vp, i64, vp, i32, vp, i32, vp, sz, vp], i32),
        "sk_linear_bwd_lut_noalloc": ([vp, i32, i32, i64, i64, vp, vp, i64, vp, i32, vp, i32, vp], i32),
        "sk_bin_counts": ([vp, i32, i32, i64, i64, vp, vp], i32),
        "sk_lut_adamw": ([vp, vp, vp, vp, vp, i32, i64, i32, i32, f32, f32, f32, f32, f32, i32, vp, vp], i32),
        "sk_lut_sgd": ([vp, vp, vp, i32, i64, i32, i32, f32, vp, vp], i32),
        "sk_device_check": ([ctypes.POINTER(ctypes.c_uint32), i32, vp], i32),
        "sk_inverse_factor_workspace_bytes": ([i64], sz),
        "sk_sketch_round_workspace_bytes": ([i64, i64], sz),
        "sk_gram": ([vp, i64, i64, vp, i32, vp], i32),
        "sk_inverse_factor": ([vp, i64, f64, vp, vp, vp, sz, vp], i32),
        "sk_lloyd": ([vp, vp, i32, i32, i64, i64, i32, vp, vp, vp], i32),
        "sk_sketch_round": ([vp, vp, vp, i32, i32, i64, i64, vp, vp, sz, vp], i32),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def _check(status: int) -> None:
    if status != SK_OK:
        name = lib.sk_status_string(status).decode()
        raise SketchError(status, f"{name}: {lib.sk_last_error().decode()}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, ndim: Optional[int] = None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def packed_row_bytes(d: int, bits: int) -> int:
    return int(lib.sk_packed_row_bytes(d, bits))


def packed_bytes(n: int, d: int, bits: int) -> int:
    return int(lib.sk_packed_bytes(n, d, bits))


def workspace_bytes(op: int, n: int, d: int, bits: int, gpr: int, T: int, ntask: int) -> int:
    return int(lib.sk_workspace_bytes(op, n, d, bits, gpr, T, ntask))


def _workspace(op, n, d, bits, gpr, T, ntask, device):
    nb = workspace_bytes(op, n, d, bits, gpr, T, ntask)
    if nb == 0:
        return None, 0
    return torch.empty(nb, dtype=torch.uint8, device=device), nb


def pack(idx: torch.Tensor, bits: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """uint8 [n, d] indices -> uint8 [n, packed_row_bytes] packed rows (on the GPU)."""
    _need(idx, torch.uint8, "idx", 2)
    n, d = idx.shape
    rb = packed_row_bytes(d, bits)
    if out is None:
        out = torch.empty((n, max(rb, 1)), dtype=torch.uint8, device=idx.device)
    _need(out, torch.uint8, "out")
    _check(lib.sk_pack(_ptr(idx), n, d, bits, _ptr(out), out.numel(), _stream(idx.device)))
    return out


def unpack(packed: torch.Tensor, n: int, d: int, bits: int) -> torch.Tensor:
    _need(packed, torch.uint8, "packed")
    out = torch.empty((n, d), dtype=torch.uint8, device=packed.device)
    _check(lib.sk_unpack(_ptr(packed), n, d, bits, _ptr(out), _stream(packed.device)))
    return out


def _lut_shape(lut: torch.Tensor, bits: int):
    _need(lut, torch.float16, "lut", 4)
    ntask, n, gpr, k = lut.shape
    if k != (1 << bits):
        raise ValueError(f"lut's last dimension must be 2**bits = {1 << bits}")
    return ntask, n, gpr


def dequant(packed: torch.Tensor, lut: torch.Tensor, bits: int, d: int, task: int = 0) -> torch.Tensor:
    """Dense bf16 [n, d] effective weight of LUT set `task` (test / comparison aid)."""
    ntask, n, gpr = _lut_shape(lut, bits)
    _need(packed, torch.uint8, "packed")
    out = torch.empty((n, d), dtype=torch.bfloat16, device=lut.device)
    _check(lib.sk_dequant(_ptr(packed), _ptr(lut), bits, gpr, n, d, task, ntask, _ptr(out), _stream(lut.device)))
    return out


def _task_arg(task: Optional[torch.Tensor], T: int):
    if task is None:
        return None
    _need(task, torch.int32, "task", 1)
    if task.numel() != T:
        raise ValueError("task must hold one id per token")
    return task


def linear_fwd(packed: torch.Tensor, lut: torch.Tensor, bits: int, X: torch.Tensor,
               task: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y [T, n] = X Theta_hat^T (bf16 in, bf16 out, fp32 accumulation)."""
    ntask, n, gpr = _lut_shape(lut, bits)
    _need(X, torch.bfloat16, "X", 2)
    _need(packed, torch.uint8, "packed")
    T, d = X.shape
    task = _task_arg(task, T)
    if out is None:
        out = torch.empty((T, n), dtype=torch.bfloat16, device=X.device)
    _need(out, torch.bfloat16, "out", 2)
    ws, nb = _workspace(SK_OP_FWD, n, d, bits, gpr, T, ntask, X.device)
    _check(lib.sk_linear_fwd(_ptr(packed), _ptr(lut), bits, gpr, n, d, _ptr(X), T, _ptr(task), ntask,
                             _ptr(out), _ptr(ws), nb, _stream(X.device)))
    return out


def linear_fwd_group(layers, bits: int, task: Optional[torch.Tensor] = None, outs=None):
    """Y_l = X_l Theta_hat_l^T for a list of layers (packed, lut, X) that see the
    same number of tokens, in one library call (one launch at decode sizes).
    Returns the list of Y_l; `outs` may give them."""
    if not 1 <= len(layers) <= SK_MAX_GROUP_LAYERS:
        raise ValueError(f"1 to {SK_MAX_GROUP_LAYERS} layers per group")
    arr = (_Layer * len(layers))()
    T = None
    ntask = None
    ys = []
    for i, (packed, lut, X) in enumerate(layers):
        nt, n, gpr = _lut_shape(lut, bits)
        _need(X, torch.bfloat16, "X", 2)
        _need(packed, torch.uint8, "packed")
        if T is None:
            T, ntask = X.shape[0], nt
        elif X.shape[0] != T or nt != ntask:
            raise ValueError("every layer of a group must see the same tokens and LUT sets")
        Y = outs[i] if outs is not None else torch.empty((T, n), dtype=torch.bfloat16, device=X.device)
        _need(Y, torch.bfloat16, "out", 2)
        ys.append(Y)
        arr[i] = _Layer(packed.data_ptr(), lut.data_ptr(), gpr, n, X.shape[1], X.data_ptr(), Y.data_ptr())
    task = _task_arg(task, T)
    _check(lib.sk_linear_fwd_group(arr, len(layers), bits, T, _ptr(task), ntask, _stream(layers[0][2].device)))
    return ys


def linear_bwd_input(packed: torch.Tensor, lut: torch.Tensor, bits: int, d: int, dY: torch.Tensor,
                     task: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """dX [T, d] = dY Theta_hat."""
    ntask, n, gpr = _lut_shape(lut, bits)
    _need(dY, torch.bfloat16, "dY", 2)
    _need(packed, torch.uint8, "packed")
    T = dY.shape[0]
    if dY.shape[1] != n:
        raise ValueError("dY must be [T, n]")
    task = _task_arg(task, T)
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=dY.device)
    _need(out, torch.bfloat16, "out", 2)
    ws, nb = _workspace(SK_OP_BWD_INPUT, n, d, bits, gpr, T, ntask, dY.device)
    _check(lib.sk_linear_bwd_input(_ptr(packed), _ptr(lut), bits, gpr, n, d, _ptr(dY), T, _ptr(task), ntask,
                                   _ptr(out), _ptr(ws), nb, _stream(dY.device)))
    return out


def linear_bwd_lut(packed: torch.Tensor, bits: int, gpr: int, X: torch.Tensor, dY: torch.Tensor,
                   task: Optional[torch.Tensor] = None, ntask: int = 1, out: Optional[torch.Tensor] = None,
                   accumulate: bool = False) -> torch.Tensor:
    """dlut [ntask, n, gpr, k] fp32: the binned dY^T X of the corrected Eq. 6."""
    _need(X, torch.bfloat16, "X", 2)
    _need(dY, torch.bfloat16, "dY", 2)
    _need(packed, torch.uint8, "packed")
    T, d = X.shape
    n = dY.shape[1]
    if dY.shape[0] != T:
        raise ValueError("X and dY must have the same number of tokens")
    task = _task_arg(task, T)
    k = 1 << bits
    if out is None:
        out = torch.empty((ntask, n, gpr, k), dtype=torch.float32, device=X.device)
    _need(out, torch.float32, "out")
    ws, nb = _workspace(SK_OP_BWD_LUT, n, d, bits, gpr, T, ntask, X.device)
    _check(lib.sk_linear_bwd_lut(_ptr(packed), bits, gpr, n, d, _ptr(X), _ptr(dY), T, _ptr(task), ntask,
                                 _ptr(out), int(accumulate), _ptr(ws), nb, _stream(X.device)))
    return out


def device_check(clear: bool = True, device=None) -> int:
    """Synchronise and return the device check word (SK_CHECK_* bits)."""
    device = torch.device("cuda") if device is None else torch.device(device)
    flags = ctypes.c_uint32(0)
    st = lib.sk_device_check(ctypes.byref(flags), int(clear), _stream(device))
    if st not in (SK_OK, 4):
        _check(st)
    return int(flags.value)


def bin_counts(packed: torch.Tensor, bits: int, gpr: int, n: int, d: int) -> torch.Tensor:
    """Static bin sizes counts[i][g][c] of the index map (int32 [n, gpr, 2^bits])."""
    _need(packed, torch.uint8, "packed")
    out = torch.empty((n, gpr, 1 << bits), dtype=torch.int32, device=packed.device)
    _check(lib.sk_bin_counts(_ptr(packed), bits, gpr, n, d, _ptr(out), _stream(packed.device)))
    return out


def _lut_update_shape(master: torch.Tensor, bits: int):
    if master.dtype != torch.float32 or master.dim() != 4 or master.shape[-1] != (1 << bits) or not master.is_contiguous():
        raise ValueError("master LUTs must be contiguous fp32 [ntask, n, gpr, 2^bits]")
    return master.shape[0], master.shape[1], master.shape[2]


def lut_adamw_(master: torch.Tensor, m: torch.Tensor, v: torch.Tensor, grad: torch.Tensor, bits: int, step: int,
               lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
               counts: Optional[torch.Tensor] = None, lut: Optional[torch.Tensor] = None) -> None:
    """One AdamW step on fp32 master LUTs (in place); writes the fp16 LUTs when given.
    counts (from bin_counts) selects the averaging variant of the gradient."""
    ntask, n, gpr = _lut_update_shape(master, bits)
    for t, name in ((m, "m"), (v, "v"), (grad, "grad")):
        if t.shape != master.shape or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name} must match the master LUTs")
    if lut is not None and (lut.shape != master.shape or lut.dtype != torch.float16 or not lut.is_contiguous()):
        raise ValueError("lut must be contiguous fp16 of the master's shape")
    _check(lib.sk_lut_adamw(_ptr(master), _ptr(m), _ptr(v), _ptr(grad), _ptr(counts), ntask, n, gpr, bits, lr, beta1,
                            beta2, eps, weight_decay, step, _ptr(lut), _stream(master.device)))


def lut_sgd_(master: torch.Tensor, grad: torch.Tensor, bits: int, lr: float, counts: Optional[torch.Tensor] = None,
             lut: Optional[torch.Tensor] = None) -> None:
    """One SGD step on fp32 master LUTs (in place); writes the fp16 LUTs when given."""
    ntask, n, gpr = _lut_update_shape(master, bits)
    if grad.shape != master.shape or grad.dtype != torch.float32 or not grad.is_contiguous():
        raise ValueError("grad must match the master LUTs")
    if lut is not None and (lut.shape != master.shape or lut.dtype != torch.float16 or not lut.is_contiguous()):
        raise ValueError("lut must be contiguous fp16 of the master's shape")
    _check(lib.sk_lut_sgd(_ptr(master), _ptr(grad), _ptr(counts), ntask, n, gpr, bits, lr, _ptr(lut),
                          _stream(master.device)))


# ---------------------------------------------------------------------------
# Sketching stage: dense weight + calibration activations -> index map + LUTs
# ---------------------------------------------------------------------------

def gram(X: torch.Tensor, H: Optional[torch.Tensor] = None, accumulate: bool = False) -> torch.Tensor:
    """H = X^T X (fp32 [d, d]) of bf16 calibration activations X [s, d];
    H += X^T X when accumulate."""
    _need(X, torch.bfloat16, "X", 2)
    s, d = X.shape
    if H is None:
        H = torch.empty((d, d), dtype=torch.float32, device=X.device)
    _need(H, torch.float32, "H", 2)
    _check(lib.sk_gram(_ptr(X), s, d, _ptr(H), int(accumulate), _stream(X.device)))
    return H


def inverse_factor(H: torch.Tensor, damp: float = 0.01):
    """(U, hinv_diag): the upper factor U of the damped H^-1 (H^-1 = U^T U,
    float64 [d, d]) and the diagonal of H^-1 (float64 [d])."""
    _need(H, torch.float32, "H", 2)
    d = H.shape[0]
    U = torch.empty((d, d), dtype=torch.float64, device=H.device)
    hd = torch.empty(d, dtype=torch.float64, device=H.device)
    nb = int(lib.sk_inverse_factor_workspace_bytes(d))
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=H.device)
    _check(lib.sk_inverse_factor(_ptr(H), d, float(damp), _ptr(U), _ptr(hd), _ptr(ws), nb, _stream(H.device)))
    return U, hd


def lloyd(theta: torch.Tensor, hinv_diag: torch.Tensor, bits: int, gpr: int, max_iter: int = 100):
    """(lut fp16 [n, gpr, 2^bits], updates run int32 [n, gpr]): weighted
    Lloyd's centroids of every (row, group) of theta (fp32 [n, d])."""
    _need(theta, torch.float32, "theta", 2)
    _need(hinv_diag, torch.float64, "hinv_diag", 1)
    n, d = theta.shape
    lut = torch.empty((n, gpr, 1 << bits), dtype=torch.float16, device=theta.device)
    iters = torch.empty((n, gpr), dtype=torch.int32, device=theta.device)
    _check(lib.sk_lloyd(_ptr(theta), _ptr(hinv_diag), bits, gpr, n, d, max_iter, _ptr(lut), _ptr(iters),
                        _stream(theta.device)))
    return lut, iters


def sketch_round(theta: torch.Tensor, U: torch.Tensor, lut: torch.Tensor, bits: int) -> torch.Tensor:
    """Index map (uint8 [n, d]) of theta against the ascending fp16 LUTs
    [n, gpr, 2^bits], with error compensation through U."""
    _need(theta, torch.float32, "theta", 2)
    _need(U, torch.float64, "U", 2)
    _need(lut, torch.float16, "lut", 3)
    n, d = theta.shape
    gpr = lut.shape[1]
    idx = torch.empty((n, d), dtype=torch.uint8, device=theta.device)
    nb = int(lib.sk_sketch_round_workspace_bytes(n, d))
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=theta.device)
    _check(lib.sk_sketch_round(_ptr(theta), _ptr(U), _ptr(lut), bits, gpr, n, d, _ptr(idx), _ptr(ws), nb,
                               _stream(theta.device)))
    return idx


def sketch_layer(theta: torch.Tensor, X: torch.Tensor, bits: int, gpr: int, damp: float = 0.01,
                 max_iter: int = 100, H: Optional[torch.Tensor] = None):
    """The sketching stage of one layer: (packed index map, fp16 LUTs
    [n, gpr, 2^bits], index map uint8 [n, d]).  H, when given, is the
    calibration Gram matrix already accumulated (X is then ignored)."""
    if H is None:
        H = gram(X)
    U, hd = inverse_factor(H, damp)
    lut, _ = lloyd(theta, hd, bits, gpr, max_iter)
    idx = sketch_round(theta, U, lut, bits)
    return pack(idx, bits), lut, idx


class SketchedLinearFunction(torch.autograd.Function):
    """Y = X Theta_hat^T with gradients for X and for the LUT values only.

    `lut` is the trainable tensor that receives the LUT gradient; `lut16` holds
    the fp16 tables the kernels read (the same tensor when `lut` is fp16, else
    the round-to-nearest-even fp16 of an fp32 master).  The LUT gradient is
    computed in fp32 and returned in `lut`'s dtype: an fp32 master gets it
    unrounded."""

    @staticmethod
    def forward(ctx, X, lut, lut16, packed, bits, task):
        Y = linear_fwd(packed, lut16, bits, X.contiguous(), task)
        ctx.save_for_backward(X, lut16, packed, task if task is not None else torch.empty(0))
        ctx.bits = bits
        ctx.has_task = task is not None
        ctx.lut_dtype = lut.dtype
        return Y

    @staticmethod
    def backward(ctx, dY):
        X, lut16, packed, task = ctx.saved_tensors
        task = task if ctx.has_task else None
        dY = dY.contiguous().to(torch.bfloat16)
        dX = dlut = None
        if ctx.needs_input_grad[0]:
            dX = linear_bwd_input(packed, lut16, ctx.bits, X.shape[1], dY, task)
        if ctx.needs_input_grad[1]:
            ntask, n, gpr, _ = lut16.shape
            dlut = linear_bwd_lut(packed, ctx.bits, gpr, X, dY, task, ntask)
            if dlut.dtype != ctx.lut_dtype:
                dlut = dlut.to(ctx.lut_dtype)
        return dX, dlut, None, None, None, None


def sketched_linear(X: torch.Tensor, lut: torch.Tensor, packed: torch.Tensor, bits: int,
                    task: Optional[torch.Tensor] = None, lut16: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = X Theta_hat^T as an autograd function of X and of the LUT values.

    lut: fp32 master LUTs (their gradient stays fp32) or fp16 LUTs (their
    gradient is rounded to fp16).  lut16: the fp16 tables of an fp32 master,
    when the caller keeps them (else they are rounded from `lut` here)."""
    if lut16 is None:
        lut16 = lut if lut.dtype == torch.float16 else lut.detach().to(torch.float16)
    return SketchedLinearFunction.apply(X, lut, lut16, packed, bits, task)


class SketchedLinear(torch.nn.Module):
    """A linear layer (no bias) whose weight is the sketch Theta_hat: a frozen
    packed index map (buffer), trainable fp32 master LUTs [ntask, n, gpr,
    2**bits] (parameter `lut`, whose gradient is the library's fp32 LUT
    gradient) and the fp16 tables the kernels read (buffer `lut16`, the
    round-to-nearest-even of the master).  forward(X, task) takes bf16
    activations [..., d]; task holds one LUT-set id per token (int32), or None
    for set 0.

    `lut16` follows the master: `adamw_step` / `sgd_step` update both in one
    library call; any other in-place change of `lut` (a torch optimizer) is
    noticed by its version counter and `lut16` is rounded again before the
    next forward."""

    def __init__(self, packed: torch.Tensor, lut: torch.Tensor, bits: int, in_features: int):
        super().__init__()
        self.register_buffer("packed", packed)
        self.lut = torch.nn.Parameter(lut.detach().to(torch.float32).contiguous())
        self.register_buffer("lut16", lut.detach().to(torch.float16).contiguous())
        self.bits = bits
        self.in_features = in_features
        self.out_features = lut.shape[1]
        self._synced = self._lut_state()

    def _lut_state(self):
        return (self.lut.data_ptr(), self.lut._version)

    def _sync_lut16(self):
        if self._lut_state() != self._synced:
            with torch.no_grad():
                self.lut16.copy_(self.lut)
            self._synced = self._lut_state()

    @classmethod
    def from_dense(cls, weight: torch.Tensor, X_calib: torch.Tensor, bits: int, gpr: int, ntask: int = 1,
                   damp: float = 0.01, max_iter: int = 100) -> "SketchedLinear":
        """Sketch a dense weight [n, d] with calibration activations [s, d]
        (bf16); every LUT set starts from the same learned centroids."""
        packed, lut, _ = sketch_layer(weight.float().contiguous(), X_calib, bits, gpr, damp, max_iter)
        return cls(packed, lut.unsqueeze(0).repeat(ntask, 1, 1, 1).contiguous(), bits, weight.shape[1])

    def forward(self, X: torch.Tensor, task: Optional[torch.Tensor] = None) -> torch.Tensor:
        self._sync_lut16()
        lead = X.shape[:-1]
        Y = sketched_linear(X.reshape(-1, self.in_features).to(torch.bfloat16).contiguous(), self.lut, self.packed,
                            self.bits, task, lut16=self.lut16)
        return Y.reshape(*lead, self.out_features)

    def adamw_step(self, m: torch.Tensor, v: torch.Tensor, step: int, lr: float, beta1: float = 0.9,
                   beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
                   counts: Optional[torch.Tensor] = None) -> None:
        """One AdamW step of the master LUTs from their gradient; rewrites lut16."""
        self._sync_lut16()
        lut_adamw_(self.lut.data, m, v, self.lut.grad, self.bits, step, lr, beta1, beta2, eps, weight_decay,
                   counts, self.lut16)

    def sgd_step(self, lr: float, counts: Optional[torch.Tensor] = None) -> None:
        """One SGD step of the master LUTs from their gradient; rewrites lut16."""
        self._sync_lut16()
        lut_sgd_(self.lut.data, self.lut.grad, self.bits, lr, counts, self.lut16)
