"""Thin ctypes binding of libgecko.so (the C ABI declared in include/gecko.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There
is no fallback: if the library is missing or cannot load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgecko.so")

# Symbols declared in include/gecko.h
EXPORTS = (
    "gecko_sca_awm_forward",
    "gecko_sca_awm_forward_continue",
    "gecko_sca_awm_forward_noalloc",
    "gecko_sca_awm_forward_train",
    "gecko_sca_awm_backward",
    "gecko_awm_state",
    "gecko_cema_forward",
    "gecko_tdnorm_forward",
    "gecko_awm_segment_logsum",
    "gecko_awm_segment_maps",
    "gecko_awm_cp_logz",
    "gecko_awm_cp_state",
    "gecko_device_status",
    "gecko_timing_enable",
    "gecko_timing_read",
    "gecko_timing_read_backward",
    "gecko_last_error",
    "gecko_release",
)

# Stages timed by gecko_timing_read, in order.
STAGES = ("awm_stats", "awm_chunk", "awm_carry", "awm_readout", "sca")
# Stages timed by gecko_timing_read_backward, in order.
BWD_STAGES = ("awm_rebuild", "awm_backward", "sca_delta", "sca_dkdv", "sca_dq")

GECKO_F32, GECKO_BF16 = 0, 1
STATUS = {
    0: "GECKO_OK", 1: "GECKO_ERR_ARG", 2: "GECKO_ERR_SHAPE", 3: "GECKO_ERR_ALIGN",
    4: "GECKO_ERR_ALLOC", 5: "GECKO_ERR_CUDA", 6: "GECKO_ERR_NO_STATE", 7: "GECKO_ERR_TIMEOUT",
    8: "GECKO_ERR_LIMIT",
}

_lib = None


class GeckoError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


def load() -> ctypes.CDLL:
    """Load libgecko.so once; raise if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m long_context_sequence_sca_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    lib.gecko_sca_awm_forward.argtypes = [vp] * 7 + [i64] * 5 + [ctypes.c_int, vp]
    lib.gecko_sca_awm_forward.restype = ctypes.c_int
    lib.gecko_sca_awm_forward_continue.argtypes = [vp] * 9 + [i64] * 5 + [ctypes.c_int, vp]
    lib.gecko_sca_awm_forward_continue.restype = ctypes.c_int
    lib.gecko_sca_awm_forward_noalloc.argtypes = [vp] * 7 + [i64] * 5 + [ctypes.c_int, vp]
    lib.gecko_sca_awm_forward_noalloc.restype = ctypes.c_int
    lib.gecko_sca_awm_forward_train.argtypes = [vp] * 9 + [i64] * 5 + [ctypes.c_int, vp]
    lib.gecko_sca_awm_forward_train.restype = ctypes.c_int
    lib.gecko_sca_awm_backward.argtypes = [vp] * 15 + [i64] * 5 + [ctypes.c_int, vp]
    lib.gecko_sca_awm_backward.restype = ctypes.c_int
    lib.gecko_awm_state.argtypes = [vp, vp, i64, i64, i64, vp]
    lib.gecko_awm_state.restype = ctypes.c_int
    lib.gecko_cema_forward.argtypes = [vp] * 10 + [i64] * 4 + [ctypes.c_int, vp]
    lib.gecko_cema_forward.restype = ctypes.c_int
    f32 = ctypes.c_float
    lib.gecko_tdnorm_forward.argtypes = [vp] * 4 + [i64] * 4 + [f32, f32, f32, ctypes.c_int, vp]
    lib.gecko_tdnorm_forward.restype = ctypes.c_int
    ci = ctypes.c_int
    lib.gecko_awm_segment_logsum.argtypes = [vp, vp] + [i64] * 5 + [ci, vp]
    lib.gecko_awm_segment_logsum.restype = ci
    lib.gecko_awm_segment_maps.argtypes = [vp] * 4 + [i64] * 5 + [ci, vp]
    lib.gecko_awm_segment_maps.restype = ci
    lib.gecko_awm_cp_logz.argtypes = [vp, ci, ci, vp, i64, i64, i64, vp]
    lib.gecko_awm_cp_logz.restype = ci
    lib.gecko_awm_cp_state.argtypes = [vp, vp, ci, ci, vp, i64, i64, i64, vp]
    lib.gecko_awm_cp_state.restype = ci
    lib.gecko_device_status.argtypes = [vp]
    lib.gecko_device_status.restype = ctypes.c_int
    lib.gecko_timing_enable.argtypes = [ctypes.c_int]
    lib.gecko_timing_enable.restype = ctypes.c_int
    lib.gecko_timing_read.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
    lib.gecko_timing_read.restype = ctypes.c_int
    lib.gecko_timing_read_backward.argtypes = lib.gecko_timing_read.argtypes
    lib.gecko_timing_read_backward.restype = ctypes.c_int
    lib.gecko_last_error.argtypes = []
    lib.gecko_last_error.restype = ctypes.c_char_p
    lib.gecko_release.argtypes = []
    lib.gecko_release.restype = None
    _lib = lib
    return lib


def _check(rc: int):
    if rc != 0:
        raise GeckoError(rc, load().gecko_last_error().decode())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


# ------------------------------------------------------- raw C entry points --

def gecko_sca_awm_forward(q, k, v, qm, km, out_sca, out_mem, B, H, T, c, d, dtype, stream) -> int:
    """Direct call of the C entry point with integer pointers; returns the status."""
    return load().gecko_sca_awm_forward(q, k, v, qm, km, out_sca, out_mem, B, H, T, c, d, dtype, stream)


def gecko_sca_awm_forward_continue(q, k, v, qm, km, out_sca, out_mem, state_in, state_out, B, H, T, c, d, dtype,
                                   stream) -> int:
    """Forward of one segment of a longer sequence (state_in 0 = fresh)."""
    return load().gecko_sca_awm_forward_continue(q, k, v, qm, km, out_sca, out_mem, state_in, state_out,
                                                 B, H, T, c, d, dtype, stream)


def gecko_sca_awm_forward_noalloc(q, k, v, qm, km, out_sca, out_mem, B, H, T, c, d, dtype, stream) -> int:
    """The no-allocation entry point (fixed library scratch instead of a
    growable workspace), with integer pointers; returns the status."""
    return load().gecko_sca_awm_forward_noalloc(q, k, v, qm, km, out_sca, out_mem, B, H, T, c, d, dtype, stream)


def gecko_sca_awm_forward_train(q, k, v, qm, km, out_sca, out_mem, lse, out_sca_lo, B, H, T, c, d, dtype,
                                stream) -> int:
    """The forward that also writes SCA's row log-sum-exp and (if out_sca_lo
    is not 0) the rounding residual of out_sca, for the backward."""
    return load().gecko_sca_awm_forward_train(q, k, v, qm, km, out_sca, out_mem, lse, out_sca_lo, B, H, T, c, d,
                                              dtype, stream)


def gecko_sca_awm_backward(q, k, v, qm, km, out_sca, out_sca_lo, lse, dout_sca, dout_mem, dq, dk, dv, dqm, dkm,
                           B, H, T, c, d, dtype, stream) -> int:
    """Gradients of q, k, v, qm, km with integer pointers; returns the status."""
    return load().gecko_sca_awm_backward(q, k, v, qm, km, out_sca, out_sca_lo, lse, dout_sca, dout_mem, dq, dk, dv,
                                         dqm, dkm, B, H, T, c, d, dtype, stream)


def gecko_awm_state(M_out, logz_out, B, H, d, stream) -> int:
    return load().gecko_awm_state(M_out, logz_out, B, H, d, stream)


def gecko_cema_forward(x, y, alpha, delta, theta, beta, eta, reset, state_in, state_out, B, L, D, h, dtype,
                       stream) -> int:
    """Direct call of the CEMA entry point with integer pointers (0 = NULL)."""
    return load().gecko_cema_forward(x, y, alpha, delta, theta, beta, eta, reset, state_in, state_out,
                                     B, L, D, h, dtype, stream)


def gecko_tdnorm_forward(x, y, gamma, bias, B, L, D, G, beta1, beta2, eps, dtype, stream) -> int:
    """Direct call of the timestep-normalisation entry point with integer pointers."""
    return load().gecko_tdnorm_forward(x, y, gamma, bias, B, L, D, G, beta1, beta2, eps, dtype, stream)


def gecko_awm_segment_logsum(km, lsum_out, B, H, T, c, d, dtype, stream) -> int:
    return load().gecko_awm_segment_logsum(km, lsum_out, B, H, T, c, d, dtype, stream)


def gecko_awm_segment_maps(km, v, logz_in, maps_out, B, H, T, c, d, dtype, stream) -> int:
    return load().gecko_awm_segment_maps(km, v, logz_in, maps_out, B, H, T, c, d, dtype, stream)


def gecko_awm_cp_logz(lsum_all, P, rank, logz_out, B, H, d, stream) -> int:
    return load().gecko_awm_cp_logz(lsum_all, P, rank, logz_out, B, H, d, stream)


def gecko_awm_cp_state(lsum_all, maps_all, P, rank, state_out, B, H, d, stream) -> int:
    return load().gecko_awm_cp_state(lsum_all, maps_all, P, rank, state_out, B, H, d, stream)


def gecko_device_status(stream) -> int:
    return load().gecko_device_status(stream)


def gecko_timing_enable(enable: int) -> int:
    return load().gecko_timing_enable(enable)


def gecko_timing_read(ms_per_stage, capacity: int, n_calls) -> int:
    return load().gecko_timing_read(ms_per_stage, capacity, n_calls)


def gecko_timing_read_backward(ms_per_stage, capacity: int, n_calls) -> int:
    return load().gecko_timing_read_backward(ms_per_stage, capacity, n_calls)


def gecko_last_error() -> str:
    return load().gecko_last_error().decode()


def gecko_release() -> None:
    load().gecko_release()


# ------------------------------------------------------- tensor front end --

_DT = {torch.float32: GECKO_F32, torch.bfloat16: GECKO_BF16}


def sca_awm_forward(q, k, v, qm, km, c: int, out_sca=None, out_mem=None, stream=None):
    """Fused SCA + AWM forward on [B, H, T, d] CUDA tensors.

    Returns (out_sca, out_mem); the layer output is their sum.  Outputs are
    allocated with torch if not given.  Runs asynchronously on `stream`
    (default: torch's current stream).
    """
    xs = (q, k, v, qm, km)
    _check_inputs(xs)
    B, H, T, d = q.shape
    _check_outputs((out_sca, out_mem), q)
    if out_sca is None:
        out_sca = torch.empty_like(q)
    if out_mem is None:
        out_mem = torch.empty_like(q)
    with torch.cuda.device(q.device):
        rc = gecko_sca_awm_forward(*(x.data_ptr() for x in xs), out_sca.data_ptr(), out_mem.data_ptr(),
                                   B, H, T, c, d, _DT[q.dtype], _stream_handle(stream))
    _check(rc)
    return out_sca, out_mem


def _check_outputs(outs, like):
    """Caller-given output buffers must be what the kernels write: the
    inputs' shape, dtype and device, contiguous (a smaller buffer would be
    written past its end)."""
    for o in outs:
        if o is None:
            continue
        if not (isinstance(o, torch.Tensor) and o.is_contiguous() and o.shape == like.shape
                and o.dtype == like.dtype and o.device == like.device):
            raise ValueError(f"output buffers must be contiguous {tuple(like.shape)} {like.dtype} "
                             f"tensors on {like.device}")


def _check_inputs(xs):
    q = xs[0]
    for x in xs:
        if not (isinstance(x, torch.Tensor) and x.is_cuda and x.is_contiguous()):
            raise ValueError("inputs must be contiguous CUDA tensors")
        if x.shape != q.shape or x.dtype != q.dtype or x.device != q.device:
            raise ValueError("inputs must share shape, dtype and device")
    if q.dim() != 4 or q.dtype not in _DT:
        raise ValueError("inputs must be [B, H, T, d] float32 or bfloat16")


def sca_awm_forward_train(q, k, v, qm, km, c: int, stream=None, keep_residual: bool = True):
    """Forward for training: returns (out_sca, out_mem, lse, out_sca_lo) with
    lse the [B, H, T] fp32 row log-sum-exp of SCA and out_sca_lo the rounding
    residual of out_sca (None if keep_residual is False), both for
    sca_awm_backward."""
    xs = (q, k, v, qm, km)
    _check_inputs(xs)
    B, H, T, d = q.shape
    out_sca, out_mem = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    lo = torch.empty_like(q) if keep_residual else None
    with torch.cuda.device(q.device):
        rc = gecko_sca_awm_forward_train(*(x.data_ptr() for x in xs), out_sca.data_ptr(), out_mem.data_ptr(),
                                         lse.data_ptr(), lo.data_ptr() if lo is not None else 0, B, H, T, c, d,
                                         _DT[q.dtype], _stream_handle(stream))
    _check(rc)
    return out_sca, out_mem, lse, lo


def sca_awm_backward(q, k, v, qm, km, out_sca, lse, dout_sca, dout_mem, c: int, out_sca_lo=None, stream=None):
    """Gradients (dq, dk, dv, dqm, dkm) of the fused forward for the output
    gradients dout_sca, dout_mem; out_sca, lse and out_sca_lo come from
    sca_awm_forward_train on the same inputs."""
    xs = (q, k, v, qm, km, out_sca, dout_sca.contiguous(), dout_mem.contiguous())
    _check_inputs(xs)
    if out_sca_lo is not None:
        _check_inputs((q, out_sca_lo))
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == q.shape[:3]):
        raise ValueError("lse must be a contiguous [B, H, T] float32 CUDA tensor")
    B, H, T, d = q.shape
    grads = [torch.empty_like(q) for _ in range(5)]
    with torch.cuda.device(q.device):
        rc = gecko_sca_awm_backward(*(x.data_ptr() for x in xs[:6]), out_sca_lo.data_ptr() if out_sca_lo is not None
                                    else 0, lse.data_ptr(), xs[6].data_ptr(), xs[7].data_ptr(),
                                    *(g.data_ptr() for g in grads), B, H, T, c, d, _DT[q.dtype],
                                    _stream_handle(stream))
    _check(rc)
    return tuple(grads)


class ScaAwmFunction(torch.autograd.Function):
    """torch.autograd wrapper of the fused forward and backward:
    (out_sca, out_mem) = ScaAwmFunction.apply(q, k, v, qm, km, c)."""

    @staticmethod
    def forward(ctx, q, k, v, qm, km, c):
        out_sca, out_mem, lse, lo = sca_awm_forward_train(q, k, v, qm, km, c)
        ctx.save_for_backward(q, k, v, qm, km, out_sca, lse, lo)
        ctx.c = c
        return out_sca, out_mem

    @staticmethod
    def backward(ctx, dout_sca, dout_mem):
        q, k, v, qm, km, out_sca, lse, lo = ctx.saved_tensors
        grads = sca_awm_backward(q, k, v, qm, km, out_sca, lse, dout_sca, dout_mem, ctx.c, out_sca_lo=lo)
        return (*grads, None)


def sca_awm_forward_segment(q, k, v, qm, km, c: int, state_in=None, out_sca=None, out_mem=None, stream=None):
    """One segment of a long sequence.  q, qm, km: [B, H, T, d].  Without
    state_in, k and v are [B, H, T, d] (fresh start); with it they are
    [B, H, c + T, d], the previous segment's last chunk first.  Returns
    (out_sca, out_mem, state) where state [B, H, 2 d^2 + d] fp32 feeds the
    next segment."""
    xs = (q, k, v, qm, km)
    for x in xs:
        if not (isinstance(x, torch.Tensor) and x.is_cuda and x.is_contiguous() and x.dtype == q.dtype):
            raise ValueError("inputs must be contiguous CUDA tensors of one dtype")
    B, H, T, d = q.shape
    kv_rows = T + (c if state_in is not None else 0)
    if tuple(k.shape) != (B, H, kv_rows, d) or tuple(v.shape) != (B, H, kv_rows, d):
        raise ValueError(f"k and v must be [B, H, {kv_rows}, d]")
    if qm.shape != q.shape or km.shape != q.shape or q.dim() != 4 or q.dtype not in _DT \
            or any(x.device != q.device for x in xs):
        raise ValueError("q, qm, km must be [B, H, T, d] float32 or bfloat16 tensors on one device")
    if state_in is not None and not (isinstance(state_in, torch.Tensor) and state_in.is_contiguous()
                                     and state_in.dtype == torch.float32
                                     and tuple(state_in.shape) == (B, H, 2 * d * d + d)):
        raise ValueError(f"state_in must be a contiguous [B, H, {2 * d * d + d}] float32 tensor")
    _check_outputs((out_sca, out_mem), q)
    if out_sca is None:
        out_sca = torch.empty_like(q)
    if out_mem is None:
        out_mem = torch.empty_like(q)
    state = torch.empty(B, H, 2 * d * d + d, dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        rc = gecko_sca_awm_forward_continue(*(x.data_ptr() for x in xs), out_sca.data_ptr(), out_mem.data_ptr(),
                                            0 if state_in is None else state_in.data_ptr(), state.data_ptr(),
                                            B, H, T, c, d, _DT[q.dtype], _stream_handle(stream))
    _check(rc)
    return out_sca, out_mem, state


def awm_state(B: int, H: int, d: int, device=None, stream=None):
    """(M'_{S+1} [B, H, d, d], log z^S [B, H, d]) of the last forward, fp32."""
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    M = torch.empty(B, H, d, d, dtype=torch.float32, device=device)
    lz = torch.empty(B, H, d, dtype=torch.float32, device=device)
    with torch.cuda.device(device):
        _check(gecko_awm_state(M.data_ptr(), lz.data_ptr(), B, H, d, _stream_handle(stream)))
    return M, lz


def device_status(stream=None) -> int:
    """Synchronise, read and clear the device status word (0 = OK)."""
    return gecko_device_status(_stream_handle(stream))


def release() -> None:
    gecko_release()


def timing_enable(on: bool = True) -> None:
    _check(gecko_timing_enable(1 if on else 0))


def timing_read():
    """({stage: summed ms}, number of forwards) since the last read."""
    buf = (ctypes.c_float * len(STAGES))()
    n = ctypes.c_int(0)
    _check(gecko_timing_read(buf, len(STAGES), ctypes.byref(n)))
    return {name: float(buf[i]) for i, name in enumerate(STAGES)}, int(n.value)


def timing_read_backward():
    """({stage: total ms}, n_calls) of the backwards timed since the last read."""
    buf = (ctypes.c_float * len(BWD_STAGES))()
    n = ctypes.c_int(0)
    _check(gecko_timing_read_backward(buf, len(BWD_STAGES), ctypes.byref(n)))
    return {name: float(buf[i]) for i, name in enumerate(BWD_STAGES)}, int(n.value)


def cema_forward(x, alpha, delta, theta, beta, eta, reset=None, state_in=None, return_state=False, y=None,
                 stream=None):
    """CEMA over x [B, L, D] (float32 or bfloat16 CUDA tensor).  alpha,
    delta, theta, beta: [D, 16] float32; eta: [D, 16, 2] float32 (real,
    imaginary); reset: [B, L] uint8 or None; state_in: [B, D, 16, 2] float32
    or None.  Returns y (and the final state [B, D, 16, 2] if return_state)."""
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.is_contiguous() and x.dim() == 3 and x.dtype in _DT):
        raise ValueError("x must be a contiguous [B, L, D] float32 or bfloat16 CUDA tensor")
    B, L, D = x.shape
    params = (alpha, delta, theta, beta, eta)
    for prm in params:
        if not (isinstance(prm, torch.Tensor) and prm.is_cuda and prm.is_contiguous() and prm.dtype == torch.float32):
            raise ValueError("parameters must be contiguous float32 CUDA tensors")
    h = alpha.shape[-1]
    for prm, shape in zip(params, ((D, h),) * 4 + ((D, h, 2),)):
        if tuple(prm.shape) != shape or prm.device != x.device:
            raise ValueError(f"CEMA parameters must be [D, h] (eta [D, h, 2]) on {x.device}; got {tuple(prm.shape)}")
    if reset is not None and not (isinstance(reset, torch.Tensor) and reset.dtype == torch.uint8
                                  and tuple(reset.shape) == (B, L) and reset.is_contiguous()
                                  and reset.device == x.device):
        raise ValueError(f"reset must be a contiguous [B, L] uint8 tensor on {x.device}")
    if state_in is not None and not (isinstance(state_in, torch.Tensor) and state_in.dtype == torch.float32
                                     and tuple(state_in.shape) == (B, D, h, 2) and state_in.is_contiguous()
                                     and state_in.device == x.device):
        raise ValueError(f"state_in must be a contiguous [B, D, h, 2] float32 tensor on {x.device}")
    _check_outputs((y,), x)
    if y is None:
        y = torch.empty_like(x)
    state_out = torch.empty(B, D, h, 2, dtype=torch.float32, device=x.device) if return_state else None
    ptr = lambda t: 0 if t is None else t.data_ptr()
    with torch.cuda.device(x.device):
        rc = gecko_cema_forward(x.data_ptr(), y.data_ptr(), *(prm.data_ptr() for prm in params), ptr(reset),
                                ptr(state_in), ptr(state_out), B, L, D, h, _DT[x.dtype], _stream_handle(stream))
    _check(rc)
    return (y, state_out) if return_state else y


def tdnorm_forward(x, gamma, bias, G: int, beta1: float, beta2: float, eps: float, y=None, stream=None):
    """Timestep decay normalisation of x [B, L, D] (float32 or bfloat16 CUDA
    tensor) over G feature groups; gamma, bias: [D] float32.  Returns y."""
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.is_contiguous() and x.dim() == 3 and x.dtype in _DT):
        raise ValueError("x must be a contiguous [B, L, D] float32 or bfloat16 CUDA tensor")
    for prm in (gamma, bias):
        if not (isinstance(prm, torch.Tensor) and prm.is_cuda and prm.is_contiguous() and prm.dtype == torch.float32):
            raise ValueError("gamma and bias must be contiguous float32 CUDA tensors")
    B, L, D = x.shape
    if gamma.shape != (D,) or bias.shape != (D,) or gamma.device != x.device or bias.device != x.device:
        raise ValueError(f"gamma and bias must be [D] = [{D}] on {x.device}")
    _check_outputs((y,), x)
    if y is None:
        y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        rc = gecko_tdnorm_forward(x.data_ptr(), y.data_ptr(), gamma.data_ptr(), bias.data_ptr(), B, L, D, G,
                                  beta1, beta2, eps, _DT[x.dtype], _stream_handle(stream))
    _check(rc)
    return y


# ------------------------------------------------ context parallelism -----

def awm_segment_logsum(km, c: int, stream=None):
    """[B, H, d] fp32: log sum over the segment's tokens of exp(km)."""
    _check_inputs((km,))
    B, H, T, d = km.shape
    out = torch.empty((B, H, d), dtype=torch.float32, device=km.device)
    with torch.cuda.device(km.device):
        rc = gecko_awm_segment_logsum(km.data_ptr(), out.data_ptr(), B, H, T, c, d, _DT[km.dtype],
                                      _stream_handle(stream))
    _check(rc)
    return out


def _f32_on(t, shape, device, name):
    """t as a contiguous fp32 tensor of `shape` on `device` (the caller keeps
    the returned tensor alive until the call is enqueued)."""
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.float32
            and tuple(t.shape) == tuple(shape) and t.device == device):
        raise ValueError(f"{name} must be a float32 CUDA tensor of shape {tuple(shape)} on {device}")
    return t.contiguous()


def awm_segment_maps(km, v, logz_in, c: int, stream=None):
    """[B, H, 4, d, d] fp32 maps (A, b, A', b') of the segment for the log z
    entering it (logz_in [B, H, d] fp32)."""
    _check_inputs((km, v))
    B, H, T, d = km.shape
    lz = _f32_on(logz_in, (B, H, d), km.device, "logz_in")
    out = torch.empty((B, H, 4, d, d), dtype=torch.float32, device=km.device)
    with torch.cuda.device(km.device):
        rc = gecko_awm_segment_maps(km.data_ptr(), v.data_ptr(), lz.data_ptr(), out.data_ptr(),
                                    B, H, T, c, d, _DT[km.dtype], _stream_handle(stream))
    _check(rc)
    return out


def awm_cp_logz(lsum_all, rank: int, stream=None):
    """log z entering segment `rank` from every rank's log-sum [P, B, H, d]."""
    P, B, H, d = lsum_all.shape
    ls = _f32_on(lsum_all, (P, B, H, d), lsum_all.device, "lsum_all")
    out = torch.empty((B, H, d), dtype=torch.float32, device=lsum_all.device)
    with torch.cuda.device(lsum_all.device):
        rc = gecko_awm_cp_logz(ls.data_ptr(), P, rank, out.data_ptr(), B, H, d, _stream_handle(stream))
    _check(rc)
    return out


def awm_cp_state(lsum_all, maps_all, rank: int, stream=None):
    """state_in [B, H, 2 d^2 + d] of segment `rank` (M'_prev, M'_in, log z)."""
    P, B, H, d = lsum_all.shape
    ls = _f32_on(lsum_all, (P, B, H, d), lsum_all.device, "lsum_all")
    mp = _f32_on(maps_all, (P, B, H, 4, d, d), lsum_all.device, "maps_all")
    out = torch.empty((B, H, 2 * d * d + d), dtype=torch.float32, device=lsum_all.device)
    with torch.cuda.device(lsum_all.device):
        rc = gecko_awm_cp_state(ls.data_ptr(), mp.data_ptr(), P, rank, out.data_ptr(), B, H, d,
                                _stream_handle(stream))
    _check(rc)
    return out

