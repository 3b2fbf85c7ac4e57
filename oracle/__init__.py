"""fp64 CPU oracle for the DCNv4 spatial aggregation, forward and backward.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU-baseline leg
of the benchmark may import this package; the product path (the CUDA library
and its Python binding) never does. The arithmetic lives in ``dcnv4_oracle.c``
(plain C, fp64), compiled here with gcc into ``liboracle.so`` and called
through ctypes with numpy arrays. It shares no code with the CUDA path.

Definition followed: "不只是卷积的平替：我把DCNv4塞进Stable Diffusion的U-Net里"
(jsqmd.com), section 1 (no softmax over the modulation scalars; the simplified
forward listing: regular grid + offsets, bilinear sampling, mask-weighted sum
over the K*K points per group) and "掌握DCNv4技术" (pwwt.cn), tuning section
(offset_scale scales the offsets). The readings taken where the pages are
silent are stated at the top of ``dcnv4_oracle.c``.

Every function here is pinned by tests that do not reuse its code (identity,
integer-offset brute force, torch ``grid_sample``, hand-expanded cases in
``tests/golden/``, linearity, out-of-bounds, partition of unity, group
equivalence, translation equivariance).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dcnv4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``dcnv4_oracle.c`` into ``liboracle.so`` (gcc, no fused multiply-add)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i, f, p = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        lib.oracle_output_size.argtypes = [i, i, i, i, i]
        lib.oracle_output_size.restype = i
        lib.oracle_dcnv4_forward.argtypes = [p, p, p] + [i] * 9 + [f]
        lib.oracle_dcnv4_forward.restype = i
        lib.oracle_dcnv4_forward_images.argtypes = [p, p, p] + [i] * 9 + [f, i, i]
        lib.oracle_dcnv4_forward_images.restype = i
        lib.oracle_dcnv4_forward_images_mt.argtypes = [p, p, p] + [i] * 9 + [f, i, i, i]
        lib.oracle_dcnv4_forward_images_mt.restype = i
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i
        lib.oracle_dcnv4_sampling_index.argtypes = [p, p, p] + [i] * 8 + [f]
        lib.oracle_dcnv4_sampling_index.restype = i
        lib.oracle_dcnv4_backward.argtypes = [p] * 5 + [i] * 9 + [f]
        lib.oracle_dcnv4_backward.restype = i
        lib.oracle_dcnv4_forward_variants.argtypes = [p] * 4 + [i] * 9 + [f, i, i, i]
        lib.oracle_dcnv4_forward_variants.restype = i
        lib.oracle_dcnv4_backward_variants.argtypes = [p] * 7 + [i] * 9 + [f, i, i, i]
        lib.oracle_dcnv4_backward_variants.restype = i
        lib.oracle_dcnv4_predictor.argtypes = [p] * 4 + [i] * 4
        lib.oracle_dcnv4_predictor.restype = i
        _lib = lib
    return _lib


def output_size(size: int, K: int, stride: int = 1, pad: int = 0, dilation: int = 1) -> int:
    """Output extent along one axis, convolution style (<= 0 when empty)."""
    return _load().oracle_output_size(size, K, stride, pad, dilation)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    """Threads the oracle's parallel forward uses by default (OpenMP)."""
    return _load().oracle_max_threads()


def dcnv4_forward(x, offset_mask, G: int, K: int, stride: int = 1, pad: int = 0,
                  dilation: int = 1, offset_scale: float = 1.0,
                  n_begin: int | None = None, n_end: int | None = None, threads: int = 1) -> np.ndarray:
    """fp64 forward. ``x``: [N,H,W,C]; ``offset_mask``: [N,Hout,Wout,G,3*K*K].

    Returns out [N,Hout,Wout,C] (fp64). With ``n_begin``/``n_end`` only those
    images are computed (the rest of the result stays zero). ``threads`` != 1
    shares the output rows out among that many OpenMP threads (0: all); every
    element is computed by the same code in the same order, so the result is
    the same bits.
    """
    x = _f64(x)
    om = _f64(offset_mask)
    N, H, W, C = x.shape
    Hout, Wout = output_size(H, K, stride, pad, dilation), output_size(W, K, stride, pad, dilation)
    if om.shape != (N, Hout, Wout, G, 3 * K * K):
        raise ValueError(f"offset_mask shape {om.shape} != {(N, Hout, Wout, G, 3 * K * K)}")
    out = np.zeros((N, Hout, Wout, C), dtype=np.float64)
    if N == 0:
        return out
    lib = _load()
    if threads != 1:
        rc = lib.oracle_dcnv4_forward_images_mt(_ptr(x), _ptr(om), _ptr(out), N, H, W, C, G, K,
                                                stride, pad, dilation, float(offset_scale),
                                                0 if n_begin is None else n_begin,
                                                N if n_end is None else n_end, int(threads))
    elif n_begin is None and n_end is None:
        rc = lib.oracle_dcnv4_forward(_ptr(x), _ptr(om), _ptr(out), N, H, W, C, G, K,
                                      stride, pad, dilation, float(offset_scale))
    else:
        rc = lib.oracle_dcnv4_forward_images(_ptr(x), _ptr(om), _ptr(out), N, H, W, C, G, K,
                                             stride, pad, dilation, float(offset_scale),
                                             0 if n_begin is None else n_begin,
                                             N if n_end is None else n_end)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def dcnv4_forward_variants(x, offset_mask, G: int, K: int, stride: int = 1, pad: int = 0, dilation: int = 1,
                           offset_scale: float = 1.0, softmax: bool = False, remove_center: bool = False,
                           center_logit=None) -> np.ndarray:
    """fp64 forward with the variant switches (see dcnv4_oracle.c for the readings).

    softmax: DCNv3-style softmax over each unit's masks; remove_center: P = K*K-1
    points per unit, record [N,Hout,Wout,G,3*P]; center_logit [N,Hout,Wout,G]:
    centre feature scaling with gate sigmoid(center_logit) (None: off).
    """
    x = _f64(x)
    om = _f64(offset_mask)
    N, H, W, C = x.shape
    Hout, Wout = output_size(H, K, stride, pad, dilation), output_size(W, K, stride, pad, dilation)
    P = K * K - (1 if remove_center else 0)
    if om.shape != (N, Hout, Wout, G, 3 * P):
        raise ValueError(f"offset_mask shape {om.shape} != {(N, Hout, Wout, G, 3 * P)}")
    z = None
    if center_logit is not None:
        z = _f64(center_logit)
        if z.shape != (N, Hout, Wout, G):
            raise ValueError("center_logit must be [N,Hout,Wout,G]")
    out = np.zeros((N, Hout, Wout, C), dtype=np.float64)
    if N == 0:
        return out
    rc = _load().oracle_dcnv4_forward_variants(_ptr(x), _ptr(om), None if z is None else _ptr(z), _ptr(out),
                                               N, H, W, C, G, K, stride, pad, dilation, float(offset_scale),
                                               int(bool(softmax)), int(bool(remove_center)), int(z is not None))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def dcnv4_backward_variants(x, offset_mask, grad_out, G: int, K: int, stride: int = 1, pad: int = 0,
                            dilation: int = 1, offset_scale: float = 1.0, softmax: bool = False,
                            remove_center: bool = False, center_logit=None):
    """fp64 backward of ``dcnv4_forward_variants``: returns (grad_x, grad_offset_mask, grad_center_logit),
    the last None without centre scaling."""
    x = _f64(x)
    om = _f64(offset_mask)
    go = _f64(grad_out)
    N, H, W, C = x.shape
    Hout, Wout = output_size(H, K, stride, pad, dilation), output_size(W, K, stride, pad, dilation)
    P = K * K - (1 if remove_center else 0)
    if om.shape != (N, Hout, Wout, G, 3 * P) or go.shape != (N, Hout, Wout, C):
        raise ValueError("offset_mask / grad_out shapes do not match x")
    z = None if center_logit is None else _f64(center_logit)
    gx = np.zeros_like(x)
    gom = np.zeros_like(om)
    gz = None if z is None else np.zeros_like(z)
    if N:
        rc = _load().oracle_dcnv4_backward_variants(_ptr(x), _ptr(om), None if z is None else _ptr(z), _ptr(go),
                                                    _ptr(gx), _ptr(gom), None if gz is None else _ptr(gz),
                                                    N, H, W, C, G, K, stride, pad, dilation, float(offset_scale),
                                                    int(bool(softmax)), int(bool(remove_center)), int(z is not None))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
    return gx, gom, gz


def dcnv4_predictor(y, weight, bias, G: int, P: int) -> np.ndarray:
    """fp64 1x1 projection + repacking into offset_mask records.

    y: [..., C] (any leading pixel shape), weight: [3*G*P, C] in the pages'
    channel order (all groups' offsets, (g, comp, point), then all groups'
    masks, (g, point)), bias: [3*G*P] or None. Returns [..., G, 3*P].
    """
    y = _f64(y)
    w = _f64(weight)
    lead, C = y.shape[:-1], y.shape[-1]
    M = int(np.prod(lead)) if lead else 1
    if w.shape != (3 * G * P, C):
        raise ValueError(f"weight shape {w.shape} != {(3 * G * P, C)}")
    b = None if bias is None else _f64(bias)
    if b is not None and b.shape != (3 * G * P,):
        raise ValueError("bias must be [3*G*P]")
    rec = np.zeros((M, G, 3 * P), dtype=np.float64)
    if M:
        rc = _load().oracle_dcnv4_predictor(_ptr(y), _ptr(w), None if b is None else _ptr(b), _ptr(rec), M, C, G, P)
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
    return rec.reshape(*lead, G, 3 * P)


def sampling_index(offset_mask, H: int, W: int, G: int, K: int, stride: int = 1, pad: int = 0,
                   dilation: int = 1, offset_scale: float = 1.0):
    """Integer corner (y0, x0) [..., K*K, 2] int32 and 4-bit validity [..., K*K] uint8.

    Bit 2*a+b of the validity byte is set when corner (y0+a, x0+b) is inside the
    image; samples with no corner inside report (INT32_MIN, INT32_MIN).
    """
    om = _f64(offset_mask)
    N, Hout, Wout, G_, R = om.shape
    if G_ != G or R != 3 * K * K:
        raise ValueError("offset_mask shape does not match G, K")
    if (Hout, Wout) != (output_size(H, K, stride, pad, dilation), output_size(W, K, stride, pad, dilation)):
        raise ValueError("offset_mask spatial shape does not match the output size")
    corner = np.zeros((N, Hout, Wout, G, K * K, 2), dtype=np.int32)
    valid = np.zeros((N, Hout, Wout, G, K * K), dtype=np.uint8)
    if N:
        rc = _load().oracle_dcnv4_sampling_index(_ptr(om), _ptr(corner), _ptr(valid), N, H, W, G, K,
                                                 stride, pad, dilation, float(offset_scale))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
    return corner, valid


def dcnv4_backward(x, offset_mask, grad_out, G: int, K: int, stride: int = 1, pad: int = 0, dilation: int = 1,
                   offset_scale: float = 1.0):
    """fp64 backward: returns (grad_x [N,H,W,C], grad_offset_mask [N,Hout,Wout,G,3*K*K]).

    The exact derivative of ``dcnv4_forward`` for a loss whose gradient with
    respect to the output is ``grad_out`` (see dcnv4_oracle.c for the
    formulas and the convention at integer positions)."""
    x = _f64(x)
    om = _f64(offset_mask)
    go = _f64(grad_out)
    N, H, W, C = x.shape
    Hout, Wout = output_size(H, K, stride, pad, dilation), output_size(W, K, stride, pad, dilation)
    if om.shape != (N, Hout, Wout, G, 3 * K * K) or go.shape != (N, Hout, Wout, C):
        raise ValueError("offset_mask / grad_out shapes do not match x")
    gx = np.zeros_like(x)
    gom = np.zeros_like(om)
    if N:
        rc = _load().oracle_dcnv4_backward(_ptr(x), _ptr(om), _ptr(go), _ptr(gx), _ptr(gom), N, H, W, C, G, K,
                                           stride, pad, dilation, float(offset_scale))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
    return gx, gom
