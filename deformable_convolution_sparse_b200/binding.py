"""ctypes binding of libdcnv4.so (the C ABI in include/dcnv4.h).

Argument marshalling only: tensors are checked (device, dtype, shape,
contiguity) and their data pointers are handed to the library together with
the current CUDA stream; every step of the computation runs in the library's
kernels. There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_PKG, "libdcnv4.so")

DCNV4_F32, DCNV4_F16, DCNV4_BF16 = 0, 1, 2
DCNV4_OK = 0
STATUS_NAMES = {
    0: "DCNV4_OK", 1: "DCNV4_ERR_NULL", 2: "DCNV4_ERR_SHAPE", 3: "DCNV4_ERR_GROUPS",
    4: "DCNV4_ERR_DTYPE", 5: "DCNV4_ERR_ALIGN", 6: "DCNV4_ERR_ALIAS", 7: "DCNV4_ERR_SCALE",
    8: "DCNV4_ERR_TOO_LARGE", 9: "DCNV4_ERR_LAUNCH", 10: "DCNV4_ERR_CUDA", 11: "DCNV4_ERR_STAGING",
    12: "DCNV4_ERR_FLAGS",
}
# variant switches of dcnv4_forward_ex
FLAG_SOFTMAX, FLAG_REMOVE_CENTER, FLAG_CENTER_SCALE = 1, 2, 4
STATUS = {v: k for k, v in STATUS_NAMES.items()}
TORCH_DTYPE = {torch.float32: DCNV4_F32, torch.float16: DCNV4_F16, torch.bfloat16: DCNV4_BF16}

# every symbol include/dcnv4.h declares
EXPORTS = ("dcnv4_output_shape", "dcnv4_validate", "dcnv4_validate_ex", "dcnv4_forward", "dcnv4_forward_ex",
           "dcnv4_forward_trace",
           "dcnv4_backward", "dcnv4_backward_ex", "dcnv4_predictor", "dcnv4_sampling_index",
           "dcnv4_forward_host", "dcnv4_forward_host_noalloc", "dcnv4_device_status", "dcnv4_selftest_wait_timeout",
           "dcnv4_probe_smem_gather", "dcnv4_probe_red_global", "dcnv4_probe_red_shared", "dcnv4_forward_plan", "dcnv4_strerror", "dcnv4_abi_version")
DEVSTATUS_COPY_TIMEOUT, DEVSTATUS_SELFTEST_TIMEOUT = 1, 2

_lib = None


class DCNv4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where}: {name} ({strerror(status)})")


def load_library():
    """Load libdcnv4.so (built in-tree by ``deformable_convolution_sparse_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY_PATH):
        raise RuntimeError(f"{LIBRARY_PATH} is missing: build it with "
                           "`python -m deformable_convolution_sparse_b200.build`")
    lib = ctypes.CDLL(LIBRARY_PATH)
    i, f, p = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
    ip = ctypes.POINTER(ctypes.c_int)
    lib.dcnv4_output_shape.argtypes = [i, i, i, i, i, i, ip, ip]
    lib.dcnv4_output_shape.restype = i
    lib.dcnv4_validate.argtypes = [p, p, p] + [i] * 9 + [f, i]
    lib.dcnv4_validate.restype = i
    lib.dcnv4_forward.argtypes = [p, p, p] + [i] * 9 + [f, i, p]
    lib.dcnv4_forward.restype = i
    lib.dcnv4_forward_trace.argtypes = [p] * 4 + [i] * 9 + [f, i, p]
    lib.dcnv4_forward_trace.restype = i
    lib.dcnv4_validate_ex.argtypes = [p] * 4 + [i] * 9 + [f, i, ctypes.c_uint]
    lib.dcnv4_validate_ex.restype = i
    lib.dcnv4_forward_ex.argtypes = [p] * 4 + [i] * 9 + [f, i, ctypes.c_uint, p]
    lib.dcnv4_forward_ex.restype = i
    lib.dcnv4_predictor.argtypes = [p] * 4 + [i] * 4 + [ctypes.c_uint, i, p]
    lib.dcnv4_predictor.restype = i
    lib.dcnv4_backward.argtypes = [p] * 5 + [i] * 9 + [f, i, p]
    lib.dcnv4_backward_ex.argtypes = [p] * 7 + [i] * 9 + [f, i, ctypes.c_uint, p]
    lib.dcnv4_backward_ex.restype = i
    lib.dcnv4_backward.restype = i
    lib.dcnv4_sampling_index.argtypes = [p, p, p] + [i] * 8 + [f, i, p]
    lib.dcnv4_sampling_index.restype = i
    lib.dcnv4_forward_host.argtypes = [p] * 6 + [i] * 9 + [f, i, p]
    lib.dcnv4_forward_host.restype = i
    lib.dcnv4_forward_host_noalloc.argtypes = [p] * 3 + [i] * 9 + [f, i, p]
    lib.dcnv4_forward_host_noalloc.restype = i
    lib.dcnv4_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), i]
    lib.dcnv4_device_status.restype = i
    lib.dcnv4_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, p]
    lib.dcnv4_selftest_wait_timeout.restype = i
    lib.dcnv4_probe_smem_gather.argtypes = [i, ctypes.POINTER(ctypes.c_double)]
    lib.dcnv4_probe_smem_gather.restype = i
    lib.dcnv4_probe_red_global.argtypes = [i, ctypes.POINTER(ctypes.c_double)]
    lib.dcnv4_probe_red_global.restype = i
    lib.dcnv4_probe_red_shared.argtypes = [i, ctypes.POINTER(ctypes.c_double)]
    lib.dcnv4_probe_red_shared.restype = i
    lib.dcnv4_forward_plan.argtypes = [i] * 10 + [ctypes.c_uint, i, ctypes.POINTER(ctypes.c_int), i]
    lib.dcnv4_forward_plan.restype = i
    lib.dcnv4_strerror.argtypes = [i]
    lib.dcnv4_strerror.restype = ctypes.c_char_p
    lib.dcnv4_abi_version.argtypes = []
    lib.dcnv4_abi_version.restype = i
    _lib = lib
    return lib


def strerror(status: int) -> str:
    return load_library().dcnv4_strerror(int(status)).decode()


def abi_version() -> int:
    return load_library().dcnv4_abi_version()


def device_status(clear: bool = False) -> int:
    """Device status word of the current device (waits for the device)."""
    v = ctypes.c_uint(0)
    rc = load_library().dcnv4_device_status(ctypes.byref(v), int(bool(clear)))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_device_status")
    return v.value


def selftest_wait_timeout(limit_ns: int = 1_000_000, stream=None) -> None:
    """Launches the bounded-wait self test (sets DEVSTATUS_SELFTEST_TIMEOUT)."""
    rc = load_library().dcnv4_selftest_wait_timeout(int(limit_ns), _stream_handle(stream))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_selftest_wait_timeout")


def probe_smem_gather(pattern: int = 0) -> float:
    """Shared-memory gather bytes per SM clock per SM (dcnv4_probe_smem_gather; synchronous)."""
    v = ctypes.c_double(0.0)
    rc = load_library().dcnv4_probe_smem_gather(int(pattern), ctypes.byref(v))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_probe_smem_gather")
    return v.value


def probe_red_global(segment_bytes: int = 64) -> float:
    """fp32 vector-reduction payload bytes per SM clock per SM into L2 (dcnv4_probe_red_global; synchronous)."""
    v = ctypes.c_double(0.0)
    rc = load_library().dcnv4_probe_red_global(int(segment_bytes), ctypes.byref(v))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_probe_red_global")
    return v.value


def probe_red_shared(fp32: bool = True) -> float:
    """Shared-memory atomic adds per SM clock per SM, fp32 or 32-bit integer (dcnv4_probe_red_shared)."""
    v = ctypes.c_double(0.0)
    rc = load_library().dcnv4_probe_red_shared(1 if fp32 else 0, ctypes.byref(v))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_probe_red_shared")
    return v.value


PLAN_FIELDS = ("kernel", "image_windows", "halo", "groups_per_strip", "band_columns", "item_rows", "ring_rows",
               "items_in_flight", "units_per_item", "threads", "smem_bytes", "unit_window_rows",
               "unit_window_cols", "window_pixels", "pixel_bytes")


def forward_plan(N: int, H: int, W: int, C: int, G: int, K: int, stride: int = 1, pad: int = 0, dilation: int = 1,
                 dtype: int = DCNV4_F32, flags: int = 0, nsm: int = 148) -> dict:
    """The forward's plan for a geometry (dcnv4_forward_plan; no GPU needed): the kernel
    choice and the ring kernel's shape, as a dict keyed by PLAN_FIELDS."""
    buf = (ctypes.c_int * len(PLAN_FIELDS))()
    rc = load_library().dcnv4_forward_plan(N, H, W, C, G, K, stride, pad, dilation, int(dtype), int(flags), int(nsm),
                                           buf, len(PLAN_FIELDS))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_forward_plan")
    d = dict(zip(PLAN_FIELDS, list(buf)))
    d["kernel"] = "ring" if d["kernel"] == 0 else "gather"
    return d


def output_shape(H: int, W: int, K: int, stride: int = 1, pad: int = 0, dilation: int = 1):
    """(Hout, Wout) from the library; raises DCNv4Error on invalid geometry."""
    ho, wo = ctypes.c_int(0), ctypes.c_int(0)
    rc = load_library().dcnv4_output_shape(H, W, K, stride, pad, dilation, ctypes.byref(ho), ctypes.byref(wo))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_output_shape")
    return ho.value, wo.value


def validate(x_ptr: int, om_ptr: int, out_ptr: int, N: int, H: int, W: int, C: int, G: int, K: int,
             stride: int = 1, pad: int = 0, dilation: int = 1, offset_scale: float = 1.0,
             dtype: int = DCNV4_F32) -> int:
    """Raw status of dcnv4_validate for the given pointers and sizes (no launch)."""
    return load_library().dcnv4_validate(x_ptr, om_ptr, out_ptr, N, H, W, C, G, K, stride, pad, dilation,
                                         float(offset_scale), int(dtype))


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check_tensor(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype not in TORCH_DTYPE:
        raise TypeError(f"{name} has unsupported dtype {t.dtype}")


def forward(x: torch.Tensor, offset_mask: torch.Tensor, G: int, K: int, stride: int = 1, pad: int = 0,
            dilation: int = 1, offset_scale: float = 1.0, out: torch.Tensor | None = None,
            stream=None, softmax: bool = False, remove_center: bool = False,
            center_logit: torch.Tensor | None = None) -> torch.Tensor:
    """DCNv4 forward aggregation on the GPU through ``dcnv4_forward`` / ``dcnv4_forward_ex``.

    x: [N,H,W,C]; offset_mask: [N,Hout,Wout,G,3*P] (per group: P x-offsets,
    P y-offsets, P masks; P = K*K, or K*K-1 with ``remove_center``); returns
    out [N,Hout,Wout,C] in x's dtype. Variants: ``softmax`` (DCNv3-style
    softmax over each unit's masks), ``remove_center`` (the centre grid point
    is left out), ``center_logit`` [N,Hout,Wout,G] (centre feature scaling with
    gate sigmoid(center_logit)). The launch is asynchronous on ``stream``
    (default: the current stream).
    """
    _check_tensor(x, "x")
    _check_tensor(offset_mask, "offset_mask")
    if x.dim() != 4:
        raise ValueError("x must be [N,H,W,C]")
    if offset_mask.dtype != x.dtype or offset_mask.device != x.device:
        raise ValueError("offset_mask must match x in dtype and device")
    N, H, W, C = x.shape
    Hout, Wout = output_shape(H, W, K, stride, pad, dilation)
    P = K * K - (1 if remove_center else 0)
    want = (N, Hout, Wout, G, 3 * P)
    if tuple(offset_mask.shape) != want:
        raise ValueError(f"offset_mask shape {tuple(offset_mask.shape)} != {want}")
    flags = (FLAG_SOFTMAX if softmax else 0) | (FLAG_REMOVE_CENTER if remove_center else 0)
    zp = 0
    if center_logit is not None:
        _check_tensor(center_logit, "center_logit")
        if tuple(center_logit.shape) != (N, Hout, Wout, G) or center_logit.dtype != x.dtype or \
                center_logit.device != x.device:
            raise ValueError(f"center_logit must be [N,Hout,Wout,G] = {(N, Hout, Wout, G)} in x's dtype and device")
        flags |= FLAG_CENTER_SCALE
        zp = center_logit.data_ptr()
    if out is None:
        out = torch.empty((N, Hout, Wout, C), dtype=x.dtype, device=x.device)
    else:
        _check_tensor(out, "out")
        if tuple(out.shape) != (N, Hout, Wout, C) or out.dtype != x.dtype or out.device != x.device:
            raise ValueError("out has the wrong shape, dtype or device")
    with torch.cuda.device(x.device):
        lib = load_library()
        if flags:
            rc = lib.dcnv4_forward_ex(x.data_ptr(), offset_mask.data_ptr(), zp, out.data_ptr(), N, H, W, C, G, K,
                                      stride, pad, dilation, float(offset_scale), TORCH_DTYPE[x.dtype], flags,
                                      _stream_handle(stream))
        else:
            rc = lib.dcnv4_forward(x.data_ptr(), offset_mask.data_ptr(), out.data_ptr(), N, H, W, C, G, K,
                                   stride, pad, dilation, float(offset_scale), TORCH_DTYPE[x.dtype],
                                   _stream_handle(stream))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_forward_ex" if flags else "dcnv4_forward")
    return out


def backward(x: torch.Tensor, offset_mask: torch.Tensor, grad_out: torch.Tensor, G: int, K: int, stride: int = 1,
             pad: int = 0, dilation: int = 1, offset_scale: float = 1.0, grad_x: torch.Tensor | None = None,
             grad_offset_mask: torch.Tensor | None = None, stream=None, softmax: bool = False,
             remove_center: bool = False, center_logit: torch.Tensor | None = None):
    """DCNv4 backward on the GPU through ``dcnv4_backward`` / ``dcnv4_backward_ex``.

    x: [N,H,W,C]; offset_mask: [N,Hout,Wout,G,3*P]; grad_out: [N,Hout,Wout,C],
    all of one dtype; the variant switches as in ``forward``. Returns
    (grad_x [N,H,W,C], grad_offset_mask [N,Hout,Wout,G,3*P]), both fp32, plus
    grad_center_logit [N,Hout,Wout,G] (fp32) as a third element when
    ``center_logit`` is given. Asynchronous on ``stream`` (default: current).
    """
    for t, name in ((x, "x"), (offset_mask, "offset_mask"), (grad_out, "grad_out")):
        _check_tensor(t, name)
    if x.dim() != 4:
        raise ValueError("x must be [N,H,W,C]")
    if offset_mask.dtype != x.dtype or grad_out.dtype != x.dtype or offset_mask.device != x.device or \
            grad_out.device != x.device:
        raise ValueError("offset_mask and grad_out must match x in dtype and device")
    N, H, W, C = x.shape
    Hout, Wout = output_shape(H, W, K, stride, pad, dilation)
    P = K * K - (1 if remove_center else 0)
    if tuple(offset_mask.shape) != (N, Hout, Wout, G, 3 * P):
        raise ValueError(f"offset_mask shape {tuple(offset_mask.shape)} != {(N, Hout, Wout, G, 3 * P)}")
    if tuple(grad_out.shape) != (N, Hout, Wout, C):
        raise ValueError(f"grad_out shape {tuple(grad_out.shape)} != {(N, Hout, Wout, C)}")
    flags = (FLAG_SOFTMAX if softmax else 0) | (FLAG_REMOVE_CENTER if remove_center else 0)
    gz = None
    if center_logit is not None:
        _check_tensor(center_logit, "center_logit")
        if tuple(center_logit.shape) != (N, Hout, Wout, G) or center_logit.dtype != x.dtype or \
                center_logit.device != x.device:
            raise ValueError(f"center_logit must be [N,Hout,Wout,G] = {(N, Hout, Wout, G)} in x's dtype and device")
        flags |= FLAG_CENTER_SCALE
        gz = torch.empty((N, Hout, Wout, G), dtype=torch.float32, device=x.device)
    outs = []
    for t, shape, name in ((grad_x, x.shape, "grad_x"), (grad_offset_mask, offset_mask.shape, "grad_offset_mask")):
        if t is None:
            t = torch.empty(tuple(shape), dtype=torch.float32, device=x.device)
        else:
            _check_tensor(t, name)
            if tuple(t.shape) != tuple(shape) or t.dtype != torch.float32 or t.device != x.device:
                raise ValueError(f"{name} must be fp32 of shape {tuple(shape)} on {x.device}")
        outs.append(t)
    gx, gom = outs
    with torch.cuda.device(x.device):
        lib = load_library()
        if flags:
            rc = lib.dcnv4_backward_ex(x.data_ptr(), offset_mask.data_ptr(),
                                       0 if center_logit is None else center_logit.data_ptr(), grad_out.data_ptr(),
                                       gx.data_ptr(), gom.data_ptr(), 0 if gz is None else gz.data_ptr(),
                                       N, H, W, C, G, K, stride, pad, dilation, float(offset_scale),
                                       TORCH_DTYPE[x.dtype], flags, _stream_handle(stream))
        else:
            rc = lib.dcnv4_backward(x.data_ptr(), offset_mask.data_ptr(), grad_out.data_ptr(), gx.data_ptr(),
                                    gom.data_ptr(), N, H, W, C, G, K, stride, pad, dilation, float(offset_scale),
                                    TORCH_DTYPE[x.dtype], _stream_handle(stream))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_backward_ex" if flags else "dcnv4_backward")
    return (gx, gom) if gz is None else (gx, gom, gz)


def predictor(y: torch.Tensor, weight: torch.Tensor, bias: torch.Tensor | None, G: int, K: int,
              remove_center: bool = False, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Offset/mask predictor step through ``dcnv4_predictor``: 1x1 projection + packing.

    y: [..., C] channels-last (leading dims are the pixels); weight: [3*G*P, C]
    in the pages' channel order (all groups' offsets, then all groups'
    masks); bias: fp32 [3*G*P] or None. Returns offset_mask [..., G, 3*P] in
    y's dtype (P = K*K, or K*K-1 with ``remove_center``).
    """
    _check_tensor(y, "y")
    _check_tensor(weight, "weight")
    P = K * K - (1 if remove_center else 0)
    C = y.shape[-1]
    if weight.dtype != y.dtype or weight.device != y.device or tuple(weight.shape) != (3 * G * P, C):
        raise ValueError(f"weight must be [{3 * G * P}, {C}] in y's dtype and device")
    bp = 0
    if bias is not None:
        _check_tensor(bias, "bias")
        if bias.dtype != torch.float32 or tuple(bias.shape) != (3 * G * P,) or bias.device != y.device:
            raise ValueError(f"bias must be fp32 [{3 * G * P}] on y's device")
        bp = bias.data_ptr()
    lead = tuple(y.shape[:-1])
    M = 1
    for d in lead:
        M *= d
    shape = lead + (G, 3 * P)
    if out is None:
        out = torch.empty(shape, dtype=y.dtype, device=y.device)
    else:
        _check_tensor(out, "out")
        if tuple(out.shape) != shape or out.dtype != y.dtype or out.device != y.device:
            raise ValueError("out has the wrong shape, dtype or device")
    with torch.cuda.device(y.device):
        rc = load_library().dcnv4_predictor(y.data_ptr(), weight.data_ptr(), bp, out.data_ptr(), M, C, G, K,
                                            FLAG_REMOVE_CENTER if remove_center else 0, TORCH_DTYPE[y.dtype],
                                            _stream_handle(stream))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_predictor")
    return out


def forward_host(x: torch.Tensor, offset_mask: torch.Tensor, G: int, K: int, stride: int = 1, pad: int = 0,
                 dilation: int = 1, offset_scale: float = 1.0, out: torch.Tensor | None = None,
                 staging=None, device=None, stream=None) -> torch.Tensor:
    """Forward from host tensors through ``dcnv4_forward_host``.

    x, offset_mask: CPU tensors (pin them for overlapped copies); returns the
    CPU tensor ``out`` once the work is complete. ``staging`` = (x_dev,
    offset_mask_dev, out_dev) device tensors of the full sizes; allocated on
    ``device`` when not given.
    """
    for t, name in ((x, "x"), (offset_mask, "offset_mask")):
        if t.device.type != "cpu" or not t.is_contiguous() or t.dtype not in TORCH_DTYPE:
            raise ValueError(f"{name} must be a contiguous CPU tensor of a supported dtype")
    if offset_mask.dtype != x.dtype:
        raise ValueError("offset_mask must match x in dtype")
    N, H, W, C = x.shape
    Hout, Wout = output_shape(H, W, K, stride, pad, dilation)
    if tuple(offset_mask.shape) != (N, Hout, Wout, G, 3 * K * K):
        raise ValueError("offset_mask has the wrong shape")
    if out is None:
        out = torch.empty((N, Hout, Wout, C), dtype=x.dtype, pin_memory=x.is_pinned())
    if tuple(out.shape) != (N, Hout, Wout, C) or out.dtype != x.dtype or out.device.type != "cpu" \
            or not out.is_contiguous():
        raise ValueError("out must be a contiguous CPU tensor of the output shape and x's dtype")
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if staging is None:
        staging = (torch.empty_like(x, device=device), torch.empty_like(offset_mask, device=device),
                   torch.empty_like(out, device=device))
    xd, omd, od = staging
    for t, ref, name in ((xd, x, "x_dev"), (omd, offset_mask, "offset_mask_dev"), (od, out, "out_dev")):
        _check_tensor(t, name)
        if t.shape != ref.shape or t.dtype != ref.dtype or t.device != xd.device:
            raise ValueError(f"{name} must match the host tensor's shape and dtype on one device")
    with torch.cuda.device(xd.device):
        handle = _stream_handle(stream)
        rc = load_library().dcnv4_forward_host(x.data_ptr(), offset_mask.data_ptr(), out.data_ptr(),
                                               xd.data_ptr(), omd.data_ptr(), od.data_ptr(), N, H, W, C, G, K,
                                               stride, pad, dilation, float(offset_scale), TORCH_DTYPE[x.dtype],
                                               handle)
        if rc != DCNV4_OK:
            raise DCNv4Error(rc, "dcnv4_forward_host")
        (stream or torch.cuda.current_stream()).synchronize()
    return out


NOALLOC_STAGING_BYTES = 32 << 20


def forward_host_noalloc(x: torch.Tensor, offset_mask: torch.Tensor, G: int, K: int, stride: int = 1,
                         pad: int = 0, dilation: int = 1, offset_scale: float = 1.0,
                         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Forward from host tensors through ``dcnv4_forward_host_noalloc``.

    For callers that must not allocate device memory at call time: the
    library stages through its own fixed 32 MiB device array per GPU (shared
    by every call on that GPU; calls that overlap on the GPU race on it). The
    output tensor is allocated on the host here when not given; pass ``out``
    to allocate nothing at all. Returns ``out`` once the work is complete.
    """
    for t, name in ((x, "x"), (offset_mask, "offset_mask")):
        if t.device.type != "cpu" or not t.is_contiguous() or t.dtype not in TORCH_DTYPE:
            raise ValueError(f"{name} must be a contiguous CPU tensor of a supported dtype")
    if offset_mask.dtype != x.dtype:
        raise ValueError("offset_mask must match x in dtype")
    N, H, W, C = x.shape
    Hout, Wout = output_shape(H, W, K, stride, pad, dilation)
    if tuple(offset_mask.shape) != (N, Hout, Wout, G, 3 * K * K):
        raise ValueError("offset_mask has the wrong shape")
    if out is None:
        out = torch.empty((N, Hout, Wout, C), dtype=x.dtype, pin_memory=x.is_pinned())
    if tuple(out.shape) != (N, Hout, Wout, C) or out.dtype != x.dtype or out.device.type != "cpu" \
            or not out.is_contiguous():
        raise ValueError("out must be a contiguous CPU tensor of the output shape and x's dtype")
    handle = _stream_handle(stream)
    rc = load_library().dcnv4_forward_host_noalloc(x.data_ptr(), offset_mask.data_ptr(), out.data_ptr(), N, H, W,
                                                   C, G, K, stride, pad, dilation, float(offset_scale),
                                                   TORCH_DTYPE[x.dtype], handle)
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_forward_host_noalloc")
    (stream or torch.cuda.current_stream()).synchronize()
    return out


def sampling_index(offset_mask: torch.Tensor, H: int, W: int, G: int, K: int, stride: int = 1, pad: int = 0,
                   dilation: int = 1, offset_scale: float = 1.0, stream=None):
    """Corner (y0, x0) [N,Hout,Wout,G,K*K,2] int32 and validity bits [N,Hout,Wout,G,K*K] uint8
    through ``dcnv4_sampling_index``."""
    _check_tensor(offset_mask, "offset_mask")
    N, Hout, Wout, G_, R = offset_mask.shape
    if G_ != G or R != 3 * K * K or (Hout, Wout) != output_shape(H, W, K, stride, pad, dilation):
        raise ValueError("offset_mask shape does not match H, W, G, K")
    corner = torch.empty((N, Hout, Wout, G, K * K, 2), dtype=torch.int32, device=offset_mask.device)
    valid = torch.empty((N, Hout, Wout, G, K * K), dtype=torch.uint8, device=offset_mask.device)
    with torch.cuda.device(offset_mask.device):
        rc = load_library().dcnv4_sampling_index(offset_mask.data_ptr(), corner.data_ptr(), valid.data_ptr(),
                                                 N, H, W, G, K, stride, pad, dilation, float(offset_scale),
                                                 TORCH_DTYPE[offset_mask.dtype], _stream_handle(stream))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_sampling_index")
    return corner, valid

# path codes of forward_trace
TRACE_WINDOW, TRACE_GLOBAL_PASS, TRACE_GATHER_KERNEL = 0, 1, 2


def forward_trace(x: torch.Tensor, offset_mask: torch.Tensor, G: int, K: int, stride: int = 1, pad: int = 0,
                  dilation: int = 1, offset_scale: float = 1.0, stream=None):
    """The forward through ``dcnv4_forward_trace``: returns (out, trace).

    out is what ``forward`` returns, bit for bit; trace [N,Hout,Wout,G,K*K,4]
    int32 holds, per sampling point, the top-left corner (y0, x0) and the
    validity bits that the gather used, and the path it took (0: the ring
    kernel's shared-memory window, 1: its global-memory pass, 2: the
    global-gather kernel).
    """
    _check_tensor(x, "x")
    _check_tensor(offset_mask, "offset_mask")
    if offset_mask.dtype != x.dtype or offset_mask.device != x.device:
        raise ValueError("offset_mask must match x in dtype and device")
    N, H, W, C = x.shape
    Hout, Wout = output_shape(H, W, K, stride, pad, dilation)
    if tuple(offset_mask.shape) != (N, Hout, Wout, G, 3 * K * K):
        raise ValueError("offset_mask shape does not match H, W, G, K")
    out = torch.empty((N, Hout, Wout, C), dtype=x.dtype, device=x.device)
    trace = torch.empty((N, Hout, Wout, G, K * K, 4), dtype=torch.int32, device=x.device)
    with torch.cuda.device(x.device):
        rc = load_library().dcnv4_forward_trace(x.data_ptr(), offset_mask.data_ptr(), out.data_ptr(),
                                                trace.data_ptr(), N, H, W, C, G, K, stride, pad, dilation,
                                                float(offset_scale), TORCH_DTYPE[x.dtype], _stream_handle(stream))
    if rc != DCNV4_OK:
        raise DCNv4Error(rc, "dcnv4_forward_trace")
    return out, trace
