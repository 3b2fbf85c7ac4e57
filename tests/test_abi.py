"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every symbol include/dcnv4.h declares, and its argument checks return the
documented status for every error class without launching anything."""
import ctypes
import os
import re

import pytest

import oracle
from deformable_convolution_sparse_b200 import binding as B
from deformable_convolution_sparse_b200.workloads import WORKLOADS

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "dcnv4.h")


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DCNV4_API\s+[\w\s\*]*?\b(dcnv4_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert _declared_symbols() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = B.load_library()
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert B.abi_version() == 1


def test_strerror_covers_every_status():
    for code, name in B.STATUS_NAMES.items():
        msg = B.strerror(code)
        assert msg and msg != "unknown status", name
    assert B.strerror(12345) == "unknown status"


@pytest.mark.parametrize("H,W,K,s,p,d", [(56, 56, 3, 1, 1, 1), (256, 256, 3, 1, 1, 2), (14, 9, 3, 2, 1, 1),
                                         (9, 11, 5, 3, 2, 2), (4, 4, 2, 2, 0, 2), (1, 1, 1, 1, 0, 1),
                                         (7, 5, 1, 4, 0, 1), (3, 3, 16, 1, 8, 1)])
def test_output_shape_matches_oracle(H, W, K, s, p, d):
    assert B.output_shape(H, W, K, s, p, d) == (oracle.output_size(H, K, s, p, d), oracle.output_size(W, K, s, p, d))


def test_named_workloads_state_the_right_output_size():
    for w in WORKLOADS.values():
        assert (w.Hout, w.Wout) == B.output_shape(w.H, w.W, w.K, w.stride, w.pad, w.dilation), w.name
        assert w.Hout == oracle.output_size(w.H, w.K, w.stride, w.pad, w.dilation), w.name


@pytest.mark.parametrize("args", [(0, 5, 3, 1, 1, 1), (5, 0, 3, 1, 1, 1), (5, 5, 0, 1, 1, 1), (5, 5, 3, 0, 1, 1),
                                  (5, 5, 3, 1, -1, 1), (5, 5, 3, 1, 1, 0), (2, 2, 5, 1, 0, 1), (5, 5, 17, 1, 8, 1),
                                  (1 << 23, 5, 3, 1, 1, 1)])
def test_output_shape_rejects_bad_geometry(args):
    lib = B.load_library()
    ho, wo = ctypes.c_int(-7), ctypes.c_int(-7)
    assert lib.dcnv4_output_shape(*args, ctypes.byref(ho), ctypes.byref(wo)) == B.STATUS["DCNV4_ERR_SHAPE"]
    assert (ho.value, wo.value) == (-7, -7)


# fake, never dereferenced device addresses
X, OM, OUT = 0x10000000, 0x20000000, 0x30000000
GOOD = dict(N=2, H=8, W=8, C=16, G=2, K=3, stride=1, pad=1, dilation=1, offset_scale=1.0, dtype=B.DCNV4_F16)


def _v(x=X, om=OM, out=OUT, **kw):
    a = dict(GOOD)
    a.update(kw)
    return B.validate(x, om, out, a["N"], a["H"], a["W"], a["C"], a["G"], a["K"], a["stride"], a["pad"],
                      a["dilation"], a["offset_scale"], a["dtype"])


def test_validate_accepts_good_arguments():
    assert _v() == B.DCNV4_OK
    assert _v(dtype=B.DCNV4_F32) == B.DCNV4_OK
    assert _v(dtype=B.DCNV4_BF16, offset_scale=-0.5) == B.DCNV4_OK
    assert _v(x=0, om=0, out=0, N=0) == B.DCNV4_OK  # empty batch: nothing is touched


@pytest.mark.parametrize("kw,status", [
    (dict(x=0), "DCNV4_ERR_NULL"), (dict(om=0), "DCNV4_ERR_NULL"), (dict(out=0), "DCNV4_ERR_NULL"),
    (dict(N=-1), "DCNV4_ERR_SHAPE"), (dict(H=0), "DCNV4_ERR_SHAPE"), (dict(C=0), "DCNV4_ERR_SHAPE"),
    (dict(G=0), "DCNV4_ERR_SHAPE"), (dict(K=0), "DCNV4_ERR_SHAPE"), (dict(stride=0), "DCNV4_ERR_SHAPE"),
    (dict(pad=-1), "DCNV4_ERR_SHAPE"), (dict(dilation=-2), "DCNV4_ERR_SHAPE"),
    (dict(H=2, W=2, pad=0), "DCNV4_ERR_SHAPE"),
    (dict(C=18, G=4), "DCNV4_ERR_GROUPS"),
    (dict(dtype=3), "DCNV4_ERR_DTYPE"), (dict(dtype=-1), "DCNV4_ERR_DTYPE"),
    (dict(x=X + 1), "DCNV4_ERR_ALIGN"), (dict(om=OM + 1), "DCNV4_ERR_ALIGN"), (dict(out=OUT + 3), "DCNV4_ERR_ALIGN"),
    (dict(x=X + 2, dtype=B.DCNV4_F32), "DCNV4_ERR_ALIGN"),
    (dict(out=X), "DCNV4_ERR_ALIAS"), (dict(out=OM + 64), "DCNV4_ERR_ALIAS"), (dict(x=OUT - 32), "DCNV4_ERR_ALIAS"),
    (dict(offset_scale=float("nan")), "DCNV4_ERR_SCALE"), (dict(offset_scale=float("inf")), "DCNV4_ERR_SCALE"),
    (dict(N=1 << 20, H=64, W=64, C=64, G=4), "DCNV4_ERR_TOO_LARGE"),
])
def test_validate_reports_each_error_class(kw, status):
    assert _v(**kw) == B.STATUS[status]


def test_inputs_may_overlap_each_other():
    # x and offset_mask are both read only: sharing memory is allowed
    assert _v(om=X) == B.DCNV4_OK


def test_forward_returns_validation_errors_before_any_cuda_call():
    lib = B.load_library()
    a = dict(GOOD)
    rc = lib.dcnv4_forward(X, OM, OUT, a["N"], a["H"], a["W"], 18, 4, a["K"], 1, 1, 1, 1.0, a["dtype"], None)
    assert rc == B.STATUS["DCNV4_ERR_GROUPS"]
    rc = lib.dcnv4_forward(X, OM, X, a["N"], a["H"], a["W"], 16, 2, 3, 1, 1, 1, 1.0, a["dtype"], None)
    assert rc == B.STATUS["DCNV4_ERR_ALIAS"]
    # an empty batch launches nothing and succeeds, also without a GPU
    assert lib.dcnv4_forward(0, 0, 0, 0, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, a["dtype"], None) == B.DCNV4_OK


def test_sampling_index_checks():
    lib = B.load_library()
    assert lib.dcnv4_sampling_index(OM, X, OUT, 1, 8, 8, 2, 3, 1, 1, 1, 1.0, 5, None) == B.STATUS["DCNV4_ERR_DTYPE"]
    assert lib.dcnv4_sampling_index(0, X, OUT, 1, 8, 8, 2, 3, 1, 1, 1, 1.0, 1, None) == B.STATUS["DCNV4_ERR_NULL"]
    assert lib.dcnv4_sampling_index(OM, X + 2, OUT, 1, 8, 8, 2, 3, 1, 1, 1, 1.0, 1, None) == B.STATUS["DCNV4_ERR_ALIGN"]
    assert lib.dcnv4_sampling_index(OM, OM, OUT, 1, 8, 8, 2, 3, 1, 1, 1, 1.0, 1, None) == B.STATUS["DCNV4_ERR_ALIAS"]
    assert lib.dcnv4_sampling_index(0, 0, 0, 0, 8, 8, 2, 3, 1, 1, 1, 1.0, 1, None) == B.DCNV4_OK


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 8, 8, 16)
    om = torch.zeros(1, 8, 8, 2, 27)
    with pytest.raises(ValueError, match="CUDA"):
        B.forward(x, om, G=2, K=3, pad=1)


GX, GOM = 0x40000000, 0x50000000


def _bw(x=X, om=OM, go=OUT, gx=GX, gom=GOM, **kw):
    a = dict(GOOD)
    a.update(kw)
    return B.load_library().dcnv4_backward(x, om, go, gx, gom, a["N"], a["H"], a["W"], a["C"], a["G"], a["K"],
                                           a["stride"], a["pad"], a["dilation"], a["offset_scale"], a["dtype"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=0), "DCNV4_ERR_NULL"), (dict(go=0), "DCNV4_ERR_NULL"), (dict(gx=0), "DCNV4_ERR_NULL"),
    (dict(gom=0), "DCNV4_ERR_NULL"),
    (dict(N=-1), "DCNV4_ERR_SHAPE"), (dict(K=17), "DCNV4_ERR_SHAPE"), (dict(C=18, G=4), "DCNV4_ERR_GROUPS"),
    (dict(dtype=7), "DCNV4_ERR_DTYPE"), (dict(offset_scale=float("nan")), "DCNV4_ERR_SCALE"),
    (dict(go=OUT + 1), "DCNV4_ERR_ALIGN"), (dict(gx=GX + 2), "DCNV4_ERR_ALIGN"), (dict(gom=GOM + 2), "DCNV4_ERR_ALIGN"),
    # outputs may not overlap any input nor each other
    (dict(gx=X), "DCNV4_ERR_ALIAS"), (dict(gx=OUT + 64), "DCNV4_ERR_ALIAS"), (dict(gom=OM + 16), "DCNV4_ERR_ALIAS"),
    (dict(gom=GX + 64), "DCNV4_ERR_ALIAS"),
    (dict(N=1 << 20, H=64, W=64, C=64, G=4), "DCNV4_ERR_TOO_LARGE"),
])
def test_backward_reports_each_error_class_before_any_cuda_call(kw, status):
    assert _bw(**kw) == B.STATUS[status]


def test_backward_empty_batch_touches_nothing():
    assert _bw(x=0, om=0, go=0, gx=0, gom=0, N=0) == B.DCNV4_OK


def test_backward_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 8, 8, 16)
    om = torch.zeros(1, 8, 8, 2, 27)
    with pytest.raises(ValueError, match="CUDA"):
        B.backward(x, om, torch.zeros(1, 8, 8, 16), G=2, K=3, pad=1)


def _vex(x=X, om=OM, z=0x60000000, out=OUT, flags=0, **kw):
    a = dict(GOOD)
    a.update(kw)
    return B.load_library().dcnv4_validate_ex(x, om, z, out, a["N"], a["H"], a["W"], a["C"], a["G"], a["K"],
                                              a["stride"], a["pad"], a["dilation"], a["offset_scale"], a["dtype"],
                                              flags)


def test_validate_ex_checks_the_variant_flags():
    assert _vex(flags=0) == B.DCNV4_OK
    assert _vex(flags=B.FLAG_SOFTMAX | B.FLAG_REMOVE_CENTER | B.FLAG_CENTER_SCALE) == B.DCNV4_OK
    assert _vex(flags=8) == B.STATUS["DCNV4_ERR_FLAGS"]
    assert _vex(flags=0x80000000) == B.STATUS["DCNV4_ERR_FLAGS"]
    # no centre to remove for an even kernel or K = 1
    assert _vex(flags=B.FLAG_REMOVE_CENTER, K=2, pad=0) == B.STATUS["DCNV4_ERR_SHAPE"]
    assert _vex(flags=B.FLAG_REMOVE_CENTER, K=1, pad=0) == B.STATUS["DCNV4_ERR_SHAPE"]
    # the gate logits are needed, aligned and disjoint from out only with centre scaling
    assert _vex(z=0, flags=B.FLAG_CENTER_SCALE) == B.STATUS["DCNV4_ERR_NULL"]
    assert _vex(z=0, flags=B.FLAG_SOFTMAX) == B.DCNV4_OK
    assert _vex(z=0x60000001, flags=B.FLAG_CENTER_SCALE) == B.STATUS["DCNV4_ERR_ALIGN"]
    assert _vex(z=OUT + 64, flags=B.FLAG_CENTER_SCALE) == B.STATUS["DCNV4_ERR_ALIAS"]
    assert _vex(z=OUT + 64, flags=B.FLAG_SOFTMAX) == B.DCNV4_OK


def test_forward_ex_returns_flag_errors_before_any_cuda_call():
    lib = B.load_library()
    a = dict(GOOD)
    rc = lib.dcnv4_forward_ex(X, OM, 0, OUT, a["N"], a["H"], a["W"], 16, 2, 3, 1, 1, 1, 1.0, a["dtype"], 16, None)
    assert rc == B.STATUS["DCNV4_ERR_FLAGS"]
    rc = lib.dcnv4_forward_ex(X, OM, 0, OUT, a["N"], a["H"], a["W"], 16, 2, 4, 1, 1, 1, 1.0, a["dtype"],
                              B.FLAG_REMOVE_CENTER, None)
    assert rc == B.STATUS["DCNV4_ERR_SHAPE"]
    assert lib.dcnv4_forward_ex(0, 0, 0, 0, 0, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, a["dtype"], 7, None) == B.DCNV4_OK


def _pred(y=X, w=OM, b=0, rec=OUT, M=1000, C=64, G=4, K=3, flags=0, dtype=B.DCNV4_F16):
    return B.load_library().dcnv4_predictor(y, w, b, rec, M, C, G, K, flags, dtype, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=-1), "DCNV4_ERR_SHAPE"), (dict(C=0), "DCNV4_ERR_SHAPE"), (dict(G=0), "DCNV4_ERR_SHAPE"),
    (dict(K=17), "DCNV4_ERR_SHAPE"), (dict(K=2, flags=B.FLAG_REMOVE_CENTER), "DCNV4_ERR_SHAPE"),
    (dict(flags=B.FLAG_SOFTMAX), "DCNV4_ERR_FLAGS"), (dict(dtype=9), "DCNV4_ERR_DTYPE"),
    (dict(y=0), "DCNV4_ERR_NULL"), (dict(w=0), "DCNV4_ERR_NULL"), (dict(rec=0), "DCNV4_ERR_NULL"),
    (dict(y=X + 1), "DCNV4_ERR_ALIGN"), (dict(b=0x70000002), "DCNV4_ERR_ALIGN"),
    (dict(rec=X + 64), "DCNV4_ERR_ALIAS"), (dict(rec=OM), "DCNV4_ERR_ALIAS"), (dict(b=OUT + 16), "DCNV4_ERR_ALIAS"),
    (dict(M=1 << 25, C=128), "DCNV4_ERR_TOO_LARGE"),
])
def test_predictor_reports_each_error_class_before_any_cuda_call(kw, status):
    assert _pred(**kw) == B.STATUS[status]


def test_predictor_empty_batch_touches_nothing():
    assert _pred(y=0, w=0, rec=0, M=0) == B.DCNV4_OK


def _bwx(x=X, om=OM, z=0x60000000, go=OUT, gx=GX, gom=GOM, gz=0x70000000, flags=0, **kw):
    a = dict(GOOD)
    a.update(kw)
    return B.load_library().dcnv4_backward_ex(x, om, z, go, gx, gom, gz, a["N"], a["H"], a["W"], a["C"], a["G"],
                                              a["K"], a["stride"], a["pad"], a["dilation"], a["offset_scale"],
                                              a["dtype"], flags, None)


@pytest.mark.parametrize("kw,status", [
    (dict(flags=8), "DCNV4_ERR_FLAGS"), (dict(flags=B.FLAG_REMOVE_CENTER, K=4, pad=1), "DCNV4_ERR_SHAPE"),
    (dict(flags=B.FLAG_CENTER_SCALE, z=0), "DCNV4_ERR_NULL"), (dict(flags=B.FLAG_CENTER_SCALE, gz=0), "DCNV4_ERR_NULL"),
    (dict(flags=B.FLAG_CENTER_SCALE, gz=0x70000002), "DCNV4_ERR_ALIGN"),
    (dict(flags=B.FLAG_CENTER_SCALE, z=0x60000001), "DCNV4_ERR_ALIGN"),
    (dict(flags=B.FLAG_CENTER_SCALE, gz=GX + 64), "DCNV4_ERR_ALIAS"),
    (dict(flags=B.FLAG_CENTER_SCALE, gz=X), "DCNV4_ERR_ALIAS"),
    (dict(flags=B.FLAG_CENTER_SCALE, gx=0x60000000), "DCNV4_ERR_ALIAS"),
    (dict(gx=0), "DCNV4_ERR_NULL"), (dict(go=OUT + 1), "DCNV4_ERR_ALIGN"),
])
def test_backward_ex_reports_each_error_class_before_any_cuda_call(kw, status):
    assert _bwx(**kw) == B.STATUS[status]


def test_backward_ex_empty_batch_touches_nothing():
    assert _bwx(x=0, om=0, z=0, go=0, gx=0, gom=0, gz=0, N=0, flags=7) == B.DCNV4_OK


def test_forward_trace_checks():
    lib = B.load_library()
    TR = 0x40000000
    a = dict(GOOD)
    args = (a["N"], a["H"], a["W"], a["C"], a["G"], a["K"], 1, 1, 1, ctypes.c_float(1.0), a["dtype"], None)
    # the forward's own checks come first
    assert lib.dcnv4_forward_trace(X, OM, X, TR, *args) == B.STATUS["DCNV4_ERR_ALIAS"]
    # then the trace buffer: present, 16-byte aligned, overlapping nothing
    assert lib.dcnv4_forward_trace(X, OM, OUT, 0, *args) == B.STATUS["DCNV4_ERR_NULL"]
    assert lib.dcnv4_forward_trace(X, OM, OUT, TR + 4, *args) == B.STATUS["DCNV4_ERR_ALIGN"]
    assert lib.dcnv4_forward_trace(X, OM, OUT, OUT, *args) == B.STATUS["DCNV4_ERR_ALIAS"]
    assert lib.dcnv4_forward_trace(X, OM, OUT, OM - 64, *args) == B.STATUS["DCNV4_ERR_ALIAS"]
    # an empty batch launches nothing and succeeds, also without a GPU
    assert lib.dcnv4_forward_trace(0, 0, 0, 0, 0, 8, 8, 16, 2, 3, 1, 1, 1, ctypes.c_float(1.0), a["dtype"],
                                   None) == B.DCNV4_OK


def test_probe_smem_gather_checks_before_any_cuda_call():
    lib = B.load_library()
    v = ctypes.c_double(0.0)
    assert lib.dcnv4_probe_smem_gather(0, None) == B.STATUS["DCNV4_ERR_NULL"]
    assert lib.dcnv4_probe_smem_gather(7, ctypes.byref(v)) == B.STATUS["DCNV4_ERR_SHAPE"]


def test_probe_red_global_checks_before_any_cuda_call():
    lib = B.load_library()
    v = ctypes.c_double(0.0)
    assert lib.dcnv4_probe_red_global(64, None) == B.STATUS["DCNV4_ERR_NULL"]
    for bad in (0, 16, 48, 256):
        assert lib.dcnv4_probe_red_global(bad, ctypes.byref(v)) == B.STATUS["DCNV4_ERR_SHAPE"]


def test_probe_red_shared_checks_before_any_cuda_call():
    lib = B.load_library()
    v = ctypes.c_double(0.0)
    assert lib.dcnv4_probe_red_shared(1, None) == B.STATUS["DCNV4_ERR_NULL"]
    assert lib.dcnv4_probe_red_shared(2, ctypes.byref(v)) == B.STATUS["DCNV4_ERR_SHAPE"]
