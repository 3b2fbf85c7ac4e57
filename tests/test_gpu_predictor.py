"""GPU parity of the offset/mask predictor step (dcnv4_predictor through the C
ABI: 1x1 projection + packing into offset_mask records; tcgen05 tensor-core
kernel for fp16/bf16, CUDA-core kernel otherwise) against the oracle, and the
predictor -> aggregation pipeline. Bars as the forward's: max|err| <= 4e-3 *
max|ref| for fp16/bf16 (one rounding of an fp32 sum), 1e-5 for fp32."""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 4e-3, "bf16": 4e-3}
TD = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(params=["auto", "wring", "epi8", "stages8", "plain"])
def pred_variant(request, monkeypatch):
    """The default choice (tensor cores where the shape allows, 16 epilogue
    warps, 4 stages, weights staged through the idle output area), the same
    with the weights staged through the activation ring, with 8 epilogue
    warps, with an 8-deep activation ring, and the CUDA-core kernel forced
    with DCNV4_PRED_VARIANT=plain."""
    for v in ("DCNV4_PRED_VARIANT", "DCNV4_PRED_EPI", "DCNV4_PRED_STAGES", "DCNV4_PRED_WSTAGE"):
        monkeypatch.delenv(v, raising=False)
    if request.param == "plain":
        monkeypatch.setenv("DCNV4_PRED_VARIANT", "plain")
    elif request.param == "epi8":
        monkeypatch.setenv("DCNV4_PRED_EPI", "8")
    elif request.param == "wring":   # the weights staged through the activation ring
        monkeypatch.setenv("DCNV4_PRED_WSTAGE", "0")
    elif request.param == "stages8":   # an 8-deep activation ring where it fits
        monkeypatch.setenv("DCNV4_PRED_STAGES", "8")
    return request.param


def _tensors(M, C, G, P, dtype, seed, bias=True, scale=None):
    g = torch.Generator().manual_seed(seed)
    y = torch.randn(M, C, generator=g).to(TD[dtype])
    w = (torch.randn(3 * G * P, C, generator=g) * (scale if scale else C ** -0.5)).to(TD[dtype])
    b = torch.randn(3 * G * P, generator=g) if bias else None
    return y, w, b


def _check(got, y, w, b, G, P, dtype):
    ref = oracle.dcnv4_predictor(y.double().numpy(), w.double().numpy(), None if b is None else b.double().numpy(),
                                 G=G, P=P)
    g = got.double().cpu().numpy()
    assert g.shape == ref.shape
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(g - ref).max()
    assert err <= TOL[dtype] * scale, f"max|err| {err:.3e} > {TOL[dtype]} * {scale:.3e}"


CASES = [
    # M, C, G, K, remove_center, bias
    (200704, 64, 4, 3, False, True),    # the stage-1 predictor: 64*56*56 pixels, 108 channels
    (1000, 64, 4, 3, False, False),     # ragged last tile, no bias
    (129, 128, 8, 3, False, True),      # 216 channels, 2 k-blocks
    (128, 256, 2, 3, False, True),      # exactly one tile, 4 k-blocks
    (4097, 192, 4, 3, True, True),      # no centre: 96 channels
    (300, 64, 1, 1, False, True),       # 3 channels (N padded to 16)
    (77, 320, 8, 3, False, True),       # 5 k-blocks (the SD latent width)
    (500, 48, 2, 3, False, True),       # C not a multiple of 64: CUDA-core kernel
    (333, 64, 16, 3, False, True),      # 432 channels: CUDA-core kernel
    (1, 64, 4, 3, False, True),         # one pixel
    (40, 2048, 1, 1, False, True),      # 32 k-blocks do not fit shared memory: CUDA-core kernel
]


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_predictor_matches_the_oracle(case, dtype, pred_variant, cuda_device):
    M, C, G, K, rc, bias = case
    P = K * K - (1 if rc else 0)
    y, w, b = _tensors(M, C, G, P, dtype, seed=M + C + G)
    got = dcn.predictor(y.to(cuda_device), w.to(cuda_device), None if b is None else b.to(cuda_device), G=G, K=K,
                        remove_center=rc)
    torch.cuda.synchronize()
    _check(got, y, w, b, G, P, dtype)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_outputs_overwritten_guard_bands_untouched_and_misaligned_output(dtype, cuda_device):
    M, C, G, K = 1000, 64, 4, 3
    P = K * K
    y, w, b = _tensors(M, C, G, P, dtype, seed=3)
    n, guard = M * G * 3 * P, 64
    for shift in (0, 1):   # 1: a 2-byte offset, so the output is not 16-byte aligned
        buf = torch.full((n + 2 * guard + shift,), 7.0, dtype=TD[dtype], device=cuda_device)
        out = buf[guard + shift:guard + shift + n].view(M, G, 3 * P)
        dcn.predictor(y.to(cuda_device), w.to(cuda_device), b.to(cuda_device), G=G, K=K, out=out)
        torch.cuda.synchronize()
        assert torch.all(buf[:guard + shift] == 7.0) and torch.all(buf[guard + shift + n:] == 7.0)
        _check(out, y, w, b, G, P, dtype)


def test_predictor_then_aggregation_matches_the_oracle_pipeline(cuda_device):
    # y (the depthwise output) -> records -> forward over x, stage-1 geometry on 4 images
    wl = WORKLOADS["stage1_f16"]
    x, _ = make_inputs(4, wl.H, wl.W, wl.C, wl.G, wl.K, wl.Hout, wl.Wout, "f16", seed=5)
    P = wl.K * wl.K
    y, w, b = _tensors(4 * wl.Hout * wl.Wout, wl.C, wl.G, P, "f16", seed=6, scale=0.3)
    y = y.view(4, wl.Hout, wl.Wout, wl.C)
    rec = dcn.predictor(y.to(cuda_device), w.to(cuda_device), b.to(cuda_device), G=wl.G, K=wl.K)
    out = dcn.forward(x.to(cuda_device), rec, **wl.kwargs())
    torch.cuda.synchronize()
    # the oracle pipeline on the GPU's (rounded) records isolates the aggregation ...
    ref = oracle.dcnv4_forward(x.double().numpy(), rec.double().cpu().numpy(), **wl.kwargs())
    assert np.abs(out.double().cpu().numpy() - ref).max() <= 4e-3 * np.abs(ref).max()
    # ... and the records themselves match the oracle's predictor
    _check(rec.view(-1, wl.G, 3 * P), y.view(-1, wl.C), w, b, wl.G, P, "f16")


def test_predictor_and_aggregation_chained_without_synchronisation(monkeypatch, cuda_device):
    """predictor -> forward -> predictor -> forward ... on one stream with no
    synchronisation: both kernels are launched with programmatic stream
    serialisation and wait for the kernel before them, so every forward reads
    the records its predictor wrote and every predictor the activations it was
    given. The chain must give the bits of the same chain with a device
    synchronisation after every launch, and of plain serialisation
    (DCNV4_PDL=0)."""
    for v in ("DCNV4_PRED_VARIANT", "DCNV4_PRED_EPI", "DCNV4_PRED_STAGES", "DCNV4_PRED_WSTAGE", "DCNV4_VARIANT"):
        monkeypatch.delenv(v, raising=False)
    wl = WORKLOADS["stage1_f16"]
    n = 8
    P = wl.K * wl.K
    x, _ = make_inputs(n, wl.H, wl.W, wl.C, wl.G, wl.K, wl.Hout, wl.Wout, "f16", seed=15)
    ws = []
    for i in range(4):
        _, w, b = _tensors(8, wl.C, wl.G, P, "f16", seed=20 + i, scale=0.05)
        ws.append((w.to(cuda_device), b.to(cuda_device)))
    x0 = x.to(cuda_device)

    def chain(sync):
        cur = x0
        for w, b in ws:
            rec = dcn.predictor(cur, w, b, G=wl.G, K=wl.K)      # the activations themselves as the predictor input
            if sync:
                torch.cuda.synchronize()
            cur = dcn.forward(cur, rec, **wl.kwargs())
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return cur

    fast = chain(False)
    step = chain(True)
    monkeypatch.setenv("DCNV4_PDL", "0")
    plain = chain(False)
    assert torch.equal(fast.view(torch.int16), step.view(torch.int16))
    assert torch.equal(fast.view(torch.int16), plain.view(torch.int16))
    assert torch.isfinite(fast).all()
