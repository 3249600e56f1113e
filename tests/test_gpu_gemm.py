"""tcgen05 GEMM (sl_gemm_bf16) against the plain definition C = A B^T in fp64,
over every epilogue, tile width and K split, with ragged M tails."""
import numpy as np
import pytest
import torch

from token_locking_b200 import _abi as A
from token_locking_b200 import runtime as rt

pytestmark = pytest.mark.gpu


def _mk(shape, seed, dev):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(dev, torch.bfloat16)


def _ref(a, b):
    return a.double().cpu() @ b.double().cpu().T


def _close(got, ref, K, bf16_out):
    got = got.double().cpu()
    scale = ref.abs().max().item() + 1e-6
    err = (got - ref).abs().max().item()
    # fp32 accumulation of K bf16 products; bf16 output rounding 2^-8 relative
    tol = (4e-3 * scale) if bf16_out else (1e-5 * np.sqrt(K) * scale + 1e-4)
    assert err <= tol, f"max err {err} > tol {tol} (scale {scale})"


VARIANTS = [(64, 0), (128, 0), (192, 0), (256, 0), (64, 1), (128, 1), (192, 1), (256, 1), (128, 2),
            (192, 2), (256, 2)]


@pytest.mark.parametrize("bn,variant", VARIANTS)
@pytest.mark.parametrize("M", [1, 37, 128, 301])
def test_store_rowmap(cuda_dev, bn, variant, M):
    K, N = 512, 768
    a, b = _mk((M, K), 1, cuda_dev), _mk((N, K), 2, cuda_dev)
    perm = torch.randperm(M + 5, generator=torch.Generator().manual_seed(3))[:M].to(torch.int32)
    out = torch.full((M + 5, N), 7.0, device=cuda_dev, dtype=torch.bfloat16)
    rt.gemm_bf16(A.GEMM_STORE, a, b, out, row_map=perm.to(cuda_dev), bn=bn, splits=1,
                 variant=variant)
    torch.cuda.synchronize()
    ref = _ref(a, b)
    _close(out[perm.long()], ref, K, True)
    untouched = torch.ones(M + 5, dtype=torch.bool)
    untouched[perm.long()] = False
    assert torch.all(out[untouched.to(cuda_dev)] == 7.0)
    rt.device_check()


@pytest.mark.parametrize("bn,splits,variant", [(64, 1, 0), (128, 3, 0), (256, 2, 0), (128, 8, 0),
                                               (256, 3, 1), (128, 1, 1), (64, 2, 1), (256, 1, 2),
                                               (256, 3, 2), (128, 2, 2), (256, -1, 0), (64, -1, 0),
                                               (128, -1, 1), (256, -1, 2), (128, -1, 2), (192, 1, 0),
                                               (192, 3, 1), (192, -1, 0), (192, 2, 2), (192, -1, 2)])
@pytest.mark.parametrize("M", [5, 130, 600])
def test_resid_split(cuda_dev, bn, splits, variant, M):
    K, N = 1024, 768
    a, b = _mk((M, K), 4, cuda_dev), _mk((N, K), 5, cuda_dev)
    h0 = torch.randn((M, N), generator=torch.Generator().manual_seed(6)).to(cuda_dev)
    h = h0.clone()
    rt.gemm_bf16(A.GEMM_RESID, a, b, h, bn=bn, splits=splits, variant=variant)
    torch.cuda.synchronize()
    _close(h - h0, _ref(a, b), K, False)
    rt.device_check()


@pytest.mark.parametrize("bn,variant", [(64, 0), (128, 0), (192, 0), (256, 0), (128, 1), (192, 1),
                                        (256, 1), (128, 2), (192, 2), (256, 2)])
@pytest.mark.parametrize("M", [3, 129, 300])
def test_swiglu(cuda_dev, bn, variant, M):
    K, F = 256, 384
    if F % (bn // 2):
        pytest.skip("F must split into bn/2 halves")
    a = _mk((M, K), 7, cuda_dev)
    wg, wu = _mk((F, K), 8, cuda_dev) * 0.1, _mk((F, K), 9, cuda_dev) * 0.1
    out = torch.zeros((M, F), device=cuda_dev, dtype=torch.bfloat16)
    rt.gemm_bf16(A.GEMM_SWIGLU, a, wg, out, b2=wu, bn=bn, splits=1, variant=variant)
    torch.cuda.synchronize()
    g, u = _ref(a, wg), _ref(a, wu)
    ref = g / (1 + torch.exp(-g)) * u
    _close(out, ref, K, True)
    rt.device_check()


@pytest.mark.parametrize("swiglu", [False, True])
@pytest.mark.parametrize("splits,variant,bn", [(4, 0, 128), (4, 2, 128), (-1, 0, 128), (-1, 1, 128),
                                               (-1, 2, 128), (3, 0, 192), (-1, 2, 192)])
def test_accum_split(cuda_dev, swiglu, splits, variant, bn):
    M, K, F = 77, 768, 384
    a = _mk((M, K), 10, cuda_dev)
    b = _mk((F, K), 11, cuda_dev)
    b2 = _mk((F, K), 12, cuda_dev) if swiglu else None
    N = 2 * F if swiglu else F
    ws = torch.zeros((M, N), device=cuda_dev)
    rt.gemm_bf16(A.GEMM_ACCUM, a, b, ws, b2=b2, bn=bn, splits=splits, variant=variant)
    torch.cuda.synchronize()
    ref = torch.cat([_ref(a, b), _ref(a, b2)], dim=1) if swiglu else _ref(a, b)
    _close(ws, ref, K, False)
    rt.device_check()


def test_large_k_full_shape_tile(cuda_dev):
    """LLaDA-8B FFN-down shape slice: K = 12288, several M tiles."""
    M, K, N = 260, 12288, 512
    a, b = _mk((M, K), 13, cuda_dev) * 0.05, _mk((N, K), 14, cuda_dev) * 0.05
    h = torch.zeros((M, N), device=cuda_dev)
    rt.gemm_bf16(A.GEMM_RESID, a, b, h, bn=256, splits=1)
    torch.cuda.synchronize()
    _close(h, _ref(a, b), K, False)
    h.zero_()
    rt.gemm_bf16(A.GEMM_RESID, a, b, h, bn=256, splits=1, variant=2)
    torch.cuda.synchronize()
    _close(h, _ref(a, b), K, False)
    rt.device_check()


@pytest.mark.parametrize("variant", [0, 2])
def test_stream_k_many_tiles(cuda_dev, variant):
    """Stream-K where worker shares cross several tile boundaries (more tiles
    than SMs) and where a share is a few K-blocks of one tile."""
    for M, K, N in ((700, 256, 2048), (200, 4096, 768)):
        a, b = _mk((M, K), 15, cuda_dev) * 0.1, _mk((N, K), 16, cuda_dev) * 0.1
        h = torch.zeros((M, N), device=cuda_dev)
        rt.gemm_bf16(A.GEMM_RESID, a, b, h, bn=128, splits=-1, variant=variant)
        torch.cuda.synchronize()
        _close(h, _ref(a, b), K, False)
    rt.device_check()


def test_stream_k_rejected_for_store(cuda_dev):
    a, b = _mk((8, 64), 1, cuda_dev), _mk((128, 64), 2, cuda_dev)
    out = torch.zeros((8, 128), device=cuda_dev, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        rt.gemm_bf16(A.GEMM_STORE, a, b, out, bn=128, splits=-1)


@pytest.mark.parametrize("variant,splits", [(0, 1), (2, -1)])
def test_resid_strided_output(cuda_dev, variant, splits):
    """fp32 output rows with a pitch wider than N (columns past N untouched)."""
    M, K, N, ldo = 150, 512, 256, 288
    a, b = _mk((M, K), 17, cuda_dev), _mk((N, K), 18, cuda_dev)
    buf = torch.full((M, ldo), 3.0, device=cuda_dev)
    rt.gemm_bf16(A.GEMM_RESID, a, b, buf, ldo=ldo, bn=128, splits=splits, variant=variant)
    torch.cuda.synchronize()
    _close(buf[:, :N] - 3.0, _ref(a, b), K, False)
    assert torch.all(buf[:, N:] == 3.0)
    rt.device_check()


# Swapped operands (variant 3): the weight tile is the MMA's 128-row operand
# and the M rows its N dimension (rounded up to 32), for M <= 256.
@pytest.mark.parametrize("splits", [1, 2, 5])
@pytest.mark.parametrize("M", [1, 5, 31, 33, 128, 130, 200, 255, 256])
def test_swap_resid(cuda_dev, splits, M):
    K, N = 1024, 768
    a, b = _mk((M, K), 21, cuda_dev), _mk((N, K), 22, cuda_dev)
    h0 = torch.randn((M, N), generator=torch.Generator().manual_seed(23)).to(cuda_dev)
    h = h0.clone()
    rt.gemm_bf16(A.GEMM_RESID, a, b, h, bn=128, splits=splits, variant=3)
    torch.cuda.synchronize()
    _close(h - h0, _ref(a, b), K, False)
    rt.device_check()


@pytest.mark.parametrize("swiglu", [False, True])
@pytest.mark.parametrize("splits", [1, 3])
@pytest.mark.parametrize("M", [7, 129, 256])
def test_swap_accum(cuda_dev, swiglu, splits, M):
    """ACCUM into a zeroed fp32 buffer; gate/up halves into columns [0, F) and
    [F, 2F), as the gate/up finishing pass reads them."""
    K, F = 2048, 384
    a = _mk((M, K), 24, cuda_dev)
    if swiglu:
        wg, wu = _mk((F, K), 25, cuda_dev), _mk((F, K), 26, cuda_dev)
        out = torch.zeros((M, 2 * F), device=cuda_dev, dtype=torch.float32)
        rt.gemm_bf16(A.GEMM_ACCUM, a, wg, out, b2=wu, bn=128, splits=splits, variant=3)
        torch.cuda.synchronize()
        _close(out[:, :F], _ref(a, wg), K, False)
        _close(out[:, F:], _ref(a, wu), K, False)
    else:
        b = _mk((3 * F, K), 27, cuda_dev)
        out = torch.zeros((M, 3 * F), device=cuda_dev, dtype=torch.float32)
        rt.gemm_bf16(A.GEMM_ACCUM, a, b, out, bn=128, splits=splits, variant=3)
        torch.cuda.synchronize()
        _close(out, _ref(a, b), K, False)
    rt.device_check()


def test_swap_rejects_what_it_cannot_do(cuda_dev):
    a, b = _mk((300, 256), 28, cuda_dev), _mk((256, 256), 29, cuda_dev)
    h = torch.zeros((300, 256), device=cuda_dev)
    with pytest.raises(Exception):            # more than 256 rows
        rt.gemm_bf16(A.GEMM_RESID, a, b, h, bn=128, splits=1, variant=3)
    out = torch.zeros((200, 256), device=cuda_dev, dtype=torch.bfloat16)
    with pytest.raises(Exception):            # a bf16 store epilogue
        rt.gemm_bf16(A.GEMM_STORE, a[:200], b, out, bn=128, splits=1, variant=3)
    with pytest.raises(Exception):            # another tile width
        rt.gemm_bf16(A.GEMM_RESID, a[:200], b, h[:200], bn=256, splits=1, variant=3)
