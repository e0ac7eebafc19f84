"""GPU parity: NF4 codebook, quantize and dequantize are bit-exact with the oracle."""
import numpy as np
import pytest

from oracle import nf4 as onf4
from layer_streamed_qlora_nf4_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch  # noqa: F401
    from layer_streamed_qlora_nf4_b200 import lib
    lib.load()
    return lib


def _quant_gpu(L, W):
    import torch
    from gpu_util import dev
    N, K = W.shape
    Wd = dev(W)
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(N * K // 64, dtype=torch.float32, device="cuda")
    L.nf4_quantize(Wd, codes, absmax)
    return codes, absmax


def test_codebook_bit_exact(L):
    got = np.array(L.lsq_nf4_codebook(), np.float32)
    assert np.array_equal(got.view(np.uint32), onf4.codebook().view(np.uint32))


@pytest.mark.parametrize("N,K", [(1024, 1024), (77, 192), (4096, 4096), (1024, 14336)])
def test_quantize_bit_exact(L, N, K):
    g = synth.rng(100 + N)
    W = synth.normal_f32(g, (N, K), 0.02)
    W[0, :64] = 0.0                                  # a zero block
    W[1, 5] = W[1, :64].max() * 1.0                  # duplicate of the max
    codes, absmax = _quant_gpu(L, W)
    rc, ra = onf4.quantize(W)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), ra.view(np.uint32))


def test_quantize_midpoint_ties_and_levels(L):
    m = onf4.midpoints()
    c = onf4.codebook()
    row = np.zeros(64, np.float32)
    row[0] = 1.0
    row[1:16] = m
    row[16:31] = np.nextafter(m, np.float32(np.inf))
    row[31:47] = c
    W = np.stack([row, -row, row * np.float32(0.125)])
    codes, absmax = _quant_gpu(L, W)
    rc, ra = onf4.quantize(W)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_dequantize_bit_exact(L):
    import torch
    g = synth.rng(7)
    N, K = 256, 1024
    W = synth.normal_f32(g, (N, K), 0.02)
    codes, absmax = _quant_gpu(L, W)
    out = torch.empty(N, K, dtype=torch.float32, device="cuda")
    L.nf4_dequantize(codes, absmax, N, K, out)
    ref = onf4.dequantize(*onf4.quantize(W), N, K)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_quantize_rejects_nonfinite_and_bad_shapes(L):
    import torch
    W = np.zeros((2, 64), np.float32)
    W[1, 3] = np.inf
    with pytest.raises(L.LsqError) as e:
        _quant_gpu(L, W)
    assert e.value.code == L.LSQ_ERR_INVALID
    # finite but beyond the fp16 range of the fused GEMM's forward operand
    W[1, 3] = 65520.0
    with pytest.raises(L.LsqError) as e:
        _quant_gpu(L, W)
    assert e.value.code == L.LSQ_ERR_INVALID
    W[1, 3] = 65504.0           # the largest finite fp16 value is accepted
    _quant_gpu(L, W)
    Wd = torch.zeros(4, 96, device="cuda")
    codes = torch.empty(4 * 96 // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(6, dtype=torch.float32, device="cuda")
    with pytest.raises(L.LsqError) as e:
        L.nf4_quantize(Wd, codes, absmax)
    assert e.value.code == L.LSQ_ERR_SHAPE
    # a later valid call still works and the status word is clean
    codes, absmax = _quant_gpu(L, np.ones((2, 64), np.float32))
    assert L.lsq_device_status() == 0


def _absmax8_case(n, seed):
    a = np.abs(synth.normal_f32(synth.rng(seed), (n,), 0.05))
    a[:256] = 0.0                                       # a zero run
    a[256:512] = np.float32(2.0 ** -10) * np.arange(256, dtype=np.float32)   # exact grid
    a[300] = np.float32(2.5 * 2.0 ** -10)              # tie -> even
    return a


@pytest.mark.parametrize("n", [1024, 256 * 37 + 77, 4096 * 4096 // 64])
def test_absmax_quantize8_bit_exact(L, n):
    import torch
    from gpu_util import dev
    a = _absmax8_case(n, 200 + n % 97)
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.full(((n + 255) // 256,), float("nan"), dtype=torch.float32, device="cuda")
    L.nf4_absmax_quantize8(dev(a), q, s)
    rq, rs = onf4.quantize_absmax8(a)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("N,K", [(512, 1024), (1024, 14336)])
def test_dequantize_dq_bit_exact(L, N, K):
    import torch
    W = synth.normal_f32(synth.rng(300 + N), (N, K), 0.02)
    codes, absmax = _quant_gpu(L, W)
    nb = N * K // 64
    q = torch.empty(nb, dtype=torch.uint8, device="cuda")
    s = torch.empty((nb + 255) // 256, dtype=torch.float32, device="cuda")
    L.nf4_absmax_quantize8(absmax, q, s)
    out = torch.empty(N, K, dtype=torch.float32, device="cuda")
    L.nf4_dequantize_dq(codes, q, s, N, K, out)
    rc, ra = onf4.quantize(W)
    rq, rs = onf4.quantize_absmax8(ra)
    ref = onf4.dequantize_dq(rc, rq, rs, N, K)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
