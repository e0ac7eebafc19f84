"""GPU parity: the fused NF4 + LoRA linear (forward and backward) against the oracle.

Tolerance (stated by the workload): normwise max|gpu - ref| / max|ref| <= 2e-2
for activations and gradients against the fp64 oracle.  The workload's bf16
activations are handed to the library in fp16 (its forward operand type); both
the library and the oracle see the same fp16 values.
"""
import numpy as np
import pytest

from oracle import model as om
from oracle import nf4 as onf4
from layer_streamed_qlora_nf4_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def L():
    from layer_streamed_qlora_nf4_b200 import lib
    lib.load()
    return lib


def _run(L, N, K, T, r=16, alpha=32.0, seed=0, residual=False, accumulate=False, check_bwd=True):
    import torch
    from gpu_util import dev, dev_bf16, dev_f16, host_bf16_to_f32, normwise_err, workspace
    case = synth.linear_case(seed, N, K, T, r)
    s = alpha / r
    codes, absmax = onf4.quantize(case["W"])
    Wt = onf4.dequantize(codes, absmax, N, K)
    x16 = synth.to_f16(synth.bf16_bits_to_f32(case["x"]))
    x = x16.astype(np.float64)
    dy = synth.bf16_bits_to_f32(case["dy"])
    res = synth.bf16_bits_to_f32(synth.normal_bf16(synth.rng(seed + 1), (T, N))) if residual else None
    ref_y = om.lora_linear_fwd(x, Wt, case["A"], case["B"], s)
    if residual:
        ref_y = ref_y + res
    ws = workspace(L.nf4_lora_linear_workspace_bytes(T, K, N, r))
    xd, Ad, Bd = dev_f16(x16), dev(case["A"]), dev(case["B"])
    cd, ad = dev(codes), dev(absmax)
    # fp32 output with a residual (the residual stream), fp16 otherwise
    y = torch.empty(T, N, dtype=torch.float32 if residual else torch.float16, device="cuda")
    u = torch.empty(T, r, dtype=torch.float32, device="cuda")
    L.nf4_lora_linear_fwd(xd, cd, ad, Ad, Bd, s, y, residual=dev(res) if residual else None,
                          u_out=u, ws=ws)
    torch.cuda.synchronize()
    e_y = normwise_err(y.float().cpu().numpy(), ref_y)
    e_u = normwise_err(u.cpu().numpy(), x @ case["A"].astype(np.float64).T)
    assert e_y <= TOL, e_y
    # u = x A^T on tensor cores: x is exact in fp16, A is rounded once to fp16
    # (an independent error of at most 2^-11 relative per element), accumulation
    # in fp32; so du/u is about 3e-4 and the check allows 2^-8
    assert e_u <= 2.0 ** -8, e_u
    if not check_bwd:
        return
    ref_dx, ref_dA, ref_dB = om.lora_linear_bwd(dy, x, Wt, case["A"], case["B"], s)
    dx = torch.empty(T, K, dtype=torch.bfloat16, device="cuda")
    dA = torch.full((r, K), 0.5 if accumulate else np.nan, dtype=torch.float32, device="cuda")
    dB = torch.full((N, r), 0.25 if accumulate else np.nan, dtype=torch.float32, device="cuda")
    L.nf4_lora_linear_bwd(dev_bf16(case["dy"]), xd, cd, ad, Ad, Bd, s, dx, dA, dB,
                          accumulate=accumulate, ws=ws)
    torch.cuda.synchronize()
    if accumulate:
        ref_dA = ref_dA + 0.5
        ref_dB = ref_dB + 0.25
    e_dx = normwise_err(host_bf16_to_f32(dx), ref_dx)
    e_dA = normwise_err(dA.cpu().numpy(), ref_dA)
    e_dB = normwise_err(dB.cpu().numpy(), ref_dB)
    assert e_dx <= TOL, e_dx
    assert e_dA <= TOL, e_dA
    assert e_dB <= TOL, e_dB
    assert L.lsq_device_status() == 0


def test_linear_single_config(L):
    # the single NF4+LoRA linear workload: W 1024x1024, x [128, 1024], r 16, alpha 32
    _run(L, N=1024, K=1024, T=128)


@pytest.mark.parametrize("T", [1, 37, 200, 300, 512, 777])
def test_linear_ragged_tokens(L, T):
    _run(L, N=384, K=512, T=T, seed=T)


def test_linear_ragged_features_and_residual(L):
    _run(L, N=1000, K=320, T=96, residual=True, seed=3)


def test_linear_accumulate(L):
    _run(L, N=256, K=256, T=64, accumulate=True, seed=4)


def test_linear_rank_32(L):
    _run(L, N=512, K=1024, T=130, r=32, alpha=64.0, seed=5)


@pytest.mark.parametrize("N,K,T,r", [
    (96, 128, 200, 96),     # every rank-r product unsplit (written directly), 128-column tile
    (384, 512, 130, 192),   # one 192-column tile; u and v split, dA and dB direct
    (256, 256, 64, 256),    # two column tiles (192 + 64)
])
def test_linear_wide_ranks(L, N, K, T, r):
    _run(L, N=N, K=K, T=T, r=r, alpha=2.0 * r, seed=N + r)


@pytest.mark.parametrize("N,K", [(4096, 4096), (1024, 4096), (4096, 14336)])
def test_linear_8b_shapes(L, N, K):
    _run(L, N=N, K=K, T=512, seed=N + K)


def test_linear_bad_arguments(L):
    import torch
    from gpu_util import workspace
    x = torch.zeros(16, 100, dtype=torch.float16, device="cuda")   # K % 64 != 0
    y = torch.zeros(16, 64, dtype=torch.float16, device="cuda")
    A = torch.zeros(16, 100, device="cuda")
    B = torch.zeros(64, 16, device="cuda")
    codes = torch.zeros(64 * 100 // 2, dtype=torch.uint8, device="cuda")
    am = torch.zeros(100, device="cuda")
    with pytest.raises(L.LsqError) as e:
        L.nf4_lora_linear_fwd(x, codes, am, A, B, 2.0, y, ws=workspace(1 << 20))
    assert e.value.code == L.LSQ_ERR_SHAPE
    x = torch.zeros(16, 128, dtype=torch.float16, device="cuda")
    A = torch.zeros(16, 128, device="cuda")
    with pytest.raises(L.LsqError) as e:
        L.nf4_lora_linear_fwd(x, codes, am, A, B, 2.0, y, ws=workspace(16))
    assert e.value.code == L.LSQ_ERR_WORKSPACE
    # a residual is added in fp32 and needs an fp32 output
    with pytest.raises(L.LsqError) as e:
        L.nf4_lora_linear_fwd(x, codes, am, A, B, 2.0, y, residual=torch.zeros(16, 64, device="cuda"),
                              ws=workspace(1 << 20))
    assert e.value.code == L.LSQ_ERR_INVALID
