"""GPU parity: one decoder layer (forward, and backward with recomputation)
against the fp64 oracle.  Tolerance: normwise 2e-2 on activations and gradients.
The layer's input and output are the fp32 residual stream; the seeded input has
bf16 values (exact in fp32)."""
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


def _oracle_weight(W, absmax_bits, weight_bits=4):
    """The weight the layer sees: NF4 with fp32 absmax, or with the 8-bit absmax, or
    the weight rounded to bf16 (an unquantised stack)."""
    if weight_bits == 16:
        return synth.bf16_bits_to_f32(synth.to_bf16_bits(W))
    N, K = W.shape
    codes, am = onf4.quantize(W)
    if absmax_bits == 8:
        return onf4.dequantize_dq(codes, *onf4.quantize_absmax8(am), N, K)
    return onf4.dequantize(codes, am, N, K)


def _oracle_params(lw, cfg):
    W = {p: _oracle_weight(lw["W"][p], cfg.get("absmax_bits", 32), cfg.get("weight_bits", 4))
         for p in synth.PROJ}
    return dict(W=W, A=lw["A"], B=lw["B"], g1=synth.bf16_bits_to_f32(lw["g1"]),
                g2=synth.bf16_bits_to_f32(lw["g2"]))


def _device_layer(L, cfg, lw):
    import torch
    from gpu_util import dev, dev_bf16
    from layer_streamed_qlora_nf4_b200 import pack
    lay = L.lsq_layer_layout_get(cfg)
    blob = torch.zeros(lay.bytes, dtype=torch.uint8, device="cuda")
    pack.pack_layer(cfg, {p: dev(lw["W"][p]) for p in synth.PROJ}, dev_bf16(lw["g1"]),
                    dev_bf16(lw["g2"]), blob)
    lora = pack.lora_block(cfg, lw["A"], lw["B"])
    return blob, lora


def _run_layer(L, cfg, batch, seq, seed, check_bwd=True):
    import torch
    from gpu_util import dev, dev_bf16, host_bf16_to_f32, normwise_err, workspace
    from layer_streamed_qlora_nf4_b200 import pack
    T = batch * seq
    lw = synth.layer_weights(seed, cfg)
    x_bits = synth.activations(seed + 1, T, cfg["hidden"])
    dout = synth.normal_f32(synth.rng(seed + 2), (T, cfg["hidden"]), 1.0)
    blob, lora = _device_layer(L, cfg, lw)
    ws = workspace(L.decoder_layer_workspace_bytes(cfg, batch, seq))
    x = synth.bf16_bits_to_f32(x_bits)
    xd = dev(x)
    y = torch.empty(T, cfg["hidden"], dtype=torch.float32, device="cuda")
    L.decoder_layer_fwd(cfg, blob, lora, xd, batch, seq, y, ws)
    torch.cuda.synchronize()
    p = _oracle_params(lw, cfg)
    ref, _ = om.decoder_layer_fwd(p, x, cfg, seq)
    e = normwise_err(y.cpu().numpy(), ref)
    assert e <= TOL, ("fwd", e)
    if not check_bwd:
        return
    dx = torch.empty(T, cfg["hidden"], dtype=torch.float32, device="cuda")
    grad = torch.full_like(lora, float("nan"))
    L.decoder_layer_bwd(cfg, blob, lora, xd, dev(dout), batch, seq, dx, grad, ws)
    torch.cuda.synchronize()
    rdx, rg = om.decoder_layer_bwd(p, x, dout, cfg, seq)
    e = normwise_err(dx.cpu().numpy(), rdx)
    assert e <= TOL, ("dx", e)
    gv = pack.lora_views(cfg, grad)
    for name in synth.PROJ:
        eA = normwise_err(gv[name][0].cpu().numpy(), rg[name][0])
        eB = normwise_err(gv[name][1].cpu().numpy(), rg[name][1])
        assert eA <= TOL and eB <= TOL, (name, eA, eB)
    assert L.lsq_device_status() == 0


def test_layer_small_ragged_seq(L):
    # several GEMM tiles, attention blocks with a ragged tail, two sequences
    _run_layer(L, synth.SMALL, batch=2, seq=100, seed=11)


def test_layer_head_dim_128(L):
    cfg = dict(synth.SMALL, hidden=512, ffn=1024, n_heads=4, n_kv_heads=2, head_dim=128)
    _run_layer(L, cfg, batch=1, seq=192, seed=12)


def test_layer_rank_32_single_token_tail(L):
    cfg = dict(synth.SMALL, lora_r=32, lora_alpha=64.0)
    _run_layer(L, cfg, batch=3, seq=65, seed=13)


def test_layer_llama8b_shapes(L):
    # one Llama-3.1-8B-shaped layer, batch 1, seq 512 (the single-layer workload)
    _run_layer(L, synth.LLAMA8B, batch=1, seq=512, seed=1)


def test_layer_bwd_accumulates(L):
    import torch
    from gpu_util import dev, dev_bf16, workspace
    cfg = synth.SMALL
    batch, seq = 1, 64
    lw = synth.layer_weights(21, cfg)
    blob, lora = _device_layer(L, cfg, lw)
    ws = workspace(L.decoder_layer_workspace_bytes(cfg, batch, seq))
    x = dev(synth.bf16_bits_to_f32(synth.activations(22, seq, cfg["hidden"])))
    dout = dev(synth.normal_f32(synth.rng(23), (seq, cfg["hidden"]), 1.0))
    dx = torch.empty(seq, cfg["hidden"], device="cuda")
    g1 = torch.zeros_like(lora)
    L.decoder_layer_bwd(cfg, blob, lora, x, dout, batch, seq, dx, g1, ws)
    g2 = g1.clone()
    L.decoder_layer_bwd(cfg, blob, lora, x, dout, batch, seq, dx, g2, ws, accumulate=True)
    torch.cuda.synchronize()
    # deterministic kernels: g + g computed in fp32 equals 2 g exactly
    assert torch.equal(g2, g1 + g1)


def test_layer_rejects_bad_config(L):
    cfg = dict(synth.SMALL, hidden=500)
    with pytest.raises(L.LsqError) as e:
        L.lsq_layer_layout_get(cfg)
    assert e.value.code == L.LSQ_ERR_SHAPE


def test_layer_small_absmax8(L):
    # the 8-bit double-quantised absmax, dequantised inside the GEMM operand stage
    _run_layer(L, dict(synth.SMALL, absmax_bits=8), batch=2, seq=100, seed=17)


def test_layer_small_bf16_weights_rank64(L):
    # an unquantised (bf16) stack's layer, LoRA rank 64 (the Qwen2.5-3B configuration)
    cfg = dict(synth.SMALL, weight_bits=16, lora_r=64, lora_alpha=128.0)
    _run_layer(L, cfg, batch=2, seq=100, seed=19)
