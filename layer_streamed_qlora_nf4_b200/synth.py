"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and stores them in the workload's storage
types (bf16 bit patterns for activations, fp32 for weights and LoRA masters).  It
holds none of the method's arithmetic, imports neither the CUDA library nor the
oracle, and both sides receive exactly the arrays made here.

Distributions (the pages run on a real checkpoint and a text dataset; these
stand in for them, at the shapes of the pages' Llama-3.1-8B run):
  * frozen weights W ~ N(0, 0.02^2), fp32, quantised to NF4 by the caller;
  * LoRA A ~ N(0, (1/r)^2), B ~ N(0, 0.01^2), fp32 masters (B != 0 so dA != 0);
  * RMSNorm gains = 1 (bf16);
  * activations x and upstream gradients dY ~ N(0, 1), rounded to bf16;
  * embedding and lm_head ~ N(0, 0.02^2), bf16, untied;
  * token ids uniform in [0, vocab).
"""

import numpy as np

# ----------------------------------------------------------------------- configs
LLAMA8B = dict(hidden=4096, ffn=14336, n_heads=32, n_kv_heads=8, head_dim=128,
               n_layers=32, vocab=128256, rope_theta=500000.0, rms_eps=1e-5,
               lora_r=16, lora_alpha=32.0, block=64)

# Qwen2.5-3B shapes, streamed unquantised (bf16 weights), tied embedding, LoRA
# r 64 on all seven projections.  RoPE base and RMSNorm epsilon are the Qwen2.5
# family's published values; QKV biases are left out (the layer has none).
QWEN3B = dict(hidden=2048, ffn=11008, n_heads=16, n_kv_heads=2, head_dim=128,
              n_layers=36, vocab=151936, rope_theta=1000000.0, rms_eps=1e-6,
              lora_r=64, lora_alpha=128.0, block=64, weight_bits=16)

# Small Llama-shaped configs for oracle-sized parity cases (same structure,
# several GEMM tiles plus ragged tails).
SMALL = dict(hidden=512, ffn=1408, n_heads=8, n_kv_heads=2, head_dim=64,
             n_layers=3, vocab=1000, rope_theta=500000.0, rms_eps=1e-5,
             lora_r=16, lora_alpha=32.0, block=64)
TINY = dict(hidden=64, ffn=128, n_heads=4, n_kv_heads=2, head_dim=16,
            n_layers=2, vocab=97, rope_theta=500000.0, rms_eps=1e-5,
            lora_r=2, lora_alpha=4.0, block=64)

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def proj_shapes(cfg):
    """(N, K) of each frozen projection weight, in q,k,v,o,gate,up,down order."""
    D, F = cfg["hidden"], cfg["ffn"]
    qd = cfg["n_heads"] * cfg["head_dim"]
    kvd = cfg["n_kv_heads"] * cfg["head_dim"]
    return dict(q=(qd, D), k=(kvd, D), v=(kvd, D), o=(D, qd),
                gate=(F, D), up=(F, D), down=(D, F))


# ----------------------------------------------------------------- bf16 storage
def to_bf16_bits(a):
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (storage only)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b):
    """bf16 bit patterns (uint16) -> the fp32 values they encode (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def to_f16(a):
    """fp32 -> fp16 (numpy float16, round to nearest even): the storage of forward
    activations handed to the library (storage only)."""
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16)


# ------------------------------------------------------------------- generators
def rng(seed):
    return np.random.default_rng(seed)


def normal_f32(g, shape, std):
    return (g.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def normal_bf16(g, shape, std=1.0):
    """N(0, std^2) rounded to bf16; returns the uint16 bit patterns."""
    return to_bf16_bits(normal_f32(g, shape, std))


def linear_case(seed, N, K, T, r, w_std=0.02):
    """One NF4 + LoRA linear: W fp32 [N,K], x/dY bf16 bits, A [r,K], B [N,r] fp32."""
    g = rng(seed)
    return dict(W=normal_f32(g, (N, K), w_std),
                x=normal_bf16(g, (T, K)),
                A=normal_f32(g, (r, K), 1.0 / r),
                B=normal_f32(g, (N, r), 0.01),
                dy=normal_bf16(g, (T, N)))


def layer_weights(seed, cfg):
    """Frozen fp32 weights (to be NF4-quantised), gains and LoRA masters of one layer."""
    g = rng(seed)
    r = cfg["lora_r"]
    shapes = proj_shapes(cfg)
    W = {p: normal_f32(g, shapes[p], 0.02) for p in PROJ}
    A = {p: normal_f32(g, (r, shapes[p][1]), 1.0 / r) for p in PROJ}
    B = {p: normal_f32(g, (shapes[p][0], r), 0.01) for p in PROJ}
    ones = to_bf16_bits(np.ones(cfg["hidden"], np.float32))
    return dict(W=W, A=A, B=B, g1=ones.copy(), g2=ones.copy())


def activations(seed, T, D):
    return normal_bf16(rng(seed), (T, D))


def tokens(seed, batch, seq, vocab):
    return rng(seed).integers(0, vocab, size=(batch, seq), dtype=np.int32)


def embeddings(seed, vocab, D):
    """Untied embedding and lm_head, bf16 bits, each ~ N(0, 0.02^2)."""
    g = rng(seed)
    return normal_bf16(g, (vocab, D), 0.02), normal_bf16(g, (vocab, D), 0.02)
