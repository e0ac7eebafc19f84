"""The C-ABI library loads on a machine without a GPU, exports every function
include/lsq.h declares, and its host-only entry points behave: the library's
own NF4 codebook derivation equals the oracle's bit for bit, the layout queries
give the documented sizes, and invalid arguments are rejected before any CUDA
call."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import nf4 as onf4
from layer_streamed_qlora_nf4_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from layer_streamed_qlora_nf4_b200 import build, lib
    if not os.path.exists(lib.LIB_PATH):
        build.build()
    lib.load()
    return lib


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "lsq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\**\s+([a-z_][a-z_0-9]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 19
    lib = L.load()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.EXPORTS)


def test_library_codebook_equals_oracle_bitwise(L):
    got = np.array(L.lsq_nf4_codebook(), np.float32)
    assert np.array_equal(got.view(np.uint32), onf4.codebook().view(np.uint32))


def test_layer_layout_matches_the_documented_sizes(L):
    cfg = synth.LLAMA8B
    lay = L.lsq_layer_layout_get(cfg)
    P = 218103808                    # NF4 weights per 8B layer
    expect = P // 2 + 4 * P // 64 + 2 * 4096 * 2
    assert lay.bytes == expect == 122699776
    shapes = synth.proj_shapes(cfg)
    for p, name in enumerate(synth.PROJ):
        assert (lay.rows[p], lay.cols[p]) == shapes[name]
    # q|k|v and gate|up codes are contiguous (stacked GEMM operands)
    assert lay.codes_off[1] == lay.codes_off[0] + 4096 * 4096 // 2
    assert lay.codes_off[2] == lay.codes_off[1] + 1024 * 4096 // 2
    assert lay.codes_off[5] == lay.codes_off[4] + 14336 * 4096 // 2
    for o in list(lay.codes_off) + list(lay.absmax_off) + [lay.g1_off, lay.g2_off]:
        assert o % 256 == 0
    ll = L.lsq_lora_layout_get(cfg)
    r = 16
    n_lora = sum(r * (shapes[p][0] + shapes[p][1]) for p in synth.PROJ)
    assert ll.floats_per_layer >= n_lora and ll.floats_per_layer - n_lora < 64 * 8
    assert n_lora * 32 == 41943040   # 41.9 M LoRA parameters for the 32-layer stack


def test_layer_layout_with_8bit_absmax_gives_the_pages_store_size(L):
    # The pages: a 3.60 GB store for the 32 layers, 113 MB layer buffers (article
    # "架构解读：layer streaming 如何塞进 4 GB").  An fp32 absmax gives 122.7 MB and
    # 3.93 GB; an 8-bit absmax with one fp32 scale per 256 blocks gives the pages'.
    cfg = dict(synth.LLAMA8B, absmax_bits=8)
    lay = L.lsq_layer_layout_get(cfg)
    P = 218103808
    expect = P // 2 + P // 64 + 4 * (P // 64 // 256) + 2 * 4096 * 2
    assert lay.bytes == expect == 112529408 and lay.absmax_bits == 8
    assert round(lay.bytes / 1e6) == 113 and round(32 * lay.bytes / 1e9, 2) == 3.60
    assert round(32 * L.lsq_layer_layout_get(synth.LLAMA8B).bytes / 1e9, 2) == 3.93
    for p in range(7):
        nb = lay.rows[p] * lay.cols[p] // 64
        assert nb % 256 == 0           # a scale run never straddles two projections
        if p + 1 < 7:
            assert lay.absmax_off[p + 1] == lay.absmax_off[p] + nb          # uint8, stacked
            assert lay.scale_off[p + 1] == lay.scale_off[p] + nb // 256 * 4
    for o in list(lay.absmax_off) + list(lay.scale_off) + [lay.g1_off, lay.g2_off]:
        assert o % 256 == 0
    with pytest.raises(L.LsqError):
        L.lsq_layer_layout_get(dict(synth.LLAMA8B, absmax_bits=16))


def test_layer_layout_of_the_bf16_stack(L):
    # Qwen2.5-3B shapes streamed unquantised: 77,070,336 bf16 weights + two gains per layer
    lay = L.lsq_layer_layout_get(synth.QWEN3B)
    assert lay.weight_bits == 16
    assert lay.bytes == 2 * 77070336 + 2 * 2048 * 2 == 154148864
    shapes = synth.proj_shapes(synth.QWEN3B)
    for p, name in enumerate(synth.PROJ):
        assert (lay.rows[p], lay.cols[p]) == shapes[name] and lay.absmax_off[p] == 0
        if p + 1 < 7:
            assert lay.codes_off[p + 1] == lay.codes_off[p] + 2 * shapes[name][0] * shapes[name][1]
    with pytest.raises(L.LsqError):
        L.lsq_layer_layout_get(dict(synth.QWEN3B, weight_bits=8))


def test_workspace_queries_are_host_only(L):
    assert L.nf4_lora_linear_workspace_bytes(128, 1024, 1024, 16) > 0
    assert L.decoder_layer_workspace_bytes(synth.LLAMA8B, 1, 512) > 0
    assert L.stream_stack_workspace_bytes(synth.LLAMA8B, 1, 512) > 0
    assert L.nf4_lora_linear_workspace_bytes(0, 1024, 1024, 16) == 0
    assert L.stream_stack_dpo_workspace_bytes(synth.LLAMA8B, 2, 512) > \
        L.stream_stack_workspace_bytes(synth.LLAMA8B, 4, 512)
    assert L.stream_stack_dpo_workspace_bytes(synth.LLAMA8B, 0, 512) == 0
    assert L.stream_stack_dpo_workspace_bytes(synth.LLAMA8B, 33, 512) == 0


def test_stack_workspace_holds_one_lm_head_chunk(L):
    # The lm_head / loss run over chunks of whole sequences whose fp32 logits and bf16 logit
    # gradients fit 4 GiB: below that, every sequence adds its V * seq * 6 bytes of logits to
    # the step's workspace; above it, a sequence adds only its per-token tensors.
    cfg = dict(synth.SMALL, vocab=128000)
    seq = 64
    per_seq_logits = cfg["vocab"] * seq * 6
    per_chunk = (4 << 30) // per_seq_logits        # whole sequences per chunk
    w = lambda b: L.stream_stack_workspace_bytes(cfg, b, seq)
    below = w(per_chunk - 1) - w(per_chunk - 2)
    above = w(per_chunk + 11) - w(per_chunk + 10)
    assert below >= per_seq_logits
    assert above < per_seq_logits // 4
    assert w(4 * per_chunk) < w(per_chunk) + 3 * per_chunk * per_seq_logits // 4


def test_invalid_arguments_are_rejected_without_a_gpu(L):
    lib = L.load()
    p = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    assert lib.nf4_quantize(p, 4, 96, 64, p, p, None) == L.LSQ_ERR_SHAPE
    assert lib.nf4_quantize(p, 4, 128, 32, p, p, None) == L.LSQ_ERR_SHAPE
    assert lib.nf4_quantize(None, 4, 128, 64, p, p, None) == L.LSQ_ERR_INVALID
    assert lib.nf4_lora_linear_fwd(p, 8, 128, 64, p, p, 64, p, p, 8, 2.0, None, p, 0, None, p,
                                   1 << 20, None) == L.LSQ_ERR_SHAPE       # r % 16 != 0
    assert b"r must be" in lib.lsq_last_error()
    # an fp32 residual needs an fp32 output (y_fp32 = 1)
    assert lib.nf4_lora_linear_fwd(p, 8, 128, 64, p, p, 64, p, p, 16, 2.0, p, p, 0, None, p,
                                   1 << 20, None) == L.LSQ_ERR_INVALID
    assert b"residual" in lib.lsq_last_error()
    bad = dict(synth.SMALL, head_dim=96)
    with pytest.raises(L.LsqError) as e:
        L.lsq_layer_layout_get(bad)
    assert e.value.code == L.LSQ_ERR_SHAPE
    h = ctypes.c_void_p()
    c = L.cfg_struct(synth.SMALL)
    arr = (ctypes.c_void_p * 2)(16, 32)
    assert lib.stream_stack_create(ctypes.byref(c), arr, 2, p, p, 0, ctypes.byref(h)) == L.LSQ_ERR_SHAPE
    assert lib.stream_stack_destroy(None) == L.LSQ_OK


def test_shard_bytes(L):
    assert L.lsq_shard_bytes(122_699_776, 8) == 15_337_472          # 1/8 of an 8B layer
    assert L.lsq_shard_bytes(122_699_776, 1) == 122_699_776
    assert L.lsq_shard_bytes(1000, 3) == 512                        # ceil(1000/3) -> 256 B units
    assert L.lsq_shard_bytes(0, 4) == 0 and L.lsq_shard_bytes(100, 0) == 0
    for b in (1, 255, 257, 4096, 112_529_408):
        for w in (1, 2, 3, 7, 8):
            S = L.lsq_shard_bytes(b, w)
            assert S % 256 == 0 and S * w >= b and (S - 256) * w < b



def test_big_layer_config_is_above_165mib(L):
    # the configuration of the large-layer gradient test (hidden 5120, FFN 27648)
    from layer_streamed_qlora_nf4_b200 import synth
    big = dict(synth.LLAMA8B, hidden=5120, ffn=27648, n_heads=40, n_kv_heads=8, head_dim=128)
    lay = L.lsq_layer_layout_get(big)
    n_w = 5120 * (5120 + 2 * 1024) + 5120 * 5120 + 3 * 27648 * 5120
    assert lay.bytes == n_w // 2 + 4 * n_w // 64 + 2 * 5120 * 2     # codes + absmax + gains
    assert lay.bytes > 165 * 2 ** 20
