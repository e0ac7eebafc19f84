"""The launch planners of the two tensor-core kernels, checked on the CPU (host
only, no GPU): the fused NF4 GEMM and the LoRA rank-r product kernel.

Every plan must fit the kernel's shared-memory cap (with room for the GEMM
epilogue's staging slots, or for the rank-r kernel's cluster sum), cover every
row, column and reduction tile exactly once, and never launch an empty slice; the
TMEM allocation must hold the tile's accumulators.  The shapes span the decoder
projections of the 8B- and Qwen2.5-3B-shaped stacks, their input gradients, the
lm_head, the LoRA products, the split cases and ragged token counts.
"""
import itertools

import pytest


@pytest.fixture(scope="module")
def L():
    from layer_streamed_qlora_nf4_b200 import lib
    lib.load()
    return lib


MODES = (0, 1, 2, 3, 4)   # NF4 fwd, NF4 dX, bf16 fwd, bf16 dX, bf16 as fp16 fwd
MS = (128, 256, 2048, 2560, 4096, 6144, 11008, 22016, 28672, 128256)
TS = (1, 16, 100, 256, 257, 512, 513, 2048, 16384)
KS = (64, 2048, 4096, 11008, 14336, 28672)


def _check_plan(p, mode, M, T, Kc, sms):
    # shared memory: the stages, the code ring and the absmax ring after a 1 KB
    # alignment pad, within the kernel's cap, and room for the epilogue's slots
    used = 1024 + p["stages"] * (p["x_stage_bytes"] + p["w_stage_bytes"]) + \
        p["ring_stages"] * p["ring_bytes"] + p["absmax_ring_bytes"]
    assert used <= p["smem_bytes"] <= p["smem_limit"]
    assert p["smem_limit"] + 2048 <= 227 * 1024
    assert p["smem_bytes"] >= p["epilogue_bytes"] == 1024 + 12 * 4 * 4096
    assert 2 <= p["stages"] <= 4 and 1 <= p["ring_stages"] <= 8
    nf4 = mode in (0, 1)
    assert p["ring_bytes"] == (4096 if nf4 else 0)
    if nf4:
        assert p["ring_stages"] >= 2
    # token tiles: every token once, no empty tile; a pair halves each accumulator
    bt = p["nacc"] * p["bn"]
    assert p["nacc"] in (1, 2) and 0 < p["bn"] <= 256
    assert p["bn"] % (32 if p["pair"] else 16) == 0
    assert p["t_tiles"] * bt >= T and (p["t_tiles"] - 1) * bt < T
    assert p["x_stage_bytes"] == (bt // 2 if p["pair"] else bt) * 128
    # feature tiles: 128 per CTA, an even count in pairs
    assert p["m_tiles"] * 128 >= M and (p["m_tiles"] - (2 if p["pair"] else 1)) * 128 < M
    if p["pair"]:
        assert p["m_tiles"] % 2 == 0
    # contraction: 64-wide tiles, slices that cover them with none empty
    assert p["kt_total"] == (Kc + 63) // 64
    assert p["splits"] * p["kt_per_split"] >= p["kt_total"]
    assert (p["splits"] - 1) * p["kt_per_split"] < p["kt_total"]
    assert 1 <= p["splits"] <= 16
    if p["m_tiles"] * p["t_tiles"] >= sms:
        assert p["splits"] == 1               # a full wave already: no split
    assert p["partial_bytes"] == (p["splits"] * T * M * 4 if p["splits"] > 1 else 0)
    # TMEM: a power of two of at least 32 columns, holding every accumulator
    c = p["tmem_cols"]
    assert 32 <= c <= 512 and c & (c - 1) == 0 and c >= bt
    # the epilogue gives each warp at most 8 chunks: 3 warps share a lane quarter
    assert p["nacc"] * ((p["bn"] + 31) // 32) <= 3 * 8
    # launch grid limits
    assert p["t_tiles"] <= 65535 and p["splits"] <= 65535


def test_plans_fit_and_cover_the_problem(L):
    n = 0
    for mode, M, T, Kc in itertools.product(MODES, MS, TS, KS):
        for sms, pair in ((148, True), (148, False), (132, True)):
            p = L.lsq_gemm_plan_get(mode, M, T, Kc, sms, pair)
            assert p["pair"] == (1 if pair and (M + 127) // 128 >= 2 else 0)
            _check_plan(p, mode, M, T, Kc, sms)
            n += 1
    assert n == len(MODES) * len(MS) * len(TS) * len(KS) * 3


def test_full_tiles_take_operand_stages_before_ring_depth(L):
    # 512 tokens per pair tile: 4 stages of 48 KB and a 3-slot NF4 code ring, the
    # 226,304 bytes of dynamic shared memory the gate|up capture reports
    for mode in (0, 1):
        p = L.lsq_gemm_plan_get(mode, 28672, 512, 4096)
        assert (p["stages"], p["ring_stages"], p["smem_bytes"]) == (4, 3, 226304)
    # a bf16 weight needs no ring
    p = L.lsq_gemm_plan_get(2, 128256, 512, 4096)
    assert p["stages"] == 4 and p["ring_bytes"] == 0


def test_small_products_split_k_over_the_sms(L):
    # o projection of the 8B layer at T = 512: 32 CTAs of one token tile, split over K
    p = L.lsq_gemm_plan_get(0, 4096, 512, 4096)
    assert p["m_tiles"] * p["t_tiles"] == 32 and p["splits"] == 4
    assert p["partial_bytes"] == 4 * 512 * 4096 * 4
    # gate|up at T = 512: 224 CTAs, no split
    p = L.lsq_gemm_plan_get(0, 28672, 512, 4096)
    assert p["m_tiles"] * p["t_tiles"] == 224 and p["splits"] == 1


def test_bad_queries_are_rejected(L):
    with pytest.raises(L.LsqError):
        L.lsq_gemm_plan_get(5, 128, 16, 64)
    with pytest.raises(L.LsqError):
        L.lsq_gemm_plan_get(0, 0, 16, 64)
    with pytest.raises(L.LsqError):
        L.lsq_gemm_plan_get(0, 128, 16, 64, num_sms=0)


# ---------------------------------------------------------------- rank-r products
# The LoRA products: C [M, N] = A [M, K] . B [N, K]^T with N the (stacked) rank or,
# for dA / dB, M the rank side; M, N and K span the 8B and Qwen2.5-3B shapes.
LM = (16, 48, 128, 512, 2048, 4096, 16384, 28672)
LN = (8, 16, 48, 64, 96, 128, 192, 256, 384, 4096, 14336)
LK = (64, 128, 512, 2048, 4096, 16384, 28672)


def _check_lora_plan(p, M, N, K, sms):
    assert p["n_pad"] == min(256, (N + 15) // 16 * 16)
    assert p["col_tiles"] * p["n_pad"] >= N and (p["col_tiles"] - 1) * p["n_pad"] < N
    assert p["row_tiles"] * 128 >= M and (p["row_tiles"] - 1) * 128 < M
    assert p["kt_total"] == (K + 63) // 64
    # shared memory: a 1 KB alignment pad and the stages, within the kernel's cap
    assert p["stages"] == 4                       # the kernel keeps 4 stage barriers
    assert p["stage_bytes"] == 128 * 64 * 2 + (p["n_pad"] * 128 + 1023) // 1024 * 1024
    assert p["smem_bytes"] == 1024 + p["stages"] * p["stage_bytes"] <= p["smem_limit"]
    assert p["smem_limit"] <= 227 * 1024
    # two resident CTAs per SM only where both fit the SM's shared memory and TMEM
    assert p["ctas_per_sm"] in (1, 2)
    if p["ctas_per_sm"] == 2:
        assert 2 * p["smem_bytes"] <= 228 * 1024 and 2 * p["tmem_cols"] <= 512
    c = p["tmem_cols"]
    assert 32 <= c <= 512 and c & (c - 1) == 0 and c >= p["n_pad"]
    # split reduction: a portable cluster whose slices share the 128 rows evenly, each
    # at least two stages long, only where the tiles alone leave half the slots empty
    z = p["splits"]
    slots = sms * p["ctas_per_sm"]
    tiles = p["row_tiles"] * p["col_tiles"]
    assert z in (1, 2, 4, 8) and 128 % z == 0
    if z > 1:
        assert tiles * 2 <= slots and tiles * z <= slots
        assert p["kt_total"] // z >= 2
        # the cluster sum's fp32 [128][n_pad + 4] buffer fits the drained stages
        assert p["reduce_bytes"] == 128 * (p["n_pad"] + 4) * 4
        assert p["reduce_bytes"] <= p["stages"] * p["stage_bytes"]
    else:
        assert p["reduce_bytes"] == 0
    assert p["row_tiles"] <= 2 ** 31 - 1 and p["col_tiles"] <= 65535


def test_rank_r_plans_fit_and_cover_the_product(L):
    n = 0
    for M, N, K in itertools.product(LM, LN, LK):
        for sms in (148, 132):
            _check_lora_plan(L.lsq_lora_plan_get(M, N, K, sms), M, N, K, sms)
            n += 1
    assert n == len(LM) * len(LN) * len(LK) * 2


def test_rank_r_split_choices_at_the_8b_shapes(L):
    # u = x A^T of the 8B q|k|v group at T = 512 (N = 3 r = 48): 4 row tiles split 8 ways
    p = L.lsq_lora_plan_get(512, 48, 4096)
    assert (p["row_tiles"], p["splits"], p["ctas_per_sm"]) == (4, 8, 2)
    # a product that fills the GPU by its tiles is not split
    p = L.lsq_lora_plan_get(16384, 256, 4096)
    assert p["splits"] == 1 and p["reduce_bytes"] == 0


def test_bad_rank_r_queries_are_rejected(L):
    with pytest.raises(L.LsqError):
        L.lsq_lora_plan_get(0, 16, 64)
    with pytest.raises(L.LsqError):
        L.lsq_lora_plan_get(128, 16, 64, num_sms=0)
