"""Host-side logic of bench.py (no GPU): which kernel class the roofline object describes."""
import importlib.util
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(HERE, "..", "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_roofline_subject_is_a_single_kernel():
    b = _bench()
    # the rank-r region (three kernels per timed region) has the most event time here,
    # but the roofline object must name one kernel: the NF4 forward GEMM
    prof = {"lora_rank_r_u": dict(total_ms=168.0, launches=4160),
            "gemm_nf4_fwd": dict(total_ms=137.5, launches=1120),
            "gemm_nf4_dx": dict(total_ms=76.0, launches=640)}
    assert b.dominant_kernel(prof)[0] == "gemm_nf4_fwd"
    prof["attention_fwd"] = dict(total_ms=140.0, launches=320)
    assert b.dominant_kernel(prof)[0] == "attention_fwd"
    # a profile holding only multi-kernel classes still yields a subject
    assert b.dominant_kernel({"lora_rank_r_dB": dict(total_ms=1.0, launches=1)})[0] == \
        "lora_rank_r_dB"


def test_kernel_table_sums_the_rank_r_kinds_once():
    b = _bench()
    prof = {"lora_rank_r_u": dict(total_ms=2.0, launches=4, flops=4e9, bytes=8e6),
            "lora_rank_r_dB": dict(total_ms=6.0, launches=12, flops=8e9, bytes=24e6),
            "gemm_nf4_fwd": dict(total_ms=10.0, launches=2, flops=1e12, bytes=1e8)}
    t = b.kernel_table(prof, steps=2)
    assert set(t) == {"lora_rank_r_u", "lora_rank_r_dB", "gemm_nf4_fwd", "lora_rank_r"}
    assert t["lora_rank_r"]["launches_per_step"] == 8 and t["lora_rank_r"]["ms_per_step"] == 4.0
    assert abs(t["lora_rank_r"]["tflops"] - 1.5) < 1e-12       # 12e9 FLOP / 8 ms
    assert abs(t["lora_rank_r"]["gbs"] - 4.0) < 1e-12          # 32e6 B / 8 ms
    assert len(prof) == 3                                      # the input is not modified
