"""Helpers shared by the GPU parity tests: host<->device marshalling and the
comparison metrics (no method arithmetic here)."""
import numpy as np
import torch

from layer_streamed_qlora_nf4_b200 import synth


def dev_bf16(bits):
    """uint16 bf16 bit patterns (numpy) -> torch.bfloat16 on cuda."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bf16_to_f32(t):
    """torch.bfloat16 (any device) -> numpy fp32 values."""
    return synth.bf16_bits_to_f32(t.detach().view(torch.int16).cpu().numpy().view(np.uint16))


def dev_f16(a16):
    """numpy float16 -> torch.float16 on cuda (the same values)."""
    return torch.from_numpy(np.ascontiguousarray(a16, dtype=np.float16)).cuda()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def normwise_err(got, ref):
    """max |got - ref| / max |ref| (the tolerance metric for fp results)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref)) / den) if den > 0 else float(np.max(np.abs(got)))


def frobenius_err(got, ref):
    """||got - ref||_F / ||ref||_F (relative error of the tensor as a whole)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


# Stack-level LoRA gradients: every tensor within 2e-2 by the max-element reading
# (max |err| / max |ref|) and in the Frobenius norm.
STACK_GRAD_TOL = 2e-2


def check_stack_grad(got, ref, name, where):
    f = frobenius_err(got, ref)
    m = normwise_err(got, ref)
    assert f <= STACK_GRAD_TOL and m <= STACK_GRAD_TOL, (where, name, f, m)


def elementwise_err(got, ref, floor=1e-3):
    """max |got - ref| / max(|ref|, floor * max|ref|)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.maximum(np.abs(ref), floor * np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref) / den))


def workspace(nbytes):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")
