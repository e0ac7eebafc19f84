"""Building the streamed store: layer blobs and LoRA blocks (marshalling only).

``pack_layer`` quantises a layer's seven frozen weights into one blob with the
library's ``nf4_quantize`` (the offline NF4 shard step of the Soup layer-streaming
tutorial, "四段資料路徑" part 1), writing at the offsets ``lsq_layer_layout_get``
returns (with an 8-bit absmax, ``nf4_absmax_quantize8`` then stores the absmax
in 8 bits; an unquantised bf16 stack stores each weight with ``lsq_bf16_from_f32``),
and copies the two RMSNorm gains.  ``lora_block`` places the fp32 LoRA
masters at the offsets of ``lsq_lora_layout_get``.  No arithmetic happens here.
"""
import torch

from . import lib

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def pack_layer(cfg, W, g1, g2, blob, stream=None):
    """W: dict proj -> fp32 cuda tensor [N, K]; g1, g2: bf16 cuda [D];
    blob: uint8 cuda tensor of layout.bytes (written in place)."""
    lay = lib.lsq_layer_layout_get(cfg)
    assert blob.dtype == torch.uint8 and blob.numel() >= lay.bytes and blob.is_cuda
    for p, name in enumerate(PROJ):
        N, K = lay.rows[p], lay.cols[p]
        w = W[name]
        assert tuple(w.shape) == (N, K) and w.dtype == torch.float32 and w.is_contiguous()
        if lay.weight_bits == 16:     # unquantised: the weight stored as bf16
            wb = blob[lay.codes_off[p]: lay.codes_off[p] + N * K * 2].view(torch.int16)
            lib.lsq_bf16_from_f32(w, wb, stream=stream)
            continue
        codes = blob[lay.codes_off[p]: lay.codes_off[p] + N * K // 2]
        nb = N * K // 64
        if lay.absmax_bits == 8:
            # codes from the fp32 absmax, then the absmax itself to 8 bits
            absmax = torch.empty(nb, dtype=torch.float32, device=blob.device)
            lib.nf4_quantize(w, codes, absmax, stream=stream)
            q = blob[lay.absmax_off[p]: lay.absmax_off[p] + nb]
            sc = blob[lay.scale_off[p]: lay.scale_off[p] + (nb + 255) // 256 * 4].view(torch.float32)
            lib.nf4_absmax_quantize8(absmax, q, sc, stream=stream)
        else:
            absmax = blob[lay.absmax_off[p]: lay.absmax_off[p] + nb * 4].view(torch.float32)
            lib.nf4_quantize(w, codes, absmax, stream=stream)
    D = cfg["hidden"]
    blob[lay.g1_off: lay.g1_off + 2 * D].copy_(g1.contiguous().view(torch.uint8))
    blob[lay.g2_off: lay.g2_off + 2 * D].copy_(g2.contiguous().view(torch.uint8))
    return lay


def lora_block(cfg, A, B, out=None, device="cuda"):
    """A, B: dict proj -> fp32 tensors ([r, K], [N, r]) -> one layer's LoRA block (fp32)."""
    lay = lib.lsq_lora_layout_get(cfg)
    if out is None:
        out = torch.zeros(lay.floats_per_layer, dtype=torch.float32, device=device)
    for p, name in enumerate(PROJ):
        a = torch.as_tensor(A[name], dtype=torch.float32).reshape(-1)
        b = torch.as_tensor(B[name], dtype=torch.float32).reshape(-1)
        out[lay.a_off[p]: lay.a_off[p] + a.numel()].copy_(a)
        out[lay.b_off[p]: lay.b_off[p] + b.numel()].copy_(b)
    return out


def lora_views(cfg, buf):
    """Inverse of lora_block: dict proj -> (A view [r, K], B view [N, r])."""
    lay = lib.lsq_lora_layout_get(cfg)
    ll = lib.lsq_layer_layout_get(cfg)
    r = cfg["lora_r"]
    out = {}
    for p, name in enumerate(PROJ):
        N, K = ll.rows[p], ll.cols[p]
        out[name] = (buf[lay.a_off[p]: lay.a_off[p] + r * K].view(r, K),
                     buf[lay.b_off[p]: lay.b_off[p] + N * r].view(N, r))
    return out
