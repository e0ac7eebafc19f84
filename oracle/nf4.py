"""NF4 codebook, blockwise-absmax quantisation and dequantisation (CPU oracle).

Test infrastructure only (see the package docstring).

Source: the Soup layer-streaming tutorial, section "為什麼一般 QLoRA 在 4GB 還是可能
放不下 8B？" (the frozen base is stored as 4-bit NormalFloat, NF4, and LoRA is trained
on top) and section "Soup layer streaming 的四段資料路徑", part 1 "NF4" (the decoder's
quantisable Linear weights are quantised offline to NF4 shards; norms stay at
higher precision).  The pages name the data type but print none of its constants,
so every constant below is a stated reading:

  * Codebook: the QLoRA "4-bit NormalFloat" construction with an exact zero.
    Positive levels are standard-normal quantiles Phi^-1(p) at the 8 points
    p = delta + i*(1/2 - delta)/8, i = 0..7; negative levels are -Phi^-1(p) at the
    7 points p = delta + i*(1/2 - delta)/7, i = 0..6; 0 is added, the 16 values are
    sorted and divided by Phi^-1(delta), so the ends are exactly -1 and +1.
    delta = ((1 - 1/30) + (1 - 1/32)) / 2.  Phi^-1 is evaluated in fp64 and each
    level is rounded once to fp32.
  * Blocking: W [N, K] row-major is cut into runs of BLOCK = 64 consecutive
    elements (K % 64 == 0, so a block never straddles a row); absmax is the
    block's max |w|, stored as fp32 (no double quantisation).
  * Code choice: v = fl32(w / absmax) (one IEEE fp32 division, round to nearest
    even); code = number of fp32 midpoints m_i = fl32((c_i + c_{i+1}) / 2) that are
    strictly below v, so a value exactly on a midpoint takes the lower code.  A
    block whose absmax is 0 gets code 7 (the zero level) everywhere.
  * Packing: byte j holds element 2j in its high nibble and element 2j+1 in its
    low nibble.
  * Dequantisation: w~ = fl32(c[code] * absmax), a single fp32 multiply.

Optional second stage (double quantisation of the absmax).  The pages give only
sizes for it: a 3.60 GB store for 32 layers and 113 MB layer buffers (article
"架构解读：layer streaming 如何塞进 4 GB" and the "工作原理" list), which is what an
8-bit absmax with one fp32 scale per 256 blocks gives for Llama-3.1-8B shapes
(fp32 absmax would give 3.93 GB).  The scheme itself is not printed, so it is a
reading, the plainest linear one:

  * Groups: runs of ABSMAX_GROUP = 256 consecutive absmax values of one weight
    matrix (block order, row-major); the last run may be shorter.
  * Scale: s = fl32(max(run) / 255) (IEEE fp32 division); q = rint(fl32(a / s))
    rounded half to even, at most 255; a run whose max is 0 gets s = 0, q = 0.
  * The NF4 codes are still chosen with the fp32 absmax; dequantisation uses
    a~ = fl32(q * s) and then w~ = fl32(c[code] * a~).
"""

from statistics import NormalDist

import numpy as np

BLOCK = 64
ABSMAX_GROUP = 256
DELTA = ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0)) / 2.0


def codebook_f64():
    """The 16 NF4 levels in fp64, ascending (before rounding to fp32)."""
    inv = NormalDist().inv_cdf
    pos = [inv(DELTA + i * (0.5 - DELTA) / 8.0) for i in range(8)]
    neg = [-inv(DELTA + i * (0.5 - DELTA) / 7.0) for i in range(7)]
    top = inv(DELTA)
    levels = sorted(pos + neg + [0.0])
    return np.array([x / top for x in levels], dtype=np.float64)


def codebook():
    """The 16 NF4 levels as fp32 (each fp64 level rounded once)."""
    return codebook_f64().astype(np.float32)


def midpoints():
    """The 15 fp32 decision thresholds between neighbouring levels."""
    c = codebook()
    return ((c[:-1] + c[1:]) * np.float32(0.5)).astype(np.float32)


def quantize(W, block=BLOCK):
    """Quantise fp32 W [N, K] -> (codes uint8 [N*K/2], absmax fp32 [N*K/block]).

    The code of each element is its nearest level after dividing by its block's
    absmax (decided in fp32); two codes are packed per byte, high nibble first.
    """
    W = np.asarray(W, dtype=np.float32)
    assert W.ndim == 2, "W must be 2-D [N, K]"
    N, K = W.shape
    assert K % block == 0, "K must be a multiple of the block size"
    assert (N * K) % 2 == 0, "N*K must be even to pack two codes per byte"
    assert np.all(np.isfinite(W)), "NF4 quantisation takes finite weights only"
    blocks = W.reshape(-1, block)
    absmax = np.max(np.abs(blocks), axis=1).astype(np.float32)
    mids = midpoints()
    codes = np.full(blocks.shape, 7, dtype=np.uint8)
    nz = absmax > 0
    # code = number of midpoints strictly below v: searchsorted(side="left")
    # returns exactly that count.  Processed in chunks to bound memory.
    step = 1 << 20
    for b0 in range(0, blocks.shape[0], step):
        sl = slice(b0, b0 + step)
        z = nz[sl]
        v = (blocks[sl][z] / absmax[sl][z, None]).astype(np.float32)
        c = codes[sl]
        c[z] = np.searchsorted(mids, v, side="left").astype(np.uint8)
        codes[sl] = c
    flat = codes.reshape(-1)
    packed = ((flat[0::2] << 4) | flat[1::2]).astype(np.uint8)
    return packed, absmax


def unpack(codes, n_elems):
    """Packed bytes -> one code per element (high nibble = even element)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(n_elems, dtype=np.uint8)
    out[0::2] = codes >> 4
    out[1::2] = codes & 0x0F
    return out


def dequantize(codes, absmax, N, K, block=BLOCK):
    """(codes, absmax) -> fp32 W~ [N, K], with w~ = fl32(level[code] * absmax)."""
    c = codebook()
    idx = unpack(codes, N * K).reshape(-1, block)
    am = np.asarray(absmax, dtype=np.float32)[:, None]
    return (c[idx] * am).astype(np.float32).reshape(N, K)


def quantize_absmax8(absmax, group=ABSMAX_GROUP):
    """fp32 absmax [nb] -> (q uint8 [nb], scale fp32 [ceil(nb / group)])."""
    a = np.asarray(absmax, dtype=np.float32).reshape(-1)
    assert np.all(np.isfinite(a)) and np.all(a >= 0), "absmax values are finite and >= 0"
    ng = (a.size + group - 1) // group
    q = np.zeros(a.size, dtype=np.uint8)
    scale = np.zeros(ng, dtype=np.float32)
    for g in range(ng):
        run = a[g * group:(g + 1) * group]
        mx = np.float32(run.max())
        if mx == 0:
            continue
        s = np.float32(mx / np.float32(255.0))
        scale[g] = s
        v = (run / s).astype(np.float32)
        q[g * group:(g + 1) * group] = np.minimum(np.rint(v), 255).astype(np.uint8)
    return q, scale


def dequantize_absmax8(q, scale, group=ABSMAX_GROUP):
    """(q, scale) -> fp32 a~ [nb], a~ = fl32(q * scale[run])."""
    q = np.asarray(q, dtype=np.uint8).reshape(-1)
    s = np.asarray(scale, dtype=np.float32)[np.arange(q.size) // group]
    return (q.astype(np.float32) * s).astype(np.float32)


def dequantize_dq(codes, q, scale, N, K, block=BLOCK, group=ABSMAX_GROUP):
    """NF4 with a double-quantised absmax -> fp32 W~ [N, K]."""
    return dequantize(codes, dequantize_absmax8(q, scale, group), N, K, block)
