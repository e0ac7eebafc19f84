"""Thin Python binding of the C ABI in include/lsq.h (argument marshalling only).

Every function here has the name of the C entry point it calls, takes torch
tensors (or plain ints/floats), passes their data pointers and the current CUDA
stream, and raises LsqError on a non-zero status.  No computation happens here:
every step of the path runs in the CUDA library.  Importing this module loads
liblsq.so and fails loudly if it has not been built.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblsq.so")

LSQ_OK, LSQ_ERR_INVALID, LSQ_ERR_SHAPE, LSQ_ERR_CUDA = 0, 1, 2, 3
LSQ_ERR_TIMEOUT, LSQ_ERR_WORKSPACE, LSQ_ERR_ALIGN, LSQ_ERR_DEVICE = 4, 5, 6, 7

# Every symbol include/lsq.h declares (checked by tests/test_abi.py).
EXPORTS = (
    "lsq_last_error", "lsq_version", "lsq_device_status", "lsq_nf4_codebook",
    "nf4_quantize", "nf4_dequantize", "nf4_lora_linear_workspace_bytes",
    "nf4_lora_linear_fwd", "nf4_lora_linear_bwd", "lsq_layer_layout_get",
    "lsq_lora_layout_get", "decoder_layer_workspace_bytes", "decoder_layer_fwd",
    "decoder_layer_bwd", "stream_stack_create", "stream_stack_destroy",
    "stream_stack_workspace_bytes", "stream_stack_step", "stream_stack_last_stats",
    "lora_adamw_step", "lsq_launch_counter", "lsq_profile_enable", "lsq_profile_read",
    "nf4_lora_linear_fwd_noalloc", "nf4_absmax_quantize8", "nf4_dequantize_dq",
    "stream_stack_dpo_workspace_bytes", "stream_stack_dpo_step", "lsq_bf16_from_f32",
    "lsq_shard_bytes", "lsq_nccl_unique_id", "stream_stack_shard", "lsq_stream_plan",
    "stream_stack_reduce_grads", "lsq_gemm_plan_get", "lsq_lora_plan_get",
)
LSQ_NCCL_ID_BYTES = 128


class LsqError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("lsq error %d: %s" % (code, msg))
        self.code = code


class lsq_cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int64), ("ffn", ctypes.c_int64), ("vocab", ctypes.c_int64),
                ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("lora_r", ctypes.c_int32), ("block", ctypes.c_int32),
                ("lora_alpha", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("absmax_bits", ctypes.c_int32),
                ("weight_bits", ctypes.c_int32)]


class lsq_layer_layout(ctypes.Structure):
    _fields_ = [("codes_off", ctypes.c_uint64 * 7), ("absmax_off", ctypes.c_uint64 * 7),
                ("g1_off", ctypes.c_uint64), ("g2_off", ctypes.c_uint64),
                ("rows", ctypes.c_int64 * 7), ("cols", ctypes.c_int64 * 7),
                ("bytes", ctypes.c_uint64), ("scale_off", ctypes.c_uint64 * 7),
                ("absmax_bits", ctypes.c_int32), ("weight_bits", ctypes.c_int32)]


class lsq_lora_layout(ctypes.Structure):
    _fields_ = [("a_off", ctypes.c_int64 * 7), ("b_off", ctypes.c_int64 * 7),
                ("floats_per_layer", ctypes.c_int64)]


class lsq_adamw(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("step", ctypes.c_int32), ("m", ctypes.c_void_p), ("v", ctypes.c_void_p)]


class lsq_prof_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


class lsq_step_stats(ctypes.Structure):
    _fields_ = [("layer_copies", ctypes.c_int32), ("h2d_bytes", ctypes.c_int64),
                ("step_ms", ctypes.c_float), ("copy_wait_ms", ctypes.c_float)]


class lsq_gemm_plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "pair", "bn", "nacc", "m_tiles", "t_tiles", "splits", "kt_total", "kt_per_split",
        "stages", "ring_stages", "x_stage_bytes", "w_stage_bytes", "ring_bytes",
        "absmax_ring_bytes", "smem_bytes", "smem_limit", "epilogue_bytes", "tmem_cols")] + [
        ("partial_bytes", ctypes.c_int64)]


class lsq_lora_plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_pad", "row_tiles", "col_tiles", "splits", "kt_total", "stages", "stage_bytes",
        "smem_bytes", "smem_limit", "ctas_per_sm", "tmem_cols", "reduce_bytes")]


# operand modes of lsq_gemm_plan_get
LSQ_GEMM_NF4_FWD, LSQ_GEMM_NF4_DX, LSQ_GEMM_BF16_FWD, LSQ_GEMM_BF16_DX = 0, 1, 2, 3
LSQ_GEMM_BF16_AS_F16_FWD = 4


_P = ctypes.c_void_p
_I32, _I64, _F, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_PROTOS = {
    "lsq_last_error": (ctypes.c_char_p, []),
    "lsq_version": (ctypes.c_int, []),
    "lsq_device_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int), ctypes.c_int]),
    "lsq_nf4_codebook": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float)]),
    "nf4_quantize": (ctypes.c_int, [_P, _I64, _I64, _I32, _P, _P, _P]),
    "nf4_dequantize": (ctypes.c_int, [_P, _P, _I64, _I64, _I32, _P, _P]),
    "nf4_absmax_quantize8": (ctypes.c_int, [_P, _I64, _P, _P, _P]),
    "lsq_bf16_from_f32": (ctypes.c_int, [_P, _I64, _P, _P]),
    "nf4_dequantize_dq": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I32, _P, _P]),
    "nf4_lora_linear_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I32]),
    "nf4_lora_linear_fwd": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I32, _P, _P, _I32, _F,
                                           _P, _P, _I32, _P, _P, _SZ, _P]),
    "nf4_lora_linear_bwd": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _I32, _P, _P, _I32,
                                           _F, _P, _P, _P, _I32, _P, _SZ, _P]),
    "lsq_layer_layout_get": (ctypes.c_int, [ctypes.POINTER(lsq_cfg),
                                            ctypes.POINTER(lsq_layer_layout)]),
    "lsq_lora_layout_get": (ctypes.c_int, [ctypes.POINTER(lsq_cfg),
                                           ctypes.POINTER(lsq_lora_layout)]),
    "decoder_layer_workspace_bytes": (_SZ, [ctypes.POINTER(lsq_cfg), _I32, _I32]),
    "decoder_layer_fwd": (ctypes.c_int, [ctypes.POINTER(lsq_cfg), _P, _P, _P, _I32, _I32, _P, _P,
                                         _SZ, _P]),
    "decoder_layer_bwd": (ctypes.c_int, [ctypes.POINTER(lsq_cfg), _P, _P, _P, _P, _I32, _I32, _P,
                                         _P, _I32, _P, _SZ, _P]),
    "stream_stack_create": (ctypes.c_int, [ctypes.POINTER(lsq_cfg), ctypes.POINTER(_P), _I32, _P,
                                           _P, _I32, ctypes.POINTER(_P)]),
    "stream_stack_destroy": (ctypes.c_int, [_P]),
    "stream_stack_workspace_bytes": (_SZ, [ctypes.POINTER(lsq_cfg), _I32, _I32]),
    "stream_stack_step": (ctypes.c_int, [_P, _P, _I32, _I32, _I32, _P, _P, _P, _P, _P,
                                         ctypes.POINTER(lsq_adamw), ctypes.POINTER(ctypes.c_float),
                                         _P, _P, _SZ, _P, _I64]),
    "stream_stack_last_stats": (ctypes.c_int, [_P, ctypes.POINTER(lsq_step_stats)]),
    "stream_stack_dpo_workspace_bytes": (_SZ, [ctypes.POINTER(lsq_cfg), _I32, _I32]),
    "stream_stack_dpo_step": (ctypes.c_int, [_P, _P, _I32, _I32, _F, _P, _P, _P, _P, _P,
                                             ctypes.POINTER(lsq_adamw),
                                             ctypes.POINTER(ctypes.c_float),
                                             ctypes.POINTER(ctypes.c_float), _P, _P, _SZ, _P,
                                             _I64]),
    "lora_adamw_step": (ctypes.c_int, [_P, _P, ctypes.POINTER(lsq_adamw), _I64, _P]),
    "lsq_shard_bytes": (_I64, [_I64, _I32]),
    "lsq_stream_plan": (ctypes.c_int, [_I32, _I32, _I32, _I32, _P, _P, _P, _I32,
                                       ctypes.POINTER(ctypes.c_int32)]),
    "lsq_nccl_unique_id": (ctypes.c_int, [_P, _I64]),
    "stream_stack_shard": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _I64]),
    "stream_stack_reduce_grads": (ctypes.c_int, [_P, _P, _I64, _I32, _I32]),
    "lsq_launch_counter": (ctypes.c_int64, []),
    "lsq_gemm_plan_get": (ctypes.c_int, [_I32, _I64, _I64, _I64, _I32, _I32,
                                         ctypes.POINTER(lsq_gemm_plan)]),
    "lsq_lora_plan_get": (ctypes.c_int, [_I64, _I64, _I64, _I32, ctypes.POINTER(lsq_lora_plan)]),
    "nf4_lora_linear_fwd_noalloc": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I32, _P, _P, _I32,
                                                   _F, _P, _P, _I32, _P, _P]),
    "lsq_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "lsq_profile_read": (ctypes.c_int, [ctypes.POINTER(lsq_prof_entry), _I32,
                                        ctypes.POINTER(ctypes.c_int32)]),
}

_lib = None


def load():
    """Loads liblsq.so (once) and declares the prototypes; raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("liblsq.so is not built (run: python -m "
                               "layer_streamed_qlora_nf4_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            if not hasattr(lib, name):
                continue   # tests/test_abi.py checks that every declared symbol exists
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _check(rc):
    if rc != LSQ_OK:
        raise LsqError(rc, load().lsq_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is not None:
        return ctypes.c_void_p(stream)
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def cfg_struct(cfg):
    """A synth-style config dict -> lsq_cfg."""
    return lsq_cfg(hidden=cfg["hidden"], ffn=cfg["ffn"], vocab=cfg["vocab"],
                   n_heads=cfg["n_heads"], n_kv_heads=cfg["n_kv_heads"],
                   head_dim=cfg["head_dim"], n_layers=cfg["n_layers"], lora_r=cfg["lora_r"],
                   block=cfg["block"], lora_alpha=cfg["lora_alpha"],
                   rope_theta=cfg["rope_theta"], rms_eps=cfg["rms_eps"],
                   absmax_bits=cfg.get("absmax_bits", 32),
                   weight_bits=cfg.get("weight_bits", 4))


# ------------------------------------------------------------------ entry points
def lsq_version():
    return load().lsq_version()


def lsq_device_status(clear=False):
    v = ctypes.c_int(0)
    _check(load().lsq_device_status(ctypes.byref(v), 1 if clear else 0))
    return v.value


def lsq_nf4_codebook():
    out = (ctypes.c_float * 16)()
    _check(load().lsq_nf4_codebook(out))
    return list(out)


def nf4_quantize(W, codes, absmax, block=64, stream=None):
    N, K = W.shape
    _check(load().nf4_quantize(_ptr(W), N, K, block, _ptr(codes), _ptr(absmax), _stream(stream)))


def nf4_dequantize(codes, absmax, N, K, W_out, block=64, stream=None):
    _check(load().nf4_dequantize(_ptr(codes), _ptr(absmax), N, K, block, _ptr(W_out),
                                 _stream(stream)))


def lsq_bf16_from_f32(x, y, stream=None):
    _check(load().lsq_bf16_from_f32(_ptr(x), x.numel(), _ptr(y), _stream(stream)))


def nf4_absmax_quantize8(absmax, q, scale, stream=None):
    _check(load().nf4_absmax_quantize8(_ptr(absmax), absmax.numel(), _ptr(q), _ptr(scale),
                                       _stream(stream)))


def nf4_dequantize_dq(codes, q, scale, N, K, W_out, block=64, stream=None):
    _check(load().nf4_dequantize_dq(_ptr(codes), _ptr(q), _ptr(scale), N, K, block, _ptr(W_out),
                                    _stream(stream)))


def nf4_lora_linear_workspace_bytes(T, K, N, r):
    return load().nf4_lora_linear_workspace_bytes(T, K, N, r)


def _y_fp32(y):
    """1 for an fp32 output tensor, 0 for an fp16 one (the y_fp32 argument)."""
    import torch
    if y.dtype not in (torch.float32, torch.float16):
        raise TypeError("y must be float16 or float32")
    return 1 if y.dtype == torch.float32 else 0


def nf4_lora_linear_fwd(x, codes, absmax, A, B, scale, y, residual=None, u_out=None, ws=None,
                        block=64, stream=None):
    """x: fp16 [T, K]; y: fp16 [T, N], or fp32 [T, N] (required with an fp32 residual)."""
    T, K = x.shape
    N = y.shape[1]
    r = A.shape[0]
    _check(load().nf4_lora_linear_fwd(_ptr(x), T, K, N, _ptr(codes), _ptr(absmax), block,
                                      _ptr(A), _ptr(B), r, scale, _ptr(residual), _ptr(y),
                                      _y_fp32(y), _ptr(u_out), _ptr(ws),
                                      0 if ws is None else ws.numel(), _stream(stream)))


def nf4_lora_linear_bwd(dy, x, codes, absmax, A, B, scale, dx, dA, dB, accumulate=False,
                        ws=None, block=64, stream=None):
    """dy: bf16 [T, N]; x: fp16 [T, K] (the forward input); dx: bf16 [T, K]."""
    T, K = x.shape
    N = dy.shape[1]
    r = A.shape[0]
    _check(load().nf4_lora_linear_bwd(_ptr(dy), _ptr(x), T, K, N, _ptr(codes), _ptr(absmax),
                                      block, _ptr(A), _ptr(B), r, scale, _ptr(dx), _ptr(dA),
                                      _ptr(dB), 1 if accumulate else 0, _ptr(ws),
                                      0 if ws is None else ws.numel(), _stream(stream)))


def lsq_layer_layout_get(cfg):
    out = lsq_layer_layout()
    c = cfg_struct(cfg)
    _check(load().lsq_layer_layout_get(ctypes.byref(c), ctypes.byref(out)))
    return out


def lsq_lora_layout_get(cfg):
    out = lsq_lora_layout()
    c = cfg_struct(cfg)
    _check(load().lsq_lora_layout_get(ctypes.byref(c), ctypes.byref(out)))
    return out


def decoder_layer_workspace_bytes(cfg, batch, seq):
    c = cfg_struct(cfg)
    return load().decoder_layer_workspace_bytes(ctypes.byref(c), batch, seq)


def decoder_layer_fwd(cfg, blob, lora, x_in, batch, seq, x_out, ws, stream=None):
    """x_in, x_out: fp32 [batch * seq, D] (the residual stream)."""
    c = cfg_struct(cfg)
    _check(load().decoder_layer_fwd(ctypes.byref(c), _ptr(blob), _ptr(lora), _ptr(x_in), batch,
                                    seq, _ptr(x_out), _ptr(ws), ws.numel(), _stream(stream)))


def decoder_layer_bwd(cfg, blob, lora, x_in, dx_out, batch, seq, dx_in, lora_grad, ws,
                      accumulate=False, stream=None):
    c = cfg_struct(cfg)
    _check(load().decoder_layer_bwd(ctypes.byref(c), _ptr(blob), _ptr(lora), _ptr(x_in),
                                    _ptr(dx_out), batch, seq, _ptr(dx_in), _ptr(lora_grad),
                                    1 if accumulate else 0, _ptr(ws), ws.numel(),
                                    _stream(stream)))


class StreamStack:
    """Owns an lsq_stack handle (stream_stack_create / stream_stack_destroy)."""

    def __init__(self, cfg, layer_blobs, buf0, buf1, resident):
        self.cfg = cfg_struct(cfg)
        self._blobs = list(layer_blobs)   # keep the tensors alive
        arr = (ctypes.c_void_p * len(self._blobs))(*[b.data_ptr() for b in self._blobs])
        self.handle = ctypes.c_void_p()
        _check(load().stream_stack_create(ctypes.byref(self.cfg), arr, len(self._blobs),
                                          _ptr(buf0), _ptr(buf1), 1 if resident else 0,
                                          ctypes.byref(self.handle)))

    def shard(self, nccl_id, world, rank, buf_bytes):
        """stream_stack_shard: spread every layer copy over `world` ranks."""
        stream_stack_shard(self, nccl_id, world, rank, buf_bytes)

    def reduce_grads(self, nccl_id, world, rank):
        """stream_stack_reduce_grads: average the LoRA gradients over `world` ranks in each step."""
        stream_stack_reduce_grads(self, nccl_id, world, rank)

    def close(self):
        if self.handle:
            _check(load().stream_stack_destroy(self.handle))
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lsq_stream_plan(n_layers, micro_batches, held0=-1, held1=-1):
    """-> list of (layer, buf, copy) per visit of one streamed step."""
    n = max(0, 2 * int(n_layers) * int(micro_batches))
    arrs = [(ctypes.c_int32 * max(n, 1))() for _ in range(3)]
    nv = ctypes.c_int32(0)
    _check(load().lsq_stream_plan(int(n_layers), int(micro_batches), int(held0), int(held1),
                                  arrs[0], arrs[1], arrs[2], n, ctypes.byref(nv)))
    return [(arrs[0][i], arrs[1][i], arrs[2][i]) for i in range(nv.value)]


def lsq_gemm_plan_get(mode, M, T, Kc, num_sms=148, allow_pair=True):
    """-> dict of the fused GEMM's launch plan for one product (host only)."""
    out = lsq_gemm_plan()
    _check(load().lsq_gemm_plan_get(int(mode), int(M), int(T), int(Kc), int(num_sms),
                                    1 if allow_pair else 0, ctypes.byref(out)))
    return {n: getattr(out, n) for n, _ in lsq_gemm_plan._fields_}


def lsq_lora_plan_get(M, N, K, num_sms=148):
    """-> dict of the rank-r product kernel's launch plan (host only)."""
    out = lsq_lora_plan()
    _check(load().lsq_lora_plan_get(int(M), int(N), int(K), int(num_sms), ctypes.byref(out)))
    return {n: getattr(out, n) for n, _ in lsq_lora_plan._fields_}


def lsq_shard_bytes(layer_bytes, world):
    return int(load().lsq_shard_bytes(int(layer_bytes), int(world)))


def lsq_nccl_unique_id():
    """-> bytes (LSQ_NCCL_ID_BYTES) of a new NCCL communicator id."""
    buf = ctypes.create_string_buffer(LSQ_NCCL_ID_BYTES)
    _check(load().lsq_nccl_unique_id(buf, LSQ_NCCL_ID_BYTES))
    return buf.raw


def stream_stack_shard(stack, nccl_id, world, rank, buf_bytes):
    nccl_id = bytes(nccl_id)
    if len(nccl_id) != LSQ_NCCL_ID_BYTES:
        raise ValueError("the NCCL id has %d bytes" % LSQ_NCCL_ID_BYTES)
    buf = ctypes.create_string_buffer(nccl_id, LSQ_NCCL_ID_BYTES)
    _check(load().stream_stack_shard(stack.handle, buf, LSQ_NCCL_ID_BYTES, int(world), int(rank),
                                     int(buf_bytes)))


def stream_stack_reduce_grads(stack, nccl_id, world, rank):
    nccl_id = bytes(nccl_id)
    if len(nccl_id) != LSQ_NCCL_ID_BYTES:
        raise ValueError("the NCCL id has %d bytes" % LSQ_NCCL_ID_BYTES)
    buf = ctypes.create_string_buffer(nccl_id, LSQ_NCCL_ID_BYTES)
    _check(load().stream_stack_reduce_grads(stack.handle, buf, LSQ_NCCL_ID_BYTES, int(world),
                                            int(rank)))


def stream_stack_workspace_bytes(cfg, batch, seq):
    c = cfg_struct(cfg)
    return load().stream_stack_workspace_bytes(ctypes.byref(c), batch, seq)


def stream_stack_step(stack, tokens, micro_batches, batch, seq, emb, lm_head, final_norm, lora,
                      lora_grad, opt, ws, logits_out=None, timeout_ms=600000, stream=None):
    """Returns the mean loss (host float).  opt: dict(lr, beta1, beta2, eps, weight_decay,
    step, m, v) or None."""
    loss = ctypes.c_float(0.0)
    o = _adamw_struct(opt) if opt is not None else None
    _check(load().stream_stack_step(stack.handle, _ptr(tokens), micro_batches, batch, seq,
                                    _ptr(emb), _ptr(lm_head), _ptr(final_norm), _ptr(lora),
                                    _ptr(lora_grad), ctypes.byref(o) if o is not None else None,
                                    ctypes.byref(loss), _ptr(logits_out), _ptr(ws), ws.numel(),
                                    _stream(stream), timeout_ms))
    return loss.value


def stream_stack_dpo_workspace_bytes(cfg, pairs, seq):
    c = cfg_struct(cfg)
    return load().stream_stack_dpo_workspace_bytes(ctypes.byref(c), pairs, seq)


def stream_stack_dpo_step(stack, tokens, pairs, seq, beta, emb, lm_head, final_norm, lora,
                          lora_grad, opt, ws, logits_out=None, timeout_ms=600000, stream=None):
    """tokens: int32 device [pairs, 2, seq] (chosen, rejected).  Returns (loss, logps) with
    logps a list of (policy chosen, policy rejected, reference chosen, reference rejected)
    per pair."""
    loss = ctypes.c_float(0.0)
    lp = (ctypes.c_float * (4 * pairs))()
    o = _adamw_struct(opt) if opt is not None else None
    _check(load().stream_stack_dpo_step(stack.handle, _ptr(tokens), pairs, seq, beta, _ptr(emb),
                                        _ptr(lm_head), _ptr(final_norm), _ptr(lora),
                                        _ptr(lora_grad),
                                        ctypes.byref(o) if o is not None else None,
                                        ctypes.byref(loss), lp, _ptr(logits_out), _ptr(ws),
                                        ws.numel(), _stream(stream), timeout_ms))
    return loss.value, [tuple(lp[4 * p: 4 * p + 4]) for p in range(pairs)]


def stream_stack_last_stats(stack):
    s = lsq_step_stats()
    _check(load().stream_stack_last_stats(stack.handle, ctypes.byref(s)))
    return dict(layer_copies=s.layer_copies, h2d_bytes=s.h2d_bytes, step_ms=s.step_ms,
                copy_wait_ms=s.copy_wait_ms)


def _adamw_struct(opt):
    return lsq_adamw(lr=opt["lr"], beta1=opt["beta1"], beta2=opt["beta2"], eps=opt["eps"],
                     weight_decay=opt["weight_decay"], step=opt["step"],
                     m=opt["m"].data_ptr(), v=opt["v"].data_ptr())


def lora_adamw_step(lora, grad, opt, stream=None):
    o = _adamw_struct(opt)
    _check(load().lora_adamw_step(_ptr(lora), _ptr(grad), ctypes.byref(o), lora.numel(),
                                  _stream(stream)))


def lsq_launch_counter():
    return load().lsq_launch_counter()


def lsq_profile_enable(enable=True):
    _check(load().lsq_profile_enable(1 if enable else 0))


def lsq_profile_read():
    """-> dict kernel class -> dict(launches, total_ms, flops, bytes)."""
    arr = (lsq_prof_entry * 64)()
    n = ctypes.c_int32(0)
    _check(load().lsq_profile_read(arr, 64, ctypes.byref(n)))
    return {arr[i].name.decode(): dict(launches=arr[i].launches, total_ms=arr[i].total_ms,
                                       flops=arr[i].flops, bytes=arr[i].bytes)
            for i in range(n.value)}


def nf4_lora_linear_fwd_noalloc(x, codes, absmax, A, B, scale, y, residual=None, u_out=None,
                                block=64, stream=None):
    """nf4_lora_linear_fwd with the library's built-in scratch instead of a workspace."""
    T, K = x.shape
    N = y.shape[1]
    r = A.shape[0]
    _check(load().nf4_lora_linear_fwd_noalloc(_ptr(x), T, K, N, _ptr(codes), _ptr(absmax), block,
                                              _ptr(A), _ptr(B), r, scale, _ptr(residual), _ptr(y),
                                              _y_fp32(y), _ptr(u_out), _stream(stream)))
