"""ctypes binding of libzo.so: the C ABI of include/zo.h with the same names.

Argument marshalling only: torch tensors are passed as raw device pointers and the
current torch CUDA stream as the context's stream.  Every step of the hot path runs in
the library's CUDA kernels; there is no Python or CPU fallback.  If libzo.so is
missing, importing this module raises ImportError.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzo.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libzo.so is not built; run `python zero_order_forward_b200/build.py` "
        "(nvcc, sm_100a) before using zero_order_forward_b200")

_L = ctypes.CDLL(LIB_PATH)

ZO_F32, ZO_BF16 = 0, 1
(ZO_OK, ZO_ERR_INVALID, ZO_ERR_STATE, ZO_ERR_CUDA, ZO_ERR_OOM, ZO_ERR_NONFINITE,
 ZO_ERR_UNSUPPORTED, ZO_ERR_TIMEOUT) = range(8)
ZO_FLAG_NONFINITE = 0x1
ZO_FLAG_TIMEOUT = 0x2
ZO_EPI_BIAS_BF16, ZO_EPI_RELU_BF16, ZO_EPI_RESID_F32 = 0, 1, 2
ZO_KT_GEMM, ZO_KT_ATTENTION, ZO_KT_PERTURB, ZO_KT_UPDATE, ZO_KT_COUNT = 0, 1, 2, 3, 4
KERNEL_CLASSES = ("gemm", "attention", "perturb", "update")
ZO_MAX_PROBES = 1024
ZO_NOALLOC_MAX_BATCH = 4096

_vp, _i32, _i64, _u32, _u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64
_f32, _f64, _int = ctypes.c_float, ctypes.c_double, ctypes.c_int

_SIGS = {
    "zo_create": [ctypes.POINTER(_vp), _vp, _i64, _int, _u64, _vp],
    "zo_destroy": [_vp],
    "zo_set_alpha": [_vp, _f32],
    "zo_set_live_buffer": [_vp, _int],
    "zo_sync": [_vp, ctypes.POINTER(_u32)],
    "zo_get_step": [_vp, ctypes.POINTER(_u32)],
    "zo_set_step": [_vp, _u32],
    "zo_set_element_offset": [_vp, _i64],
    "zo_pack_probe": [_vp, _u32, _i32, _i64, _i64, _vp],
    "zo_perturb": [_vp, _int, _f32, _i32],
    "zo_restore": [_vp],
    "zo_perturb_range": [_vp, _i64, _i64, _vp],
    "zo_quad_loss": [_vp, _vp, _vp, _int],
    "zo_quad_loss_pair": [_vp, _vp, _i32, _f32, _vp, _vp],
    "zo_mlp_loss": [_vp, _vp, _vp, _int, _int, _int, _int, _f64, _vp, _int],
    "zo_step": [_vp, _vp, _vp, _i32, _vp, _f32, _f32, _f32],
    "zo_update": [_vp, _vp, _i32],
    "zo_get_precond": [_vp, _i32, _vp, _vp, _vp, _vp],
    "zo_quad_step": [_vp, _vp, _i32, _f32, _f32, _f32, _int, _vp],
    "zo_quad_step_host": [_vp, _vp, _i32, _f32, _f32, _f32, _int, _vp],
    "zo_quad_step_host_async": [_vp, _vp, _i32, _f32, _f32, _f32, _int, _vp],
    "zo_mlp_step": [_vp, _vp, _vp, _int, _int, _int, _int, _i32, _f32, _f32, _f32, _int, _vp],
    "zo_mlp_losses": [_vp, _vp, _vp, _int, _int, _int, _int, _i32, _f32, _f64, _vp, _vp, _vp],
    "zo_mlp_loss_noalloc": [_vp, _vp, _vp, _int, _int, _int, _int, _f64, _vp, _int, _vp],
    "zo_enable_phase_timing": [_vp, _i32],
    "zo_phase_times": [_vp, _i32, _vp],
    "zo_model_param_count": [_vp, ctypes.POINTER(_i64)],
    "zo_model_create": [ctypes.POINTER(_vp), _vp, _vp, _i64],
    "zo_model_destroy": [_vp],
    "zo_model_loss": [_vp, _vp, _vp, _i32, _i32, _f64, _vp, _int],
    "zo_model_hidden": [_vp, _vp, _i32, _i32, _i32, _vp],
    "zo_model_step": [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _f32, _f32, _f32, _int, _vp],
    "zo_gemm_bf16": [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32],
    "zo_gemm_bf16_perturbed": [_vp, _vp, _i64, _vp, _vp, _i32, _i32, _i32, _i32, _i32],
    "zo_attention": [_vp, _vp, _vp, _i32, _i32, _i32, _i32],
    "zo_attention_gqa": [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32],
    "zo_model_set_pruning": [_vp, _int],
    "zo_quad_loss_octet": [_vp, _vp, _i32, _i32, _f32, _vp, _vp, _vp],
    "zo_lowrank_loss": [_vp, _vp, _vp, _vp, _int],
    "zo_lowrank_loss_pair": [_vp, _vp, _vp, _i32, _f32, _vp, _vp],
    "zo_lowrank_step": [_vp, _vp, _vp, _i32, _f32, _f32, _f32, _int, _vp],
    "zo_rmsnorm": [_vp, _vp, _vp, _vp, _i32, _i32, _f32],
    "zo_debug_gemm_timeout": [_vp, _vp, _vp, _vp, _i32, _i32, _i32],
    "zo_layernorm": [_vp, _vp, _vp, _vp, _vp, _i32, _i32],
    "zo_enable_kernel_timing": [_vp, _int],
    "zo_kernel_times": [_vp, _vp, ctypes.POINTER(_i64)],
    "zo_launch_count": [_vp, ctypes.POINTER(_i64)],
    "zo_set_loss_location": [_vp, _int],
    "zo_model_step_host": [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _f32, _f32, _f32, _int, _vp],
}
for _name, _args in _SIGS.items():
    _fn = getattr(_L, _name)
    _fn.argtypes = _args
    _fn.restype = _int
_L.zo_last_error.argtypes = [_vp]
_L.zo_last_error.restype = ctypes.c_char_p
_L.zo_status_name.argtypes = [_int]
_L.zo_status_name.restype = ctypes.c_char_p
_L.zo_live_params.argtypes = [_vp]
_L.zo_live_params.restype = _vp

lib = _L


class ZoError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_L.zo_status_name(status).decode()}: {msg}")
        self.status = status


def _ptr(t):
    """Device (or host) address of a tensor / numpy array / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if hasattr(t, "ctypes"):
        return t.ctypes.data
    raise TypeError(type(t))


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


class Ctx:
    """Owns a zo_ctx*; keeps the parameter tensor alive."""

    def __init__(self, handle, params, M, dtype):
        self.handle, self.params, self.M, self.dtype = handle, params, M, dtype

    def check(self, status):
        if status != ZO_OK:
            msg = _L.zo_last_error(self.handle) if self.handle else b""
            raise ZoError(status, msg.decode() if msg else "")
        return status

    def close(self):
        if self.handle:
            _L.zo_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def zo_create(params, seed=0, stream=None, M=None, dtype=None):
    """params: a CUDA tensor (float32 or bfloat16) holding the flat theta."""
    import torch
    if dtype is None:
        dtype = {torch.float32: ZO_F32, torch.bfloat16: ZO_BF16}[params.dtype]
    if M is None:
        M = params.numel()
    h = _vp()
    st = _L.zo_create(ctypes.byref(h), _ptr(params), int(M), int(dtype), int(seed) & (2**64 - 1),
                      _stream(stream))
    if st != ZO_OK:
        raise ZoError(st, "zo_create failed")
    return Ctx(h, params, M, dtype)


def zo_destroy(ctx):
    ctx.close()


def zo_last_error(ctx):
    return _L.zo_last_error(ctx.handle).decode()


def zo_status_name(status):
    return _L.zo_status_name(status).decode()


def zo_set_alpha(ctx, alpha):
    return ctx.check(_L.zo_set_alpha(ctx.handle, alpha))


def zo_set_live_buffer(ctx, enable):
    return ctx.check(_L.zo_set_live_buffer(ctx.handle, int(bool(enable))))


def zo_live_params(ctx):
    return _L.zo_live_params(ctx.handle)


def zo_sync(ctx, raise_nonfinite=True):
    flags = _u32()
    st = _L.zo_sync(ctx.handle, ctypes.byref(flags))
    if st == ZO_ERR_NONFINITE and not raise_nonfinite:
        return flags.value
    ctx.check(st)
    return flags.value


def zo_get_step(ctx):
    s = _u32()
    ctx.check(_L.zo_get_step(ctx.handle, ctypes.byref(s)))
    return s.value


def zo_set_step(ctx, step):
    return ctx.check(_L.zo_set_step(ctx.handle, step))


def zo_set_element_offset(ctx, first_element):
    return ctx.check(_L.zo_set_element_offset(ctx.handle, int(first_element)))


def zo_pack_probe(ctx, step, probe, first_byte, nbytes, out):
    return ctx.check(_L.zo_pack_probe(ctx.handle, int(step) & 0xFFFFFFFF, probe, first_byte, nbytes,
                                      _ptr(out)))


def zo_perturb(ctx, sign, eps, probe):
    return ctx.check(_L.zo_perturb(ctx.handle, sign, eps, probe))


def zo_restore(ctx):
    return ctx.check(_L.zo_restore(ctx.handle))


def zo_perturb_range(ctx, first, count, out):
    return ctx.check(_L.zo_perturb_range(ctx.handle, first, count, _ptr(out)))


def zo_quad_loss(ctx, D, loss_out, accumulate=False):
    return ctx.check(_L.zo_quad_loss(ctx.handle, _ptr(D), _ptr(loss_out), int(accumulate)))


def zo_quad_loss_pair(ctx, D, probe, eps, loss_plus, loss_minus):
    return ctx.check(_L.zo_quad_loss_pair(ctx.handle, _ptr(D), probe, eps, _ptr(loss_plus),
                                          _ptr(loss_minus)))


def zo_mlp_loss(ctx, X, labels, batch, n_in, n_hidden, n_out, scale, loss_out, accumulate=False):
    return ctx.check(_L.zo_mlp_loss(ctx.handle, _ptr(X), _ptr(labels), batch, n_in, n_hidden,
                                    n_out, scale, _ptr(loss_out), int(accumulate)))


def zo_step(ctx, loss_plus, loss_minus, n_pert, loss0, lr, eps, damping):
    return ctx.check(_L.zo_step(ctx.handle, _ptr(loss_plus), _ptr(loss_minus), n_pert,
                                _ptr(loss0), lr, eps, damping))


def zo_set_loss_location(ctx, on_device):
    """on_device False: zo_step takes host arrays (numpy) for its losses."""
    return ctx.check(_L.zo_set_loss_location(ctx.handle, 1 if on_device else 0))


def zo_update(ctx, coef, n_pert):
    return ctx.check(_L.zo_update(ctx.handle, _ptr(coef), n_pert))


def zo_get_precond(ctx, n):
    """Returns (g, c, w, a) as numpy arrays from the last zo_step (synchronises)."""
    import numpy as np
    g, c, w = (np.zeros(n, np.float64) for _ in range(3))
    a = np.zeros(n, np.float32)
    ctx.check(_L.zo_get_precond(ctx.handle, n, g.ctypes.data, c.ctypes.data, w.ctypes.data, a.ctypes.data))
    return g, c, w, a


def zo_quad_step(ctx, D, n_pert, eps, lr, damping, preconditioned, losses_out):
    return ctx.check(_L.zo_quad_step(ctx.handle, _ptr(D), n_pert, eps, lr, damping,
                                     int(preconditioned), _ptr(losses_out)))


def zo_quad_step_host(ctx, D_host, n_pert, eps, lr, damping, preconditioned, losses_host):
    return ctx.check(_L.zo_quad_step_host(ctx.handle, _ptr(D_host), n_pert, eps, lr, damping,
                                          int(preconditioned), _ptr(losses_host)))


def zo_quad_step_host_async(ctx, D_host, n_pert, eps, lr, damping, preconditioned, losses_host):
    return ctx.check(_L.zo_quad_step_host_async(ctx.handle, _ptr(D_host), n_pert, eps, lr, damping,
                                          int(preconditioned), _ptr(losses_host)))


def zo_mlp_step(ctx, X, labels, batch, n_in, n_hidden, n_out, n_pert, eps, lr, damping,
                preconditioned, losses_out):
    return ctx.check(_L.zo_mlp_step(ctx.handle, _ptr(X), _ptr(labels), batch, n_in, n_hidden,
                                    n_out, n_pert, eps, lr, damping, int(preconditioned),
                                    _ptr(losses_out)))


def zo_mlp_losses(ctx, X, labels, batch, n_in, n_hidden, n_out, n_pert, eps, scale, loss_plus,
                  loss_minus, loss_clean=None):
    return ctx.check(_L.zo_mlp_losses(ctx.handle, _ptr(X), _ptr(labels), batch, n_in, n_hidden,
                                      n_out, n_pert, eps, scale, _ptr(loss_plus),
                                      _ptr(loss_minus), _ptr(loss_clean)))


def zo_mlp_loss_noalloc(P, X, labels, batch, n_in, n_hidden, n_out, scale, loss_out,
                        accumulate=False, stream=None):
    """MLP loss for callers that cannot allocate device memory (see include/zo.h): no
    context, scratch in the library's static device memory.  stream=None enqueues on
    torch.cuda.current_stream(); stream=0 passes NULL, the legacy default stream.  Raises
    ZoError on failure."""
    st = _L.zo_mlp_loss_noalloc(_ptr(P), _ptr(X), _ptr(labels), batch, n_in, n_hidden, n_out,
                                scale, _ptr(loss_out), int(accumulate), _stream(stream))
    if st != ZO_OK:
        raise ZoError(st, "zo_mlp_loss_noalloc failed")
    return st


# ------------------------------------------------------------------ decoder


ZO_FAMILY_OPT, ZO_FAMILY_QWEN3 = 0, 1


class zo_lowrank(ctypes.Structure):
    _fields_ = [("rank", _i32), ("lam", _f32 * 4), ("vseed", ctypes.c_uint64)]

    @classmethod
    def make(cls, lam, vseed):
        lam = list(lam)
        if not 1 <= len(lam) <= 4:
            raise ValueError("rank must be 1..4")
        return cls(len(lam), (_f32 * 4)(*(lam + [0.0] * (4 - len(lam)))), vseed)


class zo_model_cfg(ctypes.Structure):
    _fields_ = [("n_layers", _i32), ("d_model", _i32), ("n_heads", _i32), ("d_ffn", _i32),
                ("vocab", _i32), ("max_pos", _i32), ("class_ids", _i32 * 2), ("family", _i32),
                ("n_kv_heads", _i32), ("head_dim", _i32), ("rope_theta", _f32),
                ("norm_eps", _f32)]

    @classmethod
    def from_dict(cls, c):
        qwen = c.get("family") == "qwen3"
        return cls(c["n_layers"], c["d_model"], c["n_heads"], c["d_ffn"], c["vocab"],
                   c["max_pos"], (_i32 * 2)(*c["class_ids"]),
                   ZO_FAMILY_QWEN3 if qwen else ZO_FAMILY_OPT,
                   c.get("n_kv_heads", c["n_heads"]),
                   c.get("head_dim", c["d_model"] // c["n_heads"]),
                   float(c.get("rope_theta", 0.0)), float(c.get("norm_eps", 0.0)))


class Model:
    """Owns a zo_model*; keeps its context alive."""

    def __init__(self, handle, ctx, cfg):
        self.handle, self.ctx, self.cfg = handle, ctx, cfg

    def close(self):
        if self.handle:
            _L.zo_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def zo_model_param_count(cfg):
    m = _i64()
    c = zo_model_cfg.from_dict(cfg)
    st = _L.zo_model_param_count(ctypes.byref(c), ctypes.byref(m))
    if st != ZO_OK:
        raise ZoError(st, "invalid model configuration")
    return m.value


def zo_model_create(ctx, cfg, max_tokens):
    h = _vp()
    c = zo_model_cfg.from_dict(cfg)
    ctx.check(_L.zo_model_create(ctypes.byref(h), ctx.handle, ctypes.byref(c), int(max_tokens)))
    return Model(h, ctx, cfg)


def zo_quad_loss_octet(ctx, D, first_probe, count, eps, loss_plus, loss_minus, loss_clean=None):
    return ctx.check(_L.zo_quad_loss_octet(ctx.handle, _ptr(D), first_probe, count, eps,
                                           _ptr(loss_plus), _ptr(loss_minus), _ptr(loss_clean)))


def zo_lowrank_loss(ctx, D, lam, vseed, loss_out, accumulate=False):
    q = zo_lowrank.make(lam, vseed)
    return ctx.check(_L.zo_lowrank_loss(ctx.handle, _ptr(D), ctypes.byref(q), _ptr(loss_out),
                                        1 if accumulate else 0))


def zo_lowrank_loss_pair(ctx, D, lam, vseed, probe, eps, loss_plus, loss_minus):
    q = zo_lowrank.make(lam, vseed)
    return ctx.check(_L.zo_lowrank_loss_pair(ctx.handle, _ptr(D), ctypes.byref(q), probe, eps,
                                             _ptr(loss_plus), _ptr(loss_minus)))


def zo_lowrank_step(ctx, D, lam, vseed, n_pert, eps, lr, damping, preconditioned, losses_out):
    q = zo_lowrank.make(lam, vseed)
    return ctx.check(_L.zo_lowrank_step(ctx.handle, _ptr(D), ctypes.byref(q), n_pert, eps, lr,
                                        damping, 1 if preconditioned else 0, _ptr(losses_out)))


def zo_model_set_pruning(model, enabled):
    return model.ctx.check(_L.zo_model_set_pruning(model.handle, 1 if enabled else 0))


def zo_model_destroy(model):
    model.close()


def zo_model_loss(model, tokens, labels, batch, seq, scale, loss_out, accumulate=False):
    return model.ctx.check(_L.zo_model_loss(model.handle, _ptr(tokens), _ptr(labels), batch, seq,
                                            scale, _ptr(loss_out), int(accumulate)))


def zo_model_hidden(model, tokens, batch, seq, n_layers_run, h_out):
    return model.ctx.check(_L.zo_model_hidden(model.handle, _ptr(tokens), batch, seq,
                                              n_layers_run, _ptr(h_out)))


def zo_model_step(model, tokens, labels, batch, seq, n_micro, n_pert, eps, lr, damping,
                  preconditioned, losses_out):
    return model.ctx.check(_L.zo_model_step(model.handle, _ptr(tokens), _ptr(labels), batch, seq,
                                            n_micro, n_pert, eps, lr, damping,
                                            int(preconditioned), _ptr(losses_out)))


def zo_model_step_host(model, tokens_host, labels_host, batch, seq, n_micro, n_pert, eps, lr,
                       damping, preconditioned, losses_host):
    """zo_model_step from host int32 tokens/labels (numpy or pinned CPU tensors) with the
    2 n_pert + 1 losses copied back to losses_host (host float64); synchronises."""
    return model.ctx.check(_L.zo_model_step_host(model.handle, _ptr(tokens_host), _ptr(labels_host),
                                                 batch, seq, n_micro, n_pert, eps, lr, damping,
                                                 int(preconditioned), _ptr(losses_host)))


def zo_gemm_bf16(ctx, A, B, bias, out, M, N, K, ldo, epilogue):
    return ctx.check(_L.zo_gemm_bf16(ctx.handle, _ptr(A), _ptr(B), _ptr(bias), _ptr(out), M, N,
                                     K, ldo, epilogue))


def zo_gemm_bf16_perturbed(ctx, A, w_offset, bias, out, M, N, K, ldo, epilogue):
    """The GEMM with B = ctx's parameters [w_offset, w_offset + N K) under ctx's current
    perturbation, fused into the operand path (zo.h)."""
    return ctx.check(_L.zo_gemm_bf16_perturbed(ctx.handle, _ptr(A), w_offset, _ptr(bias), _ptr(out),
                                               M, N, K, ldo, epilogue))


def zo_attention(ctx, qkv, out, batch, seq, n_heads, d_model):
    return ctx.check(_L.zo_attention(ctx.handle, _ptr(qkv), _ptr(out), batch, seq, n_heads,
                                     d_model))


def zo_attention_gqa(ctx, qkv, out, batch, seq, n_heads, n_kv_heads, head_dim):
    return ctx.check(_L.zo_attention_gqa(ctx.handle, _ptr(qkv), _ptr(out), batch, seq, n_heads,
                                         n_kv_heads, head_dim))


def zo_rmsnorm(ctx, x, w, out, rows, d, eps):
    return ctx.check(_L.zo_rmsnorm(ctx.handle, _ptr(x), _ptr(w), _ptr(out), rows, d, eps))


def zo_layernorm(ctx, x, gamma, beta, out, rows, d):
    return ctx.check(_L.zo_layernorm(ctx.handle, _ptr(x), _ptr(gamma), _ptr(beta), _ptr(out),
                                     rows, d))


def zo_enable_phase_timing(ctx, n_steps):
    return ctx.check(_L.zo_enable_phase_timing(ctx.handle, n_steps))


def zo_phase_times(ctx, n_steps):
    """[n_steps][3] ms (clean loss, perturbed losses, precond + update) of recorded steps."""
    import numpy as np
    ms = np.zeros((n_steps, 3), np.float32)
    ctx.check(_L.zo_phase_times(ctx.handle, n_steps, ms.ctypes.data))
    return ms


class zo_kernel_time(ctypes.Structure):
    _fields_ = [("ms", _f64), ("launches", _i64), ("work", _f64)]


def zo_enable_kernel_timing(ctx, enable):
    return ctx.check(_L.zo_enable_kernel_timing(ctx.handle, 1 if enable else 0))


def zo_kernel_times(ctx):
    """Per kernel class ({"gemm", "attention", "perturb", "update"}): summed ms, launches and
    algorithmic work of the launches recorded since the last call (synchronises), and the
    number of launches not recorded."""
    out = (zo_kernel_time * ZO_KT_COUNT)()
    dropped = _i64()
    ctx.check(_L.zo_kernel_times(ctx.handle, out, ctypes.byref(dropped)))
    return ({name: {"ms": out[i].ms, "launches": out[i].launches, "work": out[i].work}
             for i, name in enumerate(KERNEL_CLASSES)}, dropped.value)


def zo_launch_count(ctx):
    n = _i64()
    ctx.check(_L.zo_launch_count(ctx.handle, ctypes.byref(n)))
    return n.value


def zo_debug_gemm_timeout(ctx, A, B, out, M, N, K):
    return ctx.check(_L.zo_debug_gemm_timeout(ctx.handle, _ptr(A), _ptr(B), _ptr(out), M, N, K))
