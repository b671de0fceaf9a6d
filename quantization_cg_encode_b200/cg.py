"""Thin Python binding of libcg (C ABI in include/cg.h).

Argument marshalling only: every function checks the torch tensors it is given
(device, dtype, contiguity, size), passes their raw device pointers and the
current CUDA stream to the C entry point of the same name, and raises on a
non-OK status.  All computation happens in the CUDA library; there is no
fallback of any kind.  torch is used for device memory and streams only.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcg.so")

CG_OK, CG_ERR_INVALID, CG_ERR_UNSUPPORTED, CG_ERR_CUDA, CG_ERR_TIMEOUT, CG_ERR_TOO_LARGE, CG_ERR_BOUND = range(7)
BLOCK_UNIFORM, KIVI = 0, 1
ENGINE_AUTO, ENGINE_CUDA_CORES, ENGINE_CHAIN_TENSOR = 0, 1, 2

# Every symbol include/cg.h declares.
EXPORTS = ("cg_sizes_for", "cg_gauge_build", "cg_gauge_grad", "cg_adamw_step", "cg_group_gram", "cg_encode",
           "cg_decode", "cg_roundtrip_workspace_size", "cg_roundtrip_host", "cg_decode_attention_workspace_size",
           "cg_decode_attention", "cg_spectral_workspace_size",
           "cg_spectral_stats", "cg_spectral_stats_noalloc", "cg_selftest_wait_timeout", "cg_sync_status",
           "cg_last_cuda_error", "cg_status_string", "cg_version")


class KvDesc(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int32), ("batch", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("tokens", ctypes.c_int32), ("d_head", ctypes.c_int32)]


class CodecDesc(ctypes.Structure):
    _fields_ = [("g", ctypes.c_int32), ("bits", ctypes.c_int32), ("tb", ctypes.c_int32),
                ("range_cols", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("kivi_key_tokens", ctypes.c_int32), ("kivi_val_channels", ctypes.c_int32),
                ("engine", ctypes.c_int32)]


class Sizes(ctypes.Structure):
    _fields_ = [("code_bytes", ctypes.c_uint64), ("scale_count", ctypes.c_uint64)]


class StatsDesc(ctypes.Structure):
    _fields_ = [("tb", ctypes.c_int32), ("g", ctypes.c_int32), ("x_is_fp32", ctypes.c_int32),
                ("lambda_f", ctypes.c_float), ("lambda_r", ctypes.c_float), ("tau", ctypes.c_float)]


class AdamwDesc(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float)]


def adamw_desc(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01):
    return AdamwDesc(lr, beta1, beta2, eps, weight_decay)


class AttnDesc(ctypes.Structure):
    _fields_ = [("q_heads", ctypes.c_int32), ("n_tokens", ctypes.c_int32), ("layer0", ctypes.c_int32),
                ("n_layers", ctypes.c_int32), ("scale", ctypes.c_float)]


class CgError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        extra = ""
        if status == CG_ERR_CUDA:
            extra = ": " + lib().cg_last_cuda_error().decode()
        super().__init__("%s: %s (status %d)%s" % (where, status_string(status), status, extra))


_lib = None


def lib():
    """The loaded libcg.  Raises if the library has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libcg.so not found at %s: build it with `python -m quantization_cg_encode_b200.build`"
                              % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64
        L.cg_sizes_for.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(CodecDesc), ctypes.POINTER(Sizes)]
        L.cg_gauge_build.argtypes = [vp, vp, i32, i32, vp]
        L.cg_gauge_grad.argtypes = [vp, vp, vp, i32, i32, vp]
        L.cg_adamw_step.argtypes = [vp, vp, vp, vp, ctypes.c_int64, ctypes.POINTER(AdamwDesc), i32, vp]
        L.cg_group_gram.argtypes = [ctypes.POINTER(KvDesc), i32, vp, i32, i32, vp, vp]
        L.cg_encode.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(CodecDesc), vp, vp, i32, i32, vp, vp, vp, vp, vp]
        L.cg_decode.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(CodecDesc), vp, vp, vp, vp, i32, i32, vp, vp]
        L.cg_roundtrip_workspace_size.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(ctypes.c_uint64)]
        L.cg_roundtrip_host.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(CodecDesc), vp, vp, vp, vp, vp, vp, vp,
                                        ctypes.c_uint64, vp]
        L.cg_decode_attention_workspace_size.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(AttnDesc),
                                                         ctypes.POINTER(u64)]
        L.cg_decode_attention.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(CodecDesc), ctypes.POINTER(AttnDesc),
                                          vp, vp, vp, vp, vp, vp, vp, u64, vp]
        L.cg_spectral_workspace_size.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(StatsDesc), i32,
                                                 ctypes.POINTER(u64)]
        L.cg_spectral_stats.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(StatsDesc), vp, vp, vp, vp, vp, vp,
                                        vp, u64, vp]
        L.cg_spectral_stats_noalloc.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(StatsDesc), vp, vp, vp, vp, vp,
                                                vp, vp]
        L.cg_selftest_wait_timeout.argtypes = [ctypes.c_int64, vp, vp]
        L.cg_sync_status.argtypes = [vp]
        L.cg_status_string.argtypes = [ctypes.c_int]
        L.cg_status_string.restype = ctypes.c_char_p
        L.cg_version.restype = ctypes.c_int32
        L.cg_last_cuda_error.restype = ctypes.c_char_p
        for name in ("cg_sizes_for", "cg_gauge_build", "cg_gauge_grad", "cg_adamw_step", "cg_group_gram",
                     "cg_encode", "cg_decode", "cg_decode_attention_workspace_size", "cg_decode_attention",
                     "cg_spectral_workspace_size",
                     "cg_spectral_stats", "cg_spectral_stats_noalloc", "cg_selftest_wait_timeout",
                     "cg_sync_status"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status):
    return lib().cg_status_string(int(status)).decode()


def _check(status, where):
    if status != CG_OK:
        raise CgError(status, where)


def _ptr(t, dtype, name, numel=None):
    """Device pointer of a contiguous CUDA tensor of the given dtype (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if numel is not None and t.numel() < numel:
        raise ValueError("%s holds %d elements, needs %d" % (name, t.numel(), numel))
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def kv_desc(layers, batch, heads, tokens, d_head):
    return KvDesc(layers, batch, heads, tokens, d_head)


def codec_desc(g=16, bits=4, tb=16, range_cols=None, mode=BLOCK_UNIFORM, kivi_key_tokens=32, kivi_val_channels=32,
               engine=ENGINE_AUTO):
    return CodecDesc(g, bits, tb, g if range_cols is None else range_cols, mode, kivi_key_tokens, kivi_val_channels,
                     engine)


def kv_desc_of(kv):
    """KvDesc of a [L, 2, B, H, T, d] tensor."""
    L, two, B, H, T, d = kv.shape
    assert two == 2
    return KvDesc(L, B, H, T, d)


def cg_sizes_for(kvd, codec):
    out = Sizes()
    _check(lib().cg_sizes_for(ctypes.byref(kvd), ctypes.byref(codec), ctypes.byref(out)), "cg_sizes_for")
    return int(out.code_bytes), int(out.scale_count)


def gauge_numel(kvd, g):
    """Elements of a [L, 2, H, d/g, g, g] gauge array."""
    return kvd.layers * 2 * kvd.heads * kvd.d_head * g


def alloc_encoded(kvd, codec, device="cuda"):
    """Caller-owned output buffers (codes uint8, scales fp16, zeros fp16)."""
    cb, sc = cg_sizes_for(kvd, codec)
    return (torch.zeros(cb, dtype=torch.uint8, device=device),
            torch.zeros(sc, dtype=torch.float16, device=device),
            torch.zeros(sc, dtype=torch.float16, device=device))


def cg_gauge_build(A, G, stream=None):
    """G = exp(A - A^T) for A of shape [..., g, g] (fp32)."""
    g = A.shape[-1]
    n = A.numel() // (g * g)
    _check(lib().cg_gauge_build(_ptr(A, torch.float32, "A"), _ptr(G, torch.float32, "G", A.numel()), n, g,
                                _stream(stream)), "cg_gauge_build")
    return G


def cg_gauge_grad(A, dG, dA, stream=None):
    """dL/dA from dL/dG for G = exp(A - A^T); A, dG, dA fp32 of shape [..., g, g]."""
    g = A.shape[-1]
    n = A.numel() // (g * g)
    _check(lib().cg_gauge_grad(_ptr(A, torch.float32, "A"), _ptr(dG, torch.float32, "dG", A.numel()),
                               _ptr(dA, torch.float32, "dA", A.numel()), n, g, _stream(stream)), "cg_gauge_grad")
    return dA


def cg_adamw_step(param, grad, m, v, hp, step, stream=None):
    """One AdamW step in place on fp32 CUDA tensors of equal size (step is 1-based)."""
    n = param.numel()
    _check(lib().cg_adamw_step(_ptr(param, torch.float32, "param"), _ptr(grad, torch.float32, "grad", n),
                               _ptr(m, torch.float32, "m", n), _ptr(v, torch.float32, "v", n), n, ctypes.byref(hp),
                               int(step), _stream(stream)), "cg_adamw_step")


def cg_group_gram(kvd, g, kv, gram, t0=0, nt=None, stream=None):
    """fp64 Gram matrices [L, 2, H, d/g, g, g] of the groups of tokens [t0, t0 + nt)."""
    nt = kvd.tokens - t0 if nt is None else nt
    n = kvd.layers * 2 * kvd.batch * kvd.heads * kvd.tokens * kvd.d_head
    _check(lib().cg_group_gram(ctypes.byref(kvd), int(g), _ptr(kv, torch.bfloat16, "kv", n), int(t0), int(nt),
                               _ptr(gram, torch.float64, "gram", kvd.layers * 2 * kvd.heads * kvd.d_head * g),
                               _stream(stream)), "cg_group_gram")
    return gram


def cg_encode(kvd, codec, kv, G, t0, nt, codes, scales, zeros, gauged=None, stream=None):
    n = kvd.layers * 2 * kvd.batch * kvd.heads * kvd.tokens * kvd.d_head
    cb, sc = cg_sizes_for(kvd, codec)
    _check(lib().cg_encode(ctypes.byref(kvd), ctypes.byref(codec), _ptr(kv, torch.bfloat16, "kv", n),
                           _ptr(G, torch.float32, "G", gauge_numel(kvd, codec.g)),
                           int(t0), int(nt), _ptr(codes, torch.uint8, "codes", cb),
                           _ptr(scales, torch.float16, "scales", sc), _ptr(zeros, torch.float16, "zeros", sc),
                           _ptr(gauged, torch.float32, "gauged", n), _stream(stream)), "cg_encode")


def cg_decode(kvd, codec, codes, scales, zeros, G, t0, nt, kv_out, stream=None):
    n = kvd.layers * 2 * kvd.batch * kvd.heads * kvd.tokens * kvd.d_head
    cb, sc = cg_sizes_for(kvd, codec)
    _check(lib().cg_decode(ctypes.byref(kvd), ctypes.byref(codec), _ptr(codes, torch.uint8, "codes", cb),
                           _ptr(scales, torch.float16, "scales", sc), _ptr(zeros, torch.float16, "zeros", sc),
                           _ptr(G, torch.float32, "G", gauge_numel(kvd, codec.g)), int(t0), int(nt), _ptr(kv_out, torch.bfloat16, "kv_out", n),
                           _stream(stream)), "cg_decode")


def cg_roundtrip_workspace_size(kvd):
    out = ctypes.c_uint64()
    _check(lib().cg_roundtrip_workspace_size(ctypes.byref(kvd), ctypes.byref(out)), "cg_roundtrip_workspace_size")
    return int(out.value)


def _host_ptr(t, dtype, name, numel):
    """Host pointer of a contiguous CPU tensor of the given dtype."""
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError("%s must be a CPU tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.numel() < numel:
        raise ValueError("%s holds %d elements, needs %d" % (name, t.numel(), numel))
    return ctypes.c_void_p(t.data_ptr())


def cg_roundtrip_host(kvd, codec, kv_host, G, codes, scales, zeros, out_host, workspace, stream=None):
    """Encode a host-resident cache (bf16 CPU tensor, pinned for overlap) into device codes and
    decode it back into out_host, pipelined by layer."""
    n = kvd.layers * 2 * kvd.batch * kvd.heads * kvd.tokens * kvd.d_head
    cb, sc = cg_sizes_for(kvd, codec)
    _check(lib().cg_roundtrip_host(ctypes.byref(kvd), ctypes.byref(codec), _host_ptr(kv_host, torch.bfloat16, "kv_host", n),
                                   _ptr(G, torch.float32, "G", gauge_numel(kvd, codec.g)),
                                   _ptr(codes, torch.uint8, "codes", cb), _ptr(scales, torch.float16, "scales", sc),
                                   _ptr(zeros, torch.float16, "zeros", sc),
                                   _host_ptr(out_host, torch.bfloat16, "out_host", n),
                                   _ptr(workspace, torch.uint8, "workspace"),
                                   workspace.numel(), _stream(stream)), "cg_roundtrip_host")


def attn_desc(q_heads, n_tokens, layer0=0, n_layers=1, scale=None, d_head=128):
    return AttnDesc(q_heads, n_tokens, layer0, n_layers, (1.0 / d_head ** 0.5) if scale is None else scale)


def cg_decode_attention_workspace_size(kvd, at):
    out = ctypes.c_uint64()
    _check(lib().cg_decode_attention_workspace_size(ctypes.byref(kvd), ctypes.byref(at), ctypes.byref(out)),
           "cg_decode_attention_workspace_size")
    return int(out.value)


def cg_decode_attention(kvd, codec, at, q, codes, scales, zeros, G, out, workspace, stream=None):
    """Decode-step attention from the encoded cache: q bf16 [n_layers, B, Hq, d] ->
    out fp32 [n_layers, B, Hq, d]."""
    cb, sc = cg_sizes_for(kvd, codec)
    nq = at.n_layers * kvd.batch * at.q_heads * kvd.d_head
    _check(lib().cg_decode_attention(ctypes.byref(kvd), ctypes.byref(codec), ctypes.byref(at),
                                     _ptr(q, torch.bfloat16, "q", nq), _ptr(codes, torch.uint8, "codes", cb),
                                     _ptr(scales, torch.float16, "scales", sc), _ptr(zeros, torch.float16, "zeros", sc),
                                     _ptr(G, torch.float32, "G", gauge_numel(kvd, codec.g)),
                                     _ptr(out, torch.float32, "out", nq), ctypes.c_void_p(workspace.data_ptr()),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "cg_decode_attention")
    return out


def cg_spectral_workspace_size(kvd, st, want_grad):
    out = ctypes.c_uint64()
    _check(lib().cg_spectral_workspace_size(ctypes.byref(kvd), ctypes.byref(st), int(bool(want_grad)),
                                            ctypes.byref(out)), "cg_spectral_workspace_size")
    return int(out.value)


def cg_spectral_stats(kvd, st, x, G, lfreq, lrate, totals, dG=None, workspace=None, stream=None):
    xdt = torch.float32 if st.x_is_fp32 else torch.bfloat16
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().cg_spectral_stats(ctypes.byref(kvd), ctypes.byref(st), _ptr(x, xdt, "x"), _ptr(G, torch.float32, "G"),
                                   _ptr(lfreq, torch.float32, "lfreq"), _ptr(lrate, torch.float32, "lrate"),
                                   _ptr(totals, torch.float64, "totals", 4), _ptr(dG, torch.float32, "dG"),
                                   None if workspace is None else ctypes.c_void_p(workspace.data_ptr()),
                                   ws_bytes, _stream(stream)), "cg_spectral_stats")


def cg_spectral_stats_noalloc(kvd, st, x, G, lfreq, lrate, totals, dG=None, stream=None):
    """cg_spectral_stats without a workspace argument: for callers that cannot
    allocate device memory, the library's built-in scratch array is used."""
    xdt = torch.float32 if st.x_is_fp32 else torch.bfloat16
    _check(lib().cg_spectral_stats_noalloc(ctypes.byref(kvd), ctypes.byref(st), _ptr(x, xdt, "x"),
                                           _ptr(G, torch.float32, "G"), _ptr(lfreq, torch.float32, "lfreq"),
                                           _ptr(lrate, torch.float32, "lrate"), _ptr(totals, torch.float64, "totals", 4),
                                           _ptr(dG, torch.float32, "dG"), _stream(stream)), "cg_spectral_stats_noalloc")


def cg_selftest_wait_timeout(limit_ns, result, stream=None):
    """Enqueue the bounded-wait self-test (see include/cg.h); result is a 1-element
    int32 CUDA tensor that receives 0 when the wait gave up."""
    _check(lib().cg_selftest_wait_timeout(int(limit_ns), _ptr(result, torch.int32, "result", 1), _stream(stream)),
           "cg_selftest_wait_timeout")


def cg_sync_status(stream=None):
    _check(lib().cg_sync_status(_stream(stream)), "cg_sync_status")


def cg_version():
    return int(lib().cg_version())
