"""Python binding of ``libvggt_attn.so`` (VGGT frame / global / descriptor
attention with fused QK LayerNorm + 2D RoPE, for B200 / sm_100a).

The functions carry the C ABI's names and arguments and only marshal them:
torch tensors become device pointers, the stream defaults to torch's current
stream, and a negative status becomes :class:`VggtError`. All computation
happens in the CUDA library; there is no other implementation behind these
names. Importing the package fails if the library has not been built
(``python feed_forward_view_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB_PATH

__all__ = [
    "VggtError",
    "DescCache",
    "lib",
    "vggt_attn_frame",
    "vggt_attn_global",
    "vggt_attn_descriptor",
    "vggt_kv_pool",
    "vggt_kv_pool_tokens",
    "vggt_qk_prologue",
    "vggt_attn_core",
    "vggt_attn_core_online",
    "vggt_attn_global_noalloc",
    "vggt_get_device_status",
    "vggt_release_scratch",
    "vggt_scratch_pool_info",
    "vggt_desc_cache_create",
    "vggt_desc_cache_destroy",
    "vggt_desc_cache_frames",
    "vggt_desc_cache_reset",
    "vggt_attn_descriptor_chunk",
    "vggt_status_string",
    "vggt_set_wait_limit",
    "vggt_debug_wait_timeout",
    "vggt_attn_frame_ex",
    "vggt_attn_global_ex",
    "vggt_attn_descriptor_ex",
    "vggt_kv_pool_ex",
    "vggt_kv_pool_tokens_ex",
    "vggt_qk_prologue_ex",
    "vggt_descriptor_keys",
    "vggt_desc_cache_create_ex",
    "vggt_attn_subset",
    "vggt_attn_frame_f32",
    "vggt_attn_global_f32",
    "vggt_attn_global_batch",
    "vggt_attn_descriptor_batch",
    "FrameLayout",
    "QKNorm",
    "EXPORTED_SYMBOLS",
]

# every symbol include/vggt_attn.h declares
EXPORTED_SYMBOLS = (
    "vggt_qk_prologue",
    "vggt_attn_core",
    "vggt_attn_core_online",
    "vggt_attn_global_noalloc",
    "vggt_attn_frame",
    "vggt_attn_global",
    "vggt_attn_descriptor",
    "vggt_kv_pool",
    "vggt_kv_pool_tokens",
    "vggt_get_device_status",
    "vggt_release_scratch",
    "vggt_scratch_pool_info",
    "vggt_desc_cache_create",
    "vggt_desc_cache_destroy",
    "vggt_desc_cache_frames",
    "vggt_desc_cache_reset",
    "vggt_attn_descriptor_chunk",
    "vggt_status_string",
    "vggt_set_wait_limit",
    "vggt_debug_wait_timeout",
    "vggt_attn_frame_ex",
    "vggt_attn_global_ex",
    "vggt_attn_descriptor_ex",
    "vggt_kv_pool_ex",
    "vggt_kv_pool_tokens_ex",
    "vggt_qk_prologue_ex",
    "vggt_descriptor_keys",
    "vggt_desc_cache_create_ex",
    "vggt_attn_subset",
    "vggt_attn_frame_f32",
    "vggt_attn_global_f32",
    "vggt_attn_global_batch",
    "vggt_attn_descriptor_batch",
)

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python feed_forward_view_b200/build.py`"
    )

lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_ATTN_ARGS = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
for _name in ("vggt_attn_frame", "vggt_attn_global", "vggt_attn_descriptor",
              "vggt_attn_global_noalloc"):
    getattr(lib, _name).argtypes = _ATTN_ARGS
    getattr(lib, _name).restype = _i
lib.vggt_kv_pool.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
lib.vggt_kv_pool.restype = _i
lib.vggt_qk_prologue.argtypes = [_p, _p, _p, _i, _i, _i, _p]
lib.vggt_qk_prologue.restype = _i
for _name in ("vggt_attn_core", "vggt_attn_core_online"):
    getattr(lib, _name).argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
    getattr(lib, _name).restype = _i
lib.vggt_kv_pool_tokens.argtypes = [_i, _i]
lib.vggt_kv_pool_tokens.restype = _i
lib.vggt_desc_cache_create.argtypes = [ctypes.POINTER(_p), _i, _i, _i, _i, _i]
lib.vggt_desc_cache_create.restype = _i
lib.vggt_desc_cache_destroy.argtypes = [_p]
lib.vggt_desc_cache_destroy.restype = _i
lib.vggt_desc_cache_frames.argtypes = [_p]
lib.vggt_desc_cache_frames.restype = _i
lib.vggt_desc_cache_reset.argtypes = [_p]
lib.vggt_desc_cache_reset.restype = _i
lib.vggt_attn_descriptor_chunk.argtypes = [_p, _p, _p, _p, _p, _p, _i, _p]
lib.vggt_attn_descriptor_chunk.restype = _i
lib.vggt_release_scratch.argtypes = []
lib.vggt_release_scratch.restype = _i
lib.vggt_scratch_pool_info.argtypes = [ctypes.POINTER(_i), ctypes.POINTER(ctypes.c_ulonglong)]
lib.vggt_scratch_pool_info.restype = _i
lib.vggt_get_device_status.argtypes = [_p]
lib.vggt_get_device_status.restype = _i
lib.vggt_status_string.argtypes = [_i]
lib.vggt_status_string.restype = ctypes.c_char_p
lib.vggt_set_wait_limit.argtypes = [ctypes.c_longlong]
lib.vggt_set_wait_limit.restype = ctypes.c_longlong
lib.vggt_debug_wait_timeout.argtypes = [_p]
lib.vggt_debug_wait_timeout.restype = _i


class FrameLayout(ctypes.Structure):
    """``vggt_frame_layout``: n_front special tokens, a grid_h x grid_w patch
    grid (row-major), n_back trailing tokens per frame."""
    _fields_ = [("n_front", _i), ("grid_h", _i), ("grid_w", _i), ("n_back", _i)]


_f32p = ctypes.POINTER(ctypes.c_float)


class QKNorm(ctypes.Structure):
    """``vggt_qk_norm``: host fp32 arrays of D values (or NULL) for the QK
    LayerNorm affine."""
    _fields_ = [("q_weight", _f32p), ("q_bias", _f32p), ("k_weight", _f32p), ("k_bias", _f32p)]


_LP = ctypes.POINTER(FrameLayout)
_NP = ctypes.POINTER(QKNorm)
for _name in ("vggt_attn_frame_ex", "vggt_attn_global_ex"):
    getattr(lib, _name).argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _NP, _p]
    getattr(lib, _name).restype = _i
lib.vggt_attn_descriptor_ex.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _LP, _NP, _p]
lib.vggt_attn_descriptor_ex.restype = _i
lib.vggt_kv_pool_ex.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _LP, _p]
lib.vggt_kv_pool_ex.restype = _i
lib.vggt_kv_pool_tokens_ex.argtypes = [_i, _i, _LP]
lib.vggt_kv_pool_tokens_ex.restype = _i
lib.vggt_qk_prologue_ex.argtypes = [_p, _p, _p, _i, _i, _i, _f32p, _f32p, _p]
lib.vggt_qk_prologue_ex.restype = _i
lib.vggt_descriptor_keys.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _LP, _f32p, _f32p, _p]
lib.vggt_descriptor_keys.restype = _i
for _name in ("vggt_attn_frame_f32", "vggt_attn_global_f32"):
    getattr(lib, _name).argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _NP, _i, _p]
    getattr(lib, _name).restype = _i
lib.vggt_attn_global_batch.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _NP, _p]
lib.vggt_attn_global_batch.restype = _i
lib.vggt_attn_descriptor_batch.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _LP, _NP, _p]
lib.vggt_attn_descriptor_batch.restype = _i
lib.vggt_attn_subset.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _NP, _p]
lib.vggt_attn_subset.restype = _i
lib.vggt_desc_cache_create_ex.argtypes = [ctypes.POINTER(_p), _i, _i, _i, _i, _i, _LP, _NP]
lib.vggt_desc_cache_create_ex.restype = _i


class VggtError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {vggt_status_string(status)} ({status})")


def vggt_status_string(status: int) -> str:
    return lib.vggt_status_string(int(status)).decode()


def _ptr(t, dtype, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise VggtError(rc, where)


def _attn(fn, q, k, v, pos, out, S, T, H, D, kv_down, stream):
    if out is None:
        out = torch.empty_like(q)
    rc = fn(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
            _ptr(pos, torch.float32, "pos"), _ptr(out, torch.bfloat16, "out"),
            int(S), int(T), int(H), int(D), int(kv_down), _stream(stream))
    _check(rc, fn.__name__)
    return out


def vggt_attn_frame(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, kv_down=0, stream=None):
    """Frame attention (see include/vggt_attn.h). q, k, v: [S*T, H, D] bf16,
    pos: [S*T, 2] fp32. Returns ``out``."""
    return _attn(lib.vggt_attn_frame, q, k, v, pos, out, S, T, H, D, kv_down, stream)


def vggt_attn_global(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, kv_down=0, stream=None):
    """Global attention over all S*T tokens. Returns ``out``."""
    return _attn(lib.vggt_attn_global, q, k, v, pos, out, S, T, H, D, kv_down, stream)


def vggt_attn_descriptor(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, kv_down=4,
                         stream=None):
    """Compressed-descriptor attention (pooled K/V). Returns ``out``."""
    return _attn(lib.vggt_attn_descriptor, q, k, v, pos, out, S, T, H, D, kv_down, stream)


def vggt_attn_global_noalloc(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, kv_down=0,
                             stream=None):
    """Global attention drawing its scratch from the library's fixed array
    instead of allocating (see include/vggt_attn.h). Returns ``out``."""
    return _attn(lib.vggt_attn_global_noalloc, q, k, v, pos, out, S, T, H, D, kv_down, stream)


def vggt_qk_prologue(x, pos, x_hat=None, N=None, H=16, D=64, stream=None):
    """LayerNorm + 2D RoPE of x [N, H, D]; returns x_hat [H, N, D] (head-major)."""
    N = x.shape[0] if N is None else N
    if x_hat is None:
        x_hat = torch.empty((H, N, D), dtype=torch.bfloat16, device=x.device)
    rc = lib.vggt_qk_prologue(_ptr(x, torch.bfloat16, "x"), _ptr(pos, torch.float32, "pos"),
                              _ptr(x_hat, torch.bfloat16, "x_hat"), int(N), int(H), int(D),
                              _stream(stream))
    _check(rc, "vggt_qk_prologue")
    return x_hat


def vggt_attn_core(q_hat, k_hat, v, out, n_seg, q_len, k_len, H=16, D=64, stream=None):
    """Attention on prologue outputs (head-major q_hat / k_hat). Returns ``out``."""
    rc = lib.vggt_attn_core(_ptr(q_hat, torch.bfloat16, "q_hat"), _ptr(k_hat, torch.bfloat16, "k_hat"),
                            _ptr(v, torch.bfloat16, "v"), _ptr(out, torch.bfloat16, "out"),
                            int(n_seg), int(q_len), int(k_len), int(H), int(D), _stream(stream))
    _check(rc, "vggt_attn_core")
    return out


def vggt_attn_core_online(q_hat, k_hat, v, out, n_seg, q_len, k_len, H=16, D=64, stream=None):
    """vggt_attn_core for any finite q_hat / k_hat (running row maximum).
    Returns ``out``."""
    rc = lib.vggt_attn_core_online(_ptr(q_hat, torch.bfloat16, "q_hat"), _ptr(k_hat, torch.bfloat16, "k_hat"),
                                   _ptr(v, torch.bfloat16, "v"), _ptr(out, torch.bfloat16, "out"),
                                   int(n_seg), int(q_len), int(k_len), int(H), int(D), _stream(stream))
    _check(rc, "vggt_attn_core_online")
    return out


def vggt_kv_pool_tokens(T: int, kv_down: int) -> int:
    return int(lib.vggt_kv_pool_tokens(int(T), int(kv_down)))


def vggt_kv_pool(k, v, pos, k_out=None, v_out=None, pos_out=None, S=None, T=None, H=16, D=64,
                 kv_down=4, stream=None):
    """Per-frame pooled descriptors. Returns ``(k_out, v_out, pos_out)``."""
    Tk = vggt_kv_pool_tokens(T, kv_down)
    if Tk < 0:
        raise VggtError(Tk, "vggt_kv_pool_tokens")
    if k_out is None:
        k_out = torch.empty((S * Tk, H, D), dtype=torch.bfloat16, device=k.device)
    if v_out is None:
        v_out = torch.empty((S * Tk, H, D), dtype=torch.bfloat16, device=k.device)
    if pos_out is None:
        pos_out = torch.empty((S * Tk, 2), dtype=torch.float32, device=k.device)
    rc = lib.vggt_kv_pool(_ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
                          _ptr(pos, torch.float32, "pos"), _ptr(k_out, torch.bfloat16, "k_out"),
                          _ptr(v_out, torch.bfloat16, "v_out"), _ptr(pos_out, torch.float32, "pos_out"),
                          int(S), int(T), int(H), int(D), int(kv_down), _stream(stream))
    _check(rc, "vggt_kv_pool")
    return k_out, v_out, pos_out


# ----------------------------------------------------------------- _ex calls


def _host_f32(x, name):
    """A host fp32 array for an affine argument (None stays NULL); returns
    (ctypes pointer, owner to keep alive during the call)."""
    if x is None:
        return None, None
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float32).contiguous()
        if x.numel() != 64:
            raise ValueError(f"{name} must hold 64 values")
        return ctypes.cast(x.data_ptr(), _f32p), x
    arr = (ctypes.c_float * 64)(*[float(t) for t in x])
    return ctypes.cast(arr, _f32p), arr


def _layout(layout):
    if layout is None:
        return None
    if isinstance(layout, FrameLayout):
        return ctypes.pointer(layout)
    return ctypes.pointer(FrameLayout(*[int(t) for t in layout]))


def _norm(ln):
    """``ln = (q_weight, q_bias, k_weight, k_bias)`` (entries may be None) ->
    (pointer to QKNorm or None, owners)."""
    if ln is None:
        return None, ()
    parts = [_host_f32(x, n) for x, n in zip(ln, ("q_weight", "q_bias", "k_weight", "k_bias"))]
    return ctypes.pointer(QKNorm(*[p for p, _ in parts])), tuple(o for _, o in parts)


def _attn_ex(fn, q, k, v, pos, out, S, T, H, D, ln, stream):
    if out is None:
        out = torch.empty_like(q)
    norm, keep = _norm(ln)
    rc = fn(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
            _ptr(pos, torch.float32, "pos"), _ptr(out, torch.bfloat16, "out"),
            int(S), int(T), int(H), int(D), norm, _stream(stream))
    del keep
    _check(rc, fn.__name__)
    return out


def vggt_attn_frame_ex(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, ln=None, stream=None):
    """Frame attention, any T, optional QK LayerNorm affine ``ln = (q_weight,
    q_bias, k_weight, k_bias)`` (host values; entries may be None)."""
    return _attn_ex(lib.vggt_attn_frame_ex, q, k, v, pos, out, S, T, H, D, ln, stream)


def vggt_attn_global_ex(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, ln=None, stream=None):
    """Global attention, any T, optional QK LayerNorm affine."""
    return _attn_ex(lib.vggt_attn_global_ex, q, k, v, pos, out, S, T, H, D, ln, stream)


def vggt_attn_descriptor_ex(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, kv_down=4, layout=None,
                            ln=None, stream=None):
    """Descriptor attention with a frame layout ``(n_front, grid_h, grid_w,
    n_back)`` and an optional QK LayerNorm affine."""
    if out is None:
        out = torch.empty_like(q)
    norm, keep = _norm(ln)
    rc = lib.vggt_attn_descriptor_ex(
        _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
        _ptr(pos, torch.float32, "pos"), _ptr(out, torch.bfloat16, "out"), int(S), int(T), int(H), int(D),
        int(kv_down), _layout(layout), norm, _stream(stream))
    del keep
    _check(rc, "vggt_attn_descriptor_ex")
    return out


def vggt_attn_subset(q, k, v, pos, out=None, S=None, T=None, n_skip_back=0, n_extra=0, H=16, D=64,
                     kind="global", ln=None, stream=None):
    """Attention over a token subset (VGGT-Omega layout): S frames of T tokens
    whose last ``n_skip_back`` take no part, then ``n_extra`` sequence tokens
    (global attention only). ``kind``: "frame" or "global". Rows that take no
    part are left as they are in ``out``. Returns ``out``."""
    if out is None:
        out = torch.zeros_like(q)
    norm, keep = _norm(ln)
    rc = lib.vggt_attn_subset(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                              _ptr(v, torch.bfloat16, "v"), _ptr(pos, torch.float32, "pos"),
                              _ptr(out, torch.bfloat16, "out"), int(S), int(T), int(n_skip_back), int(n_extra),
                              int(H), int(D), {"frame": 0, "global": 1}[kind], norm, _stream(stream))
    del keep
    _check(rc, "vggt_attn_subset")
    return out


def vggt_attn_global_batch(q, k, v, pos, out=None, B=None, S=None, T=None, H=16, D=64, ln=None, stream=None):
    """B scenes of S frames of T tokens (q, k, v [B*S*T, H, D]); each scene's
    global attention on its own. Returns ``out``."""
    if out is None:
        out = torch.empty_like(q)
    norm, keep = _norm(ln)
    rc = lib.vggt_attn_global_batch(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                                    _ptr(v, torch.bfloat16, "v"), _ptr(pos, torch.float32, "pos"),
                                    _ptr(out, torch.bfloat16, "out"), int(B), int(S), int(T), int(H), int(D), norm,
                                    _stream(stream))
    del keep
    _check(rc, "vggt_attn_global_batch")
    return out


def vggt_attn_descriptor_batch(q, k, v, pos, out=None, B=None, S=None, T=None, H=16, D=64, kv_down=4, layout=None,
                               ln=None, stream=None):
    """B scenes; each scene's descriptor attention over its own pooled frames."""
    if out is None:
        out = torch.empty_like(q)
    norm, keep = _norm(ln)
    rc = lib.vggt_attn_descriptor_batch(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                                        _ptr(v, torch.bfloat16, "v"), _ptr(pos, torch.float32, "pos"),
                                        _ptr(out, torch.bfloat16, "out"), int(B), int(S), int(T), int(H), int(D),
                                        int(kv_down), _layout(layout), norm, _stream(stream))
    del keep
    _check(rc, "vggt_attn_descriptor_batch")
    return out


def _attn_f32(fn, q, k, v, pos, out, S, T, H, D, ln, terms, stream):
    if out is None:
        out = torch.empty_like(q)
    norm, keep = _norm(ln)
    rc = fn(_ptr(q, torch.float32, "q"), _ptr(k, torch.float32, "k"), _ptr(v, torch.float32, "v"),
            _ptr(pos, torch.float32, "pos"), _ptr(out, torch.float32, "out"),
            int(S), int(T), int(H), int(D), norm, int(terms), _stream(stream))
    del keep
    _check(rc, fn.__name__)
    return out


def vggt_attn_frame_f32(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, ln=None, terms=2, stream=None):
    """Frame attention in the fp32 mode: fp32 q, k, v [S*T, H, D] in, fp32 out;
    operands carried as `terms` (2 or 3) bf16 terms."""
    return _attn_f32(lib.vggt_attn_frame_f32, q, k, v, pos, out, S, T, H, D, ln, terms, stream)


def vggt_attn_global_f32(q, k, v, pos, out=None, S=None, T=None, H=16, D=64, ln=None, terms=2, stream=None):
    """Global attention in the fp32 mode: fp32 q, k, v [S*T, H, D] in, fp32 out;
    operands carried as `terms` (2 or 3) bf16 terms."""
    return _attn_f32(lib.vggt_attn_global_f32, q, k, v, pos, out, S, T, H, D, ln, terms, stream)


def vggt_kv_pool_tokens_ex(T: int, kv_down: int, layout=None) -> int:
    return int(lib.vggt_kv_pool_tokens_ex(int(T), int(kv_down), _layout(layout)))


def _pooled_shapes(T, kv_down, layout, where):
    Tk = vggt_kv_pool_tokens_ex(T, kv_down, layout)
    if Tk < 0:
        raise VggtError(Tk, where)
    return Tk


def vggt_kv_pool_ex(k, v, pos, k_out=None, v_out=None, pos_out=None, S=None, T=None, H=16, D=64,
                    kv_down=4, layout=None, stream=None):
    """Pooled descriptors for a frame layout. Returns ``(k_out, v_out, pos_out)``."""
    Tk = _pooled_shapes(T, kv_down, layout, "vggt_kv_pool_tokens_ex")
    k_out = torch.empty((S * Tk, H, D), dtype=torch.bfloat16, device=k.device) if k_out is None else k_out
    v_out = torch.empty((S * Tk, H, D), dtype=torch.bfloat16, device=k.device) if v_out is None else v_out
    pos_out = torch.empty((S * Tk, 2), dtype=torch.float32, device=k.device) if pos_out is None else pos_out
    rc = lib.vggt_kv_pool_ex(_ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
                             _ptr(pos, torch.float32, "pos"), _ptr(k_out, torch.bfloat16, "k_out"),
                             _ptr(v_out, torch.bfloat16, "v_out"), _ptr(pos_out, torch.float32, "pos_out"),
                             int(S), int(T), int(H), int(D), int(kv_down), _layout(layout), _stream(stream))
    _check(rc, "vggt_kv_pool_ex")
    return k_out, v_out, pos_out


def vggt_qk_prologue_ex(x, pos, x_hat=None, N=None, H=16, D=64, ln_weight=None, ln_bias=None, stream=None):
    """LayerNorm (+ optional host affine) + 2D RoPE; returns x_hat [H, N, D]."""
    N = x.shape[0] if N is None else N
    if x_hat is None:
        x_hat = torch.empty((H, N, D), dtype=torch.bfloat16, device=x.device)
    w, kw = _host_f32(ln_weight, "ln_weight")
    b, kb = _host_f32(ln_bias, "ln_bias")
    rc = lib.vggt_qk_prologue_ex(_ptr(x, torch.bfloat16, "x"), _ptr(pos, torch.float32, "pos"),
                                 _ptr(x_hat, torch.bfloat16, "x_hat"), int(N), int(H), int(D), w, b,
                                 _stream(stream))
    del kw, kb
    _check(rc, "vggt_qk_prologue_ex")
    return x_hat


def vggt_descriptor_keys(k, v, pos, k_hat=None, v_out=None, pos_out=None, S=None, T=None, H=16, D=64,
                         kv_down=4, layout=None, ln_weight=None, ln_bias=None, stream=None):
    """Pooling fused with the key prologue. Returns ``(k_hat [H, S*T_k, D],
    v_out [S*T_k, H, D], pos_out [S*T_k, 2])``."""
    Tk = _pooled_shapes(T, kv_down, layout, "vggt_kv_pool_tokens_ex")
    k_hat = torch.empty((H, S * Tk, D), dtype=torch.bfloat16, device=k.device) if k_hat is None else k_hat
    v_out = torch.empty((S * Tk, H, D), dtype=torch.bfloat16, device=k.device) if v_out is None else v_out
    pos_out = torch.empty((S * Tk, 2), dtype=torch.float32, device=k.device) if pos_out is None else pos_out
    w, kw = _host_f32(ln_weight, "ln_weight")
    b, kb = _host_f32(ln_bias, "ln_bias")
    rc = lib.vggt_descriptor_keys(_ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
                                  _ptr(pos, torch.float32, "pos"), _ptr(k_hat, torch.bfloat16, "k_hat"),
                                  _ptr(v_out, torch.bfloat16, "v_out"), _ptr(pos_out, torch.float32, "pos_out"),
                                  int(S), int(T), int(H), int(D), int(kv_down), _layout(layout), w, b,
                                  _stream(stream))
    del kw, kb
    _check(rc, "vggt_descriptor_keys")
    return k_hat, v_out, pos_out


def vggt_get_device_status(stream=None) -> int:
    return int(lib.vggt_get_device_status(_stream(stream)))


class DescCache:
    """A streaming descriptor cache (see include/vggt_attn.h): holds the
    normalised pooled keys, values and positions of the frames seen so far
    of one sequence, on the device that was current at creation."""

    def __init__(self, max_frames: int, T: int, H: int = 16, D: int = 64, kv_down: int = 4,
                 layout=None, ln=None):
        """``layout = (n_front, grid_h, grid_w, n_back)`` and ``ln = (q_weight,
        q_bias, k_weight, k_bias)`` (host values) select the _ex form."""
        if layout is None and ln is None:
            self._h = vggt_desc_cache_create(max_frames, T, H, D, kv_down)
        else:
            self._h = vggt_desc_cache_create_ex(max_frames, T, H, D, kv_down, layout, ln)
        self.T, self.H, self.D = int(T), int(H), int(D)

    @property
    def frames(self) -> int:
        n = lib.vggt_desc_cache_frames(self._h)
        _check(min(n, 0), "vggt_desc_cache_frames")
        return int(n)

    def reset(self) -> None:
        _check(lib.vggt_desc_cache_reset(self._h), "vggt_desc_cache_reset")

    def attend(self, q, k, v, pos, out=None, C=None, stream=None):
        """One chunk of C frames: q, k, v [C*T, H, D] bf16, pos [C*T, 2] fp32.
        Appends the chunk's descriptors and returns ``out`` (the chunk's
        tokens attending to every cached descriptor)."""
        C = q.shape[0] // self.T if C is None else C
        if out is None:
            out = torch.empty_like(q)
        return vggt_attn_descriptor_chunk(self._h, q, k, v, pos, out, C, stream)

    def close(self) -> None:
        if self._h:
            vggt_desc_cache_destroy(self._h)
            self._h = _p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def vggt_desc_cache_create(max_frames: int, T: int, H: int = 16, D: int = 64, kv_down: int = 4):
    """Returns an opaque cache handle (see :class:`DescCache` for the managed form)."""
    h = _p()
    _check(lib.vggt_desc_cache_create(ctypes.byref(h), int(max_frames), int(T), int(H), int(D), int(kv_down)),
           "vggt_desc_cache_create")
    return h


def vggt_desc_cache_create_ex(max_frames: int, T: int, H: int = 16, D: int = 64, kv_down: int = 4,
                              layout=None, ln=None):
    """Cache handle with a frame layout and a QK LayerNorm affine (either may be None)."""
    h = _p()
    norm, keep = _norm(ln)
    rc = lib.vggt_desc_cache_create_ex(ctypes.byref(h), int(max_frames), int(T), int(H), int(D), int(kv_down),
                                       _layout(layout), norm)
    del keep
    _check(rc, "vggt_desc_cache_create_ex")
    return h


def vggt_desc_cache_destroy(h) -> None:
    _check(lib.vggt_desc_cache_destroy(h), "vggt_desc_cache_destroy")


def vggt_desc_cache_frames(h) -> int:
    n = lib.vggt_desc_cache_frames(h)
    _check(min(n, 0), "vggt_desc_cache_frames")
    return int(n)


def vggt_desc_cache_reset(h) -> None:
    _check(lib.vggt_desc_cache_reset(h), "vggt_desc_cache_reset")


def vggt_attn_descriptor_chunk(h, q, k, v, pos, out, C, stream=None):
    """One chunk of C frames through cache ``h``; returns ``out``."""
    rc = lib.vggt_attn_descriptor_chunk(h, _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                                        _ptr(v, torch.bfloat16, "v"), _ptr(pos, torch.float32, "pos"),
                                        _ptr(out, torch.bfloat16, "out"), int(C), _stream(stream))
    _check(rc, "vggt_attn_descriptor_chunk")
    return out


def vggt_release_scratch() -> None:
    """Return the library's unused scratch memory on the current device."""
    _check(lib.vggt_release_scratch(), "vggt_release_scratch")


def vggt_scratch_pool_info() -> tuple[bool, int]:
    """(exists, reserved bytes) of the library's scratch pool on the current
    device."""
    exists = ctypes.c_int(0)
    reserved = ctypes.c_ulonglong(0)
    _check(lib.vggt_scratch_pool_info(ctypes.byref(exists), ctypes.byref(reserved)), "vggt_scratch_pool_info")
    return bool(exists.value), int(reserved.value)


def vggt_set_wait_limit(cycles: int) -> int:
    return int(lib.vggt_set_wait_limit(int(cycles)))


def vggt_debug_wait_timeout(stream=None) -> None:
    _check(lib.vggt_debug_wait_timeout(_stream(stream)), "vggt_debug_wait_timeout")
