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
    "vggt_attn_global_noalloc",
    "vggt_get_device_status",
    "vggt_release_scratch",
    "vggt_desc_cache_create",
    "vggt_desc_cache_destroy",
    "vggt_desc_cache_frames",
    "vggt_desc_cache_reset",
    "vggt_attn_descriptor_chunk",
    "vggt_status_string",
    "vggt_set_wait_limit",
    "vggt_debug_wait_timeout",
    "EXPORTED_SYMBOLS",
]

# every symbol include/vggt_attn.h declares
EXPORTED_SYMBOLS = (
    "vggt_qk_prologue",
    "vggt_attn_core",
    "vggt_attn_global_noalloc",
    "vggt_attn_frame",
    "vggt_attn_global",
    "vggt_attn_descriptor",
    "vggt_kv_pool",
    "vggt_kv_pool_tokens",
    "vggt_get_device_status",
    "vggt_release_scratch",
    "vggt_desc_cache_create",
    "vggt_desc_cache_destroy",
    "vggt_desc_cache_frames",
    "vggt_desc_cache_reset",
    "vggt_attn_descriptor_chunk",
    "vggt_status_string",
    "vggt_set_wait_limit",
    "vggt_debug_wait_timeout",
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
lib.vggt_attn_core.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
lib.vggt_attn_core.restype = _i
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
lib.vggt_get_device_status.argtypes = [_p]
lib.vggt_get_device_status.restype = _i
lib.vggt_status_string.argtypes = [_i]
lib.vggt_status_string.restype = ctypes.c_char_p
lib.vggt_set_wait_limit.argtypes = [ctypes.c_longlong]
lib.vggt_set_wait_limit.restype = ctypes.c_longlong
lib.vggt_debug_wait_timeout.argtypes = [_p]
lib.vggt_debug_wait_timeout.restype = _i


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


def vggt_get_device_status(stream=None) -> int:
    return int(lib.vggt_get_device_status(_stream(stream)))


class DescCache:
    """A streaming descriptor cache (see include/vggt_attn.h): holds the
    normalised pooled keys, values and positions of the frames seen so far
    of one sequence, on the device that was current at creation."""

    def __init__(self, max_frames: int, T: int, H: int = 16, D: int = 64, kv_down: int = 4):
        self._h = _p()
        _check(lib.vggt_desc_cache_create(ctypes.byref(self._h), int(max_frames), int(T), int(H),
                                          int(D), int(kv_down)), "vggt_desc_cache_create")
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
        rc = lib.vggt_attn_descriptor_chunk(self._h, _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                                            _ptr(v, torch.bfloat16, "v"), _ptr(pos, torch.float32, "pos"),
                                            _ptr(out, torch.bfloat16, "out"), int(C), _stream(stream))
        _check(rc, "vggt_attn_descriptor_chunk")
        return out

    def close(self) -> None:
        if self._h:
            _check(lib.vggt_desc_cache_destroy(self._h), "vggt_desc_cache_destroy")
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


def vggt_release_scratch() -> None:
    """Return the library's unused scratch memory on the current device."""
    _check(lib.vggt_release_scratch(), "vggt_release_scratch")


def vggt_set_wait_limit(cycles: int) -> int:
    return int(lib.vggt_set_wait_limit(int(cycles)))


def vggt_debug_wait_timeout(stream=None) -> None:
    _check(lib.vggt_debug_wait_timeout(_stream(stream)), "vggt_debug_wait_timeout")
