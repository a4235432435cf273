"""Python binding of liblla -- Looped Latent Attention decode/encode on B200 (sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``liblla.so`` behind the C ABI declared in ``include/lla.h``.  Tensors are
passed as raw device pointers (``tensor.data_ptr()``) together with the current
torch CUDA stream; torch is used for device memory and streams, nothing else.
There is no CPU path: importing this package fails loudly when the compiled
library is missing.

Names follow the C ABI: ``cache_bytes``, ``slot_layout``, ``codec_bias``,
``encode``, ``decode_attn``, ``decode_workspace_bytes``, ``decode_num_splits``,
``decode_attn_static``, ``decode_attn_hybrid``, ``decode_hybrid_workspace_bytes``, ``decode_attn_rope``,
``codec_residual``, ``codec_fit``, ``codec_fit_workspace_bytes``, ``decode_attn_decoupled``, ``decode_decoupled_workspace_bytes``,
``status_fetch``, ``status_string``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblla.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first "
        "(python decode_attention_12_b200/_build.py, or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

LLA_OK = 0
LLA_ERR_INVALID = -1
LLA_ERR_UNSUPPORTED = -2
LLA_ERR_MISALIGNED = -3
LLA_ERR_WORKSPACE = -4
LLA_ERR_CUDA = -5
LLA_ERR_DEVICE_TIMEOUT = -6
LLA_ERR_NO_CONVERGENCE = -7
PER_HEAD, FOLD_2D = 0, 1
F32, BF16 = 0, 1
ABSORB, RECONSTRUCT = 0, 1
ROPE_HALF, ROPE_INTERLEAVED = 0, 1

EXPORTED = ("lla_cache_bytes", "lla_slot_layout", "lla_codec_bias", "lla_encode",
            "lla_decode_attn", "lla_decode_workspace_bytes", "lla_decode_num_splits",
            "lla_decode_attn_static", "lla_decode_attn_hybrid", "lla_decode_hybrid_workspace_bytes",
            "lla_decode_attn_rope", "lla_codec_residual", "lla_decode_attn_decoupled", "lla_decode_attn_timed",
            "lla_codec_fit", "lla_codec_fit_workspace_bytes", "lla_selftest_wait_timeout",
            "lla_decode_decoupled_workspace_bytes",
            "lla_status_fetch", "lla_status_fetch_static", "lla_status_string")
STATIC_SCRATCH_BYTES = 8 << 20


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "L", "H", "d_head", "r_k", "r_v", "fold", "dtype",
                                              "out_dtype")]


class Codec(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_down_k", "W_down_v", "bias_k", "bias_v",
                                               "W_up_k", "W_up_v", "mu_k", "mu_v")]


class Cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("slots", ctypes.c_int64)]


class Window(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("len", ctypes.c_void_p),
                ("w_max", ctypes.c_int32), ("seqs", ctypes.c_int32)]


class Rope(ctypes.Structure):
    _fields_ = [("q_pos", ctypes.c_void_p), ("base", ctypes.c_float), ("style", ctypes.c_int32)]


class Decoupled(ctypes.Structure):
    _fields_ = [("k_rope", ctypes.c_void_p), ("q_rope", ctypes.c_void_p), ("d_rope", ctypes.c_int32)]


_i32, _i64, _u64p = ctypes.c_int32, ctypes.c_int64, ctypes.POINTER(ctypes.c_uint64)
_vp, _sz = ctypes.c_void_p, ctypes.c_size_t
_P = ctypes.POINTER
_lib.lla_cache_bytes.argtypes = [_P(Dims), _P(_i32), _i32, _u64p, _u64p, _u64p, _u64p]
_lib.lla_slot_layout.argtypes = [_P(_i32), _i32, _i64, _P(_i64), _P(_i64)]
_lib.lla_codec_bias.argtypes = [_P(Dims), _P(Codec), _vp, _vp, _vp]
_lib.lla_encode.argtypes = [_P(Dims), _i32, _i32, _vp, _vp, _i64, _vp, _P(Codec), _P(Cache), _vp]
_lib.lla_decode_attn.argtypes = [_P(Dims), _i32, _i32, _i32, _vp, _P(Cache), _vp, _vp, _i32, _i32,
                                 _P(Codec), ctypes.c_float, _i32, _i32, _vp, _vp, _vp, _sz, _vp]
_lib.lla_decode_attn_static.argtypes = [_P(Dims), _i32, _i32, _i32, _vp, _P(Cache), _vp, _vp, _i32,
                                        _i32, _P(Codec), ctypes.c_float, _i32, _i32, _vp, _vp, _vp]
_lib.lla_decode_attn_hybrid.argtypes = [_P(Dims), _i32, _i32, _i32, _vp, _P(Cache), _vp, _vp, _i32,
                                        _i32, _P(Codec), _P(Window), ctypes.c_float, _i32, _i32, _vp,
                                        _vp, _vp, _sz, _vp]
_lib.lla_codec_fit.argtypes = [_P(Dims), _i32, _i32, _vp, _vp, _i64, _P(Codec), _vp, _vp, _vp, _sz, _vp]
_lib.lla_codec_fit_workspace_bytes.argtypes = [_P(Dims), _i32, _i64]
_lib.lla_codec_fit_workspace_bytes.restype = _sz
_lib.lla_decode_attn_timed.argtypes = [_P(Dims), _i32, _i32, _i32, _vp, _P(Cache), _vp, _vp, _i32, _i32,
                                       _P(Codec), ctypes.c_float, _i32, _i32, _vp, _vp, _vp, _sz, _vp, _vp, _vp]
_lib.lla_decode_attn_decoupled.argtypes = [_P(Dims), _i32, _i32, _i32, _vp, _P(Cache), _vp, _vp, _i32, _i32,
                                           _P(Codec), _P(Decoupled), _P(Rope), ctypes.c_float, _i32, _vp, _vp,
                                           _vp, _sz, _vp]
_lib.lla_decode_decoupled_workspace_bytes.argtypes = [_P(Dims), _i32, _i32, _i32, _i32, _i32]
_lib.lla_decode_decoupled_workspace_bytes.restype = _sz
_lib.lla_codec_residual.argtypes = [_P(Dims), _i32, _i32, _vp, _vp, _i64, _P(Codec), _vp, _vp, _vp, _vp, _vp]
_lib.lla_decode_attn_rope.argtypes = [_P(Dims), _i32, _i32, _i32, _vp, _P(Cache), _vp, _vp, _i32, _i32,
                                      _P(Codec), _P(Rope), ctypes.c_float, _i32, _vp, _vp, _vp, _sz, _vp]
_lib.lla_decode_hybrid_workspace_bytes.argtypes = [_P(Dims), _i32, _i32, _i32, _i32, _i32]
_lib.lla_decode_hybrid_workspace_bytes.restype = _sz
_lib.lla_decode_workspace_bytes.argtypes = [_P(Dims), _i32, _i32, _i32, _i32, _i32]
_lib.lla_decode_workspace_bytes.restype = _sz
_lib.lla_decode_num_splits.argtypes = [_P(Dims), _i32, _i32, _i32, _i32, _i32]
_lib.lla_status_fetch.argtypes = [_vp, _vp, _P(_i32)]
_lib.lla_status_fetch_static.argtypes = [_vp, _P(_i32)]
_lib.lla_selftest_wait_timeout.argtypes = [_vp, _vp]
_lib.lla_selftest_wait_timeout.restype = ctypes.c_int
_lib.lla_status_string.argtypes = [ctypes.c_int]
_lib.lla_status_string.restype = ctypes.c_char_p
for _n in ("lla_cache_bytes", "lla_slot_layout", "lla_codec_bias", "lla_encode", "lla_decode_attn",
           "lla_decode_attn_static", "lla_decode_attn_hybrid", "lla_decode_attn_rope", "lla_codec_residual",
           "lla_decode_attn_decoupled", "lla_decode_attn_timed", "lla_codec_fit",
           "lla_decode_num_splits",
           "lla_status_fetch", "lla_status_fetch_static"):
    getattr(_lib, _n).restype = ctypes.c_int


class LLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} ({code})")
        self.code = code


def status_string(code: int) -> str:
    return _lib.lla_status_string(code).decode()


def _check(rc: int, where: str) -> int:
    if rc < 0:
        raise LLAError(rc, where)
    return rc


def make_dims(T, L, H, d_head, r_k, r_v, fold=PER_HEAD, dtype=BF16, out_dtype=F32) -> Dims:
    return Dims(T, L, H, d_head, r_k, r_v, int(fold), int(dtype), int(out_dtype))


def _ptr(t) -> Optional[int]:
    """Device address of a buffer: None, a raw address, or a tensor.  The library takes
    dense row-major buffers (no strides cross the ABI), so a strided view is refused
    rather than read as if it were dense."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError(f"liblla takes dense row-major buffers; got a strided view of shape "
                         f"{tuple(t.shape)} with strides {tuple(t.stride())} (call .contiguous())")
    return t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def make_codec(W_down_k=None, W_down_v=None, bias_k=None, bias_v=None, W_up_k=None, W_up_v=None,
               mu_k=None, mu_v=None) -> Codec:
    return Codec(*[_ptr(t) for t in (W_down_k, W_down_v, bias_k, bias_v, W_up_k, W_up_v, mu_k, mu_v)])


def make_cache(k, v, slots: int) -> Cache:
    return Cache(_ptr(k), _ptr(v), int(slots))


def make_window(k, v, win_len, w_max: int, seqs: int) -> Window:
    """Exact window planes k, v [L][seqs][H][T][w_max][d] and rows in use win_len [seqs]."""
    return Window(_ptr(k), _ptr(v), _ptr(win_len), int(w_max), int(seqs))


# ---- a7 -------------------------------------------------------------------------------
def cache_bytes(dims: Dims, ctx_lens: Sequence[int]):
    """(latent_bytes, uncompressed_bytes, rho_num, rho_den) -- exact integers."""
    n = len(ctx_lens)
    arr = (_i32 * max(n, 1))(*[int(v) for v in ctx_lens])
    out = [ctypes.c_uint64(0) for _ in range(4)]
    _check(_lib.lla_cache_bytes(ctypes.byref(dims), arr, n, *[ctypes.byref(o) for o in out]),
           "lla_cache_bytes")
    return tuple(int(o.value) for o in out)


def slot_layout(ctx_lens: Sequence[int], gap: int = 0):
    """(seq_start list, total_slots) -- exclusive prefix sum with an optional gap."""
    n = len(ctx_lens)
    arr = (_i32 * max(n, 1))(*[int(v) for v in ctx_lens])
    starts = (_i64 * max(n, 1))()
    total = _i64(0)
    _check(_lib.lla_slot_layout(arr, n, int(gap), starts, ctypes.byref(total)), "lla_slot_layout")
    return [int(starts[i]) for i in range(n)], int(total.value)


# ---- a6 -------------------------------------------------------------------------------
def codec_bias(dims: Dims, codec: Codec, bias_k, bias_v, stream=None) -> None:
    _check(_lib.lla_codec_bias(ctypes.byref(dims), ctypes.byref(codec), _ptr(bias_k), _ptr(bias_v),
                               _stream(stream)), "lla_codec_bias")


def encode(dims: Dims, layer0: int, n_layers: int, x_k, x_v, n_tok: int, slot_idx, codec: Codec,
           cache: Cache, stream=None) -> None:
    _check(_lib.lla_encode(ctypes.byref(dims), layer0, n_layers, _ptr(x_k), _ptr(x_v), int(n_tok),
                           _ptr(slot_idx), ctypes.byref(codec), ctypes.byref(cache), _stream(stream)),
           "lla_encode")


def codec_fit_workspace_bytes(dims: Dims, n_layers: int, n_cal: int) -> int:
    n = _lib.lla_codec_fit_workspace_bytes(ctypes.byref(dims), n_layers, n_cal)
    if n == 0:
        raise LLAError(LLA_ERR_INVALID, "lla_codec_fit_workspace_bytes")
    return int(n)


def codec_fit(dims: Dims, layer0: int, n_layers: int, x_k, x_v, n_cal: int, codec: Codec, workspace,
              ws_bytes: Optional[int] = None, sigma_k=None, sigma_v=None, stream=None) -> None:
    """SVD initialisation of the codec on the GPU: writes codec.W_down_{k,v}, W_up_{k,v}, mu_{k,v}."""
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.lla_codec_fit(ctypes.byref(dims), layer0, n_layers, _ptr(x_k), _ptr(x_v), n_cal,
                              ctypes.byref(codec), _ptr(sigma_k), _ptr(sigma_v), _ptr(workspace), int(ws_bytes),
                              _stream(stream)),
           "lla_codec_fit")


def codec_residual(dims: Dims, layer0: int, n_layers: int, x_k, x_v, n_tok: int, codec: Codec,
                   err_k, norm_k, err_v, norm_v, stream=None) -> None:
    """Per-token reconstruction residual ||x - x_hat|| and norm ||x|| per (layer, token, head')."""
    _check(_lib.lla_codec_residual(ctypes.byref(dims), layer0, n_layers, _ptr(x_k), _ptr(x_v), n_tok,
                                   ctypes.byref(codec), _ptr(err_k), _ptr(norm_k), _ptr(err_v),
                                   _ptr(norm_v), _stream(stream)),
           "lla_codec_residual")


# ---- a1-a5, a8 ------------------------------------------------------------------------------
def decode_num_splits(dims: Dims, B: int, Tq: int, max_ctx: int, variant: int = ABSORB,
                      num_splits: int = 0) -> int:
    return _check(_lib.lla_decode_num_splits(ctypes.byref(dims), B, Tq, max_ctx, variant, num_splits),
                  "lla_decode_num_splits")


def decode_workspace_bytes(dims: Dims, B: int, Tq: int, max_ctx: int, variant: int = ABSORB,
                           num_splits: int = 0) -> int:
    n = _lib.lla_decode_workspace_bytes(ctypes.byref(dims), B, Tq, max_ctx, variant, num_splits)
    if n == 0:
        raise LLAError(LLA_ERR_INVALID, "lla_decode_workspace_bytes")
    return int(n)


def decode_attn(dims: Dims, layer: int, t0: int, Tq: int, q, cache: Cache, seq_start, ctx_lens,
                B: int, max_ctx: int, codec: Codec, softmax_scale: float, out, lse=None,
                workspace=None, ws_bytes: Optional[int] = None, variant: int = ABSORB,
                num_splits: int = 0, stream=None) -> None:
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.lla_decode_attn(ctypes.byref(dims), layer, t0, Tq, _ptr(q), ctypes.byref(cache),
                                _ptr(seq_start), _ptr(ctx_lens), B, max_ctx, ctypes.byref(codec),
                                float(softmax_scale), variant, num_splits, _ptr(out), _ptr(lse),
                                _ptr(workspace), int(ws_bytes), _stream(stream)),
           "lla_decode_attn")


def decode_hybrid_workspace_bytes(dims: Dims, B: int, Tq: int, max_ctx: int, variant: int = ABSORB,
                                  num_splits: int = 0) -> int:
    n = _lib.lla_decode_hybrid_workspace_bytes(ctypes.byref(dims), B, Tq, max_ctx, variant, num_splits)
    if n == 0:
        raise LLAError(LLA_ERR_INVALID, "lla_decode_hybrid_workspace_bytes")
    return int(n)


def decode_attn_hybrid(dims: Dims, layer: int, t0: int, Tq: int, q, cache: Cache, seq_start, ctx_lens,
                       B: int, max_ctx: int, codec: Codec, window: Window, softmax_scale: float, out,
                       lse=None, workspace=None, ws_bytes: Optional[int] = None, variant: int = ABSORB,
                       num_splits: int = 0, stream=None) -> None:
    """Hybrid latent attention: one softmax over the latent tokens and the exact window rows."""
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.lla_decode_attn_hybrid(ctypes.byref(dims), layer, t0, Tq, _ptr(q), ctypes.byref(cache),
                                       _ptr(seq_start), _ptr(ctx_lens), B, max_ctx, ctypes.byref(codec),
                                       ctypes.byref(window), float(softmax_scale), variant, num_splits,
                                       _ptr(out), _ptr(lse), _ptr(workspace), int(ws_bytes),
                                       _stream(stream)),
           "lla_decode_attn_hybrid")


def make_rope(q_pos, base: float = 10000.0, style: int = ROPE_HALF) -> Rope:
    """Query positions q_pos int32 [B] (device), rotary base and pairing style."""
    return Rope(_ptr(q_pos), float(base), int(style))


def decode_attn_rope(dims: Dims, layer: int, t0: int, Tq: int, q, cache: Cache, seq_start, ctx_lens,
                     B: int, max_ctx: int, codec: Codec, rope: Rope, softmax_scale: float, out, lse=None,
                     workspace=None, ws_bytes: Optional[int] = None, num_splits: int = 0,
                     stream=None) -> None:
    """Faithful read: rebuilt keys and the query rotated at their positions (reconstruct form)."""
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.lla_decode_attn_rope(ctypes.byref(dims), layer, t0, Tq, _ptr(q), ctypes.byref(cache),
                                     _ptr(seq_start), _ptr(ctx_lens), B, max_ctx, ctypes.byref(codec),
                                     ctypes.byref(rope), float(softmax_scale), num_splits, _ptr(out),
                                     _ptr(lse), _ptr(workspace), int(ws_bytes), _stream(stream)),
           "lla_decode_attn_rope")


def decode_decoupled_workspace_bytes(dims: Dims, B: int, Tq: int, max_ctx: int, d_rope: int,
                                     num_splits: int = 0) -> int:
    n = _lib.lla_decode_decoupled_workspace_bytes(ctypes.byref(dims), B, Tq, max_ctx, d_rope, num_splits)
    if n == 0:
        raise LLAError(LLA_ERR_INVALID, "lla_decode_decoupled_workspace_bytes")
    return int(n)


def decode_attn_decoupled(dims: Dims, layer: int, t0: int, Tq: int, q, cache: Cache, seq_start, ctx_lens,
                          B: int, max_ctx: int, codec: Codec, k_rope, q_rope, d_rope: int, rope: Rope,
                          softmax_scale: float, out, lse=None, workspace=None, ws_bytes: Optional[int] = None,
                          num_splits: int = 0, stream=None) -> None:
    """Absorbed read with a decoupled rotary sub-key plane k_rope [L][H][slots][d_rope] (stored
    rotated) and the queries' rotary parts q_rope [B][Tq][H][d_rope] (rotated at rope.q_pos)."""
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    dec = Decoupled(_ptr(k_rope), _ptr(q_rope), int(d_rope))
    _check(_lib.lla_decode_attn_decoupled(ctypes.byref(dims), layer, t0, Tq, _ptr(q), ctypes.byref(cache),
                                          _ptr(seq_start), _ptr(ctx_lens), B, max_ctx, ctypes.byref(codec),
                                          ctypes.byref(dec), ctypes.byref(rope), float(softmax_scale),
                                          num_splits, _ptr(out), _ptr(lse), _ptr(workspace), int(ws_bytes),
                                          _stream(stream)),
           "lla_decode_attn_decoupled")


def decode_attn_timed(dims: Dims, layer: int, t0: int, Tq: int, q, cache: Cache, seq_start, ctx_lens,
                      B: int, max_ctx: int, codec: Codec, softmax_scale: float, out, lse, workspace,
                      ws_bytes: int, ev_start, ev_end, variant: int = ABSORB, num_splits: int = 0,
                      stream=None) -> None:
    """lla_decode_attn with CUDA events around the latent-streaming grid alone (timing aid).
    ev_start / ev_end: torch.cuda.Event(enable_timing=True), already created (recorded once)."""
    _check(_lib.lla_decode_attn_timed(ctypes.byref(dims), layer, t0, Tq, _ptr(q), ctypes.byref(cache),
                                      _ptr(seq_start), _ptr(ctx_lens), B, max_ctx, ctypes.byref(codec),
                                      float(softmax_scale), variant, num_splits, _ptr(out), _ptr(lse),
                                      _ptr(workspace), int(ws_bytes), _stream(stream), ev_start.cuda_event,
                                      ev_end.cuda_event),
           "lla_decode_attn_timed")


def decode_attn_static(dims: Dims, layer: int, t0: int, Tq: int, q, cache: Cache, seq_start,
                       ctx_lens, B: int, max_ctx: int, codec: Codec, softmax_scale: float, out,
                       lse=None, variant: int = ABSORB, num_splits: int = 0, stream=None) -> None:
    """lla_decode_attn without a workspace argument: for callers that cannot allocate
    device memory.  The scratch is an 8 MiB array inside the library, shared by every
    call (serialise calls that could overlap on the GPU).  Device-side errors land in
    the array's status word: read them with :func:`status_fetch_static`."""
    _check(_lib.lla_decode_attn_static(ctypes.byref(dims), layer, t0, Tq, _ptr(q), ctypes.byref(cache),
                                       _ptr(seq_start), _ptr(ctx_lens), B, max_ctx,
                                       ctypes.byref(codec), float(softmax_scale), variant, num_splits,
                                       _ptr(out), _ptr(lse), _stream(stream)),
           "lla_decode_attn_static")


def selftest_wait_timeout(workspace, stream=None) -> None:
    """Run the bounded-wait self-test: a wait that nothing completes gives up (about 2 s)
    and records LLA_ERR_DEVICE_TIMEOUT in the workspace's status word."""
    _check(_lib.lla_selftest_wait_timeout(_ptr(workspace), _stream(stream)), "lla_selftest_wait_timeout")


def status_fetch(workspace, stream=None) -> int:
    v = _i32(0)
    _check(_lib.lla_status_fetch(_ptr(workspace), _stream(stream), ctypes.byref(v)), "lla_status_fetch")
    return int(v.value)


def status_fetch_static(stream=None) -> int:
    """Read and clear the status word of decode_attn_static's library-owned array on the
    current device (synchronises the stream)."""
    v = _i32(0)
    _check(_lib.lla_status_fetch_static(_stream(stream), ctypes.byref(v)), "lla_status_fetch_static")
    return int(v.value)
