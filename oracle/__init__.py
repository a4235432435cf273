"""Plain fp64 CPU oracle for Looped Latent Attention (LLA) -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does: it shares no code with this oracle, and the
oracle imports nothing from it.

The arithmetic lives in ``lla_oracle.c`` (plain loops, double precision, one
problem instance per call, each routine citing the passage it follows).  This
module only marshals numpy arrays into it and loops over independent
(sequence, head, loop) problem instances, optionally on a thread pool (ctypes
releases the GIL during the call, so the pool really runs in parallel).

Citations use the page title and section:
  "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers",
  Pith review page, "What carries the argument" (Eqs. 2-4) -- encode,
  reconstruction, exact ratio; Pith verdict record, desk-editor letter --
  absorbed-attention variant; arXiv abstract -- LLA-2D.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lla_oracle.c")
_LIB = os.path.join(_HERE, "liblla_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile lla_oracle.c into liblla_oracle.so (plain -O2, no fast-math)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                                   "-fno-fast-math", "-ffp-contract=off",
                                   _SRC, "-o", tmp, "-lm"])
            os.replace(tmp, _LIB)
    return _LIB


def configure(lib):
    """Declare the C signatures on a loaded oracle library (also used for test mutants)."""
    i64, i32 = ctypes.c_int64, ctypes.c_int
    u64p = ctypes.POINTER(ctypes.c_uint64)
    lib.oracle_cache_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i64,
                                       u64p, u64p, u64p, u64p]
    lib.oracle_cache_bytes.restype = i32
    lib.oracle_encode.argtypes = [i64, i32, i32, _dp, _dp, _dp, _dp]
    lib.oracle_encode.restype = None
    lib.oracle_reconstruct.argtypes = [i64, i32, i32, _dp, _dp, _dp, _dp]
    lib.oracle_reconstruct.restype = None
    for name in ("oracle_attend_reconstruct", "oracle_attend_absorb"):
        f = getattr(lib, name)
        f.argtypes = [i64, i32, i32, i32, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                      ctypes.c_double, _dp, _dp]
        f.restype = i32
    lib.oracle_attend_hybrid.argtypes = [i64, i64, i32, i32, i32, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                         _dp, ctypes.c_double, _dp, _dp]
    lib.oracle_attend_hybrid.restype = i32
    lib.oracle_attend_rope.argtypes = [i64, i32, i32, i32, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                       ctypes.c_double, i32, ctypes.c_double, ctypes.c_double,
                                       ctypes.c_double, _dp, _dp]
    lib.oracle_attend_rope.restype = i32
    lib.oracle_attend_decoupled.argtypes = [i64, i32, i32, i32, i32, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                            _dp, ctypes.c_double, i32, ctypes.c_double, ctypes.c_double,
                                            _dp, _dp]
    lib.oracle_attend_decoupled.restype = i32
    lib.oracle_codec_residual.argtypes = [i64, i32, i32, i32, _dp, _dp, _dp, _dp, _dp, _dp]
    lib.oracle_codec_residual.restype = i32
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


# --------------------------------------------------------------------------
# Eq. 4 / Figure 10: exact cache accounting
# --------------------------------------------------------------------------
def cache_bytes(T, L, H, d, r_k, r_v, fold2d, elem_bytes, n_tokens):
    """Return (latent_bytes, uncompressed_bytes, rho_num, rho_den)."""
    lib = _load()
    out = [ctypes.c_uint64(0) for _ in range(4)]
    rc = lib.oracle_cache_bytes(T, L, H, d, r_k, r_v, int(bool(fold2d)), elem_bytes,
                                int(n_tokens), *[ctypes.byref(o) for o in out])
    if rc != 0:
        raise ValueError("invalid dimensions")
    return tuple(int(o.value) for o in out)


# --------------------------------------------------------------------------
# Eq. 2: encode;  Eq. 3: per-loop reconstruction
# --------------------------------------------------------------------------
def encode(x, mu, W_down):
    """c = (x - mu) W_down.  x [n, W], mu [W], W_down [W, r] -> c [n, r]."""
    x, mu, W_down = _f64(x), _f64(mu), _f64(W_down)
    n, W = x.shape
    r = W_down.shape[1]
    assert mu.shape == (W,) and W_down.shape[0] == W
    c = np.empty((n, r), dtype=np.float64)
    _load().oracle_encode(n, W, r, _ptr(x), _ptr(mu), _ptr(W_down), _ptr(c))
    return c


def reconstruct(c, W_up_t, mu_t):
    """x_hat_t = c W_up,t + mu_t.  c [n, r], W_up_t [r, d], mu_t [d] -> [n, d]."""
    c, W_up_t, mu_t = _f64(c), _f64(W_up_t), _f64(mu_t)
    n, r = c.shape
    d = W_up_t.shape[1]
    assert W_up_t.shape[0] == r and mu_t.shape == (d,)
    out = np.empty((n, d), dtype=np.float64)
    _load().oracle_reconstruct(n, r, d, _ptr(c), _ptr(W_up_t), _ptr(mu_t), _ptr(out))
    return out


# --------------------------------------------------------------------------
# Decode attention for one (sequence, head, loop) instance
# --------------------------------------------------------------------------
def attend(variant, c_K, c_V, W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q, scale):
    """One query over n cached latents.  variant in {"absorb", "reconstruct"}.

    c_K [n, r_k], c_V [n, r_v], W_up_K_t [r_k, d], mu_K_t [d], W_up_V_t [r_v, d],
    mu_V_t [d], q [d]  ->  (o [d], lse).
    """
    c_K, c_V = _f64(c_K), _f64(c_V)
    W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q = map(_f64, (W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q))
    n = c_K.shape[0]
    r_k, r_v, d = W_up_K_t.shape[0], W_up_V_t.shape[0], q.shape[0]
    if n == 0:
        c_K = np.zeros((1, r_k)); c_V = np.zeros((1, r_v))
    assert c_K.shape[1] == r_k and c_V.shape[1] == r_v
    assert W_up_K_t.shape == (r_k, d) and W_up_V_t.shape == (r_v, d)
    o = np.empty(d, dtype=np.float64)
    lse = ctypes.c_double(0.0)
    lib = _load()
    fn = {"absorb": lib.oracle_attend_absorb,
          "reconstruct": lib.oracle_attend_reconstruct}[variant]
    rc = fn(n, r_k, r_v, d, _ptr(c_K), _ptr(c_V), _ptr(W_up_K_t), _ptr(mu_K_t),
            _ptr(W_up_V_t), _ptr(mu_V_t), _ptr(q), float(scale), _ptr(o), ctypes.byref(lse))
    if rc != 0:
        raise MemoryError("oracle scratch allocation failed")
    return o, float(lse.value)


def attend_hybrid(c_K, c_V, W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, k_win, v_win, q, scale):
    """One loop query over n older tokens (latents) and w window tokens (exact K/V).

    c_K [n, r_k], c_V [n, r_v], codec slices as in ``attend``, k_win / v_win [w, d],
    q [d]  ->  (o [d], lse).
    """
    c_K, c_V = _f64(c_K), _f64(c_V)
    W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q = map(_f64, (W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q))
    k_win, v_win = _f64(k_win), _f64(v_win)
    n, w = c_K.shape[0], k_win.shape[0]
    r_k, r_v, d = W_up_K_t.shape[0], W_up_V_t.shape[0], q.shape[0]
    if n == 0:
        c_K = np.zeros((1, r_k)); c_V = np.zeros((1, r_v))
    if w == 0:
        k_win = np.zeros((1, d)); v_win = np.zeros((1, d))
    assert k_win.shape[1] == d and v_win.shape == k_win.shape
    o = np.empty(d, dtype=np.float64)
    lse = ctypes.c_double(0.0)
    rc = _load().oracle_attend_hybrid(n, w, r_k, r_v, d, _ptr(c_K), _ptr(c_V), _ptr(W_up_K_t),
                                      _ptr(mu_K_t), _ptr(W_up_V_t), _ptr(mu_V_t), _ptr(k_win),
                                      _ptr(v_win), _ptr(q), float(scale), _ptr(o), ctypes.byref(lse))
    if rc != 0:
        raise MemoryError("oracle scratch allocation failed")
    return o, float(lse.value)


def attend_decoupled(c_K, c_V, W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, k_rope, q, q_rope, scale, style,
                     base, q_pos):
    """Decoupled rotary sub-key: k_rope [n, d_r] stored rotated, q_rope [d_r] rotated at
    q_pos here; score = scale (q . k_hat + rope(q_rope) . k_rope).  -> (o [d], lse)."""
    c_K, c_V, k_rope = _f64(c_K), _f64(c_V), _f64(k_rope)
    W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q, q_rope = map(_f64, (W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q, q_rope))
    n = c_K.shape[0]
    r_k, r_v, d, d_r = W_up_K_t.shape[0], W_up_V_t.shape[0], q.shape[0], q_rope.shape[0]
    if d_r % 2:
        raise ValueError("the rotary part needs an even width")
    if n == 0:
        c_K = np.zeros((1, r_k)); c_V = np.zeros((1, r_v)); k_rope = np.zeros((1, max(d_r, 1)))
    if d_r == 0:
        q_rope = np.zeros(1); k_rope = np.zeros((max(n, 1), 1))
    o = np.empty(d, dtype=np.float64)
    lse = ctypes.c_double(0.0)
    rc = _load().oracle_attend_decoupled(n, r_k, r_v, d, d_r, _ptr(c_K), _ptr(c_V), _ptr(W_up_K_t),
                                         _ptr(mu_K_t), _ptr(W_up_V_t), _ptr(mu_V_t), _ptr(k_rope), _ptr(q),
                                         _ptr(q_rope), float(scale), int(style), float(base), float(q_pos),
                                         _ptr(o), ctypes.byref(lse))
    if rc != 0:
        raise MemoryError("oracle scratch allocation failed")
    return o, float(lse.value)


def codec_fit(x_cal, r, T):
    """SVD initialisation of the codec from calibration tokens ("Looped Latent Attention",
    review page, What carries the argument: the codec starts from the top right singular
    vectors of the centred teacher activations).

    x_cal [n, W] stacked vectors (W = T * Dp, loop-major), rank r ->
    (mu [W], W_down [W, r], W_up [T, r, Dp], sigma [min(n, W)]):
      mu = column mean; Y = x_cal - mu = U diag(sigma) V^T (numpy SVD, fp64);
      W_down = V[:, :r], each column signed so that its largest-magnitude entry (the first
      one on a tie) is positive; W_up,t = transpose of the loop-t row block of W_down.
    """
    x = _f64(x_cal)
    n, W = x.shape
    if W % T or not (0 < r <= min(n, W)):
        raise ValueError("bad rank or width")
    mu = x.mean(axis=0)
    _, sigma, Vt = np.linalg.svd(x - mu[None, :], full_matrices=False)
    W_down = Vt[:r].T.copy()
    lead = np.argmax(np.abs(W_down), axis=0)
    sign = np.sign(W_down[lead, np.arange(r)])
    sign[sign == 0] = 1.0
    W_down *= sign[None, :]
    W_up = W_down.reshape(T, W // T, r).transpose(0, 2, 1).copy()
    return mu, W_down, W_up, sigma


def codec_residual(x, mu, W_down, W_up):
    """Per-token reconstruction residual of a codec.

    x [n, W] stacked vectors (W = T * Dp, loop-major), mu [W], W_down [W, r],
    W_up [T, r, Dp]  ->  (err [n], norm [n]) with err = ||x - x_hat||, norm = ||x||.
    """
    x, mu, W_down, W_up = _f64(x), _f64(mu), _f64(W_down), _f64(W_up)
    n, W = x.shape
    T, r, Dp = W_up.shape
    assert W == T * Dp and mu.shape == (W,) and W_down.shape == (W, r)
    err = np.empty(n, dtype=np.float64)
    norm = np.empty(n, dtype=np.float64)
    if n:
        rc = _load().oracle_codec_residual(n, T, Dp, r, _ptr(x), _ptr(mu), _ptr(W_down), _ptr(W_up),
                                           _ptr(err), _ptr(norm))
        if rc != 0:
            raise MemoryError("oracle scratch allocation failed")
    return err, norm


ROPE_HALF, ROPE_INTERLEAVED = 0, 1


def attend_rope(c_K, c_V, W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q, scale, style, base, q_pos,
                k_pos0=0):
    """Faithful read: rebuilt keys and the query rotated at their positions (token i of
    the context at k_pos0 + i, the query at q_pos), then plain attention.  -> (o, lse)."""
    c_K, c_V = _f64(c_K), _f64(c_V)
    W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q = map(_f64, (W_up_K_t, mu_K_t, W_up_V_t, mu_V_t, q))
    n = c_K.shape[0]
    r_k, r_v, d = W_up_K_t.shape[0], W_up_V_t.shape[0], q.shape[0]
    if d % 2:
        raise ValueError("rotary embedding needs an even head dimension")
    if n == 0:
        c_K = np.zeros((1, r_k)); c_V = np.zeros((1, r_v))
    o = np.empty(d, dtype=np.float64)
    lse = ctypes.c_double(0.0)
    rc = _load().oracle_attend_rope(n, r_k, r_v, d, _ptr(c_K), _ptr(c_V), _ptr(W_up_K_t), _ptr(mu_K_t),
                                    _ptr(W_up_V_t), _ptr(mu_V_t), _ptr(q), float(scale), int(style),
                                    float(base), float(q_pos), float(k_pos0), _ptr(o), ctypes.byref(lse))
    if rc != 0:
        raise MemoryError("oracle scratch allocation failed")
    return o, float(lse.value)


# --------------------------------------------------------------------------
# A whole decode call for one layer: loop over (b, loop t, head) instances
# --------------------------------------------------------------------------
def decode_layer(variant, q, c_K, c_V, seq_start, ctx_lens, W_up_K, mu_K, W_up_V, mu_V,
                 t0, scale, fold2d=False, units=None, threads=None, window=None, rope=None,
                 decoupled=None):
    """Decode attention of every (b, tq, h) query of one layer.

    q        [B, Tq, H, d]           loop queries t0 .. t0+Tq-1
    c_K/c_V  [H', S, r]              latent planes (H' = H, or 1 for LLA-2D)
    seq_start[B], ctx_lens[B]        sequence b owns slots seq_start[b] .. +len-1
    W_up_K   per-head [H, T, r_k, d]    LLA-2D [T, r_k, H*d]   (same for V)
    mu_K     per-head [H, T, d]         LLA-2D [T, H*d]
    units    optional iterable of (b, h) pairs to evaluate (default: all)
    window   optional (win_k, win_v, win_len): exact loop keys / values of each
             sequence's window tokens, win_k [B, H, T, w_max, d], win_len [B]; the
             hybrid form then attends over the ctx_lens[b] latents and the
             win_len[b] window tokens together (variant is ignored)
    rope     optional (q_pos [B], base, style): the faithful read with rotary embedding,
             cached token i of sequence b at position i, its queries at q_pos[b]
             (variant is ignored)
    decoupled optional (k_rope [H', S, d_r], q_rope [B, Tq, H, d_r], q_pos [B], base, style):
             the decoupled rotary sub-key beside each latent (stored rotated), the
             queries' rotary parts rotated at q_pos[b] (variant is ignored)
    Returns (o [B, Tq, H, d], lse [B, Tq, H]); entries outside ``units`` are NaN.
    """
    q = np.asarray(q)
    B, Tq, H, d = q.shape
    o = np.full((B, Tq, H, d), np.nan)
    lse = np.full((B, Tq, H), np.nan)
    if units is None:
        units = [(b, h) for b in range(B) for h in range(H)]

    def slices(h, t):
        if fold2d:
            cols = slice(h * d, (h + 1) * d)
            return (W_up_K[t][:, cols], mu_K[t][cols], W_up_V[t][:, cols], mu_V[t][cols])
        return W_up_K[h][t], mu_K[h][t], W_up_V[h][t], mu_V[h][t]

    def run(unit):
        b, h = unit
        s0, n = int(seq_start[b]), int(ctx_lens[b])
        hp = 0 if fold2d else h
        cK = c_K[hp, s0:s0 + n]
        cV = c_V[hp, s0:s0 + n]
        for tq in range(Tq):
            wk, mk, wv, mv = slices(h, t0 + tq)
            if decoupled is not None:
                k_rope, q_rope, q_pos, base, style = decoupled
                o[b, tq, h], lse[b, tq, h] = attend_decoupled(
                    cK, cV, wk, mk, wv, mv, k_rope[hp, s0:s0 + n], q[b, tq, h], q_rope[b, tq, h], scale,
                    style, base, float(q_pos[b]))
            elif rope is not None:
                q_pos, base, style = rope
                o[b, tq, h], lse[b, tq, h] = attend_rope(cK, cV, wk, mk, wv, mv, q[b, tq, h], scale,
                                                         style, base, float(q_pos[b]))
            elif window is None:
                o[b, tq, h], lse[b, tq, h] = attend(variant, cK, cV, wk, mk, wv, mv,
                                                    q[b, tq, h], scale)
            else:
                win_k, win_v, win_len = window
                nw = int(win_len[b])
                o[b, tq, h], lse[b, tq, h] = attend_hybrid(
                    cK, cV, wk, mk, wv, mv, win_k[b, h, t0 + tq, :nw], win_v[b, h, t0 + tq, :nw],
                    q[b, tq, h], scale)

    units = list(units)
    if threads is None:
        threads = os.cpu_count() or 1
    if threads <= 1:
        for u in units:
            run(u)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(run, units))
    return o, lse
