"""Helpers for GPU parity tests: run the CUDA path through the C ABI, run the fp64
oracle on the same inputs, compare with the stated tolerances.

Tolerances (attention output stored in bf16 with fp32 accumulation): max-abs <= 1e-2
and relative L2 <= 5e-3 against the fp64 oracle; encode latents relative L2 <= 5e-3.
lse is compared with an absolute bound of 2e-3 (it is computed in fp32 from fp32
scores; -inf must match exactly for empty contexts).
"""
import numpy as np
import torch

import decode_attention_12_b200 as lla
import oracle

ATOL_MAX = 1e-2
RTOL_L2 = 5e-3
LSE_ATOL = 2e-3


def to64(t):
    return t.detach().to(torch.float32).cpu().double().numpy()


def dims_of(w, out_dtype=lla.F32):
    return lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v, int(w.fold2d),
                         lla.F32 if w.dtype == "f32" else lla.BF16, out_dtype)


def codec_of(p):
    return lla.make_codec(W_down_k=p["W_down_k"], W_down_v=p["W_down_v"], bias_k=p.get("bias_k"),
                          bias_v=p.get("bias_v"), W_up_k=p["W_up_k"], W_up_v=p["W_up_v"],
                          mu_k=p["mu_k"], mu_v=p["mu_v"])


def run_decode(p, w, layer, t0, Tq, scale, num_splits=0, variant=lla.ABSORB, q=None,
               out_dtype=lla.F32):
    """Decode through the C ABI; returns (out, lse, device status)."""
    dims = dims_of(w, out_dtype)
    q = p["q"] if q is None else q
    B = len(p["lens"])
    max_ctx = int(p["lens"].max()) if B else 0
    ws_bytes = lla.decode_workspace_bytes(dims, B, Tq, max_ctx, variant, num_splits)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    odt = torch.float32 if out_dtype == lla.F32 else torch.bfloat16
    out = torch.full((B, Tq, w.H, w.d), float("nan"), dtype=odt, device="cuda")
    lse = torch.full((B, Tq, w.H), float("nan"), dtype=torch.float32, device="cuda")
    lla.decode_attn(dims, layer, t0, Tq, q, lla.make_cache(p["k"], p["v"], p["slots"]),
                    p["seq_start"], p["ctx_lens"], B, max_ctx, codec_of(p), scale, out, lse,
                    ws, ws_bytes, variant=variant, num_splits=num_splits)
    torch.cuda.synchronize()
    status = lla.status_fetch(ws)
    return out, lse, status


def oracle_decode(p, w, layer, t0, Tq, scale, units=None, variant="absorb", q=None, threads=None,
                  win=None, rope=None):
    q = p["q"] if q is None else q
    q64 = to64(q)
    cK, cV = to64(p["k"][layer]), to64(p["v"][layer])
    WK, WV = to64(p["W_up_k"][layer]), to64(p["W_up_v"][layer])
    mK, mV = to64(p["mu_k"][layer]), to64(p["mu_v"][layer])
    if w.fold2d:
        WK, WV, mK, mV = WK[0], WV[0], mK[0], mV[0]
    window = None
    if win is not None:
        window = (to64(win["win_k"][layer]), to64(win["win_v"][layer]), win["win_lens"])
    return oracle.decode_layer(variant, q64, cK, cV, p["starts"], p["lens"], WK, mK, WV, mV,
                               t0, scale, fold2d=w.fold2d, units=units, threads=threads,
                               window=window, rope=rope)


def run_decode_rope(p, w, layer, t0, Tq, scale, q_pos, base, style, num_splits=0, q=None,
                    out_dtype=lla.F32):
    """Faithful (rotary) decode through the C ABI; returns (out, lse, device status)."""
    dims = dims_of(w, out_dtype)
    q = p["q"] if q is None else q
    B = len(p["lens"])
    max_ctx = int(p["lens"].max()) if B else 0
    ws_bytes = lla.decode_workspace_bytes(dims, B, Tq, max_ctx, lla.RECONSTRUCT, num_splits)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    odt = torch.float32 if out_dtype == lla.F32 else torch.bfloat16
    out = torch.full((B, Tq, w.H, w.d), float("nan"), dtype=odt, device="cuda")
    lse = torch.full((B, Tq, w.H), float("nan"), dtype=torch.float32, device="cuda")
    qp = torch.as_tensor(np.asarray(q_pos, dtype=np.int32), device="cuda")
    lla.decode_attn_rope(dims, layer, t0, Tq, q, lla.make_cache(p["k"], p["v"], p["slots"]),
                         p["seq_start"], p["ctx_lens"], B, max_ctx, codec_of(p),
                         lla.make_rope(qp, base, style), scale, out, lse, ws, ws_bytes,
                         num_splits=num_splits)
    torch.cuda.synchronize()
    status = lla.status_fetch(ws)
    return out, lse, status


def rotate_pairs(x, pos, base, style):
    """Rotary map in RoFormer's complex form, fp64 numpy, in the real layout of ``style``."""
    x = np.asarray(x, dtype=np.float64)
    dr = x.shape[-1]
    theta = base ** (-2.0 * np.arange(dr // 2) / dr)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    if style == lla.ROPE_HALF:
        a, b = x[..., :dr // 2], x[..., dr // 2:]
    else:
        a, b = x[..., 0::2], x[..., 1::2]
    z = (a + 1j * b) * np.exp(1j * ang)
    out = np.empty_like(x)
    if style == lla.ROPE_HALF:
        out[..., :dr // 2], out[..., dr // 2:] = z.real, z.imag
    else:
        out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def stored_subkeys(raw, starts, lens, base, style, dtype):
    """Sub-key plane as the cache stores it: slot seq_start[b] + n rotated at position n."""
    raw = np.asarray(raw, dtype=np.float64)         # [H', slots, d_r]
    pos = np.zeros(raw.shape[1])
    for s0, n in zip(starts, lens):
        pos[int(s0):int(s0) + int(n)] = np.arange(int(n))
    rot = rotate_pairs(raw, pos[None, :], base, style)
    return torch.as_tensor(rot, dtype=torch.float32).to(dtype)


def run_decode_decoupled(p, w, layer, t0, Tq, scale, k_rope, q_rope, q_pos, base, style, num_splits=0,
                         out_dtype=lla.F32):
    """Decoupled-RoPE absorbed decode through the C ABI; k_rope [L][H][slots][d_r] on the device."""
    dims = dims_of(w, out_dtype)
    B = len(p["lens"])
    d_r = k_rope.shape[-1]
    max_ctx = int(p["lens"].max()) if B else 0
    ws_bytes = lla.decode_decoupled_workspace_bytes(dims, B, Tq, max_ctx, d_r, num_splits)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    odt = torch.float32 if out_dtype == lla.F32 else torch.bfloat16
    out = torch.full((B, Tq, w.H, w.d), float("nan"), dtype=odt, device="cuda")
    lse = torch.full((B, Tq, w.H), float("nan"), dtype=torch.float32, device="cuda")
    qp = torch.as_tensor(np.asarray(q_pos, dtype=np.int32), device="cuda")
    lla.decode_attn_decoupled(dims, layer, t0, Tq, p["q"], lla.make_cache(p["k"], p["v"], p["slots"]),
                              p["seq_start"], p["ctx_lens"], B, max_ctx, codec_of(p), k_rope, q_rope, d_r,
                              lla.make_rope(qp, base, style), scale, out, lse, ws, ws_bytes,
                              num_splits=num_splits)
    torch.cuda.synchronize()
    status = lla.status_fetch(ws)
    return out, lse, status


def run_decode_hybrid(p, win, w, layer, t0, Tq, scale, num_splits=0, variant=lla.ABSORB, q=None,
                      out_dtype=lla.F32):
    """Hybrid decode through the C ABI; returns (out, lse, device status)."""
    dims = dims_of(w, out_dtype)
    q = p["q"] if q is None else q
    B = len(p["lens"])
    max_ctx = int(p["lens"].max()) if B else 0
    ws_bytes = lla.decode_hybrid_workspace_bytes(dims, B, Tq, max_ctx, variant, num_splits)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    odt = torch.float32 if out_dtype == lla.F32 else torch.bfloat16
    out = torch.full((B, Tq, w.H, w.d), float("nan"), dtype=odt, device="cuda")
    lse = torch.full((B, Tq, w.H), float("nan"), dtype=torch.float32, device="cuda")
    window = lla.make_window(win["win_k"], win["win_v"], win["win_len"], win["w_max"],
                             win["win_k"].shape[1])
    lla.decode_attn_hybrid(dims, layer, t0, Tq, q, lla.make_cache(p["k"], p["v"], p["slots"]),
                           p["seq_start"], p["ctx_lens"], B, max_ctx, codec_of(p), window, scale,
                           out, lse, ws, ws_bytes, variant=variant, num_splits=num_splits)
    torch.cuda.synchronize()
    status = lla.status_fetch(ws)
    return out, lse, status


def attn_errors(out_gpu, o_ref):
    o = to64(out_gpu)
    mask = ~np.isnan(o_ref)
    err = o[mask] - o_ref[mask]
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    den = float(np.linalg.norm(o_ref[mask]))
    rel = float(np.linalg.norm(err)) / den if den > 0 else float(np.linalg.norm(err))
    return max_abs, rel


def assert_attn_close(out_gpu, lse_gpu, o_ref, lse_ref):
    assert not torch.isnan(out_gpu.float()).any(), "NaN in GPU output"
    max_abs, rel = attn_errors(out_gpu, o_ref)
    assert max_abs <= ATOL_MAX, f"max-abs {max_abs:.3e} > {ATOL_MAX}"
    assert rel <= RTOL_L2, f"rel-L2 {rel:.3e} > {RTOL_L2}"
    l = to64(lse_gpu)
    m = ~np.isnan(lse_ref)
    inf_ref = np.isinf(lse_ref) & m
    assert np.array_equal(np.isinf(l) & m, inf_ref), "lse -inf pattern differs"
    fin = m & ~inf_ref
    if fin.any():
        d = np.abs(l[fin] - lse_ref[fin]).max()
        assert d <= LSE_ATOL, f"lse max-abs {d:.3e}"
    return max_abs, rel


def oracle_decode_units(p, w, layer, t0, Tq, scale, units, variant="absorb", q=None, threads=None,
                        win=None, rope=None, decoupled=None):
    """Oracle on sampled (b, h) units only: their latent rows are gathered to the host.

    Works for caches far larger than host memory; the result arrays are NaN outside
    ``units``.  Uses the same stored inputs as the GPU run.
    """
    q = p["q"] if q is None else q
    q64 = to64(q)
    B, _, H, d = q64.shape
    o = np.full((B, Tq, H, d), np.nan)
    lse = np.full((B, Tq, H), np.nan)
    WK, WV = to64(p["W_up_k"][layer]), to64(p["W_up_v"][layer])
    mK, mV = to64(p["mu_k"][layer]), to64(p["mu_v"][layer])
    if w.fold2d:
        WK, WV, mK, mV = WK[0], WV[0], mK[0], mV[0]
    for (b, h) in units:
        s0, n = int(p["starts"][b]), int(p["lens"][b])
        hp = 0 if w.fold2d else h
        cK = to64(p["k"][layer, hp, s0:s0 + n])[None]
        cV = to64(p["v"][layer, hp, s0:s0 + n])[None]
        window = None
        if win is not None:
            nw = int(win["win_lens"][b])
            hsel = slice(None) if w.fold2d else slice(h, h + 1)
            window = (to64(win["win_k"][layer, b:b + 1, hsel, :, :nw]),
                      to64(win["win_v"][layer, b:b + 1, hsel, :, :nw]), [nw])
        rope_b = None if rope is None else ([rope[0][b]], rope[1], rope[2])
        dec_b = None
        if decoupled is not None:  # (k_rope plane [H', slots, d_r] of the layer, q_rope, q_pos, base, style)
            kr, qr, qpos, base_, style_ = decoupled
            dec_b = (to64(kr[hp:hp + 1, s0:s0 + n]), to64(qr[b:b + 1, :, h:h + 1]), [qpos[b]], base_, style_)
        if w.fold2d:
            ob, lb = oracle.decode_layer(variant, q64[b:b + 1], cK, cV, [0], [n], WK, mK, WV, mV, t0, scale,
                                         fold2d=True, units=[(0, h)], threads=1, window=window,
                                         rope=rope_b)
        else:
            sel = [h]
            ob, lb = oracle.decode_layer(variant, q64[b:b + 1, :, sel], cK, cV, [0], [n], WK[sel], mK[sel],
                                         WV[sel], mV[sel], t0, scale, fold2d=False, threads=1,
                                         window=window, rope=rope_b, decoupled=dec_b)
            o[b, :, h] = ob[0, :, 0]
            lse[b, :, h] = lb[0, :, 0]
            continue
        o[b, :, h] = ob[0, :, h]
        lse[b, :, h] = lb[0, :, h]
    return o, lse


def sample_units(B, H, n, seed=0):
    rng = np.random.default_rng(seed)
    units = {(0, 0), (B - 1, H - 1)}
    while len(units) < min(n, B * H):
        units.add((int(rng.integers(0, B)), int(rng.integers(0, H))))
    return sorted(units)
