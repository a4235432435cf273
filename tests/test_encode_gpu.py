"""GPU parity: lla_codec_bias + lla_encode (write path, Eq. 2) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
import oracle
from gpu_util import dims_of, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
ENC_RTOL_L2 = 5e-3


def _setup(w, layers, n_tok, slots=None, seed_tag="tokens"):
    """Codec for `layers`, tokens for each, bias via the library, empty cache."""
    p = S.decode_inputs(w, layers, DEV, lens=[1], Tq=1)  # codec tensors of the layers
    slots = n_tok if slots is None else slots
    p["bias_k"] = torch.zeros(w.L, w.heads_stored, w.r_k, device=DEV)
    p["bias_v"] = torch.zeros(w.L, w.heads_stored, w.r_v, device=DEV)
    dims = dims_of(w)
    codec = lla.make_codec(W_down_k=p["W_down_k"], W_down_v=p["W_down_v"], mu_k=p["mu_k"],
                           mu_v=p["mu_v"])
    lla.codec_bias(dims, codec, p["bias_k"], p["bias_v"])
    p["ck"] = torch.full((w.L, w.heads_stored, slots, w.r_k), float("nan"), dtype=w.torch_dtype,
                         device=DEV)
    p["cv"] = torch.full((w.L, w.heads_stored, slots, w.r_v), float("nan"), dtype=w.torch_dtype,
                         device=DEV)
    return p


def _oracle_latents(w, p, layer, x, axis, rows):
    """Oracle encode of token rows `rows` for every stored head: [H', len(rows), r]."""
    xs = to64(x[rows])                                  # [n, T, H, d]
    Wd = to64(p[f"W_down_{axis}"][layer])               # [H', r, W]
    mu = to64(p[f"mu_{axis}"][layer]).reshape(w.heads_stored, -1)   # [H', W]
    out = []
    for hs in range(w.heads_stored):
        xr = xs.reshape(len(rows), -1) if w.fold2d else xs[:, :, hs, :].reshape(len(rows), -1)
        out.append(oracle.encode(xr, mu[hs], Wd[hs].T))
    return np.stack(out)


def _check(w, p, layer, x, axis, rows, slot_of_row):
    ref = _oracle_latents(w, p, layer, x, axis, rows)
    plane = p["ck" if axis == "k" else "cv"][layer]
    got = to64(plane[:, torch.as_tensor(slot_of_row, device=DEV)])
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all()
    assert err <= ENC_RTOL_L2, f"encode rel-L2 {err:.3e}"
    return err


@pytest.mark.parametrize("name", ["tiny-fp32", "ouro1.4b-layer", "rho4-prefill", "deep-T32", "lla2d"])
def test_encode_matches_oracle(name):
    w = S.WORKLOADS[name]
    if w.L > 1:
        w = S.shrink(w, L=2)
    n_tok = 1000
    layer = w.L - 1
    p = _setup(w, [layer], n_tok, slots=n_tok + 7)
    xk = S.draw_encode_tokens(w, layer, "k", n_tok, DEV)
    xv = S.draw_encode_tokens(w, layer, "v", n_tok, DEV)
    perm = np.random.default_rng(1).permutation(n_tok + 7)[:n_tok]   # scattered slots
    slot_idx = torch.as_tensor(perm, dtype=torch.int64, device=DEV)
    lla.encode(dims_of(w), layer, 1, xk, xv, n_tok, slot_idx, _codec(p), _cache(p, n_tok + 7))
    torch.cuda.synchronize()
    rows = np.arange(n_tok)
    for axis, x in (("k", xk), ("v", xv)):
        _check(w, p, layer, x, axis, rows, perm)


def test_encode_skips_out_of_range_slots():
    w = S.WORKLOADS["ouro1.4b-layer"]
    n_tok = 64
    p = _setup(w, [0], n_tok, slots=n_tok)
    xk = S.draw_encode_tokens(w, 0, "k", n_tok, DEV)
    xv = S.draw_encode_tokens(w, 0, "v", n_tok, DEV)
    slots = np.arange(n_tok)
    slots[5], slots[9] = -1, n_tok + 100
    lla.encode(dims_of(w), 0, 1, xk, xv, n_tok, torch.as_tensor(slots, device=DEV), _codec(p),
               _cache(p, n_tok))
    torch.cuda.synchronize()
    assert torch.isnan(p["ck"][0, :, 5].float()).all() and torch.isnan(p["ck"][0, :, 9].float()).all()
    ok = [i for i in range(n_tok) if i not in (5, 9)]
    _check(w, p, 0, xk, "k", np.array(ok), slots[ok])


def test_encode_of_the_mean_is_zero():
    """Encoding mu itself must give c = 0 (bias = -mu W_down exactly cancels)."""
    w = S.WORKLOADS["tiny-fp32"]
    p = _setup(w, [0], 4)
    mu = p["mu_k"][0]                         # [H, T, d] fp32
    x = mu.permute(1, 0, 2).unsqueeze(0).expand(4, -1, -1, -1).contiguous()  # [4, T, H, d]
    slot_idx = torch.arange(4, device=DEV)
    lla.encode(dims_of(w), 0, 1, x, x, 4, slot_idx, _codec(p), _cache(p, 4))
    torch.cuda.synchronize()
    scale = float(p["mu_k"].abs().max())
    assert float(p["ck"][0].abs().max()) <= 1e-5 * scale * 64


def _codec(p):
    return lla.make_codec(W_down_k=p["W_down_k"], W_down_v=p["W_down_v"], bias_k=p["bias_k"],
                          bias_v=p["bias_v"], W_up_k=p["W_up_k"], W_up_v=p["W_up_v"],
                          mu_k=p["mu_k"], mu_v=p["mu_v"])


def _cache(p, slots):
    return lla.make_cache(p["ck"], p["cv"], slots)


def test_codec_bias_matches_definition():
    w = S.shrink(S.WORKLOADS["rho4-prefill"], L=2)
    p = _setup(w, [0, 1], 1)
    for axis in ("k", "v"):
        Wd = to64(p[f"W_down_{axis}"])                 # [L, H, r, W]
        mu = to64(p[f"mu_{axis}"]).reshape(w.L, w.H, -1)
        for l in range(w.L):
            for h in (0, 7, 15):
                # the bias is the encode of the zero vector: (0 - mu) W_down
                ref = oracle.encode(np.zeros((1, Wd.shape[-1])), mu[l, h], Wd[l, h].T)[0]
                got = to64(p[f"bias_{axis}"][l, h])
                np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-6)


def test_prefill_encode_full_layer_sampled_rows():
    """rho4-prefill: one layer of the full prefill (32 x 4096 tokens x 16 heads, K and V),
    checked on sampled token rows."""
    w = S.WORKLOADS["rho4-prefill"]
    n_tok = w.B * 4096
    layer = w.L - 1
    p = _setup(w, [layer], n_tok)
    xk = S.draw_encode_tokens(w, layer, "k", n_tok, DEV)
    xv = S.draw_encode_tokens(w, layer, "v", n_tok, DEV)
    slot_idx = torch.arange(n_tok, device=DEV)
    lla.encode(dims_of(w), layer, 1, xk, xv, n_tok, slot_idx, _codec(p), _cache(p, n_tok))
    torch.cuda.synchronize()
    assert lla.status_fetch(None) == 0
    rows = np.unique(np.concatenate([[0, n_tok - 1], np.random.default_rng(5).integers(0, n_tok, 62)]))
    for axis, x in (("k", xk), ("v", xv)):
        _check(w, p, layer, x, axis, rows, rows)
