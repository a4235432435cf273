"""Canary-padded buffers for the write paths: lla_encode, lla_codec_fit and
lla_codec_residual write nothing outside the buffers (and rows) they are given.

Every output buffer is the dense prefix of a larger allocation whose tail holds
sentinels; the fit workspace likewise.  Encode scatters to slot indices that include
out-of-range entries (-1, the slot count, far past it): those rows must write nothing,
every untargeted slot keeps its sentinel, and the targeted rows equal an unpadded run's.
The fit and the residual write one layer of a two-layer codec: the other layer's rows
keep their sentinels and the results equal an unpadded run's.  Paths covered: the
tcgen05 encode (ranks 16/32 and 96/160, one grid for K and V; LLA-2D with few tokens,
where a tile's K slabs are split over a cluster), the fp32 CUDA-core encode, the fit
(per-head and LLA-2D) and the residual diagnostic.
"""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import dims_of

pytestmark = pytest.mark.gpu
DEV = "cuda"
PAD = 4096                # extra elements after each buffer
SENT_F = 1234.5           # sentinel of fp32 / bf16 buffers (exact in bf16)
SENT_B = 0x5A             # sentinel byte of the workspace


def _padded(shape, dtype):
    n = int(np.prod(shape))
    full = torch.full((n + PAD,), SENT_F, dtype=dtype, device=DEV)
    return full, full[:n].view(*shape)


def _codec_inputs(w, layers):
    p = S.decode_inputs(w, layers, DEV, lens=[1], Tq=1)
    p["bias_k"] = torch.zeros(w.L, w.heads_stored, w.r_k, device=DEV)
    p["bias_v"] = torch.zeros(w.L, w.heads_stored, w.r_v, device=DEV)
    codec = lla.make_codec(W_down_k=p["W_down_k"], W_down_v=p["W_down_v"], bias_k=p["bias_k"],
                           bias_v=p["bias_v"], W_up_k=p["W_up_k"], W_up_v=p["W_up_v"],
                           mu_k=p["mu_k"], mu_v=p["mu_v"])
    lla.codec_bias(dims_of(w), codec, p["bias_k"], p["bias_v"])
    return p, codec


@pytest.mark.parametrize("name,n_tok", [("ouro1.4b-layer", 300), ("rho4-prefill", 130),
                                         ("lla2d", 16), ("tiny-fp32", 70)])
def test_encode_writes_only_its_slots(name, n_tok):
    w = S.shrink(S.WORKLOADS[name], L=2)
    layer, slots = 1, n_tok + 9
    p, codec = _codec_inputs(w, [layer])
    xk = S.draw_encode_tokens(w, layer, "k", n_tok, DEV)
    xv = S.draw_encode_tokens(w, layer, "v", n_tok, DEV)
    rng = np.random.default_rng(7)
    slot = rng.permutation(slots)[:n_tok].astype(np.int64)
    slot[3], slot[n_tok // 2], slot[-1] = -1, slots, slots + 100        # out of range: no write
    slot_idx = torch.as_tensor(slot, device=DEV)
    Hs = w.heads_stored
    ck_full, ck = _padded((w.L, Hs, slots, w.r_k), w.torch_dtype)
    cv_full, cv = _padded((w.L, Hs, slots, w.r_v), w.torch_dtype)
    lla.encode(dims_of(w), layer, 1, xk, xv, n_tok, slot_idx, codec, lla.make_cache(ck, cv, slots))
    ref_k = torch.zeros(w.L, Hs, slots, w.r_k, dtype=w.torch_dtype, device=DEV)
    ref_v = torch.zeros(w.L, Hs, slots, w.r_v, dtype=w.torch_dtype, device=DEV)
    lla.encode(dims_of(w), layer, 1, xk, xv, n_tok, slot_idx, codec, lla.make_cache(ref_k, ref_v, slots))
    torch.cuda.synchronize()
    assert lla.status_fetch(None) == 0
    for full, plane, ref in ((ck_full, ck, ref_k), (cv_full, cv, ref_v)):
        n = plane.numel()
        assert bool((full[n:] == SENT_F).all()), "write past the plane"
        assert bool((plane[0] == SENT_F).all()), "write into another layer"
        target = torch.zeros(slots, dtype=torch.bool, device=DEV)
        ok = slot[(slot >= 0) & (slot < slots)]
        target[torch.as_tensor(ok, device=DEV)] = True
        assert bool((plane[layer][:, ~target] == SENT_F).all()), "write to an untargeted slot"
        assert torch.equal(plane[layer][:, target], ref[layer][:, target])


@pytest.mark.parametrize("name,n_cal", [("ouro1.4b-layer", 64), ("lla2d", 256)])
def test_codec_fit_writes_only_its_layer(name, n_cal):
    w = S.shrink(S.WORKLOADS[name], L=2)
    layer, Hs, Dp = 1, w.heads_stored, w.d * (w.H if w.fold2d else 1)
    dims = dims_of(w)
    xs = {ax: S.draw_encode_tokens(w, layer, ax, n_cal, DEV, seed_tag="calib").unsqueeze(0) for ax in ("k", "v")}

    def run(padded):
        bufs, outs = {}, {}
        for ax, r in (("k", w.r_k), ("v", w.r_v)):
            for key, shape, dt in ((f"W_down_{ax}", (w.L, Hs, r, w.W), w.torch_dtype),
                                   (f"W_up_{ax}", (w.L, Hs, w.T, r, Dp), torch.float32),
                                   (f"mu_{ax}", (w.L, Hs, w.T, Dp), torch.float32),
                                   (f"sigma_{ax}", (1, Hs, n_cal), torch.float32)):
                if padded:
                    bufs[key], outs[key] = _padded(shape, dt)
                else:
                    outs[key] = torch.full(shape, SENT_F, dtype=dt, device=DEV)
        codec = lla.make_codec(**{k: v for k, v in outs.items() if not k.startswith("sigma")})
        wsb = lla.codec_fit_workspace_bytes(dims, 1, n_cal)
        ws_full = torch.full((wsb + PAD,), SENT_B, dtype=torch.uint8, device=DEV)
        ws_full[:8] = 0                       # status word and sweep counter start at zero
        lla.codec_fit(dims, layer, 1, xs["k"], xs["v"], n_cal, codec, ws_full[:wsb], wsb,
                      sigma_k=outs["sigma_k"], sigma_v=outs["sigma_v"])
        torch.cuda.synchronize()
        assert lla.status_fetch(ws_full[:wsb]) == 0
        assert bool((ws_full[wsb:] == SENT_B).all()), "workspace overrun"
        return bufs, outs

    bufs, outs = run(True)
    _, ref = run(False)
    for key, full in bufs.items():
        n = outs[key].numel()
        assert bool((full[n:] == SENT_F).all()), f"{key}: write past the buffer"
        if not key.startswith("sigma"):
            assert bool((outs[key][0] == SENT_F).all()), f"{key}: write into another layer"
        assert torch.equal(outs[key], ref[key]), key


@pytest.mark.parametrize("name,n_tok", [("ouro1.4b-layer", 65), ("rho4-prefill", 64), ("lla2d", 33)])
def test_codec_residual_writes_only_its_outputs(name, n_tok):
    w = S.shrink(S.WORKLOADS[name], L=2)
    layer, Hs = 1, w.heads_stored
    _, codec = _codec_inputs(w, [layer])
    xk = S.draw_encode_tokens(w, layer, "k", n_tok, DEV, seed_tag="held-out").unsqueeze(0)
    xv = S.draw_encode_tokens(w, layer, "v", n_tok, DEV, seed_tag="held-out").unsqueeze(0)
    padded = [_padded((1, n_tok, Hs), torch.float32) for _ in range(4)]
    lla.codec_residual(dims_of(w), layer, 1, xk, xv, n_tok, codec, *[v for _, v in padded])
    ref = [torch.full((1, n_tok, Hs), float("nan"), device=DEV) for _ in range(4)]
    lla.codec_residual(dims_of(w), layer, 1, xk, xv, n_tok, codec, *ref)
    torch.cuda.synchronize()
    for (full, view), r in zip(padded, ref):
        assert bool((full[view.numel():] == SENT_F).all()), "write past the output"
        assert torch.equal(view, r)
