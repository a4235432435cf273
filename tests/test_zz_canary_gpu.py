"""Canary-padded buffers: a decode writes nothing past the buffers it is given.

The workspace is followed by 4 KB of sentinel bytes and `out` / `lse` by one extra
sequence row of sentinel values; the call gets the dense prefix views.  After the call
the sentinels must be intact and the result must equal the one computed with exactly
sized buffers.  Covers the kernels a decode call can route to: the per-head tensor-core
kernel, the fp32 CUDA-core kernel, the reconstruct form, LLA-2D and the hybrid window
pass, on ragged contexts (empty and one-token sequences included).
"""
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import codec_of, dims_of, run_decode, run_decode_hybrid

pytestmark = pytest.mark.gpu
DEV = "cuda"

CTX_LENS = [0, 5, 300, 129, 2048, 64, 1]
WIN_LENS = [0, 7, 128, 1, 100, 64, 0]
PAD_BYTES = 4096
SENTINEL_BYTE = 0x5A
SENTINEL = 1234.5


def _padded(shape):
    full = torch.full((shape[0] + 1,) + tuple(shape[1:]), SENTINEL, dtype=torch.float32, device=DEV)
    return full, full[:shape[0]]


@pytest.mark.parametrize("name,variant,window", [
    ("ouro1.4b-layer", lla.ABSORB, False),
    ("ouro1.4b-layer", lla.RECONSTRUCT, False),
    ("tiny-fp32", lla.ABSORB, False),
    ("lla2d", lla.ABSORB, False),
    ("ouro1.4b-layer", lla.ABSORB, True),
])
def test_decode_writes_nothing_past_its_buffers(name, variant, window):
    Tq, layer = 4, 1
    w = S.shrink(S.WORKLOADS[name], L=2, B=len(CTX_LENS))
    p = S.decode_inputs(w, layer, DEV, Tq=Tq, lens=CTX_LENS, gap=5)
    dims = dims_of(w)
    B, max_ctx = len(CTX_LENS), max(CTX_LENS)
    if window:
        win = S.window_inputs(w, layer, B, 128, DEV, win_lens=WIN_LENS)
        nb = lla.decode_hybrid_workspace_bytes(dims, B, Tq, max_ctx, variant, 0)
    else:
        nb = lla.decode_workspace_bytes(dims, B, Tq, max_ctx, variant, 0)
    ws_full = torch.full((nb + PAD_BYTES,), SENTINEL_BYTE, dtype=torch.uint8, device=DEV)
    ws_full[:4] = 0  # status word
    ws = ws_full[:nb]
    out_full, out = _padded((B, Tq, w.H, w.d))
    lse_full, lse = _padded((B, Tq, w.H))
    args = (dims, layer, 0, Tq, p["q"], lla.make_cache(p["k"], p["v"], p["slots"]), p["seq_start"],
            p["ctx_lens"], B, max_ctx, codec_of(p))
    if window:
        wnd = lla.make_window(win["win_k"], win["win_v"], win["win_len"], win["w_max"], win["win_k"].shape[1])
        lla.decode_attn_hybrid(*args, wnd, 1.0, out, lse, ws, nb, variant=variant)
    else:
        lla.decode_attn(*args, 1.0, out, lse, ws, nb, variant=variant)
    torch.cuda.synchronize()
    assert lla.status_fetch(ws) == 0
    assert bool((ws_full[nb:] == SENTINEL_BYTE).all()), "workspace overrun"
    assert bool((out_full[B] == SENTINEL).all()), "output overrun"
    assert bool((lse_full[B] == SENTINEL).all()), "lse overrun"
    if window:
        ref = run_decode_hybrid(p, win, w, layer, 0, Tq, 1.0, variant=variant)
    else:
        ref = run_decode(p, w, layer, 0, Tq, 1.0, variant=variant)
    assert ref[2] == 0
    torch.testing.assert_close(out, ref[0], rtol=0, atol=1e-6)
    torch.testing.assert_close(lse, ref[1], rtol=0, atol=1e-6)
