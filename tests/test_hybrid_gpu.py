"""GPU parity of the hybrid form ("Hybrid Latent Attention for Looped Language Models",
abstract): exact K/V for each sequence's window rows plus latents for the older tokens,
one softmax over both, against the fp64 oracle on the same stored inputs.

Cases: ragged latent contexts x ragged windows (both empty, one empty, full window), the
three kernels of the latent part (tensor-core per-head, LLA-2D, CUDA-core fp32) and the
reconstruct form, multi-pass loop counts, a full-size layer on sampled units, and two
properties: an all-empty window reproduces lla_decode_attn, and the window row order does
not matter.
"""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import (assert_attn_close, oracle_decode, oracle_decode_units, run_decode,
                      run_decode_hybrid, sample_units)

pytestmark = pytest.mark.gpu
DEV = "cuda"

CTX_LENS = [0, 5, 0, 300, 1000, 129, 2048, 64]
WIN_LENS = [0, 0, 7, 128, 1, 33, 100, 64]


def _case(name, Tq=None, w_max=128, lens=CTX_LENS, wins=WIN_LENS, **kw):
    w = S.shrink(S.WORKLOADS[name], L=2, B=len(lens), **kw)
    layer = 1
    p = S.decode_inputs(w, layer, DEV, Tq=Tq, lens=lens, gap=5)
    win = S.window_inputs(w, layer, len(lens), w_max, DEV, win_lens=wins)
    return w, layer, p, win


@pytest.mark.parametrize("name,Tq,t0", [("ouro1.4b-layer", 4, 0), ("ouro1.4b-layer", 1, 3),
                                        ("lla2d", 4, 0), ("lla2d", 2, 1),
                                        ("tiny-fp32", 4, 0), ("deep-T32", 20, 5)])
def test_hybrid_ragged_contexts_and_windows(name, Tq, t0):
    w, layer, p, win = _case(name, Tq=Tq)
    out, lse, st = run_decode_hybrid(p, win, w, layer, t0, Tq, 0.9)
    assert st == 0
    if w.B * w.H <= 64:
        o_ref, l_ref = oracle_decode(p, w, layer, t0, Tq, 0.9, win=win)
    else:
        units = [(b, h) for b in range(w.B) for h in (0, w.H // 2, w.H - 1)]
        o_ref, l_ref = oracle_decode_units(p, w, layer, t0, Tq, 0.9, units, win=win)
    assert_attn_close(out, lse, o_ref, l_ref)
    # no latents and no window rows: out = 0, lse = -inf
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


def test_hybrid_reconstruct_form():
    w, layer, p, win = _case("ouro1.4b-layer", Tq=4, lens=[0, 700, 33, 0], wins=[9, 0, 128, 0])
    out, lse, st = run_decode_hybrid(p, win, w, layer, 0, 4, 1.0, variant=lla.RECONSTRUCT)
    assert st == 0
    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    o_ref, l_ref = oracle_decode_units(p, w, layer, 0, 4, 1.0, units, variant="reconstruct", win=win)
    assert_attn_close(out, lse, o_ref, l_ref)


def test_hybrid_full_layer_sampled_units():
    """Decode-step sizes: 64 sequences of 2-4k latent tokens, 16 heads, W = 128 window
    rows (ragged), bf16 output."""
    w = S.WORKLOADS["ouro1.4b-layer"]
    layer = 0
    p = S.decode_inputs(w, layer, DEV)
    win = S.window_inputs(w, layer, w.B, 128, DEV)
    out, lse, st = run_decode_hybrid(p, win, w, layer, 0, 4, 1.0, out_dtype=lla.BF16)
    assert st == 0
    units = sample_units(w.B, w.H, 40, seed=7)
    o_ref, l_ref = oracle_decode_units(p, w, layer, 0, 4, 1.0, units, win=win)
    assert_attn_close(out, lse, o_ref, l_ref)


def test_hybrid_with_empty_windows_equals_latent_decode():
    """len = 0 everywhere: the window part is empty and the output is the latent decode's,
    bit for bit (lse up to the rounding of its two formulas)."""
    w, layer, p, win = _case("ouro1.4b-layer", Tq=4, wins=[0] * len(CTX_LENS))
    out_h, lse_h, st = run_decode_hybrid(p, win, w, layer, 0, 4, 1.0)
    assert st == 0
    out, lse, st = run_decode(p, w, layer, 0, 4, 1.0)
    assert st == 0
    assert torch.equal(out_h, out)
    torch.testing.assert_close(lse_h, lse, atol=2e-5, rtol=0)


def test_hybrid_window_row_order_is_irrelevant():
    w, layer, p, win = _case("lla2d", Tq=4, wins=[128] * len(CTX_LENS))
    out_a, lse_a, _ = run_decode_hybrid(p, win, w, layer, 0, 4, 1.0)
    perm = torch.randperm(128, generator=torch.Generator().manual_seed(3)).to(DEV)
    win2 = dict(win)
    win2["win_k"] = win["win_k"][:, :, :, :, perm].contiguous()
    win2["win_v"] = win["win_v"][:, :, :, :, perm].contiguous()
    out_b, lse_b, st = run_decode_hybrid(p, win2, w, layer, 0, 4, 1.0)
    assert st == 0
    torch.testing.assert_close(out_b, out_a, atol=2e-5, rtol=1e-5)
    torch.testing.assert_close(lse_b, lse_a, atol=2e-5, rtol=0)


def test_hybrid_window_only_and_long_window():
    """No latents at all (a fresh sequence lives in its window) and a window longer than
    the latent context."""
    w, layer, p, win = _case("ouro1.4b-layer", Tq=4, w_max=1024, lens=[0, 0, 17],
                             wins=[1024, 1, 1000])
    out, lse, st = run_decode_hybrid(p, win, w, layer, 0, 4, 0.5)
    assert st == 0
    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    o_ref, l_ref = oracle_decode_units(p, w, layer, 0, 4, 0.5, units, win=win)
    assert_attn_close(out, lse, o_ref, l_ref)
