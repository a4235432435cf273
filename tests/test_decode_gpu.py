"""GPU parity: lla_decode_attn (absorb form) against the fp64 oracle on seeded inputs."""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import assert_attn_close, codec_of, dims_of, oracle_decode, run_decode

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def tiny():
    w = S.WORKLOADS["tiny-fp32"]
    return w, S.decode_inputs(w, 0, DEV)


@pytest.mark.parametrize("splits", [1, 2, 0])
def test_tiny_fp32_all_loops_fused(tiny, splits):
    w, p = tiny
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0, num_splits=splits)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("t0", [0, 1, 2, 3])
def test_tiny_fp32_one_loop_per_call(tiny, t0):
    w, p = tiny
    q1 = p["q"][:, t0:t0 + 1].contiguous()
    out, lse, st = run_decode(p, w, 0, t0, 1, 0.125, q=q1)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, t0, 1, 0.125, q=q1)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.fixture(scope="module")
def ouro():
    w = S.WORKLOADS["ouro1.4b-layer"]
    return w, S.decode_inputs(w, 0, DEV)


def test_ouro_layer_fused_loops_full(ouro):
    """Full Ouro-1.4B-shaped layer, 64 ragged sequences, all 4 loop queries in one
    pass, the split count the benchmark uses (automatic)."""
    w, p = ouro
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("t0", [0, 3])
def test_ouro_layer_model_order_single_loop(ouro, t0):
    w, p = ouro
    q1 = p["q"][:, t0:t0 + 1].contiguous()
    out, lse, st = run_decode(p, w, 0, t0, 1, 1.0, q=q1)
    assert st == 0
    units = [(b, h) for b in range(0, 64, 5) for h in range(16)]
    o_ref, l_ref = oracle_decode(p, w, 0, t0, 1, 1.0, q=q1, units=units)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("splits", [0, 3])
def test_decode_is_deterministic(ouro, splits):
    w, p = ouro
    a = run_decode(p, w, 0, 0, 4, 1.0, num_splits=splits)
    b = run_decode(p, w, 0, 0, 4, 1.0, num_splits=splits)
    assert a[2] == 0 and b[2] == 0
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_decode_with_dirty_workspace(ouro):
    """The workspace needs no initialisation beyond its status word: one full of stale
    bytes (here 0xff) gives the same result."""
    w, p = ouro
    dims = dims_of(w)
    B, Tq = len(p["lens"]), 4
    max_ctx = int(p["lens"].max())
    nb = lla.decode_workspace_bytes(dims, B, Tq, max_ctx, lla.ABSORB, 0)
    ws = torch.full((nb,), 255, dtype=torch.uint8, device="cuda")
    ws[:4] = 0  # status word
    out = torch.empty(B, Tq, w.H, w.d, device="cuda")
    lse = torch.empty(B, Tq, w.H, device="cuda")
    lla.decode_attn(dims, 0, 0, Tq, p["q"], lla.make_cache(p["k"], p["v"], p["slots"]), p["seq_start"],
                    p["ctx_lens"], B, max_ctx, codec_of(p), 1.0, out, lse, ws, nb)
    torch.cuda.synchronize()
    assert lla.status_fetch(ws) == 0
    ref = run_decode(p, w, 0, 0, 4, 1.0)
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])


# ---- edge cases -------------------------------------------------------------------------
EDGE_LENS = [0, 1, 2, 31, 255, 256, 257, 1000, 4097]


@pytest.mark.parametrize("rk,rv", [(16, 32), (8, 16), (16, 16)])
@pytest.mark.parametrize("splits", [0, 1, 3, 8])
def test_ragged_edges_bf16(rk, rv, splits):
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name=f"edge-{rk}-{rv}", r_k=rk, r_v=rv,
                 B=len(EDGE_LENS))
    p = S.decode_inputs(w, 0, DEV, lens=EDGE_LENS, gap=5)
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0, num_splits=splits)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)
    # empty context: out == 0 exactly, lse == -inf
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


@pytest.mark.parametrize("Tq,t0", [(2, 1), (3, 0), (3, 1)])
def test_partial_loop_ranges(Tq, t0):
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="tq", B=6, len_lo=100, len_hi=3000)
    p = S.decode_inputs(w, 0, DEV, Tq=Tq)
    out, lse, st = run_decode(p, w, 0, t0, Tq, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, t0, Tq, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("scale", [30.0, 1.0 / np.sqrt(128)])
def test_large_and_small_logit_scales(scale):
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="scale", B=4, len_lo=500, len_hi=2500)
    p = S.decode_inputs(w, 0, DEV)
    out, lse, st = run_decode(p, w, 0, 0, 4, scale, num_splits=2)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, scale)
    assert_attn_close(out, lse, o_ref, l_ref)


def test_distilled_codec_up_projection_not_transpose():
    """W_up perturbed away from W_down^T (a distilled codec): still exact attention."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="perturb", B=4, len_lo=300, len_hi=1500)
    p = S.decode_inputs(w, 0, DEV, perturb=0.3)
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)


def test_second_layer_of_a_multilayer_cache():
    w = S.shrink(S.WORKLOADS["capacity-768x4k"], name="ml", L=3, B=5, len_lo=10, len_hi=900)
    p = S.decode_inputs(w, [0, 2], DEV)
    for layer in (0, 2):
        out, lse, st = run_decode(p, w, layer, 0, 4, 1.0)
        assert st == 0
        o_ref, l_ref = oracle_decode(p, w, layer, 0, 4, 1.0)
        assert_attn_close(out, lse, o_ref, l_ref)


def test_bf16_output_storage(ouro):
    """bf16 outputs: the only extra error is the final round-to-nearest-even (<= 2^-9 |o|)."""
    w, p = ouro
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0, out_dtype=lla.BF16)
    assert st == 0 and out.dtype == torch.bfloat16
    units = [(b, h) for b in range(0, 64, 7) for h in range(16)]
    o_ref, _ = oracle_decode(p, w, 0, 0, 4, 1.0, units=units)
    o = out.float().cpu().double().numpy()
    m = ~np.isnan(o_ref)
    bound = np.abs(o_ref[m]) * 2.0 ** -8 + 5e-3
    assert np.all(np.abs(o[m] - o_ref[m]) <= bound)


def test_timed_entry_matches_decode_and_times_the_grid():
    """lla_decode_attn_timed: the same results, bit for bit, and a positive event interval
    around the decode grid that is shorter than the whole call."""
    import torch
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="timed", B=8, len_lo=500, len_hi=3000)
    p = S.decode_inputs(w, 0, "cuda")
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0)
    assert st == 0
    dims = dims_of(w)
    B, max_ctx = w.B, int(p["lens"].max())
    wsb = lla.decode_workspace_bytes(dims, B, 4, max_ctx)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for e in (e0, e1):
        e.record()
    torch.cuda.synchronize()
    c0.record()
    lla.decode_attn_timed(dims, 0, 0, 4, p["q"], lla.make_cache(p["k"], p["v"], p["slots"]), p["seq_start"],
                          p["ctx_lens"], B, max_ctx, codec_of(p), 1.0, out2, lse2, ws, wsb, e0, e1)
    c1.record()
    torch.cuda.synchronize()
    assert lla.status_fetch(ws) == 0
    assert torch.equal(out2, out) and torch.equal(lse2, lse)
    assert 0 < e0.elapsed_time(e1) < c0.elapsed_time(c1)


@pytest.mark.parametrize("Tq,t0", [(12, 0), (9, 3)])
def test_more_than_eight_loop_queries_small_ranks(Tq, t0):
    """T = 12 loops at ranks 16/32: fragment rows g + 8 of the tensor-core tile carry loop
    queries (the 16-row variant of the small-rank kernel)."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="T12", T=12, L=1, B=6, len_lo=100, len_hi=2000)
    p = S.decode_inputs(w, 0, "cuda", Tq=Tq)
    out, lse, st = run_decode(p, w, 0, t0, Tq, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, t0, Tq, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("T,Tq,t0", [(24, 20, 2), (32, 32, 0), (40, 37, 1)])
def test_two_row_tiles_in_one_latent_pass_small_ranks(T, Tq, t0):
    """17 to 32 loop queries fill two m16 row tiles that share each staged latent tile (one
    read of the latents); 37 queries take a second pass of 5."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name=f"T{T}", T=T, L=1, B=5, len_lo=60, len_hi=1700)
    p = S.decode_inputs(w, 0, "cuda", Tq=Tq)
    out, lse, st = run_decode(p, w, 0, t0, Tq, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, t0, Tq, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)


def test_two_row_tiles_big_ranks_ragged():
    """Ranks 96/160 (64-token tiles, two consumer warps per row tile), 17 loop queries and
    ragged contexts including empty and one-token sequences."""
    lens = [0, 1, 63, 64, 65, 700, 1500]
    w = S.shrink(S.WORKLOADS["deep-T32"], name="T32-ragged", L=1, B=len(lens))
    p = S.decode_inputs(w, 0, "cuda", Tq=17, lens=lens, gap=2)
    out, lse, st = run_decode(p, w, 0, 9, 17, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 9, 17, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


# ---- head dimensions other than 128 ------------------------------------------------------
@pytest.mark.parametrize("d", [64, 96, 192, 256, 512])
@pytest.mark.parametrize("rk,rv", [(16, 32), (96, 160)])
def test_head_dims_prologue_and_projection(d, rk, rv):
    """The q_tilde prologue covers d in 128-wide register chunks (several passes for d > 256)
    and the combine projects d / 4 column groups over its warps; both depend on d."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name=f"d{d}-{rk}-{rv}", d=d, r_k=rk, r_v=rv, H=4, B=5,
                 len_lo=60, len_hi=700)
    p = S.decode_inputs(w, 0, DEV)
    scale = 1.0 / np.sqrt(d)
    if rv * d * 4 > 190 * 1024:  # W_up,t^V too large for the combine: refused, nothing queued
        with pytest.raises(lla.LLAError) as e:
            run_decode(p, w, 0, 0, 4, scale)
        assert e.value.code == lla.LLA_ERR_UNSUPPORTED
        return
    out, lse, st = run_decode(p, w, 0, 0, 4, scale)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, scale)
    assert_attn_close(out, lse, o_ref, l_ref)


def test_head_dim_256_deep_loops_sixteen_sequence_combine():
    """32 loop queries (two row tiles) at d = 256: W_up,t^V of 160 KB, staged once per 16
    sequences by the combine; 17 sequences so a second, partial combine CTA exists."""
    w = S.shrink(S.WORKLOADS["deep-T32"], name="d256-T32", d=256, H=2, L=1, B=17, len_lo=40, len_hi=600)
    p = S.decode_inputs(w, 0, DEV, Tq=32)
    out, lse, st = run_decode(p, w, 0, 0, 32, 1.0 / 16)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 32, 1.0 / 16)
    assert_attn_close(out, lse, o_ref, l_ref)
