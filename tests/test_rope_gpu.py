"""GPU parity of the faithful read with rotary embedding (RoPE applied after reconstruction:
LLA paper, Pith verdict record, key_machinery and domain assumptions; RoFormer's rotary
map) against the fp64 oracle on the same stored inputs.

Cases: both pairings, ragged contexts (empty, one token, tile edges), query positions at,
after and far past the context, rotary bases from 500 to 5e5, d = 64 and 128, LLA-2D, and
positions past 16k where the angles reach 1e4 radians.
"""
import numpy as np
import pytest

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import assert_attn_close, oracle_decode_units, run_decode_rope

pytestmark = pytest.mark.gpu
DEV = "cuda"
HALF, INTER = lla.ROPE_HALF, lla.ROPE_INTERLEAVED

CTX_LENS = [0, 1, 31, 32, 33, 128, 129, 700, 2048, 3000]


def _run(w, lens, q_pos, base, style, Tq, t0, units_per_seq=None, scale=1.0, num_splits=0):
    w = S.shrink(w, L=2, B=len(lens))
    layer = 1
    p = S.decode_inputs(w, layer, DEV, Tq=Tq, lens=lens, gap=3)
    out, lse, st = run_decode_rope(p, w, layer, t0, Tq, scale, q_pos, base, style, num_splits=num_splits)
    assert st == 0
    heads = range(w.H) if units_per_seq is None else np.linspace(0, w.H - 1, units_per_seq).astype(int)
    units = [(b, int(h)) for b in range(w.B) for h in heads]
    o_ref, l_ref = oracle_decode_units(p, w, layer, t0, Tq, scale, units, variant="reconstruct",
                                       rope=(np.asarray(q_pos), base, style))
    assert_attn_close(out, lse, o_ref, l_ref)
    return out, lse


@pytest.mark.parametrize("style", [HALF, INTER])
def test_rope_ragged_query_after_context(style):
    """The usual decode step: the new token sits right after its sequence's context."""
    _run(S.WORKLOADS["ouro1.4b-layer"], CTX_LENS, CTX_LENS, 10000.0, style, Tq=4, t0=0, units_per_seq=3)


@pytest.mark.parametrize("style,base,Tq,t0", [(HALF, 500000.0, 2, 1), (INTER, 500.0, 1, 3)])
def test_rope_bases_and_loop_ranges(style, base, Tq, t0):
    q_pos = [n + 5000 for n in CTX_LENS]
    _run(S.WORKLOADS["ouro1.4b-layer"], CTX_LENS, q_pos, base, style, Tq=Tq, t0=t0, units_per_seq=3,
         scale=0.6)


@pytest.mark.parametrize("rk,rv", [(16, 16), (32, 32)])
def test_rope_head_dim_64(rk, rv):
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], d=64, r_k=rk, r_v=rv)
    _run(w, CTX_LENS, [0, 9, 31, 100, 7, 128, 1, 700, 4000, 2999], 10000.0, INTER, Tq=4, t0=0,
         units_per_seq=4)


def test_rope_lla2d():
    """LLA-2D codec (heads folded into one latent, ranks 16/32): head h rotates its own
    rebuilt key slice."""
    w = S.shrink(S.WORKLOADS["lla2d"], r_k=16, r_v=32)
    _run(w, CTX_LENS, CTX_LENS, 10000.0, HALF, Tq=4, t0=0, units_per_seq=4)


def test_rope_long_positions_and_fixed_splits():
    """Contexts past 16k tokens and a query position of 7e4: base angles of 1e4-7e4 rad are
    formed in double precision; fixed split counts change only the work split."""
    lens = [16384, 3, 9000]
    q_pos = [16384, 70000, 9000]
    for ns in (0, 5):
        _run(S.WORKLOADS["longctx-8x16k"], lens, q_pos, 10000.0, HALF, Tq=4, t0=0, units_per_seq=2,
             num_splits=ns)
