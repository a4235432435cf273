"""lla_decode_attn_static: decode attention for callers that cannot allocate device memory.

Some callers have no way to get device memory for a workspace -- a plugin inside a
host framework that owns the whole device pool, or a serving loop that forbids
allocation after start-up.  lla_decode_attn_static keeps its scratch in a fixed 8 MiB
array inside the library instead.  These tests call it through the C ABI and check
that two calls in a row (different loop ranges and queries, so stale scratch from the
first call would show) give the same results as lla_decode_attn with a caller-provided
workspace, within the parity tolerances the other tests use.  The file name makes
pytest collect it last; it needs nothing from the other test files' state.
"""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import ATOL_MAX, LSE_ATOL, RTOL_L2, codec_of, dims_of, run_decode, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _static_call(p, w, t0, Tq, q):
    dims = dims_of(w)
    B = len(p["lens"])
    out = torch.full((B, Tq, w.H, w.d), float("nan"), dtype=torch.float32, device=DEV)
    lse = torch.full((B, Tq, w.H), float("nan"), dtype=torch.float32, device=DEV)
    lla.decode_attn_static(dims, 0, t0, Tq, q, lla.make_cache(p["k"], p["v"], p["slots"]),
                           p["seq_start"], p["ctx_lens"], B, int(p["lens"].max()), codec_of(p), 1.0,
                           out, lse)
    torch.cuda.synchronize()
    return out, lse


def _assert_same(out_a, lse_a, out_b, lse_b):
    a, b = to64(out_a), to64(out_b)
    err = a - b
    assert np.isfinite(a).all()
    assert np.abs(err).max() <= ATOL_MAX
    assert np.linalg.norm(err) / np.linalg.norm(b) <= RTOL_L2
    la, lb = to64(lse_a), to64(lse_b)
    assert np.array_equal(np.isinf(la), np.isinf(lb))
    fin = np.isfinite(lb)
    assert np.abs(la[fin] - lb[fin]).max() <= LSE_ATOL


def test_static_scratch_matches_workspace_entry_point_twice():
    w = S.WORKLOADS["ouro1.4b-layer"]
    p = S.decode_inputs(w, 0, DEV)
    q1 = p["q"]                                            # all 4 loop queries
    q2 = S.draw_queries(w.B, 1, w.H, w.d, 12345, DEV, w.torch_dtype)   # loop 2 only
    ref1 = run_decode(p, w, 0, 0, 4, 1.0, q=q1)
    ref2 = run_decode(p, w, 0, 2, 1, 1.0, q=q2)
    assert ref1[2] == 0 and ref2[2] == 0
    got1 = _static_call(p, w, 0, 4, q1)
    got2 = _static_call(p, w, 2, 1, q2)
    _assert_same(got1[0], got1[1], ref1[0], ref1[1])
    _assert_same(got2[0], got2[1], ref2[0], ref2[1])


def test_static_scratch_rejects_problems_beyond_its_size():
    w = S.WORKLOADS["ouro1.4b-layer"]
    dims = dims_of(w)
    need = lla.decode_workspace_bytes(dims, 64, 4, 4096, lla.ABSORB, 64)
    assert need > lla.STATIC_SCRATCH_BYTES
    p = S.decode_inputs(S.shrink(w, B=2, len_lo=10, len_hi=20), 0, DEV)
    out = torch.empty(64, 4, w.H, w.d, device=DEV)
    with pytest.raises(lla.LLAError) as ei:
        lla.decode_attn_static(dims, 0, 0, 4, p["q"], lla.make_cache(p["k"], p["v"], p["slots"]),
                               p["seq_start"], p["ctx_lens"], 64, 4096, codec_of(p), 1.0, out,
                               None, num_splits=64)
    assert ei.value.code == lla.LLA_ERR_WORKSPACE


def test_static_scratch_reports_device_errors_and_clears_them_per_call():
    """A context longer than max_ctx is a device-side error (LLA_ERR_INVALID in the status
    word).  The static call's word is read with status_fetch_static; a call refused on the
    host queues nothing and leaves the word alone; the next accepted call clears it."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], B=2, len_lo=300, len_hi=500)
    p = S.decode_inputs(w, 0, DEV)
    dims = dims_of(w)
    B = len(p["lens"])
    cache = lla.make_cache(p["k"], p["v"], p["slots"])
    out = torch.full((B, 4, w.H, w.d), float("nan"), dtype=torch.float32, device=DEV)
    lla.status_fetch_static()                      # start from a clear word
    # every context is longer than the max_ctx the scratch was planned for
    assert int(p["lens"].min()) > 100
    lla.decode_attn_static(dims, 0, 0, 4, p["q"], cache, p["seq_start"], p["ctx_lens"], B, 100,
                           codec_of(p), 1.0, out, None)
    torch.cuda.synchronize()
    # refused on the host (no query): nothing is queued, the word keeps the error
    with pytest.raises(lla.LLAError) as ei:
        lla.decode_attn_static(dims, 0, 0, 4, None, cache, p["seq_start"], p["ctx_lens"], B,
                               int(p["lens"].max()), codec_of(p), 1.0, out, None)
    assert ei.value.code == lla.LLA_ERR_INVALID
    assert lla.status_fetch_static() == lla.LLA_ERR_INVALID
    assert lla.status_fetch_static() == 0          # the fetch cleared it
    # an accepted call with the right max_ctx: status clear, results right
    got = _static_call(p, w, 0, 4, p["q"])
    assert lla.status_fetch_static() == 0
    ref = run_decode(p, w, 0, 0, 4, 1.0, q=p["q"])
    assert ref[2] == 0
    _assert_same(got[0], got[1], ref[0], ref[1])
