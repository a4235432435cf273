"""CPU tests of the C-ABI library: it loads, exports every declared symbol, its
integer accounting is bit-exact against the oracle, and argument checks reject bad
calls before any device work (fake pointers are never dereferenced)."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

import decode_attention_12_b200 as lla
import lla_synth as S
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(lla_\w+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert {"lla_cache_bytes", "lla_encode", "lla_decode_attn"} <= set(names)
    lib = ctypes.CDLL(lla.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lla.status_string(code) and lla.status_string(code) != "unknown status"
    assert lla.status_string(12345) == "unknown status"


@pytest.mark.parametrize("name", sorted(S.WORKLOADS))
def test_cache_bytes_bit_exact_vs_oracle(name):
    w = S.WORKLOADS[name]
    lens = S.context_lengths(w)
    dims = lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v, int(w.fold2d),
                         lla.F32 if w.dtype == "f32" else lla.BF16)
    got = lla.cache_bytes(dims, lens)
    ref = oracle.cache_bytes(w.T, w.L, w.H, w.d, w.r_k, w.r_v, w.fold2d, w.elem_bytes,
                             int(lens.sum()))
    assert got == ref


def test_cache_bytes_random_dims_bit_exact():
    rng = np.random.default_rng(0)
    for _ in range(300):
        T, L, H = (int(v) for v in rng.integers(1, 33, 3))
        d = int(rng.choice([16, 64, 128, 256]))
        rk, rv = (int(v) for v in rng.integers(1, 513, 2))
        fold = int(rng.integers(0, 2))
        dt = int(rng.integers(0, 2))
        lens = rng.integers(0, 20000, size=int(rng.integers(0, 50)))
        dims = lla.make_dims(T, L, H, d, rk, rv, fold, dt)
        got = lla.cache_bytes(dims, lens)
        ref = oracle.cache_bytes(T, L, H, d, rk, rv, bool(fold), 4 if dt == 0 else 2,
                                 int(lens.sum()))
        assert got == ref


def test_capacity_workload_bytes():
    w = S.WORKLOADS["capacity-768x4k"]
    dims = lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v)
    lat, unc, num, den = lla.cache_bytes(dims, [4096] * 768)
    assert lat == 115_964_116_992 and (num, den) == (64, 3)


def test_cache_bytes_errors():
    dims = lla.make_dims(4, 1, 2, 64, 8, 16)
    with pytest.raises(lla.LLAError):
        lla.cache_bytes(dims, [5, -1])
    with pytest.raises(lla.LLAError):
        lla.cache_bytes(lla.make_dims(0, 1, 2, 64, 8, 16), [5])


@pytest.mark.parametrize("gap", [0, 3])
def test_slot_layout_exact(gap):
    lens = np.array([5, 0, 7, 1, 4096, 3], dtype=np.int32)
    starts, total = lla.slot_layout(lens, gap)
    assert starts == list(S.slot_starts(lens, gap))
    assert total == int(lens.sum()) + gap * len(lens)
    big = [2 ** 31 - 1] * 8
    starts, total = lla.slot_layout(big, 0)
    assert total == 8 * (2 ** 31 - 1) and starts[-1] == 7 * (2 ** 31 - 1)


# ---- argument checks (no device memory is touched: fake aligned pointers) ------------
FAKE = 1 << 40   # 16-byte aligned, never dereferenced


def _decode_args(**over):
    dims = lla.make_dims(4, 1, 16, 128, 16, 32)
    codec = lla.make_codec(W_up_k=FAKE, W_up_v=FAKE, mu_k=FAKE, mu_v=FAKE)
    cache = lla.make_cache(FAKE, FAKE, 1000)
    a = dict(dims=dims, layer=0, t0=0, Tq=4, q=FAKE, cache=cache, seq_start=FAKE, ctx_lens=FAKE,
             B=2, max_ctx=100, codec=codec, softmax_scale=1.0, out=FAKE, lse=None,
             workspace=FAKE, ws_bytes=1 << 30, variant=lla.ABSORB, num_splits=0, stream=0)
    a.update(over)
    return a


def _rc(**over):
    try:
        lla.decode_attn(**_decode_args(**over))
    except lla.LLAError as e:
        return e.code
    return 0


def test_decode_argument_errors():
    assert _rc(layer=1) == lla.LLA_ERR_INVALID
    assert _rc(t0=1) == lla.LLA_ERR_INVALID          # t0 + Tq > T
    assert _rc(Tq=0) == lla.LLA_ERR_INVALID
    assert _rc(max_ctx=-1) == lla.LLA_ERR_INVALID
    assert _rc(variant=7) == lla.LLA_ERR_INVALID
    assert _rc(q=0) == lla.LLA_ERR_INVALID
    assert _rc(q=FAKE + 2) == lla.LLA_ERR_MISALIGNED
    assert _rc(out=FAKE + 8) == lla.LLA_ERR_MISALIGNED
    assert _rc(ws_bytes=64) == lla.LLA_ERR_WORKSPACE
    assert _rc(workspace=0) == lla.LLA_ERR_WORKSPACE
    assert _rc(dims=lla.make_dims(4, 1, 16, 128, 0, 32)) == lla.LLA_ERR_INVALID
    assert _rc(dims=lla.make_dims(4, 1, 16, 128, 12, 32)) == lla.LLA_ERR_UNSUPPORTED  # 24 B rows
    assert _rc(dims=lla.make_dims(4, 1, 16, 128, 16, 32, 0, 5)) == lla.LLA_ERR_INVALID
    # d_head above the combine's 512 columns: refused before anything is queued
    assert _rc(dims=lla.make_dims(4, 1, 16, 1024, 16, 32)) == lla.LLA_ERR_UNSUPPORTED
    assert _rc(B=0) == 0  # nothing to do, nothing launched


def _hybrid_rc(window=None, **over):
    a = _decode_args(**over)
    if window is None:
        window = lla.make_window(FAKE, FAKE, FAKE, 128, a["B"])
    try:
        lla.decode_attn_hybrid(window=window, **a)
    except lla.LLAError as e:
        return e.code
    return 0


def test_hybrid_argument_errors():
    assert _hybrid_rc(layer=1) == lla.LLA_ERR_INVALID
    assert _hybrid_rc(window=lla.make_window(FAKE, FAKE, FAKE, -1, 2)) == lla.LLA_ERR_INVALID
    assert _hybrid_rc(window=lla.make_window(FAKE, FAKE, FAKE, 128, 1)) == lla.LLA_ERR_INVALID  # seqs < B
    assert _hybrid_rc(window=lla.make_window(FAKE, FAKE, 0, 128, 2)) == lla.LLA_ERR_INVALID
    assert _hybrid_rc(window=lla.make_window(0, FAKE, FAKE, 128, 2)) == lla.LLA_ERR_INVALID
    assert _hybrid_rc(window=lla.make_window(FAKE + 8, FAKE, FAKE, 128, 2)) == lla.LLA_ERR_MISALIGNED
    assert _hybrid_rc(window=lla.make_window(FAKE, FAKE, FAKE + 4, 128, 2)) == lla.LLA_ERR_MISALIGNED
    # bf16 rows of 512 bytes at most (d_head <= 256)
    assert _hybrid_rc(dims=lla.make_dims(4, 1, 16, 512, 16, 32)) == lla.LLA_ERR_UNSUPPORTED
    assert _hybrid_rc(B=0) == 0
    # a NULL window is rejected by the hybrid entry itself
    rc = lla._lib.lla_decode_attn_hybrid(None, 0, 0, 4, None, None, None, None, 2, 100, None, None,
                                         1.0, 0, 0, None, None, None, 0, None)
    assert rc == lla.LLA_ERR_INVALID


def _rope_rc(rope=None, **over):
    a = _decode_args(**over)
    a.pop("variant")
    if rope is None:
        rope = lla.make_rope(FAKE, 10000.0, lla.ROPE_HALF)
    try:
        lla.decode_attn_rope(rope=rope, **a)
    except lla.LLAError as e:
        return e.code
    return 0


def test_rope_argument_errors():
    assert _rope_rc(layer=1) == lla.LLA_ERR_INVALID
    assert _rope_rc(rope=lla.make_rope(0, 10000.0, lla.ROPE_HALF)) == lla.LLA_ERR_INVALID
    assert _rope_rc(rope=lla.make_rope(FAKE, 10000.0, 7)) == lla.LLA_ERR_INVALID
    assert _rope_rc(rope=lla.make_rope(FAKE, 1.0, lla.ROPE_HALF)) == lla.LLA_ERR_INVALID
    assert _rope_rc(rope=lla.make_rope(FAKE, float("nan"), lla.ROPE_HALF)) == lla.LLA_ERR_INVALID
    assert _rope_rc(rope=lla.make_rope(FAKE + 4, 10000.0, lla.ROPE_HALF)) == lla.LLA_ERR_MISALIGNED
    # ranks the reconstruct kernels do not cover
    assert _rope_rc(dims=lla.make_dims(4, 1, 16, 128, 96, 160)) == lla.LLA_ERR_UNSUPPORTED
    assert _rope_rc(B=0) == 0
    rc = lla._lib.lla_decode_attn_rope(None, 0, 0, 4, None, None, None, None, 2, 100, None, None,
                                       1.0, 0, None, None, None, 0, None)
    assert rc == lla.LLA_ERR_INVALID


def test_codec_residual_argument_errors():
    codec = lla.make_codec(W_down_k=FAKE, W_down_v=FAKE, bias_k=FAKE, bias_v=FAKE, W_up_k=FAKE,
                           W_up_v=FAKE, mu_k=FAKE, mu_v=FAKE)

    def rc(dims=None, codec=codec, **over):
        dims = dims or lla.make_dims(4, 2, 16, 128, 16, 32)
        a = dict(layer0=0, n_layers=1, x_k=FAKE, x_v=FAKE, n_tok=10, err_k=FAKE, norm_k=FAKE,
                 err_v=FAKE, norm_v=FAKE, stream=0)
        a.update(over)
        try:
            lla.codec_residual(dims, codec=codec, **a)
        except lla.LLAError as e:
            return e.code
        return 0

    assert rc(layer0=2) == lla.LLA_ERR_INVALID
    assert rc(n_tok=-1) == lla.LLA_ERR_INVALID
    assert rc(x_k=0) == lla.LLA_ERR_INVALID
    assert rc(err_v=0) == lla.LLA_ERR_INVALID
    assert rc(codec=lla.make_codec(W_down_k=FAKE, W_down_v=FAKE)) == lla.LLA_ERR_INVALID
    assert rc(x_v=FAKE + 2) == lla.LLA_ERR_MISALIGNED
    assert rc(dims=lla.make_dims(4, 2, 16, 128, 16, 24)) == lla.LLA_ERR_UNSUPPORTED   # rank 24
    assert rc(dims=lla.make_dims(4, 2, 16, 96, 16, 32)) == lla.LLA_ERR_UNSUPPORTED    # d = 96
    assert rc(dims=lla.make_dims(4, 2, 16, 128, 16, 32, 0, lla.F32)) == lla.LLA_ERR_UNSUPPORTED
    assert rc(n_tok=0) == 0 and rc(n_layers=0) == 0


def test_decoupled_argument_errors():
    def rc(d_rope=64, k_rope=FAKE, q_rope=FAKE, rope=None, **over):
        a = _decode_args(**over)
        a.pop("variant")
        rope = rope if rope is not None else lla.make_rope(FAKE, 10000.0, lla.ROPE_HALF)
        try:
            lla.decode_attn_decoupled(k_rope=k_rope, q_rope=q_rope, d_rope=d_rope, rope=rope, **a)
        except lla.LLAError as e:
            return e.code
        return 0

    assert rc(layer=1) == lla.LLA_ERR_INVALID
    assert rc(k_rope=0) == lla.LLA_ERR_INVALID
    assert rc(d_rope=0) == lla.LLA_ERR_INVALID
    assert rc(q_rope=FAKE + 2) == lla.LLA_ERR_MISALIGNED
    assert rc(d_rope=48) == lla.LLA_ERR_UNSUPPORTED
    assert rc(dims=lla.make_dims(4, 1, 16, 128, 32, 32)) == lla.LLA_ERR_UNSUPPORTED
    assert rc(rope=lla.make_rope(0, 10000.0, lla.ROPE_HALF)) == lla.LLA_ERR_INVALID
    assert rc(B=0) == 0
    dims = lla.make_dims(4, 1, 16, 128, 16, 32)
    base = lla.decode_workspace_bytes(dims, 64, 4, 4096)
    assert lla.decode_decoupled_workspace_bytes(dims, 64, 4, 4096, 64) >= base + 64 * 16 * 4 * 64 * 4


def test_hybrid_workspace_adds_one_window_record_per_query():
    dims = lla.make_dims(4, 1, 16, 128, 16, 32)
    base = lla.decode_workspace_bytes(dims, 64, 4, 4096)
    hyb = lla.decode_hybrid_workspace_bytes(dims, 64, 4, 4096)
    assert hyb >= base + 64 * 16 * 4 * (128 + 4) * 4
    assert hyb - base < 64 * 16 * 4 * (128 + 4) * 4 + 256


def test_timed_entry_needs_both_events():
    a = _decode_args()
    rc = lla._lib.lla_decode_attn_timed(ctypes.byref(a["dims"]), 0, 0, 4, FAKE, ctypes.byref(a["cache"]), FAKE,
                                        FAKE, 2, 100, ctypes.byref(a["codec"]), 1.0, 0, 0, FAKE, None, FAKE,
                                        1 << 30, None, None, FAKE)
    assert rc == lla.LLA_ERR_INVALID


def test_codec_fit_argument_errors():
    codec = lla.make_codec(W_down_k=FAKE, W_down_v=FAKE, W_up_k=FAKE, W_up_v=FAKE, mu_k=FAKE, mu_v=FAKE)
    dims = lla.make_dims(4, 2, 16, 128, 16, 32)

    def rc(n_cal=256, **over):
        a = dict(layer0=0, n_layers=1, x_k=FAKE, x_v=FAKE, workspace=FAKE, ws_bytes=1 << 40, stream=0)
        a.update(over)
        try:
            lla.codec_fit(over.pop("dims", dims), a["layer0"], a["n_layers"], a["x_k"], a["x_v"], n_cal,
                          over.get("codec", codec), a["workspace"], a["ws_bytes"], stream=0)
        except lla.LLAError as e:
            return e.code
        return 0

    assert rc(layer0=2) == lla.LLA_ERR_INVALID
    assert rc(n_cal=255) == lla.LLA_ERR_INVALID          # odd
    assert rc(n_cal=2048) == lla.LLA_ERR_INVALID         # above 1024
    assert rc(n_cal=32) == lla.LLA_ERR_INVALID           # r_v = 32 > n - 1
    assert rc(x_v=0) == lla.LLA_ERR_INVALID
    assert rc(x_k=FAKE + 8) == lla.LLA_ERR_MISALIGNED
    assert rc(ws_bytes=1024) == lla.LLA_ERR_WORKSPACE
    assert rc(n_layers=0) == 0
    n = lla.codec_fit_workspace_bytes(dims, 1, 256)
    assert n >= 16 * (2 * 256 * 256 * 8)


def test_selftest_argument_errors():
    assert lla._lib.lla_selftest_wait_timeout(None, None) == lla.LLA_ERR_INVALID
    assert lla._lib.lla_selftest_wait_timeout(FAKE + 4, None) == lla.LLA_ERR_MISALIGNED


def test_workspace_bytes_and_splits():
    dims = lla.make_dims(4, 1, 16, 128, 16, 32)
    s = lla.decode_num_splits(dims, 64, 4, 4096)
    assert s >= 1
    ws = lla.decode_workspace_bytes(dims, 64, 4, 4096)
    assert ws >= 256 + 64 * 16 * 4 * s * (32 + 4) * 4
    # 7 shares of >= ceil(4096/7) = 586 tokens: a context spans at most 8 of them
    assert lla.decode_num_splits(dims, 64, 4, 4096, num_splits=7) == 8
    with pytest.raises(lla.LLAError):
        lla.decode_workspace_bytes(dims, 64, 0, 4096)


def test_encode_argument_errors():
    dims = lla.make_dims(4, 2, 16, 128, 96, 160)
    codec = lla.make_codec(W_down_k=FAKE, W_down_v=FAKE, bias_k=FAKE, bias_v=FAKE)
    cache = lla.make_cache(FAKE, FAKE, 10)

    def rc(**over):
        a = dict(dims=dims, layer0=0, n_layers=1, x_k=FAKE, x_v=FAKE, n_tok=4, slot_idx=FAKE,
                 codec=codec, cache=cache, stream=0)
        a.update(over)
        try:
            lla.encode(**a)
        except lla.LLAError as e:
            return e.code
        return 0

    assert rc(layer0=2) == lla.LLA_ERR_INVALID
    assert rc(layer0=1, n_layers=2) == lla.LLA_ERR_INVALID
    assert rc(x_k=FAKE + 4) == lla.LLA_ERR_MISALIGNED
    assert rc(x_v=0) == lla.LLA_ERR_INVALID
    assert rc(n_tok=0) == 0
    assert rc(dims=lla.make_dims(4, 2, 16, 128, 320, 160)) == lla.LLA_ERR_UNSUPPORTED


def test_plain_c_program_links_and_calls_the_library(tmp_path):
    """The header is plain C99 and a C program linked against liblla.so gets the exact
    accounting of the 768 x 4096-token capacity case (no device needed)."""
    import subprocess
    src = tmp_path / "main.c"
    src.write_text(r'''
#include <stdio.h>
#include "lla.h"
int main(void)
{
    lla_dims d = {4, 24, 16, 128, 16, 32, LLA_PER_HEAD, LLA_BF16, LLA_F32};
    int32_t lens[768];
    for (int i = 0; i < 768; ++i) lens[i] = 4096;
    uint64_t lat = 0, unc = 0, num = 0, den = 0;
    int rc = lla_cache_bytes(&d, lens, 768, &lat, &unc, &num, &den);
    printf("%d %llu %llu %llu\n", rc, (unsigned long long)lat, (unsigned long long)num, (unsigned long long)den);
    return rc;
}
''')
    exe = tmp_path / "main"
    libdir = os.path.dirname(lla.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-I", os.path.join(ROOT, "include"),
                           str(src), "-L", libdir, "-llla", "-Wl,-rpath," + libdir, "-o", str(exe)])
    out = subprocess.check_output([str(exe)], text=True).split()
    assert out == ["0", "115964116992", "64", "3"]


def test_binding_refuses_strided_views():
    """No strides cross the ABI: the binding passes dense buffers' addresses and refuses a
    strided view instead of letting the library read it as dense."""
    import torch
    dense = torch.zeros(4, 6)
    assert lla._ptr(dense) == dense.data_ptr()
    assert lla._ptr(dense[1:3]) == dense[1:3].data_ptr()       # a row range is still dense
    assert lla._ptr(None) is None and lla._ptr(12345) == 12345
    for view in (dense.t(), dense[:, 1:3], dense[:, None].expand(4, 2, 6)):
        with pytest.raises(ValueError, match="dense row-major"):
            lla._ptr(view)
    with pytest.raises(ValueError):
        lla.make_cache(dense.t(), dense, 4)
