"""The C-ABI library loads and exports every declared entry point (no GPU needed).

Only host-side logic runs here: symbol table, parameter validation and the
buffer-size query, none of which touches a device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"PRISM_API\s+[\w\s\*]*?\b(prism_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from dynamic_block_sparse_zone_b200 import build as b
    b.build()
    from dynamic_block_sparse_zone_b200.binding import load_library
    return load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert {"prism_plan_create", "prism_plan_build", "prism_attn_fwd", "prism_attn_bwd"} <= names
    for n in names:
        assert hasattr(lib, n), n


def test_binding_names_match_header():
    from dynamic_block_sparse_zone_b200 import binding
    assert set(binding.EXPORTED) == declared_symbols()


def _params(**kw):
    from dynamic_block_sparse_zone_b200.binding import Params
    base = dict(batch=1, T=24, H=96, W=160, heads=24, head_dim=128, top_k=32, top_p=0.95, max_frac=0.0625)
    base.update(kw)
    return Params(**base)


def test_plan_bytes_and_validation(lib):
    from dynamic_block_sparse_zone_b200.binding import prism_plan_bytes
    n = prism_plan_bytes(_params())
    # three permuted copies + dO copy (bf16) + dQ accumulator (fp32) dominate
    N, C = 24 * 96 * 160, 24 * 128
    assert n > N * C * (4 * 2 + 4)
    assert n < 20e9
    assert prism_plan_bytes(_params(T=20)) == 0          # not a multiple of 8
    assert prism_plan_bytes(_params(head_dim=96)) == 0   # unsupported head_dim
    assert prism_plan_bytes(_params(top_k=0)) == 0
    assert prism_plan_bytes(_params(top_p=0.0)) == 0
    assert prism_plan_bytes(_params(top_p=1.5)) == 0
    assert prism_plan_bytes(_params(fixed_shape=(4, 4, 2))) == 0   # volume 32: not a candidate
    assert prism_plan_bytes(_params(fixed_shape=(4, 4, 4))) > 0
    assert prism_plan_bytes(_params(hilbert_block=128)) > 0          # Hilbert-order baseline
    assert prism_plan_bytes(_params(hilbert_block=96)) == 0          # not 64 / 128 / 256
    assert prism_plan_bytes(_params(hilbert_block=64, fixed_shape=(4, 4, 4))) == 0
    assert prism_plan_bytes(_params(T=8, H=8, W=1024, hilbert_block=64)) == 0   # cube side 1024 > 512


def test_create_rejects_bad_params_before_touching_the_device(lib):
    from dynamic_block_sparse_zone_b200.binding import PrismError, PrismPlan
    with pytest.raises(PrismError) as ei:
        PrismPlan(_params(W=12))
    assert "PRISM_ERR_UNSUPPORTED" in str(ei.value) and "macro-zone" in str(ei.value)
    with pytest.raises(PrismError) as ei:
        PrismPlan(_params(top_p=-1.0))
    assert "PRISM_ERR_INVALID_ARG" in str(ei.value)


def test_null_arguments_are_rejected(lib):
    P = ctypes.c_void_p
    assert lib.prism_plan_create(None, None) == 1
    assert lib.prism_plan_build(None, None, None, None, None, None) == 1
    assert lib.prism_attn_fwd(None, None, None, None) == 1
    assert lib.prism_attn_fwd_taylor(None, None, None, None) == 1
    assert lib.prism_attn_bwd(None, None, None, None, None, None, None) == 1
    assert lib.prism_plan_build_stats(None, None, None, None) == 1
    assert lib.prism_plan_build_finish(None, None, None, None, None) == 1
    assert lib.prism_plan_stats_slice(None, None, None, None, None) == 1
    assert lib.prism_plan_build_with_zones(None, None, None, None, None, None, None) == 1
    assert b"NULL" in lib.prism_last_error()
    lib.prism_plan_destroy(None)  # no-op


def test_audio_norm_arguments_are_checked_on_the_host(lib):
    assert lib.prism_audio_norms(None, None, 1, 8, 8, 8, 16, None) == 1
    dummy = ctypes.c_void_p(16)  # never dereferenced: the sizes are rejected first
    assert lib.prism_audio_norms(dummy, dummy, 0, 8, 8, 8, 16, None) == 1
    assert lib.prism_audio_norms(dummy, dummy, 1, 8, 8, 8, 0, None) == 1
    assert b"channels" in lib.prism_last_error()


def test_host_step_arguments_are_checked_on_the_host(lib):
    from dynamic_block_sparse_zone_b200.binding import prism_host_io
    io = prism_host_io()
    tk = ctypes.c_ulonglong()
    assert lib.prism_step_host(None, ctypes.byref(io), None, ctypes.byref(tk)) == 1
    assert lib.prism_step_host(None, None, None, None) == 1
    assert lib.prism_step_join(None, 1, None) == 1
    assert lib.prism_step_wait(None, 1) == 1
    assert b"NULL" in lib.prism_last_error()


def test_timer_names_cover_every_id(lib):
    from dynamic_block_sparse_zone_b200.binding import NUM_TIMERS
    names = [lib.prism_timer_name(k).decode() for k in range(NUM_TIMERS)]
    assert len(set(names)) == NUM_TIMERS and all(names)
    assert {"zone_stats_v", "permute_pool", "select", "attn_fwd", "attn_bwd", "attn_fwd_taylor"} <= set(names)
    assert lib.prism_timer_name(NUM_TIMERS) == b"" and lib.prism_timer_name(-1) == b""
