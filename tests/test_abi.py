"""The C-ABI library builds, loads and exports every entry point of
include/loopkv.h, and rejects bad arguments before touching the GPU.

No test here launches a kernel: argument errors return before any CUDA call,
so these run on a machine without a GPU.
"""

import ctypes
import math
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    import mixed_precision_kv_loopkv_b200 as pkg  # built at session start (conftest)
    return pkg


def _header_functions():
    text = open(os.path.join(ROOT, "include", "loopkv.h")).read()
    return re.findall(r"LOOPKV_API\s+[\w\s\*]+?\b(loopkv_\w+)\s*\(", text)


def test_every_header_function_is_exported(m):
    names = _header_functions()
    assert len(names) == 10, names
    lib = ctypes.CDLL(m.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings(m):
    assert m.loopkv_status_string(0) == "ok"
    assert "invalid" in m.loopkv_status_string(1)
    assert m.loopkv_status_string(99) == "unknown status"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
def test_record_bytes_agree_with_oracle_layout(m, d, kind):
    assert m.loopkv_record_bytes(d, kind) == O.record_bytes(kind, d)


def test_record_bytes_rejects_unsupported(m):
    assert m.loopkv_record_bytes(96, "q4") == 0
    assert m.loopkv_record_bytes(128, "q4", block_size=32) == 0
    assert m.loopkv_record_bytes(128, "reuse") == 0


def _cfg(m, plan, L, N, **kw):
    buf = (ctypes.c_uint8 * len(plan))(*plan)
    args = dict(num_loops=L, num_layers=N, num_heads=2, head_dim=128, block_size=16, num_blocks=8,
                max_batch=2, max_blocks_per_seq=4, flags=0, decode_splits=0)
    args.update(kw)
    from mixed_precision_kv_loopkv_b200.loopkv import loopkv_config
    cfg = loopkv_config(**args, plan=ctypes.cast(buf, ctypes.POINTER(ctypes.c_uint8)))
    cfg._buf = buf
    return cfg


def _cells(m, n):
    from mixed_precision_kv_loopkv_b200.loopkv import loopkv_cells
    fake = 0x10000  # never dereferenced: every call below fails validation first
    a = (ctypes.c_void_p * n)(*([fake] * n))
    r = (ctypes.c_void_p * n)(*([fake] * n))
    c = loopkv_cells(ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p)),
                     ctypes.cast(r, ctypes.POINTER(ctypes.c_void_p)))
    c._keep = (a, r)
    return c


FAKE = ctypes.c_void_p(0x20000)


def _decode(m, cfg, cells, loop=0, layer=0, tau=0.01, batch=1, max_seq_len=0, q=FAKE, sm_scale=1.0,
            k_cur=None, v_cur=None):
    lib = m.library()
    return lib.loopkv_decode_attention(ctypes.byref(cfg), ctypes.byref(cells), loop, layer, q, k_cur, v_cur,
                                       FAKE, FAKE, batch, max_seq_len, tau, sm_scale, FAKE, None, None, None,
                                       None)


def _append(m, cfg, cells, loop=0, layer=0, batch=1, T=1, k=FAKE):
    lib = m.library()
    return lib.loopkv_quantize_append(ctypes.byref(cfg), ctypes.byref(cells), loop, layer, k, FAKE, FAKE,
                                      FAKE, batch, T, None, None)


Q4, Q2, REUSE, BF16 = 0, 1, 2, 3


def test_reuse_in_final_loop_is_bad_plan(m):
    cfg = _cfg(m, [Q4, Q2, REUSE, Q4], 2, 2)
    assert _decode(m, cfg, _cells(m, 4)) == 2
    assert _append(m, cfg, _cells(m, 4)) == 2


def test_unknown_kind_is_bad_plan(m):
    cfg = _cfg(m, [Q4, 7], 1, 2)
    assert _decode(m, cfg, _cells(m, 2)) == 2


def test_append_to_reuse_cell_is_invalid(m):
    cfg = _cfg(m, [REUSE, Q4], 2, 1)
    assert _append(m, cfg, _cells(m, 2), loop=0) == 1


@pytest.mark.parametrize("tau", [-1e-3, float("nan"), -math.inf])
def test_bad_tau_is_invalid(m, tau):
    cfg = _cfg(m, [Q4], 1, 1)
    assert _decode(m, cfg, _cells(m, 1), tau=tau) == 1


def test_infinite_sm_scale_is_invalid(m):
    cfg = _cfg(m, [Q4], 1, 1)
    assert _decode(m, cfg, _cells(m, 1), sm_scale=math.inf) == 1


@pytest.mark.parametrize("d,bs,expect", [(96, 16, 3), (128, 32, 3), (32, 16, 3)])
def test_unsupported_shapes(m, d, bs, expect):
    cfg = _cfg(m, [Q4], 1, 1, head_dim=d, block_size=bs)
    assert _decode(m, cfg, _cells(m, 1)) == expect


def test_out_of_range_cell_and_batch(m):
    cfg = _cfg(m, [Q4, Q4], 1, 2)
    assert _decode(m, cfg, _cells(m, 2), layer=2) == 1
    assert _decode(m, cfg, _cells(m, 2), loop=-1) == 1
    assert _decode(m, cfg, _cells(m, 2), batch=3) == 1
    assert _append(m, cfg, _cells(m, 2), batch=-1) == 1
    assert _append(m, cfg, _cells(m, 2), T=-2) == 1


def test_max_seq_len_checks(m):
    cfg = _cfg(m, [Q4], 1, 1, max_blocks_per_seq=8)
    assert _decode(m, cfg, _cells(m, 1), max_seq_len=8 * 16 + 1) == 1
    big = _cfg(m, [Q4], 1, 1, max_blocks_per_seq=8192)
    assert _decode(m, big, _cells(m, 1), max_seq_len=8192 * 16) == 3


def test_misaligned_or_null_buffers(m):
    cfg = _cfg(m, [Q4], 1, 1)
    assert _decode(m, cfg, _cells(m, 1), q=ctypes.c_void_p(0x20004)) == 1
    assert _decode(m, cfg, _cells(m, 1), q=None) == 1
    assert _append(m, cfg, _cells(m, 1), k=ctypes.c_void_p(0x20002)) == 1


def test_bad_split_override(m):
    cfg = _cfg(m, [Q4], 1, 1, decode_splits=3)
    assert _decode(m, cfg, _cells(m, 1)) == 1


def test_split_choice(m):
    from mixed_precision_kv_loopkv_b200.loopkv import library
    lib = library()
    for batch, heads, n in [(8, 16, 2048), (64, 16, 8192), (16, 16, 16384), (1, 2, 256), (1, 1, 65536)]:
        cfg = _cfg(m, [Q4], 1, 1, num_heads=heads, max_batch=batch, max_blocks_per_seq=n // 16)
        s = lib.loopkv_decode_splits(ctypes.byref(cfg), Q4, batch, n)
        assert s in (1, 2, 4, 8)
        assert math.ceil(math.ceil(n / 32) / s) <= 512
    cfg = _cfg(m, [Q4], 1, 1, decode_splits=4)
    assert lib.loopkv_decode_splits(ctypes.byref(cfg), Q4, 2, 64) == 4


def _fused(m, cfg, cells, loop=0, layer=0, k=FAKE, v=FAKE, batch=1, tau=0.01):
    lib = m.library()
    return lib.loopkv_append_decode_attention(ctypes.byref(cfg), ctypes.byref(cells), loop, layer, k, v, FAKE,
                                              FAKE, FAKE, batch, 0, tau, 1.0, FAKE, None, None, None, None)


def test_fused_step_argument_errors(m):
    cfg = _cfg(m, [REUSE, Q4], 2, 1)
    assert _fused(m, cfg, _cells(m, 2), loop=0) == 1          # reuse cells store nothing
    assert _fused(m, cfg, _cells(m, 2), loop=1, k=None) == 1  # the new token is required
    assert _fused(m, cfg, _cells(m, 2), loop=1, v=ctypes.c_void_p(0x20008)) == 1
    assert _fused(m, cfg, _cells(m, 2), loop=1, tau=-1.0) == 1
    bad = _cfg(m, [Q4, REUSE], 2, 1)
    assert _fused(m, bad, _cells(m, 2), loop=0) == 2


def test_two_selection_units_are_invalid(m):
    cfg = _cfg(m, [Q4], 1, 1, flags=0x2 | 0x4)
    assert _decode(m, cfg, _cells(m, 1)) == 1


def test_grouped_query_config_checks(m):
    """KV heads must divide the query heads, with 1, 2, 4 or 8 query heads
    per KV head; a 4-bit source clusters G heads x splits <= 16 CTAs; the
    fused append + decode takes no grouped queries."""
    assert _decode(m, _cfg(m, [Q4], 1, 1, num_heads=6, num_kv_heads=4), _cells(m, 1)) == 1
    assert _decode(m, _cfg(m, [Q4], 1, 1, num_kv_heads=-1), _cells(m, 1)) == 1
    assert _decode(m, _cfg(m, [Q4], 1, 1, num_heads=6, num_kv_heads=2), _cells(m, 1)) == 3   # G = 3
    assert _decode(m, _cfg(m, [Q4], 1, 1, num_heads=32, num_kv_heads=2), _cells(m, 1)) == 3  # G = 16
    assert _append(m, _cfg(m, [Q4], 1, 1, num_heads=6, num_kv_heads=2), _cells(m, 1)) == 3
    assert _decode(m, _cfg(m, [Q4], 1, 1, num_heads=8, num_kv_heads=2, decode_splits=8), _cells(m, 1)) == 3
    assert _fused(m, _cfg(m, [Q4], 1, 1, num_heads=4, num_kv_heads=2), _cells(m, 1)) == 3


def test_grouped_query_sizes_and_splits(m):
    lib = m.library()
    gqa = _cfg(m, [Q4], 1, 1, num_heads=8, num_kv_heads=2)
    mha = _cfg(m, [Q4], 1, 1, num_heads=2)
    for kind in (Q4, Q2, BF16):
        assert lib.loopkv_arena_bytes(ctypes.byref(gqa), kind) == lib.loopkv_arena_bytes(ctypes.byref(mha), kind)
    assert lib.loopkv_residual_bytes(ctypes.byref(gqa)) == lib.loopkv_residual_bytes(ctypes.byref(mha))
    for g, smax in [(2, 8), (4, 4), (8, 2)]:
        cfg = _cfg(m, [Q4], 1, 1, num_heads=2 * g, num_kv_heads=2, max_blocks_per_seq=4096)
        for n in (256, 8192, 65536):
            assert 1 <= lib.loopkv_decode_splits(ctypes.byref(cfg), Q4, 1, n) <= smax
        # 2-bit sources select nothing: their splits are not capped
        assert lib.loopkv_decode_splits(ctypes.byref(cfg), Q2, 1, 65536) == 8
        over = _cfg(m, [Q4], 1, 1, num_heads=2 * g, num_kv_heads=2, decode_splits=2 * smax)
        if 2 * smax <= 8:
            assert lib.loopkv_decode_splits(ctypes.byref(over), Q4, 1, 64) == 0


def test_grouped_query_split_cap(m):
    """Eight query heads per KV head leave two splits per cluster of 16."""
    big = _cfg(m, [Q4], 1, 1, num_heads=16, num_kv_heads=2, max_blocks_per_seq=4096)
    lib = m.library()
    assert lib.loopkv_decode_splits(ctypes.byref(big), Q4, 1, 16384) == 2
    assert lib.loopkv_decode_splits(ctypes.byref(big), Q4, 1, 65536) == 2


def test_current_token_needs_both_rows(m):
    """k_cur and v_cur come together: one without the other is an argument
    error, reported before anything is launched."""
    cfg = _cfg(m, [Q4, Q2, REUSE, Q4], 2, 2)
    cfg.plan[2] = Q4
    cells = _cells(m, 4)
    assert _decode(m, cfg, cells, k_cur=FAKE) == 1
    assert _decode(m, cfg, cells, v_cur=FAKE) == 1
