"""Python binding of the LoopKV C ABI (include/loopkv.h).

Argument marshalling only: every function here converts torch tensors to
device pointers and calls the same-named entry point of libloopkv.so, whose
CUDA kernels do all the work.  PyTorch provides device memory and streams.
There is no fallback: if the library is missing, importing this module fails.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libloopkv.so")

LOOPKV_CELL_Q4, LOOPKV_CELL_Q2, LOOPKV_CELL_REUSE, LOOPKV_CELL_BF16 = 0, 1, 2, 3
KIND_CODES = {"q4": LOOPKV_CELL_Q4, "q2": LOOPKV_CELL_Q2, "reuse": LOOPKV_CELL_REUSE,
              "bf16": LOOPKV_CELL_BF16}
LOOPKV_DEVERR_BLOCK_ID, LOOPKV_DEVERR_SEQ_LEN, LOOPKV_DEVERR_TIMEOUT, LOOPKV_DEVERR_RANGE = 0x1, 0x2, 0x4, 0x8
LOOPKV_FLAG_PDL, LOOPKV_FLAG_SELECT_BLOCK, LOOPKV_FLAG_SELECT_GROUP = 0x1, 0x2, 0x4
STATUS_NAMES = {0: "LOOPKV_OK", 1: "LOOPKV_ERR_INVALID_ARG", 2: "LOOPKV_ERR_BAD_PLAN",
                3: "LOOPKV_ERR_UNSUPPORTED", 4: "LOOPKV_ERR_CUDA"}


class LoopKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} "
                         f"({_lib.loopkv_status_string(status).decode()})")


class loopkv_config(ctypes.Structure):
    _fields_ = [("num_loops", ctypes.c_int32), ("num_layers", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("decode_splits", ctypes.c_int32),
                ("plan", ctypes.POINTER(ctypes.c_uint8)), ("num_kv_heads", ctypes.c_int32)]


class loopkv_cells(ctypes.Structure):
    _fields_ = [("arena", ctypes.POINTER(ctypes.c_void_p)),
                ("key_residual", ctypes.POINTER(ctypes.c_void_p))]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run mixed_precision_kv_loopkv_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, F32, VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p
    sig = {
        "loopkv_record_bytes": (ctypes.c_size_t, [I32, I32, I32]),
        "loopkv_arena_bytes": (ctypes.c_size_t, [P(loopkv_config), I32]),
        "loopkv_residual_bytes": (ctypes.c_size_t, [P(loopkv_config)]),
        "loopkv_quantize_append": (ctypes.c_int, [P(loopkv_config), P(loopkv_cells), I32, I32, VP, VP,
                                                  VP, VP, I32, I32, VP, VP]),
        "loopkv_decode_attention": (ctypes.c_int, [P(loopkv_config), P(loopkv_cells), I32, I32, VP, VP, VP,
                                                   VP, VP, I32, I32, F32, F32, VP, VP, VP, VP, VP]),
        "loopkv_append_decode_attention": (ctypes.c_int, [P(loopkv_config), P(loopkv_cells), I32, I32, VP, VP,
                                                          VP, VP, VP, I32, I32, F32, F32, VP, VP, VP, VP,
                                                          VP]),
        "loopkv_decode_splits": (I32, [P(loopkv_config), I32, I32, I32]),
        "loopkv_plan_cells": (ctypes.c_int, [I32, I32, VP, I32, I32, I32, VP, VP]),
        "loopkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "loopkv_selftest_wait_timeout": (ctypes.c_int, [VP, VP, VP]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def _ptr(t, what, dtype=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{what} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def loopkv_record_bytes(head_dim: int, kind, block_size: int = 16) -> int:
    kind = KIND_CODES.get(kind, kind)
    return int(_lib.loopkv_record_bytes(head_dim, block_size, kind))


def loopkv_status_string(status: int) -> str:
    return _lib.loopkv_status_string(status).decode()


class KVCells:
    """Device storage of every (loop, layer) cell of a looped model.

    Holds one arena uint8[num_blocks * Hkv * record] per stored cell and one
    key residual bf16[max_batch, Hkv, 32, D] per 4-bit or 2-bit cell (torch
    tensors), plus the C structs the entry points take.  ``num_heads`` counts
    query heads; ``num_kv_heads`` (0: as many as query heads) the KV heads
    the cells store.  ``allocate`` (a set of cell indices) restricts storage
    to those cells; the others get null pointers, which the entry points
    reject.
    """

    def __init__(self, plan, num_loops: int, num_layers: int, num_heads: int, head_dim: int,
                 num_blocks: int, max_batch: int, max_blocks_per_seq: int, device="cuda",
                 flags: int = 0, decode_splits: int = 0, block_size: int = 16, allocate=None,
                 num_kv_heads: int = 0):
        codes = [KIND_CODES.get(k, k) for k in plan]
        if len(codes) != num_loops * num_layers:
            raise ValueError("plan must have num_loops * num_layers entries")
        self.plan_codes = codes
        self.num_loops, self.num_layers = num_loops, num_layers
        self.num_heads, self.head_dim = num_heads, head_dim
        self.num_kv_heads = num_kv_heads or num_heads
        self.num_blocks, self.max_batch = num_blocks, max_batch
        self.max_blocks_per_seq, self.block_size = max_blocks_per_seq, block_size
        self._plan_buf = (ctypes.c_uint8 * len(codes))(*codes)
        self.cfg = loopkv_config(num_loops, num_layers, num_heads, head_dim, block_size, num_blocks,
                                 max_batch, max_blocks_per_seq, flags, decode_splits,
                                 ctypes.cast(self._plan_buf, ctypes.POINTER(ctypes.c_uint8)), num_kv_heads)
        self.arenas, self.residuals = [], []
        ptr_a = (ctypes.c_void_p * len(codes))()
        ptr_r = (ctypes.c_void_p * len(codes))()
        for c, kind in enumerate(codes):
            arena = residual = None
            if kind != LOOPKV_CELL_REUSE and (allocate is None or c in allocate):
                nbytes = int(_lib.loopkv_arena_bytes(ctypes.byref(self.cfg), kind))
                arena = torch.zeros(nbytes, dtype=torch.uint8, device=device)
                ptr_a[c] = arena.data_ptr()
                if kind in (LOOPKV_CELL_Q4, LOOPKV_CELL_Q2):
                    residual = torch.zeros((max_batch, self.num_kv_heads, 32, head_dim), dtype=torch.bfloat16,
                                           device=device)
                    ptr_r[c] = residual.data_ptr()
            self.arenas.append(arena)
            self.residuals.append(residual)
        self._ptr_a, self._ptr_r = ptr_a, ptr_r
        self.cells = loopkv_cells(ctypes.cast(ptr_a, ctypes.POINTER(ctypes.c_void_p)),
                                  ctypes.cast(ptr_r, ctypes.POINTER(ctypes.c_void_p)))

    @property
    def flags(self) -> int:
        return self.cfg.flags

    @flags.setter
    def flags(self, v: int):
        self.cfg.flags = v

    @property
    def decode_splits(self) -> int:
        return self.cfg.decode_splits

    @decode_splits.setter
    def decode_splits(self, v: int):
        self.cfg.decode_splits = v

    def source_cell(self, cell: int) -> int:
        if self.plan_codes[cell] == LOOPKV_CELL_REUSE:
            return (self.num_loops - 1) * self.num_layers + cell % self.num_layers
        return cell

    def record_bytes(self, kind) -> int:
        return loopkv_record_bytes(self.head_dim, kind, self.block_size)

    def arena_view(self, cell: int) -> torch.Tensor:
        """Arena of a stored cell as uint8[num_blocks, Hkv, record]."""
        a = self.arenas[cell]
        return a.view(self.num_blocks, self.num_kv_heads, -1)


def loopkv_quantize_append(kv: KVCells, loop: int, layer: int, k_new, v_new, block_table, start_pos,
                           err_flag=None, stream=None):
    """Append k_new, v_new bf16[B, T, Hkv, D] at positions start_pos[b].. (device int32)."""
    if k_new.dim() != 4:
        raise ValueError("k_new must be [batch, tokens, heads, head_dim]")
    batch, tokens = int(k_new.shape[0]), int(k_new.shape[1])
    st = _lib.loopkv_quantize_append(
        ctypes.byref(kv.cfg), ctypes.byref(kv.cells), loop, layer,
        _ptr(k_new, "k_new", torch.bfloat16), _ptr(v_new, "v_new", torch.bfloat16),
        _ptr(block_table, "block_table", torch.int32), _ptr(start_pos, "start_pos", torch.int32),
        batch, tokens, _ptr(err_flag, "err_flag", torch.int32, optional=True), _stream(stream))
    if st:
        raise LoopKVError(st, "loopkv_quantize_append")


def loopkv_decode_attention(kv: KVCells, loop: int, layer: int, q, block_table, seq_lens, tau: float,
                            sm_scale: float = 1.0, out=None, max_seq_len: int = 0, sel_mask=None,
                            sel_count=None, err_flag=None, stream=None, k_cur=None, v_cur=None):
    """Decode attention of q bf16[B, H, D] over cell (loop, layer); returns out bf16[B, H, D].
    k_cur, v_cur (optional bf16 [B, Hkv, D] or [B, 1, Hkv, D]): the current
    token's own K/V, attended exactly after the stored tokens."""
    if out is None:
        out = torch.empty_like(q)
    batch = int(q.shape[0])
    st = _lib.loopkv_decode_attention(
        ctypes.byref(kv.cfg), ctypes.byref(kv.cells), loop, layer, _ptr(q, "q", torch.bfloat16),
        _ptr(k_cur, "k_cur", torch.bfloat16, optional=True), _ptr(v_cur, "v_cur", torch.bfloat16, optional=True),
        _ptr(block_table, "block_table", torch.int32), _ptr(seq_lens, "seq_lens", torch.int32),
        batch, int(max_seq_len), float(tau), float(sm_scale), _ptr(out, "out", torch.bfloat16),
        _ptr(sel_mask, "sel_mask", torch.int32, optional=True),
        _ptr(sel_count, "sel_count", torch.int32, optional=True),
        _ptr(err_flag, "err_flag", torch.int32, optional=True), _stream(stream))
    if st:
        raise LoopKVError(st, "loopkv_decode_attention")
    return out


def loopkv_append_decode_attention(kv: KVCells, loop: int, layer: int, k_new, v_new, q, block_table, start_pos,
                                   tau: float, sm_scale: float = 1.0, out=None, max_seq_len: int = 0,
                                   sel_mask=None, sel_count=None, err_flag=None, stream=None):
    """Append token start_pos[b] (k_new, v_new bf16[B, 1, Hkv, D]) to a stored
    cell and attend q bf16[B, H, D] over start_pos[b] + 1 tokens, in one
    launch; returns out bf16[B, H, D]."""
    if out is None:
        out = torch.empty_like(q)
    if k_new.dim() != 4 or k_new.shape[1] != 1:
        raise ValueError("k_new must be [batch, 1, heads, head_dim]")
    batch = int(q.shape[0])
    st = _lib.loopkv_append_decode_attention(
        ctypes.byref(kv.cfg), ctypes.byref(kv.cells), loop, layer,
        _ptr(k_new, "k_new", torch.bfloat16), _ptr(v_new, "v_new", torch.bfloat16), _ptr(q, "q", torch.bfloat16),
        _ptr(block_table, "block_table", torch.int32), _ptr(start_pos, "start_pos", torch.int32),
        batch, int(max_seq_len), float(tau), float(sm_scale), _ptr(out, "out", torch.bfloat16),
        _ptr(sel_mask, "sel_mask", torch.int32, optional=True),
        _ptr(sel_count, "sel_count", torch.int32, optional=True),
        _ptr(err_flag, "err_flag", torch.int32, optional=True), _stream(stream))
    if st:
        raise LoopKVError(st, "loopkv_append_decode_attention")
    return out


def loopkv_decode_splits(kv: KVCells, kind, batch: int, max_seq_len: int) -> int:
    return int(_lib.loopkv_decode_splits(ctypes.byref(kv.cfg), KIND_CODES.get(kind, kind), batch,
                                         max_seq_len))


def loopkv_plan_cells(damage, damage_budget: int, storage_budget: int, q4_read_bytes: int = 128):
    """Plan every (loop, layer) cell from an integer damage table
    ``damage[loop][layer][choice]`` (choice 0: 4-bit, 1: 2-bit, 2: reuse).
    Returns (plan as kind names in cell order, total reads per token-head)."""
    import numpy as np
    d = np.ascontiguousarray(np.asarray(damage, dtype=np.int32))
    if d.ndim != 3 or d.shape[2] != 3:
        raise ValueError("damage must be [num_loops, num_layers, 3]")
    L, N = int(d.shape[0]), int(d.shape[1])
    plan = (ctypes.c_uint8 * (L * N))()
    reads = ctypes.c_int64(0)
    st = _lib.loopkv_plan_cells(L, N, d.ctypes.data_as(ctypes.c_void_p), int(damage_budget), int(storage_budget),
                                int(q4_read_bytes), ctypes.cast(plan, ctypes.c_void_p), ctypes.byref(reads))
    if st:
        raise LoopKVError(st, "loopkv_plan_cells")
    names = {v: k for k, v in KIND_CODES.items()}
    return [names[int(x)] for x in plan], int(reads.value)


def mask_words(kv: KVCells) -> int:
    return math.ceil(kv.max_blocks_per_seq * kv.block_size / 32)


def loopkv_selftest_wait_timeout(err_flag, elapsed_ns, stream=None):
    """Run the bounded-wait self-test: err_flag int32[1] and elapsed_ns
    int64[1] on the device receive LOOPKV_DEVERR_TIMEOUT and the wait's
    duration (about 2 s)."""
    st = _lib.loopkv_selftest_wait_timeout(_ptr(err_flag, "err_flag", torch.int32),
                                           _ptr(elapsed_ns, "elapsed_ns", torch.int64), _stream(stream))
    if st:
        raise LoopKVError(st, "loopkv_selftest_wait_timeout")
