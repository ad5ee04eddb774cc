"""Python binding of libpkv.so (include/pkv.h): argument marshalling only.

Every step of the hot path runs in the library's sm_100a kernels; torch supplies device memory and
the current CUDA stream. There is no fallback: if the shared library is missing or cannot be loaded,
importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m paged_kv_cache_446_b200.build` "
                      "(or __graft_entry__.build())")
_lib = ctypes.CDLL(LIB_PATH)

PKV_OK = 0
STATUS = {0: "PKV_OK", 1: "PKV_ERR_INVALID_ARG", 2: "PKV_ERR_UNSUPPORTED", 3: "PKV_ERR_CUDA",
          4: "PKV_ERR_WORKSPACE_TOO_SMALL", 5: "PKV_ERR_DEVICE_TIMEOUT", 6: "PKV_ERR_DEVICE_RANGE",
          7: "PKV_ERR_OUT_OF_BLOCKS"}
PKV_ERR_OUT_OF_BLOCKS = 7
DTYPE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
DTYPE_NAME = {"f32": 0, "f16": 1, "bf16": 2}

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t


class PlanOptions(ctypes.Structure):
    _fields_ = [("split_blocks", ctypes.c_int32), ("no_split", ctypes.c_int32),
                ("cuda_core_only", ctypes.c_int32), ("num_sms", ctypes.c_int32), ("heads_per_item", ctypes.c_int32),
                ("rows_per_item", ctypes.c_int32), ("tc_min_rows", ctypes.c_int32), ("decode_kernel", ctypes.c_int32),
                ("h_block_tables", ctypes.c_void_p), ("block_table_stride", ctypes.c_int32),
                ("min_shared_blocks", ctypes.c_int32), ("decode_sms", ctypes.c_int32)]


class Plan(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32)] + [(n, ctypes.c_int32) for n in (
        "num_reqs", "num_q_tokens", "num_q_heads", "num_kv_heads", "head_dim", "dtype", "num_decode_rows",
        "num_prefill_rows", "num_items", "num_tiles", "num_merge_rows", "num_partials", "split_blocks",
        "max_blocks", "heads_per_item", "rows_per_item", "decode_kernel", "part_stride", "merge_slots")] + [(n, ctypes.c_int64) for n in (
        "off_items", "off_tiles", "off_merge", "off_part_o", "off_part_ml", "meta_bytes", "ws_bytes", "kv_bytes",
        "attn_flops", "core_kv_bytes", "tile_kv_bytes", "tile_flops")] + [
        ("decode_sms", ctypes.c_int32), ("flags", ctypes.c_uint32)]


def _sig(name, restype, argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = argtypes
    return f


_lib.pkv_status_string.restype = ctypes.c_char_p
_lib.pkv_status_string.argtypes = [_I]
_lib.pkv_last_error.restype = ctypes.c_char_p
_lib.pkv_version.restype = ctypes.c_char_p
_slot_mapping = _sig("pkv_slot_mapping", _I, [_P, _I, _P, _P, _I, _I, _P, _I, _P])
_kv_cache_write = _sig("pkv_kv_cache_write", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P])
_copy_blocks = _sig("pkv_copy_blocks", _I, [_P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P])
_ws_size = _sig("pkv_attention_workspace_size", _I, [_P, _P, _I, _I, _I, _I, _I, _P, ctypes.POINTER(_SZ)])
_plan_host = _sig("pkv_attention_plan_host", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _SZ, ctypes.POINTER(Plan)])
_plan = _sig("pkv_attention_plan", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _SZ, ctypes.POINTER(Plan), _P])
_plan_async = _sig("pkv_attention_plan_async", _I,
                   [_P, _P, _I, _I, _I, _I, _I, _P, _P, _SZ, _P, _SZ, _P, _P, ctypes.POINTER(Plan), _P])
_attention = _sig("pkv_paged_attention", _I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _F, ctypes.POINTER(Plan), _P, _SZ, _P])
_validate_tables = _sig("pkv_validate_tables", _I, [_P, _P, _I, _I, _I])
_validate_slots = _sig("pkv_validate_slots", _I, [_P, _I, _I])
_validate_pairs = _sig("pkv_validate_copy_pairs", _I, [_P, _I, _I])
_device_error = _sig("pkv_device_error", _I, [ctypes.POINTER(_I), ctypes.POINTER(_I64), _P])
_profile_start = _sig("pkv_profile_start", _I, [_I])
_profile_stop = _sig("pkv_profile_stop", _I, [_P, _P, _P])
KERNEL_KINDS = ("slot_mapping", "kv_write", "copy_blocks", "decode", "merge", "prefill_tc")


class PkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.pkv_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")


def _check(status: int, where: str):
    if status != PKV_OK:
        raise PkvError(status, where)


def version() -> str:
    return _lib.pkv_version().decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(_P)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in DTYPE:
        raise TypeError(f"unsupported element type {t.dtype}")
    return DTYPE[t.dtype]


def _opts(split_blocks=0, no_split=False, cuda_core_only=False, num_sms=0, heads_per_item=0, rows_per_item=0,
          tc_min_rows=0, decode_kernel=0, shared_tables=None, min_shared_blocks=0, decode_sms=0) -> PlanOptions:
    """Planner options. shared_tables: host int32 block tables [R, max_blocks] for shared-prefix
    detection (the caller keeps the array alive while planning), or None. decode_sms: SMs of the
    split-K kernel when it runs concurrently with the tcgen05 tiles (0 planner's choice, -1 serial)."""
    o = PlanOptions(int(split_blocks), int(bool(no_split)), int(bool(cuda_core_only)), int(num_sms),
                    int(heads_per_item), int(rows_per_item), int(tc_min_rows), int(decode_kernel))
    if shared_tables is not None:
        assert shared_tables.dtype == np.int32 and shared_tables.flags["C_CONTIGUOUS"] and shared_tables.ndim == 2
        o.h_block_tables = shared_tables.ctypes.data
        o.block_table_stride = int(shared_tables.shape[1])
    o.min_shared_blocks = int(min_shared_blocks)
    o.decode_sms = int(decode_sms)
    return o


# ---- a13: mixed-batch flattening -------------------------------------------------------------

def flatten_batch(batch: dict, prior_lens) -> tuple[np.ndarray, np.ndarray]:
    """{request_id: num_tokens} (dict order) + each request's prior context ->
    (query_start_loc int32 [R+1], context_lens int32 [R]) on the host."""
    counts = np.fromiter(batch.values(), dtype=np.int64, count=len(batch))
    qsl = np.zeros(len(batch) + 1, dtype=np.int64)
    np.cumsum(counts, out=qsl[1:])
    ctx = np.asarray(prior_lens, dtype=np.int64).reshape(-1) + counts
    return qsl.astype(np.int32), ctx.astype(np.int32)


# ---- a1 / a2 / a12 -----------------------------------------------------------------------------

def slot_mapping(block_tables: torch.Tensor, query_start_loc: torch.Tensor, context_lens: torch.Tensor,
                 num_blocks: int, num_tokens: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Physical slot (int64) of every token the step appends; device tensors in and out."""
    if out is None:
        out = torch.empty(num_tokens, dtype=torch.int64, device=block_tables.device)
    R = context_lens.shape[0]
    mb = block_tables.shape[1] if block_tables.dim() == 2 else 0
    _check(_slot_mapping(_ptr(block_tables), mb, _ptr(query_start_loc), _ptr(context_lens), R, int(num_blocks),
                         _ptr(out), int(num_tokens), _stream(stream)), "pkv_slot_mapping")
    return out


def kv_cache_write(k_new: torch.Tensor, v_new: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                   slot_mapping: torch.Tensor, stream=None) -> None:
    """k_pool[slot // 16, h, slot % 16] = k_new[t, h] (and V) for every slot >= 0."""
    NB, Hkv, BS, D = k_pool.shape
    T = slot_mapping.shape[0]
    _check(_kv_cache_write(_ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(slot_mapping), T, NB, Hkv, D,
                           BS, _dtype_code(k_pool), _stream(stream)), "pkv_kv_cache_write")


def copy_blocks(k_pools: list, v_pools: list, block_mapping: torch.Tensor, stream=None) -> None:
    """Copy-on-write: for every layer, block dst := block src for each (src, dst) row of block_mapping."""
    L = len(k_pools)
    NB, Hkv, BS, D = k_pools[0].shape
    kp = (_P * L)(*[_ptr(p) for p in k_pools])
    vp = (_P * L)(*[_ptr(p) for p in v_pools])
    P = block_mapping.shape[0]
    _check(_copy_blocks(kp, vp, L, _ptr(block_mapping), P, NB, Hkv, D, BS, _dtype_code(k_pools[0]), _stream(stream)),
           "pkv_copy_blocks")


# ---- paged attention ---------------------------------------------------------------------------

def plan_host(query_start_loc: np.ndarray, context_lens: np.ndarray, num_q_heads: int, num_kv_heads: int,
              head_dim: int, dtype: str, with_meta: bool = True, **opts) -> tuple[Plan, np.ndarray | None]:
    """Host-only planning (no CUDA): the plan and the metadata image the upload would copy."""
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    plan = Plan()
    if opts.get("shared_tables") is not None:
        opts = dict(opts, shared_tables=np.ascontiguousarray(opts["shared_tables"], dtype=np.int32))
    o = _opts(**opts)
    _check(_plan_host(_np_ptr(qsl), _np_ptr(ctx), ctx.shape[0], num_q_heads, num_kv_heads, head_dim,
                      DTYPE_NAME[dtype], ctypes.byref(o), None, 0, ctypes.byref(plan)), "pkv_attention_plan_host")
    meta = None
    if with_meta:
        meta = np.zeros(plan.meta_bytes, dtype=np.uint8)
        _check(_plan_host(_np_ptr(qsl), _np_ptr(ctx), ctx.shape[0], num_q_heads, num_kv_heads, head_dim,
                          DTYPE_NAME[dtype], ctypes.byref(o), _np_ptr(meta), meta.nbytes, ctypes.byref(plan)),
               "pkv_attention_plan_host")
    return plan, meta


class AttentionPlan:
    """A planned batch: host plan, device workspace and device copies of the batch description.

    The workspace is reused across plans and grows only when a batch needs more than it holds.
    replan() uploads the new work lists and batch description on `stream`, ordered after the
    kernels of the previous batch when those ran on the same stream.
    """

    def __init__(self, batch: dict, prior_lens, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 dtype: torch.dtype, device, workspace: torch.Tensor | None = None, stream=None, **opts):
        self.num_q_heads, self.num_kv_heads, self.head_dim, self.dtype = num_q_heads, num_kv_heads, head_dim, dtype
        self._code = _dtype_code(torch.empty(0, dtype=dtype))
        self.device = torch.device(device)
        shared = opts.pop("shared_tables", None)
        self._shared = None if shared is None else np.ascontiguousarray(shared, dtype=np.int32)
        self.opts = _opts(shared_tables=self._shared, **opts)
        if self.opts.num_sms == 0:
            self.opts.num_sms = torch.cuda.get_device_properties(self.device).multi_processor_count
        self.workspace = workspace
        self.plan = Plan()
        self._meta = None       # pinned image of the work lists
        self._staged = None     # pinned query_start_loc + context_lens
        self._dev = None        # their device copy
        self._views = (-1, None, None)  # (R, query_start_loc, context_lens) views of _dev
        self._uploaded = None   # event after the last upload from the pinned buffers
        self.replan(batch, prior_lens, stream=stream)

    def replan(self, batch: dict, prior_lens, stream=None, shared_tables=None) -> "AttentionPlan":
        """Plans the batch on the host straight into pinned memory and enqueues the uploads of the
        work lists and of the batch description on `stream` (pkv_attention_plan_async: one library
        call, no host wait). shared_tables: the batch's host block tables, when they changed (for
        shared-prefix detection)."""
        if shared_tables is not None:
            self._shared = np.ascontiguousarray(shared_tables, dtype=np.int32)
            self.opts.h_block_tables = self._shared.ctypes.data
            self.opts.block_table_stride = int(self._shared.shape[1])
        qsl, ctx = flatten_batch(batch, prior_lens)
        self.h_query_start_loc, self.h_context_lens = qsl, ctx
        self.num_q_tokens = int(qsl[-1])
        R = ctx.shape[0]
        n = 2 * R + 1
        if self._uploaded is not None:
            self._uploaded.synchronize()          # the pinned buffers are free again
        if self._staged is None or self._staged.numel() < n:
            cap = max(n, 64)
            self._staged = torch.empty(cap, dtype=torch.int32).pin_memory()
            self._dev = torch.empty(cap, dtype=torch.int32, device=self.device)
            self._views = (-1, None, None)
        if isinstance(stream, torch.cuda.Stream):
            s = stream
        elif stream is None:
            s = torch.cuda.current_stream(self.device)
        else:
            s = torch.cuda.ExternalStream(_stream(stream))
        qp, cp = qsl.ctypes.data, ctx.ctypes.data
        for _ in range(3):
            meta_cap = self._meta.numel() if self._meta is not None else 0
            ws_cap = self.workspace.numel() if self.workspace is not None else 0
            status = _plan_async(qp, cp, R, self.num_q_heads, self.num_kv_heads, self.head_dim, self._code,
                                 ctypes.byref(self.opts), self._meta.data_ptr() if meta_cap else None, meta_cap,
                                 self.workspace.data_ptr() if ws_cap else None, ws_cap, self._staged.data_ptr(),
                                 self._dev.data_ptr(), ctypes.byref(self.plan), s.cuda_stream)
            if status != 4:
                break
            if meta_cap < self.plan.meta_bytes:
                self._meta = torch.empty(max(int(self.plan.meta_bytes) * 5 // 4, 4096), dtype=torch.uint8).pin_memory()
            if ws_cap < self.plan.ws_bytes:
                self.workspace = torch.empty(max(int(self.plan.ws_bytes), 256), dtype=torch.uint8, device=self.device)
        _check(status, "pkv_attention_plan_async")
        if self._uploaded is None:
            self._uploaded = torch.cuda.Event()
        self._uploaded.record(s)
        if self._views[0] != R:
            self._views = (R, self._dev[:R + 1], self._dev[R + 1:n])
        self.query_start_loc, self.context_lens = self._views[1], self._views[2]
        return self


def paged_attention(plan: AttentionPlan, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                    block_tables: torch.Tensor, scale: float, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Attention of every row of the planned batch; q/out [T, Hq, D], pools [NB, Hkv, 16, D]."""
    if out is None:
        out = torch.empty_like(q)
    NB = k_pool.shape[0]
    _check(_attention(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
                      _ptr(plan.context_lens), _ptr(plan.query_start_loc), NB, float(scale), ctypes.byref(plan.plan),
                      _ptr(plan.workspace), plan.workspace.numel(), _stream(stream)), "pkv_paged_attention")
    return out


def attend(batch: dict, prior_lens, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
           block_tables: torch.Tensor, scale: float, out: torch.Tensor | None = None, stream=None,
           **opts) -> torch.Tensor:
    """One call for a {request_id: num_tokens} batch (dict order): builds query_start_loc and
    context_lens from it and each request's prior context, plans on the host and runs
    pkv_paged_attention. Callers that run many steps keep an AttentionPlan and replan it instead."""
    plan = AttentionPlan(batch, prior_lens, q.shape[1], k_pool.shape[1], q.shape[2], q.dtype, q.device,
                         stream=stream, **opts)
    return paged_attention(plan, q, k_pool, v_pool, block_tables, scale, out=out, stream=stream)


# ---- host validators and the device error word -----------------------------------------------

def validate_tables(block_tables: np.ndarray, context_lens: np.ndarray, num_blocks: int) -> None:
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    _check(_validate_tables(_np_ptr(bt), _np_ptr(ctx), ctx.shape[0], bt.shape[1] if bt.ndim == 2 else 0,
                            int(num_blocks)), "pkv_validate_tables")


def validate_slots(slots: np.ndarray, num_blocks: int) -> None:
    s = np.ascontiguousarray(slots, dtype=np.int64)
    _check(_validate_slots(_np_ptr(s), s.shape[0], int(num_blocks)), "pkv_validate_slots")


def validate_copy_pairs(pairs: np.ndarray, num_blocks: int) -> None:
    p = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    _check(_validate_pairs(_np_ptr(p), p.shape[0], int(num_blocks)), "pkv_validate_copy_pairs")


def device_error(stream=None) -> tuple[int, int]:
    """(code, detail) of the first device-side error since the last read; (0, -1) when none."""
    code = _I(0)
    detail = _I64(0)
    _check(_device_error(ctypes.byref(code), ctypes.byref(detail), _stream(stream)), "pkv_device_error")
    return code.value, detail.value


def profile_start(capacity: int = 4096) -> None:
    """Time every library kernel launched from this thread with CUDA events on its stream."""
    _check(_profile_start(int(capacity)), "pkv_profile_start")


def profile_stop() -> dict:
    """{kind: (total_ms, launches)} since profile_start; also 'dropped' (launches not timed)."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    dropped = ctypes.c_int(0)
    _check(_profile_stop(ms, cnt, ctypes.byref(dropped)), "pkv_profile_stop")
    out = {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}
    out["dropped"] = dropped.value
    return out


# ---- host block manager ------------------------------------------------------------------------

class BmStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "num_blocks", "free_blocks", "used_blocks", "shared_blocks", "num_sequences", "logical_tokens",
        "stored_tokens", "wasted_slots", "cow_copies", "cached_blocks", "cache_queries", "cache_hits")]


_BM = ctypes.c_void_p
_I32P = ctypes.POINTER(ctypes.c_int32)
_bm_create = _sig("pkv_bm_create_ex", _I, [_I, _I, _I, ctypes.POINTER(_BM)])
_bm_add_cached = _sig("pkv_bm_add_cached_prefix", _I, [_BM, _I64, _P, _I64, ctypes.POINTER(_I64)])
_bm_append_tokens = _sig("pkv_bm_append_tokens", _I, [_BM, _I64, _P, _I64, _I32P])
_bm_destroy = _sig("pkv_bm_destroy", None, [_BM])
_bm_add = _sig("pkv_bm_add_sequence", _I, [_BM, _I64, _I64])
_bm_fork = _sig("pkv_bm_fork", _I, [_BM, _I64, _I64])
_bm_append = _sig("pkv_bm_append", _I, [_BM, _I64, _I64, _I32P])
_bm_free = _sig("pkv_bm_free", _I, [_BM, _I64])
_bm_sequence = _sig("pkv_bm_sequence", _I, [_BM, _I64, ctypes.POINTER(_I64), _P, _I, ctypes.POINTER(_I)])
_bm_tables = _sig("pkv_bm_block_tables", _I, [_BM, _P, _I, _P, _I])
_bm_refcount = _sig("pkv_bm_refcount", _I, [_BM, ctypes.c_int32, _I32P])
_bm_stats = _sig("pkv_bm_stats", _I, [_BM, ctypes.POINTER(BmStats)])
_bm_step = _sig("pkv_bm_step", _I, [_BM, _P, _P, _I, _P, _P, _I, _P, _P, _P, ctypes.POINTER(_I)])
PKV_BM_PREFIX_CACHE = 1


class BlockManager:
    """Allocation state of one block pool (pkv_bm_* in include/pkv.h): on-demand blocks,
    reference-counted sharing between forked sequences, copy-on-write of shared last blocks and,
    with prefix_cache=True, reuse of cached full blocks for prompts that begin alike."""

    def __init__(self, num_blocks: int, block_size: int = 16, prefix_cache: bool = False):
        h = _BM()
        _check(_bm_create(int(num_blocks), int(block_size), PKV_BM_PREFIX_CACHE if prefix_cache else 0,
                          ctypes.byref(h)), "pkv_bm_create_ex")
        self._h = h
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def __del__(self, _destroy=_bm_destroy):
        if getattr(self, "_h", None):
            _destroy(self._h)
            self._h = None

    def add(self, seq_id: int, num_tokens: int) -> None:
        _check(_bm_add(self._h, int(seq_id), int(num_tokens)), "pkv_bm_add_sequence")

    def fork(self, parent: int, child: int) -> None:
        _check(_bm_fork(self._h, int(parent), int(child)), "pkv_bm_fork")

    def add_cached_prefix(self, seq_id: int, tokens) -> int:
        """Starts a token-tracked sequence from the longest cached prefix of `tokens`; returns how
        many leading tokens are cached (the rest are appended, with their ids, by the caller)."""
        ids = np.ascontiguousarray(tokens, dtype=np.int32)
        cached = _I64(0)
        _check(_bm_add_cached(self._h, int(seq_id), _np_ptr(ids), ids.shape[0], ctypes.byref(cached)),
               "pkv_bm_add_cached_prefix")
        return cached.value

    def append(self, seq_id: int, num_tokens: int, tokens=None) -> tuple[int, int] | None:
        """Returns the (src, dst) copy the append needs, or None. `tokens`: the new tokens' ids."""
        pair = (ctypes.c_int32 * 2)()
        if tokens is None:
            _check(_bm_append(self._h, int(seq_id), int(num_tokens), pair), "pkv_bm_append")
        else:
            ids = np.ascontiguousarray(tokens, dtype=np.int32)
            if ids.shape[0] != int(num_tokens):
                raise ValueError("len(tokens) != num_tokens")
            _check(_bm_append_tokens(self._h, int(seq_id), _np_ptr(ids), int(num_tokens), pair), "pkv_bm_append_tokens")
        return None if pair[0] < 0 else (pair[0], pair[1])

    def free(self, seq_id: int) -> None:
        _check(_bm_free(self._h, int(seq_id)), "pkv_bm_free")

    def sequence(self, seq_id: int) -> tuple[int, list]:
        """(tokens, block ids) of one sequence."""
        tokens = _I64(0)
        nb = _I(0)
        _check(_bm_sequence(self._h, int(seq_id), ctypes.byref(tokens), None, 0, ctypes.byref(nb)), "pkv_bm_sequence")
        blocks = np.empty(max(nb.value, 1), np.int32)
        _check(_bm_sequence(self._h, int(seq_id), ctypes.byref(tokens), _np_ptr(blocks), blocks.shape[0],
                            ctypes.byref(nb)), "pkv_bm_sequence")
        return tokens.value, blocks[:nb.value].tolist()

    def block_tables(self, seq_ids, max_blocks_per_seq: int) -> np.ndarray:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        out = np.empty((ids.shape[0], int(max_blocks_per_seq)), np.int32)
        _check(_bm_tables(self._h, _np_ptr(ids), ids.shape[0], _np_ptr(out), int(max_blocks_per_seq)),
               "pkv_bm_block_tables")
        return out

    def refcount(self, block: int) -> int:
        c = ctypes.c_int32(0)
        _check(_bm_refcount(self._h, int(block), ctypes.byref(c)), "pkv_bm_refcount")
        return c.value

    def stats(self) -> dict:
        st = BmStats()
        _check(_bm_stats(self._h, ctypes.byref(st)), "pkv_bm_stats")
        return {n: getattr(st, n) for n, _ in BmStats._fields_}

    def step(self, batch: dict, max_blocks_per_seq: int, new_tokens=None):
        """Appends batch {seq_id: num_new_tokens} (dict order) and returns the step's host inputs:
        (block_tables int32 [R, max_blocks_per_seq], context_lens int32 [R], query_start_loc int32 [R+1],
        copy pairs int32 [P, 2]). new_tokens: the new tokens' ids concatenated in batch order."""
        ids = np.fromiter(batch.keys(), np.int64, len(batch))
        n = np.fromiter(batch.values(), np.int32, len(batch))
        tok = None
        if new_tokens is not None:
            tok = np.ascontiguousarray(new_tokens, dtype=np.int32)
            if tok.shape[0] != int(n.sum()):
                raise ValueError("new_tokens must hold sum(batch.values()) ids")
        R = ids.shape[0]
        tables = np.empty((R, int(max_blocks_per_seq)), np.int32)
        ctx = np.empty(R, np.int32)
        qsl = np.empty(R + 1, np.int32)
        pairs = np.empty((max(R, 1), 2), np.int32)
        npairs = _I(0)
        _check(_bm_step(self._h, _np_ptr(ids), _np_ptr(n), R, None if tok is None else _np_ptr(tok), _np_ptr(tables),
                        int(max_blocks_per_seq), _np_ptr(ctx), _np_ptr(qsl), _np_ptr(pairs), ctypes.byref(npairs)),
               "pkv_bm_step")
        return tables, ctx, qsl, pairs[:npairs.value].copy()
