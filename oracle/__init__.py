"""CPU oracle for paged attention over a block-pooled KV cache -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference arm may import this
package. The product library (paged_kv_cache_446_b200) never imports it and shares no code with it.

Two independent implementations live here:
  * pkv_oracle.c (loaded below through ctypes): gathers K/V through the block tables and runs naive
    max-subtracted softmax attention in double precision; also the slot mapping, the KV append, the
    copy-on-write block copy and the block accounting of the pages.
  * brute.py: NumPy float64 attention over contiguous per-request K/V with no tables at all, used to
    pin the C oracle on tiny inputs.

Arrays are NumPy; 16-bit storage types are passed as uint16 bit patterns.
"""
import ctypes

import numpy as np

from . import build as _build

F32, F16, BF16 = 0, 1, 2
DTYPE_CODES = {"f32": F32, "f16": F16, "bf16": BF16}

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_D = ctypes.c_double

_libs: dict = {}


def load(mutant: str | None = None) -> ctypes.CDLL:
    """Load (building on first use) the oracle library, or a planted-mistake variant of it."""
    key = mutant or ""
    if key not in _libs:
        path = _build.build(mutant)
        lib = ctypes.CDLL(path)
        lib.oracle_paged_attention.restype = _I
        lib.oracle_paged_attention.argtypes = [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _D, _I, _P, _I, _I]
        lib.oracle_slot_mapping.restype = _I
        lib.oracle_slot_mapping.argtypes = [_P, _I, _P, _P, _I, _I, _P]
        lib.oracle_kv_cache_write.restype = _I
        lib.oracle_kv_cache_write.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I]
        lib.oracle_copy_blocks.restype = _I
        lib.oracle_copy_blocks.argtypes = [_P, _P, _I, _P, _I, _I, _I, _I, _I, _I]
        lib.oracle_blocks_for_tokens.restype = _I64
        lib.oracle_blocks_for_tokens.argtypes = [_I64, _I]
        lib.oracle_wasted_slots.restype = _I64
        lib.oracle_wasted_slots.argtypes = [_I64, _I]
        lib.oracle_half_to_double.restype = _D
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = _D
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_max_threads.restype = _I
        _libs[key] = lib
    return _libs[key]


def _ptr(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(_P)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


class OracleError(RuntimeError):
    pass


def _check(code: int, what: str):
    if code != 0:
        raise OracleError(f"{what} returned {code}")


def paged_attention(q, k_pool, v_pool, block_tables, context_lens, query_start_loc, scale, dtype,
                    rows=None, nthreads=0, mutant=None) -> np.ndarray:
    """Attention output in float64, [rows or T, Hq, D].

    q: [T, Hq, D]; k_pool, v_pool: [NB, Hkv, 16, D] (float32, or uint16 bits of f16/bf16);
    block_tables: int32 [R, max_blocks]; context_lens: int32 [R]; query_start_loc: int32 [R+1].
    """
    lib = load(mutant)
    q = np.ascontiguousarray(q)
    k_pool = np.ascontiguousarray(k_pool)
    v_pool = np.ascontiguousarray(v_pool)
    bt = _i32(block_tables)
    ctx = _i32(context_lens)
    qsl = _i32(query_start_loc)
    T, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_pool.shape
    assert D2 == D and v_pool.shape == k_pool.shape
    R = ctx.shape[0]
    max_blocks = bt.shape[1] if bt.ndim == 2 and bt.shape[0] > 0 else max(1, bt.size)
    code = DTYPE_CODES[dtype] if isinstance(dtype, str) else int(dtype)
    if rows is None:
        out = np.zeros((T, Hq, D), dtype=np.float64)
        rl, nr = None, 0
    else:
        rl = _i32(rows)
        nr = rl.shape[0]
        out = np.zeros((nr, Hq, D), dtype=np.float64)
    if bt.size == 0:
        bt = np.zeros((1, 1), dtype=np.int32)
    _check(lib.oracle_paged_attention(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(bt), max_blocks,
                                      _ptr(ctx), _ptr(qsl), R, Hq, Hkv, D, BS, NB, float(scale), code,
                                      _ptr(rl) if rl is not None else None, nr, int(nthreads)),
           "oracle_paged_attention")
    return out


def slot_mapping(block_tables, query_start_loc, context_lens, block_size=16, mutant=None) -> np.ndarray:
    """int64 slot of every new token of the batch (physical block * block_size + offset)."""
    lib = load(mutant)
    bt = _i32(block_tables)
    qsl = _i32(query_start_loc)
    ctx = _i32(context_lens)
    T = int(qsl[-1]) if qsl.size else 0
    out = np.full(T, -1, dtype=np.int64)
    max_blocks = bt.shape[1] if bt.ndim == 2 else bt.size
    _check(lib.oracle_slot_mapping(_ptr(bt), max_blocks, _ptr(qsl), _ptr(ctx), ctx.shape[0], block_size, _ptr(out)),
           "oracle_slot_mapping")
    return out


def kv_cache_write(k_new, v_new, k_pool, v_pool, slots, mutant=None) -> None:
    """In place: pool[slot // bs, h, slot % bs, :] = new[t, h, :] for every slot >= 0, in token order."""
    lib = load(mutant)
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    k_new = np.ascontiguousarray(k_new)
    v_new = np.ascontiguousarray(v_new)
    s = np.ascontiguousarray(np.asarray(slots, dtype=np.int64))
    NB, Hkv, BS, D = k_pool.shape
    _check(lib.oracle_kv_cache_write(_ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(s), s.shape[0],
                                     NB, Hkv, D, BS, k_pool.itemsize), "oracle_kv_cache_write")


def copy_blocks(k_pools, v_pools, pairs, mutant=None) -> None:
    """In place, for every layer and every (src, dst) pair in order: block dst := block src (K and V)."""
    lib = load(mutant)
    pr = _i32(pairs).reshape(-1, 2)
    L = len(k_pools)
    kp = (_P * L)(*[p.ctypes.data for p in k_pools])
    vp = (_P * L)(*[p.ctypes.data for p in v_pools])
    NB, Hkv, BS, D = k_pools[0].shape
    _check(lib.oracle_copy_blocks(kp, vp, L, _ptr(np.ascontiguousarray(pr)), pr.shape[0], NB, Hkv, D, BS,
                                  k_pools[0].itemsize), "oracle_copy_blocks")


def blocks_for_tokens(n: int, block_size: int = 16, mutant=None) -> int:
    return int(load(mutant).oracle_blocks_for_tokens(int(n), int(block_size)))


def wasted_slots(n: int, block_size: int = 16, mutant=None) -> int:
    return int(load(mutant).oracle_wasted_slots(int(n), int(block_size)))


def half_to_double(bits: int, mutant=None) -> float:
    return float(load(mutant).oracle_half_to_double(int(bits)))


def bf16_to_double(bits: int, mutant=None) -> float:
    return float(load(mutant).oracle_bf16_to_double(int(bits)))


def max_threads() -> int:
    return int(load().oracle_max_threads())


__all__ = ["paged_attention", "slot_mapping", "kv_cache_write", "copy_blocks", "blocks_for_tokens",
           "wasted_slots", "half_to_double", "bf16_to_double", "max_threads", "load", "F32", "F16", "BF16",
           "OracleError", "flatten_batch"]


def flatten_batch(batch: dict, prior_lens, mutant=None) -> tuple[np.ndarray, np.ndarray]:
    """{request_id: num_tokens} (insertion order) -> (query_start_loc [R+1], context_lens [R]).

    blog.mckayzhao.com/?p=56, "V1 架构：推倒重来的勇气": one step is a dict giving each request's token
    count; rows of request r are consecutive, in dict order; its context after the step is its prior
    context plus its tokens. prior_lens[r] belongs to the r-th entry of the dict.

    mutant (tests only) plants one mistake: "FLAT_CTX_PRIOR" leaves the step's tokens out of the
    context, "FLAT_SORTED_IDS" lays rows out in request-id order instead of dict order,
    "FLAT_QSL_SHIFT" drops the leading zero of the prefix sum.
    """
    items = list(batch.items())
    if mutant == "FLAT_SORTED_IDS":
        items.sort(key=lambda kv: kv[0])
    counts = [int(v) for _, v in items]
    qsl = [0]
    for c in counts:
        qsl.append(qsl[-1] + c)
    if mutant == "FLAT_QSL_SHIFT":
        qsl = qsl[1:] + [qsl[-1]]
    prior = [int(p) for p in prior_lens]
    ctx = [p if mutant == "FLAT_CTX_PRIOR" else p + c for p, c in zip(prior, counts)]
    return np.asarray(qsl, dtype=np.int32), np.asarray(ctx, dtype=np.int32)
