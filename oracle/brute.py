"""Brute-force contiguous attention in float64 -- TEST INFRASTRUCTURE (pins the C oracle).

This is the storage scheme the pages contrast paging with: each request's K and V as one contiguous
[ctx, Hkv, D] array (blog.mckayzhao.com/?p=56, "故事要从 KV Cache 说起"; 一文搞懂vLLM, "朴素 serving 方式为啥
这么浪费"). The pages state that the paged kernel's result equals this contiguous computation
(blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感"). No block table appears here:
the attention is written in matrix form with NumPy, independently of pkv_oracle.c's loops.
"""
import numpy as np


def contiguous_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, prior: int, scale: float) -> np.ndarray:
    """Attention of n query rows over one request's contiguous cache.

    q: [n, Hq, D] float64 rows at positions prior .. prior+n-1; K, V: [ctx, Hkv, D] float64 with
    ctx >= prior + n. Query head h uses KV head h // (Hq // Hkv). Row i attends keys 0..prior+i.
    Returns [n, Hq, D] float64.
    """
    n, Hq, D = q.shape
    ctx, Hkv, _ = K.shape
    group = Hq // Hkv
    Kh = np.repeat(K, group, axis=1)                  # [ctx, Hq, D]
    Vh = np.repeat(V, group, axis=1)
    S = np.einsum("nhd,thd->hnt", q, Kh) * scale      # [Hq, n, ctx]
    visible = np.arange(ctx)[None, :] <= (prior + np.arange(n))[:, None]
    S = np.where(visible[None, :, :], S, -np.inf)
    S = S - S.max(axis=-1, keepdims=True)
    W = np.exp(S)
    W = W / W.sum(axis=-1, keepdims=True)
    return np.einsum("hnt,thd->nhd", W, Vh)


def naive_reserved_waste(used: int, reserved: int) -> int:
    """Slots a contiguous max-length reservation leaves unused (一文搞懂vLLM, "朴素 serving 方式为啥这么浪费")."""
    return reserved - used
