"""Independent brute-force attention for tiny shapes (a pin for the oracle).

Written separately from the oracle: numpy fancy indexing for the page
gather, np.repeat for the grouped heads, einsum for the products, and the
softmax taken as exp(s) / sum exp(s) with no maximum subtracted, which is
exact enough for the small, bounded scores of tiny N(0,1) inputs.
Widening to float64 goes through torch's own casts.
"""
import numpy as np
import torch


def brute_attention(q, k_cache, v_cache, block_table, cache_seqlens, *, Hkv, page_size,
                    scale, causal):
    qd = q.double().numpy()
    kd = k_cache.double().numpy()
    vd = v_cache.double().numpy()
    B, q_len, Hq, D = qd.shape
    G = Hq // Hkv
    L = np.asarray(cache_seqlens, dtype=np.int64)
    Lmax = int(L.max()) if B else 0
    out = np.zeros((B, q_len, Hq, D))
    lse = np.full((B, Hq, q_len), -np.inf)
    if Lmax == 0:
        return out, lse
    j = np.arange(Lmax)
    if block_table is None:
        pages = np.repeat(np.arange(B)[:, None], Lmax, axis=1)
    else:
        bt = np.asarray(block_table, dtype=np.int64)
        pages = bt[:, np.minimum(j // page_size, bt.shape[1] - 1)]
    slots = np.broadcast_to(j % page_size, (B, Lmax))
    K = kd[pages, slots]            # [B, Lmax, Hkv, D]
    V = vd[pages, slots]
    K = np.repeat(K, G, axis=2)     # [B, Lmax, Hq, D]
    V = np.repeat(V, G, axis=2)
    s = np.einsum("bthd,bjhd->bhtj", qd, K) * scale
    t = np.arange(q_len)
    limit = L[:, None] - q_len + t[None, :] + 1 if causal else np.broadcast_to(L[:, None], (B, q_len))
    limit = np.minimum(limit, L[:, None])
    visible = j[None, None, :] < limit[:, :, None]          # [B, q_len, Lmax]
    w = np.exp(s) * visible[:, None, :, :]                  # [B, Hq, q_len, Lmax]
    den = w.sum(-1)                                         # [B, Hq, q_len]
    num = np.einsum("bhtj,bjhd->bthd", w, V)
    nz = den > 0
    o = np.where(np.transpose(nz, (0, 2, 1))[..., None], num / np.where(den > 0, den, 1).transpose(0, 2, 1)[..., None], 0.0)
    out[:] = o
    lse[nz] = np.log(den[nz])
    return out, lse
