"""Independent numpy brute force for packed attention (test-only).

Written apart from the C oracle and the CUDA path: the packed batch is
scattered into a padded [B, Lmax, H, D] tensor, the scores of every
(query, key) pair are formed densely, keys beyond each request's length get
a -inf mask, and the softmax is taken with numpy along the key axis.
"""

import numpy as np


def attention_padded(Qp, Kp, Vp, lens, scale):
    """Dense attention over padded [B, Lmax, H, D] tensors whose rows at and
    beyond lens[b] hold anything (they are masked). Returns padded
    (O [B, Lmax, H, D], LSE [B, H, Lmax])."""
    lens = np.asarray(lens)
    B, Lmax = Qp.shape[:2]
    S = np.einsum("bqhd,bkhd->bhqk", Qp, Kp) * scale
    keymask = np.arange(Lmax)[None, :] < lens[:, None]          # [B, Lmax]
    S = np.where(keymask[:, None, None, :], S, -np.inf)
    mx = S.max(axis=-1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    E = np.exp(S - mx)
    Z = E.sum(axis=-1, keepdims=True)
    P = E / np.where(Z > 0, Z, 1.0)
    Vz = np.where(keymask[:, :, None, None], Vp, 0.0)            # masked rows never reach O
    Op = np.einsum("bhqk,bkhd->bqhd", P, Vz)
    Lp = (mx + np.log(np.where(Z > 0, Z, 1.0)))[..., 0]
    return Op, Lp


def padded_masked_attention(q, k, v, cu_seqlens, scale, pad_value=0.0):
    """q, k, v float64 [T, H, D] packed. Returns (o [T, H, D], lse [T, H])."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = len(cu) - 1
    T, H, D = q.shape
    lens = np.diff(cu)
    Lmax = int(lens.max()) if B else 0
    o = np.zeros((T, H, D))
    lse = np.zeros((T, H))
    if Lmax == 0:
        return o, lse
    Qp, Kp, Vp = (np.full((B, Lmax, H, D), pad_value) for _ in range(3))
    for b in range(B):
        n = lens[b]
        Qp[b, :n], Kp[b, :n], Vp[b, :n] = q[cu[b]:cu[b + 1]], k[cu[b]:cu[b + 1]], v[cu[b]:cu[b + 1]]
    Op, Lp = attention_padded(Qp, Kp, Vp, lens, scale)
    for b in range(B):
        n = lens[b]
        o[cu[b]:cu[b + 1]] = Op[b, :n]
        lse[cu[b]:cu[b + 1]] = Lp[b, :, :n].T
    return o, lse
