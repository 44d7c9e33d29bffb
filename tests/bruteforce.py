"""Dense numpy fp64 brute force for tiny grids, written independently of the
C oracle: it builds the full N x N token mask by broadcasting coordinates,
finds radii by counting mask rows, and evaluates entropy and attention with
dense softmax.  Used only to pin the oracle.

Definitions restated from "Token Radius Attention for Efficient Video
Generation" (gist.science summary), section 2: Intuition I (entropy ->
budget), Intuition II (query-centred radius with temporal decay), "Le
Pipeline TRA" (radius mask, tile-major blocks, token voting).
"""
from __future__ import annotations

import math

import numpy as np


def coords(T, H, W):
    n = np.arange(T * H * W)
    return n // (H * W), (n // W) % H, n % W


def decay(gamma, rte):
    return np.array([math.pow(gamma, k) for k in range(rte + 1)], dtype=np.float64)


def halfwidth(r, g):
    # r * g then + 1e-9, each a separately rounded fp64 op (numpy never fuses)
    prod = np.asarray(r, dtype=np.float64) * np.asarray(g, dtype=np.float64)
    return np.floor(prod + 1e-9).astype(np.int64)


def token_mask(T, H, W, gamma, Rt, r, disk=False):
    """Dense boolean M[i, j] for radii r[i] (natural order).  disk=True takes
    the Euclidean test dh^2 + dw^2 <= s^2 instead of the Chebyshev one."""
    t, h, w = coords(T, H, W)
    rte = min(Rt, T - 1)
    g = decay(gamma, rte)
    dt = np.abs(t[:, None] - t[None, :])
    dh = np.abs(h[:, None] - h[None, :])
    dw = np.abs(w[:, None] - w[None, :])
    inside = dt <= rte
    s = halfwidth(np.asarray(r)[:, None], g[np.minimum(dt, rte)])
    if disk:
        return inside & (dh * dh + dw * dw <= s * s)
    return inside & (np.maximum(dh, dw) <= s)


def bhat(Hent, a, b, N, Bmin):
    out = []
    for h in np.asarray(Hent, dtype=np.float32).reshape(-1):
        x = (a * float(h)) + b
        e = math.exp(x) if x < 700 else math.inf
        out.append(math.ceil(min(float(N), max(float(Bmin), e))))
    return np.array(out, dtype=np.int64)


def r_cap(T, H, W, gamma, Rt, disk=False):
    """Smallest r at which no query's mask row can grow any more: the
    farthest-frame test reaches the whole frame from every position."""
    rte = min(Rt, T - 1)
    g = decay(gamma, rte)[rte]
    r = 0
    if disk:
        while int(halfwidth(r, g)) ** 2 < (H - 1) ** 2 + (W - 1) ** 2:
            r += 1
        return r
    need = max(H, W) - 1
    while int(halfwidth(r, g)) < need:
        r += 1
    return r


def radius(Hent, T, H, W, a, b, gamma, Rt, Bmin, disk=False):
    """Smallest r whose dense token-mask row holds >= Bhat keys, else r_cap.
    Returns (r, counts) for one head (Hent of length N)."""
    N = T * H * W
    bh = bhat(Hent, a, b, N, Bmin)
    rc = r_cap(T, H, W, gamma, Rt, disk)
    r = np.full(N, -1, dtype=np.int64)
    cnt = np.zeros(N, dtype=np.int64)
    for rr in range(rc + 1):
        c = token_mask(T, H, W, gamma, Rt, np.full(N, rr), disk).sum(axis=1)
        newly = (r < 0) & (c >= bh)
        r[newly] = rr
        cnt[newly] = c[newly]
        if rr == rc:
            cnt[r < 0] = c[r < 0]
            r[r < 0] = rc
    return r, cnt


def entropy_dense(q, k):
    """-sum p ln p of softmax(q k^T / sqrt d) per row, one head."""
    d = q.shape[-1]
    s = (q.astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        lp = np.where(p > 0, np.log(p), 0.0)
    return -(p * lp).sum(axis=1)


def attention_masked(q, k, v, M):
    d = q.shape[-1]
    s = (q.astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(d)
    s = np.where(M, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v.astype(np.float64)


def tile_ids(T, H, W, th, tw):
    t, h, w = coords(T, H, W)
    nTh, nTw = -(-H // th), -(-W // tw)
    return (t * nTh + h // th) * nTw + w // tw, T * nTh * nTw


def block_mask(M, T, H, W, qtile, ktile):
    """0 inactive / 1 active / 3 full for every (query tile, key tile)."""
    qid, nQ = tile_ids(T, H, W, *qtile)
    kid, nK = tile_ids(T, H, W, *ktile)
    out = np.zeros((nQ, nK), dtype=np.uint8)
    for a in range(nQ):
        rows = np.nonzero(qid == a)[0]
        sub = M[rows]
        for b in range(nK):
            cols = np.nonzero(kid == b)[0]
            blk = sub[:, cols]
            if blk.any():
                out[a, b] = 3 if blk.all() else 1
    return out


def topk_count(q, k, mass):
    """Fewest top keys whose dense softmax probabilities reach `mass`, per row
    (numpy sort, one head)."""
    d = q.shape[-1]
    s = (q.astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    c = np.cumsum(-np.sort(-p, axis=1), axis=1)
    return (c < mass).sum(axis=1) + 1
