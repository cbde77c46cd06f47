"""Token-level brute force in numpy (float64), for tiny inputs only.

Written independently of the oracle's C loops: pooling by reshaping, the metric
from a dense masked score matrix and scipy's softmax, selection by a full
lexicographic sort, attention from a dense token-level mask. It is a pin for the
oracle, not a second oracle: tests compare the two on small random cases.
"""

from __future__ import annotations

import numpy as np
import scipy.special
import torch


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def pool(q, k, v, block):
    """Block means by slicing; a partial last block (S % block != 0) is the mean of its rows."""
    Q, K, V = f64(q), f64(k), f64(v)
    B, Hq, S, D = Q.shape
    Hkv = K.shape[1]
    nb = -(-S // block)
    blocks = [slice(i * block, min(S, (i + 1) * block)) for i in range(nb)]
    qbar = np.stack([Q[:, :, sl].mean(axis=2) for sl in blocks], axis=2)
    kbar = np.stack([K[:, :, sl].mean(axis=2) for sl in blocks], axis=2)
    norms = np.linalg.norm(V, axis=-1)
    vnorm = np.stack([norms[:, :, sl].mean(axis=2) for sl in blocks], axis=2)
    return qbar, kbar, vnorm


def metric_dense(qbar, kbar, vnorm):
    """m [B, Hq, nb, nb]; entries above the diagonal are 0."""
    B, Hq, nb, D = qbar.shape
    G = Hq // kbar.shape[1]
    kb = np.repeat(kbar, G, axis=1)
    vn = np.repeat(vnorm, G, axis=1)
    s = np.einsum("bhid,bhjd->bhij", qbar, kb) / np.sqrt(D)
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    s = np.where(causal, s, -np.inf)
    p = scipy.special.softmax(s, axis=-1)
    return p * vn[:, :, None, :]


def select_rows(m_dense, k):
    """Per (b, h, i): sorted list of kept blocks."""
    B, Hq, nb, _ = m_dense.shape
    out = {}
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                if i == 0:
                    out[(b, h, i)] = [0]
                    continue
                js = np.arange(1, i)
                vals = m_dense[b, h, i, 1:i]
                order = np.lexsort((js, -vals))  # primary: -m, secondary: j
                best = js[order][: k[i] - 2].tolist()
                out[(b, h, i)] = sorted(set([0, i] + best))
    return out


def attention_masked(q, k, v, block, kept):
    """Dense token-level attention under the block mask implied by `kept`
    ({(b,h,i): [blocks]}); returns out [B, Hq, S, D] float64."""
    Q, K, V = f64(q), f64(k), f64(v)
    B, Hq, S, D = Q.shape
    G = Hq // K.shape[1]
    nb = -(-S // block)
    tok_block = np.arange(S) // block
    out = np.zeros_like(Q)
    for b in range(B):
        for h in range(Hq):
            allowed = np.zeros((S, S), dtype=bool)
            for i in range(nb):
                blocks = np.zeros(nb, dtype=bool)
                blocks[kept[(b, h, i)]] = True
                allowed[i * block:(i + 1) * block, :] = blocks[tok_block][None, :]
            allowed &= np.tril(np.ones((S, S), dtype=bool))
            logits = Q[b, h] @ K[b, h // G].T / np.sqrt(D)
            logits = np.where(allowed, logits, -np.inf)
            w = scipy.special.softmax(logits, axis=-1)
            out[b, h] = w @ V[b, h // G]
    return out


def antidiag(q, k, block, stride):
    """Anti-diagonal block probabilities from the full token logit matrix: the samples are
    picked out of Q K^T / sqrt(D) (numpy matmul) by index, averaged per sub-tile, softmaxed
    per query group (scipy) and summed per block. Returns [B, Hq, nb, nb] (0 above i)."""
    B, Hq, S, D = q.shape
    G = Hq // k.shape[1]
    nb = -(-S // block)
    R = block // stride
    nred = S // stride
    t = np.arange(stride)
    out = np.zeros((B, Hq, nb, nb))
    for b in range(B):
        for h in range(Hq):
            Q = q[b, h].double().numpy()
            K = k[b, h // G].double().numpy()
            X = Q @ K.T / np.sqrt(D)
            u = np.arange(nred)
            rows = u[:, None, None] * stride + t[None, None, :]                  # [u, 1, t]
            cols = u[None, :, None] * stride + (stride - 1 - t)[None, None, :]   # [1, w, t]
            A = X[rows, cols].mean(axis=2)                                       # [u, w]
            A = np.where(np.tril(np.ones((nred, nred), bool)), A, -np.inf)
            P = scipy.special.softmax(A, axis=1)
            for i in range(nb):
                us = range(i * R, min((i + 1) * R, nred))
                for j in range(i + 1):
                    out[b, h, i, j] = np.mean([P[uu, j * R:(j + 1) * R].sum() for uu in us])
    return out
