"""fp64 CPU oracle of the Wan DiT full spatio-temporal self-attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this module.  It shares no code
with the CUDA path (``video_dit_full_b200``) and imports nothing from it.

What it computes, and where the pages fix it:

* Bidirectional (non-causal), full (not windowed) multi-head self-attention
  over all latent tokens of all frames:
  Wan 2.1 paper-podcast summary, section "先看现象" (cost model
  C = L(a*b*s*h^2 + b*b*s^2*h), "non-causal attention, beta = 4 forward,
  8 backward") and section "干预与形式化" (the DiT uses full spatio-temporal
  self-attention, not windowed);  kwkr.cn Wan explainer, section 2.2.
* The same definition with queries and keys of different lengths is the DiT
  block's cross-attention from the video tokens to the 512-token umT5 text
  embedding (Wan 2.1 paper-podcast summary, section "干预与形式化": c_txt is
  umT5's 512-token text embedding; the DiT backbone injects umT5 by
  cross-attention).  Q and dO hold Sq rows, K and V hold Sk rows; self-
  attention is Sk = Sq.
* The softmax scale 1/sqrt(D), D = 128, the [B, S, H, D] layout and the
  natural-log LSE [B, H, S] are readings (the pages give no formula); the
  design notes list them.

For each batch b, head h and query row i (inputs widened exactly from bf16):
    s_ij  = (q_i . k_j) / sqrt(D)             for every key j in [0, Sk)
    lse_i = m_i + ln sum_j exp(s_ij - m_i),    m_i = max_j s_ij
    o_i   = sum_j exp(s_ij - lse_i) v_j

Backward of f = sum(O * dO) (textbook differentiation of the definition):
    P_ij  = exp(s_ij - lse_i),  Dl_i = sum_d dO_id o_id
    dP_ij = dO_i . v_j,          dS_ij = P_ij (dP_ij - Dl_i)
    dQ_i  = sum_j dS_ij k_j / sqrt(D),  dK_j = sum_i dS_ij q_i / sqrt(D),
    dV_j  = sum_i P_ij dO_i

Rows are independent in the definition, so rows are processed in groups of
``ROW_CHUNK`` (each row still sees all S keys in one piece); a matmul from
numpy's BLAS serves as the dot-product step.  Nothing is reordered across keys.
"""
from __future__ import annotations

import numpy as np

ROW_CHUNK = 512


def widen(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values; fp arrays -> fp64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def _head(x: np.ndarray, b: int, h: int, rows=None) -> np.ndarray:
    sl = x[b, :, h, :] if rows is None else x[b, rows, h, :]
    return np.ascontiguousarray(widen(sl))


def _rows_fwd(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Definition above for the rows of Q against all keys of K, V (fp64)."""
    s = (Q @ K.T) * scale
    m = s.max(axis=1)
    lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    p = np.exp(s - lse[:, None])
    return p @ V, lse


def attn_fwd(q, k, v, rows=None, heads=None):
    """Forward attention.

    q: [B, Sq, H, D], k and v: [B, Sk, H, D] arrays (bf16 bit patterns or floats).
    rows: query token indices to evaluate (default: all Sq).
    heads: head indices to evaluate (default: all H).
    Returns (o [B, R, Hs, D] fp64, lse [B, Hs, R] fp64).
    """
    B, S, H, D = q.shape
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(H)) if heads is None else list(heads)
    scale = 1.0 / np.sqrt(D)
    o = np.empty((B, len(rows), len(heads), D))
    lse = np.empty((B, len(heads), len(rows)))
    for b in range(B):
        for hi, h in enumerate(heads):
            K = _head(k, b, h)
            V = _head(v, b, h)
            for r0 in range(0, len(rows), ROW_CHUNK):
                r = rows[r0:r0 + ROW_CHUNK]
                ob, lb = _rows_fwd(_head(q, b, h, r), K, V, scale)
                o[b, r0:r0 + len(r), hi, :] = ob
                lse[b, hi, r0:r0 + len(r)] = lb
    return o, lse


def attn_bwd(q, k, v, do, q_rows=None, k_rows=None, heads=None):
    """Backward attention of f = sum(O * dO).

    q, do: [B, Sq, H, D]; k, v: [B, Sk, H, D].
    q_rows: query rows whose dQ is wanted (default all Sq; empty = none).
    k_rows: key rows whose dK, dV are wanted (default all Sk; empty = none).
    heads:  heads to evaluate (default all).
    Returns dict with dq [B, Rq, Hs, D], dk and dv [B, Rk, Hs, D], and the
    forward's lse [B, Hs, Sq] and Dl = rowsum(dO * O) [B, Hs, Sq] when key rows
    were asked for (they need every query row), else for the query rows only.
    """
    B, S, H, D = q.shape
    Sk = k.shape[1]
    q_rows = np.arange(S) if q_rows is None else np.asarray(q_rows, dtype=np.int64)
    k_rows = np.arange(Sk) if k_rows is None else np.asarray(k_rows, dtype=np.int64)
    heads = list(range(H)) if heads is None else list(heads)
    scale = 1.0 / np.sqrt(D)
    Hs = len(heads)
    dq = np.zeros((B, len(q_rows), Hs, D))
    dk = np.zeros((B, len(k_rows), Hs, D))
    dv = np.zeros((B, len(k_rows), Hs, D))
    need_all = len(k_rows) > 0
    lse_out = np.empty((B, Hs, S if need_all else len(q_rows)))
    dl_out = np.empty_like(lse_out)
    for b in range(B):
        for hi, h in enumerate(heads):
            K = _head(k, b, h)
            V = _head(v, b, h)
            if need_all:
                # lse_i and Dl_i of every row i (every query sees key j)
                Q = _head(q, b, h)
                dO = _head(do, b, h)
                lse = np.empty(S)
                dl = np.empty(S)
                for r0 in range(0, S, ROW_CHUNK):
                    r1 = min(S, r0 + ROW_CHUNK)
                    ob, lb = _rows_fwd(Q[r0:r1], K, V, scale)
                    lse[r0:r1] = lb
                    dl[r0:r1] = (dO[r0:r1] * ob).sum(axis=1)
                lse_out[b, hi] = lse
                dl_out[b, hi] = dl
                # key rows: the columns j of P, dP, dS
                Kc, Vc = K[k_rows], V[k_rows]
                for r0 in range(0, S, ROW_CHUNK):
                    r1 = min(S, r0 + ROW_CHUNK)
                    s_c = (Q[r0:r1] @ Kc.T) * scale
                    p_c = np.exp(s_c - lse[r0:r1, None])
                    dp_c = dO[r0:r1] @ Vc.T
                    ds_c = p_c * (dp_c - dl[r0:r1, None])
                    dv[b, :, hi, :] += p_c.T @ dO[r0:r1]
                    dk[b, :, hi, :] += (ds_c.T @ Q[r0:r1]) * scale
                lse_q, dl_q = lse[q_rows], dl[q_rows]
            if len(q_rows):
                Qr = _head(q, b, h, q_rows)
                dOr = _head(do, b, h, q_rows)
                if not need_all:
                    orow, lse_q = _rows_fwd(Qr, K, V, scale)
                    dl_q = (dOr * orow).sum(axis=1)
                    lse_out[b, hi] = lse_q
                    dl_out[b, hi] = dl_q
                s = (Qr @ K.T) * scale
                p = np.exp(s - lse_q[:, None])
                dp = dOr @ V.T
                ds = p * (dp - dl_q[:, None])
                dq[b, :, hi, :] = (ds @ K) * scale
    return {"dq": dq, "dk": dk, "dv": dv, "lse": lse_out, "dl": dl_out}


def softmax_matrix(q, k, b: int = 0, h: int = 0) -> np.ndarray:
    """The full S x S matrix P_ij = exp(s_ij - lse_i) of one (b, h): tiny cases only."""
    D = q.shape[3]
    Q, K = _head(q, b, h), _head(k, b, h)
    s = (Q @ K.T) / np.sqrt(D)
    m = s.max(axis=1)
    lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return np.exp(s - lse[:, None])
