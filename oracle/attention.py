"""fp64 oracle: exact attention written out from its definition (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` use this module. Page keys ([card], [interview], [essay],
[explainer]) are defined in ``oracle/__init__.py``.

Every function takes float64 arrays and materialises what the definition names.
Matrix products go through numpy (a library primitive); no blocking, fusion or
reordering is applied beyond what a definition states, except that rows of S are
independent by definition, so the long-sequence mode computes them a group of
rows at a time.

Readings of points the pages leave open:
  * scale: S = scale·QKᵀ with the scale passed in (1/√d in every workload);
    [essay] section 二 writes softmax(QKᵀ/√d), [interview] 二.1 omits the scale.
  * the statistic saved for the backward is lse = m + ln ℓ (natural log, in the
    units of the scaled scores); [essay] 二 and [interview] 三.3 save (m, ℓ),
    which carries the same information.
  * softmax gradient: dS = P∘(dP − rowsum(P∘dP)) with dP = dO·Vᵀ (textbook
    softmax Jacobian); the formula printed in [explainer] "梯度计算优化" is not
    dimensionally consistent and is not used.
  * causal: query i sees keys j ≤ i ([essay] 三.1) when N_q = N_k. With
    N_q ≠ N_k (pages silent) the mask is bottom-right aligned: query i sees keys
    j ≤ i + (N_k − N_q), i.e. the queries are the last N_q positions of the key
    sequence; with N_q = N_k it is the rule above.
  * block mask: one uint8 entry per 128×128 tile of S, shared by every batch
    and head, composed with the causal mask by AND ([card] Block-Sparse).
  * a row with no allowed key: O = 0, lse = −inf, zero gradient (pages silent).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

TILE = 128  # one block-mask entry covers a TILE x TILE tile of S


# --------------------------------------------------------------------------- masks

def allowed_mask(nq: int, nk: int, causal: bool = False, block_mask=None, tile: int = TILE) -> np.ndarray:
    """Boolean [nq, nk]: True where query i may attend to key j.

    Causal ([essay] 三.1): P_ij = 0 for j > i + (nk − nq) (bottom-right aligned;
    j > i when nq = nk). Block mask ([card] Block-Sparse): entry (I, J) = 0
    removes every pair (i, j) with i // tile == I and j // tile == J. The two
    compose by AND.
    """
    a = np.ones((nq, nk), dtype=bool)
    if causal:
        a &= np.arange(nk)[None, :] <= np.arange(nq)[:, None] + (nk - nq)
    if block_mask is not None:
        bm = np.asarray(block_mask).astype(bool)
        a &= bm[np.arange(nq)[:, None] // tile, np.arange(nk)[None, :] // tile]
    return a


# --------------------------------------------------------------------------- forward

def _softmax_rows(S: np.ndarray):
    """Safe softmax of each row ([explainer] 工作原理; [interview] 三.2).

    Subtract the row maximum, exponentiate, divide by the row sum. Returns P and
    lse = max + ln(sum). A row of only −inf gives P = 0 and lse = −inf.
    """
    m = S.max(axis=-1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - m_safe)
    l = E.sum(axis=-1, keepdims=True)
    P = np.divide(E, l, out=np.zeros_like(E), where=l > 0)
    l1 = l[..., 0]
    lse = np.full(l1.shape, -np.inf)
    pos = l1 > 0
    lse[pos] = m_safe[..., 0][pos] + np.log(l1[pos])
    return P, lse


def _head_forward(q, k, v, scale, allowed):
    S = scale * (q @ k.T)                       # S = scale·QKᵀ   ([interview] 二.1, [essay] 二)
    S = np.where(allowed, S, -np.inf)           # masked scores
    P, lse = _softmax_rows(S)                   # P = softmax(S)
    O = P @ v                                   # O = PV
    return O, lse, P


def forward(q, k, v, scale: float, causal: bool = False, block_mask=None, tile: int = TILE,
            return_p: bool = False):
    """Exact attention forward for q, k, v of shape [..., N, d] (float64).

    Returns (O [..., N, d], lse [..., N]) and, if ``return_p``, P [..., N, N].
    Leading dimensions (batch, heads) are independent problems.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    allowed = allowed_mask(n, k.shape[-2], causal, block_mask, tile)
    O = np.empty(lead + (n, v.shape[-1]))
    lse = np.empty(lead + (n,))
    Ps = np.empty(lead + (n, k.shape[-2])) if return_p else None
    for idx in np.ndindex(*lead):
        o, s, P = _head_forward(q[idx], k[idx], v[idx], scale, allowed)
        O[idx], lse[idx] = o, s
        if return_p:
            Ps[idx] = P
    return (O, lse, Ps) if return_p else (O, lse)


def forward_rows(q, k, v, scale: float, rows, causal: bool = False, block_mask=None, tile: int = TILE):
    """O and lse of the query rows ``rows`` only, for inputs [..., N, d].

    The definition restricted to those rows: S[rows, :] = scale·Q[rows] Kᵀ,
    masked, softmax per row, times V. Rows are independent, so nothing else is
    needed; used where the full N×N problem is too large for the CPU.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    rows = np.asarray(rows)
    lead = q.shape[:-2]
    n = k.shape[-2]
    allowed = _allowed_pairs(rows, np.arange(n), causal, block_mask, tile, n - q.shape[-2])
    O = np.empty(lead + (rows.size, v.shape[-1]))
    lse = np.empty(lead + (rows.size,))
    for idx in np.ndindex(*lead):
        S = scale * (q[idx][rows] @ k[idx].T)
        S = np.where(allowed, S, -np.inf)
        P, lse[idx] = _softmax_rows(S)
        O[idx] = P @ v[idx]
    return O, lse


# --------------------------------------------------------------------------- backward

def _head_backward(q, k, v, do, scale, allowed):
    _, _, P = _head_forward(q, k, v, scale, allowed)   # P recomputed from the definition
    dV = P.T @ do                                      # dV = Pᵀ dO
    dP = do @ v.T                                      # dP = dO Vᵀ
    D = (P * dP).sum(axis=1, keepdims=True)            # D_i = Σ_j P_ij dP_ij
    dS = P * (dP - D)                                  # softmax Jacobian
    dQ = scale * (dS @ k)                              # S = scale·QKᵀ
    dK = scale * (dS.T @ q)
    return dQ, dK, dV, D[:, 0]


def backward(q, k, v, do, scale: float, causal: bool = False, block_mask=None, tile: int = TILE,
             return_d: bool = False):
    """Gradients of a loss L with ∂L/∂O = dO, by the chain rule through the definition.

    dV = Pᵀ dO, dP = dO Vᵀ, dS = P∘(dP − rowsum(P∘dP)), dQ = scale·dS K,
    dK = scale·dSᵀ Q. P is recomputed here from Q and K ([card] 反向：重算而非存储).
    Returns (dQ, dK, dV) and, if ``return_d``, D = rowsum(P∘dP) [..., N].
    """
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    lead = q.shape[:-2]
    n = q.shape[-2]
    allowed = allowed_mask(n, k.shape[-2], causal, block_mask, tile)
    dQ, dK, dV = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    D = np.empty(lead + (n,))
    for idx in np.ndindex(*lead):
        dQ[idx], dK[idx], dV[idx], D[idx] = _head_backward(q[idx], k[idx], v[idx], do[idx], scale, allowed)
    return (dQ, dK, dV, D) if return_d else (dQ, dK, dV)


def backward_rows(q, k, v, do, scale: float, rows, causal: bool = False, block_mask=None, tile: int = TILE):
    """Forward and gradients of L = Σ_{i ∈ rows} <dO_i, O_i> for one head [N, d].

    The same definitions as :func:`forward` and :func:`backward`, applied to the
    query rows ``rows`` only: S_rows = scale·Q_rows Kᵀ (masked), P_rows =
    softmax(S_rows), O_rows = P_rows V, dV = P_rowsᵀ dO_rows, dP = dO_rows Vᵀ,
    dS = P∘(dP − rowsum(P∘dP)), dQ_rows = scale·dS K, dK = scale·dSᵀ Q_rows.
    With ``rows`` = all rows this is the full backward. Returns
    (O_rows, lse_rows, dQ_rows, dK, dV).
    """
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    rows = np.asarray(rows)
    allowed = _allowed_pairs(rows, np.arange(k.shape[0]), causal, block_mask, tile, k.shape[0] - q.shape[0])
    S = scale * (q[rows] @ k.T)
    S = np.where(allowed, S, -np.inf)
    P, lse = _softmax_rows(S)
    O = P @ v
    dV = P.T @ do[rows]
    dP = do[rows] @ v.T
    D = (P * dP).sum(axis=1, keepdims=True)
    dS = P * (dP - D)
    return O, lse, scale * (dS @ k), scale * (dS.T @ q[rows]), dV


# --------------------------------------------------------------------------- online recurrence

def online_forward(q, k, v, scale: float, bounds, causal: bool = False, block_mask=None,
                   tile: int = TILE):
    """Forward by the online-softmax recurrence of [interview] 三.2, for one head [N, d].

    Keys are split into consecutive blocks at ``bounds`` (0 = b_0 < … < b_T = N).
    Each block gives local statistics m̃ = rowmax(S_blk), ℓ̃ = rowsum(exp(S_blk − m̃))
    and an unnormalised local output Õ = exp(S_blk − m̃)·V_blk. They are merged
    into the running (m, ℓ, O):
        m' = max(m, m̃),  ℓ' = e^{m−m'}·ℓ + e^{m̃−m'}·ℓ̃,  O' = e^{m−m'}·O + e^{m̃−m'}·Õ,
    and O/ℓ is returned at the end with lse = m + ln ℓ. A factor e^{x−m'} whose
    exponent is −inf − (−inf) (no allowed key seen yet on either side) is taken as 0.
    This routine exists to check the two-pass oracle; it is not used for parity.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    n = q.shape[0]
    allowed = allowed_mask(n, k.shape[0], causal, block_mask, tile)
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    O = np.zeros((n, v.shape[1]))

    def factor(a, b):
        out = np.zeros_like(a)
        ok = np.isfinite(a)
        out[ok] = np.exp(a[ok] - b[ok])
        return out

    bounds = list(bounds)
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        S = scale * (q @ k[lo:hi].T)
        S = np.where(allowed[:, lo:hi], S, -np.inf)
        m_t = S.max(axis=1)
        m_t_safe = np.where(np.isfinite(m_t), m_t, 0.0)
        E = np.exp(S - m_t_safe[:, None])
        l_t = E.sum(axis=1)
        O_t = E @ v[lo:hi]
        m_new = np.maximum(m, m_t)
        a_old = factor(m, m_new)
        a_new = factor(m_t, m_new)
        l = a_old * l + a_new * l_t
        O = a_old[:, None] * O + a_new[:, None] * O_t
        m = m_new
    lse = np.full(n, -np.inf)
    pos = l > 0
    O = np.divide(O, l[:, None], out=np.zeros_like(O), where=pos[:, None])
    lse[pos] = m[pos] + np.log(l[pos])
    return O, lse


# --------------------------------------------------------------------------- split-KV merge

def merge_partials(Os, lses):
    """Merge partial results of disjoint key splits of the same query rows.

    Each split s contributes O_s (its softmax-weighted average of its values) and
    lse_s (the log of its exp-sum). The whole is
        lse = log Σ_s exp(lse_s),   O = Σ_s exp(lse_s − lse)·O_s,
    the online-softmax update of [interview] 三.2 applied to whole splits at once.
    A split with no allowed key has lse_s = −inf and weight 0; a row whose splits
    all have none gets O = 0, lse = −inf.
    """
    lses = np.stack([np.asarray(x, dtype=np.float64) for x in lses])   # [S, ..., N]
    Os = np.stack([np.asarray(x, dtype=np.float64) for x in Os])       # [S, ..., N, dv]
    m = lses.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lses - m_safe)                                          # exp(−inf) = 0
    z = w.sum(axis=0)
    lse = np.full(z.shape, -np.inf)
    pos = z > 0
    lse[pos] = m_safe[pos] + np.log(z[pos])
    O = np.divide((w[..., None] * Os).sum(axis=0), z[..., None],
                  out=np.zeros(Os.shape[1:]), where=pos[..., None])
    return O, lse


def split_kv_forward(q, k, v, scale: float, bounds, causal: bool = False, block_mask=None,
                     tile: int = TILE):
    """Forward for one head (q [N_q, d], k, v [N_k, d]) with the keys cut into
    consecutive splits at ``bounds`` (0 = b_0 < … < b_S = N_k): each split is
    computed on its own by the definition restricted to its keys, then the
    partials are merged (:func:`merge_partials`) — the split-KV form used for
    decoding, where one query row meets a long key sequence. Masks are those of
    :func:`allowed_mask` on the whole problem. Returns (O, lse, Os, lses).
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    allowed = allowed_mask(q.shape[0], k.shape[0], causal, block_mask, tile)
    Os, lses = [], []
    bounds = list(bounds)
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        S = scale * (q @ k[lo:hi].T)
        S = np.where(allowed[:, lo:hi], S, -np.inf)
        P, lse_s = _softmax_rows(S)
        Os.append(P @ v[lo:hi])
        lses.append(lse_s)
    O, lse = merge_partials(Os, lses)
    return O, lse, Os, lses


# --------------------------------------------------------------------------- tile enumeration

def causal_tile_set(n: int, br: int, bc: int, nk: int | None = None):
    """The valid-tile set of [essay] 三.1: {(i, j) | j·B_c ≤ i·B_r + B_r − 1}.

    i ranges over the ⌈n/B_r⌉ query tiles and j over the ⌈n/B_c⌉ key tiles.
    With ``nk`` keys (N_q = n ≠ N_k) the diagonal is shifted by N_k − N_q and
    the last row of tile i is the last real query row: j·B_c ≤
    min(i·B_r + B_r − 1, n − 1) + N_k − N_q. Returned as a sorted list of (i, j) pairs.
    """
    nk = n if nk is None else nk
    tr, tc = -(-n // br), -(-nk // bc)
    return [(i, j) for i in range(tr) for j in range(tc)
            if j * bc <= min(i * br + br - 1, n - 1) + (nk - n)]


def _visited(n, causal, block_mask, br, bc, mask_tile=TILE, nk=None):
    """Set of (i, j) tile pairs the method processes: the causal valid-tile set
    (or all pairs) intersected with the non-zero entries of the block mask.
    A query tile of B_r rows inside mask row I = i·B_r // mask_tile (B_r divides mask_tile)."""
    nk = n if nk is None else nk
    tr, tc = -(-n // br), -(-nk // bc)
    pairs = set(causal_tile_set(n, br, bc, nk)) if causal else {(i, j) for i in range(tr) for j in range(tc)}
    if block_mask is not None:
        bm = np.asarray(block_mask)
        pairs = {(i, j) for (i, j) in pairs
                 if bm[(i * br) // mask_tile, (j * bc) // mask_tile]}
    return pairs


def forward_tile_lists(n: int, causal: bool, block_mask=None, br: int = 128, bc: int = 128, nk: int | None = None):
    """For each query tile i, the sorted key tiles j it streams ([essay] 三.1; [card] Block-Sparse:
    zero tiles skipped). ``n`` queries, ``nk`` keys (default ``n``)."""
    tr = -(-n // br)
    pairs = _visited(n, causal, block_mask, br, bc, nk=nk)
    return [sorted(j for (ii, j) in pairs if ii == i) for i in range(tr)]


def backward_tile_lists(n: int, causal: bool, block_mask=None, br: int = 128, bc: int = 128, nk: int | None = None):
    """For each key tile j, the sorted query tiles i that reach it (the transpose of the forward lists)."""
    tc = -(-(n if nk is None else nk) // bc)
    pairs = _visited(n, causal, block_mask, br, bc, nk=nk)
    return [sorted(i for (i, jj) in pairs if jj == j) for j in range(tc)]


# --------------------------------------------------------------------------- long sequences

def _head_sampled(q, k, v, do, scale, causal, block_mask, tile, rows_q, rows_k, chunk):
    n = q.shape[0]
    O = np.empty_like(q)
    lse = np.empty(n)
    # Pass 1: O and lse of every row, a group of rows at a time (rows are independent).
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        kend = r1 if causal else n          # keys beyond r1 are masked for every row of the group
        allowed = _allowed_pairs(np.arange(r0, r1), np.arange(kend), causal, block_mask, tile)
        S = scale * (q[r0:r1] @ k[:kend].T)
        S = np.where(allowed, S, -np.inf)
        P, lse[r0:r1] = _softmax_rows(S)
        O[r0:r1] = P @ v[:kend]
    D = (do * O).sum(axis=1)                # D_i = rowsum(dO∘O)
    out = {"o": O[rows_q], "lse": lse[rows_q]}
    # dQ at the sampled query rows: dQ_i = scale·Σ_j dS_ij k_j.
    Sq = scale * (q[rows_q] @ k.T)
    aq = _allowed_pairs(rows_q, np.arange(n), causal, block_mask, tile)
    Pq = np.where(aq, np.exp(np.where(aq, Sq, 0.0) - lse[rows_q][:, None]), 0.0)
    dPq = do[rows_q] @ v.T
    dSq = Pq * (dPq - D[rows_q][:, None])
    out["dq"] = scale * (dSq @ k)
    # dK, dV at the sampled key rows: dK_j = scale·Σ_i dS_ij q_i, dV_j = Σ_i P_ij dO_i.
    Sk = scale * (q @ k[rows_k].T)
    ak = _allowed_pairs(np.arange(n), rows_k, causal, block_mask, tile)
    Pk = np.where(ak, np.exp(np.where(ak, Sk, 0.0) - lse[:, None]), 0.0)
    dPk = do @ v[rows_k].T
    dSk = Pk * (dPk - D[:, None])
    out["dk"] = scale * (dSk.T @ q)
    out["dv"] = Pk.T @ do
    return out


def _allowed_pairs(rows, cols, causal, block_mask, tile, offset=0):
    """allowed_mask restricted to query rows ``rows`` and key columns ``cols``;
    ``offset`` = N_k − N_q (the causal diagonal's shift)."""
    a = np.ones((rows.size, cols.size), dtype=bool)
    if causal:
        a &= cols[None, :] <= rows[:, None] + offset
    if block_mask is not None:
        bm = np.asarray(block_mask).astype(bool)
        a &= bm[rows[:, None] // tile, cols[None, :] // tile]
    return a


def sampled_forward_backward(q, k, v, do, scale: float, causal: bool, rows_q, rows_k,
                             block_mask=None, tile: int = TILE, chunk: int = 1024,
                             workers: int | None = None):
    """Long-sequence mode for inputs [..., N, d]: full-N×N matrices never exist.

    Pass 1 computes O and lse for every row of every head, a group of ``chunk``
    rows at a time, and D = rowsum(dO∘O). Then the same formulas as
    :func:`backward`, restricted to the rows ``rows_q`` (O, lse, dQ) and the key
    rows ``rows_k`` (dK, dV). Heads run in a thread pool (numpy releases the GIL
    in its kernels); the arithmetic of each head is unchanged by that.
    Returns a dict of arrays with leading dims [..., len(rows)].
    """
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    if q.shape[-2] != k.shape[-2]:
        raise ValueError("the long-sequence mode covers N_q = N_k only")
    rows_q, rows_k = np.asarray(rows_q), np.asarray(rows_k)
    lead = q.shape[:-2]
    heads = list(np.ndindex(*lead))
    if workers is None:
        workers = max(1, min(len(heads), os.cpu_count() or 1))

    def run(idx):
        return idx, _head_sampled(q[idx], k[idx], v[idx], do[idx], scale, causal, block_mask, tile,
                                  rows_q, rows_k, chunk)

    results = {}
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(1) if workers > 1 else None
    except ImportError:  # pragma: no cover
        limiter = None
    try:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            for idx, res in ex.map(run, heads):
                results[idx] = res
    finally:
        if limiter is not None:
            limiter.restore_original_limits()
    out = {}
    for key in ("o", "lse", "dq", "dk", "dv"):
        first = results[heads[0]][key]
        arr = np.empty(lead + first.shape)
        for idx in heads:
            arr[idx] = results[idx][key]
        out[key] = arr
    return out
