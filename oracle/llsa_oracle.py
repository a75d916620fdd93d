"""Plain, slow CPU oracle of the LLSA hot path (test infrastructure only).

Source: "Trainable Log-linear Sparse Attention for Efficient Diffusion
Transformers", howistudyai explainer: Building Blocks (Hierarchical
Compression, Hierarchical Top-K Selection, Hierarchical KV Enrichment, KV
Reweighting, Sparse Index Transpose) and Steps 1-4.  Readings of points the
pages leave open are stated next to the code that takes them.

Conventions shared with the CUDA library's C header (conventions of the
interface, not shared code):
  * tensors are [B, H, tokens, D] with D innermost; tokens are in Z-order;
  * level 0 is the N fine tokens, level l has N / 16**l tokens, and the
    level-1 tokens are the 16-token query/key blocks;
  * an index list I(l) is int [B, H, N_l, K]: for each level-l query token the
    selected level-l key tokens in ascending order, -1 padding at the tail;
  * level_w is None (every key weighs 1) or a sequence indexed by level whose
    entries 2..L weight the coarse keys of that level.
"""

from __future__ import annotations

import math

import numpy as np

FACTOR = 16  # pooling factor per level and tokens per block


def default_scale(D: int) -> float:
    """Softmax scale 1/sqrt(D) for every key, fine or coarse (the pages do not
    state one; this is the usual attention scale)."""
    return 1.0 / math.sqrt(D)


# --------------------------------------------------------------------------
# Step 1: hierarchical compression
# --------------------------------------------------------------------------
def pool(X: np.ndarray, L: int, factor: int = FACTOR) -> dict[int, np.ndarray]:
    """Mean-pool X level by level (Step 1, Hierarchical Compression).

    Level l is made from level l-1 by averaging non-overlapping groups of
    ``factor`` consecutive tokens, so level l has N / factor**l tokens and each
    summarises factor**l fine tokens.  The pages build each level from the
    one below it, and so does this function.

    Precision: fp32, the precision of the pyramid that the selection scores
    read.  Each group is summed left to right, one rounding per addition, and
    the sum is multiplied by 1/factor (exact for a power of two).

    Returns {l: float32 [B, H, N_l, D]} for l = 1..L.
    """
    out = {}
    prev = np.asarray(X, dtype=np.float32)
    for l in range(1, L + 1):
        B, H, n, D = prev.shape
        assert n % factor == 0, "token count must be divisible by the factor"
        groups = prev.reshape(B, H, n // factor, factor, D)
        acc = groups[:, :, :, 0, :].copy()
        for j in range(1, factor):
            acc = acc + groups[:, :, :, j, :]  # float32 + float32 -> float32
        prev = acc * np.float32(1.0 / factor)
        out[l] = prev
    return out


# --------------------------------------------------------------------------
# Step 2: hierarchical Top-K selection
# --------------------------------------------------------------------------
def candidates_for_level(parent_idx: np.ndarray, factor: int = FACTOR) -> np.ndarray:
    """Candidate key tokens at level l for every level-(l+1) parent.

    A parent p that kept key tokens c (its row of I(l+1)) passes on the
    children factor*c .. factor*c + factor-1 of each kept c: the parent's
    choice expanded one level down (Step 2).  Padding (-1) in
    the parent row gives -1 candidates.  Returns int64 [B, H, N_{l+1}, K*factor].
    """
    p = np.asarray(parent_idx, dtype=np.int64)
    j = np.arange(factor, dtype=np.int64)
    cand = p[..., :, None] * factor + j  # [B,H,Np,K,factor]
    cand = np.where(p[..., :, None] >= 0, cand, -1)
    return cand.reshape(*p.shape[:-1], p.shape[-1] * factor)


def _scores_fp32(q: np.ndarray, kc: np.ndarray) -> np.ndarray:
    """Unscaled dot products q . k in fp32, summed over d = 0..D-1 in order.

    q: float32 [n, D]; kc: float32 [n, C, D] -> float32 [n, C].
    s_0 = fl(q_0 k_0), s_d = fl(s_{d-1} + fl(q_d k_d)): every product and every
    partial sum is rounded to fp32 (no fused multiply-add).
    """
    s = q[:, None, 0] * kc[:, :, 0]
    for d in range(1, q.shape[1]):
        s = s + q[:, None, d] * kc[:, :, d]
    return s


def select_level(
    Ql: np.ndarray,
    Kl: np.ndarray,
    parent_idx: np.ndarray | None,
    topk: int,
    factor: int = FACTOR,
) -> np.ndarray:
    """One level of hierarchical Top-K selection (Step 2).

    Ql, Kl: float32 [B, H, N_l, D], the level-l pooled queries and keys.
    parent_idx: I(l+1) as int [B, H, N_l/factor, K], or None at the coarsest
    level, where every query scores every key.

    For each level-l query token q the candidates are all level-l keys (top
    level) or the children of the keys its parent q // factor kept.  Each
    candidate c scores Q(l)[q] . K(l)[c] (unscaled: the softmax is monotone,
    so scaling cannot change the order).  The K_eff = min(K, #candidates)
    highest scores are kept; equal scores go to the lower key index.  The
    kept keys are stored in ascending order with -1 padding after them.

    Returns int32 [B, H, N_l, topk].
    """
    Ql = np.asarray(Ql, dtype=np.float32)
    Kl = np.asarray(Kl, dtype=np.float32)
    B, H, n, D = Ql.shape
    out = np.full((B, H, n, topk), -1, dtype=np.int32)
    if parent_idx is None:
        cand_q = np.broadcast_to(np.arange(n, dtype=np.int64), (B, H, n, n))
    else:
        cand_p = candidates_for_level(parent_idx, factor)  # [B,H,n/factor,C]
        cand_q = np.repeat(cand_p, factor, axis=2)  # query q takes parent q // factor
    C = cand_q.shape[-1]
    chunk = max(1, (1 << 22) // max(1, C * D))
    for b in range(B):
        for h in range(H):
            for q0 in range(0, n, chunk):
                q1 = min(n, q0 + chunk)
                cand = np.asarray(cand_q[b, h, q0:q1])  # [m, C]
                valid = cand >= 0
                kc = Kl[b, h][np.where(valid, cand, 0)]  # [m, C, D]
                s = _scores_fp32(Ql[b, h, q0:q1], kc)
                # order: score descending, then key index ascending; invalid last
                neg = np.where(valid, -s.astype(np.float64), np.inf)
                order = np.lexsort((cand, neg), axis=-1)
                ranked = np.take_along_axis(cand, order, axis=-1)
                k_eff = np.minimum(topk, valid.sum(axis=-1))  # [m]
                keep = np.full((q1 - q0, topk), -1, dtype=np.int64)
                w = min(topk, C)
                keep[:, :w] = ranked[:, :w]
                keep[np.arange(topk)[None, :] >= k_eff[:, None]] = -1
                # ascending block order, padding after the kept keys
                keep = np.where(keep < 0, np.iinfo(np.int64).max, keep)
                keep.sort(axis=-1)
                keep = np.where(keep == np.iinfo(np.int64).max, -1, keep)
                out[b, h, q0:q1] = keep
    return out


def level_topk(topk, l: int) -> int:
    """K_l, the number of keys kept at level l: topk itself when it is an
    int, else topk[l] (a dict or a sequence indexed by level).  The pages fix
    one K for every level; a K per level is the plainest reading of letting
    K vary (Open Questions: adaptive K), with the same descent."""
    return int(topk) if np.isscalar(topk) else int(topk[l])


def select_all(pyr_q: dict, pyr_k: dict, L: int, topk, factor: int = FACTOR) -> dict[int, np.ndarray]:
    """Hierarchical Top-K from the coarsest level L down to level 1 (Step 2).

    topk: one K for every level, or K_l per level (level_topk).  Level l then
    keeps K_l of the factor * K_{l+1} children of its parent's kept keys.

    Returns {l: I(l)} for l = 1..L, I(l) int32 [B, H, N_l, K_l].
    """
    idx = {}
    parent = None
    for l in range(L, 0, -1):
        idx[l] = select_level(pyr_q[l], pyr_k[l], parent, level_topk(topk, l), factor)
        parent = idx[l]
    return idx


# --------------------------------------------------------------------------
# Step 3: sparse attention with hierarchical KV enrichment and reweighting
# --------------------------------------------------------------------------
def enriched_top(L: int, enrich=None) -> int:
    """Highest level whose pooled tokens enrich the keys, for an enrichment
    depth Le (Limitations: "enrichment depth Le"; Surprising Findings: more
    enrichment levels, a little more quality for a little more time).
    Reading taken: depth Le uses levels 2..1+Le; None or 0 means every
    coarse level (2..L), a negative value none."""
    if enrich is None or enrich == 0:
        return L
    if enrich < 0:
        return 1
    return min(L, 1 + int(enrich))


def key_sets(idx: dict, L: int, n_blocks: int, enrich=None):
    """The key set of every 16-token query block b (Step 3).

    Fine part: the 16 fine tokens of every level-1 block in I(1)[b].
    Coarse part, for each level l = 2..Lc (Lc = enriched_top(L, enrich)): the
    level-l tokens in I(l)[a], where a = b // 16**(l-1) is the level-l
    ancestor of block b.  Level-1 pooled tokens are never keys (the fine
    tokens of the selected blocks stand for them).

    Returns (fine_tok int64 [B,H,n_blocks,16*K], coarse {l: int64
    [B,H,n_blocks,K]}) with -1 for padding.
    """
    I1 = np.asarray(idx[1], dtype=np.int64)
    j = np.arange(FACTOR, dtype=np.int64)
    fine = np.where(I1[..., None] >= 0, I1[..., None] * FACTOR + j, -1)
    fine = fine.reshape(*I1.shape[:-1], I1.shape[-1] * FACTOR)
    coarse = {}
    for l in range(2, enriched_top(L, enrich) + 1):
        anc = np.arange(n_blocks) // FACTOR ** (l - 1)
        coarse[l] = np.asarray(idx[l], dtype=np.int64)[:, :, anc, :]
    return fine, coarse


def _gather_keys(Kbh, Vbh, pk, pv, fine, coarse, L, level_w):
    """Keys, values, log-weights and validity of the key sets of some blocks."""
    ks = [Kbh[np.maximum(fine, 0)]]
    vs = [Vbh[np.maximum(fine, 0)]]
    lw = [np.zeros(fine.shape)]
    ok = [fine >= 0]
    for l in sorted(coarse):
        c = coarse[l]
        ks.append(pk[l][np.maximum(c, 0)])
        vs.append(pv[l][np.maximum(c, 0)])
        w = 1.0 if level_w is None else float(level_w[l])
        lw.append(np.full(c.shape, math.log(w)))
        ok.append(c >= 0)
    return (np.concatenate(ks, axis=1), np.concatenate(vs, axis=1),
            np.concatenate(lw, axis=1), np.concatenate(ok, axis=1))


def attn_fwd(Q, K, V, pyr_k, pyr_v, idx, L, scale, level_w=None, block_chunk=512, enrich=None):
    """Forward of LLSA attention (Step 3), as dense attention over each query
    block's explicit key list, in fp64.

    For query i in block b with key set S_b (fine keys weight 1, level-l
    coarse keys weight w_l):
        s_ij   = scale * q_i . k_j
        O_i    = sum_j w_j exp(s_ij) v_j / sum_j w_j exp(s_ij)
        LSE_i  = ln sum_j w_j exp(s_ij)
    A weight w multiplies the key's exponential, which is what counting the
    token w times does (KV Reweighting).  A query with an empty key set gets
    O_i = 0 and LSE_i = -inf.

    pyr_k, pyr_v: {l: [B,H,N_l,D]} for l = 2..L (any float type).
    enrich: enrichment depth (enriched_top).
    Returns O float64 [B,H,N,D], LSE float64 [B,H,N].
    """
    B, H, N, D = Q.shape
    nb = N // FACTOR
    fine, coarse = key_sets(idx, L, nb, enrich)
    O = np.zeros((B, H, N, D))
    LSE = np.full((B, H, N), -np.inf)
    for b in range(B):
        for h in range(H):
            Kbh = np.asarray(K[b, h], dtype=np.float64)
            Vbh = np.asarray(V[b, h], dtype=np.float64)
            pk = {l: np.asarray(pyr_k[l][b, h], dtype=np.float64) for l in range(2, L + 1)}
            pv = {l: np.asarray(pyr_v[l][b, h], dtype=np.float64) for l in range(2, L + 1)}
            for b0 in range(0, nb, block_chunk):
                b1 = min(nb, b0 + block_chunk)
                ks, vs, lw, ok = _gather_keys(
                    Kbh, Vbh, pk, pv, fine[b, h, b0:b1],
                    {l: coarse[l][b, h, b0:b1] for l in coarse}, L, level_w)
                q = np.asarray(Q[b, h, b0 * FACTOR:b1 * FACTOR], dtype=np.float64)
                q = q.reshape(b1 - b0, FACTOR, D)
                s = scale * np.matmul(q, ks.transpose(0, 2, 1)) + lw[:, None, :]
                s = np.where(ok[:, None, :], s, -np.inf)
                m = s.max(axis=-1, keepdims=True)
                has = np.isfinite(m)
                e = np.where(ok[:, None, :], np.exp(s - np.where(has, m, 0.0)), 0.0)
                den = e.sum(axis=-1, keepdims=True)
                o = np.matmul(e, vs) / np.where(has, den, 1.0)
                lse = np.where(has, m + np.log(np.where(has, den, 1.0)), -np.inf)
                O[b, h, b0 * FACTOR:b1 * FACTOR] = o.reshape(-1, D)
                LSE[b, h, b0 * FACTOR:b1 * FACTOR] = lse.reshape(-1)
    return O, LSE


# --------------------------------------------------------------------------
# Step 4: sparse index transpose
# --------------------------------------------------------------------------
def index_transpose(idx_l: np.ndarray, n_keys: int):
    """Query-major index lists -> key-major lists (Step 4, Sparse Index Transpose).

    For each (b, h): count how many query tokens kept each key token, take the
    exclusive prefix sum of the counts as row offsets, and list under each key
    the query tokens that kept it, in ascending order (CSR of the transposed
    selection).  Padding (-1) is skipped.

    Returns row_ptr int32 [B,H,n_keys+1] and col int32 [B,H,Nq*K]; col entries
    past row_ptr[n_keys] are -1.
    """
    I = np.asarray(idx_l, dtype=np.int64)
    B, H, nq, K = I.shape
    row_ptr = np.zeros((B, H, n_keys + 1), dtype=np.int32)
    col = np.full((B, H, nq * K), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            q_of = np.repeat(np.arange(nq), K)
            c_of = I[b, h].reshape(-1)
            keep = c_of >= 0
            q_of, c_of = q_of[keep], c_of[keep]
            counts = np.bincount(c_of, minlength=n_keys)
            row_ptr[b, h, 1:] = np.cumsum(counts)
            order = np.lexsort((q_of, c_of))  # by key, then by query
            col[b, h, : q_of.size] = q_of[order]
    return row_ptr, col


# --------------------------------------------------------------------------
# Backward of Step 3 (the pass that the transpose serves)
# --------------------------------------------------------------------------
def attn_bwd(Q, K, V, pyr_k, pyr_v, O, LSE, dO, idx, L, scale, level_w=None, block_chunk=512, enrich=None):
    """Gradients of the LLSA attention (fp64), with the indices held fixed.

    With P_ij = w_j exp(s_ij - LSE_i) on the key set of i's block:
        Delta_i = sum_d dO_id O_id
        dS_ij   = P_ij (dO_i . v_j - Delta_i)
        dQ_i    = scale * sum_j dS_ij k_j
        dk_j    = scale * sum_i dS_ij q_i,   dv_j = sum_i P_ij dO_i
    A fine key's gradient goes to its token.  A level-l coarse key is the mean
    of 16**l fine tokens, so its gradient reaches each of them divided by
    16**l.  Selection is discrete and passes no gradient, so the pooled Q(l)
    and the level-1 pooled K get none.

    Returns dQ, dK, dV float64 [B,H,N,D].
    """
    B, H, N, D = Q.shape
    nb = N // FACTOR
    fine, coarse = key_sets(idx, L, nb, enrich)
    dQ = np.zeros((B, H, N, D))
    dK = np.zeros((B, H, N, D))
    dV = np.zeros((B, H, N, D))
    for b in range(B):
        for h in range(H):
            Kbh = np.asarray(K[b, h], dtype=np.float64)
            Vbh = np.asarray(V[b, h], dtype=np.float64)
            pk = {l: np.asarray(pyr_k[l][b, h], dtype=np.float64) for l in range(2, L + 1)}
            pv = {l: np.asarray(pyr_v[l][b, h], dtype=np.float64) for l in range(2, L + 1)}
            dpk = {l: np.zeros_like(pk[l]) for l in range(2, L + 1)}
            dpv = {l: np.zeros_like(pv[l]) for l in range(2, L + 1)}
            for b0 in range(0, nb, block_chunk):
                b1 = min(nb, b0 + block_chunk)
                fi = fine[b, h, b0:b1]
                co = {l: coarse[l][b, h, b0:b1] for l in coarse}
                ks, vs, lw, ok = _gather_keys(Kbh, Vbh, pk, pv, fi, co, L, level_w)
                sl = slice(b0 * FACTOR, b1 * FACTOR)
                q = np.asarray(Q[b, h, sl], dtype=np.float64).reshape(b1 - b0, FACTOR, D)
                o = np.asarray(O[b, h, sl], dtype=np.float64).reshape(b1 - b0, FACTOR, D)
                do = np.asarray(dO[b, h, sl], dtype=np.float64).reshape(b1 - b0, FACTOR, D)
                lse = np.asarray(LSE[b, h, sl], dtype=np.float64).reshape(b1 - b0, FACTOR)
                s = scale * np.matmul(q, ks.transpose(0, 2, 1)) + lw[:, None, :]
                fin = np.isfinite(lse)[..., None] & ok[:, None, :]
                P = np.where(fin, np.exp(np.where(fin, s - lse[..., None], 0.0)), 0.0)
                delta = (do * o).sum(axis=-1)  # [nb, 16]
                dP = np.matmul(do, vs.transpose(0, 2, 1))
                dS = P * (dP - delta[..., None])
                dQ[b, h, sl] = (scale * np.matmul(dS, ks)).reshape(-1, D)
                dk = scale * np.matmul(dS.transpose(0, 2, 1), q)  # [nb, S, D]
                dv = np.matmul(P.transpose(0, 2, 1), do)
                nf = fi.shape[-1]
                m = fi >= 0
                np.add.at(dK[b, h], fi[m], dk[:, :nf][m])
                np.add.at(dV[b, h], fi[m], dv[:, :nf][m])
                off = nf
                for l in sorted(co):
                    c = co[l]
                    kk = c.shape[-1]
                    m = c >= 0
                    np.add.at(dpk[l], c[m], dk[:, off:off + kk][m])
                    np.add.at(dpv[l], c[m], dv[:, off:off + kk][m])
                    off += kk
            for l in range(2, L + 1):
                span = FACTOR ** l
                dK[b, h] += np.repeat(dpk[l], span, axis=0) / span
                dV[b, h] += np.repeat(dpv[l], span, axis=0) / span
    return dQ, dK, dV


# --------------------------------------------------------------------------
# The whole forward path, for tests and the CPU baseline
# --------------------------------------------------------------------------
def run_forward(Q, K, V, L, topk, scale=None, level_w=None):
    """pool -> hierarchical Top-K -> enriched sparse attention: the forward
    pipeline of the howistudyai explainer's overview, from Q, K, V to O.
    Returns a dict with the pyramid, indices, O and LSE."""
    D = Q.shape[-1]
    if scale is None:
        scale = default_scale(D)
    pq = pool(Q, L)
    pk = pool(K, L)
    pv = pool(V, L)
    idx = select_all(pq, pk, L, topk)
    O, LSE = attn_fwd(Q, K, V, pk, pv, idx, L, scale, level_w)
    return {"pq": pq, "pk": pk, "pv": pv, "idx": idx, "O": O, "LSE": LSE, "scale": scale}


# --------------------------------------------------------------------------
# Step 5: index reordering for images (raster <-> Z-order)
# --------------------------------------------------------------------------
def zorder_index(img_h: int, img_w: int) -> np.ndarray:
    """Z-order token of every raster position y * img_w + x (Step 5, Index
    Reordering for Images: group 2x2 pixels, then 4x4, ...).  The Z-order
    index interleaves the bits of x and y, x taking the even bits and y the
    odd bits, so 4 consecutive tokens are a 2x2 tile, 16 a 4x4 tile and so
    on.  Reading taken: square images whose side is a power of two (the
    pages' images are square); other shapes are rejected."""
    if img_h != img_w or img_h < 1 or (img_h & (img_h - 1)) != 0:
        raise ValueError("square power-of-two images only")
    z = np.zeros(img_h * img_w, dtype=np.int64)
    bits = img_w.bit_length() - 1
    for y in range(img_h):
        for x in range(img_w):
            t = 0
            for b in range(bits):
                t |= ((x >> b) & 1) << (2 * b)
                t |= ((y >> b) & 1) << (2 * b + 1)
            z[y * img_w + x] = t
    return z


def reorder(X: np.ndarray, img_h: int, img_w: int, to_zorder: bool) -> np.ndarray:
    """Permute the token axis of X [B, H, N, D] between raster order
    (y * img_w + x) and Z-order (zorder_index); a pure permutation."""
    z = zorder_index(img_h, img_w)
    out = np.empty_like(X)
    if to_zorder:
        out[:, :, z, :] = X
    else:
        out[:, :, :, :] = X[:, :, z, :]
    return out
