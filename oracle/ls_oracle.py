"""Plain, slow, obviously-correct CPU oracle for one decode step of a DSA-style
sparse-attention layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module; the
CUDA library shares no code, table or constant with it.  Everything here is
written from the definitions, in float64; the one encoding step (block summaries)
is defined by exact comparisons, which float64 evaluates exactly.

Sources (web pages the method is described on):
  * "LeanSparse: Memory-Efficient Serving for Native Sparse-Attention LLMs"
    (arXiv 2611.04671), abstract: sparse attention limits the history each query
    reads; the indexer keys and the KV are separate caches; coarse-to-fine indexing
    searches compact representations and re-reads original indexer keys only to
    refine candidates.
  * "XM-Sparse: Pushing the Throughput Frontier of Sparse Attention with Netpreme
    X-Mem" (LMSYS / Netpreme), section "the hot buffer reduces reads but cannot
    replace the full history": a per-request HBM hot KV buffer plus the indexer
    key cache stay on the GPU; after each step's sparse selection only the
    selected-but-missed KV is fetched; 4,096-token hot buffer, 2,048 selected per
    step.  Section "the integration point is the whole KV lifecycle": decode
    fetches only selected-but-missed KV.
  * "Related papers: SparseServe ..." page, DSA abstract: dynamic sparse attention
    restricts computation to a top-k subset of the cached KV entries.

The pages print no formula for the indexer score, the summaries, the bound or the
eviction policy.  The readings used (each stated again where it is used):
  * indexer score  S_s = sum_h w_h * ReLU(q_h . k_s)  (the DSA "lightning indexer"
    form), with q_h = sq_h * q8_h and k_s = sk_s * k8_s dequantised;
  * top-k: the k largest scores, ties broken by lower position, returned in
    ascending position order, padded with -1;
  * block summaries: per 64-token block and per dim, the max and min of the
    dequantised keys, stored as e4m3 codes times one fp32 block scale about
    amax/448, rounded outward (max up, min down) in exact arithmetic;
  * block bound: UB_j = sum_h w_h * ReLU(sum_d max(q_hd*Kmax_jd, q_hd*Kmin_jd)) for
    w_h >= 0, and w_h * ReLU(sum_d min(...)) for w_h < 0;
  * hot-buffer policy: selected resident slots are pinned; victims are the
    unpinned slots, empty ones first (by slot), then by (recent score asc, slot
    asc); the i-th miss (ascending position) takes the i-th victim; every selected
    slot's recent score becomes this step's score;
  * attention: softmax(scale * q K^T) V over the selected rows only; for MLA the
    latent row is K (576 dims) and its first 512 dims are V.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "e4m3_values", "e4m3_decode", "bf16_decode", "f32_round_up_to_e4m3_code",
    "f32_round_down_to_e4m3_code", "index_score", "topk_select", "block_summaries",
    "block_bound", "c2f_prune", "hotbuf_resolve", "gather_misses",
    "sparse_attn_decode", "decode_step", "ORACLE_PAGE",
]

ORACLE_PAGE = 64  # tokens per page / per summary block


# --------------------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------------------
def e4m3_values() -> np.ndarray:
    """float64 value of each of the 256 e4m3 codes (OCP 8-bit floating point spec,
    E4M3: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
    S.1111.111 is NaN, exponent field 0 encodes subnormals m/8 * 2^-6)."""
    out = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if (code >> 7) & 1 else 1.0
        exp_field = (code >> 3) & 0xF
        man = code & 0x7
        if exp_field == 0xF and man == 0x7:
            out[code] = np.nan
        elif exp_field == 0:
            out[code] = sign * (man / 8.0) * 2.0 ** (1 - 7)
        else:
            out[code] = sign * (1.0 + man / 8.0) * 2.0 ** (exp_field - 7)
    return out


_E4M3 = e4m3_values()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Decode uint8 e4m3 codes to float64."""
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 is the upper half of an IEEE binary32: widen the 16 bits and reinterpret."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


# finite e4m3 values in ascending order, with one canonical code per value (+0 -> 0x00)
def _e4m3_sorted():
    vals, codes = [], []
    for code in range(256):
        v = _E4M3[code]
        if np.isnan(v) or code == 0x80:  # NaNs and the negative zero are never produced
            continue
        vals.append(v)
        codes.append(code)
    order = np.argsort(np.array(vals), kind="stable")
    return np.array(vals)[order], np.array(codes, dtype=np.uint8)[order]


_E4M3_SORTED_VALS, _E4M3_SORTED_CODES = _e4m3_sorted()


def f32_round_up_to_e4m3_code(x: np.ndarray) -> np.ndarray:
    """Code of the smallest finite e4m3 value >= x (x already clamped to [-448, 448])."""
    i = np.searchsorted(_E4M3_SORTED_VALS, np.asarray(x, dtype=np.float64), side="left")
    return _E4M3_SORTED_CODES[i]


def f32_round_down_to_e4m3_code(x: np.ndarray) -> np.ndarray:
    """Code of the largest finite e4m3 value <= x (x already clamped to [-448, 448])."""
    i = np.searchsorted(_E4M3_SORTED_VALS, np.asarray(x, dtype=np.float64), side="right") - 1
    return _E4M3_SORTED_CODES[i]


# --------------------------------------------------------------------------------------
# Paged history helpers
# --------------------------------------------------------------------------------------
def _rows_of_request(pool: np.ndarray, page_table_row: np.ndarray, length: int) -> np.ndarray:
    """Rows 0..length-1 of one request's history, read through its page table.
    ``pool`` is [num_pages, page, ...]; logical position p lives in page
    page_table_row[p // page] at offset p % page."""
    page = pool.shape[1]
    n_pages = -(-length // page)
    pages = np.asarray(page_table_row[:n_pages], dtype=np.int64)
    rows = pool[pages].reshape((n_pages * page,) + pool.shape[2:])
    return rows[:length]


# --------------------------------------------------------------------------------------
# a1: indexer score
# --------------------------------------------------------------------------------------
def index_score(q, w, key_pool, page_table, lens, *, q_scale=None, key_scale_pool=None,
                key_format="e4m3", w_format="bf16"):
    """Indexer score of every cached token of every request.

    S[b, s] = sum_h w[b,h] * max(0, sum_d q[b,h,d] * k[b,s,d])   for s < lens[b]

    The pages give no scoring formula (LeanSparse, abstract, only speaks of
    "indexer keys" and "indexer scores"); this is the DSA lightning-indexer form,
    read with dequantised operands: q[b,h,:] = q_scale[b,h] * e4m3(q8[b,h,:]) and
    k[s,:] = key_scale[s] * e4m3(k8[s,:]).  With ``key_format='f32'`` q and keys are
    float32 values and no scales apply.

    Returns a list of float64 arrays, one per request, of length lens[b].
    """
    B = len(lens)
    out = []
    for b in range(B):
        L = int(lens[b])
        if key_format == "e4m3":
            qb = e4m3_decode(q[b]) * np.asarray(q_scale[b], dtype=np.float64)[:, None]
            k8 = _rows_of_request(key_pool, page_table[b], L)
            ks = _rows_of_request(key_scale_pool, page_table[b], L).astype(np.float64)
            kb = e4m3_decode(k8) * ks[:, None]
        else:
            qb = np.asarray(q[b], dtype=np.float64)
            kb = _rows_of_request(key_pool, page_table[b], L).astype(np.float64)
        wb = bf16_decode(w[b]) if w_format == "bf16" else np.asarray(w[b], dtype=np.float64)
        logits = kb @ qb.T                      # [L, H]: q_h . k_s
        out.append(np.maximum(logits, 0.0) @ wb)  # sum_h w_h ReLU(.)
    return out


# --------------------------------------------------------------------------------------
# a2: top-k selection
# --------------------------------------------------------------------------------------
def topk_select(scores_b: np.ndarray, k: int):
    """The k highest-scoring positions of one request (the DSA top-k subset of the
    cached entries), ties broken by lower position, emitted in ascending position
    order and padded with -1 when the request has fewer than k positions.

    Returns (idx int32 [k], sel_score float64 [k] with NaN padding)."""
    s = np.asarray(scores_b, dtype=np.float64)
    L = s.shape[0]
    pos = np.arange(L)
    order = np.lexsort((pos, -s))        # primary: score descending, secondary: position
    chosen = np.sort(order[: min(k, L)])
    idx = np.full(k, -1, dtype=np.int32)
    sel = np.full(k, np.nan, dtype=np.float64)
    idx[: chosen.size] = chosen
    sel[: chosen.size] = s[chosen]
    return idx, sel


# --------------------------------------------------------------------------------------
# a3: coarse-to-fine indexing
# --------------------------------------------------------------------------------------
def block_summaries(key_pool, key_scale_pool, page_table_row, length: int):
    """Compact per-block representation of one request's indexer keys (LeanSparse,
    abstract: "coarse-to-fine indexing searches compact representations").

    Per 64-token block j and dim d: Kmax_jd = max_s k_sd and Kmin_jd = min_s k_sd over
    the block's valid tokens, with k_sd = key_scale_s * e4m3(k8_sd) (an exact
    product, held in float64).  Stored as e4m3 codes times one float32 block scale:
      bs_j = amax_j / 448 rounded to float32, raised by one float32 step if then
             448 * bs_j < amax_j (so every key fits), bs_j = 1 when amax_j = 0;
      kmax code = the smallest e4m3 value v with v * bs_j >= Kmax_jd,
      kmin code = the largest  e4m3 value v with v * bs_j <= Kmin_jd,
    all comparisons exact, so the stored box contains every key of the block and
    the codes have one correct answer whatever the arithmetic used to find them.

    Returns (kmax8 uint8 [NB,D], kmin8 uint8 [NB,D], block_scale float32 [NB])."""
    k8 = _rows_of_request(key_pool, page_table_row, length)
    ks = _rows_of_request(key_scale_pool, page_table_row, length).astype(np.float64)
    keys = e4m3_decode(k8) * ks[:, None]            # exact: 4-bit x 24-bit mantissas
    nb = -(-length // ORACLE_PAGE)
    D = keys.shape[1]
    kmax8 = np.zeros((nb, D), dtype=np.uint8)
    kmin8 = np.zeros((nb, D), dtype=np.uint8)
    bscale = np.ones(nb, dtype=np.float32)
    for j in range(nb):
        blk = keys[j * ORACLE_PAGE: (j + 1) * ORACLE_PAGE]
        kmax = blk.max(axis=0)
        kmin = blk.min(axis=0)
        amax = max(np.abs(kmax).max(), np.abs(kmin).max())
        if amax == 0:
            bs = np.float32(1.0)
        else:
            bs = np.float32(amax / 448.0)
            if 448.0 * np.float64(bs) < amax:
                bs = np.nextafter(bs, np.float32(np.inf))
        scaled = _E4M3_SORTED_VALS * np.float64(bs)  # exact products, ascending
        up = np.searchsorted(scaled, kmax, side="left")
        dn = np.searchsorted(scaled, kmin, side="right") - 1
        kmax8[j] = _E4M3_SORTED_CODES[up]
        kmin8[j] = _E4M3_SORTED_CODES[dn]
        bscale[j] = bs
    return kmax8, kmin8, bscale


def block_bound(q8, q_scale, w_bits, kmax8, kmin8, bscale):
    """Per-block upper bound on the indexer score of every token in the block.

    For each head, each term q_hd*k_sd of a token in block j lies between
    min(q_hd*Kmax_jd, q_hd*Kmin_jd) and max(...), so the head's dot product lies in
    [lo_hj, hi_hj] with hi = sum_d max(...), lo = sum_d min(...).  ReLU is monotone,
    so w_h*ReLU(q_h.k_s) <= w_h*ReLU(hi_hj) when w_h >= 0 and <= w_h*ReLU(lo_hj)
    when w_h < 0.  For w_h >= 0 (the coarse-to-fine workload) this is
    UB_j = sum_h w_h ReLU(sum_d max(q_hd Kmax_jd, q_hd Kmin_jd)).

    Returns float64 [NB]."""
    q = e4m3_decode(q8) * np.asarray(q_scale, dtype=np.float64)[:, None]   # [H, D]
    w = bf16_decode(w_bits)                                               # [H]
    Kmax = e4m3_decode(kmax8) * bscale.astype(np.float64)[:, None]         # [NB, D]
    Kmin = e4m3_decode(kmin8) * bscale.astype(np.float64)[:, None]
    nb = Kmax.shape[0]
    ub = np.zeros(nb, dtype=np.float64)
    for h in range(q.shape[0]):
        a = Kmax * q[h][None, :]
        c = Kmin * q[h][None, :]
        hi = np.maximum(a, c).sum(axis=1)
        lo = np.minimum(a, c).sum(axis=1)
        if w[h] >= 0:
            ub += w[h] * np.maximum(hi, 0.0)
        else:
            ub += w[h] * np.maximum(lo, 0.0)
    return ub


def c2f_prune(scores_b, ub, k: int):
    """Coarse-to-fine pruning of one request, in two phases (the "running k-th
    threshold" read as: take the k-th best exact score over the blocks with the
    largest bounds as tau0, then keep every block whose bound reaches tau0).

    Phase 1: the ceil(k/64)+1 blocks with the largest bound (ties: lower block) are
    scored exactly; tau0 = the k-th largest of those scores (-inf if they hold fewer
    than k tokens).  Any k tokens' k-th score is at most the true k-th score, so
    tau0 never exceeds it.
    Phase 2: survivors = blocks with UB >= tau0; the top-k over the survivors'
    tokens equals the full-scan top-k, because every true top-k token has score
    >= true k-th score >= tau0 and its block's bound is at least its score.

    Returns (tau0, survivors int32 ascending, idx [k], sel [k])."""
    s = np.asarray(scores_b, dtype=np.float64)
    L = s.shape[0]
    nb = ub.shape[0]
    nb0 = min(nb, -(-k // ORACLE_PAGE) + 1)
    order = np.lexsort((np.arange(nb), -ub))
    first = np.sort(order[:nb0])
    cand = np.concatenate([s[j * ORACLE_PAGE: min(L, (j + 1) * ORACLE_PAGE)] for j in first]) \
        if nb0 else np.zeros(0)
    tau0 = -np.inf if cand.size < k else np.sort(cand)[::-1][k - 1]
    survivors = np.nonzero(ub >= tau0)[0].astype(np.int32)
    pos = np.concatenate([np.arange(j * ORACLE_PAGE, min(L, (j + 1) * ORACLE_PAGE))
                          for j in survivors]) if survivors.size else np.zeros(0, np.int64)
    sub_idx, sub_sel = topk_select(s[pos], k)
    idx = np.full(k, -1, dtype=np.int32)
    valid = sub_idx >= 0
    idx[valid] = pos[sub_idx[valid]]
    return tau0, survivors, idx, sub_sel


# --------------------------------------------------------------------------------------
# a4: hot-buffer resolve
# --------------------------------------------------------------------------------------
def hotbuf_resolve(idx_b, sel_score_b, pos_of_slot_b, recent_score_b, slot_of_pos_b):
    """One request's hit/miss classification and slot replacement against its HBM hot
    buffer (XM-Sparse, "the hot buffer reduces reads but cannot replace the full
    history": after each step's sparse selection only selected KV that misses the
    hot buffer is fetched).

    Policy (the pages name none beyond a hot buffer of recently used KV; reading):
      hit  = the selected position is resident (slot_of_pos >= 0); its slot is pinned;
      misses are listed in selection order (ascending position);
      victims = unpinned slots, empty ones first (by slot), then occupied ones by
                (recent score asc, slot asc); the i-th miss takes the i-th victim;
      the victim's old position leaves the buffer, the miss moves in;
      every selected slot's recent score is set to this step's score.

    Inputs are left untouched.  Returns a dict with sel_slot, miss_pos, miss_slot
    (each [k], -1 padded), n_miss, and the new pos_of_slot, recent_score,
    slot_of_pos."""
    k = len(idx_b)
    pos_of_slot = np.array(pos_of_slot_b, dtype=np.int32, copy=True)
    recent = np.array(recent_score_b, dtype=np.float32, copy=True)
    slot_of_pos = np.array(slot_of_pos_b, dtype=np.int32, copy=True)
    S = pos_of_slot.shape[0]
    sel = [(j, int(p)) for j, p in enumerate(idx_b) if p >= 0]
    pinned = set()
    misses = []
    sel_slot = np.full(k, -1, dtype=np.int32)
    for j, p in sel:
        s = int(slot_of_pos[p])
        if s >= 0:
            pinned.add(s)
            sel_slot[j] = s
        else:
            misses.append((j, p))
    candidates = [s for s in range(S) if s not in pinned]

    def victim_key(s):
        empty = pos_of_slot[s] < 0
        return (0, 0.0, s) if empty else (1, float(recent[s]), s)

    candidates.sort(key=victim_key)
    if len(misses) > len(candidates):
        raise ValueError("more misses than unpinned slots")
    miss_pos = np.full(k, -1, dtype=np.int32)
    miss_slot = np.full(k, -1, dtype=np.int32)
    for i, (j, p) in enumerate(misses):
        v = candidates[i]
        old = int(pos_of_slot[v])
        if old >= 0:
            slot_of_pos[old] = -1
        pos_of_slot[v] = p
        slot_of_pos[p] = v
        sel_slot[j] = v
        miss_pos[i] = p
        miss_slot[i] = v
    for j, p in sel:
        recent[sel_slot[j]] = np.float32(sel_score_b[j])
    return dict(sel_slot=sel_slot, miss_pos=miss_pos, miss_slot=miss_slot,
                n_miss=len(misses), pos_of_slot=pos_of_slot, recent_score=recent,
                slot_of_pos=slot_of_pos)


# --------------------------------------------------------------------------------------
# a5: miss gather
# --------------------------------------------------------------------------------------
def gather_misses(host_kv, page_table_row, miss_pos_b, miss_slot_b, n_miss: int, hbuf_b):
    """Copy each missed position's KV row from the full history (XM-Sparse: the full
    history lives outside HBM and decode fetches only selected-but-missed KV) into
    the slot the replacement policy gave it.  A byte copy; returns the new hot
    buffer of the request."""
    out = np.array(hbuf_b, copy=True)
    page = host_kv.shape[1]
    for i in range(n_miss):
        p = int(miss_pos_b[i])
        out[int(miss_slot_b[i])] = host_kv[int(page_table_row[p // page]), p % page]
    return out


# --------------------------------------------------------------------------------------
# a6: sparse attention
# --------------------------------------------------------------------------------------
def sparse_attn_decode(q_b, k_rows, v_rows, scale: float):
    """Attention of one decode query over only the selected rows (LeanSparse,
    abstract: sparse attention limits the history read by each query).

        s_hj = scale * q_h . K_j ;  o_h = sum_j softmax_j(s_h) V_j ;  lse_h = log sum_j e^{s_hj}

    q_b [H, Dk], k_rows [n, Dk], v_rows [n, Dv] as float64.  An empty selection gives
    o = 0 and lse = -inf.  Returns (o [H, Dv], lse [H])."""
    H = q_b.shape[0]
    n = k_rows.shape[0]
    if n == 0:
        return np.zeros((H, v_rows.shape[1])), np.full(H, -np.inf)
    s = scale * (q_b @ k_rows.T)                   # [H, n]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ v_rows) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def selected_rows(pool, page_table_row, idx_b):
    """Rows of the selected positions (ascending; -1 entries skipped), read through
    the page table from a [num_pages, page, width] pool."""
    page = pool.shape[1]
    sel = [int(p) for p in idx_b if p >= 0]
    if not sel:
        return np.zeros((0, pool.shape[2]), dtype=pool.dtype)
    return np.stack([pool[int(page_table_row[p // page]), p % page] for p in sel])


# --------------------------------------------------------------------------------------
# a7: one decode step, composed
# --------------------------------------------------------------------------------------
def decode_step(*, q8, q_scale, w_bits, key_pool, key_scale_pool, page_table, lens, k,
                q_attn_bits, kv_pool_bits, scale, dv):
    """Indexer -> top-k -> sparse MLA attention for every request, without a hot
    buffer (the history read straight from the paged KV pool).  bf16 inputs are
    given as uint16 bit patterns.  Returns (scores, idx [B,k], o [B,H,dv], lse [B,H])."""
    scores = index_score(q8, w_bits, key_pool, page_table, lens, q_scale=q_scale,
                         key_scale_pool=key_scale_pool)
    B = len(lens)
    H = q_attn_bits.shape[1]
    idx = np.full((B, k), -1, dtype=np.int32)
    o = np.zeros((B, H, dv))
    lse = np.zeros((B, H))
    for b in range(B):
        idx[b], _ = topk_select(scores[b], k)
        rows = bf16_decode(selected_rows(kv_pool_bits, page_table[b], idx[b]))
        o[b], lse[b] = sparse_attn_decode(bf16_decode(q_attn_bits[b]), rows, rows[:, :dv], scale)
    return scores, idx, o, lse


def softmax_scale_default(dk: int) -> float:
    """1/sqrt(dk): the scale stated for the fp32 workload, used for MLA too."""
    return 1.0 / math.sqrt(dk)
