"""Plain fp64 attention forward on the CPU, written from the definition.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing on the product
path may import this module.

Sources (page title, section):

* "带你了解Attention,从MHA到DeepSeek", section 1.2: score = q.k, weights =
  softmax(score / sqrt(d_k)), output = weighted sum of the value rows.
* "GQA和MLA详解", section 1: ``softmax(att / sqrt(d) + causal_mask)``; section 2:
  GQA shares one K/V head among a group of query heads, K/V broadcast with
  ``repeat_interleave`` along the head axis.
* "Full 路线：保留 softmax，压缩 K/V 表示", section 三: ``repeat_kv`` expands
  [B, H_kv, S, d] to [B, H_kv * n_rep, S, d] on a new axis right after H_kv, so
  query head h reads kv head h // n_rep.
* Same page, sections 4.2-4.3, and "GQA和MLA详解" section 3: MLA caches one
  row [c_kv (512) | k_pe (64)] per token; after absorbing W_UK into the query
  the scores are q'.[c_kv | k_pe] and the values are c_kv itself.

Readings where the pages are silent (each one is a choice, listed with the
others in the design notes):

* causal alignment when Sq != Skv is bottom-right: query i of Sq sees key j
  of Skv iff j <= i + Skv - Sq (decode with Sq = 1 sees every key);
* LSE is the natural log of the sum of exp(scale * q.k) over visible keys;
  a row with no visible key has output 0 and LSE -inf;
* keys at or past a sequence's length are ignored.

Everything is computed in float64 on the exact values handed in (callers pass
the bf16/fp16 values the GPU receives, upcast).  Scores are materialised per
(batch, head): no tiling, no online softmax.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def repeat_kv(x, n_rep: int) -> np.ndarray:
    """[B, H_kv, S, d] -> [B, H_kv * n_rep, S, d], each kv head repeated n_rep
    times in place ("Full 路线" section 三 ``repeat_kv``; "GQA和MLA详解"
    section 2 ``repeat_interleave(group, dim=1)``)."""
    return np.repeat(_f64(x), n_rep, axis=1)


def visible_keys(i: int, Sq: int, skv: int, causal: bool) -> int:
    """Number of keys query row i may attend to (keys 0 .. n-1).

    Non-causal: all skv keys.  Causal, bottom-right aligned: keys j with
    j <= i + skv - Sq, clipped to [0, skv]."""
    if not causal:
        return skv
    return max(0, min(skv, i + skv - Sq + 1))


def scores(q, k, skv_lens, scale: float, causal: bool):
    """Scaled scores with masked entries set to -inf, per (b, h).

    Returns a list over b of arrays [Hq, Sq, skv_b] (float64)."""
    q, k = _f64(q), _f64(k)
    B, Hq, Sq, _ = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    out = []
    for b in range(B):
        L = int(skv_lens[b])
        s = np.full((Hq, Sq, L), -np.inf)
        for h in range(Hq):
            raw = scale * (q[b, h] @ k[b, h // G, :L].T)  # [Sq, L]
            for i in range(Sq):
                n = visible_keys(i, Sq, L, causal)
                s[h, i, :n] = raw[i, :n]
        out.append(s)
    return out


def softmax_probs(q, k, skv_lens, scale: float, causal: bool):
    """Attention weights P (rows sum to 1; masked entries 0), per b."""
    probs = []
    for s in scores(q, k, skv_lens, scale, causal):
        m = s.max(axis=-1, keepdims=True) if s.shape[-1] else np.full(s.shape[:-1] + (1,), -np.inf)
        with np.errstate(invalid="ignore"):
            e = np.where(np.isfinite(m), np.exp(s - np.where(np.isfinite(m), m, 0.0)), 0.0)
        l = e.sum(axis=-1, keepdims=True)
        probs.append(np.divide(e, l, out=np.zeros_like(e), where=l > 0))
    return probs


def attention_fwd(q, k, v, skv_lens, scale: float, causal: bool):
    """out[b,h,i,:] = sum_j softmax_j(scale * q[b,h,i].k[b,h//G,j]) v[b,h//G,j].

    q: [B, Hq, Sq, d_k]; k: [B, Hkv, >=max(skv), d_k]; v: [B, Hkv, >=max(skv), d_v].
    Returns (out [B, Hq, Sq, d_v], lse [B, Hq, Sq]) in float64.

    Two passes per row over fully materialised scores: max, then
    exp(s - max), sum, weighted sum of v, division; lse = max + log(sum)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Sq, _ = q.shape
    Hkv, d_v = k.shape[1], v.shape[-1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    out = np.zeros((B, Hq, Sq, d_v))
    lse = np.full((B, Hq, Sq), -np.inf)
    for b in range(B):
        L = int(skv_lens[b])
        for h in range(Hq):
            kh, vh = k[b, h // G, :L], v[b, h // G, :L]
            raw = scale * (q[b, h] @ kh.T)  # [Sq, L]
            for i in range(Sq):
                n = visible_keys(i, Sq, L, causal)
                if n == 0:
                    continue
                s = raw[i, :n]
                m = s.max()
                e = np.exp(s - m)
                l = e.sum()
                out[b, h, i] = (e @ vh[:n]) / l
                lse[b, h, i] = m + np.log(l)
    return out, lse


def attention_rows(q, k, v, skv_lens, scale: float, causal: bool, rows):
    """Same definition as :func:`attention_fwd`, evaluated only at the listed
    (b, h, i) rows.  Returns (out [n, d_v], lse [n]).  Used to check sampled
    outputs of full-size workloads."""
    q_t, k_t, v_t = q, k, v
    Hq = q_t.shape[1]
    Sq = q_t.shape[2]
    Hkv = k_t.shape[1]
    G = Hq // Hkv
    d_v = v_t.shape[-1]
    outs = np.zeros((len(rows), d_v))
    lses = np.full(len(rows), -np.inf)
    for r, (b, h, i) in enumerate(rows):
        L = int(skv_lens[b])
        n = visible_keys(int(i), Sq, L, causal)
        if n == 0:
            continue
        qi = _f64(q_t[b, h, i])
        kh = _f64(k_t[b, h // G, :n])
        vh = _f64(v_t[b, h // G, :n])
        s = scale * (kh @ qi)
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        outs[r] = (e @ vh) / l
        lses[r] = m + np.log(l)
    return outs, lses


def split_combine(o_parts, lse_parts):
    """Merge partial results computed over disjoint key subsets.

    o_parts [S, ..., d_v] are the per-subset normalised outputs and lse_parts
    [S, ...] their log-sum-exps.  L = log sum_s exp(lse_s);
    out = sum_s exp(lse_s - L) o_s, summed in subset order.  Subsets with
    lse = -inf contribute nothing; if all are -inf the result is (0, -inf)."""
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    m = lse_parts.max(axis=0)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    w_un = np.where(np.isfinite(lse_parts), np.exp(lse_parts - safe_m), 0.0)
    tot = w_un.sum(axis=0)
    L = np.where(tot > 0, safe_m + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    w = np.where(tot > 0, w_un / np.where(tot > 0, tot, 1.0), 0.0)
    out = np.zeros(o_parts.shape[1:])
    for s in range(o_parts.shape[0]):
        out = out + w[s][..., None] * o_parts[s]
    return out, L


def topk_attention_fwd(q, k, v, skv_lens, idx, n_sel, scale: float):
    """Attention of each query over a selected subset of its sequence's keys.

    "带你了解Attention,从MHA到DeepSeek" section 5.1 (DSA): an indexer picks the
    top-k cached entries per new token and attention is computed over those
    entries only.  The indexer itself is not modelled: the selection is an
    input.  For sequence b the selected keys are the positions
    idx[b, t], t < n_sel[b]; every query row i of every head h of b gets

        out = sum_t exp(s_t - m) v[b, h//G, idx[b,t]] / sum_t exp(s_t - m),
        s_t = scale * q[b,h,i] . k[b, h//G, idx[b,t]],  lse = m + log sum_t exp(s_t - m)

    (one selection per sequence, shared by its query rows and heads; no
    causal mask beyond the selection).  A position listed twice counts twice.
    n_sel[b] == 0 gives out 0, lse -inf.  Positions outside [0, skv[b]) raise.
    Returns (out [B, Hq, Sq, d_v], lse [B, Hq, Sq]) in float64."""
    q = _f64(q)
    idx = np.asarray(idx.tolist() if hasattr(idx, "tolist") else idx, dtype=np.int64)
    B, Hq, Sq, _ = q.shape
    Hkv, d_v = k.shape[1], v.shape[-1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, Sq, d_v))
    lse = np.full((B, Hq, Sq), -np.inf)
    for b in range(B):
        n = int(n_sel[b])
        if n == 0:
            continue
        sel = idx[b, :n]
        if sel.min() < 0 or sel.max() >= int(skv_lens[b]):
            raise ValueError(f"sequence {b}: a selected position lies outside [0, skv)")
        # only the selected rows are widened to float64 (long caches stay compact)
        ti = sel.tolist()
        ks, vs = _f64(k[b][:, ti]), _f64(v[b][:, ti])  # [Hkv, n, d]
        for h in range(Hq):
            kh, vh = ks[h // G], vs[h // G]  # [n, d]
            s = scale * (q[b, h] @ kh.T)  # [Sq, n]
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            out[b, h] = (e @ vh) / l
            lse[b, h] = (m + np.log(l))[:, 0]
    return out, lse


# --------------------------------------------------------------------------
# MLA: naive reconstruction versus attention over the absorbed latent rows.
# "Full 路线" sections 4.2-4.3; "GQA和MLA详解" section 3 (matrix absorption:
# q^T (W_uk c) = (W_uk^T q)^T c; W_uv folds into the output side).
# --------------------------------------------------------------------------

def mla_naive_decode(c_kv, k_pe, q_nope, q_rope, W_uk, W_uv, scale: float):
    """One decode query per head against T cached tokens, K and V rebuilt.

    c_kv [T, d_c], k_pe [T, d_R] (already rotated), q_nope [H, d_nope],
    q_rope [H, d_R], W_uk [d_c, H*d_nope], W_uv [d_c, H*d_v].
    K_h = [c_kv W_uk_h | k_pe], V_h = c_kv W_uv_h.  Returns [H, d_v]."""
    c_kv, k_pe, q_nope, q_rope = map(_f64, (c_kv, k_pe, q_nope, q_rope))
    W_uk, W_uv = _f64(W_uk), _f64(W_uv)
    H, d_nope = q_nope.shape
    d_v = W_uv.shape[1] // H
    out = np.zeros((H, d_v))
    for h in range(H):
        k_nope = c_kv @ W_uk[:, h * d_nope:(h + 1) * d_nope]  # [T, d_nope]
        K = np.concatenate([k_nope, k_pe], axis=1)           # [T, d_nope + d_R]
        V = c_kv @ W_uv[:, h * d_v:(h + 1) * d_v]            # [T, d_v]
        qh = np.concatenate([q_nope[h], q_rope[h]])
        s = scale * (K @ qh)
        e = np.exp(s - s.max())
        out[h] = (e @ V) / e.sum()
    return out


def mla_absorb_query(q_nope, q_rope, W_uk):
    """q'_h = [W_uk_h q_nope_h | q_rope_h], a 576-wide query per head."""
    q_nope, q_rope, W_uk = _f64(q_nope), _f64(q_rope), _f64(W_uk)
    H, d_nope = q_nope.shape
    d_c = W_uk.shape[0]
    qp = np.zeros((H, d_c + q_rope.shape[1]))
    for h in range(H):
        qp[h, :d_c] = W_uk[:, h * d_nope:(h + 1) * d_nope] @ q_nope[h]
        qp[h, d_c:] = q_rope[h]
    return qp


def mla_absorbed_decode(c_kv, k_pe, q_nope, q_rope, W_uk, W_uv, scale: float):
    """Absorbed form: MQA over cached rows [c_kv | k_pe] with V = c_kv
    (the first d_c columns of the row), then o_h = W_uv_h^T o_lat_h."""
    c_kv, k_pe = _f64(c_kv), _f64(k_pe)
    W_uv = _f64(W_uv)
    qp = mla_absorb_query(q_nope, q_rope, W_uk)         # [H, 576]
    H = qp.shape[0]
    T, d_c = c_kv.shape
    rows = np.concatenate([c_kv, k_pe], axis=1)          # [T, 576]
    o_lat, _ = attention_fwd(qp[None, :, None, :], rows[None, None], c_kv[None, None],
                             [T], scale, causal=False)
    o_lat = o_lat[0, :, 0, :]                            # [H, d_c]
    d_v = W_uv.shape[1] // H
    return np.stack([W_uv[:, h * d_v:(h + 1) * d_v].T @ o_lat[h] for h in range(H)])


# --------------------------------------------------------------------------
# KV-cache byte model ("Full 路线" sections 4.4-4.5).
# --------------------------------------------------------------------------

def kv_bytes_per_token(kind: str, H: int = 128, d_h: int = 128, G: int = 8,
                       d_c: int = 512, d_R: int = 64, elem_bytes: int = 2) -> int:
    """Bytes cached per token per layer: MHA 2*H*d_h, GQA 2*G*d_h, MQA 2*d_h,
    MLA (d_c + d_R), each times the element size."""
    if kind == "mha":
        return 2 * H * d_h * elem_bytes
    if kind == "gqa":
        return 2 * G * d_h * elem_bytes
    if kind == "mqa":
        return 2 * d_h * elem_bytes
    if kind == "mla":
        return (d_c + d_R) * elem_bytes
    raise ValueError(kind)


def mla_decode_bytes(T: int, H: int = 128, d_nope: int = 128, d_R: int = 64,
                     d_v: int = 128, d_c: int = 512, elem_bytes: int = 2):
    """Bytes of KV one decode step reads: naive = rebuilt per-head K (d_nope +
    d_R) and V (d_v) for T tokens; absorbed = the T cached latent rows."""
    naive = T * (H * (d_nope + d_R) + H * d_v) * elem_bytes
    absorbed = T * (d_c + d_R) * elem_bytes
    return naive, absorbed
