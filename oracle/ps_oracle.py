"""Float64 CPU oracle for the Prefix Sliding attention hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py``.  It is plain numpy in float64, written
from the pages' definitions, with no blocking, fusion or reordering; it shares no
code with the CUDA library (``prefix_sliding_window_b200``) and imports nothing from it.

Sources (page title, section, equation):

* "Prefix Sliding 完全拆解" (pinghaoyang blog), §核心机制, eq. A(i):
  query i may attend key j iff j <= L_prefix or i - W < j <= i (1-indexed);
  every other score is -inf before the softmax.  Same section, eq. L_total:
  at most L_prefix + W keys are visible, independent of the generated length.
  Same section: the window begins after the prefix (no key counted twice);
  hidden keys are evicted outright, not down-weighted; while the sequence is
  shorter than L_total the mask is plain causal attention (warm-up).
* same page, §位置编码 (Continue PE): every token keeps its absolute position
  id; keys rotated once when cached are reused without re-rotation.
* same page, §Kernel 实现 (two-level filtering): tiles wholly in the evicted
  region are skipped (neither loaded nor computed); boundary tiles get an
  element-wise mask.
* same page, §截断回传: the trainer receives the last 4*W tokens of a rollout;
  the loss falls on the last W of them.
* same page, §引子, eq. M_KV: KV bytes per token = 2 * layers * kv_heads * head_dim
  * bytes_per_element.
* "Prefix Sliding for efficient test-time scaling" (agihunt summary): a prefix of
  100 tokens with a window of 4096 holds at most 4196 tokens.

Readings where the pages are silent (each listed in the design notes):

* Indices are 0-based here.  The 1-indexed A(i) with i = p + 1, j = k + 1 becomes
  V(p) = {k : 0 <= k <= p and (k < L_prefix or k > p - W)}; the window is the W
  positions ending at, and including, the query.
* RoPE is the rotate-half form: for i < D/2, inv_f[i] = theta^(-2i/D), angle =
  position * inv_f[i]; (x1, x2) = (x[:D/2], x[D/2:]) maps to
  (x1 cos - x2 sin, x2 cos + x1 sin).  Each query is rotated at its own
  absolute position.  theta = 1e6.
* GQA: query head h reads KV head floor(h / g), g = n_q_heads / n_kv_heads.
* softmax scale defaults to 1/sqrt(D); lse is the natural log of the
  softmax denominator including the max (lse = m + log(sum exp(s - m))).
* Ring layout (not on the pages, which use vLLM paged blocks): position p < L_prefix
  is stored in prefix row p; position p >= L_prefix in ring slot (p - L_prefix) mod W.
* Tile classification counts in-range visible (row, col) pairs of the unclipped
  Bq x Bk tile: 0 -> SKIP, Bq*Bk -> FULL, otherwise PARTIAL (ragged tail tiles are
  therefore PARTIAL).

Parity status: every function below is pinned by tests/test_oracle_pins.py except
where its docstring says "parity unpinned".
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "TILE_FULL",
    "TILE_PARTIAL",
    "rope_inv_freq",
    "rope_rotate",
    "visible_positions",
    "RingKVCache",
    "attend_gqa",
    "decode_reference",
    "full_attention_decode",
    "reset_pe_positions",
    "pinned_visible_positions",
    "pinned_decode_reference",
    "reset_pe_decode_reference",
    "prefill_reference",
    "prefill_backward_reference",
    "tile_plan",
    "tile_counts",
    "kv_bytes_per_token",
    "truncated_context",
    "default_scale",
]

TILE_FULL = 1
TILE_PARTIAL = 2


def default_scale(head_dim: int) -> float:
    """Softmax scale 1/sqrt(D) (reading: the pages leave the model's scale implicit)."""
    return 1.0 / math.sqrt(head_dim)


# ----------------------------------------------------------------------------- RoPE
def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """inv_f[i] = theta^(-2i/D) for i < D/2, float64 (rotate-half RoPE; reading)."""
    assert head_dim % 2 == 0
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * i / np.float64(head_dim))


def rope_rotate(x: np.ndarray, positions, theta: float) -> np.ndarray:
    """Rotate ``x[..., D]`` by RoPE at absolute ``positions`` (broadcast over x[..., 0]).

    Continue PE ("Prefix Sliding 完全拆解", §位置编码): the angle uses the token's
    absolute position, in float64, with no wrap-around or renumbering.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    pos = np.asarray(positions, dtype=np.float64)
    ang = pos[..., None] * rope_inv_freq(d, theta)  # [..., D/2]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ------------------------------------------------------------------- visibility
def visible_positions(p: int, l_prefix: int, window: int) -> np.ndarray:
    """Sorted key positions that query position ``p`` may attend (eq. A(i), 0-indexed).

    Brute force over every earlier position: k is kept iff k <= p and
    (k < l_prefix or k > p - window).
    """
    k = np.arange(p + 1, dtype=np.int64)
    keep = (k < l_prefix) | (k > p - window)
    return k[keep]


class RingKVCache:
    """Simulator of one sequence's bounded KV store: a pinned prefix plus W ring slots.

    Every slot remembers the absolute position it holds, so eviction can be checked
    against eq. A(i) directly.  Appending position p overwrites whatever the slot held
    before (hard eviction, "Prefix Sliding 完全拆解", §核心机制); cached keys are
    never re-rotated (Continue PE, §位置编码).
    """

    def __init__(self, l_prefix: int, window: int, n_kv_heads: int, head_dim: int,
                 theta: float):
        self.l_prefix = int(l_prefix)
        self.window = int(window)
        self.theta = float(theta)
        self.prefix: List[Optional[Tuple[int, np.ndarray, np.ndarray]]] = [None] * self.l_prefix
        self.ring: List[Optional[Tuple[int, np.ndarray, np.ndarray]]] = [None] * self.window
        self.shape = (n_kv_heads, head_dim)

    def slot_of(self, p: int) -> Tuple[str, int]:
        """Where position p lives: ("prefix", p) or ("ring", (p - L_prefix) mod W)."""
        if p < self.l_prefix:
            return "prefix", p
        return "ring", (p - self.l_prefix) % self.window

    def append(self, p: int, k_raw: np.ndarray, v: np.ndarray) -> None:
        """Rotate the raw key once at absolute position p and store (p, k_rot, v)."""
        k_rot = rope_rotate(np.asarray(k_raw, np.float64), p, self.theta)
        kind, idx = self.slot_of(p)
        entry = (int(p), k_rot, np.asarray(v, np.float64))
        if kind == "prefix":
            self.prefix[idx] = entry
        else:
            self.ring[idx] = entry

    def held_positions(self) -> List[int]:
        out = [e[0] for e in self.prefix if e is not None]
        out += [e[0] for e in self.ring if e is not None]
        return sorted(out)

    def visible_entries(self, p: int):
        """(kind, slot, position, k, v) of every stored entry visible from query p,
        ordered by position.  Found by scanning every slot."""
        vis = set(visible_positions(p, self.l_prefix, self.window).tolist())
        out = []
        for kind, store in (("prefix", self.prefix), ("ring", self.ring)):
            for idx, e in enumerate(store):
                if e is not None and e[0] in vis:
                    out.append((kind, idx, e[0], e[1], e[2]))
        out.sort(key=lambda t: t[2])
        return out

    def descriptor(self, p: int) -> Tuple[int, int, int, int]:
        """(pre_len, seg0_start, seg0_len, seg1_len) of query p, read off the slots.

        pre_len counts visible prefix rows; the visible ring slots, in position
        order, form one run from seg0_start up to the end of the ring and an
        optional second run from slot 0.  An empty window reports seg0_start 0.
        """
        ents = self.visible_entries(p)
        pre = [e for e in ents if e[0] == "prefix"]
        ring_slots = [e[1] for e in ents if e[0] == "ring"]
        if not ring_slots:
            return len(pre), 0, 0, 0
        start = ring_slots[0]
        seg0 = 1
        while seg0 < len(ring_slots) and ring_slots[seg0] == ring_slots[seg0 - 1] + 1:
            seg0 += 1
        rest = ring_slots[seg0:]
        # the remainder must be one run starting at slot 0 (after the wrap)
        for i, s in enumerate(rest):
            if s != i:
                raise AssertionError("visible ring slots do not form <= 2 runs")
        return len(pre), start, seg0, len(rest)


# -------------------------------------------------------------------- attention
def attend_gqa(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Textbook softmax attention of one query row over N keys, with GQA sharing.

    q: [Hq, D]; k, v: [N, Hkv, D] (already rotated).  Query head h reads KV head
    h // (Hq / Hkv).  Returns (out [Hq, D], lse [Hq]) in float64.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    hq = q.shape[0]
    hkv = k.shape[1]
    g = hq // hkv
    out = np.empty((hq, q.shape[1]), np.float64)
    lse = np.empty((hq,), np.float64)
    for h in range(hq):
        kv = h // g
        s = (k[:, kv, :] @ q[h]) * scale
        m = s.max()
        e = np.exp(s - m)
        den = e.sum()
        out[h] = (e @ v[:, kv, :]) / den
        lse[h] = m + math.log(den)
    return out, lse


def decode_reference(q: np.ndarray, k_rot: np.ndarray, v: np.ndarray, p: int,
                     l_prefix: int, window: int, scale: float):
    """Output of the query at absolute position p under the Prefix Sliding mask.

    q: [Hq, D] rotated at p; k_rot, v: [>= p+1, Hkv, D] indexed by absolute position
    (keys already rotated at their own positions).  Gathers V(p) and attends.
    """
    vis = visible_positions(p, l_prefix, window)
    return attend_gqa(q, k_rot[vis], v[vis], scale)


def full_attention_decode(q: np.ndarray, k_rot: np.ndarray, v: np.ndarray, p: int,
                          scale: float):
    """Full causal attention of the query at position p over keys [0, p]."""
    return attend_gqa(q, k_rot[: p + 1], v[: p + 1], scale)


def pinned_visible_positions(p: int, l_prefix: int, window: int, pinned) -> np.ndarray:
    """Visible keys when tokens are appended to the pinned prefix at run time
    ("Prefix Sliding 完全拆解", §局限: a mechanism for the model to append important tokens to
    the prefix; multi-turn: pinning later user messages into the prefix).

    The pinned set becomes the prompt rows [0, L_prefix) plus the promoted positions; a
    pinned token is never evicted.  V(p) = eq. A(i)'s set united with the promoted
    positions <= p (a promoted token still inside the window is counted once).
    """
    base = visible_positions(p, l_prefix, window)
    extra = np.asarray([t for t in pinned if t <= p], dtype=np.int64)
    return np.union1d(base, extra).astype(np.int64)


def pinned_decode_reference(q: np.ndarray, k_rot: np.ndarray, v: np.ndarray, p: int,
                            l_prefix: int, window: int, pinned, scale: float):
    """Decode output of the query at p over pinned_visible_positions (Continue PE: keys
    already rotated at their absolute positions).  Returns (out [Hq, D], lse [Hq])."""
    vis = pinned_visible_positions(p, l_prefix, window, pinned)
    return attend_gqa(q, k_rot[vis], v[vis], scale)


def reset_pe_positions(p: int, l_prefix: int, window: int):
    """Reset PE ("Prefix Sliding 完全拆解", §位置编码): the visible keys of the query at
    absolute position p, and the position ids Reset PE gives them and the query.

    The prefix keeps its ids; the window tokens are renumbered to follow the prefix
    directly (the first window token gets id L_prefix, the next L_prefix + 1, ...), and the
    query, the newest window token, gets the last of those ids.
    Returns (visible absolute positions, their Reset-PE ids, the query's Reset-PE id).
    """
    vis = visible_positions(p, l_prefix, window)
    ids = vis.copy()
    win = vis >= l_prefix
    ids[win] = l_prefix + np.arange(int(win.sum()), dtype=np.int64)
    q_id = int(ids[-1])  # the query is the last visible position (itself)
    return vis, ids, q_id


def reset_pe_decode_reference(q_raw: np.ndarray, k_raw: np.ndarray, v: np.ndarray, p: int,
                              l_prefix: int, window: int, theta: float, scale: float):
    """Decode output under Reset PE: every visible key and the query rotated at its Reset-PE
    id (reset_pe_positions), then softmax attention (eq. A(i) for the visible set).

    q_raw: [Hq, D] un-rotated query; k_raw, v: [>= p+1, Hkv, D] un-rotated keys and values
    indexed by absolute position.  Returns (out [Hq, D], lse [Hq]).
    """
    vis, ids, q_id = reset_pe_positions(p, l_prefix, window)
    q = rope_rotate(np.asarray(q_raw, np.float64), q_id, theta)
    k = rope_rotate(np.asarray(k_raw, np.float64)[vis], ids[:, None], theta)
    return attend_gqa(q, k, np.asarray(v, np.float64)[vis], scale)


def prefill_reference(Q: np.ndarray, K: np.ndarray, V: np.ndarray, l_prefix: int,
                      window: int, scale: float, rows: Optional[Sequence[int]] = None):
    """Masked prefill over sequence indices: row i attends V(i) (eq. A(i)).

    Q: [S, Hq, D], K, V: [S, Hkv, D], all already rotated.  ``rows`` selects which
    query rows to compute (default: all).  Returns (O [R, Hq, D], lse [R, Hq]).
    """
    S = Q.shape[0]
    rows = range(S) if rows is None else rows
    outs, lses = [], []
    for i in rows:
        o, l = decode_reference(Q[i], K, V, int(i), l_prefix, window, scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def prefill_backward_reference(Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray,
                               l_prefix: int, window: int, scale: float,
                               rows: Optional[Sequence[int]] = None,
                               keys: Optional[Sequence[int]] = None):
    """Gradients of the masked prefill with respect to Q, K and V.

    The truncated-backprop trainer ("Prefix Sliding 完全拆解", §截断回传) back-propagates
    through the same masked attention it ran forward; this is the chain rule of
    O_i = sum_{j in V(i)} softmax_j(s_ij) V_j with s_ij = scale * <Q_i, K_j>, written out
    per query head h (KV head h // g):

        P_ij  = softmax over j in V(i) of s_ij              (0 for j not in V(i))
        dV_j  = sum_i P_ij dO_i                             (summed over the heads of a group)
        dP_ij = <dO_i, V_j>
        D_i   = sum_j P_ij dP_ij  (= <dO_i, O_i>)
        dS_ij = P_ij (dP_ij - D_i)
        dQ_i  = scale * sum_j dS_ij K_j
        dK_j  = scale * sum_i dS_ij Q_i                     (summed over the heads of a group)

    Q, dO: [S, Hq, D]; K, V: [S, Hkv, D] (already rotated).  ``rows`` selects the query
    rows of dQ and ``keys`` the key rows of dK/dV to return (default: all).  Each head's
    masked score matrix is formed densely over the query rows that are needed (the
    selected rows plus every row that sees a selected key) and the keys [0, last row].
    Returns (dQ [R, Hq, D], dK [K, Hkv, D], dV [K, Hkv, D]) in float64.
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    dO = np.asarray(dO, np.float64)
    S, hq, d = Q.shape
    hkv = K.shape[1]
    g = hq // hkv
    rows = np.arange(S) if rows is None else np.asarray(rows, np.int64)
    keys = np.arange(S) if keys is None else np.asarray(keys, np.int64)
    # every query row that sees one of the selected keys: i >= j, and i < j + W unless
    # j is a prefix key
    need = np.zeros(S, bool)
    need[rows] = True
    for j in keys:
        hi = S if j < l_prefix else min(S, j + window)
        need[j:hi] = True
    R = np.nonzero(need)[0]
    if R.size == 0:
        return (np.zeros((0, hq, d)), np.zeros((len(keys), hkv, d)),
                np.zeros((len(keys), hkv, d)))
    ncol = int(R.max()) + 1
    j = np.arange(ncol)
    vis = (j[None, :] <= R[:, None]) & ((j[None, :] < l_prefix) | (j[None, :] > R[:, None] - window))
    where_row = {int(i): r for r, i in enumerate(R)}
    sel_rows = np.array([where_row[int(i)] for i in rows], np.int64)
    dQ = np.zeros((len(rows), hq, d))
    dK = np.zeros((len(keys), hkv, d))
    dV = np.zeros((len(keys), hkv, d))
    for h in range(hq):
        kv = h // g
        Kh, Vh = K[:ncol, kv], V[:ncol, kv]
        s = np.where(vis, (Q[R, h] @ Kh.T) * scale, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        P = e / e.sum(axis=1, keepdims=True)
        O = P @ Vh
        dP = dO[R, h] @ Vh.T
        Dr = (dO[R, h] * O).sum(axis=1, keepdims=True)
        dS = P * (dP - Dr)
        dQ[:, h] = scale * (dS[sel_rows] @ Kh)
        kin = keys < ncol
        kk = keys[kin]
        dK[kin, kv] += scale * (dS[:, kk].T @ Q[R, h])
        dV[kin, kv] += P[:, kk].T @ dO[R, h]
    return dQ, dK, dV


# ------------------------------------------------------------------- tile plan
def tile_counts(seq: int, l_prefix: int, window: int, bq: int, bk: int) -> np.ndarray:
    """Visible (row, col) pairs per (q_tile, k_tile), counted by brute force.

    Row i and column j are sequence indices < seq; a pair counts iff j is in V(i).
    """
    nq = -(-seq // bq)
    nk = -(-seq // bk)
    counts = np.zeros((nq, nk), np.int64)
    j = np.arange(seq, dtype=np.int64)
    for qt in range(nq):
        i = np.arange(qt * bq, min(seq, (qt + 1) * bq), dtype=np.int64)[:, None]
        vis = (j[None, :] <= i) & ((j[None, :] < l_prefix) | (j[None, :] > i - window))
        col = vis.sum(axis=0)  # visible rows per column
        padded = np.zeros(nk * bk, np.int64)
        padded[:seq] = col
        counts[qt] = padded.reshape(nk, bk).sum(axis=1)
    return counts


def tile_plan(seq: int, l_prefix: int, window: int, bq: int, bk: int) -> np.ndarray:
    """Two-level filtering plan ("Prefix Sliding 完全拆解", §Kernel 实现).

    Returns int32 [n, 3] rows (q_tile, k_tile, flag), q-tile-major with ascending
    k_tile, SKIP tiles omitted; flag TILE_FULL when all bq*bk pairs are visible and
    in range, TILE_PARTIAL when some but not all are.
    """
    counts = tile_counts(seq, l_prefix, window, bq, bk)
    out = []
    for qt in range(counts.shape[0]):
        for kt in range(counts.shape[1]):
            c = counts[qt, kt]
            if c == 0:
                continue
            out.append((qt, kt, TILE_FULL if c == bq * bk else TILE_PARTIAL))
    return np.asarray(out, dtype=np.int32).reshape(-1, 3)


# --------------------------------------------------------------- sizing helpers
def kv_bytes_per_token(n_layers: int, n_kv_heads: int, head_dim: int,
                       bytes_per_elem: int) -> int:
    """eq. M_KV ("Prefix Sliding 完全拆解", §引子): 2 (K and V) * L * h_kv * d * b."""
    return 2 * n_layers * n_kv_heads * head_dim * bytes_per_elem


def truncated_context(rollout_tokens: int, window: int, multiplier: int = 4):
    """Slice a trainer receives under truncated backprop ("Prefix Sliding 完全拆解", §截断回传).

    Returns (first_sent, first_loss, sent, loss_tokens): the last multiplier*W tokens
    are sent, and the loss falls on the last W of them.
    """
    sent = min(rollout_tokens, multiplier * window)
    loss = min(sent, window)
    first_sent = rollout_tokens - sent
    return first_sent, rollout_tokens - loss, sent, loss
