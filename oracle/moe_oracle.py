"""fp64 CPU oracle for the fine-grained MoE layer forward.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product path (the CUDA library and its binding) never calls it,
and this module never imports the product package.

Every function is the plain definition of one step, written from the pages
(cited by page title and section; the three pages are listed below), in
float64 on inputs widened exactly from bf16/fp32. Library primitives used as
steps: numpy matmul, numpy stable argsort, ``scipy.special.erf``.

Pages:
  [K3-A2A]  "Kimi K3 fine-grained MoE under high concurrency" (hncyxsy.com
            news 209238): sections "物理通信拓扑" (dispatch / expert FFN /
            combine phases), "通信-计算时间比的代数拐点" (Time_comp), and
            "工业级细粒度 MoE 路由与通信掩盖实战" (FineGrainedMoERouter).
  [K3-DIAG] "Kimi K3 专家路由不均衡诊断：高负载场景下的专家利用率与排队延迟实测"
            (bjdmk.com.cn news 5375932): section 三 (MoERouteDiagnostics:
            counts, capacity, overflow, Gini, skew, stragglers), section 四
            (no-aux-loss dynamic bias: Score = Softmax(Logits + B)), section 五
            (never drop tokens; resident shared experts).
  [MOE-ARCH] "MoE architecture in production" (lpqz.cn news 86129): §2.3
            (gating network), §3.1 (expert pool of Linear-GeLU-Linear FFNs,
            MoEDispatcher grouping tokens by expert into one shared buffer).

Readings where the pages are silent or disagree (all also listed in the
design notes): selection is taken on fp32 ``s = fl32(l) + B`` (fp32 add),
ties go to the lower expert index, slots are ordered by descending s; the
combine weights are the renormalised softmax of the selected s; GeLU is the
exact erf form; no residual is added; the shared expert is added with weight
1; capacity is ``floor(T*K*cf_num / (E*cf_den))``; overflow is reported, no
copy is dropped; Gini uses one fp64 division of exact integers.

Parity pins: see ``tests/test_oracle_pins.py`` (brute-force top-K,
closed-form softmax at K=E, dispatch invariants and brute-force recount,
dense-FFN reduction at E=K=1 against torch's float64 layers, identical-expert
invariant, permutation equivariance, Gini closed forms and the
mean-absolute-difference form, hand-computed capacity/overflow cases).
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf


# --------------------------------------------------------------------------
# a1  router GEMM
# --------------------------------------------------------------------------
def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """Gate logits ``l[t, e] = sum_h x[t, h] * W_r[e, h]`` (no bias).

    [K3-A2A] "工业级细粒度 MoE 路由与通信掩盖实战": the router's gate is a
    bias-free Linear(hidden_dim, num_experts) applied to x of shape (B, H).
    [MOE-ARCH] §2.3: the gating network maps the hidden state to one logit
    per expert.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_router, dtype=np.float64)
    return x @ w.T


# --------------------------------------------------------------------------
# a2  bias + top-K selection + renormalisation
# --------------------------------------------------------------------------
def selection_scores(logits: np.ndarray, bias, noise=None) -> np.ndarray:
    """The fp32 scores the selection is decided on: ``s = fl32(fl32(l) + B)``.

    [K3-DIAG] 四: the expert bias B is added to the logits before the
    softmax used for selection. Selection is taken on ``l + B`` in fp32 (the
    kernel's precision): softmax is strictly increasing, so in exact
    arithmetic it selects the same set, and deciding on fp32 ``l + B`` avoids
    ties created or merged by rounding of exp.

    [MOE-ARCH] §2.3 (inference): Gumbel noise is added to the logits before
    the softmax, so the top-K choice is randomised and hot experts do not
    stay fixed. ``noise`` is a [T, E] array of Gumbel(0, 1) draws supplied by
    the caller; the scores are then ``fl32(fl32(l + B) + g)`` and the weights
    come from the softmax of these noisy scores.
    """
    l32 = np.asarray(logits, dtype=np.float64).astype(np.float32)
    E = l32.shape[-1]
    b32 = np.zeros(E, np.float32) if bias is None else np.asarray(bias, dtype=np.float32)
    s = (l32 + b32[None, :]).astype(np.float32)
    if noise is not None:
        s = (s + np.asarray(noise, dtype=np.float32)).astype(np.float32)
    return s


def select_topk(logits: np.ndarray, bias, K: int, noise=None):
    """Top-K experts per token and their renormalised weights.

    [K3-A2A] "工业级细粒度 MoE 路由与通信掩盖实战": scores = softmax(logits),
    take the top_k scores (descending, as torch.topk returns them), then
    divide the K weights by their sum. [K3-DIAG] 四: scores are
    Softmax(Logits + B). Ties go to the lower expert index.

    Returns (idx [T, K] int32, w [T, K] float64, s [T, E] float32).
    The weights are ``exp(s_k - s_max) / sum_{j in sel} exp(s_j - s_max)``:
    the full-E softmax denominator cancels in the renormalisation.
    """
    s = selection_scores(logits, bias, noise)
    T, E = s.shape
    if not 1 <= K <= E:
        raise ValueError("need 1 <= K <= E")
    # stable sort of -s: equal scores keep ascending expert index
    # (-0.0 and +0.0 compare equal, so they are a tie as well).
    order = np.argsort(-s.astype(np.float64), axis=1, kind="stable")
    idx = order[:, :K].astype(np.int32)
    s_sel = np.take_along_axis(s, idx, axis=1).astype(np.float64)
    z = np.exp(s_sel - s_sel[:, :1])
    w = z / z.sum(axis=1, keepdims=True)
    return idx, w, s


# --------------------------------------------------------------------------
# a3 - a5  dispatch: histogram, offsets, stable permutation
# --------------------------------------------------------------------------
def expert_counts(idx: np.ndarray, E: int) -> np.ndarray:
    """``counts[e] = #{(t, k) : idx[t, k] == e}``.

    [K3-DIAG] 三: per-expert absolute hit counts accumulated over the
    flattened top-K indices (np.add.at).
    """
    counts = np.zeros(E, dtype=np.int64)
    np.add.at(counts, np.asarray(idx).reshape(-1), 1)
    return counts.astype(np.int32)


def expert_offsets(counts: np.ndarray) -> np.ndarray:
    """Exclusive prefix sum: ``off[0] = 0``, ``off[e+1] = off[e] + counts[e]``.

    [MOE-ARCH] §3.1: all experts' token copies share one pre-allocated
    buffer; expert e owns the contiguous segment off[e] .. off[e+1]-1.
    """
    off = np.zeros(len(counts) + 1, dtype=np.int64)
    off[1:] = np.cumsum(np.asarray(counts, dtype=np.int64))
    return off.astype(np.int32)


def dispatch(idx: np.ndarray, E: int):
    """Group the T*K token copies by expert.

    [MOE-ARCH] §3.1 MoEDispatcher.dispatch: for each expert id, the indices
    of the matching entries (torch.where on the mask, i.e. ascending order)
    are written into that expert's part of the shared buffer; the experts'
    results are later scattered back to the original positions.
    [K3-DIAG] 五: no copy is dropped, whatever the expert's load.

    Copy ``c = t*K + k`` of token t goes to row ``inv[c]``; ``perm[row] = c``.
    Within expert e's segment the copies are in ascending c (= ascending t).
    Returns (counts, offsets, perm, inv), all int32.
    """
    flat = np.asarray(idx).reshape(-1)
    counts = expert_counts(idx, E)
    off = expert_offsets(counts)
    perm = np.empty(flat.size, dtype=np.int32)
    for e in range(E):
        members = np.nonzero(flat == e)[0]          # ascending copy index
        perm[off[e]:off[e + 1]] = members
    inv = np.empty(flat.size, dtype=np.int32)
    inv[perm] = np.arange(flat.size, dtype=np.int32)
    return counts, off, perm, inv


# --------------------------------------------------------------------------
# a6 - a8  expert FFN and shared expert
# --------------------------------------------------------------------------
def gelu_erf(z: np.ndarray) -> np.ndarray:
    """Exact GeLU: ``0.5 * z * (1 + erf(z / sqrt(2)))``.

    [MOE-ARCH] §3.1: each expert is two Linear layers with a GeLU between
    them (the exact erf form is taken; the pages do not name an
    approximation).
    """
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def expert_ffn(rows: np.ndarray, w1: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """``GeLU(rows @ W1^T) @ W2^T`` with W1 [D, H], W2 [H, D] (nn.Linear layout).

    [MOE-ARCH] §3.1 (Linear -> GeLU -> Linear, no biases);
    [K3-A2A] "通信-计算时间比的代数拐点": the expert costs 2*H*D
    multiply-adds per routed copy.
    """
    rows = np.asarray(rows, dtype=np.float64)
    h = gelu_erf(rows @ np.asarray(w1, dtype=np.float64).T)
    return h @ np.asarray(w2, dtype=np.float64).T


def grouped_ffn(x, perm, offsets, K, w1, w2, ws1=None, ws2=None):
    """Each expert applied to its dispatched segment, plus the shared expert.

    [MOE-ARCH] §3.1: the dispatcher calls expert[e] on the rows gathered into
    its part of the shared buffer. Row ``r`` of expert e's segment
    (offsets[e] <= r < offsets[e+1]) holds copy ``perm[r]`` of token
    ``perm[r] // K``. The shared expert ([K3-A2A] opening section, resident
    expert every token passes through) is applied to every token row.
    Returns (y_rows [T*K, H], y_shared [T, H] or None), float64.
    """
    x = np.asarray(x, dtype=np.float64)
    perm = np.asarray(perm, dtype=np.int64)
    H = x.shape[1]
    y_rows = np.zeros((perm.size, H), dtype=np.float64)
    for e in range(len(offsets) - 1):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            y_rows[a:b] = expert_ffn(x[perm[a:b] // K], w1[e], w2[e])
    y_shared = expert_ffn(x, ws1, ws2) if ws1 is not None else None
    return y_rows, y_shared


def combine(y_rows, w, inv, y_shared=None):
    """``y[t] = sum_{k<K} w[t,k] * y_rows[inv[t*K+k]] (+ y_shared[t])``.

    [K3-A2A] "物理通信拓扑", combine phase: each token's expert outputs are
    brought back and summed with their routing weights (the residual the
    page also adds belongs to the surrounding transformer and is left out);
    [MOE-ARCH] §3.1: results are scattered back to their original positions.
    """
    w = np.asarray(w, dtype=np.float64)
    T, K = w.shape
    y_rows = np.asarray(y_rows, dtype=np.float64)
    inv = np.asarray(inv, dtype=np.int64).reshape(T, K)
    y = np.zeros((T, y_rows.shape[1]), dtype=np.float64)
    for k in range(K):
        y += w[:, k:k + 1] * y_rows[inv[:, k]]
    if y_shared is not None:
        y += np.asarray(y_shared, dtype=np.float64)
    return y


# --------------------------------------------------------------------------
# a9  full layer: route, dispatch, experts, weighted combine (+ shared)
# --------------------------------------------------------------------------
def moe_layer_forward(x, w_router, bias, w1, w2, ws1, ws2, K, tokens=None, noise=None,
                      logits=None):
    """Forward pass of one fine-grained MoE FFN layer.

    Steps: gate logits, Softmax(l + B) selection of the top K with
    renormalised weights ([K3-A2A] router code; [K3-DIAG] 四), dispatch of
    the T*K copies into expert-contiguous segments ([MOE-ARCH] §3.1), each
    expert's Linear-GeLU-Linear applied to its segment, then the weighted sum
    of each token's K expert outputs back in token order ([K3-A2A]
    "物理通信拓扑", combine phase; no residual), plus the always-on shared
    expert with weight 1 when ws1/ws2 are given ([K3-A2A] opening section;
    [K3-DIAG] 五).

    ``w1``/``w2`` only need ``w1[e]`` indexing (lazy widening is allowed).
    ``tokens``: optional sorted token indices; the output is computed for
    those tokens only (routing and dispatch always cover all T tokens).
    ``noise``: optional [T, E] Gumbel draws for noisy routing ([MOE-ARCH]
    §2.3; see ``selection_scores``).
    ``logits``: optional [T, E] gate logits given by the caller (for example
    the fp32 logits a GPU run produced); the selection is then taken on
    these instead of on ``x @ W_r^T``, and every later step is unchanged. A
    parity check routes the oracle this way, so that both sides decide the
    top-K on the same fp32 numbers.

    Returns dict with logits, idx, w, s, counts, offsets, perm, inv and
    ``y`` [len(tokens), H] float64.
    """
    x = np.asarray(x, dtype=np.float64)
    T, H = x.shape
    E = np.asarray(w_router).shape[0]
    if logits is None:
        logits = router_logits(x, w_router)
    else:
        logits = np.asarray(logits, dtype=np.float64)
        if logits.shape != (T, E):
            raise ValueError("given logits must have shape [T, E]")
    idx, w, s = select_topk(logits, bias, K, noise)
    counts, off, perm, inv = dispatch(idx, E)

    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    pos = -np.ones(T, dtype=np.int64)
    pos[tok] = np.arange(tok.size)
    yr = np.zeros((tok.size, K, H), dtype=np.float64)   # expert output per copy
    for e in range(E):
        seg = perm[off[e]:off[e + 1]].astype(np.int64)
        t_of = seg // K
        keep = pos[t_of] >= 0
        if not keep.any():
            continue
        t_sel = t_of[keep]
        k_sel = seg[keep] % K
        yr[pos[t_sel], k_sel, :] = expert_ffn(x[t_sel], w1[e], w2[e])

    y = np.zeros((tok.size, H), dtype=np.float64)
    for k in range(K):                                   # combine, k ascending
        y += w[tok, k][:, None] * yr[:, k, :]
    if ws1 is not None:
        y += expert_ffn(x[tok], ws1, ws2)
    return {"logits": logits, "idx": idx, "w": w, "s": s, "counts": counts,
            "offsets": off, "perm": perm, "inv": inv, "y": y, "tokens": tok}


# --------------------------------------------------------------------------
# a10  load statistics
# --------------------------------------------------------------------------
def capacity(T: int, K: int, E: int, cf_num: int = 5, cf_den: int = 4) -> int:
    """Per-expert capacity ``floor(T*K*cf / E)`` in exact integers.

    [K3-DIAG] 三: avg = T*K/E tokens per expert, capacity =
    int(avg * capacity_factor) with capacity_factor 1.25 = 5/4.
    """
    return (T * K * cf_num) // (E * cf_den)


def capacity_page_float(T: int, K: int, E: int, cf: float = 1.25) -> int:
    """The same capacity evaluated the way [K3-DIAG] 三 writes it (float)."""
    return int((T * K) / E * cf)


def gini_exact(counts: np.ndarray) -> float:
    """Gini coefficient of the expert loads, one fp64 division of integers.

    [K3-DIAG] 三 compute_gini_coefficient: with the counts sorted ascending
    and i = 1..n, G = 2*sum(i*c_(i)) / (n*sum(c)) - (n+1)/n, and 0 when the
    total is 0 (0 = perfectly even, 1 = fully concentrated). Rewritten over
    one denominator: G = (2*sum(i*c_(i)) - (n+1)*S) / (n*S).
    """
    c = np.sort(np.asarray(counts, dtype=np.int64))
    n = c.size
    S = int(c.sum())
    if S == 0:
        return 0.0
    num = 2 * int(np.sum(np.arange(1, n + 1, dtype=np.int64) * c)) - (n + 1) * S
    return float(num) / float(n * S)


def gini_page_form(counts: np.ndarray) -> float:
    """[K3-DIAG] 三 Gini formula evaluated literally in float64."""
    c = np.sort(np.asarray(counts, dtype=np.float64))
    n = c.size
    if c.sum() == 0:
        return 0.0
    i = np.arange(1, n + 1, dtype=np.float64)
    return float(2.0 * np.sum(i * c) / (n * np.sum(c)) - (n + 1) / n)


def load_stats(counts: np.ndarray, T: int, K: int, cf_num: int = 5, cf_den: int = 4):
    """Per-expert load statistics of one routing step.

    [K3-DIAG] 三 analyze_batch_routing: capacity limit, max / min expert
    load, skew max/(min + 1e-5), copies past capacity ("dropped" on the
    page; [K3-DIAG] 五 forbids dropping, so here they are only counted as
    overflow), their rate over T*K, straggler experts (count > capacity) and
    the Gini coefficient.
    """
    c = np.asarray(counts, dtype=np.int64)
    E = c.size
    cap = capacity(T, K, E, cf_num, cf_den)
    over = np.maximum(0, c - cap)
    overflow = int(over.sum())
    mx, mn = int(c.max()), int(c.min())
    return {
        "num_copies": int(T * K),
        "capacity": int(cap),
        "max_load": mx,
        "min_load": mn,
        "skew_ratio": float(mx) / (float(mn) + 1e-5),
        "gini": gini_exact(c),
        "overflow": overflow,
        "overflow_rate": float(overflow) / float(T * K) if T * K else 0.0,
        # hottest expert over the mean load T*K/E: the skew that stays finite
        # when an expert is idle (max/(min + 1e-5) is then 1e5 * max)
        "max_over_mean": float(mx) * float(E) / float(T * K) if T * K else 0.0,
        "num_stragglers": int(np.count_nonzero(c > cap)),
        "straggler_mask": (c > cap).astype(np.uint8),
    }


# --------------------------------------------------------------------------
# dynamic expert bias update (the other half of no-aux-loss routing)
# --------------------------------------------------------------------------
def bias_update(bias, counts, T: int, K: int, gamma: float, cf_num: int = 5, cf_den: int = 4):
    """One low-frequency update of the expert bias B.

    [K3-DIAG] 四: the bias B is updated rarely by a monitor; an expert that
    stays overloaded has B_i lowered by a small step, one that stays idle has
    it raised. Reading (the page gives neither step nor period): `counts` are
    the expert loads accumulated over the caller's period and T the tokens of
    that period; overloaded means count > capacity (capacity as in
    load_stats), idle means count == 0; B_i -= gamma / += gamma, in fp32.
    Returns the new bias as float32.
    """
    b = np.asarray(bias, dtype=np.float32).copy()
    c = np.asarray(counts, dtype=np.int64)
    cap = capacity(T, K, c.size, cf_num, cf_den)
    g = np.float32(gamma)
    over = c > cap
    idle = c == 0
    b[over] = (b[over] - g).astype(np.float32)
    b[idle] = (b[idle] + g).astype(np.float32)
    return b
