"""Pure-Python brute force of the grouped-query attention lab functions.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.

Source: TT Lab, "キー・バリューヘッドだけ減らしてみる" (tf-gqa-lab), steps 1-7 and
their reference subsections.  Every function below works on plain nested Python
lists of floats (``heads[head][row][col]``) and uses Python's double-precision
floats, exactly as the lab asks ("standard library only").  Where the lab is
silent the reading taken is stated in the docstring.

The lab's ``attend`` has no mask.  The causal mask is the one of the course
page "Неделя 7. Внимание", step 1 ("Масштаб и маска"): scores of future keys
become -inf *before* the softmax, so each row normalises over the past only.
"""

import math

# The lab asks for "one small linear congruential generator" of the form
# state = (a*state + c) % m, emitting state/m - 0.5, but does not print a, c,
# m.  Reading: the widely published constants a=1664525, c=1013904223, m=2**32,
# state advanced before each draw, initial state = seed.
LCG_A = 1664525
LCG_C = 1013904223
LCG_M = 2 ** 32


def make_heads(count, rows, dim, seed):
    """Deterministic sample of ``count`` heads of ``rows`` x ``dim`` values.

    Lab step 1 ("クエリヘッドをグループに分ける"): an integer-state LCG, each value
    ``state / m - 0.5`` (so |x| <= 0.5 <= 4), same arguments -> same values.
    Draw order is head, then row, then column.
    """
    if count <= 0 or rows <= 0 or dim <= 0:
        raise ValueError("count, rows and dim must be positive")
    state = seed % LCG_M
    heads = []
    for _ in range(count):
        head = []
        for _ in range(rows):
            row = []
            for _ in range(dim):
                state = (LCG_A * state + LCG_C) % LCG_M
                row.append(state / LCG_M - 0.5)
            head.append(row)
        heads.append(head)
    return heads


def group_of(head, h, g):
    """KV group read by query ``head`` when ``h`` heads form ``g`` groups.

    Lab step 1: groups are contiguous blocks, number ``head // (h // g)``;
    ``head % g`` (the interleaved assignment) is wrong.  ValueError when g does
    not divide h.  Reading: a head outside [0, h) is also a ValueError.
    """
    if g <= 0 or h <= 0 or h % g != 0:
        raise ValueError(f"{g} groups do not divide {h} heads evenly")
    if not 0 <= head < h:
        raise ValueError(f"head {head} outside [0, {h})")
    return head // (h // g)


def group_members(h, g):
    """``members[j]`` = the query heads of group j, filled by calling group_of h times."""
    if g <= 0 or h <= 0 or h % g != 0:
        raise ValueError(f"{g} groups do not divide {h} heads evenly")
    members = [[] for _ in range(g)]
    for head in range(h):
        members[group_of(head, h, g)].append(head)
    return members


def fold_kv(heads, g):
    """Fold K (or V) heads into ``g`` heads by a position-wise mean per group.

    Lab step 2 ("グループ内のキー・値を1つに畳む"): one group is the contiguous slice
    heads[start:start+size]; add position by position and divide by the group
    size.  ValueError when g does not divide the head count; g == #heads gives
    the values back unchanged.
    """
    n = len(heads)
    if g <= 0 or n == 0 or n % g != 0:
        raise ValueError(f"{g} groups do not divide {n} heads evenly")
    size = n // g
    folded = []
    for grp in range(g):
        start = grp * size
        members = heads[start:start + size]
        rows = len(members[0])
        dim = len(members[0][0])
        out = []
        for r in range(rows):
            out_row = []
            for c in range(dim):
                acc = 0.0
                for m in members:
                    acc += m[r][c]
                out_row.append(acc / size)
            out.append(out_row)
        folded.append(out)
    return folded


def expand_kv(folded, h):
    """Repeat each folded head adjacently until there are ``h`` heads.

    Lab step 3 ("クエリヘッドの数だけ再び広げる"): [A, B] -> [A, A, B, B], never
    [A, B, A, B]; the outer loop runs over folded heads, the inner one
    ``h // len(folded)`` times; rows are copied so no two heads share storage.
    ValueError when len(folded) does not divide h.
    """
    n = len(folded)
    if n == 0 or h <= 0 or h % n != 0:
        raise ValueError(f"{n} heads cannot be expanded evenly to {h}")
    rep = h // n
    out = []
    for head in folded:
        for _ in range(rep):
            out.append([list(row) for row in head])
    return out


def attend(q, k, v, causal=False, scale=None, window=0, sinks=0):
    """Single-head attention of a query table against key/value tables.

    Lab step 4 ("1ヘッドのアテンションを作る"): for every query row, dot with every
    key row, divide by sqrt(head dim), softmax after subtracting the row max,
    then the softmax-weighted mean of the value rows.  Returns a table shaped
    like ``q``.

    ``causal`` adds the course page's mask (step 1 of "Неделя 7. Внимание"):
    key j is hidden from query i when j > i + (len(k) - len(q)) (the
    bottom-right alignment, i.e. j > i when the lengths agree) and its score is
    -inf before the softmax.  A row with no visible key returns zeros.
    ``scale`` overrides 1/sqrt(head dim) (the same number when left as None).

    ``window`` > 0 (with ``causal``) adds the sliding window of the course's
    step 3 ("Sliding window, attention sinks"): query row i, at key position
    p = i + (len(k) - len(q)), sees key j only if j > p - window; the first
    ``sinks`` keys stay visible to every row that may see them (j <= p).
    """
    probs = attention_probs(q, k, causal=causal, scale=scale, window=window, sinks=sinks)
    dim_v = len(v[0])
    out = []
    for p_row in probs:
        o_row = [0.0] * dim_v
        for j, p in enumerate(p_row):
            if p != 0.0:
                vj = v[j]
                for c in range(dim_v):
                    o_row[c] += p * vj[c]
        out.append(o_row)
    return out


def visible(i, j, tq, tk, causal=False, window=0, sinks=0):
    """Whether query row i may see key j (mask applied before the softmax)."""
    p = i + (tk - tq)                       # the row's position among the keys
    if causal and j > p:
        return False
    if window > 0 and j <= p - window and j >= sinks:
        return False
    return True


def attention_probs(q, k, causal=False, scale=None, window=0, sinks=0):
    """The softmax weights ``attend`` uses: one row per query, one column per key."""
    dim = len(q[0])
    if scale is None:
        scale = 1.0 / math.sqrt(dim)
    tq, tk = len(q), len(k)
    probs = []
    for i in range(tq):
        scores = []
        for j in range(tk):
            if not visible(i, j, tq, tk, causal, window, sinks):
                scores.append(-math.inf)
                continue
            dot = 0.0
            for c in range(dim):
                dot += q[i][c] * k[j][c]
            scores.append(dot * scale)
        top = max(scores)
        if top == -math.inf:
            probs.append([0.0] * tk)
            continue
        e = [math.exp(s - top) if s != -math.inf else 0.0 for s in scores]
        total = sum(e)
        probs.append([x / total for x in e])
    return probs


def heads_out(q_heads, k_heads, v_heads, g, causal=False, scale=None):
    """Multi-head outputs with K and V folded to ``g`` groups and expanded back.

    Lab step 5 ("3つの方式を同じ重みで動かす"): fold then expand the keys, fold then
    expand the values, then one ``attend`` per query head; the query heads are
    left untouched.  g == len(q_heads) must equal plain multi-head attention.
    """
    h = len(q_heads)
    ks = expand_kv(fold_kv(k_heads, g), h)
    vs = expand_kv(fold_kv(v_heads, g), h)
    return [attend(q_heads[i], ks[i], vs[i], causal=causal, scale=scale)
            for i in range(h)]


def max_gap(left, right):
    """Largest absolute difference over every head, row and column (lab step 5)."""
    gap = 0.0
    for hl, hr in zip(left, right, strict=True):
        for rl, rr in zip(hl, hr, strict=True):
            for a, b in zip(rl, rr, strict=True):
                gap = max(gap, abs(a - b))
    return gap


def kv_cache_elems(layers, kv_heads, seq_len, head_dim):
    """KV-cache element count, lab step 6: 2 (K and V) x layers x KV heads x length x head dim.

    The query-head count does not appear: queries are not cached.
    """
    for x in (layers, kv_heads, seq_len, head_dim):
        if x < 0:
            raise ValueError("counts must be non-negative")
    return 2 * layers * kv_heads * seq_len * head_dim


def kv_table(layers, h, groups, seq_len, head_dim):
    """[(g, cache elements with g KV heads), ...]; ValueError for a g that does not divide h."""
    table = []
    for g in groups:
        if g <= 0 or h % g != 0:
            raise ValueError(f"{g} groups do not divide {h} heads evenly")
        table.append((g, kv_cache_elems(layers, g, seq_len, head_dim)))
    return table


def mults(n, d_model, h, g, head_dim):
    """Multiplications of one pass through one attention layer, lab step 7.

    Projections cost n x d_model x (heads x head_dim) with heads = h for Q and
    the output, g for K and V; scores and the weighted sum cost
    h x n x n x head_dim each (after expansion every query head runs, so g does
    not enter).  Additions and the softmax exponentials are not counted.
    """
    if g <= 0 or h <= 0 or h % g != 0:
        raise ValueError(f"{g} groups do not divide {h} heads evenly")
    proj_q = n * d_model * (h * head_dim)
    proj_k = n * d_model * (g * head_dim)
    proj_v = n * d_model * (g * head_dim)
    scores = h * n * n * head_dim
    weighted = h * n * n * head_dim
    proj_out = n * (h * head_dim) * d_model
    total = proj_q + proj_k + proj_v + scores + weighted + proj_out
    return {"proj_q": proj_q, "proj_k": proj_k, "proj_v": proj_v,
            "scores": scores, "weighted": weighted, "proj_out": proj_out,
            "total": total}


def rope(x, positions, theta=10000.0):
    """Rotary position embedding of one head's rows (course "Неделя 7. Внимание",
    step 3): coordinate pair (2i, 2i+1) of the row at position m is rotated by
    the angle m * theta_i, theta_i = theta ** (-2i / d).  Reading: adjacent
    coordinates form a pair (the complex-number form of the page).
    ``x``: rows of length d (even); ``positions``: one position per row."""
    out = []
    for row, m in zip(x, positions, strict=True):
        d = len(row)
        if d % 2:
            raise ValueError("head dim must be even for RoPE")
        r = list(row)
        for i in range(d // 2):
            ang = m * theta ** (-2.0 * i / d)
            c, s = math.cos(ang), math.sin(ang)
            a, b = row[2 * i], row[2 * i + 1]
            r[2 * i] = a * c - b * s
            r[2 * i + 1] = a * s + b * c
        out.append(r)
    return out
