"""Plain fp64 CPU oracle for exact attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import or call this module.  The product path (``libfa.so`` and its
binding) never touches it; it shares no code with the CUDA kernels.

Sources (cited by page and section):
  [ctyun]  "FlashAttention" article on ctyun.cn (developer/article/562082064035909):
           section 核心思想 (the three standard passes, eight HBM reads/writes) and
           section MAC分析 / 标准Transformer MAC分析 (the 4Nd + 4N^2 access count).
  [jiahao] "Flash Attention" on special-jiahao.github.io: section Standard Attention
           (S = QK^T, P = softmax(S), O = PV) and section 增量求解 softmax (two-block merge).
  [xinc]   xinc.fun archive 235: section 6 标准注意力为什么慢 (S = QK^T/sqrt(d)) and
           section 7 Online Softmax (running max m_t, denominator l_t, weighted sum z_t,
           o = z_N / l_N; a whole block may be added per step; the backward recomputes
           scores from saved inputs and statistics).

Readings taken where the pages are silent or garbled:
  * scale: S = scale * Q K^T with scale passed explicitly (1/sqrt(d) in every workload),
    following [xinc] section 6; [jiahao] omits the factor.
  * LSE: the saved per-row statistic is the natural-log log-sum-exp of the scaled scores,
    LSE_i = m_i + ln sum_j exp(S_ij - m_i).
  * causal: key j is allowed for query i iff j <= i (square self-attention).
  * a row with no allowed key yields O = 0 and LSE = -inf.
  * backward: plain calculus of the materialised forward (below).
  * [jiahao]'s merge: f(p2) and l(p2) are taken relative to m(p2) (the page writes m(p1) in
    two places), and s(p_i)^global = f(p_i)^global / l(x) (the page writes l(p_i)^global).

Every function here is pinned by the CPU tests in ``tests/test_oracle_pins.py`` against
closed forms, invariants, a library softmax, brute force, finite differences and torch
autograd; none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def allowed_mask(nq: int, nk: int, causal: bool) -> np.ndarray:
    """Boolean [nq, nk]: True where key j may be attended by query i (j <= i when causal)."""
    if not causal:
        return np.ones((nq, nk), dtype=bool)
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    return j <= i


def scaled_scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
                  rows: np.ndarray | None = None) -> np.ndarray:
    """S = scale * Q K^T for one head ([xinc] section 6), masked entries set to -inf.

    q: [Nq, d], k: [Nk, d].  ``rows`` selects query rows (their absolute indices are used
    for the causal mask); default all rows.
    """
    q = _f64(q)
    k = _f64(k)
    if rows is None:
        rows = np.arange(q.shape[0])
    s = scale * (q[rows] @ k.T)
    if causal:
        j = np.arange(k.shape[0])[None, :]
        s = np.where(j <= rows[:, None], s, NEG_INF)
    return s


def softmax_rows(s: np.ndarray):
    """Row softmax of a score block: returns (P, m, l) with m the row max and
    l = sum_j exp(s_ij - m_i), so that P = exp(s - m) / l.  Rows that are all -inf give
    P = 0, m = -inf, l = 0."""
    s = _f64(s)
    m = s.max(axis=-1)
    m_use = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_use[..., None])
    l = e.sum(axis=-1)
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(l[..., None] > 0, e / np.where(l > 0, l, 1.0)[..., None], 0.0)
    return p, m, l


def attention_forward_head(q, k, v, scale: float, causal: bool,
                           rows: np.ndarray | None = None, row_chunk: int = 4096):
    """Standard (unfused) exact attention for one head, materialising S and P
    ([jiahao] Standard Attention; [xinc] section 6):
        S = scale * Q K^T,  P = softmax(S) row-wise,  O = P V,
    and LSE_i = m_i + ln l_i.  Returns (O [R, d], LSE [R]) for the selected rows.

    Rows are processed in chunks of ``row_chunk`` query rows, each holding its complete
    key rows of S and P; softmax is row-wise, so this is the same computation (it only
    bounds memory for very long sequences).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    if rows is None:
        rows = np.arange(q.shape[0])
    rows = np.asarray(rows)
    o = np.zeros((rows.shape[0], v.shape[1]))
    lse = np.full(rows.shape[0], NEG_INF)
    for c0 in range(0, rows.shape[0], row_chunk):
        r = rows[c0:c0 + row_chunk]
        s = scaled_scores(q, k, scale, causal, r)
        p, m, l = softmax_rows(s)
        o[c0:c0 + row_chunk] = p @ v
        with np.errstate(divide="ignore"):
            lse[c0:c0 + row_chunk] = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), NEG_INF)
    return o, lse


def attention_forward(q, k, v, scale: float, causal: bool):
    """Exact attention over [B, H, N, d] inputs; returns O [B,H,N,d] and LSE [B,H,N]."""
    q = _f64(q)
    B, H, N, d = q.shape
    o = np.zeros((B, H, N, v.shape[-1]))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_forward_head(q[b, h], k[b, h], v[b, h], scale, causal)
    return o, lse


# ---------------------------------------------------------------------------- FP8 inputs
# [xinc] section 4 (减少访存的几种办法): matmul operands may be held in a low-precision format
# such as FP8 while accumulation and softmax stay at higher precision.  With FP8 inputs the
# attention to compute is that of the values the codes represent; the oracle decodes them
# exactly and runs the fp64 attention above on them.

def e4m3_decode(codes) -> np.ndarray:
    """fp64 values of FP8 E4M3 codes (uint8), from the format's definition (the "FN" variant:
    no infinities): bit 7 sign, bits 3-6 exponent e with bias 7, bits 0-2 mantissa m.
      e = 0          : subnormal, (m / 8) * 2^-6   (so 0x01 = 2^-9 and 0x00 = +0)
      e = 1..15      : (1 + m / 8) * 2^(e - 7)     (largest finite: e = 15, m = 6 -> 448)
      e = 15, m = 7  : NaN
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def attention_forward_fp8(q8, k8, v8, descale_q, descale_k, descale_v, scale: float,
                          causal: bool):
    """Exact attention of FP8 (E4M3) inputs [B,H,N,d] given as uint8 codes, each (b, h) slice
    representing code value * descale[b, h] (descale arrays [B, H]; None means 1).  Returns
    (O [B,H,N,d], LSE [B,H,N]) in fp64."""
    q = e4m3_decode(q8)
    k = e4m3_decode(k8)
    v = e4m3_decode(v8)
    B, H = q.shape[:2]
    ones = np.ones((B, H))
    dq = ones if descale_q is None else _f64(descale_q).reshape(B, H)
    dk = ones if descale_k is None else _f64(descale_k).reshape(B, H)
    dv = ones if descale_v is None else _f64(descale_v).reshape(B, H)
    o = np.zeros(v.shape)
    lse = np.zeros(q.shape[:3])
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_forward_head(q[b, h] * dq[b, h], k[b, h] * dk[b, h],
                                                        v[b, h] * dv[b, h], scale, causal)
    return o, lse


def attention_backward_head(q, k, v, do, scale: float, causal: bool, row_chunk: int = 4096,
                            rows: np.ndarray | None = None, o=None):
    """Gradients of O = softmax(scale * Q K^T) V for one head, by plain calculus of the
    materialised forward (the pages only say the backward recomputes the scores from the
    saved inputs and a few statistics, [xinc] section 7):
        dV = P^T dO
        dP = dO V^T
        D_i = sum_j P_ij dP_ij
        dS = P * (dP - D_i)
        dQ = scale * dS K
        dK = scale * dS^T Q
    Masked entries have P = 0 and so contribute nothing.  The sums over query rows in dV
    and dK are split into chunks of ``row_chunk`` rows only to bound memory.  ``rows``
    restricts the computation to the given query rows: dQ and D are then filled for those
    rows only and dK, dV hold those rows' contributions (used to time bounded samples).
    ``o``, when given, is a stored forward output [N, d] (for instance the bf16 O a kernel
    wrote): D_i is then rowsum(dO o O) of that O, which equals sum_j P_ij dP_ij when O = P V
    exactly, so that the gradients are those of a backward that reads the saved output (the
    pages' backward works from the saved inputs and statistics, [xinc] section 7).
    Returns (dQ, dK, dV, D).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    o = None if o is None else _f64(o)
    N = q.shape[0]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dvec = np.zeros(N)
    all_rows = np.arange(N) if rows is None else np.asarray(rows)
    for c0 in range(0, all_rows.shape[0], row_chunk):
        r = all_rows[c0:c0 + row_chunk]
        s = scaled_scores(q, k, scale, causal, r)
        p, _, _ = softmax_rows(s)
        dv += p.T @ do[r]
        dp = do[r] @ v.T
        dvec[r] = (p * dp).sum(axis=-1) if o is None else (do[r] * o[r]).sum(axis=-1)
        ds = p * (dp - dvec[r][:, None])
        dq[r] = scale * (ds @ k)
        dk += scale * (ds.T @ q[r])
    return dq, dk, dv, dvec


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Backward over [B, H, N, d]; returns (dQ, dK, dV, D) with D [B,H,N]."""
    q = _f64(q)
    B, H, N, d = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(q)
    dv = np.zeros((B, H, N, v.shape[-1]))
    dvec = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h], dvec[b, h] = attention_backward_head(
                q[b, h], k[b, h], v[b, h], do[b, h], scale, causal)
    return dq, dk, dv, dvec


# --------------------------------------------------------------------------------------
# The pages' own constructions, written out so that they can pin the oracle above.
# --------------------------------------------------------------------------------------

def two_block_softmax(x, k: int):
    """Softmax of a vector from its two blocks p1 = x[:k], p2 = x[k:] ([jiahao] 增量求解
    softmax): each block's local max m(p_i), exponentials f(p_i) and sum l(p_i); then
    m(x) = max(m(p1), m(p2)), f(p_i)^global = f(p_i) e^{m(p_i) - m(x)},
    l(p_i)^global = l(p_i) e^{m(p_i) - m(x)}, l(x) = l(p1)^global + l(p2)^global and
    s(p_i)^global = f(p_i)^global / l(x).  Returns (softmax(x), m(x), l(x))."""
    x = _f64(x)
    p1, p2 = x[:k], x[k:]
    m1, m2 = p1.max(), p2.max()
    f1, f2 = np.exp(p1 - m1), np.exp(p2 - m2)
    l1, l2 = f1.sum(), f2.sum()
    mx = max(m1, m2)
    f1g, f2g = f1 * math.exp(m1 - mx), f2 * math.exp(m2 - mx)
    l1g, l2g = l1 * math.exp(m1 - mx), l2 * math.exp(m2 - mx)
    lx = l1g + l2g
    return np.concatenate([f1g / lx, f2g / lx]), mx, lx


def online_softmax_elementwise(s, vals):
    """The element-wise recurrence of [xinc] section 7 for one query row:
        m_{t+1} = max(m_t, s_{t+1})
        l_{t+1} = e^{m_t - m_{t+1}} l_t + e^{s_{t+1} - m_{t+1}}
        z_{t+1} = e^{m_t - m_{t+1}} z_t + e^{s_{t+1} - m_{t+1}} v_{t+1}
    starting from the first element, and o = z_N / l_N.  Returns (o, m_N, l_N)."""
    s = _f64(s)
    vals = _f64(vals)
    m = s[0]
    l = 1.0
    z = vals[0].copy()
    for t in range(1, s.shape[0]):
        m_new = max(m, s[t])
        a = math.exp(m - m_new)
        e = math.exp(s[t] - m_new)
        l = a * l + e
        z = a * z + e * vals[t]
        m = m_new
    return z / l, m, l


def online_softmax_blocks(s, vals, block_sizes):
    """Block-at-a-time form of the same recurrence ([xinc] section 7: a whole block may be
    added per step): for each block, m_new = max(m, max(block)); the old l and z are
    multiplied by e^{m - m_new}; the block adds sum e^{s - m_new} and sum e^{s - m_new} v.
    Returns (o, m, l)."""
    s = _f64(s)
    vals = _f64(vals)
    m = -np.inf
    l = 0.0
    z = np.zeros(vals.shape[1])
    t = 0
    for bsz in block_sizes:
        blk = s[t:t + bsz]
        vb = vals[t:t + bsz]
        t += bsz
        m_new = max(m, blk.max())
        a = 0.0 if m == -np.inf else math.exp(m - m_new)
        e = np.exp(blk - m_new)
        l = a * l + e.sum()
        z = a * z + e @ vb
        m = m_new
    assert t == s.shape[0], "block sizes must cover the row"
    return z / l, m, l


class CountingMemory:
    """Counts single-element reads and writes of whole matrices held in "HBM"
    ([ctyun] MAC分析: the unit is one float access)."""

    def __init__(self):
        self.reads = 0
        self.writes = 0
        self.store = {}
        self.per_line = []

    def end_line(self):
        """Close one pass: record its (reads, writes) since the previous pass."""
        r0 = sum(x[0] for x in self.per_line)
        w0 = sum(x[1] for x in self.per_line)
        self.per_line.append((self.reads - r0, self.writes - w0))

    def write(self, name, arr):
        arr = _f64(arr)
        self.writes += arr.size
        self.store[name] = arr

    def read(self, name):
        arr = self.store[name]
        self.reads += arr.size
        return arr


def standard_attention_counted(q, k, v):
    """The three standard passes of [ctyun] 核心思想 / [jiahao] Standard Attention for one
    head, with every matrix read from and written to a counting memory:
        line 1: read Q, K; S = Q K^T; write S
        line 2: read S; P = softmax(S); write P
        line 3: read P, V; O = P V; write O
    (unscaled, as on those pages).  Returns (O, memory) where memory.reads + memory.writes
    is the access count the article totals as 4Nd + 4N^2 and memory.per_line holds the
    (reads, writes) of each pass."""
    mem = CountingMemory()
    mem.write("Q", q)
    mem.write("K", k)
    mem.write("V", v)
    mem.reads = mem.writes = 0
    s = mem.read("Q") @ mem.read("K").T
    mem.write("S", s)
    mem.end_line()
    p, _, _ = softmax_rows(mem.read("S"))
    mem.write("P", p)
    mem.end_line()
    o = mem.read("P") @ mem.read("V")
    mem.write("O", o)
    mem.end_line()
    return o, mem


def brute_force_attention(q, k, v, scale: float, causal: bool):
    """Pure-Python triple loop with math.exp and math.fsum, for tiny shapes only.
    q, k, v are nested lists (or arrays) [N][d].  Returns (O, LSE) as lists."""
    n = len(q)
    d = len(q[0])
    dv = len(v[0])
    out, lses = [], []
    for i in range(n):
        keys = [j for j in range(len(k)) if (not causal or j <= i)]
        if not keys:
            out.append([0.0] * dv)
            lses.append(-math.inf)
            continue
        sc = [scale * math.fsum(float(q[i][c]) * float(k[j][c]) for c in range(d)) for j in keys]
        mx = max(sc)
        ex = [math.exp(x - mx) for x in sc]
        den = math.fsum(ex)
        out.append([math.fsum(ex[t] * float(v[keys[t]][c]) for t in range(len(keys))) / den
                    for c in range(dv)])
        lses.append(mx + math.log(den))
    return out, lses
