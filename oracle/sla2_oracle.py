"""CPU oracle for the SLA2 inference forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module. The product
path (the CUDA library and its binding) never calls it and shares no code,
header, table or constant with it.

What it computes, step by step, in fp64 (quantisation emulated bit for bit in
IEEE fp32 with round-to-nearest-even, no fused multiply-add):

Sources (web pages about "SLA2: Sparse-Linear Attention with Learnable Routing
and QAT", arXiv 2602.12675):
  [S]  "SLA2：基于可学习路由和量化感知训练的稀疏-线性注意力机制" summary page
       (paper.rainbus.top), first paragraph: the four-step forward pass
       (mask construction, sparse branch, linear branch, combination).
  [D]  "SLA2: Sparse-Linear Attention v2 for Diffusion Transformers" detail
       page (zhaifeiyue.github.io): §3 flowchart, §4 symbol table and Eq. 9 /
       Eq. 11 / Eq. 17, §7 implementation notes (K smoothing at the start of
       the forward pass; per-key-block h_j precomputed then accumulated).

Readings where the pages are silent or ambiguous (each one is also listed in
the design notes):
  * masked softmax: softmax(S ⊙ M) is read as a softmax over the selected
    entries only (masked logits are -inf), as P_s = P_1 / alpha in [D] §4 forces;
  * k = clamp(floor(frac * nk + 1e-3), 1, nk) key blocks per query block;
  * ranking uses the logits s (softmax is monotone), ties go to the lower j;
  * proj is y = x @ W with W stored [d_in, d_out] per head, no bias;
  * smoothing K_s = K - colmean(K) feeds the router, K-hat and phi(K); Q is
    not smoothed; phi is an unscaled softmax over the d features;
  * quantisation granularity: Q per 128-token block and K_s per 64-token
    block, symmetric INT8 (max 127); V per channel over all tokens, FP8 e4m3
    (max 448); P with a fixed x448 scale, e4m3; the row sum l uses the
    unquantised P; the linear branch is not quantised;
  * online-softmax schedule (mode "qa"): one running-max update per selected
    key block, key blocks in ascending index order;
  * k = nk: the linear branch is defined as 0 (no unselected blocks);
  * SoftTop-k ([D] §4 Eq. 17): "each row sums to k%" is read as the row
    summing to k, the count of blocks the hard Top-k keeps; lambda by bisection.

Modes of ``forward``:
  "qa" quantised, online softmax in the tile order above (the contract);
  "qb" quantised, with each row's exact final max (schedule-free bound);
  "u"  unquantised, exact masked softmax attention.

Backward pass (``head_backward``): the gradient of the unquantised forward
with respect to Q, K, V and alpha for a given block mask ([D] §7 note 3: a
hand-derived gradient, in which the linear branch's dH_i and dZ_i are formed
once per query block; [D] §2 table: the low-bit kernels are forward-only and
the backward runs in 16-bit, so the gradient is that of the unquantised
pass). Readings: the hard Top-k mask is piecewise constant in Q, K and the
projections, so it is held fixed and the router's projections receive no
gradient from this path (in training the pages route the gradient through
SoftTop-k, which is a separate function here); K smoothing is part of the
differentiated map.
"""
from __future__ import annotations

import math

import numpy as np

BQ = 128   # b_q ([S] step 1; [D] §4 symbol table)
BK = 64    # b_k
E4M3_MAX = 448.0
INT8_MAX = 127.0


# --------------------------------------------------------------------------
# Top-k count and router ([S] step 1; [D] §3 flowchart "Learnable Router")
# --------------------------------------------------------------------------
def topk_count(nk: int, frac: float) -> int:
    """Number of key blocks kept per query block for a 'k%' setting.

    ``frac`` is the fp32 value a caller passes; the count is
    floor(frac * nk + 1e-3) clamped to [1, nk] (reading: floor, since 10% of 32
    blocks is stated as 3; the guard absorbs fp32 representation error)."""
    k = int(math.floor(float(np.float32(frac)) * nk + 1e-3))
    return min(max(k, 1), nk)


def colmean(K: np.ndarray) -> np.ndarray:
    """c = mean over tokens of K (one head, [N, d]); [D] §7 note 1."""
    return K.astype(np.float64).mean(axis=0)


def pool(X: np.ndarray, b: int) -> np.ndarray:
    """Mean pooling of consecutive b-token blocks: [N, d] -> [N/b, d]; [S] step 1."""
    N, d = X.shape
    return X.astype(np.float64).reshape(N // b, b, d).mean(axis=1)


def router_scores(Q, K, Wq, Wk, smooth=True):
    """Compressed logits s_ij = proj_q(Qbar_i) . proj_k(Kbar_j) / sqrt(d).

    P_c = softmax_j(s_ij) ([S] step 1); ranking by s is the same as ranking
    by P_c because softmax is monotone within a row."""
    Q = Q.astype(np.float64)
    K = K.astype(np.float64)
    d = Q.shape[1]
    Ks = K - colmean(K) if smooth else K
    A = pool(Q, BQ) @ Wq.astype(np.float64)
    Bk = pool(Ks, BK) @ Wk.astype(np.float64)
    return (A @ Bk.T) / math.sqrt(d)


def compressed_probs(s: np.ndarray) -> np.ndarray:
    """P_c, the row softmax of the compressed logits ([S] step 1)."""
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def topk_mask(s: np.ndarray, k: int):
    """Hard Top-k per row: the k largest logits, ties to the lower block index.

    Returns the block mask M_c (uint8 [nq, nk]) and, per row, the selected
    block indices in ascending order (int32 [nq, k])."""
    nq, nk = s.shape
    mask = np.zeros((nq, nk), dtype=np.uint8)
    idx = np.zeros((nq, k), dtype=np.int32)
    j = np.arange(nk)
    for i in range(nq):
        order = np.lexsort((j, -s[i]))     # primary: -s ascending; secondary: j ascending
        sel = np.sort(order[:k])
        mask[i, sel] = 1
        idx[i] = sel
    return mask, idx


def soft_topk(pc_row: np.ndarray, k: int, tau: float, iters: int = 200):
    """SoftTop-k of one row of P_c ([D] §4 Eq. 17; [S] step 1, the training-time
    mask): m_j = sigmoid(P_c[j] / tau + lambda), with the row offset lambda
    found by bisection so that the row sums to k (the number of blocks the hard
    Top-k keeps). The row sum is strictly increasing in lambda; because
    P_c / tau lies in [0, 1 / tau], the root lies in
    [logit(k / nk) - 1 / tau, logit(k / nk)]. Returns (mask row, lambda); for
    k = nk every entry is 1 and lambda is +inf."""
    x = np.asarray(pc_row, dtype=np.float64) / tau
    nk = x.shape[0]
    if k >= nk:
        return np.ones(nk), math.inf
    target = float(k)
    base = math.log(k / (nk - k))
    lo, hi = base - 1.0 / tau, base

    def sig(t):
        with np.errstate(over="ignore"):      # exp overflow -> sigmoid 0, as intended
            return 1.0 / (1.0 + np.exp(-t))

    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if float(np.sum(sig(x + mid))) < target:
            lo = mid
        else:
            hi = mid
    lam = 0.5 * (lo + hi)
    return sig(x + lam), lam


def router_soft(q, k, proj_q, proj_k, frac, tau):
    """SoftTop-k masks and offsets for [B, H, N, d] inputs: float64
    [B, H, nq, nk] and [B, H, nq]."""
    q, k = (np.asarray(t.float() if hasattr(t, "float") else t, dtype=np.float64) for t in (q, k))
    B, H, N, d = q.shape
    nq, nk = N // BQ, N // BK
    kk = topk_count(nk, frac)
    soft = np.zeros((B, H, nq, nk))
    lam = np.zeros((B, H, nq))
    for b in range(B):
        for hh in range(H):
            s = router_scores(q[b, hh], k[b, hh], np.asarray(proj_q[hh], np.float64), np.asarray(proj_k[hh], np.float64))
            pc = compressed_probs(s)
            for i in range(nq):
                soft[b, hh, i], lam[b, hh, i] = soft_topk(pc[i], kk, tau)
    return soft, lam


# --------------------------------------------------------------------------
# Low-bit codecs (the quantised sparse branch of [S] step 2)
# --------------------------------------------------------------------------
def e4m3_round(x) -> np.ndarray:
    """Round to the nearest FP8 E4M3 value (ties to even), saturating at +-448.

    Written from the OCP FP8 E4M3 definition: exponent bias 7, 3 mantissa
    bits, largest finite 448 = 1.75 * 2^8, smallest normal 2^-6, subnormal
    step 2^-9, no infinities. Input is fp64 (or exactly representable in it);
    the result is the decoded fp64 value, sign kept (including -0)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, E = np.frexp(a)                      # a = f * 2^E, f in [0.5, 1)
    e = np.maximum(E - 1, -6)               # unbiased exponent, subnormals share -6
    quantum = np.ldexp(1.0, e - 3)          # spacing of representable values
    r = np.rint(a / quantum) * quantum      # exact division by a power of two
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_code(x) -> np.ndarray:
    """The 8-bit E4M3 encoding (uint8) of ``e4m3_round(x)``."""
    r = e4m3_round(x)
    a = np.abs(r)
    sign = np.signbit(r).astype(np.uint8) << 7
    _, E = np.frexp(a)
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, E - 1 + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, E - 1) - 1.0, a / 2.0 ** -9) * np.where(normal, 8, 1)
    mant = np.rint(mant).astype(np.int64)
    code = (exp_field.astype(np.int64) << 3) | mant
    code = np.where(a == 0, 0, code)
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(code & 0x80, -1.0, 1.0)
    e = (code >> 3) & 0xF
    m = code & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    return s * val


def quant_int8(X32: np.ndarray):
    """Symmetric INT8 of one block, in IEEE fp32: scale = amax/127,
    q = clamp(rint(x * (127/amax)), -127, 127). amax == 0 gives scale 0, q 0."""
    X32 = np.asarray(X32, dtype=np.float32)
    a = np.float32(np.max(np.abs(X32)))
    if a == 0:
        return np.zeros(X32.shape, dtype=np.int8), np.float32(0.0)
    s = np.float32(INT8_MAX)
    scale = np.float32(a / s)
    inv = np.float32(s / a)
    q = np.rint((X32 * inv).astype(np.float32))
    q = np.clip(q, -INT8_MAX, INT8_MAX).astype(np.int8)
    return q, scale


def quantize_q(Q) -> tuple:
    """Q-hat per 128-token query block; returns int8 [N, d] and scales [nq]."""
    N, d = Q.shape
    Q32 = np.asarray(Q, dtype=np.float32)
    qh = np.zeros((N, d), dtype=np.int8)
    sq = np.zeros(N // BQ, dtype=np.float32)
    for i in range(N // BQ):
        qh[i * BQ:(i + 1) * BQ], sq[i] = quant_int8(Q32[i * BQ:(i + 1) * BQ])
    return qh, sq


def smoothed_k_fp32(K, c) -> np.ndarray:
    """K_s as the quantiser sees it: fp32(K) - fp32(c), one fp32 subtraction."""
    return (np.asarray(K, dtype=np.float32) - np.asarray(c, dtype=np.float64).astype(np.float32)).astype(np.float32)


def quantize_k(K, c) -> tuple:
    """K-hat of the smoothed keys per 64-token key block; int8 [N, d], scales [nk]."""
    N, d = K.shape
    X = smoothed_k_fp32(K, c)
    kh = np.zeros((N, d), dtype=np.int8)
    sk = np.zeros(N // BK, dtype=np.float32)
    for j in range(N // BK):
        kh[j * BK:(j + 1) * BK], sk[j] = quant_int8(X[j * BK:(j + 1) * BK])
    return kh, sk


def quantize_v(V) -> tuple:
    """V-hat per channel over all tokens, FP8 e4m3: s_v = amax/448,
    v-hat = e4m3(v * (448/amax)) with the product in fp32. Returns the uint8
    codes [N, d] and the scales [d] (a zero channel gets scale 0, codes 0)."""
    V32 = np.asarray(V, dtype=np.float32)
    a = np.max(np.abs(V32), axis=0).astype(np.float32)
    safe = np.where(a == 0, np.float32(1.0), a).astype(np.float32)
    sv = np.where(a == 0, np.float32(0.0), (a / np.float32(E4M3_MAX)).astype(np.float32)).astype(np.float32)
    inv = np.where(a == 0, np.float32(0.0), (np.float32(E4M3_MAX) / safe).astype(np.float32)).astype(np.float32)
    prod = (V32 * inv[None, :]).astype(np.float32)
    return e4m3_code(prod.astype(np.float64)), sv


# --------------------------------------------------------------------------
# Sparse branch O_s ([S] step 2; [D] §3 "Sparse Branch", §7 note 2)
# --------------------------------------------------------------------------
def sparse_quantized(qh, sq, kh, sk, vcode, sv, idx_i, i, d, exact_max=False):
    """O_s for query block i with INT8 Q/K and FP8 P/V.

    Walk the selected key blocks in ascending order; per block
      S = (q-hat . k-hat) * s_q * s_k / sqrt(d)        (dequantised logits)
      m' = max(m, rowmax S); p = exp(S - m')
      l = l * exp(m - m') + sum p                       (unquantised p)
      acc = acc * exp(m - m') + e4m3(448 p) @ v-hat     (decoded codes)
    and finally O_s = acc * s_v / 448 / l. With ``exact_max`` the running max
    is replaced by the row's final max over all selected keys (mode "qb")."""
    rows = slice(i * BQ, (i + 1) * BQ)
    qi = qh[rows].astype(np.float64)
    vdec = e4m3_decode(vcode)
    rsd = 1.0 / math.sqrt(d)

    def logits(j):
        kj = kh[j * BK:(j + 1) * BK].astype(np.float64)
        return (qi @ kj.T) * float(sq[i]) * float(sk[j]) * rsd

    m = np.full(BQ, -np.inf)
    if exact_max:
        m = np.max(np.stack([logits(j).max(axis=1) for j in idx_i]), axis=0)
    l = np.zeros(BQ)
    acc = np.zeros((BQ, d))
    for j in idx_i:
        S = logits(j)
        m_new = m if exact_max else np.maximum(m, S.max(axis=1))
        p = np.exp(S - m_new[:, None])
        corr = np.exp(m - m_new) if not exact_max else np.ones(BQ)
        l = l * corr + p.sum(axis=1)
        acc = acc * corr[:, None] + e4m3_round(E4M3_MAX * p) @ vdec[j * BK:(j + 1) * BK]
        m = m_new
    return acc * sv.astype(np.float64)[None, :] / E4M3_MAX / l[:, None]


def sparse_exact(Q, Ks, V, idx_i, i, d):
    """O_s for query block i without quantisation: softmax over the selected
    keys only (masked logits are -inf), two passes in fp64."""
    rows = slice(i * BQ, (i + 1) * BQ)
    keys = np.concatenate([np.arange(j * BK, (j + 1) * BK) for j in idx_i])
    S = (Q[rows].astype(np.float64) @ Ks[keys].T) / math.sqrt(d)
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    return P @ V[keys].astype(np.float64)


# --------------------------------------------------------------------------
# Linear branch O_l ([S] step 3; [D] §3 "Linear Branch", §4 phi, §7 note 2)
# --------------------------------------------------------------------------
def feature_softmax(X) -> np.ndarray:
    """phi(x): softmax over the d features of each row."""
    X = np.asarray(X, dtype=np.float64)
    e = np.exp(X - X.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def linear_states(Ks, V):
    """Per key block j: h_j = phi(K_j)^T V_j ([d, d]) and z_j = rowsum(phi(K_j)^T) ([d])."""
    N, d = Ks.shape
    phk = feature_softmax(Ks)
    V = V.astype(np.float64)
    nk = N // BK
    h = np.zeros((nk, d, d))
    z = np.zeros((nk, d))
    for j in range(nk):
        pj = phk[j * BK:(j + 1) * BK]
        h[j] = pj.T @ V[j * BK:(j + 1) * BK]
        z[j] = pj.sum(axis=0)
    return h, z


def linear_branch(Q, h, z, mask_i, i):
    """O_l for query block i: phi(Q_i) H_i / (phi(Q_i) Z_i) with
    H_i = sum of h_j and Z_i = sum of z_j over the UNSELECTED key blocks
    (the plain definition). All blocks selected gives O_l = 0."""
    rows = slice(i * BQ, (i + 1) * BQ)
    unsel = (mask_i == 0)
    d = h.shape[1]
    if not unsel.any():
        return np.zeros((BQ, d))
    Hi = h[unsel].sum(axis=0)
    Zi = z[unsel].sum(axis=0)
    phq = feature_softmax(Q[rows])
    return (phq @ Hi) / (phq @ Zi)[:, None]


# --------------------------------------------------------------------------
# Whole forward pass for one head, and for [B, H, N, d] tensors
# --------------------------------------------------------------------------
def head_forward(Q, K, V, Wq, Wk, alpha_h, frac, mode="qa", blocks=None, k_override=None):
    """SLA2 forward for one (batch, head): returns a dict with the output O
    (fp64, rows of the requested query blocks only when ``blocks`` is given,
    else all N rows), the logits, mask, idx and both branches.

    Steps: K smoothing ([D] §7 note 1); router ([S] step 1); sparse branch
    ([S] step 2); linear branch ([S] step 3); O = alpha O_s + (1-alpha) O_l
    ([S] step 4; [D] §2 table). ``k_override`` (tests only) allows k = 0."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N, d = Q.shape
    nq, nk = N // BQ, N // BK
    k = topk_count(nk, frac) if k_override is None else k_override
    c = colmean(K)
    Ks = K - c
    s = router_scores(Q, K, Wq, Wk)
    if k > 0:
        mask, idx = topk_mask(s, k)
    else:
        mask, idx = np.zeros((nq, nk), np.uint8), np.zeros((nq, 0), np.int32)
    blocks = list(range(nq)) if blocks is None else list(blocks)
    if mode in ("qa", "qb"):
        qh, sq = quantize_q(Q)
        kh, sk = quantize_k(K, c)
        vcode, sv = quantize_v(V)
    h, z = linear_states(Ks, V)
    O = np.zeros((len(blocks) * BQ, d))
    Os = np.zeros_like(O)
    Ol = np.zeros_like(O)
    for n, i in enumerate(blocks):
        if k == 0:
            os_i = np.zeros((BQ, d))
        elif mode == "u":
            os_i = sparse_exact(Q, Ks, V, idx[i], i, d)
        else:
            os_i = sparse_quantized(qh, sq, kh, sk, vcode, sv, idx[i], i, d, exact_max=(mode == "qb"))
        ol_i = linear_branch(Q, h, z, mask[i], i)
        a = float(alpha_h[i])
        sl = slice(n * BQ, (n + 1) * BQ)
        Os[sl] = os_i
        Ol[sl] = ol_i
        O[sl] = a * os_i + (1.0 - a) * ol_i
    return {"O": O, "O_s": Os, "O_l": Ol, "scores": s, "mask": mask, "idx": idx,
            "colmean": c, "h": h, "z": z, "k": k}


def forward(q, k, v, proj_q, proj_k, alpha, frac, mode="qa"):
    """O for [B, H, N, d] inputs (numpy or torch tensors), fp64 [B, H, N, d]."""
    q, k, v = (np.asarray(t.float() if hasattr(t, "float") else t, dtype=np.float64) for t in (q, k, v))
    Wq = np.asarray(proj_q, dtype=np.float64)
    Wk = np.asarray(proj_k, dtype=np.float64)
    al = np.asarray(alpha, dtype=np.float64)
    B, H, N, d = q.shape
    out = np.zeros((B, H, N, d))
    for b in range(B):
        for hh in range(H):
            out[b, hh] = head_forward(q[b, hh], k[b, hh], v[b, hh], Wq[hh], Wk[hh], al[hh], frac, mode)["O"]
    return out


def router(q, k, proj_q, proj_k, frac):
    """Mask, idx and logits for [B, H, N, d] inputs (router stage only)."""
    q, k = (np.asarray(t.float() if hasattr(t, "float") else t, dtype=np.float64) for t in (q, k))
    B, H, N, d = q.shape
    nq, nk = N // BQ, N // BK
    kk = topk_count(nk, frac)
    masks = np.zeros((B, H, nq, nk), np.uint8)
    idxs = np.zeros((B, H, nq, kk), np.int32)
    scores = np.zeros((B, H, nq, nk))
    for b in range(B):
        for hh in range(H):
            s = router_scores(q[b, hh], k[b, hh], np.asarray(proj_q[hh], np.float64), np.asarray(proj_k[hh], np.float64))
            scores[b, hh] = s
            masks[b, hh], idxs[b, hh] = topk_mask(s, kk)
    return masks, idxs, scores


# --------------------------------------------------------------------------
# Backward pass of the unquantised forward for a fixed mask ([D] §7 note 3)
# --------------------------------------------------------------------------
def feature_softmax_backward(Y, dY) -> np.ndarray:
    """Gradient through phi = softmax over the features: given Y = phi(X) and
    dY = dL/dY (rows), returns dL/dX = Y * (dY - rowsum(dY * Y))."""
    Y = np.asarray(Y, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    return Y * (dY - np.sum(dY * Y, axis=-1, keepdims=True))


def head_forward_masked(Q, K, V, alpha_h, mask):
    """Unquantised forward of one head for a GIVEN block mask (the function the
    backward differentiates): O = alpha O_s + (1 - alpha) O_l with O_s the
    softmax attention over the selected keys ([S] step 2) and O_l the linear
    attention over the unselected key blocks ([S] step 3), K smoothed first
    ([D] §7 note 1). Returns O [N, d]."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N, d = Q.shape
    Ks = K - colmean(K)
    h, z = linear_states(Ks, V)
    O = np.zeros((N, d))
    for i in range(N // BQ):
        sel = np.nonzero(mask[i])[0]
        rows = slice(i * BQ, (i + 1) * BQ)
        os_i = sparse_exact(Q, Ks, V, sel, i, d) if len(sel) else np.zeros((BQ, d))
        ol_i = linear_branch(Q, h, z, mask[i], i)
        a = float(alpha_h[i])
        O[rows] = a * os_i + (1.0 - a) * ol_i
    return O


def unselected_blocks(mask_row) -> np.ndarray:
    """Key blocks of one mask row whose states h_j, z_j enter H_i, Z_i (the
    unselected ones, [S] step 3)."""
    return np.nonzero(np.asarray(mask_row) == 0)[0]


def head_backward(Q, K, V, alpha_h, mask, dO):
    """dL/dQ, dL/dK, dL/dV [N, d] and dL/dalpha [nq] of one head, for the
    upstream gradient dO = dL/dO, by the chain rule through the unquantised
    forward with the mask held fixed. Per query block i (rows r of block i):

      sparse branch (softmax over the selected keys, S = Q_i K_s^T / sqrt(d)):
        dV_sel += P^T dO_s,  dP = dO_s V_sel^T,  dS = P * (dP - rowsum(dP * P)),
        dQ_i += dS K_sel / sqrt(d),  dK_sel += dS^T Q_i / sqrt(d);
      linear branch (a = phi(Q_i), num = a H_i, den = a Z_i, O_l = num / den):
        dnum = dO_l / den,  dden = -rowsum(dO_l * O_l) / den,
        da = dnum H_i^T + dden Z_i^T,  dQ_i += phi-backward(a, da),
        dH_i = a^T dnum,  dZ_i = a^T dden  (formed once per query block);
      mix: dO_s = alpha_i dO, dO_l = (1 - alpha_i) dO,
        dalpha_i = sum over the block's rows and channels of dO * (O_s - O_l).

    Then, per key block j, the plain definition dh_j = sum of dH_i and
    dz_j = sum of dZ_i over the query blocks i that did NOT select j (h_j, z_j
    enter exactly those H_i, Z_i), and through h_j = phi(K_j)^T V_j,
    z_j = phi(K_j)^T 1: dV_j += phi(K_j) dh_j, dphi(K_j) = V_j dh_j^T + dz_j,
    dK_s += phi-backward(phi(K_j), dphi(K_j)). Finally through K_s = K - colmean(K):
    dK = dK_s - colmean(dK_s)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    N, d = Q.shape
    nq, nk = N // BQ, N // BK
    Ks = K - colmean(K)
    h, z = linear_states(Ks, V)
    rs = 1.0 / math.sqrt(d)
    dQ = np.zeros((N, d))
    dKs = np.zeros((N, d))
    dV = np.zeros((N, d))
    dalpha = np.zeros(nq)
    dh = np.zeros((nk, d, d))
    dz = np.zeros((nk, d))
    for i in range(nq):
        rows = slice(i * BQ, (i + 1) * BQ)
        sel = np.nonzero(mask[i])[0]
        unsel = unselected_blocks(mask[i])
        al = float(alpha_h[i])
        dOs = al * dO[rows]
        dOl = (1.0 - al) * dO[rows]
        Qi = Q[rows]
        # sparse branch
        if len(sel):
            keys = np.concatenate([np.arange(j * BK, (j + 1) * BK) for j in sel])
            S = (Qi @ Ks[keys].T) * rs
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            Os = P @ V[keys]
            dV[keys] += P.T @ dOs
            dP = dOs @ V[keys].T
            dS = P * (dP - np.sum(dP * P, axis=1, keepdims=True))
            dQ[rows] += (dS @ Ks[keys]) * rs
            dKs[keys] += (dS.T @ Qi) * rs
        else:
            Os = np.zeros((BQ, d))
        # linear branch
        if len(unsel):
            Hi = h[unsel].sum(axis=0)
            Zi = z[unsel].sum(axis=0)
            a = feature_softmax(Qi)
            num = a @ Hi
            den = a @ Zi
            Ol = num / den[:, None]
            dnum = dOl / den[:, None]
            dden = -np.sum(dOl * Ol, axis=1) / den
            da = dnum @ Hi.T + dden[:, None] * Zi[None, :]
            dQ[rows] += feature_softmax_backward(a, da)
            dHi = a.T @ dnum
            dZi = a.T @ dden
            for j in unsel:
                dh[j] += dHi
                dz[j] += dZi
        else:
            Ol = np.zeros((BQ, d))
        dalpha[i] = float(np.sum(dO[rows] * (Os - Ol)))
    phk = feature_softmax(Ks)
    for j in range(nk):
        t = slice(j * BK, (j + 1) * BK)
        dV[t] += phk[t] @ dh[j]
        dphi = V[t] @ dh[j].T + dz[j][None, :]
        dKs[t] += feature_softmax_backward(phk[t], dphi)
    dK = dKs - dKs.mean(axis=0, keepdims=True)
    return {"dQ": dQ, "dK": dK, "dV": dV, "dalpha": dalpha}
