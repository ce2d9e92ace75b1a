"""Plain fp64 CPU oracle for the Lookahead Sparse Attention indexer step.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
baseline may import this module; the library never calls it and it calls nothing of
the library.  It is deliberately slow and literal: numpy in float64, one library
primitive (matmul, sort, exp) per step, no blocking or fusion, so that each function
can be checked by eye against the passage it cites.

Pages (cited by title and section):
  [REVIEW]  "论文综述：FlashMemory-DeepSeek-V4 用前瞻稀疏注意力压缩超长上下文KV缓存"
            (paper.oopus.info), part 二 "核心方法与创新".
  [SUMMARY] "技术摘要：通过前瞻性稀疏注意力机制实现的 FlashMemory-DeepSeek-V4"
            (gist.science), §2.1 架构设计, §2.2 数据策展与标注, §2.3 无骨干解耦训练,
            §2.4 最优配置.

Readings taken where the pages are silent (each is listed in the design notes):
  * score: z = sum_h w_h * ReLU(q_h . k_s) + b, I = sigmoid(z); no 1/sqrt(d) factor,
    no positional rotation; w = h W_w; the query is linear low rank, q = (h W_down) W_up.
  * precision boundaries of the projection for bf16 models: c = h W_down and
    q = c W_up are each rounded to bf16 (nearest even) from an exact sum; w stays exact.
  * e4m3 keys carry a per-entry scale s > 0: k = s * decode(code).
  * threshold: marked  <=>  I >= 0.5  <=>  z >= 0.
  * top-k inside the fetched set ranks by the largest logit over the layers that
    marked the entry; equal keys -> lower entry index first; |U| <= k -> all of U.
  * the native indexer's fine selection scores the fetched entries with the same
    head-fused ReLU form, its own per-token query and keys, no bias or gate.
  * nucleus: descending probability, equal probability -> lower index first; the
    smallest prefix whose mass reaches top_p (an entry is in it iff the mass strictly
    before it is < top_p).
  * loss: mean BCE and mean focal loss (gamma, no alpha), reported separately, with
    probabilities clamped to [2^-20, 1 - 2^-20].
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------- formats


def decode_bf16(u16) -> np.ndarray:
    """bf16 bit patterns -> float64 (a bf16 is the top half of an IEEE binary32)."""
    u = np.asarray(u16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):          # NaN patterns stay NaN
        return u.view(np.float32).astype(np.float64)


def decode_e4m3(u8) -> np.ndarray:
    """OCP 8-bit floating point E4M3 ("fn" variant) codes -> float64.

    Sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0 holds
    subnormals m/8 * 2**-6; S.1111.111 is NaN; there is no infinity.
    """
    c = np.asarray(u8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.power(2.0, e - 7)
    sub = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, v)


def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even (returned as float64).

    bf16: 8 significant bits, exponent range of binary32 (normals down to 2**-126,
    subnormal spacing 2**-133).  Values past the largest finite bf16 become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    fin = np.isfinite(x) & (x != 0)
    m, e = np.frexp(x[fin])                # x = m * 2**e, 0.5 <= |m| < 1
    e_q = np.maximum(e, -125)              # quantum 2**(e_q - 8); 2**-133 below 2**-126
    q = np.ldexp(np.rint(np.ldexp(m, 8 + e - e_q)), e_q - 8)   # rint: ties to even
    big = np.abs(q) > float.fromhex("0x1.fep127")
    q = np.where(big, np.copysign(np.inf, q), q)
    out[fin] = q
    out[~fin] = x[~fin]
    return out


# ----------------------------------------------------------------------------- query


def project_query(h, W_down, W_up, W_w, H: int, dI: int, bf16_boundaries: bool):
    """Low-rank dual-encoder query of one (sequence, indexer layer).

    [SUMMARY] §2.1 (memory indexer: the current token's hidden state h_t is mapped to
    a low-rank indexer query) and §2.3 (only the low-rank query projections are
    trained).  c = h W_down (rank r), q = c W_up reshaped to [H][dI], w = h W_w [H].
    """
    h = np.asarray(h, dtype=np.float64)
    c = h @ np.asarray(W_down, dtype=np.float64)
    if bf16_boundaries:
        c = round_to_bf16(c)
    q = c @ np.asarray(W_up, dtype=np.float64)
    if bf16_boundaries:
        q = round_to_bf16(q)
    w = h @ np.asarray(W_w, dtype=np.float64)
    return q.reshape(H, dI), w


# ----------------------------------------------------------------------------- score


def head_fused_logits(q, w, b: float, K) -> np.ndarray:
    """Pre-sigmoid lookahead index logit z_s for every key row of K [N][dI].

    [SUMMARY] §2.1 (scoring: a head-fused, sigmoid-gated matching score between the
    indexer query and every earlier compressed KV entry s):
        z_s = sum_h w_h * max(0, q_h . k_s) + b,   I_{t,s} = sigmoid(z_s).
    """
    q = np.asarray(q, dtype=np.float64)        # [H][dI]
    K = np.asarray(K, dtype=np.float64)        # [N][dI]
    dots = K @ q.T                             # [N][H], dots[s, h] = q_h . k_s
    return np.maximum(dots, 0.0) @ np.asarray(w, dtype=np.float64) + b


def sigmoid(z) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def threshold_mark(z) -> np.ndarray:
    """Entries to fetch: I >= 0.5 ([SUMMARY] §2.1 dynamic fetch; [REVIEW] 二).

    sigmoid is increasing with sigmoid(0) = 0.5, so I >= 0.5 exactly when z >= 0.
    """
    return np.asarray(z) >= 0.0


# ----------------------------------------------------------------------------- bit sets


def pack_bits(mark) -> np.ndarray:
    """bool [N] -> uint32 words, bit i of word j = entry 32*j + i; bits past N are 0."""
    mark = np.asarray(mark, dtype=bool)
    n = mark.shape[-1]
    nw = (n + 31) // 32
    pad = np.zeros(mark.shape[:-1] + (nw * 32,), dtype=bool)
    pad[..., :n] = mark
    bits = pad.reshape(mark.shape[:-1] + (nw, 32)).astype(np.uint64)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (bits * weights).sum(axis=-1).astype(np.uint32)


def unpack_bits(words, n: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint32)
    bits = (words[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(words.shape[:-1] + (-1,))[..., :n].astype(bool)


def or_union(marks_by_layer):
    """Multi-layer routing in OR mode ([SUMMARY] §2.4; [REVIEW] 二, conservative policy).

    Layers are taken in order; new_l = mark_l AND NOT (union of earlier layers), which
    is what an incremental fetch needs; the final union is the OR of all layers.
    Returns (union bool [N], [new_l bool [N] for each layer]).
    """
    U = np.zeros_like(np.asarray(marks_by_layer[0], dtype=bool))
    news = []
    for m in marks_by_layer:
        m = np.asarray(m, dtype=bool)
        news.append(m & ~U)
        U = U | m
    return U, news


def compact(mark) -> np.ndarray:
    """Fetch list: ascending indices of the marked entries (its length is the count)."""
    return np.flatnonzero(np.asarray(mark, dtype=bool)).astype(np.int64)


# ----------------------------------------------------------------------------- top-k


def topk_in_fetched(fetched_idx, key_of_entry, k: int) -> np.ndarray:
    """Fine top-k inside the fetched subset ([SUMMARY] §2.1, hierarchical selection).

    Candidates are the fetched entries only.  Order by descending key, equal keys by
    ascending entry index; keep the first min(k, |fetched|); return them in ascending
    index order.
    """
    idx = np.asarray(fetched_idx, dtype=np.int64)
    if idx.size == 0 or k <= 0:
        return np.zeros(0, dtype=np.int64)
    key = np.asarray(key_of_entry, dtype=np.float64)[idx]
    order = np.lexsort((idx, -key))            # primary: -key, secondary: index
    return np.sort(idx[order[:k]])


def fetched_key(z_by_layer, marks_by_layer) -> np.ndarray:
    """Per-entry key for the top-k: the largest z_l over layers l that marked the entry
    (-inf where no layer marked it)."""
    z = np.asarray(z_by_layer, dtype=np.float64)
    m = np.asarray(marks_by_layer, dtype=bool)
    return np.where(m, z, -np.inf).max(axis=0)


def fine_index_scores(q_f, w_f, K_f, fetched_idx) -> np.ndarray:
    """Native-indexer score of every fetched entry for the current token ([SUMMARY] §2.1,
    hierarchical selection: once the fetched subset is in GPU memory, the backbone's own
    Lightning Indexer makes a fine top-k choice inside it for the core attention).

    The pages name the native indexer but do not print its formula.  Reading: the same
    head-fused ReLU form as the lookahead score, with the backbone indexer's per-token
    query (q_f [H][dI], head weights w_f [H]) and its own keys K_f [N][dI]; no bias and no
    sigmoid (neither changes an ordering).  Returns the scores of fetched_idx, in its order.
    """
    idx = np.asarray(fetched_idx, dtype=np.int64)
    K = np.asarray(K_f, dtype=np.float64)[idx]
    return head_fused_logits(q_f, w_f, 0.0, K)


def fine_topk(q_f, w_f, K_f, fetched_idx, k: int) -> np.ndarray:
    """The fine top-k of the fetched subset by the native-indexer score: candidates are the
    fetched entries only; ties and ordering as in topk_in_fetched."""
    idx = np.asarray(fetched_idx, dtype=np.int64)
    key = np.full(np.asarray(K_f).shape[0], -np.inf)
    key[idx] = fine_index_scores(q_f, w_f, K_f, idx)
    return topk_in_fetched(idx, key, k)


# ----------------------------------------------------------------------------- gather


def gather_rows(cold, idx) -> np.ndarray:
    """Cold pool -> hot pool: the rows of the fetched entries, in fetch-list order
    ([SUMMARY] §2.1 dynamic fetch from the CPU cold pool into GPU memory)."""
    return np.asarray(cold)[np.asarray(idx, dtype=np.int64)]


# ----------------------------------------------------------------------------- hot pool


class HotPool:
    """Residency of fetched rows across triggers, for one sequence.

    [SUMMARY] §2.1 and [REVIEW] 二: the indexer runs every tau decode steps and keeps
    only the KV blocks it predicts as needed in GPU memory, fetching them from the CPU
    cold pool.  The pages do not say what happens to rows fetched by an earlier trigger;
    the reading taken here: a row stays in its hot-pool slot until its slot is needed
    for a row the current trigger wants and the pool has no free slot, so only rows
    not yet resident cross the host link.

    State: slot_of[e] (-1 if entry e is not resident), entry_of[s] (-1 if slot s is
    free), stamp[s] (the last trigger whose fetch set contained slot s's entry; 0 for
    a slot never used).  One update with fetch set U at trigger t >= 1:
      1. every resident entry of U gets stamp t (its slot is kept);
      2. need = entries of U not resident, ascending;
      3. if |U| > slots the update fails (nothing moves, stamps of step 1 stay);
      4. the candidate slots are those not kept, in order of (stamp, slot): free slots
         first, then the least recently needed; the first |need| of them are taken;
      5. the i-th entry of need goes to the i-th taken slot in ascending slot order,
         evicting the entry that slot held; its row is copied from the cold pool.
    """

    def __init__(self, N: int, slots: int):
        self.N, self.slots = N, slots
        self.slot_of = [-1] * N
        self.entry_of = [-1] * slots
        self.stamp = [0] * slots

    def update(self, U, t: int, cold=None, hot=None):
        """U: iterable of entry indices (the trigger's fetch set).  Returns the list of
        (entry, slot) moves in entry order, or None when |U| exceeds the pool."""
        assert t >= 1
        U = sorted(set(int(e) for e in U))
        inU = set(U)
        kept = set()
        for e in U:
            s = self.slot_of[e]
            if s >= 0:
                self.stamp[s] = t
                kept.add(s)
        need = [e for e in U if self.slot_of[e] < 0]
        if len(U) > self.slots:
            return None
        cand = sorted((self.stamp[s], s) for s in range(self.slots) if s not in kept)
        taken = sorted(s for _, s in cand[: len(need)])
        moves = []
        for e, s in zip(need, taken):
            old = self.entry_of[s]
            assert old < 0 or old not in inU
            if old >= 0:
                self.slot_of[old] = -1
            self.entry_of[s] = e
            self.slot_of[e] = s
            self.stamp[s] = t
            if cold is not None:
                hot[s] = cold[e]
            moves.append((e, s))
        return moves


# ----------------------------------------------------------------------------- labels


def nucleus(logits, top_p: float) -> np.ndarray:
    """Top-p set of one (layer, query position) ([SUMMARY] §2.2 steps 1-2).

    pi = softmax(x) over the N entries; sort by descending pi (equal pi: lower index
    first); an entry belongs to the set iff the probability mass strictly before it in
    that order is < top_p.  Returns bool [N].
    """
    x = np.asarray(logits, dtype=np.float64)
    e = np.exp(x - x.max())
    pi = e / e.sum()
    order = np.lexsort((np.arange(x.size), -pi))
    before = np.cumsum(pi[order]) - pi[order]
    sel = np.zeros(x.size, dtype=bool)
    sel[order] = before < top_p
    return sel


def vote_labels(logits, top_p: float, theta: int):
    """Cross-layer majority vote ([SUMMARY] §2.2 step 3; [REVIEW] 二 training labels).

    logits [L][P][N].  count[p, s] = number of layers whose nucleus for position p
    contains s; golden = count >= theta.  Returns (golden bool [P][N], count int [P][N]).
    """
    x = np.asarray(logits)
    L, P, N = x.shape
    count = np.zeros((P, N), dtype=np.int64)
    for l in range(L):
        for p in range(P):
            count[p] += nucleus(x[l, p], top_p)
    return count >= theta, count


PROB_EPS = 2.0 ** -20   # probabilities are clamped to [PROB_EPS, 1 - PROB_EPS]


def bce_focal(prob, label, gamma: float, eps: float = PROB_EPS):
    """Mean binary cross-entropy and mean focal loss ([SUMMARY] §2.3 loss; [REVIEW] 二).

    p = clamp(prob, eps, 1 - eps)   (sigmoid scores saturate to exactly 0 or 1 in fp32,
                                     where an unclamped log would be infinite; eps is a
                                     power of two, exact in fp32 and fp64)
    BCE = -mean[y ln p + (1-y) ln(1-p)];
    FL  = -mean[y (1-p)^gamma ln p + (1-y) p^gamma ln(1-p)].
    """
    p = np.clip(np.asarray(prob, dtype=np.float64), eps, 1.0 - eps)
    y = np.asarray(label, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        lp = np.where(y > 0, np.log(p), 0.0)
        lq = np.where(y < 1, np.log1p(-p), 0.0)
    bce = -np.mean(y * lp + (1 - y) * lq)
    fl = -np.mean(y * (1 - p) ** gamma * lp + (1 - y) * p ** gamma * lq)
    return float(bce), float(fl)


# ----------------------------------------------------------------------------- calibration


def bias_for_fraction(z_pre, frac: float) -> float:
    """Bias b putting round(frac * n) of the sample's pre-bias logits at or above 0.

    Midpoint of the two order statistics that straddle the cut, negated.
    """
    z = np.sort(np.asarray(z_pre, dtype=np.float64).ravel())
    n = z.size
    m = int(round(frac * n))
    m = min(max(m, 1), n - 1)
    return float(-(z[n - m - 1] + z[n - m]) / 2.0)
