"""Plain fp64 CPU oracle of Block-GTQ / TQ-MSE packed-KV decode attention.

TEST INFRASTRUCTURE: used only by the tests, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``. Never on the product path.

Sources (cited by page title and passage):

* [BGTQ] "Block-GTQ: RoPE-Block Rate Allocation for KV-Cache Quantization", abstract.
  Sentence 2: RoPE 2-D frequency blocks carry the key precision. Sentence 3: a blockwise
  logit-error bound motivates a label-free query-key energy score, combined with
  codec-dependent rate penalties. Sentence 4: largest-marginal-gain allocation is
  exactly optimal for the separable integer proxy under equal-cost budgets and
  diminishing gains. Sentence 5: TQ-MSE instantiation, equal-rate blocks grouped, and
  attention over packed caches with no decoded fp16 KV. Sentence 7: "K2V2" = average
  logical bits per K/V coordinate. Sentence 8: no fp16 sink or recent-token buffer.
* [TQ] "TurboQuant: paper algorithm and vLLM engineering implementation" (pipeline
  diagram). Box "input vector x" (a per-head K or V vector); box "random rotation /
  Hadamard" (makes coordinates concentrated and near-independent); box "per-coordinate
  MSE scalar quantisation" (a few centroids approximate the rotated coordinates);
  exercise box 1 (KV-cache memory for a batch/context/kv-head count); vLLM column, box
  "NC" (norm correction: corrects the distortion of the norm by the centroids; the
  "_nc" presets).
* [Philox] Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3"
  (SC'11): the Philox4x32-10 counter-based generator.
* [BoxMuller] Box and Muller (1958): two uniforms to two independent N(0,1) draws.

Readings where the pages leave a step open:
energy score = mean query block energy x mean key block energy (blockwise bound,
Cauchy-Schwarz per block); rate penalty D(b) = Gaussian Lloyd-Max per-coordinate MSE;
block j = coordinates {j, j+64} (rotate-half RoPE); groups ordered by descending rate,
blocks ascending, coordinate j before j+64; dense Haar rotation per group from a
Philox-seeded Gaussian matrix (QR, positive triangular diagonal); y = sqrt(d) R x/|x|;
code = number of thresholds <= y; one fp32 norm per (token, group); V coded as one
128-dim TQ-MSE group at the V rate. Optional layout variants: norm correction (NC) stores
|x| sqrt(d) / |c| instead of |x|, c the vector of the chosen centroids, so the decoded
group vector has the norm of the input; fp16 norms (round to nearest, saturating at the
largest finite fp16) halve the norm bytes. Beyond the pages: a block may get rate 0 (not
stored, decodes to 0, D(0) = 1); rates may be allocated per KV head from that head's term
of the energy score; n_q new query tokens attend causally (token j up to its own
position); decode attention may be split over disjoint token ranges (e.g. one per GPU)
and merged by log-sum-exp.

Parity pins (tests/test_oracle_pins.py): Philox known-answer vectors; Lloyd-Max closed
form at 1 bit, the published per-coordinate MSE figures and Monte Carlo; greedy vs
exhaustive search; rotation orthogonality / QR definition; encode-decode against the
closed-form distortion; attention against the rotated-space identity and its special
cases; NC against the norm it must restore and the mean centroid energy 1 - D(b) of a
Lloyd-Max quantiser; fp16 norms against hand-placed bytes; multi-token attention against
PyTorch's masked scaled_dot_product_attention and causality; rate-0 blocks against
exhaustive allocation, D(0) by Monte Carlo and exact zeros; per-head scores against the
layer score and a constructed scaling; partial attention and its log-sum-exp merge against
attention over the whole token set (random splits, empty parts). No function here is
"parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

HEAD_DIM = 128
FP16_MAX = 65504.0
N_BLOCKS = 64
TILE_TOKENS = 64
CHUNK_TOKENS = 16
_MASK32 = np.uint64(0xFFFFFFFF)

# ----------------------------------------------------------------------------------------
# Counter-based randomness [Philox], [BoxMuller]
# ----------------------------------------------------------------------------------------
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds [Philox, section 3]. ctr: 4 arrays, key: 2 ints/arrays.

    One round multiplies words 0 and 2 by the two Philox constants, takes the 64-bit
    products apart into high and low halves, and mixes the high halves with the other
    two counter words and the round key. The key is bumped by the Weyl constants
    before every round but the first.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK32 for c in ctr)
    k0 = np.asarray(key[0], dtype=np.uint64) & _MASK32
    k1 = np.asarray(key[1], dtype=np.uint64) & _MASK32
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _PHILOX_W0) & _MASK32
            k1 = (k1 + _PHILOX_W1) & _MASK32
        p0 = _PHILOX_M0 * c0
        p1 = _PHILOX_M1 * c2
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & _MASK32,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & _MASK32)
    return c0, c1, c2, c3


def _u53(hi, lo):
    """Uniform in (0,1) from two 32-bit words: 27 high bits of hi, 26 of lo, plus half."""
    a = (hi >> np.uint64(5)).astype(np.float64)
    b = (lo >> np.uint64(6)).astype(np.float64)
    return (a * 67108864.0 + b + 0.5) / 9007199254740992.0


def gaussian_stream(seed: int, stream: int, count: int) -> np.ndarray:
    """Draws 0..count-1 of the N(0,1) stream (seed, stream).

    Philox block n has counter (n mod 2^32, n div 2^32, stream, 0) and key (seed mod 2^32,
    seed div 2^32); its words (0,1) and (2,3) give two uniforms u1, u2 and Box-Muller
    turns them into draws 2n (radius times cosine) and 2n+1 (radius times sine).
    """
    nblk = (count + 1) // 2
    n = np.arange(nblk, dtype=np.uint64)
    x0, x1, x2, x3 = philox4x32_10((n & _MASK32, n >> np.uint64(32), np.full_like(n, stream), np.zeros_like(n)),
                                   (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    u1, u2 = _u53(x0, x1), _u53(x2, x3)
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * nblk)
    out[0::2] = r * np.cos(2.0 * math.pi * u2)
    out[1::2] = r * np.sin(2.0 * math.pi * u2)
    return out[:count]


def haar_rotation(seed: int, stream: int, d: int) -> np.ndarray:
    """Seeded random orthogonal d x d matrix [TQ, "random rotation" box].

    A[i, j] = draw i*d + j of the stream; A = Q T with T upper triangular and a positive
    diagonal; the rotation is Q (Haar distributed). numpy's QR returns some sign pattern
    on T's diagonal, fixed here by flipping the matching columns of Q.
    """
    a = gaussian_stream(seed, stream, d * d).reshape(d, d)
    q, t = np.linalg.qr(a)
    sgn = np.sign(np.diag(t))
    sgn[sgn == 0] = 1.0
    return q * sgn[None, :]


# ----------------------------------------------------------------------------------------
# Lloyd-Max scalar quantiser on N(0,1) [TQ, "per-coordinate MSE scalar quantisation" box]
# ----------------------------------------------------------------------------------------
def _phi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi) if math.isfinite(x) else 0.0


def _upper_tail(x):
    return 0.5 * math.erfc(x / math.sqrt(2.0)) if math.isfinite(x) else 0.0


def lloyd_max(bits: int, tol: float = 1e-15, max_iter: int = 200000):
    """MSE-optimal 2^bits-level quantiser for N(0,1): (centroids, thresholds, mse).

    Lloyd's two conditions, iterated to a fixed point: each threshold is the midpoint of
    its neighbouring centroids; each centroid is the conditional mean of its cell,
    E[X | a < X <= b] = (phi(a) - phi(b)) / (P(X > a) - P(X > b)). The density is
    symmetric, so only the positive half (middle threshold 0) is iterated and then
    mirrored. mse = 1 - sum_i P(cell i) c_i^2 (the centroid condition makes the cross
    term vanish).
    """
    if bits < 1 or bits > 8:
        raise ValueError("bits in 1..8")
    n = 1 << (bits - 1)
    t = [0.0] + [3.0 * i / n for i in range(1, n)] + [math.inf]
    mu = [0.0] * n
    for _ in range(max_iter):
        for i in range(n):
            mu[i] = (_phi(t[i]) - _phi(t[i + 1])) / (_upper_tail(t[i]) - _upper_tail(t[i + 1]))
        change = 0.0
        for i in range(1, n):
            nt = 0.5 * (mu[i - 1] + mu[i])
            change = max(change, abs(nt - t[i]))
            t[i] = nt
        if change < tol:
            break
    for i in range(n):
        mu[i] = (_phi(t[i]) - _phi(t[i + 1])) / (_upper_tail(t[i]) - _upper_tail(t[i + 1]))
    cent = np.array([-m for m in reversed(mu)] + mu)
    thr = np.array([-x for x in reversed(t[1:n])] + [0.0] + t[1:n])
    mse = 1.0 - 2.0 * sum((_upper_tail(t[i]) - _upper_tail(t[i + 1])) * mu[i] ** 2 for i in range(n))
    return cent, thr, mse


def lloyd_max_mse_table(max_bits: int = 4) -> dict:
    """D(b) for b = 0..max_bits. D(0) = 1: a block given no bits is not stored and decodes
    to 0, the error of predicting 0 for an N(0,1) coordinate is its variance."""
    return {0: 1.0, **{b: lloyd_max(b)[2] for b in range(1, max_bits + 1)}}


# ----------------------------------------------------------------------------------------
# Energy score and rate allocation [BGTQ sentences 2-4]
# ----------------------------------------------------------------------------------------
def block_energy(q_cal: np.ndarray, k_cal: np.ndarray) -> np.ndarray:
    """Label-free query-key energy per RoPE block [BGTQ sentence 3].

    q_cal [n_q, h_q, 128], k_cal [n_k, h_kv, 128]. Block j holds coordinates j and j+64.
    For KV head h: (mean over calibration queries and the h_q/h_kv query heads of h of
    |q_j|^2) times (mean over calibration keys of |k_j|^2); the layer score sums the KV
    heads. Cauchy-Schwarz per block bounds the logit error q.(k - k_hat) by
    sum_j |q_j| |e_j|, and E|e_j|^2 grows with D(b_j) |k_j|^2, which is this product.
    """
    q = np.asarray(q_cal, dtype=np.float64)
    k = np.asarray(k_cal, dtype=np.float64)
    h_q, h_kv = q.shape[1], k.shape[1]
    g = h_q // h_kv
    qe = q[..., :N_BLOCKS] ** 2 + q[..., N_BLOCKS:] ** 2      # [n, h_q, 64]
    ke = k[..., :N_BLOCKS] ** 2 + k[..., N_BLOCKS:] ** 2      # [n, h_kv, 64]
    s = np.zeros(N_BLOCKS)
    for h in range(h_kv):
        s += qe[:, h * g:(h + 1) * g, :].mean(axis=(0, 1)) * ke[:, h, :].mean(axis=0)
    return s


def block_energy_heads(q_cal: np.ndarray, k_cal: np.ndarray) -> np.ndarray:
    """The energy score of each KV head on its own, [h_kv, 64]: the terms that
    ``block_energy`` sums over KV heads [BGTQ sentence 3], for an allocation per KV head."""
    q = np.asarray(q_cal, dtype=np.float64)
    k = np.asarray(k_cal, dtype=np.float64)
    h_q, h_kv = q.shape[1], k.shape[1]
    g = h_q // h_kv
    out = np.zeros((h_kv, N_BLOCKS))
    for h in range(h_kv):
        qh, kh = q[:, h * g:(h + 1) * g, :], k[:, h, :]
        out[h] = ((qh[..., :N_BLOCKS] ** 2 + qh[..., N_BLOCKS:] ** 2).mean(axis=(0, 1))
                  * (kh[..., :N_BLOCKS] ** 2 + kh[..., N_BLOCKS:] ** 2).mean(axis=0))
    return out


def proxy_objective(score, rates, distortion) -> float:
    """Separable integer proxy sum_j s_j D(b_j) [BGTQ sentence 4]."""
    return float(sum(score[j] * distortion[rates[j]] for j in range(len(rates))))


def greedy_rates(score, distortion, r_min: int, r_max: int, total_bits: int) -> np.ndarray:
    """Largest-marginal-gain allocation [BGTQ sentence 4].

    Every block starts at r_min; each step gives one more bit to the block whose proxy
    drops the most, s_j (D(b_j) - D(b_j + 1)), among blocks still below r_max, until the
    rates sum to total_bits. Ties go to the lowest block index.
    """
    n = len(score)
    if total_bits < n * r_min or total_bits > n * r_max:
        raise ValueError("infeasible budget")
    rates = np.full(n, r_min, dtype=np.int64)
    for _ in range(total_bits - n * r_min):
        best, best_gain = -1, -math.inf
        for j in range(n):
            if rates[j] < r_max:
                gain = score[j] * (distortion[rates[j]] - distortion[rates[j] + 1])
                if gain > best_gain:
                    best, best_gain = j, gain
        rates[best] += 1
    return rates


def brute_force_rates(score, distortion, r_min: int, r_max: int, total_bits: int):
    """Exhaustive minimum of the proxy over every rate vector with the given sum."""
    import itertools
    n = len(score)
    best, arg = math.inf, []
    for r in itertools.product(range(r_min, r_max + 1), repeat=n):
        if sum(r) != total_bits:
            continue
        v = proxy_objective(score, r, distortion)
        tol = 1e-12 * max(1.0, abs(v))
        if not arg or v < best - tol:
            best, arg = v, [r]
        elif abs(v - best) <= tol:
            arg.append(r)
    return best, arg


# ----------------------------------------------------------------------------------------
# Layout: groups, rotations, packed format [BGTQ sentence 5], [TQ]
# ----------------------------------------------------------------------------------------
@dataclass
class Layout:
    k_rates: np.ndarray                  # [64] rate per RoPE block
    v_rate: int
    seed: int
    groups: list                         # [(rate, coords ndarray)] in descending rate order
    k_rot: list                          # R_g, d_g x d_g
    v_rot: np.ndarray                    # 128 x 128
    codebooks: dict                      # rate -> (centroids, thresholds)
    norm_correct: bool = False           # NC: stored norm |x| sqrt(d) / |c| [TQ, box "NC"]
    norm_fp16: bool = False              # norms stored as fp16 instead of fp32

    @property
    def norm_bytes(self):
        return 2 if self.norm_fp16 else 4

    @property
    def n_kgroups(self):
        return len(self.groups)

    @property
    def k_bits(self):                    # bits per token of the K code record
        return int(sum(r * len(c) for r, c in self.groups))

    @property
    def k_record_bytes(self):
        return self.k_bits // 8

    @property
    def v_record_bytes(self):
        return HEAD_DIM * self.v_rate // 8

    @property
    def bytes_per_token(self):
        """Resident bytes per (token, KV head): codes plus one norm (fp32, or fp16) per group."""
        return self.k_record_bytes + self.v_record_bytes + self.norm_bytes * (self.n_kgroups + 1)

    @property
    def tile_bytes(self):
        return TILE_TOKENS * self.bytes_per_token

    def k_quads(self):
        """Quads of the key groups in order: (first packed dim, pairs, rate, byte offset of
        the quad's block inside a tile). A group's packed dims are cut into quads of 4 pairs
        (8 dims); its last quad holds the remaining 1-3 pairs when the group's dim count is
        not a multiple of 8. A quad block holds the codes of its pairs for the tile's 64
        tokens: 64 x 2 pairs x r bits = 16 x pairs x r bytes, so blocks start 16-byte
        aligned and the K area has no padding."""
        out, p, off = [], 0, 0
        for r, coords in self.groups:
            d = len(coords)
            for c0 in range(0, d, 8):
                npairs = min(8, d - c0) // 2
                out.append((p + c0, npairs, r, off))
                off += 16 * npairs * r
            p += d
        return out

    @property
    def n_packed(self):
        """Stored key dimensions (128 minus two per rate-0 block)."""
        return int(sum(len(c) for _, c in self.groups))

    def packed_rates(self):
        return np.concatenate([np.full(len(c), r) for r, c in self.groups])

    def packed_coords(self):
        return np.concatenate([c for _, c in self.groups])


def group_coordinates(k_rates) -> list:
    """Equal-rate blocks form one group [BGTQ sentence 5]; descending rate, blocks ascending,
    coordinate j before j+64 inside block j. Rate-0 blocks are in no group (not stored)."""
    rates = np.asarray(k_rates)
    out = []
    for r in sorted(set(int(x) for x in rates if x > 0), reverse=True):
        blocks = [j for j in range(N_BLOCKS) if rates[j] == r]
        coords = np.array([c for j in blocks for c in (j, j + N_BLOCKS)], dtype=np.int64)
        out.append((r, coords))
    return out


def make_layout(k_rates, v_rate: int, seed: int, norm_correct: bool = False, norm_fp16: bool = False) -> Layout:
    """K record = a whole number of bytes: the 64 block rates (0..4, at least one block
    coded) must sum to a multiple of 4."""
    r = np.asarray(k_rates)
    if (len(r) != N_BLOCKS or (2 * int(np.sum(r))) % 8 or not 1 <= v_rate <= 4 or r.min() < 0 or r.max() > 4
            or r.max() < 1):
        raise ValueError("64 block rates in 0..4, not all 0, summing to a multiple of 4, and a V rate in 1..4")
    groups = group_coordinates(k_rates)
    k_rot = [haar_rotation(seed, r, len(c)) for r, c in groups]
    v_rot = haar_rotation(seed, 0, HEAD_DIM)
    books = {}
    for r in set([r for r, _ in groups] + [v_rate]):
        c, t, _ = lloyd_max(r)
        books[r] = (c, t)
    return Layout(np.asarray(k_rates, dtype=np.int64), int(v_rate), int(seed), groups, k_rot, v_rot, books,
                  bool(norm_correct), bool(norm_fp16))


def cache_bytes(layout: Layout, batch: int, h_kv: int, tokens: int) -> int:
    """Resident bytes of a packed cache [TQ exercise box 1]: per (token, KV head)
    128 b_K/8 + 128 b_V/8 code bytes plus 4 (n_gK + 1) norm bytes (2 (n_gK + 1) with
    fp16 norms); capacity in whole 64-token tiles."""
    tiles = -(-tokens // TILE_TOKENS)
    return batch * h_kv * tiles * layout.tile_bytes


# ----------------------------------------------------------------------------------------
# TQ-MSE encode / decode [TQ pipeline boxes], [BGTQ sentence 5]
# ----------------------------------------------------------------------------------------
def _tq_encode_group(x: np.ndarray, rot: np.ndarray, thresholds: np.ndarray):
    """x [n, d] -> (codes [n, d], norms [n], margin [n, d]).

    |x| is the group norm; the unit vector is rotated and scaled by sqrt(d) so each
    coordinate has unit variance, then each coordinate is compared with the Lloyd-Max
    thresholds: code = number of thresholds <= y (a value on a threshold goes up).
    A zero vector gives y = 0. margin = distance from y to the nearest threshold.
    """
    d = x.shape[1]
    norms = np.sqrt(np.sum(x * x, axis=1))
    y = np.zeros_like(x)
    nz = norms > 0
    y[nz] = math.sqrt(d) * (x[nz] @ rot.T) / norms[nz, None]
    codes = np.searchsorted(thresholds, y, side="right")
    margin = np.min(np.abs(y[..., None] - thresholds[None, None, :]), axis=-1)
    return codes.astype(np.int64), norms, margin


def _norm_correct(norms: np.ndarray, codes: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """Norm correction [TQ, vLLM box "NC"]. The decoded group vector (s / sqrt(d)) R^T c
    has norm s |c| / sqrt(d), and |c|^2 (the energy of the chosen centroids) is not d in
    general: the centroids distort the norm. Storing s = |x| sqrt(d) / |c| gives the
    decoded vector the norm |x| of the input. No Lloyd-Max centroid is 0, so |c| > 0."""
    d = codes.shape[1]
    cn = np.sqrt(np.sum(centroids[codes] ** 2, axis=1))
    return norms * math.sqrt(d) / cn


def encode(layout: Layout, k: np.ndarray, v: np.ndarray) -> dict:
    """k, v [n, 128] (any float; promoted to fp64). Codes are in packed-dimension order.
    Norms are fp64 (rounded to the stored type by ``pack``); with NC they are the
    corrected norms."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kc, kn, km = [], [], []
    for (r, coords), rot in zip(layout.groups, layout.k_rot):
        c, nrm, m = _tq_encode_group(k[:, coords], rot, layout.codebooks[r][1])
        if layout.norm_correct:
            nrm = _norm_correct(nrm, c, layout.codebooks[r][0])
        kc.append(c)
        kn.append(nrm)
        km.append(m)
    vc, vn, vm = _tq_encode_group(v, layout.v_rot, layout.codebooks[layout.v_rate][1])
    if layout.norm_correct:
        vn = _norm_correct(vn, vc, layout.codebooks[layout.v_rate][0])
    return {
        "k_codes": np.concatenate(kc, axis=1), "k_norms": np.stack(kn, axis=1), "k_margin": np.concatenate(km, axis=1),
        "v_codes": vc, "v_norm": vn, "v_margin": vm,
    }


def reconstruct(layout: Layout, k_codes, k_norms, v_codes, v_norm):
    """Decoded k_hat, v_hat [n, 128] in original coordinates (fp64): per group
    x_hat = (|x| / sqrt(d)) R^T c[code], scattered back to the group's coordinates."""
    n = k_codes.shape[0]
    kh = np.zeros((n, HEAD_DIM))
    col = 0
    for gi, ((r, coords), rot) in enumerate(zip(layout.groups, layout.k_rot)):
        d = len(coords)
        cvals = layout.codebooks[r][0][k_codes[:, col:col + d]]
        kh[:, coords] = (np.asarray(k_norms[:, gi], dtype=np.float64) / math.sqrt(d))[:, None] * (cvals @ rot)
        col += d
    cv = layout.codebooks[layout.v_rate][0][v_codes]
    vh = (np.asarray(v_norm, dtype=np.float64) / math.sqrt(HEAD_DIM))[:, None] * (cv @ layout.v_rot)
    return kh, vh


def attention(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray, scale: float) -> np.ndarray:
    """Exact softmax attention of queries q [G, 128] over every cached token (no sink or
    recent-token window [BGTQ sentence 8]). Returns [G, 128]; an empty cache gives 0."""
    q = np.asarray(q, dtype=np.float64)
    if k_hat.shape[0] == 0:
        return np.zeros_like(q)
    s = (q @ k_hat.T) * scale
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v_hat


def partial_attention(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray, scale: float):
    """Attention of queries q [G, 128] over one part of the cached tokens, kept in the
    form that parts over disjoint token sets can be merged from (the log-sum-exp
    bookkeeping of split attention): s_t = scale q . k_t, m = max_t s_t,
    l = sum_t exp(s_t - m), o = sum_t exp(s_t - m) v_t / l. Returns (m [G], l [G],
    o [G, 128]); an empty part gives m = -inf, l = 0, o = 0."""
    q = np.asarray(q, dtype=np.float64)
    G = q.shape[0]
    if k_hat.shape[0] == 0:
        return np.full(G, -np.inf), np.zeros(G), np.zeros((G, v_hat.shape[1]))
    s = (q @ k_hat.T) * scale
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    return m, l, (e @ v_hat) / l[:, None]


def merge_partials(parts) -> np.ndarray:
    """Merge partial attentions [(m, l, o)] over disjoint token sets into the attention over
    their union: M = max_r m_r, w_r = l_r exp(m_r - M), o = sum_r w_r o_r / sum_r w_r.
    Rows whose parts are all empty give 0."""
    m = np.stack([p[0] for p in parts])          # [R, G]
    l = np.stack([p[1] for p in parts])
    o = np.stack([p[2] for p in parts])          # [R, G, 128]
    M = m.max(axis=0)
    finite = np.isfinite(M)
    w = np.where(np.isfinite(m) & finite[None], l * np.exp(np.where(np.isfinite(m), m, 0.0) - np.where(finite, M, 0.0)[None]), 0.0)
    den = w.sum(axis=0)
    out = np.einsum("rg,rgd->gd", w, o)
    return np.where(den[:, None] > 0, out / np.where(den > 0, den, 1.0)[:, None], 0.0)


# ----------------------------------------------------------------------------------------
# Packed tile format (the byte layout both sides implement)
#
# Tile of 64 tokens = [K area][V area][K norms [group][g][m]][V norms [g][m]], the norm of
# token g + 8 m of the tile (g, m = 0..7) at entry 8 g + m of its row of 64 (so the eight
# tokens a lane's tensor-core rows cover are consecutive), norms fp32 (fp16 in a layout
# with fp16 norms). Both code areas are "fragment-major": they are cut into per-lane
# bit strings, lane l = 4 g + t of a 32-lane warp, holding exactly the codes that lane
# turns into its tensor-core operand registers, so a lane reads its codes with one or two
# aligned loads and no two lanes share a word. Words are little-endian; bit b of a bit
# string is bit b % 8 of its byte b // 8.
#
# K quad with P pairs at rate r (Layout.k_quads): lane i = g P + e (g 0..7 = token row,
# e 0..P-1 = pair) holds, for the eight tokens j = g + 8 m (m 0..7), the codes lo = dim
# 2e and hi = dim 2e + 1 of the quad. Its 16 r-bit string: rate 1: bit m = lo(m), bit
# 8 + m = hi(m); rates 2-4: field m (2 r bits) at bit 2 r m = lo(m) | hi(m) << r. Storage
# inside the quad block: rate 1: halfword i; rate 2: word i; rate 4: 8 bytes at 8 i;
# rate 3: bits 0..31 in word i, bits 32..47 in halfword i after the 8 P words.
#
# V: four 16-token chunks (tokens 16 c .. 16 c + 15), each a block of 256 b bytes. Lane
# l = 4 g + t holds 32 fields n = 4 mt + k (mt 0..7, k 0..3): value dim 16 g + 2 mt +
# (k & 1), tokens lo = 2 t + 8 (k >> 1) and hi = lo + 1 of the chunk. Its 64 b-bit
# string: rate 1: word u (0, 1) has bit f = lo(16 u + f) and bit 16 + f = hi(16 u + f);
# rates 2-4: field n at bit 2 b n = lo | hi << b. Storage: rate 1: 8 bytes at 8 l; rate
# 2: 16 bytes at 16 l; rates 3-4: bits 0..127 at 16 l and the rest (64 or 128 bits) at
# 512 + (8 or 16) l.
# ----------------------------------------------------------------------------------------
def _k_lane_bits(r: int, lo: np.ndarray, hi: np.ndarray) -> np.ndarray:
    """lo, hi [..., 8] codes of slots m = 0..7 -> [..., 16 r] bits of one K lane."""
    out = np.zeros(lo.shape[:-1] + (16 * r,), dtype=np.uint8)
    for m in range(8):
        if r == 1:
            out[..., m] = lo[..., m] & 1
            out[..., 8 + m] = hi[..., m] & 1
        else:
            for b in range(r):
                out[..., 2 * r * m + b] = (lo[..., m] >> b) & 1
                out[..., 2 * r * m + r + b] = (hi[..., m] >> b) & 1
    return out


def _k_lane_codes(r: int, bits: np.ndarray):
    """Inverse of _k_lane_bits: [..., 16 r] bits -> (lo, hi) [..., 8]."""
    bits = bits.astype(np.int64)
    lo = np.zeros(bits.shape[:-1] + (8,), dtype=np.int64)
    hi = np.zeros_like(lo)
    for m in range(8):
        if r == 1:
            lo[..., m] = bits[..., m]
            hi[..., m] = bits[..., 8 + m]
        else:
            for b in range(r):
                lo[..., m] |= bits[..., 2 * r * m + b] << b
                hi[..., m] |= bits[..., 2 * r * m + r + b] << b
    return lo, hi


def _k_lane_spans(r: int, npairs: int, i: int):
    """(lane bit range, block bit range) pieces where K lane i of a quad is stored."""
    if r == 3:
        return [((0, 32), (32 * i, 32 * i + 32)), ((32, 48), (256 * npairs + 16 * i, 256 * npairs + 16 * i + 16))]
    return [((0, 16 * r), (16 * r * i, 16 * r * (i + 1)))]


def _v_fields():
    """For lane l = 4 g + t and field n: (value dim, lo token, hi token) in a V chunk."""
    out = np.zeros((32, 32, 3), dtype=np.int64)
    for lane in range(32):
        g, t = lane // 4, lane % 4
        for n in range(32):
            mt, k = n // 4, n % 4
            lo = 2 * t + 8 * (k >> 1)
            out[lane, n] = (16 * g + 2 * mt + (k & 1), lo, lo + 1)
    return out


def _v_lane_bits(b: int, lo: np.ndarray, hi: np.ndarray) -> np.ndarray:
    """lo, hi [..., 32] codes of fields n = 0..31 -> [..., 64 b] bits of one V lane."""
    out = np.zeros(lo.shape[:-1] + (64 * b,), dtype=np.uint8)
    for n in range(32):
        if b == 1:
            u, f = divmod(n, 16)
            out[..., 32 * u + f] = lo[..., n] & 1
            out[..., 32 * u + 16 + f] = hi[..., n] & 1
        else:
            for i in range(b):
                out[..., 2 * b * n + i] = (lo[..., n] >> i) & 1
                out[..., 2 * b * n + b + i] = (hi[..., n] >> i) & 1
    return out


def _v_lane_codes(b: int, bits: np.ndarray):
    bits = bits.astype(np.int64)
    lo = np.zeros(bits.shape[:-1] + (32,), dtype=np.int64)
    hi = np.zeros_like(lo)
    for n in range(32):
        if b == 1:
            u, f = divmod(n, 16)
            lo[..., n] = bits[..., 32 * u + f]
            hi[..., n] = bits[..., 32 * u + 16 + f]
        else:
            for i in range(b):
                lo[..., n] |= bits[..., 2 * b * n + i] << i
                hi[..., n] |= bits[..., 2 * b * n + b + i] << i
    return lo, hi


def _v_lane_spans(b: int, lane: int):
    """(lane bit range, chunk-block bit range) pieces where V lane l is stored."""
    if b <= 2:
        return [((0, 64 * b), (64 * b * lane, 64 * b * (lane + 1)))]
    rest = 64 * b - 128
    return [((0, 128), (128 * lane, 128 * lane + 128)), ((128, 64 * b), (4096 + rest * lane, 4096 + rest * (lane + 1)))]


def pack(layout: Layout, enc: dict, capacity: int) -> np.ndarray:
    """Bytes of one (batch row, KV head) cache holding tokens 0..n-1 of ``enc`` in the
    fragment-major tile format described above. Unused token slots are 0."""
    n = enc["k_codes"].shape[0]
    if capacity % TILE_TOKENS or n > capacity:
        raise ValueError("capacity must be a multiple of 64 and hold the tokens")
    ntile = capacity // TILE_TOKENS
    out = np.zeros((ntile, layout.tile_bytes), dtype=np.uint8)
    kb, vb, ng, br = layout.k_record_bytes, layout.v_record_bytes, layout.n_kgroups, layout.v_rate
    # K area
    kcodes = np.zeros((ntile * TILE_TOKENS, HEAD_DIM), dtype=np.int64)
    kcodes[:n, :layout.n_packed] = enc["k_codes"]
    kcodes = kcodes.reshape(ntile, 8, 8, HEAD_DIM)          # [tile, m, g, dim]: token g + 8 m
    for p0, npairs, r, off in layout.k_quads():
        blk = np.zeros((ntile, 128 * npairs * r), dtype=np.uint8)
        for g in range(8):
            for e in range(npairs):
                lane = _k_lane_bits(r, kcodes[:, :, g, p0 + 2 * e], kcodes[:, :, g, p0 + 2 * e + 1])
                for (a0, a1), (b0, b1) in _k_lane_spans(r, npairs, g * npairs + e):
                    blk[:, b0:b1] = lane[:, a0:a1]
        out[:, off:off + 16 * npairs * r] = np.packbits(blk, axis=1, bitorder="little")
    # V area
    vcodes = np.zeros((ntile * TILE_TOKENS, HEAD_DIM), dtype=np.int64)
    vcodes[:n] = enc["v_codes"]
    vcodes = vcodes.reshape(ntile, 4, CHUNK_TOKENS, HEAD_DIM)
    fld = _v_fields()
    base = TILE_TOKENS * kb
    for c in range(4):
        blk = np.zeros((ntile, 2048 * br), dtype=np.uint8)
        for lane in range(32):
            dims, lot, hit = fld[lane, :, 0], fld[lane, :, 1], fld[lane, :, 2]
            bits = _v_lane_bits(br, vcodes[:, c, lot, dims], vcodes[:, c, hit, dims])
            for (a0, a1), (b0, b1) in _v_lane_spans(br, lane):
                blk[:, b0:b1] = bits[:, a0:a1]
        out[:, base + 256 * br * c:base + 256 * br * (c + 1)] = np.packbits(blk, axis=1, bitorder="little")
    # norms
    base += TILE_TOKENS * vb
    nb, nt = layout.norm_bytes, norm_dtype(layout)
    kn = np.zeros((ntile * TILE_TOKENS, ng), dtype=nt)
    kn[:n] = stored_norms(layout, enc["k_norms"])
    # [tile, token, group] -> [tile, group, row g, slot m] (token g + 8 m)
    kn = kn.reshape(ntile, 8, 8, ng).transpose(0, 3, 2, 1).reshape(ntile, -1)
    out[:, base:base + nb * TILE_TOKENS * ng] = kn.view(np.uint8).reshape(ntile, -1)
    base += nb * TILE_TOKENS * ng
    vn = np.zeros(ntile * TILE_TOKENS, dtype=nt)
    vn[:n] = stored_norms(layout, enc["v_norm"])
    vn = vn.reshape(ntile, 8, 8).transpose(0, 2, 1).reshape(ntile, TILE_TOKENS)
    out[:, base:base + nb * TILE_TOKENS] = vn.view(np.uint8)
    return out.reshape(-1)


def norm_dtype(layout: Layout):
    return np.float16 if layout.norm_fp16 else np.float32


def stored_norms(layout: Layout, norms) -> np.ndarray:
    """fp64 norms rounded to the layout's norm type (round to nearest even); fp16 norms
    above the largest finite fp16 are stored as that value, not as infinity."""
    x = np.asarray(norms, dtype=np.float64)
    if layout.norm_fp16:
        return np.minimum(x, FP16_MAX).astype(np.float16)
    return x.astype(np.float32)


def unpack(layout: Layout, buf: np.ndarray, n: int) -> dict:
    """Inverse of ``pack`` for tokens 0..n-1 (codes, stored norms promoted to fp64)."""
    ntile = len(buf) // layout.tile_bytes
    t = np.asarray(buf, dtype=np.uint8).reshape(ntile, layout.tile_bytes)
    kb, vb, ng, br = layout.k_record_bytes, layout.v_record_bytes, layout.n_kgroups, layout.v_rate
    kc = np.zeros((ntile, 8, 8, HEAD_DIM), dtype=np.int64)
    for p0, npairs, r, off in layout.k_quads():
        blk = np.unpackbits(t[:, off:off + 16 * npairs * r], axis=1, bitorder="little")
        for g in range(8):
            for e in range(npairs):
                lane = np.zeros((ntile, 16 * r), dtype=np.uint8)
                for (a0, a1), (b0, b1) in _k_lane_spans(r, npairs, g * npairs + e):
                    lane[:, a0:a1] = blk[:, b0:b1]
                lo, hi = _k_lane_codes(r, lane)
                kc[:, :, g, p0 + 2 * e] = lo
                kc[:, :, g, p0 + 2 * e + 1] = hi
    kc = kc.reshape(-1, HEAD_DIM)
    vc = np.zeros((ntile, 4, CHUNK_TOKENS, HEAD_DIM), dtype=np.int64)
    fld = _v_fields()
    base = TILE_TOKENS * kb
    for c in range(4):
        blk = np.unpackbits(t[:, base + 256 * br * c:base + 256 * br * (c + 1)], axis=1, bitorder="little")
        for lane in range(32):
            bits = np.zeros((ntile, 64 * br), dtype=np.uint8)
            for (a0, a1), (b0, b1) in _v_lane_spans(br, lane):
                bits[:, a0:a1] = blk[:, b0:b1]
            lo, hi = _v_lane_codes(br, bits)
            dims, lot, hit = fld[lane, :, 0], fld[lane, :, 1], fld[lane, :, 2]
            vc[:, c, lot, dims] = lo
            vc[:, c, hit, dims] = hi
    base += TILE_TOKENS * vb
    nb, nt = layout.norm_bytes, norm_dtype(layout)
    kn = t[:, base:base + nb * TILE_TOKENS * ng].copy().view(nt).reshape(ntile, ng, 8, 8)  # [group][g][m]
    kn = kn.transpose(0, 3, 2, 1).reshape(-1, ng)                                          # token g + 8 m
    base += nb * TILE_TOKENS * ng
    vn = t[:, base:base + nb * TILE_TOKENS].copy().view(nt).reshape(ntile, 8, 8).transpose(0, 2, 1).reshape(-1)
    return {"k_codes": kc[:n, :layout.n_packed], "k_norms": kn[:n].astype(np.float64),
            "v_codes": vc.reshape(-1, HEAD_DIM)[:n], "v_norm": vn[:n].astype(np.float64)}


def boundary_mask(layout: Layout, enc: dict, capacity: int, eps: float = 1e-6):
    """Byte mask (same shape as ``pack``) covering the code bits of every coordinate whose
    rotated value lies within eps of a decision threshold; also returns their count."""
    rates = layout.packed_rates()
    kmask = np.where(enc["k_margin"] < eps, (1 << rates)[None, :] - 1, 0)
    vmask = np.where(enc["v_margin"] < eps, (1 << layout.v_rate) - 1, 0)
    fake = {"k_codes": kmask, "v_codes": vmask,
            "k_norms": np.zeros_like(enc["k_norms"]), "v_norm": np.zeros_like(enc["v_norm"])}
    return pack(layout, fake, capacity), int((enc["k_margin"] < eps).sum() + (enc["v_margin"] < eps).sum())


def decode_attention(layout: Layout, q: np.ndarray, buf: np.ndarray, length: int, scale: float) -> np.ndarray:
    """Attention of the G query heads q [G, 128] of one KV head over its packed cache."""
    u = unpack(layout, buf, length)
    kh, vh = reconstruct(layout, u["k_codes"], u["k_norms"], u["v_codes"], u["v_norm"])
    return attention(q, kh, vh, scale)


def decode_attention_multi(layout: Layout, q: np.ndarray, buf: np.ndarray, length: int, scale: float) -> np.ndarray:
    """Attention of n_q consecutive query tokens q [n_q, G, 128] of one KV head over its
    packed cache of ``length`` tokens, the last n_q of which are the query tokens' own
    keys and values (multi-token decode: speculative verification, a prefill chunk).
    Causal among the new tokens: query j sits at position length - n_q + j and attends to
    tokens 0 .. length - n_q + j [BGTQ sentence 5: attention over the packed cache; the
    causal rule is the one of autoregressive attention]. Returns [n_q, G, 128]."""
    q = np.asarray(q, dtype=np.float64)
    n_q = q.shape[0]
    u = unpack(layout, buf, length)
    kh, vh = reconstruct(layout, u["k_codes"], u["k_norms"], u["v_codes"], u["v_norm"])
    out = np.zeros_like(q)
    for j in range(n_q):
        n = max(0, length - n_q + j + 1)
        out[j] = attention(q[j], kh[:n], vh[:n], scale)
    return out


def decode_scores(layout: Layout, q: np.ndarray, buf: np.ndarray, length: int, scale: float) -> np.ndarray:
    """Logits scale * q . k_hat of the G query heads q [G, 128] against every cached token of
    one KV head's packed cache [BGTQ sentence 5: scores over the packed codes]; [G, length]."""
    u = unpack(layout, buf, length)
    kh, _ = reconstruct(layout, u["k_codes"], u["k_norms"], u["v_codes"], u["v_norm"])
    return (np.asarray(q, dtype=np.float64) @ kh.T) * scale


def logit_mae(layout: Layout, q: np.ndarray, k: np.ndarray, scale: float) -> float:
    """K-only logit error of a layout [BGTQ sentence 6: layer-averaged logit MAE against
    uniform TQ-MSE]: mean over query heads and tokens of |scale q . k_hat - scale q . k|,
    where k_hat is the TQ-MSE reconstruction of the keys k [n, 128] (values unused)."""
    k = np.asarray(k, dtype=np.float64)
    enc = encode(layout, k, np.zeros_like(k))
    kh, _ = reconstruct(layout, enc["k_codes"], stored_norms(layout, enc["k_norms"]), enc["v_codes"], enc["v_norm"])
    q = np.asarray(q, dtype=np.float64)
    return float(np.mean(np.abs((q @ kh.T - q @ k.T) * scale)))
