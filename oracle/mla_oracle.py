"""fp64 CPU oracle of the DeepSeek-V2 MLA decode step (weight-absorbed and not).

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module. The product (the CUDA library and its Python
binding) never imports it, and this module imports nothing from the product package: the
two share no code. Everything here is plain numpy in float64; a matrix product is the only
library primitive used as a step.

Sources, cited by page title and section:

[V2-walk]  "DeepSeek-V2 paper walkthrough" (2kiu.com/news/6085339)
           §2.1 MHA cache arithmetic and the kv_cache_bytes estimate;
           §2.2 low-rank joint KV compression; §2.3 matrix absorption (displayed equation);
           §2.4 decoupled RoPE; §5.2 position-path check; §6 validation recipe.
[V2-arch]  "Transformer-15: DeepSeek-V2 architecture, MLA, DeepSeekMoE" (zeeklog.com)
           MHA equations (per-head softmax attention, W^O), eqs. 9-11, cache table.
[V2-notes] "DeepSeek-V2" paper notes (process-cxr.github.io ai-library), section
           "Multi-Head Latent Attention": shared k^R, cache = d_c + d_h^R = 4.5 d_h l.
[V3-walk]  "DeepSeek-V3 technical report walkthrough" (2kiu.com/news/6340724)
           §2.2 KV-side forward (only c^KV and k^R are cached); §2.3 absorption, RoPE R_p.

What the decode step computes, for sequence b with L = kv_len[b] cached tokens and
head i (non-absorbed definition, [V2-arch] MHA equations with [V2-arch] eqs. 9-11 and the
decoupled key of [V2-notes] / [V3-walk] §2.3):

    k_j,i = [ W_UK,i c_j ; k^R_j ]            c_j = c^KV_j (d_c), k^R_j shared by all heads
    v_j,i =   W_UV,i c_j
    q_i   = [ q^C_i ; RoPE_{L-1}(q^R_i) ]
    s_j   = scale * q_i . k_j,i               j = 0 .. L-1
    o_i   = sum_j softmax_j(s)_j v_j,i        (d_h)

The absorbed form ([V2-walk] §2.3 displayed equation, [V3-walk] §2.3) reaches the same
o_i through q'_i = W_UK,i^T q^C_i, a latent output sum_j p_j c_j, and W_UV,i last.

Readings where the pages are silent:
  * scale = 1/sqrt(d_h + d_h^R). The pages print only the MHA 1/sqrt(d_h); the MLA
    equations that would fix it are omitted or lost in extraction.
  * RoPE: interleaved pairs (x[2m], x[2m+1]), theta_m = base^(-2m/d_R), angle pos*theta_m,
    0-based positions. base == 0 means "no rotation" (RoPE off).
  * The query of the new token sits at position L-1 and attends to all L cached rows,
    its own included ([V2-arch]: the new token's K/V is appended, then attended). So the
    causal mask has no interior holes, only the end at L.
  * k^R in the cache is already rotated (it is rotated when it is written, [V3-walk]
    §2.2); the decode step reads it as it is.
  * kv_len == 0: the output is 0 and the log-sum-exp is -inf.
  * Several new tokens per sequence (multi-token prediction, speculative decoding; the
    pages' MTP modules, [V3-walk] section 4.1, predict extra tokens that the main model then
    verifies): the T new tokens are the last T of the kv_len cached rows, and token t sees
    rows 0 .. kv_len - T + t (see "several new tokens per sequence" below).
  * YaRN ([V2-arch] pre-training: the context is extended from 4K to 128K with YaRN, applied
    only to the decoupled RoPE part; s = 40, alpha = 1, beta = 32, target length 160K, and the
    length scaling factor sqrt(t) = 0.0707 ln s + 1; [V2-notes] Long-Context Extension repeats
    s, alpha, beta and the 160K target). The pages give only these hyper-parameters; the
    frequencies follow the YaRN method ("NTK-by-parts", Peng et al. 2023): with the original
    context L_0 (the 4K pre-training length) and a pair's wavelength 2 pi / theta_m, the ratio
    r_m = L_0 theta_m / (2 pi) sets a weight g = clip((r_m - alpha) / (beta - alpha), 0, 1) and
    theta'_m = (1 - g) theta_m / s + g theta_m: long wavelengths are interpolated by s, short
    ones kept. The scores are multiplied by t = (0.0707 ln s + 1)^2, which the default softmax
    scale takes in.
  * The cache row of a new token (the step before decode): c^KV = W^DKV h ([V2-arch] eq. 9,
    [V2-walk] §2.2), followed by an RMSNorm ([V2-notes] Architecture: an RMSNorm is added
    after the compressed latent vectors) with a learned scale gamma and eps = 1e-6 by default
    (the pages give no eps); k^R = RoPE(W^KR h) ([V3-walk] §2.2, §2.3), rotated at the new
    token's position, which is L-1 once the token is counted in L.

Cache layouts accepted (the row is [c^KV (d_c) ; k^R (d_R)], 576 values):
  * contiguous: array [B, Lmax, d_c + d_R];
  * paged: array [num_pages, page_size, d_c + d_R] plus page_table[B, max_pages]; token j
    of sequence b sits at page page_table[b, j // page_size], slot j % page_size.
A cache given as uint16 is read as bf16 bit patterns and widened exactly to float64.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np

D_HEAD = 128      # d_h
D_LATENT = 512    # d_c
D_ROPE = 64       # d_h^R


# ---------------------------------------------------------------------------
# cache-size arithmetic  ([V2-walk] §2.1, [V2-arch] cache table, [V2-notes] MLA)
# ---------------------------------------------------------------------------

def mha_cache_elements_per_token(n_heads: int, d_head: int) -> int:
    """Elements an MHA layer caches per token: one key and one value per head."""
    return 2 * n_heads * d_head


def mla_cache_elements_per_token(d_latent: int, d_rope: int) -> int:
    """Elements an MLA layer caches per token: the latent c^KV plus the shared k^R."""
    return d_latent + d_rope


def kv_cache_bytes(seq_len: int, n_layers: int, elems_per_token_per_layer: int,
                   dtype_bytes: int = 2) -> int:
    """Bytes one request's KV cache takes: tokens x layers x elements x element size."""
    return seq_len * n_layers * elems_per_token_per_layer * dtype_bytes


# ---------------------------------------------------------------------------
# input widening and row gathering
# ---------------------------------------------------------------------------

def widen(x) -> np.ndarray:
    """Return x as float64. uint16 input is taken as bf16 bit patterns (exact widening:
    a bf16 is the top 16 bits of an IEEE binary32)."""
    a = np.asarray(x)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def token_rows(cache, b: int, kv_len: int, page_table=None, page_size: int = 0) -> np.ndarray:
    """The kv_len cached rows of sequence b, in token order, as float64 [kv_len, 576]."""
    cache = np.asarray(cache)
    if kv_len == 0:
        return np.zeros((0, cache.shape[-1]), dtype=np.float64)
    if page_table is None or page_size == 0:
        return widen(cache[b, :kv_len, :])
    pt = np.asarray(page_table)
    j = np.arange(kv_len)
    pages = pt[b, j // page_size]
    slots = j % page_size
    return widen(cache[pages, slots, :])


# ---------------------------------------------------------------------------
# RoPE on the decoupled query  ([V2-walk] §2.4, [V3-walk] §2.3; convention: module doc)
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Yarn:
    """YaRN context extension of the decoupled RoPE (module doc): scale factor s, the
    original context L_0, the ramp bounds alpha < beta, and the coefficient of ln s in
    sqrt(t)."""
    factor: float
    original_len: int = 4096
    alpha: float = 1.0
    beta: float = 32.0
    mscale_coef: float = 0.0707


def rope_theta(d_rope: int, base: float, yarn: Optional[Yarn] = None) -> np.ndarray:
    """The d_rope/2 pair frequencies: theta_m = base^(-2m/d_rope), or with YaRN the blend of
    theta_m / s and theta_m weighted by the ramp of r_m = L_0 theta_m / (2 pi)."""
    m = np.arange(d_rope // 2, dtype=np.float64)
    theta = base ** (-2.0 * m / d_rope)
    if yarn is None or yarn.factor <= 1.0:
        return theta
    wavelength = 2.0 * math.pi / theta
    r = yarn.original_len / wavelength
    g = np.clip((r - yarn.alpha) / (yarn.beta - yarn.alpha), 0.0, 1.0)
    return (1.0 - g) * theta / yarn.factor + g * theta


def yarn_score_factor(yarn: Optional[Yarn]) -> float:
    """t with sqrt(t) = coef * ln s + 1 (1 without YaRN): the factor on the scores."""
    if yarn is None or yarn.factor <= 1.0:
        return 1.0
    root = yarn.mscale_coef * math.log(yarn.factor) + 1.0
    return root * root


def rope_angles(pos: int, d_rope: int, base: float, yarn: Optional[Yarn] = None) -> np.ndarray:
    """Angles pos * theta_m for the d_rope/2 pairs (rope_theta)."""
    return float(pos) * rope_theta(d_rope, base, yarn)


def rope_rotate(x, pos: int, base: float, yarn: Optional[Yarn] = None) -> np.ndarray:
    """Rotate each interleaved pair (x[2m], x[2m+1]) of the last axis by pos * theta_m.
    base == 0 leaves x unchanged (RoPE off)."""
    x = widen(x)
    if base == 0:
        return x.copy()
    ang = rope_angles(pos, x.shape[-1], base, yarn)
    c, s = np.cos(ang), np.sin(ang)
    even, odd = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = even * c - odd * s
    y[..., 1::2] = even * s + odd * c
    return y


# ---------------------------------------------------------------------------
# softmax with its log-sum-exp  ([V2-arch] MHA equation: Softmax_j over j = 1..t)
# ---------------------------------------------------------------------------

def softmax_lse(s: np.ndarray, axis: int = 0):
    """Two-pass softmax along `axis`: subtract the max, exponentiate, normalise.
    Returns (p, lse) with lse = log(sum(exp(s))). An empty axis gives lse = -inf."""
    s = np.asarray(s, dtype=np.float64)
    if s.shape[axis] == 0:
        shape = list(s.shape)
        del shape[axis]
        return s.copy(), np.full(shape, -np.inf)
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=axis, keepdims=True)
    p = e / z
    lse = np.squeeze(m + np.log(z), axis=axis)
    return p, lse


# ---------------------------------------------------------------------------
# the cache row of a new token  ([V2-arch] eq. 9, [V2-notes] Architecture, [V3-walk] §2.2)
# ---------------------------------------------------------------------------

def rms_norm(x, gamma, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gamma over the last axis."""
    x, gamma = widen(x), widen(gamma)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma


def cache_rows(hidden, w_dkv, w_kr, gamma, kv_lens, rope_base: float,
               eps: float = 1e-6, yarn: Optional[Yarn] = None) -> np.ndarray:
    """The row each sequence appends for its new token, [c^KV ; k^R] (576 values):
        c^KV = RMSNorm(W^DKV h_b) * gamma,   k^R = RoPE_{kv_len[b]-1}(W^KR h_b).
    hidden [B, d]; w_dkv [d_c, d]; w_kr [d_R, d]; gamma [d_c]. Returns [B, d_c + d_R]."""
    hidden, w_dkv, w_kr = widen(hidden), widen(w_dkv), widen(w_kr)
    kv_lens = np.asarray(kv_lens)
    rows = np.zeros((hidden.shape[0], w_dkv.shape[0] + w_kr.shape[0]))
    for b in range(hidden.shape[0]):
        c = rms_norm(w_dkv @ hidden[b], gamma, eps)
        kr = rope_rotate(w_kr @ hidden[b], int(kv_lens[b]) - 1, rope_base, yarn)
        rows[b] = np.concatenate([c, kr])
    return rows


# ---------------------------------------------------------------------------
# the quantised latent cache (FP8 rows with one power-of-two scale per token)
# ---------------------------------------------------------------------------
# The pages quantise the deployed KV cache to about 6 bits per element on average ([V2-notes]
# Inference cost; [V2-arch] summary) without giving the format. Reading: each cached row of
# 576 values is stored as OCP FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa
# bits; subnormals; no infinities; S.1111.111 is NaN; largest finite 448) and one scale 2^e
# per token, e an integer. The quantiser takes the smallest e with max|row| / 2^e <= 448 and
# rounds row / 2^e to the nearest code, ties to the even code. A power-of-two scale keeps
# the dequantised values exact in bf16 and fp32.

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """The value of one E4M3 code, from the format's definition."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    exp, man = (code >> 3) & 0xF, code & 0x7
    if exp == 0xF and man == 0x7:
        return math.nan
    if exp == 0:
        return sign * man * 2.0 ** -9            # subnormal: (man / 8) * 2^(1 - 7)
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


_E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)])


def e4m3_decode(codes) -> np.ndarray:
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Nearest finite E4M3 code to each value (|x| <= 448), ties to the code with an even last
    bit; found by comparing with every finite code's value."""
    x = np.asarray(x, dtype=np.float64)
    codes = np.array([c for c in range(256) if np.isfinite(_E4M3_TABLE[c])], dtype=np.int64)
    vals = _E4M3_TABLE[codes]
    d = np.abs(x[..., None] - vals)                                 # [..., finite codes]
    best = d.min(axis=-1, keepdims=True)
    tie = d == best
    # among equally near codes prefer an even code, then the one whose value has x's sign
    # (the two zeros, 0x00 and 0x80, are both even: keep +0 for x >= 0 and -0 for x < 0)
    score = tie * 4 + tie * ((codes & 1) == 0) * 2 + tie * (np.signbit(vals) == np.signbit(x)[..., None])
    return codes[np.argmax(score, axis=-1)].astype(np.uint8)


def fp8_row_exponent(row) -> int:
    """Smallest e with max|row| / 2^e <= 448 (0 for an all-zero row)."""
    amax = float(np.max(np.abs(widen(row))))
    if amax == 0.0:
        return 0
    e = math.ceil(math.log2(amax / E4M3_MAX))
    while amax / 2.0 ** e > E4M3_MAX:             # guard against log2 rounding
        e += 1
    while e > -200 and amax / 2.0 ** (e - 1) <= E4M3_MAX:
        e -= 1
    return e


def quantize_rows_fp8(rows):
    """rows [N, 576] -> (codes uint8 [N, 576], exponents int [N])."""
    rows = widen(rows)
    exps = np.array([fp8_row_exponent(r) for r in rows], dtype=np.int64)
    codes = np.stack([e4m3_encode(r / 2.0 ** e) for r, e in zip(rows, exps)])
    return codes, exps


def dequantize_rows_fp8(codes, exps) -> np.ndarray:
    """codes [..., 576] uint8, exps [...] -> rows in float64: 2^e * value(code)."""
    return e4m3_decode(codes) * np.exp2(np.asarray(exps, dtype=np.float64))[..., None]


def quantize_weight_fp8(w, tile: int = 128):
    """A projection weight (an nn.Linear weight [rows, d_c], e.g. W_UK or W_UV as
    [n_h * d_h, d_c]; an [n_h, d_h, d_c] array is taken row by row) as E4M3 codes with one
    power-of-two scale per 1 x `tile` tile of a row ([V3-walk] section 4.4: weights quantised in
    1 x 128 tiles): (codes uint8 [rows, d_c], exponents int [rows, d_c / tile]). Each tile's
    exponent is the smallest e with max|tile| / 2^e <= 448 and its codes the nearest E4M3
    codes of tile / 2^e (quantize_rows_fp8 applied to the tiles)."""
    w = widen(w)
    d_c = w.shape[-1]
    rows = w.reshape(-1, d_c)
    codes, exps = quantize_rows_fp8(rows.reshape(-1, tile))
    return codes.reshape(rows.shape).astype(np.uint8), exps.reshape(rows.shape[0], d_c // tile)


def dequantize_weight_fp8(codes, exps, d_head: int = D_HEAD) -> np.ndarray:
    """The weight in float64 [rows / d_head, d_head, d_c] from its E4M3 codes [rows, d_c] and
    tile exponents [rows, d_c / tile]: W[r, c] = value(code[r, c]) * 2^exp[r, c // tile]."""
    codes = np.asarray(codes, dtype=np.uint8)
    exps = np.asarray(exps, dtype=np.float64)
    rows, d_c = codes.shape
    tile = d_c // exps.shape[1]
    w = e4m3_decode(codes).reshape(rows, d_c // tile, tile) * np.exp2(exps)[:, :, None]
    return w.reshape(rows // d_head, d_head, d_c)


def default_scale(d_head: int = D_HEAD, d_rope: int = D_ROPE, yarn: Optional[Yarn] = None) -> float:
    """1/sqrt(d_h + d_h^R) (the reading of the softmax scale, module doc), times the YaRN
    score factor t when YaRN is on."""
    return yarn_score_factor(yarn) / math.sqrt(d_head + d_rope)


# ---------------------------------------------------------------------------
# the absorbed path, one stage at a time
# ---------------------------------------------------------------------------

def absorb_query(q_c, q_r, w_uk, kv_lens, rope_base: float, yarn: Optional[Yarn] = None) -> np.ndarray:
    """Absorbed query rows [B, n_h, d_c + d_R] in float64.

    q'_{b,i} = W_UK,i^T q^C_{b,i}   ([V2-walk] §2.3 displayed equation; [V3-walk] §2.3)
    followed by RoPE_{L_b - 1}(q^R_{b,i}) in the last d_R slots ([V2-walk] §2.4).
    w_uk is [n_h, d_h, d_c]: W_UK,i maps a latent c (d_c) to the head's content key (d_h).
    """
    q_c, q_r, w_uk = widen(q_c), widen(q_r), widen(w_uk)
    kv_lens = np.asarray(kv_lens)
    B, H, _ = q_c.shape
    d_c = w_uk.shape[2]
    d_r = q_r.shape[2]
    out = np.zeros((B, H, d_c + d_r))
    for b in range(B):
        pos = max(int(kv_lens[b]) - 1, 0)
        for i in range(H):
            out[b, i, :d_c] = w_uk[i].T @ q_c[b, i]
            out[b, i, d_c:] = rope_rotate(q_r[b, i], pos, rope_base, yarn)
    return out


def latent_attention(q_abs, cache, kv_lens, scale: float, page_table=None,
                     page_size: int = 0, d_latent: int = D_LATENT):
    """Attention over the shared latent cache for every (sequence, head).

    s_{i,j} = scale * q'_i . [c_j ; k^R_j], p = softmax_j(s), latent_i = sum_j p_j c_j.
    Returns (latent [B, n_h, d_c], lse [B, n_h]); lse is log sum_j exp(s_{i,j}).
    The score uses the full 576-wide row, the weighted sum only the first d_c values
    ([V2-walk] §2.3: the weighted sum stays in the latent space).
    """
    q_abs = widen(q_abs)
    kv_lens = np.asarray(kv_lens)
    B, H, _ = q_abs.shape
    latent = np.zeros((B, H, d_latent))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        L = int(kv_lens[b])
        if L == 0:
            continue
        rows = token_rows(cache, b, L, page_table, page_size)      # [L, 576]
        s = (rows @ q_abs[b].T) * scale                              # [L, H]
        p, lse[b] = softmax_lse(s, axis=0)
        latent[b] = p.T @ rows[:, :d_latent]
    return latent, lse


def apply_wuv(latent, w_uv) -> np.ndarray:
    """o_{b,i} = W_UV,i latent_{b,i}; w_uv is [n_h, d_h, d_c] ([V2-arch] eq. 11)."""
    latent, w_uv = widen(latent), widen(w_uv)
    B, H, _ = latent.shape
    out = np.zeros((B, H, w_uv.shape[1]))
    for i in range(H):
        out[:, i, :] = latent[:, i, :] @ w_uv[i].T
    return out


# ---------------------------------------------------------------------------
# the non-absorbed definition: plain MHA over materialised keys and values
# ---------------------------------------------------------------------------

def mla_decode_nonabsorbed(q_c, q_r, w_uk, w_uv, cache, kv_lens, scale: float,
                           rope_base: float, page_table=None, page_size: int = 0,
                           pairs=None, yarn: Optional[Yarn] = None) -> np.ndarray:
    """Head outputs o [B, n_h, d_h] by the non-absorbed definition (module doc).

    Per (b, i): k^C_j = W_UK,i c_j and v_j = W_UV,i c_j are materialised for every cached
    token ([V2-arch] eqs. 9-11), the key gets the shared k^R_j appended and the query its
    rotated q^R ([V2-notes] decoupled RoPE), and ordinary softmax attention follows
    ([V2-arch] MHA equation). `pairs` restricts the work to a list of (b, i); the other
    outputs are left at NaN.
    """
    q_c, q_r = widen(q_c), widen(q_r)
    w_uk, w_uv = widen(w_uk), widen(w_uv)
    kv_lens = np.asarray(kv_lens)
    B, H, d_h = q_c.shape
    d_c = w_uk.shape[2]
    out = np.full((B, H, d_h), np.nan)
    if pairs is None:
        pairs = [(b, i) for b in range(B) for i in range(H)]
    by_seq: dict[int, list[int]] = {}
    for b, i in pairs:
        by_seq.setdefault(int(b), []).append(int(i))
    for b, heads in by_seq.items():
        L = int(kv_lens[b])
        if L == 0:
            for i in heads:
                out[b, i] = 0.0
            continue
        rows = token_rows(cache, b, L, page_table, page_size)
        c, k_r = rows[:, :d_c], rows[:, d_c:]
        for i in heads:
            k_content = c @ w_uk[i].T                                   # [L, d_h]
            v = c @ w_uv[i].T                                           # [L, d_h]
            q = np.concatenate([q_c[b, i], rope_rotate(q_r[b, i], L - 1, rope_base, yarn)])
            keys = np.concatenate([k_content, k_r], axis=1)             # [L, d_h + d_R]
            p, _ = softmax_lse((keys @ q) * scale, axis=0)
            out[b, i] = p @ v
    return out


# ---------------------------------------------------------------------------
# several new tokens per sequence (multi-token prediction / speculative decoding)
# ---------------------------------------------------------------------------
# A sequence whose kv_len = L cached rows include T new tokens holds them at positions
# L - T + t, t = 0..T-1. Token t attends to the rows at positions 0 .. L - T + t: itself and
# what came before it, not the new tokens after it (the causal mask of [V2-arch]'s MHA
# equation, Softmax_j over j = 1..t, applied to each new token). A token with no visible row
# (L < T) gets a zero output and a log-sum-exp of -inf; its q^R is rotated at position 0.

def token_visible_rows(kv_len: int, q_len: int, t: int) -> int:
    """Rows that new token t (0-based, of q_len) of a sequence with kv_len rows sees."""
    return max(0, int(kv_len) - int(q_len) + t + 1)


def absorb_query_tokens(q_c, q_r, w_uk, kv_lens, rope_base: float,
                        yarn: Optional[Yarn] = None) -> np.ndarray:
    """q_c [B, T, n_h, d_h], q_r [B, T, n_h, d_R] -> absorbed rows [B, T, n_h, d_c + d_R]:
    W_UK,i^T q^C and q^R rotated at token t's position max(L - T + t, 0)."""
    q_c, q_r, w_uk = widen(q_c), widen(q_r), widen(w_uk)
    kv_lens = np.asarray(kv_lens)
    B, T, H, _ = q_c.shape
    d_c, d_r = w_uk.shape[2], q_r.shape[3]
    out = np.zeros((B, T, H, d_c + d_r))
    for b in range(B):
        for t in range(T):
            pos = max(int(kv_lens[b]) - T + t, 0)
            for i in range(H):
                out[b, t, i, :d_c] = w_uk[i].T @ q_c[b, t, i]
                out[b, t, i, d_c:] = rope_rotate(q_r[b, t, i], pos, rope_base, yarn)
    return out


def latent_attention_tokens(q_abs, cache, kv_lens, scale: float, page_table=None,
                            page_size: int = 0, d_latent: int = D_LATENT):
    """q_abs [B, T, n_h, 576] -> (latent [B, T, n_h, d_c], lse [B, T, n_h]); token t of
    sequence b attends to its first token_visible_rows(L, T, t) rows."""
    q_abs = widen(q_abs)
    kv_lens = np.asarray(kv_lens)
    B, T, H, _ = q_abs.shape
    latent = np.zeros((B, T, H, d_latent))
    lse = np.full((B, T, H), -np.inf)
    for b in range(B):
        L = int(kv_lens[b])
        rows = token_rows(cache, b, L, page_table, page_size) if L > 0 else None
        for t in range(T):
            n = token_visible_rows(L, T, t)
            if n == 0:
                continue
            s = (rows[:n] @ q_abs[b, t].T) * scale                   # [n, H]
            p, lse[b, t] = softmax_lse(s, axis=0)
            latent[b, t] = p.T @ rows[:n, :d_latent]
    return latent, lse


def mla_decode_nonabsorbed_tokens(q_c, q_r, w_uk, w_uv, cache, kv_lens, scale: float,
                                  rope_base: float, page_table=None, page_size: int = 0,
                                  yarn: Optional[Yarn] = None) -> np.ndarray:
    """Head outputs o [B, T, n_h, d_h] by the non-absorbed definition (materialised keys and
    values per head), each new token over its visible rows."""
    q_c, q_r = widen(q_c), widen(q_r)
    w_uk, w_uv = widen(w_uk), widen(w_uv)
    kv_lens = np.asarray(kv_lens)
    B, T, H, d_h = q_c.shape
    d_c = w_uk.shape[2]
    out = np.zeros((B, T, H, d_h))
    for b in range(B):
        L = int(kv_lens[b])
        rows = token_rows(cache, b, L, page_table, page_size) if L > 0 else None
        for t in range(T):
            n = token_visible_rows(L, T, t)
            if n == 0:
                continue
            c, k_r = rows[:n, :d_c], rows[:n, d_c:]
            pos = L - T + t
            for i in range(H):
                keys = np.concatenate([c @ w_uk[i].T, k_r], axis=1)
                q = np.concatenate([q_c[b, t, i], rope_rotate(q_r[b, t, i], pos, rope_base, yarn)])
                p, _ = softmax_lse((keys @ q) * scale, axis=0)
                out[b, t, i] = p @ (c @ w_uv[i].T)
    return out


def mla_decode_absorbed(q_c, q_r, w_uk, w_uv, cache, kv_lens, scale: float,
                        rope_base: float, page_table=None, page_size: int = 0,
                        yarn: Optional[Yarn] = None):
    """The absorbed path in float64: absorb_query -> latent_attention -> apply_wuv.
    Returns (out [B, n_h, d_h], latent [B, n_h, d_c], lse [B, n_h])."""
    d_latent = np.asarray(w_uk).shape[2]
    q_abs = absorb_query(q_c, q_r, w_uk, kv_lens, rope_base, yarn)
    latent, lse = latent_attention(q_abs, cache, kv_lens, scale, page_table, page_size,
                                   d_latent=d_latent)
    return apply_wuv(latent, w_uv), latent, lse
