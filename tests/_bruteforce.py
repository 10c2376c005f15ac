"""A second, independent implementation of the MLA decode step for tiny inputs.

Pure Python loops over lists of floats with the `math` module only (no numpy), used to
cross-check the numpy oracle. It follows the non-absorbed definition: per head, the
content key W_UK,i c_j and value W_UV,i c_j are formed for every cached token, the shared
k^R_j is appended to the key, the rotated q^R to the query, and softmax attention
follows (Transformer-15 DeepSeek-V2 architecture, MHA equations and eqs. 9-11; DeepSeek-V2
walkthrough 2kiu.com/news/6085339 section 2.4 for the decoupled key).

RoPE here is written as a complex product: the pair (x[2m], x[2m+1]) is the complex
number x[2m] + i x[2m+1] multiplied by exp(i * pos * base^(-2m/d_R)).
"""

import cmath
import math


def _rotate(x, pos, base):
    if base == 0:
        return list(x)
    d = len(x)
    y = [0.0] * d
    for m in range(d // 2):
        z = complex(x[2 * m], x[2 * m + 1]) * cmath.exp(1j * pos * base ** (-2.0 * m / d))
        y[2 * m], y[2 * m + 1] = z.real, z.imag
    return y


def _matvec(w, x):
    """w: list of rows; returns [sum_k w[r][k] * x[k] for r]."""
    return [math.fsum(wr[k] * x[k] for k in range(len(x))) for wr in w]


def decode(q_c, q_r, w_uk, w_uv, rows_of, kv_lens, scale, rope_base):
    """q_c[b][i] (d_h), q_r[b][i] (d_R), w_uk[i] / w_uv[i] as d_h rows of d_c,
    rows_of(b) -> list of kv_len[b] cached rows [c (d_c) ; k^R (d_R)].
    Returns out[b][i] (d_h) and lse[b][i]."""
    B, H = len(q_c), len(q_c[0])
    d_c = len(w_uk[0][0])
    out, lse = [], []
    for b in range(B):
        L = kv_lens[b]
        rows = rows_of(b)
        ob, lb = [], []
        for i in range(H):
            if L == 0:
                ob.append([0.0] * len(w_uv[i]))
                lb.append(-math.inf)
                continue
            q = list(q_c[b][i]) + _rotate(q_r[b][i], L - 1, rope_base)
            keys, vals = [], []
            for j in range(L):
                c = rows[j][:d_c]
                keys.append(_matvec(w_uk[i], c) + list(rows[j][d_c:]))
                vals.append(_matvec(w_uv[i], c))
            s = [scale * math.fsum(q[k] * kj[k] for k in range(len(q))) for kj in keys]
            mx = max(s)
            e = [math.exp(v - mx) for v in s]
            z = math.fsum(e)
            ob.append([math.fsum(e[j] / z * vals[j][d] for j in range(L))
                       for d in range(len(vals[0]))])
            lb.append(mx + math.log(z))
        out.append(ob)
        lse.append(lb)
    return out, lse


def cache_row(h, w_dkv, w_kr, gamma, kv_len, rope_base, eps=1e-6):
    """The cache row of a new token, [RMSNorm(W^DKV h) * gamma ; RoPE_{kv_len-1}(W^KR h)]
    (DeepSeek-V2 architecture page eq. 9 and its RMSNorm after the compressed latent;
    DeepSeek-V3 walkthrough section 2.2 for the rotated k^R), with math.fsum for the sums."""
    x = _matvec(w_dkv, h)
    rms = math.sqrt(math.fsum(v * v for v in x) / len(x) + eps)
    c = [v / rms * g for v, g in zip(x, gamma)]
    return c + _rotate(_matvec(w_kr, h), kv_len - 1, rope_base)


def yarn_theta(d, base, s, orig_len, alpha, beta):
    """YaRN pair frequencies, written pair by pair from the method's definition: a pair whose
    wavelength fits into the original context fewer than alpha times is slowed by s, more
    than beta times is kept, and in between the two are blended linearly in that count."""
    out = []
    for m in range(d // 2):
        theta = base ** (-2.0 * m / d)
        fits = orig_len / (2.0 * math.pi / theta)
        if fits <= alpha:
            w = 0.0
        elif fits >= beta:
            w = 1.0
        else:
            w = (fits - alpha) / (beta - alpha)
        out.append(w * theta + (1.0 - w) * theta / s)
    return out


def rotate_with(x, pos, thetas):
    """RoPE as a complex product with the given pair frequencies."""
    y = [0.0] * len(x)
    for m, th in enumerate(thetas):
        z = complex(x[2 * m], x[2 * m + 1]) * cmath.exp(1j * pos * th)
        y[2 * m], y[2 * m + 1] = z.real, z.imag
    return y
