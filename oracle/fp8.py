"""FP8-E4M3 codec and fine-grained block quantisation (test infrastructure).

E4M3 follows the OCP 8-bit floating point format definition (OFP8, "E4M3"):
1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
encodes subnormals (m/8 * 2^-6); there are no infinities and S.1111.111 is
NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.  Encoding here is
round-to-nearest-even with saturation to +-448 ("satfinite").

Quantisation follows [P1] §4.1 (精细量化策略, 在线量化): activations are
scaled per 1x128 tile and weights per 128x128 block, each scale computed
online from the tile's current max-abs.  Reading taken: scale = amax/448 and
its inverse 448/amax, both float32 (IEEE division); code =
E4M3(float32(v * inverse)); dequantised value = code * scale; a tile whose
amax is 0 gets scale 1 and all-zero codes.  The block-scaled GEMM keeps one
float64 partial sum per 128-wide K slice and applies both scales to it, which
is the exact value of sum_k (qa*sa)(qb*sb).

E5M2 (the same OCP definition, "E5M2") is the gradient format: [P3] (the
10100.com article on the V3 report, FP8 paragraph) has the forward pass in
E4M3 and the backward pass in E5M2.  1 sign bit, 5 exponent bits with bias
15, 2 mantissa bits; exponent field 0 encodes subnormals (m/4 * 2^-14);
S.11111.00 is infinity and S.11111.{01,10,11} NaN, so the largest finite
magnitude is 1.75 * 2^15 = 57344.  Readings taken: encoding is
round-to-nearest-even with saturation to +-57344 (like E4M3 here), and a
gradient tile is scaled like an activation tile with 57344 in place of 448.
"""
from __future__ import annotations

import numpy as np


def _e4m3_value(codes) -> np.ndarray:
    """The format's definition: E4M3 bit patterns (uint8) -> float64 values
    (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    E = (c >> 3) & 0xF
    M = c & 0x7
    mag = np.where(E == 0, (M / 8.0) * 2.0 ** -6, (1.0 + M / 8.0) * np.exp2(E - 7.0))
    mag = np.where((E == 15) & (M == 7), np.nan, mag)
    return sign * mag


_E4M3_TABLE = _e4m3_value(np.arange(256, dtype=np.uint8))


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 bit patterns (uint8) -> float64 values (NaN for S.1111.111): the
    entry of each code in the table of all 256 values the definition gives."""
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_all_values() -> np.ndarray:
    """Values of all 256 codes, index = code."""
    return _E4M3_TABLE.copy()


_POS_VALUES = e4m3_all_values()[:127]          # codes 0x00..0x7E: 0 .. 448, increasing


def e4m3_encode(v) -> np.ndarray:
    """float -> E4M3 code, round to nearest (ties to even mantissa),
    saturating finite overflow (infinities included) to +-448; NaN -> 0x7F.
    float32 input is rounded in float32 (every step below is exact there),
    anything else in float64."""
    v = np.asarray(v)
    if v.dtype != np.float32:
        v = v.astype(np.float64)
    a = np.abs(v)
    _, e = np.frexp(a)                         # a = m * 2**e, 0.5 <= m < 1
    step_exp = np.maximum(e - 4, -9)           # 3 mantissa bits; subnormal step 2^-9
    r = np.ldexp(np.rint(np.ldexp(a, -step_exp)), step_exp)
    r = np.fmin(r, 448.0)                      # saturate (NaN is replaced below)
    # the code of r: a subnormal r < 2^-6 is (r / 2^-9); a normal
    # r = (1 + M/8) 2^(E-7) has exponent field E and mantissa M
    mr, er = np.frexp(r)                       # r = mr 2^er, 0.5 <= mr < 1
    code = np.where(r >= 2.0 ** -6, ((er + 6) << 3) | (np.rint(mr * 16) - 8).astype(np.int64),
                    np.rint(r * 512).astype(np.int64)).astype(np.uint8)
    code = np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)
    if np.isnan(v).any():
        code = np.where(np.isnan(v), np.uint8(0x7F), code).astype(np.uint8)
    return code


def e5m2_decode(codes) -> np.ndarray:
    """E5M2 bit patterns (uint8) -> float64 values (+-inf for S.11111.00,
    NaN for S.11111.{01,10,11})."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    E = (c >> 2) & 0x1F
    M = c & 0x3
    mag = np.where(E == 0, (M / 4.0) * 2.0 ** -14, (1.0 + M / 4.0) * np.exp2(E - 15.0))
    mag = np.where(E == 31, np.where(M == 0, np.inf, np.nan), mag)
    return sign * mag


def e5m2_all_values() -> np.ndarray:
    """Values of all 256 E5M2 codes, index = code."""
    return e5m2_decode(np.arange(256, dtype=np.uint8))


_POS_VALUES_E5M2 = e5m2_all_values()[:124]     # codes 0x00..0x7B: 0 .. 57344, increasing


def e5m2_encode(v) -> np.ndarray:
    """float -> E5M2 code, round to nearest (ties to even mantissa),
    saturating overflow (infinities included) to +-57344; NaN -> 0x7F."""
    v = np.asarray(v, dtype=np.float64)
    a = np.nan_to_num(np.abs(v), nan=0.0, posinf=np.inf)
    fin = np.isfinite(a)
    _, e = np.frexp(np.where(fin, a, 0.0))     # a = m * 2**e, 0.5 <= m < 1
    step_exp = np.maximum(e - 3, -16)          # 2 mantissa bits; subnormal step 2^-16
    r = np.ldexp(np.rint(np.ldexp(np.where(fin, a, 0.0), -step_exp)), step_exp)
    r = np.where(fin, np.minimum(r, 57344.0), 57344.0)
    code = np.searchsorted(_POS_VALUES_E5M2, r).astype(np.uint8)
    assert np.all(_POS_VALUES_E5M2[np.minimum(code, 123)] == r)
    code = np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)
    return np.where(np.isnan(v), np.uint8(0x7F), code).astype(np.uint8)


def _quant_tiles(tiles32: np.ndarray, fmax: float = 448.0, encode=None):
    """Quantise tiles [..., n] (float32 values), each with its own online
    scale from its max-abs (scale = amax / fmax).  ``encode`` defaults to
    E4M3.  Returns (codes [..., n], scales [...])."""
    encode = e4m3_encode if encode is None else encode
    amax = np.max(np.abs(tiles32), axis=-1).astype(np.float32)
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    scale = np.where(zero, np.float32(1.0), safe / np.float32(fmax)).astype(np.float32)
    inv = (np.float32(fmax) / safe).astype(np.float32)
    prod = (tiles32 * inv[..., None]).astype(np.float32)
    codes = np.where(zero[..., None], np.uint8(0), encode(prod)).astype(np.uint8)
    return codes, scale


def quant_rows_1x128(a):
    """Per-row, per-128-column quantisation of activations [M, K] (K % 128 == 0).
    Returns (codes uint8 [M, K], scales float32 [M, K/128])."""
    a32 = np.asarray(a, dtype=np.float32)
    M, K = a32.shape
    codes, scales = _quant_tiles(a32.reshape(M, K // 128, 128))
    return codes.reshape(M, K), scales


def quant_rows_1x128_e5m2(g):
    """Per-row, per-128-column E5M2 quantisation of gradients [M, K]
    (K % 128 == 0), scale = amax / 57344.  Returns (codes uint8 [M, K],
    scales float32 [M, K/128])."""
    g32 = np.asarray(g, dtype=np.float32)
    M, K = g32.shape
    codes, scales = _quant_tiles(g32.reshape(M, K // 128, 128), 57344.0, e5m2_encode)
    return codes.reshape(M, K), scales


def quant_blocks_128(w):
    """Per-128x128-block quantisation of a weight matrix [R, C] (both % 128 == 0).
    Returns (codes uint8 [R, C], scales float32 [R/128, C/128])."""
    w32 = np.asarray(w, dtype=np.float32)
    R, C = w32.shape
    blocks = w32.reshape(R // 128, 128, C // 128, 128).transpose(0, 2, 1, 3)
    codes, scales = _quant_tiles(blocks.reshape(R // 128, C // 128, 128 * 128))
    codes = codes.reshape(R // 128, C // 128, 128, 128).transpose(0, 2, 1, 3).reshape(R, C)
    return codes, scales


_DECODE = {"e4m3": e4m3_decode, "e5m2": e5m2_decode}


def fp8_gemm_ref(codes_a, sa, codes_b, sb, a_format: str = "e4m3",
                 b_format: str = "e4m3") -> np.ndarray:
    """out[m, n] = sum_k (qa[m,k] sa[m,k/128]) (qb[n,k] sb[n/128,k/128]) in
    float64, for A [M, K] (1x128 scales) and B [Nn, K] (128x128 scales).
    ``a_format`` / ``b_format`` name each operand's FP8 format ("e4m3", or
    "e5m2" for a gradient operand of the backward pass, [P3])."""
    qa = _DECODE[a_format](codes_a)
    qb = _DECODE[b_format](codes_b)
    M, K = qa.shape
    Nn = qb.shape[0]
    out = np.zeros((M, Nn), dtype=np.float64)
    sbx = np.repeat(np.asarray(sb, np.float64), 128, axis=0)[:Nn]      # [Nn, K/128]
    for kb in range(K // 128):
        part = qa[:, kb * 128:(kb + 1) * 128] @ qb[:, kb * 128:(kb + 1) * 128].T
        out += part * np.asarray(sa, np.float64)[:, kb:kb + 1] * sbx[:, kb][None, :]
    return out


def fp8_swiglu_expert(a, w1, w3, w2, quant: bool = True) -> np.ndarray:
    """One SwiGLU expert with all three GEMMs in block-scaled E4M3 ([P1] §4.1):
    the rows ``a`` (bf16 values) are quantised per 1x128 tile along d, W1, W3
    ([f, d]) and W2 ([d, f]) per 128x128 block; the gate product a W1^T goes
    through silu and multiplies the up product a W3^T; the hidden activation
    h = silu(a W1^T) * (a W3^T) is held in float32 (the accumulation
    precision the pages name) and quantised per 1x128 tile along f (each of
    its rows separately) before W2.  ``quant=False`` skips every quantisation
    and the float32 holding of h: the same steps then give the exact float64
    expert."""
    from .moe import silu
    if not quant:
        a = np.asarray(a, dtype=np.float64)
        h = silu(a @ np.asarray(w1, np.float64).T) * (a @ np.asarray(w3, np.float64).T)
        return h @ np.asarray(w2, np.float64).T
    qa, sa = quant_rows_1x128(a)
    q1, s1 = quant_blocks_128(w1)
    q3, s3 = quant_blocks_128(w3)
    q2, s2 = quant_blocks_128(w2)
    h = silu(fp8_gemm_ref(qa, sa, q1, s1)) * fp8_gemm_ref(qa, sa, q3, s3)
    qh, sh = quant_rows_1x128(h.astype(np.float32))
    return fp8_gemm_ref(qh, sh, q2, s2)


def fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy, quant: bool = True,
                                  dgu_round: str = "none") -> dict:
    """Input gradient of one SwiGLU expert with the FP8 recipe of the pages:
    E4M3 operands in the forward pass and E5M2 gradients in the backward pass
    ([P3]), each scaled per 1x128 tile (activations, gradients) or 128x128
    block (weights) from its online max-abs ([P1] §4.1).  Steps:
      1. g = a W1^T, u = a W3^T recomputed from the E4M3 operands of the
         forward (a per 1x128 along d, W1 and W3 per block) and rounded to
         bf16 (the values the recompute stores);
      2. dy quantised to E5M2 per 1x128 along d; dh = dy W2 against the
         E4M3 blocks of W2 (its 128x128 blocks read transposed);
      3. dg = dh * u * silu'(g), du = dh * silu(g) from the bf16 g, u;
      4. dg and du quantised to E5M2 per 1x128 along f (each 128-feature tile
         is all gate or all up, as in the packed layout);
      5. da = dg W1 + du W3 against the E4M3 blocks of W1 and W3.
    ``quant=False`` skips every quantisation (float64 operands): the same
    steps then give the exact backward with bf16 g and u.  ``dgu_round=
    'bf16'`` rounds dg and du to bf16 first (where an implementation stores
    them before quantising).
    Returns dict(da [M, d], dh [M, f], dg, du, g, u)."""
    from .moe import round_bf16
    a = np.asarray(a, dtype=np.float64)
    w1, w3, w2 = (np.asarray(w, np.float64) for w in (w1, w3, w2))
    dy = np.asarray(dy, dtype=np.float64)

    def mm(x, w, x_format):
        """x [M, K] (rows scaled per 1x128) times w [N, K]^T (128x128 blocks)."""
        if not quant:
            return x @ w.T
        qx, sx = (quant_rows_1x128(x) if x_format == "e4m3"
                  else quant_rows_1x128_e5m2(x))
        qw, sw = quant_blocks_128(w)
        return fp8_gemm_ref(qx, sx, qw, sw, a_format=x_format, b_format="e4m3")

    g = round_bf16(mm(a, w1, "e4m3"))
    u = round_bf16(mm(a, w3, "e4m3"))
    dh = mm(dy, w2.T, "e5m2")
    sig = 1.0 / (1.0 + np.exp(-g))
    dg = dh * u * sig * (1.0 + g * (1.0 - sig))
    du = dh * g * sig
    if dgu_round == "bf16":
        dg, du = round_bf16(dg), round_bf16(du)
    da = mm(dg, w1.T, "e5m2") + mm(du, w3.T, "e5m2")
    return dict(da=da, dh=dh, dg=dg, du=du, g=g, u=u)


def quant_cols_1x128(m, fmt: str = "e4m3"):
    """Quantise the columns of m [R, C] in 128-row tiles (the contraction
    dimension of a weight-gradient product), zero-padding R up to a multiple
    of 128: each (column, 128-row tile) gets its own max-abs scale.
    Returns (codes uint8 [R, C], scales float32 [ceil(R/128), C])."""
    m32 = np.asarray(m, dtype=np.float32)
    R, C = m32.shape
    Rp = (R + 127) // 128 * 128
    pad = np.zeros((Rp, C), dtype=np.float32)
    pad[:R] = m32
    tiles = pad.reshape(Rp // 128, 128, C).transpose(0, 2, 1)          # [tiles, C, 128]
    if fmt == "e4m3":
        codes, scales = _quant_tiles(tiles)
    else:
        codes, scales = _quant_tiles(tiles, 57344.0, e5m2_encode)
    codes = codes.transpose(0, 2, 1).reshape(Rp, C)[:R]
    return codes, scales


def fp8_weight_grad(dy, h, quant: bool = True) -> np.ndarray:
    """dW = dy^T h for one expert's rows (dy [R, M] the output gradients, h
    [R, N] the layer inputs of that GEMM), with both operands in FP8 along
    the contraction over the R rows: dy in E5M2 and h in E4M3, each column
    scaled per 128-row tile from the expert's first row ([P3] E5M2 in the
    backward pass; [P1] §4.1 1x128 online scaling, the tile laid along the
    contraction as for every other FP8 product here).  Per tile kb:
        dW[i, j] += sdy[kb, i] sh[kb, j] sum_{r in kb} qdy[r, i] qh[r, j]
    in float64.  ``quant=False`` gives dy^T h exactly.  [M, N]."""
    dy = np.asarray(dy, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    if not quant:
        return dy.T @ h
    R = dy.shape[0]
    qd, sd = quant_cols_1x128(dy, "e5m2")
    qh, sh = quant_cols_1x128(h, "e4m3")
    vd, vh = e5m2_decode(qd), e4m3_decode(qh)
    out = np.zeros((dy.shape[1], h.shape[1]), dtype=np.float64)
    for kb in range((R + 127) // 128):
        rs = slice(128 * kb, min(R, 128 * (kb + 1)))
        part = vd[rs].T @ vh[rs]
        out += (part * np.asarray(sd[kb], np.float64)[:, None]
                * np.asarray(sh[kb], np.float64)[None, :])
    return out
