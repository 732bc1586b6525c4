"""FP8 E4M3 codec, block quantisation and the promoted FP8 GEMM, for the oracle.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.

Sources:
  [V3]   "DeepSeek-V3 technical report" summary (xyznot.com), "Main ideas",
         FP8 mixed-precision bullet: E4M3 for all tensors, tile-wise 1x128
         activation scaling, block-wise 128x128 weight scaling, FP32
         accumulation on CUDA cores every N_c = 128 steps of K.
  [ARCH] "DeepSeek model architecture explained" (deepseekmodel.com),
         block-quantisation pseudocode: scale = max(abs(block)) / 448, where
         448 is the E4M3 maximum; the block is divided by its scale and
         rounded to FP8.

E4M3 itself (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
subnormals, no infinities, S.1111.111 = NaN, largest finite 448) is written
here from that definition.

Readings where the pages are silent or garbled: activations use 1x128 tiles
([V3]; the pseudocode's 128x128 activation blocks are read as garbled); a
tile whose max is 0 gets scale 1; a value is rounded to fp32 before it is
quantised, and the scale and the division x/scale are evaluated in fp32 (the
scales are fp32 numbers), the fp32 quotient rounded to E4M3 to nearest-even,
saturating at +-448; dequantisation multiplies by BOTH the activation and the
weight scale of each 128-wide K block ([V3]; the pseudocode's single scale is
read as garbled); the intermediate h of an expert FFN is quantised from its
exact value (the pages give it no storage precision of its own). All other
arithmetic is fp64.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
BLOCK = 128


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code (uint8 array) as fp64; the NaN codes give NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    man = c & 0x7
    normal = sign * np.ldexp(1.0 + man / 8.0, ex - 7)
    sub = sign * np.ldexp(man / 8.0, -6)
    val = np.where(ex == 0, sub, normal)
    val = np.where((ex == 15) & (man == 7), np.nan, val)
    return val


def _rne(x: np.ndarray) -> np.ndarray:
    """Round to the nearest integer, ties to even (numpy's np.rint)."""
    return np.rint(x)


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value to each fp64 x (ties to even mantissa), saturating
    to +-448. Returned as fp64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, ex = np.frexp(a)                 # a = m * 2^ex, m in [0.5, 1)
    e = np.clip(ex - 1, -6, 8)          # binade of a; below 2^-6 the spacing stays 2^-9
    quantum = np.ldexp(1.0, e - 3)      # 3 mantissa bits
    q = _rne(a / quantum) * quantum
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, x)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code (uint8) of the rounded value of each fp64 x (see e4m3_round)."""
    x = np.asarray(x, dtype=np.float64)
    q = e4m3_round(x)
    a = np.abs(q)
    sign = np.where(np.signbit(q), 0x80, 0)
    _, ex = np.frexp(a)
    e = ex - 1
    is_sub = a < np.ldexp(1.0, -6)
    m_sub = np.rint(a / np.ldexp(1.0, -9)).astype(np.int64)
    E = np.where(is_sub, 0, e + 7)
    M = np.where(is_sub, m_sub,
                 np.rint(np.ldexp(a, -np.where(is_sub, 0, e)) * 8.0 - 8.0).astype(np.int64))
    code = np.where(is_sub, m_sub, (E << 3) | M)
    return (code | sign).astype(np.uint8)


def _scale_fp32(amax: np.ndarray) -> np.ndarray:
    """scale = max|x| / 448 evaluated in fp32; 1 for an all-zero block."""
    a = np.asarray(amax, dtype=np.float32)
    s = a / np.float32(E4M3_MAX)
    return np.where(a == 0, np.float32(1.0), s).astype(np.float32)


def quant_act_1x128(x):
    """Tile-wise activation quantisation ([V3]: 1x128 tiles).

    x [n, k] (k % 128 == 0; rounded to fp32 first, exact for bf16 or fp32
    input) -> (codes uint8 [n,k], scales fp32 [n, k/128]). Each 128-wide tile
    of a row: s = max|x|/448, code = E4M3(x / s)."""
    x32 = np.asarray(x, dtype=np.float32)
    n, k = x32.shape
    assert k % BLOCK == 0
    tiles = x32.reshape(n, k // BLOCK, BLOCK)
    s = _scale_fp32(np.max(np.abs(tiles), axis=2))
    quot = (tiles / s[:, :, None]).astype(np.float32)      # fp32 division
    codes = e4m3_encode(quot.astype(np.float64)).reshape(n, k)
    return codes, s


def quant_weight_128x128(w):
    """Block-wise weight quantisation ([V3]: 128x128 blocks).

    w [r, k] (r, k multiples of 128) -> (codes uint8 [r,k], scales fp32
    [r/128, k/128])."""
    w32 = np.asarray(w, dtype=np.float32)
    r, k = w32.shape
    assert r % BLOCK == 0 and k % BLOCK == 0
    blocks = w32.reshape(r // BLOCK, BLOCK, k // BLOCK, BLOCK)
    s = _scale_fp32(np.max(np.abs(blocks), axis=(1, 3)))
    quot = (blocks / s[:, None, :, None]).astype(np.float32)
    codes = e4m3_encode(quot.astype(np.float64)).reshape(r, k)
    return codes, s


def fp8_gemm(a_codes, a_scales, w_codes, w_scales) -> np.ndarray:
    """Promoted FP8 product ([V3]): for each 128-wide K block kb the product of
    the E4M3 values is formed, then scaled by s_a[m,kb] * s_w[n/128,kb] and
    accumulated; exact in fp64. a [m,k] with scales [m,k/128];
    w [n,k] with scales [n/128,k/128] -> [m,n]."""
    A = e4m3_decode(a_codes)
    W = e4m3_decode(w_codes)
    m, k = A.shape
    n = W.shape[0]
    sa = np.asarray(a_scales, dtype=np.float64)
    sw = np.asarray(w_scales, dtype=np.float64)
    out = np.zeros((m, n))
    for kb in range(k // BLOCK):
        ks = slice(kb * BLOCK, (kb + 1) * BLOCK)
        part = A[:, ks] @ W[:, ks].T
        col_scale = np.repeat(sw[:, kb], BLOCK)[:n]
        out += part * sa[:, kb][:, None] * col_scale[None, :]
    return out


def quant_expert(w1, w3, w2):
    """128x128-block quantisation of one expert's (w1, w3, w2)."""
    return (quant_weight_128x128(_as32(w1)), quant_weight_128x128(_as32(w3)),
            quant_weight_128x128(_as32(w2)))


def _as32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.cpu().numpy()
    return np.asarray(x, dtype=np.float32)


def ffn_fp8(xq, xs, qexpert) -> np.ndarray:
    """SwiGLU expert with FP8 operands: a = x W1^T, g = x W3^T (promoted FP8
    GEMMs), h = silu(a) * g in fp64, quantised per 1x128 tile from that
    exact value, then y = h W2^T (promoted FP8 GEMM)."""
    (w1q, w1s), (w3q, w3s), (w2q, w2s) = qexpert
    a = fp8_gemm(xq, xs, w1q, w1s)
    g = fp8_gemm(xq, xs, w3q, w3s)
    h = a / (1.0 + np.exp(-a)) * g
    hq, hs = quant_act_1x128(h)
    return fp8_gemm(hq, hs, w2q, w2s)


def layer_output_fp8(u, idx, gate, qexpert, qshared, residual: bool = True) -> np.ndarray:
    """h'_t of the FP8 variant: u quantised once per token (1x128), routed and
    shared FFNs through ffn_fp8, combined in fp64 with the gates and the
    residual. `qexpert(i)` returns quant_expert(...) of routed expert i;
    qshared is a list of quantised shared experts."""
    u32 = _as32(u)
    u64 = u32.astype(np.float64)
    uq, us = quant_act_1x128(u32)
    idx = np.asarray(idx, dtype=np.int64)
    gate = np.asarray(gate, dtype=np.float64)
    out = np.zeros_like(u64)
    for i in np.unique(idx):
        t, k = np.nonzero(idx == i)
        y = ffn_fp8(uq[t], us[t], qexpert(int(i)))
        out[t] += gate[t, k][:, None] * y
    for qs in (qshared or []):
        out += ffn_fp8(uq, us, qs)
    if residual:
        out += u64
    return out
