"""Pins for the oracle's E4M3 codec, block quantisation and promoted FP8 GEMM."""
import numpy as np
import torch

from oracle import fp8


def test_decode_closed_forms():
    v = fp8.e4m3_decode(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0xB8, 0x7E, 0xFE, 0x7F, 0x80],
                                 dtype=np.uint8))
    assert v[0] == 0.0
    assert v[1] == 2.0 ** -9            # smallest subnormal
    assert v[2] == 7 * 2.0 ** -9        # largest subnormal
    assert v[3] == 2.0 ** -6            # smallest normal
    assert v[4] == 1.0 and v[5] == -1.0
    assert v[6] == 448.0 and v[7] == -448.0
    assert np.isnan(v[8])
    assert v[9] == 0.0 and np.signbit(v[9])


def test_all_codes_round_trip():
    codes = np.arange(256, dtype=np.uint8)
    vals = fp8.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254
    assert np.array_equal(fp8.e4m3_encode(vals[finite]), codes[finite])


def test_encoder_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * 30, rng.standard_normal(50000) * 1e-2,
                        rng.uniform(-448, 448, 50000)]).astype(np.float32)
    # exact midpoints between neighbouring codes (ties go to the even mantissa)
    v = np.sort(np.unique(fp8.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))))
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = fp8.e4m3_encode(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_saturation():
    got = fp8.e4m3_round(np.array([448.0, 460.0, 1000.0, -1e9, 1e-12]))
    assert got.tolist() == [448.0, 448.0, 448.0, -448.0, 0.0]


def test_act_quant_tiles_and_error_bound():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((8, 512)) * np.array([1, 10, 0.01, 100])[None, :].repeat(128, 1)
         ).astype(np.float32)
    x[3, 128:256] = 0.0                      # an all-zero tile gets scale 1
    q, s = fp8.quant_act_1x128(x)
    assert q.shape == (8, 512) and s.shape == (8, 4)
    assert s[3, 1] == 1.0
    amax = np.abs(x.reshape(8, 4, 128)).max(2)
    nz = amax > 0
    np.testing.assert_array_equal(s[nz], (amax[nz].astype(np.float32) / np.float32(448))[...])
    deq = fp8.e4m3_decode(q).reshape(8, 4, 128) * s[:, :, None]
    xs = x.reshape(8, 4, 128).astype(np.float64)
    # max element of every tile maps to +-448 (up to the fp32 division)
    assert np.all(np.abs(fp8.e4m3_decode(q)).reshape(8, 4, 128).max(2)[nz] == 448.0)
    # relative error of a normal E4M3 value is at most 2^-4; subnormals 2^-10 * s
    err = np.abs(deq - xs)
    bound = np.maximum(np.abs(xs) * 2.0 ** -4, 2.0 ** -10 * s[:, :, None]) * 1.0001
    assert np.all(err <= bound)


def test_weight_quant_blocks():
    rng = np.random.default_rng(2)
    w = rng.standard_normal((256, 384)).astype(np.float32)
    w[128:, 256:] *= 100.0
    q, s = fp8.quant_weight_128x128(w)
    assert s.shape == (2, 3)
    for i in range(2):
        for j in range(3):
            blk = w[128 * i:128 * (i + 1), 128 * j:128 * (j + 1)]
            assert s[i, j] == np.float32(np.abs(blk).max()) / np.float32(448)


def test_promoted_gemm_equals_dequantised_matmul():
    rng = np.random.default_rng(3)
    m, n, k = 5, 256, 384
    aq = rng.integers(0, 256, (m, k)).astype(np.uint8)
    wq = rng.integers(0, 256, (n, k)).astype(np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0x10           # no NaN codes
    wq[(wq & 0x7F) == 0x7F] = 0x22
    sa = rng.uniform(0.1, 2, (m, k // 128)).astype(np.float32)
    sw = rng.uniform(0.1, 2, (n // 128, k // 128)).astype(np.float32)
    got = fp8.fp8_gemm(aq, sa, wq, sw)
    A = fp8.e4m3_decode(aq) * np.repeat(sa.astype(np.float64), 128, axis=1)
    W = fp8.e4m3_decode(wq) * np.repeat(np.repeat(sw.astype(np.float64), 128, axis=0), 128, axis=1)
    np.testing.assert_allclose(got, A @ W.T, rtol=1e-12, atol=1e-9)


def test_exact_inputs_give_exact_product():
    # values that are E4M3 numbers times a power-of-two scale pass through the
    # quantiser unchanged, so the FP8 product equals the fp64 product
    rng = np.random.default_rng(4)
    codes_a = rng.integers(0x08, 0x70, (4, 256)).astype(np.uint8)
    codes_w = rng.integers(0x08, 0x70, (128, 256)).astype(np.uint8)
    for c in (codes_a, codes_w):
        c[:, ::128] = 0x7E                    # every tile holds a 448 -> scale 1
    a = fp8.e4m3_decode(codes_a).astype(np.float32)
    w = fp8.e4m3_decode(codes_w).astype(np.float32)
    qa, sa = fp8.quant_act_1x128(a)
    qw, sw = fp8.quant_weight_128x128(w)
    assert np.all(sa == 1.0) and np.all(sw == 1.0)
    np.testing.assert_array_equal(qa, codes_a)
    np.testing.assert_allclose(fp8.fp8_gemm(qa, sa, qw, sw),
                               a.astype(np.float64) @ w.astype(np.float64).T, rtol=1e-14)


def test_fp8_ffn_close_to_exact_ffn():
    from oracle import moe_oracle as om
    rng = np.random.default_rng(5)
    d, inter = 256, 256
    x = rng.standard_normal((16, d)).astype(np.float32)
    w1, w3 = [(0.02 * rng.standard_normal((inter, d))).astype(np.float32) for _ in range(2)]
    w2 = (0.02 * rng.standard_normal((d, inter))).astype(np.float32)
    xq, xs = fp8.quant_act_1x128(x)
    y8 = fp8.ffn_fp8(xq, xs, fp8.quant_expert(w1, w3, w2))
    y = om.ffn(x, w1, w3, w2)
    # four E4M3 roundings (x, W1/W3, h, W2) of relative size <= 2^-4 each
    assert np.abs(y8 - y).max() <= 0.25 * np.abs(y).max()
    assert np.abs(y8 - y).mean() <= 0.1 * np.abs(y).mean()


def _torch_fp8_dequant(x32: torch.Tensor, rows_per_block: int) -> torch.Tensor:
    """Quantise fp32 x [r, c] to E4M3 with torch's own float8_e4m3fn cast,
    one scale max|x|/448 (fp32; 1 for an all-zero block) per
    rows_per_block x 128 block, and return the dequantised values in fp64."""
    r, c = x32.shape
    b = x32.reshape(r // rows_per_block, rows_per_block, c // 128, 128)
    amax = b.abs().amax(dim=(1, 3))
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    q = (b / s[:, None, :, None]).to(torch.float8_e4m3fn)
    return (q.to(torch.float64) * s.to(torch.float64)[:, None, :, None]).reshape(r, c)


def _torch_ffn_fp8(x32, w1, w3, w2):
    """The FP8 expert FFN restated with torch primitives: dequantised operands
    (the promoted per-block sum equals their fp64 product), h in fp64,
    quantised again per 1x128 tile (from its fp32 value: the scale and the
    quotient are fp32) for the second GEMM."""
    xd = _torch_fp8_dequant(x32, 1)
    w1d, w3d, w2d = (_torch_fp8_dequant(torch.from_numpy(w), 128) for w in (w1, w3, w2))
    a, g = xd @ w1d.T, xd @ w3d.T
    h = torch.nn.functional.silu(a) * g
    return _torch_fp8_dequant(h.to(torch.float32), 1) @ w2d.T


def test_fp8_ffn_and_layer_match_a_torch_restatement():
    """The composition of the FP8 oracle (ffn_fp8, layer_output_fp8) against
    an independent formulation: torch's E4M3 cast instead of the oracle's
    encoder, dequantise-then-multiply instead of the promoted block sum.
    A swapped W1/W3, a transposed scale grid or an extra rounding of h fails
    it (the last is planted in the test below)."""
    from oracle import moe_oracle as om
    rng = np.random.default_rng(11)
    T, d, inter, n_r, K = 24, 256, 384, 4, 2
    u = rng.standard_normal((T, d)).astype(np.float32)
    u[3, :128] = 0.0                               # an all-zero tile: scale 1
    experts = [tuple((0.02 * rng.standard_normal(shape)).astype(np.float32)
                     for shape in ((inter, d), (inter, d), (d, inter))) for _ in range(n_r)]
    shared = tuple((0.02 * rng.standard_normal(shape)).astype(np.float32)
                   for shape in ((inter, d), (inter, d), (d, inter)))
    u32 = torch.from_numpy(u)
    # one expert alone
    uq, us = fp8.quant_act_1x128(u)
    y_or = fp8.ffn_fp8(uq, us, fp8.quant_expert(*experts[1]))
    y_t = _torch_ffn_fp8(u32, *experts[1]).numpy()
    assert np.abs(y_or - y_t).max() <= 1e-12 * np.abs(y_t).max()
    # the layer: routing from the exact oracle, gates, shared expert, residual
    e = (0.5 * rng.standard_normal((n_r, d))).astype(np.float32)
    r = om.route(u, e, None, K, 2.5)
    qexp = [fp8.quant_expert(*w) for w in experts]
    out_or = fp8.layer_output_fp8(u, r.idx, r.gate, lambda i: qexp[i], [fp8.quant_expert(*shared)])
    out_t = u.astype(np.float64) + _torch_ffn_fp8(u32, *shared).numpy()
    for t in range(T):
        for k in range(K):
            i = int(r.idx[t, k])
            out_t[t] += r.gate[t, k] * _torch_ffn_fp8(u32[t:t + 1], *experts[i]).numpy()[0]
    assert np.abs(out_or - out_t).max() <= 1e-12 * np.abs(out_t).max()



def test_planted_bf16_hold_of_h_fails_the_restatement(monkeypatch):
    """The FP8 oracle quantises h from its exact value (the pages give h no
    storage precision). Plant the mistake of holding h in bf16 before its
    1x128 quantisation (an implementation's storage choice) and check that
    the torch restatement above catches it."""
    rng = np.random.default_rng(12)
    d, inter = 256, 384
    x = rng.standard_normal((24, d)).astype(np.float32)
    w = tuple((0.02 * rng.standard_normal(shape)).astype(np.float32)
              for shape in ((inter, d), (inter, d), (d, inter)))
    xq, xs = fp8.quant_act_1x128(x)
    qe = fp8.quant_expert(*w)
    y_t = _torch_ffn_fp8(torch.from_numpy(x), *w).numpy()
    y_or = fp8.ffn_fp8(xq, xs, qe)
    assert np.abs(y_or - y_t).max() <= 1e-12 * np.abs(y_t).max()
    real = fp8.quant_act_1x128

    def quant_of_bf16(v):
        hb = torch.from_numpy(np.asarray(v, dtype=np.float32)).bfloat16().float().numpy()
        return real(hb)

    monkeypatch.setattr(fp8, "quant_act_1x128", quant_of_bf16)
    y_planted = fp8.ffn_fp8(xq, xs, qe)
    assert np.abs(y_planted - y_t).max() > 1e-6 * np.abs(y_t).max()
