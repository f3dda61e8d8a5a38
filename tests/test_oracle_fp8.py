"""Pins of the oracle's FP8 path and bf16 rounding (CPU only).

* e4m3 encoder: every finite bf16 value, divided by several scales, against a
  nearest-value search over the format's decode table (table built here from
  the OCP FP8 definition: bias 7, 3 mantissa bits, S.1111.111 = NaN, no
  infinities; ties to the even code) and against torch's float8_e4m3fn cast
  wherever torch and saturation agree (|q| <= 448);
* bf16 rounding against torch's float32 -> bfloat16 conversion;
* per-block scales: scale = fp32(amax) / 448 exactly, the block maximum maps
  to +-448, every value decodes back within half an e4m3 step, an all-zero
  block gives scale 0 and zero bytes, -0 keeps its sign bit.
"""
import numpy as np
import pytest
import torch

import oracle


def e4m3_decode_table():
    vals = np.empty(256, np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        E = (c >> 3) & 0xF
        m = c & 7
        if E == 15 and m == 7:
            vals[c] = np.nan
        elif E == 0:
            vals[c] = s * m * 2.0 ** -9
        else:
            vals[c] = s * (1 + m / 8) * 2.0 ** (E - 7)
    return vals


def nearest_e4m3(q):
    """Nearest finite e4m3 code of float32 q, ties to the even code."""
    q = np.asarray(q, np.float32)
    tab = e4m3_decode_table()[:0x7F]          # codes 0x00..0x7E: 0 .. 448, increasing
    a = np.abs(q.astype(np.float64))
    hi = np.clip(np.searchsorted(tab, a, side="left"), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo = np.abs(a - tab[lo])
    d_hi = np.abs(tab[hi] - a)
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = d_lo == d_hi
    pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)
    sign = np.signbit(q).astype(np.uint8) << 7
    return (pick.astype(np.uint8) | sign)


def all_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = oracle.bits_to_f32(bits)
    return f[np.isfinite(f)]


def test_decode_table_landmarks():
    tab = e4m3_decode_table()
    assert tab[0x7E] == 448 and tab[0x08] == 2 ** -6 and tab[0x01] == 2 ** -9
    assert np.isnan(tab[0x7F]) and np.isnan(tab[0xFF])
    fin = tab[:0x7F]
    assert np.all(np.diff(fin) > 0)


@pytest.mark.parametrize("scale", [1.0, 0.001953125, 3.0 / 448, 1e-3, 7.25, 2.0 ** -20, 2.0 ** 20])
def test_e4m3_exhaustive_vs_table(scale):
    x = all_finite_bf16()
    with np.errstate(over="ignore"):
        q = (x / np.float32(scale)).astype(np.float32)
    q = q[np.isfinite(q)]
    got = oracle.e4m3_encode(q)
    want = nearest_e4m3(q)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (q[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e4m3_vs_torch_in_range():
    rng = np.random.default_rng(3)
    q = np.concatenate([
        all_finite_bf16(),
        rng.standard_normal(200000).astype(np.float32) * 100,
        rng.uniform(-448, 448, 200000).astype(np.float32),
        (rng.standard_normal(100000) * 2.0 ** -8).astype(np.float32),
        np.float32([0.0, -0.0, 448.0, -448.0, 2 ** -10, -(2 ** -10), 3 * 2 ** -10]),
    ]).astype(np.float32)
    q = q[np.abs(q) <= 448]
    want = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(q)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (q[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e4m3_saturation_and_signs():
    q = np.float32([448.0, 449.0, 463.99, 464.0, 464.01, 479.0, 480.0, 1e6, np.inf,
                    -464.01, -np.inf, -0.0, -1e-30, 1e-30])
    got = oracle.e4m3_encode(q).tolist()
    assert got == [0x7E] * 9 + [0xFE, 0xFE, 0x80, 0x80, 0x00]


def test_bf16_round_vs_torch():
    rng = np.random.default_rng(5)
    u = np.concatenate([
        rng.integers(0, 2 ** 32, 500000, dtype=np.uint64).astype(np.uint32),
        # exact ties and their neighbours
        (rng.integers(0, 2 ** 16, 20000, dtype=np.uint32) << 16) | 0x8000,
        (rng.integers(0, 2 ** 16, 20000, dtype=np.uint32) << 16) | 0x7FFF,
        (rng.integers(0, 2 ** 16, 20000, dtype=np.uint32) << 16) | 0x8001,
        np.uint32([0x7F7FFFFF, 0xFF7FFFFF, 0x7F800000, 0x00000001, 0x80000001]),
    ]).astype(np.uint32)
    f = u.view(np.float32)
    f = f[~np.isnan(f)]
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round(f)
    np.testing.assert_array_equal(got, want)
    # NaN stays NaN
    nan = oracle.bf16_round(np.float32([np.nan]))
    assert (nan[0] & 0x7F80) == 0x7F80 and (nan[0] & 0x7F) != 0


def _bf16_rows(rng, M, N, scale=1.0):
    x = (rng.standard_normal((M, N)) * scale).astype(np.float32)
    return oracle.bf16_round(x)


def test_fp8_dispatch_scales_and_roundtrip():
    rng = np.random.default_rng(11)
    M, N = 40, 512
    xb = _bf16_rows(rng, M, N)
    xb[3, 128:256] = 0                       # an all-zero block
    xb[4, 0:128] = 0x8000                    # an all -0 block
    xb[5, 7] = 0x8000                        # -0 inside a non-zero block
    xb[6, 256:384] = oracle.bf16_round(np.float32(rng.standard_normal(128) * 1e-30))
    xb[7, :128] = oracle.bf16_round(np.float32(np.full(128, 2.0 ** -130)))  # subnormal bf16
    disp_token = np.arange(M, dtype=np.int32)[::-1].copy()
    q, s = oracle.dispatch(xb, disp_token, fp8=True)
    xf = oracle.bits_to_f32(xb)
    tab = e4m3_decode_table()
    for r in range(M):
        t = disp_token[r]
        for b in range(N // 128):
            blk = xf[t, b * 128:(b + 1) * 128]
            amax = np.float32(np.max(np.abs(blk)))
            qb = q[r, b * 128:(b + 1) * 128]
            if amax == 0:
                assert s[r, b] == 0 and np.all(qb == 0)
                continue
            assert s[r, b] == np.float32(amax / np.float32(448.0))
            j = int(np.argmax(np.abs(blk)))
            assert qb[j] & 0x7F == 0x7E
            dec = tab[qb].astype(np.float64) * np.float64(s[r, b])
            # half an e4m3 step: 2^-4 relative for normals, 2^-10 * s below 2^-6
            err = np.abs(dec - blk.astype(np.float64))
            bound = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * s[r, b]) * (1 + 1e-6)
            assert np.all(err <= bound)
    assert q[M - 1 - 5, 7] == 0x80


def test_bf16_dispatch_identity():
    rng = np.random.default_rng(2)
    M, N, G, E, topk = 33, 64, 12, 5, 3
    idx = np.argsort(rng.random((M, G)), axis=1)[:, :topk].astype(np.int32)
    po = rng.integers(0, E, size=G).astype(np.int32)
    xb = _bf16_rows(rng, M, N)
    for dedup in (False, True):
        lay = oracle.layout(idx, po, G, E, dedup)
        recv = oracle.dispatch(xb, lay["disp_token"], fp8=False)
        if dedup:
            for t in range(M):
                for p in range(E):
                    r = lay["disp_row"][t, p]
                    if r >= 0:
                        np.testing.assert_array_equal(recv[r], xb[t])
        else:
            for t in range(M):
                for k in range(topk):
                    np.testing.assert_array_equal(recv[lay["exp_row"][t, k]], xb[t])
        # sampled rows give the same bytes as the full dispatch
        rows = np.array([0, lay["R_disp"] - 1, lay["R_disp"] // 2], np.int64)
        np.testing.assert_array_equal(oracle.dispatch(xb, lay["disp_token"], False, rows=rows), recv[rows])
