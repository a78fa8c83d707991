"""Pins of the oracle's quantiser, bit planes and record layout.

Each check ties the oracle to something other than itself: a library
routine (torch's bf16 cast), a brute-force search, a closed-form error bound,
or a worked example derived by hand (tests/golden).
"""

import numpy as np
import pytest
import torch

import oracle as O


def _bf16_exact(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).float().numpy()


def _read_golden(path):
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append(line)
    return rows


# --------------------------------------------------------------------- bf16

def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 100000),
        # exact ties: a bf16 value plus half an ulp
        (torch.randn(1000).to(torch.bfloat16).float().numpy().view(np.uint32) | np.uint32(0x8000)).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -3e-39, 3.3e38], np.float32),
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = O.bf16_round(x)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))


# ---------------------------------------------------------------- quantiser

@pytest.mark.parametrize("bits", [2, 4])
def test_golden_ramp(bits, golden_dir):
    rows = _read_golden(f"{golden_dir}/quant_ramp.txt")
    table = {}
    for head, codes in zip(rows[0::2], rows[1::2]):
        kv = dict(item.split("=") for item in head.split())
        table[int(kv["bits"])] = (float(kv["scale"]), float(kv["min"]),
                                  [int(c) for c in codes.split("=")[1].split()])
    scale, mn, codes = table[bits]
    x = np.arange(32, dtype=np.float32)
    c, s, m = O.quantize_group(x, bits)
    assert float(s) == scale and float(m) == mn
    assert c.tolist() == codes


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_are_nearest_level_brute_force(bits):
    rng = np.random.default_rng(1)
    x = _bf16_exact(rng, (400, 32), 3.0)
    c, s, m = O.quantize_group(x, bits)
    levels = np.arange(2 ** bits, dtype=np.float64)
    recon = m[:, None, None].astype(np.float64) + s[:, None, None].astype(np.float64) * levels
    dist = np.abs(x[..., None].astype(np.float64) - recon)          # [g, 32, levels]
    best = dist.min(axis=-1)
    chosen = np.take_along_axis(dist, c[..., None].astype(np.int64), axis=-1)[..., 0]
    # fp32 division may move a value sitting within an ulp of a half step
    assert np.all(chosen <= best + 1e-6 * np.abs(s)[:, None] + 1e-30)


@pytest.mark.parametrize("bits", [2, 4])
def test_scale_is_nearest_bf16_and_min_exact(bits):
    rng = np.random.default_rng(2)
    x = _bf16_exact(rng, (500, 32), 2.0)
    c, s, m = O.quantize_group(x, bits)
    np.testing.assert_array_equal(m, x.min(axis=1))
    exact = (x.max(axis=1).astype(np.float64) - m) / (2 ** bits - 1)
    bits_s = s.view(np.uint32)
    assert np.all((bits_s & 0xFFFF) == 0)
    up = (bits_s + np.uint32(0x10000)).view(np.float32).astype(np.float64)
    down = (bits_s - np.uint32(0x10000)).view(np.float32).astype(np.float64)
    err = np.abs(s - exact)
    assert np.all(err <= np.abs(up - exact) + 1e-12 * exact)
    assert np.all(err <= np.abs(down - exact) + 1e-12 * exact)


@pytest.mark.parametrize("bits", [2, 4])
def test_round_trip_error_bound(bits):
    """|x - xhat| <= max(s/2, top overshoot) (closed form), with the high-plane
    midpoint reconstruction adding at most 2 s for 4-bit values."""
    rng = np.random.default_rng(3)
    x = _bf16_exact(rng, (300, 32), 1.5)
    c, s, m = O.quantize_group(x, bits)
    s64, m64 = s.astype(np.float64), m.astype(np.float64)
    xhat = m64[:, None] + s64[:, None] * c
    top = x.max(axis=1) - (m64 + (2 ** bits - 1) * s64)
    bound = np.maximum(s64 / 2, top) * (1 + 1e-6) + 1e-7 * np.abs(x).max(axis=1)
    assert np.all(np.abs(x - xhat) <= bound[:, None])
    if bits == 4:
        hi = m64[:, None] + s64[:, None] * (4 * (c >> 2) + 1.5)
        assert np.all(np.abs(x - hi) <= bound[:, None] + 2 * s64[:, None])


def test_constant_group_has_zero_scale():
    x = np.full((3, 32), 0.75, np.float32)
    for bits in (2, 4):
        c, s, m = O.quantize_group(x, bits)
        assert np.all(s == 0) and np.all(m == 0.75) and np.all(c == 0)


def test_key_groups_and_residual():
    rng = np.random.default_rng(4)
    k = _bf16_exact(rng, (77, 64))
    qk = O.QuantKeys(k, 4)
    assert qk.codes.shape == (64, 64) and qk.scale.shape == (2, 64)
    np.testing.assert_array_equal(qk.residual, k[64:])
    kh = qk.dequant()
    np.testing.assert_array_equal(kh[64:], k[64:])
    # group g of channel c is quantised from exactly tokens 32g..32g+31
    c, s, m = O.quantize_group(k[32:64, 5], 4)
    np.testing.assert_array_equal(qk.codes[32:64, 5], c)
    assert qk.scale[1, 5] == s and qk.minv[1, 5] == m


def test_value_groups_are_per_token_32_channels():
    rng = np.random.default_rng(5)
    v = _bf16_exact(rng, (9, 128))
    qv = O.QuantValues(v, 2)
    c, s, m = O.quantize_group(v[7, 64:96], 2)
    np.testing.assert_array_equal(qv.codes[7, 64:96], c)
    assert qv.scale[7, 2] == s and qv.minv[7, 2] == m


# ------------------------------------------------------------ planes, layout

def test_golden_plane_packing(golden_dir):
    rows = dict(r.split("=") for r in _read_golden(f"{golden_dir}/plane_pack.txt"))
    codes2 = np.array([[int(v) for v in rows["codes2"].split()]], np.uint8)
    assert O.pack_plane(codes2).tolist() == [[int(v) for v in rows["bytes"].split()]]
    codes4 = np.array([int(v) for v in rows["codes4"].split()], np.uint8)
    assert (codes4 >> 2).tolist() == [int(v) for v in rows["hi"].split()]
    assert (codes4 & 3).tolist() == [int(v) for v in rows["lo"].split()]


def test_plane_pack_against_unpackbits():
    rng = np.random.default_rng(6)
    c = rng.integers(0, 4, size=(10, 128)).astype(np.uint8)
    packed = O.pack_plane(c)
    bits = np.unpackbits(packed[..., None], axis=-1, bitorder="little")   # [10, 32, 8]
    got = (bits[..., 0::2] + 2 * bits[..., 1::2]).reshape(10, 128)
    np.testing.assert_array_equal(got, c)


@pytest.mark.parametrize("d", [64, 128])
def test_record_sizes_per_token(d):
    """Bytes per token of each precision, from the format's definition:
    4-bit = K hi + K lo + V hi + V lo planes (4 * d/4) + key and value meta
    (4 bytes per 32 elements each); 2-bit = two planes + the two metas;
    bf16 = 4 bytes per channel."""
    meta = 2 * 4 * d // 32
    assert O.record_bytes("q4", d) == 16 * (4 * d // 4 + meta)
    assert O.record_bytes("q2", d) == 16 * (2 * d // 4 + meta)
    assert O.record_bytes("bf16", d) == 16 * 4 * d
    if d == 128:
        assert O.record_bytes("q4", d) // 16 == 160
        assert O.record_bytes("q2", d) // 16 == 96
    secs = O.record_sections("q4", d)
    assert [n for n, _, _ in secs] == ["k_hi", "k_lo", "k_meta", "v_hi", "v_meta", "v_lo"]
    assert all(off % 16 == 0 for _, off, _ in secs)


@pytest.mark.parametrize("kind", ["q4", "q2"])
def test_sequence_records_read_back(kind):
    """Read the expected records back with independent byte arithmetic and
    compare with the quantiser's codes, scales and minima."""
    rng = np.random.default_rng(7)
    d, n = 128, 75
    k, v = _bf16_exact(rng, (n, d)), _bf16_exact(rng, (n, d))
    rec, resid = O.sequence_records(kind, k, v)
    bits = O.BITS[kind]
    qk, qv = O.QuantKeys(k, bits), O.QuantValues(v, bits)
    secs = {nm: (off, sz) for nm, off, sz in O.record_sections(kind, d)}
    np.testing.assert_array_equal(resid, k[64:])

    def plane(blk, name):
        off, sz = secs[name]
        return O.unpack_plane(rec[blk, off: off + sz].reshape(16, d // 4), d)

    def column_plane(blk, name):
        # column-major: byte 16 * j + r holds row r's channels 4j .. 4j + 3
        off, sz = secs[name]
        b = rec[blk, off: off + sz]
        out = np.zeros((16, d), dtype=np.uint8)
        for r in range(16):
            for c in range(d):
                out[r, c] = (int(b[16 * (c // 4) + r]) >> (2 * (c % 4))) & 3
        return out

    def meta(blk, name):
        off, sz = secs[name]
        w = rec[blk, off: off + sz].copy().view("<u4")
        s = ((w & 0xFFFF).astype(np.uint32) << 16).view(np.float32)
        m = (w & 0xFFFF0000).astype(np.uint32).view(np.float32)
        return s, m

    for t in range(n):
        blk, r = divmod(t, 16)
        if kind == "q4":
            vc = column_plane(blk, "v_hi")[r] * 4 + plane(blk, "v_lo")[r]
        else:
            vc = column_plane(blk, "v")[r]
        np.testing.assert_array_equal(vc, qv.codes[t])
        s, m = meta(blk, "v_meta")
        np.testing.assert_array_equal(s.reshape(16, d // 32)[r], qv.scale[t])
        np.testing.assert_array_equal(m.reshape(16, d // 32)[r], qv.minv[t])
    for t in range(64):
        blk, r = divmod(t, 16)
        if kind == "q4":
            kc = plane(blk, "k_hi")[r] * 4 + plane(blk, "k_lo")[r]
        else:
            kc = plane(blk, "k")[r]
        np.testing.assert_array_equal(kc, qk.codes[t])
    for g in range(2):
        s0, m0 = meta(2 * g, "k_meta")
        s1, m1 = meta(2 * g + 1, "k_meta")
        np.testing.assert_array_equal(np.concatenate([s0, s1]), qk.scale[g])
        np.testing.assert_array_equal(np.concatenate([m0, m1]), qk.minv[g])
    # key planes of the unfinished group stay untouched (zero)
    if kind == "q4":
        assert not rec[4, secs["k_hi"][0]: secs["k_meta"][0] + secs["k_meta"][1]].any()


def test_bf16_records_are_raw_rows():
    rng = np.random.default_rng(8)
    k, v = _bf16_exact(rng, (20, 64)), _bf16_exact(rng, (20, 64))
    rec, resid = O.sequence_records("bf16", k, v)
    assert resid is None and rec.shape == (2, O.record_bytes("bf16", 64))
    kr = rec[1, : 16 * 128].copy().view("<u2").reshape(16, 64)
    np.testing.assert_array_equal(kr[3], torch.from_numpy(k[19]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_column_major_plane_worked_example():
    """A hand-worked column-major plane: channel c of row t is code
    (t + c) % 4; byte 16 j + t packs channels 4j .. 4j + 3 of row t LSB first,
    i.e. codes (t + 4j) % 4, (t + 4j + 1) % 4, ... = t % 4, (t+1) % 4, ..."""
    d = 8
    codes = np.array([[(t + c) % 4 for c in range(d)] for t in range(16)], dtype=np.uint8)
    b = O.pack_plane_columns(codes)
    assert b.shape == (d // 4 * 16,)
    for j in range(d // 4):
        for t in range(16):
            a = [(t + 4 * j + f) % 4 for f in range(4)]
            assert b[16 * j + t] == a[0] | a[1] << 2 | a[2] << 4 | a[3] << 6
    # row 1 of column 0: codes 1, 2, 3, 0 -> 0b00111001
    assert b[1] == 0x39
