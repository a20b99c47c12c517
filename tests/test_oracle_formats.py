"""Pins for the oracle's number formats (no GPU).

Each test checks the C oracle against something other than itself: values
worked out by hand (tests/golden), an independent library (numpy float16,
torch bfloat16), or invariants and bounds that follow from the format
definitions.
"""
import numpy as np
import pytest
import torch

from conftest import load_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ------------------------------------------------------------ IEEE 16-bit ---
def test_f16_decode_all_65536_codes_match_numpy(ref):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = codes.view(np.float16).astype(np.float32)
    got = np.array([ref.f16_to_f32(int(h)) for h in codes], np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


def _f32_edge_values():
    vals = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e9, -1e9,
            2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26,
            2.0 ** -26, 1e-8, 1e-30, np.inf, -np.inf,
            1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 1.0 + 2.0 ** -11 + 2.0 ** -20,
            2.0 ** -15 + 2.0 ** -25, 6.1e-5, 3 / 127, 0.5 / 127]
    return np.array(vals, np.float32)


def test_f32_to_f16_rne_matches_numpy(ref):
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, 60000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    # dense coverage of the binary16 range, including subnormals and ties
    y = (rng.standard_normal(40000) * 10.0 ** rng.uniform(-9, 5, 40000)).astype(np.float32)
    x = np.concatenate([x, y, _f32_edge_values()])
    want = x.astype(np.float16).view(np.uint16)
    got = np.array([ref.f32_to_f16(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, want)


def test_f32_to_bf16_rne_matches_torch(ref):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(30000) * 10.0 ** rng.uniform(-30, 30, 30000)).astype(np.float32)
    x = np.concatenate([x, _f32_edge_values()[np.isfinite(_f32_edge_values())],
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([ref.f32_to_bf16(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, want)
    back = np.array([ref.bf16_to_f32(int(h)) for h in got[:2000]], np.float32)
    assert np.array_equal(back, torch.from_numpy(want[:2000].view(np.int16)).view(torch.bfloat16).float().numpy())


# ------------------------------------------------------------------ Q8_0 ---
def test_q8_0_golden_blocks(ref):
    g = load_golden("q8_blocks.json")
    for case in g["weight_blocks"]:
        x = np.array(case["x"], np.float32)[None, :]
        blk = ref.quantize(ref.Q8_0, x)[0]
        assert blk.size == 34
        d = int(blk[0]) | (int(blk[1]) << 8)
        assert d == int(case["d_f16"], 16), case["name"]
        q = blk[2:].view(np.int8).astype(int).tolist()
        assert q == case["q"], case["name"]
        if "dequant" in case:
            xh = ref.dequantize(ref.Q8_0, blk[None, :], 32)[0]
            assert xh.tolist() == [float(v) for v in case["dequant"]], case["name"]


def test_q8_0_invariants_and_round_trip_bound(ref):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 256)) * 10.0 ** rng.uniform(-4, 3, (64, 1))).astype(np.float32)
    x[5, 32:64] = 0.0                       # an all-zero block
    w = ref.quantize(ref.Q8_0, x)
    assert w.shape == (64, 8 * 34)
    blocks = w.reshape(64, 8, 34)
    q = blocks[:, :, 2:].view(np.int8).astype(np.int32)
    d = blocks[:, :, :2].copy().view(np.uint16)[..., 0].view(np.float16).astype(np.float64)
    xb = x.reshape(64, 8, 32).astype(np.float64)
    amax = np.abs(xb).max(-1)
    d32 = (amax.astype(np.float32) / np.float32(127)).astype(np.float64)
    assert np.all(np.abs(q) <= 127)
    nz = amax > 0
    # the element with the largest magnitude maps to |q| = 127
    assert np.all(np.abs(q).max(-1)[nz] == 127)
    assert np.all(q[~nz] == 0) and np.all(d[~nz] == 0)
    # |x - d*q| <= d32/2 + 127*|d - d32|  (rounding of x/d32, then of d32 to fp16)
    err = np.abs(xb - d[..., None] * q)
    bound = 0.5 * d32[..., None] * (1 + 1e-6) + 127 * np.abs(d - d32)[..., None] + 1e-30
    assert np.all(err <= bound)
    # dequantization is the exact product
    xh = ref.dequantize(ref.Q8_0, w, 256).reshape(64, 8, 32)
    assert np.array_equal(xh.astype(np.float64), d[..., None] * q)


# ------------------------------------------------------------ act Q8 -------
def test_act_q8_golden_blocks(ref):
    g = load_golden("q8_blocks.json")
    for case in g["activation_blocks"]:
        xq, xd, xs = ref.quantize_act_q8(np.array(case["x"], np.float32)[None, :])
        assert xq[0].tolist() == case["q"], case["name"]
        assert float(xd[0, 0]) == case["xd"], case["name"]
        assert int(xs[0, 0]) == case["xs"], case["name"]


def test_act_q8_invariants(ref):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((8, 1024)) * 10.0 ** rng.uniform(-6, 4, (8, 1))).astype(np.float32)
    x[3, :32] = 0.0
    x[4, 64:96] = -7.25                      # constant block -> all codes -127
    xq, xd, xs = ref.quantize_act_q8(x)
    assert xq.shape == (8, 1024) and xd.shape == (8, 32) and xs.shape == (8, 32)
    q = xq.reshape(8, 32, 32).astype(np.int64)
    assert np.array_equal(xs, q.sum(-1))
    assert np.all(np.abs(q) <= 127)
    assert np.all(q[4, 2] == -127)
    xb = x.reshape(8, 32, 32).astype(np.float64)
    amax = np.abs(xb).max(-1)
    nz = amax > 0
    assert np.all(np.abs(q).max(-1)[nz] == 127)
    assert xd[3, 0] == 0 and np.all(q[3, 0] == 0)
    # the scale is amax/127 within one fp32 rounding, and each code is within
    # half a step of x/xd
    assert np.all(np.abs(xd[nz] * 127.0 - amax[nz]) <= amax[nz] * 2.0 ** -23)
    ratio = xb[nz] / xd[nz][:, None].astype(np.float64)
    assert np.all(np.abs(ratio - q[nz]) <= 0.5 + 1e-5)


# ------------------------------------------------------------------ Q4_K ---
def test_q4k_scale_field_is_a_bijection(ref):
    rng = np.random.default_rng(5)
    for j in range(8):
        for sc in range(64):
            for m in range(64):
                s = rng.integers(0, 256, 12, dtype=np.uint8)
                others = {}
                for jj in range(8):
                    if jj != j:
                        others[jj] = (int(rng.integers(64)), int(rng.integers(64)))
                        ref.q4k_set_scale_min(s, jj, *others[jj])
                ref.q4k_set_scale_min(s, j, sc, m)
                assert ref.q4k_get_scale_min(s, j) == (sc, m)
                for jj, v in others.items():
                    assert ref.q4k_get_scale_min(s, jj) == v


def _golden_q4k_block():
    g = load_golden("q4_k_block.json")
    blk = np.zeros(144, np.uint8)
    blk[0:2] = np.array([int(g["d_f16"], 16)], np.uint16).view(np.uint8)
    blk[2:4] = np.array([int(g["dmin_f16"], 16)], np.uint16).view(np.uint8)
    blk[4:16] = np.frombuffer(bytes.fromhex(g["scales_hex"]), np.uint8)
    for j in range(8):
        for l in range(32):
            q = (j + l) % 16
            byte = 16 + 32 * (j // 2) + l
            blk[byte] |= (q << 4) if (j & 1) else q
    return g, blk


def test_q4k_golden_block(ref):
    g, blk = _golden_q4k_block()
    for j in range(8):
        assert ref.q4k_get_scale_min(blk[4:16], j) == (g["sc"][j], g["m"][j])
    for k, v in g["qs_bytes_spot"].items():
        assert blk[16 + int(k)] == int(v, 16)
    xh = ref.dequantize(ref.Q4_K, blk[None, :], 256)[0]
    for e in g["expected"]:
        assert xh[32 * e["j"] + e["l"]] == e["x"], e


def test_q4k_quantizer_invariants_and_bound(ref):
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
    x[1, :256] = 0.013                    # constant positive super-block
    x[2, 256:512] = -rng.random(256).astype(np.float32)   # all-negative super-block
    x[3] += 0.05                          # shifted rows (mostly positive)
    w = ref.quantize(ref.Q4_K, x)
    assert w.shape == (16, 2 * 144)
    xh = ref.dequantize(ref.Q4_K, w, 512)
    for r in range(16):
        for sb in range(2):
            blk = w[r, sb * 144:(sb + 1) * 144]
            d = float(blk[0:2].copy().view(np.float16)[0])
            dmin = float(blk[2:4].copy().view(np.float16)[0])
            for j in range(8):
                sc, m = ref.q4k_get_scale_min(blk[4:16], j)
                assert 0 <= sc <= 63 and 0 <= m <= 63
                xs = x[r, sb * 256 + 32 * j: sb * 256 + 32 * j + 32].astype(np.float64)
                got = xh[r, sb * 256 + 32 * j: sb * 256 + 32 * j + 32].astype(np.float64)
                # every reconstructed value lies on the grid -dmin*m + d*sc*[0..15]
                assert np.all(got >= -dmin * m - 1e-12)
                assert np.all(got <= -dmin * m + 15 * d * sc + 1e-12)
                lo = min(0.0, float(xs.min()))
                s_j = (float(xs.max()) - lo) / 15.0
                mm_j = -lo
                # |x - x^| <= d*sc/2 + 15*|d*sc - s_j| + |dmin*m - mm_j|  (+ fp32 slack)
                bound = 0.5 * d * sc + 15 * abs(d * sc - s_j) + abs(dmin * m - mm_j)
                assert np.all(np.abs(xs - got) <= bound * (1 + 1e-5) + 1e-7), (r, sb, j)
    # a constant super-block: s_j = c/15 for all j, so sc = 63, q = 15 and the
    # value is recovered to the precision of the binary16 scale
    assert np.max(np.abs(xh[1, :256] - 0.013)) < 0.013 * 2 ** -9


def test_row_bytes(ref):
    assert ref.row_bytes(ref.Q8_0, 1024) == 1088
    assert ref.row_bytes(ref.Q8_0, 4096) == 4352
    assert ref.row_bytes(ref.Q4_K, 4096) == 2304
    assert ref.row_bytes(ref.Q4_K, 100) == 0
    assert ref.row_bytes(ref.Q8_0, 33) == 0
