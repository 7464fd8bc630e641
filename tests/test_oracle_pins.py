"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every check here is independent of the oracle's own code path: golden tables
from the public format definitions, hand-worked blocks, an exhaustive sweep
against separately written decision rules, torch's float8 conversion, exact
rational arithmetic, closed forms and invariants.  Source of the method:
"Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent
Half of a Hybrid 27B LLM" (page summary "Background" item 1 for the format;
abstract mechanism (i) for outlier localisation; abstract last sentence and the
news article's "Risks and caveats" for per-module global scales in fused GEMMs).
"""
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_07_b200 import synthetic

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _golden_codes():
    e2m1, e4m3 = {}, {}
    with open(os.path.join(GOLDEN, "element_codes.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            fmt, code, val = line.split()
            (e2m1 if fmt == "e2m1" else e4m3)[int(code, 16)] = float(val)
    return e2m1, e4m3


def _e4m3_table():
    """All 256 E4M3 byte values from torch's float8_e4m3fn (library decode)."""
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def _e2m1_table():
    e2m1, _ = _golden_codes()
    return np.array([e2m1[c] for c in range(16)])


# --------------------------------------------------------------------------- formats
def test_element_code_tables_match_golden(oracle_lib):
    e2m1, e4m3 = _golden_codes()
    for code, val in e2m1.items():
        got = oracle.e2m1_decode(code)
        assert got == val and np.signbit(got) == np.signbit(val), (code, got, val)
    for code, val in e4m3.items():
        got = oracle.e4m3_decode(code)
        assert got == val and np.signbit(got) == np.signbit(val), (code, got, val)
    # the library's float8 decode agrees with the oracle on every finite byte
    t = _e4m3_table()
    for code in range(256):
        if code & 0x7F == 0x7F:
            continue
        assert oracle.e4m3_decode(code) == t[code]


def test_worked_blocks_golden(oracle_lib):
    with open(os.path.join(GOLDEN, "worked_blocks.txt")) as f:
        rows = [l for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for line in rows:
        head, xs, qs = line.split("|")
        name, s_g, sf = head.split()
        x = np.array([[float(v) for v in xs.split()]], np.float32)
        q, s = oracle.quantize(x, np.float32(s_g))
        assert s[0, 0] == int(sf, 16), name
        assert q[0].tobytes().hex() == "".join(qs.split()), name


def test_exhaustive_rounding_against_decision_rules(oracle_lib, tmp_path):
    """Every FP32 in [0, 8] for E2M1; a dense sweep plus every pattern near each
    midpoint for E4M3.  The decision rules are written separately in C."""
    exe = str(tmp_path / "exhaustive")
    odir = os.path.dirname(oracle.build())
    subprocess.run(["gcc", "-O2", "-fopenmp", "-o", exe, os.path.join(HERE, "pins", "exhaustive_rounding.c"),
                    "-L" + odir, "-loracle", "-Wl,-rpath," + odir, "-lm"], check=True)
    vals = _e4m3_table()[:127]
    out = subprocess.run([exe] + [repr(float(v)) for v in vals], check=True,
                         capture_output=True, text=True).stdout.split()
    assert out[0] == "mismatches"
    bad2, bad4, n2, n4 = map(int, (out[1], out[2], out[4], out[5]))
    assert n2 > 2_000_000_000 and n4 > 70_000_000
    assert bad2 == 0 and bad4 == 0


def test_e4m3_matches_torch_float8_in_range(oracle_lib):
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 200_000)),
        rng.uniform(0, 2.0 ** -6, 20_000),                      # subnormal range
        np.array([0.0, 2.0 ** -10, 2.0 ** -9, 448.0, 450.0, 463.9]),
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    np.testing.assert_array_equal(got, want)
    # beyond torch's range the oracle saturates to the largest finite value
    assert set(oracle.e4m3_encode(np.array([464.0, 1e6, 3e38, np.inf], np.float32))) == {0x7E}


def test_e2m1_ties_and_saturation(oracle_lib):
    y = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 1e30, -0.1, -0.0, -5.0001], np.float32)
    want = [0, 2, 2, 4, 4, 6, 6, 7, 7, 8, 8, 15]
    assert list(oracle.e2m1_encode(y)) == want


# --------------------------------------------------------------------------- block scaling
def _inputs(kind, rows=48, k=256, seed=3):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        x = rng.standard_normal((rows, k))
    elif kind == "outlier":
        x = rng.standard_normal((rows, k))
        x[:, rng.choice(k, 3, replace=False)] *= 100.0
    elif kind == "lognormal":
        x = rng.lognormal(0.0, 3.0, (rows, k)) * rng.choice([-1, 1], (rows, k))
    elif kind == "tiny":
        x = rng.standard_normal((rows, k)) * 1e-30
    elif kind == "wide_range":
        x = rng.standard_normal((rows, k)) * np.exp(rng.uniform(-20, 20, (rows, 1)))
    return x.astype(np.float32)


@pytest.mark.parametrize("kind", ["normal", "outlier", "lognormal", "tiny", "wide_range"])
def test_block_scale_is_blockmax_over_six(oracle_lib, kind):
    """The effective block scale e4m3(sb) * s_g is blockmax/6 to within the E4M3
    half-ulp, and sb is the E4M3 value nearest to blockmax / (6 s_g)."""
    x = _inputs(kind)
    rows, k = x.shape
    s_g = oracle.global_scale(x)
    q, sf = oracle.quantize(x, s_g)
    t4 = _e4m3_table()
    dec = t4[sf]
    assert dec.max() <= 448.0
    bm = np.abs(x.astype(np.float64)).reshape(rows, k // 16, 16).max(-1)
    target = bm / (6.0 * float(s_g))           # wanted value of the E4M3 byte
    finite = t4[:127]
    nearest_d = np.abs(target[..., None] - finite[None, None, :]).min(-1)
    got_d = np.abs(target - dec)
    # sb is a nearest E4M3 value (up to the two FP32 roundings of t and bm/t)
    assert np.all(got_d <= nearest_d + 4e-7 * np.maximum(target, 2.0 ** -9))
    normal = (target >= 2.0 ** -6) & (target <= 448.0)
    rel = np.abs(dec - target) / np.where(target > 0, target, 1)
    assert np.all(rel[normal] <= 2.0 ** -4 + 1e-6)
    # the block holding the tensor's amax gets the largest scale, 448
    r, b = np.unravel_index(np.argmax(bm), bm.shape)
    assert sf[r, b] == 0x7E


def test_dequantize_uses_the_format_tables(oracle_lib):
    x = _inputs("outlier", rows=8, k=64)
    s_g = oracle.global_scale(x)
    q, sf = oracle.quantize(x, s_g)
    xh = oracle.dequantize(q, sf, s_g)
    codes = np.stack([q & 15, q >> 4], -1).reshape(q.shape[0], -1)
    want = _e2m1_table()[codes] * _e4m3_table()[np.repeat(sf, 16, axis=1)] * float(s_g)
    np.testing.assert_array_equal(xh, want)
    # every dequantised value divided by its block's scale is on the E2M1 grid
    scale = _e4m3_table()[np.repeat(sf, 16, axis=1)] * float(s_g)
    ratio = np.abs(xh[scale > 0] / scale[scale > 0])
    assert np.isin(ratio, E2M1_GRID).all()


def test_dequantize_is_exact_rational(oracle_lib):
    x = _inputs("lognormal", rows=2, k=32, seed=11)
    s_g = oracle.global_scale(x)
    q, sf = oracle.quantize(x, s_g)
    xh = oracle.dequantize(q, sf, s_g)
    e2, e4 = _e2m1_table(), _e4m3_table()
    for r in range(2):
        for i in range(32):
            code = (q[r, i // 2] >> (4 * (i % 2))) & 15
            exact = Fraction(float(e2[code])) * Fraction(float(e4[sf[r, i // 16]])) * Fraction(float(s_g))
            assert Fraction(float(xh[r, i])) == exact


@pytest.mark.parametrize("kind", ["normal", "outlier", "lognormal", "wide_range"])
def test_codes_are_nearest_grid_points(oracle_lib, kind):
    """Brute force over all 16 codes: each element's code is the grid point of
    its block nearest to x (ties to the even code), except within FP32 rounding
    distance of a midpoint, and the sign bit is the sign of x."""
    x = _inputs(kind, rows=64, k=128, seed=5)
    rows, k = x.shape
    s_g = oracle.global_scale(x)
    q, sf = oracle.quantize(x, s_g)
    codes = np.stack([q & 15, q >> 4], -1).reshape(rows, k)
    se = _e4m3_table()[np.repeat(sf, 16, axis=1)] * float(s_g)
    live = se > 0
    r = x.astype(np.float64)[live] / se[live]
    grid = _e2m1_table()
    d = np.abs(r[:, None] - grid[None, :])
    dmin = d.min(-1)
    chosen = np.abs(r - grid[codes[live]])
    slack = 2.0 ** -21 * np.maximum(np.abs(r), 1.0)
    assert np.all(chosen <= dmin + slack)
    # exact ties (far from FP32 noise) go to the even code
    tie = (np.sum(d <= dmin[:, None] + slack[:, None], -1) > 1)
    assert np.all((codes[live][tie] & 1) == 0) or not tie.any()
    np.testing.assert_array_equal((codes[live] >> 3).astype(bool), np.signbit(x[live]))
    # a block whose effective scale underflows encodes to +0 codes
    assert np.all(codes[~live] == 0)


def test_every_bf16_value_as_block_max(oracle_lib):
    """All finite positive BF16 values placed as the max of a block: the scale
    invariant and the nearest-code property hold for each (s_g fixed)."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32)          # positive finite BF16
    vmax = (bits << 16).view(np.float32)
    rng = np.random.default_rng(1)
    frac = rng.uniform(-1, 1, (vmax.size, 16)).astype(np.float32)
    x = (frac * vmax[:, None]).astype(np.float32)
    x[:, 0] = vmax
    s_g = np.float32(1.0)
    q, sf = oracle.quantize(x, s_g)
    t4 = _e4m3_table()
    target = vmax.astype(np.float64) / 6.0
    dec = t4[sf[:, 0]]
    nearest = np.abs(target[:, None] - t4[None, :127]).min(-1)
    assert np.all(np.abs(dec - target) <= nearest + 1e-7 * np.maximum(target, 2.0 ** -9))
    codes = np.stack([q & 15, q >> 4], -1).reshape(x.shape)
    se = dec[:, None] * np.ones((1, 16))
    live = se > 0
    r = x.astype(np.float64)[live] / se[live]
    d = np.abs(r[:, None] - _e2m1_table()[None, :]).min(-1)
    chosen = np.abs(r - _e2m1_table()[codes[live]])
    assert np.all(chosen <= d + 2.0 ** -21 * np.maximum(np.abs(r), 1.0))
    # blocks whose scale underflows encode to +0 everywhere
    assert np.all(codes[~live.any(1)] == 0)


def test_on_grid_inputs_round_trip(oracle_lib):
    rng = np.random.default_rng(2)
    rows, k = 8, 64
    nb = k // 16
    s_g = np.float32(2.0 ** -5)
    sb = rng.integers(0x20, 0x68, (rows, nb)).astype(np.uint8)   # E4M3 scales 2^-3 .. 2^5 range
    sb[3, 2] = 0x7E                                               # the tensor's largest block scale
    codes = rng.integers(0, 16, (rows, k)).astype(np.uint8)
    for r in range(rows):
        for b in range(nb):
            codes[r, b * 16 + rng.integers(16)] = rng.choice([7, 15])   # a +-6 sets blockmax
    e2, e4 = _e2m1_table(), _e4m3_table()
    x = (e2[codes] * e4[np.repeat(sb, 16, axis=1)] * float(s_g)).astype(np.float32)
    assert oracle.global_scale(x) == s_g
    q, sf = oracle.quantize(x, s_g)
    np.testing.assert_array_equal(sf, sb)
    np.testing.assert_array_equal(np.stack([q & 15, q >> 4], -1).reshape(rows, k), codes)
    xh = oracle.dequantize(q, sf, s_g)
    np.testing.assert_array_equal(xh, x.astype(np.float64))
    q2, sf2 = oracle.quantize(xh.astype(np.float32), s_g)
    np.testing.assert_array_equal(q2, q)
    np.testing.assert_array_equal(sf2, sf)


def test_outlier_stays_in_its_block(oracle_lib):
    """Mechanism (i): with a fixed global scale, a single x50 outlier changes only
    its own 16-element block; a per-tensor-only 4-bit scale instead wipes out
    the other blocks."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((32, 256)).astype(np.float32)
    s_g = np.float32(float(oracle.amax(x)) * 50.0 / 2688.0)      # static, calibrated with headroom
    x2 = x.copy()
    r0, c0 = 17, 133
    x2[r0, c0] *= 50.0
    q1, sf1 = oracle.quantize(x, s_g)
    q2, sf2 = oracle.quantize(x2, s_g)
    b0 = c0 // 16
    diff_sf = np.argwhere(sf1 != sf2)
    assert diff_sf.tolist() == [[r0, b0]]
    dq = np.argwhere(q1 != q2)
    assert len(dq) > 0 and np.all(dq[:, 0] == r0) and np.all(dq[:, 1] // 8 == b0)

    # dynamic scale: the other blocks keep their NVFP4 accuracy ...
    sd = oracle.global_scale(x2)
    qd, sfd = oracle.quantize(x2, sd)
    xh = oracle.dequantize(qd, sfd, sd)
    mask = np.ones_like(x2, bool)
    mask[r0, b0 * 16:(b0 + 1) * 16] = False
    err_nvfp4 = np.linalg.norm((xh - x2)[mask]) / np.linalg.norm(x2[mask])
    # ... while a per-tensor-only E2M1 scale (amax/6, no block scales) crushes them
    per_tensor = float(oracle.amax(x2)) / 6.0
    codes = oracle.e2m1_encode((x2 / per_tensor).astype(np.float32)).reshape(x2.shape)
    xt = _e2m1_table()[codes] * per_tensor
    err_tensor = np.linalg.norm((xt - x2)[mask]) / np.linalg.norm(x2[mask])
    assert err_nvfp4 < 0.15
    assert err_tensor > 0.9


# --------------------------------------------------------------------------- GEMM
def test_gemm_matches_exact_rational_sums(oracle_lib):
    rng = np.random.default_rng(8)
    m, n, k = 3, 5, 32
    a = rng.standard_normal((m, k))
    w = rng.standard_normal((n, k))
    c = oracle.gemm(a, w)
    for i in range(m):
        for j in range(n):
            exact = sum(Fraction(float(a[i, p])) * Fraction(float(w[j, p])) for p in range(k))
            bound = sum(abs(float(a[i, p]) * float(w[j, p])) for p in range(k)) * 2.0 ** -50
            assert abs(Fraction(float(c[i, j])) - exact) <= Fraction(bound)


def test_gemm_on_grid_equals_textbook_matmul(oracle_lib):
    """Inputs already on the NVFP4 grid with power-of-two scales: the quantised
    GEMM equals the ordinary FP64 product of the original matrices.  Non-square
    shapes so a transposed operand cannot pass."""
    rng = np.random.default_rng(9)
    m, n, k = 48, 80, 128
    e2 = _e2m1_table()

    def on_grid(rows, top_exp):
        codes = rng.integers(0, 16, (rows, k))
        codes[:, ::16] = 7                                      # every block max = 6
        bscale = 2.0 ** rng.integers(-2, 3, (rows, k // 16))
        bscale[0, 0] = 448.0                     # amax = 6 * 448 * 2^top, so s_g = 2^top exactly
        scale = np.repeat(bscale, 16, axis=1) * 2.0 ** top_exp
        return (e2[codes] * scale).astype(np.float32)

    a = on_grid(m, -3)
    w = on_grid(n, -7)
    c, _ = oracle.linear(a, [w])
    want = a.astype(np.float64) @ w.astype(np.float64).T
    np.testing.assert_allclose(c, want, rtol=1e-13, atol=0)


def test_fused_segments_follow_each_module_scale(oracle_lib):
    """The fix for the global-scale mismatch, as a definition: the fused GEMM over
    separately calibrated modules equals the per-module GEMMs concatenated, and
    applying one shared global scale to all columns does not."""
    p = synthetic.gdn_in_proj(m=16, k=256, widths=(64, 32, 16, 16), stds=(0.02, 0.02, 0.2, 0.2))
    c, info = oracle.linear(p.a, p.modules)
    s_ga = info["s_ga"]
    parts = [oracle.linear(p.a, [w], act_scale=s_ga)[0] for w in p.modules]
    np.testing.assert_array_equal(c, np.concatenate(parts, axis=1))
    qm = info["qmods"]
    scales = [float(m.s_g) for m in qm]
    assert max(scales) / min(scales) > 5                        # std 0.2 vs 0.02 modules
    for shared in (scales[0], max(scales)):
        w_bad = np.concatenate([oracle.dequantize(m.q, m.sf, shared) for m in qm], axis=0)
        c_bad = oracle.gemm(info["a_hat"], w_bad)
        rel = np.linalg.norm(c_bad - c) / np.linalg.norm(c)
        assert rel > 0.5


def test_gemm_error_magnitude_is_about_ten_percent(oracle_lib):
    """Order-of-magnitude sanity against the pages' "~11% GEMM error" on gate
    projections (abstract, mechanism (ii)): Gaussian data, NVFP4 both sides."""
    p = synthetic.prefill(m=64, k=512, n=96)
    c, _ = oracle.linear(p.a, p.modules)
    exact = p.a.double().numpy() @ p.modules[0].double().numpy().T
    rel = np.linalg.norm(c - exact) / np.linalg.norm(exact)
    assert 0.03 < rel < 0.3, rel


# --------------------------------------------------------------------------- layout, glue, inputs
def test_tiled_scale_layout_map(oracle_lib):
    assert oracle.sf_tiled_offset(33, 2, 256) == 16 + 4 + 2
    assert oracle.sf_tiled_offset(128, 0, 256) == 4 * 512
    assert oracle.sf_tiled_offset(5, 7, 256) == 512 + 5 * 16 + 3
    assert oracle.sf_tiled_offset(127, 3, 64) == 31 * 16 + 3 * 4 + 3
    rows, k = 300, 320
    size = oracle.sf_tiled_bytes(rows, k)
    assert size == 384 * 20
    offs = {oracle.sf_tiled_offset(r, b, k) for r in range(384) for b in range(20)}
    assert offs == set(range(size))
    rng = np.random.default_rng(0)
    sf = rng.integers(1, 255, (rows, k // 16)).astype(np.uint8)
    tiled = oracle.sf_to_tiled(sf, k)
    np.testing.assert_array_equal(oracle.sf_from_tiled(tiled, rows, k), sf)
    assert tiled.astype(np.int64).sum() == sf.astype(np.int64).sum()   # padding is zero


def test_silu_mul_matches_closed_form(oracle_lib):
    rng = np.random.default_rng(12)
    g = torch.from_numpy(rng.standard_normal(50_000).astype(np.float32) * 4).bfloat16()
    u = torch.from_numpy(rng.standard_normal(50_000).astype(np.float32)).bfloat16()
    h = oracle.silu_mul_bf16(g.view(torch.int16).numpy().view(np.uint16), u.view(torch.int16).numpy().view(np.uint16))
    hf = oracle.bf16_bits_to_f32(h).astype(np.float64)
    gd, ud = g.double().numpy(), u.double().numpy()
    want = gd / (1.0 + np.exp(-gd)) * ud
    assert np.all(np.abs(hf - want) <= 2.0 ** -8 * np.abs(want) + 1e-38)


def test_bf16_round_matches_torch(oracle_lib):
    rng = np.random.default_rng(13)
    x = (rng.standard_normal(100_000) * np.exp(rng.uniform(-30, 30, 100_000))).astype(np.float32)
    want = torch.from_numpy(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.bf16_round(x), want)


def test_synthetic_inputs_are_seeded_and_shaped():
    a1, c1 = synthetic.activations(64, 5120)
    a2, c2 = synthetic.activations(64, 5120)
    assert torch.equal(a1, a2) and torch.equal(c1, c2)
    assert a1.dtype == torch.bfloat16 and len(c1) == 5
    assert (a1[:, c1].float().abs().mean() > 30).item()
    p = synthetic.gdn_in_proj(m=8, k=64)
    assert p.n == 12384 and p.widths == [2048, 2048, 4096, 4096, 48, 48]


def test_gdn_gates_closed_forms(oracle_lib):
    """The Gated DeltaNet gates ("Why Gated DeltaNet Survives 4-Bit
    Quantization", page summary, "Gated DeltaNet Mechanics"; abstract,
    mechanism (ii) for the sigmoid) at points with known values."""
    ln3 = float(np.float32(np.log(3.0)))
    lnem1 = float(np.float32(np.log(np.e - 1.0)))          # softplus(ln(e - 1)) = 1
    a = np.array([[0.0, 0.0, lnem1, 1.0, 60.0, -60.0]], np.float32)
    b = np.array([[0.0, ln3, -ln3, 30.0, -30.0, 1.0]], np.float32)
    A_log = np.array([0.0, ln3, 0.0, 0.0, 0.0, 0.0], np.float32)
    dt_bias = np.array([0.0, 0.0, 0.0, -1.0, 0.0, 0.0], np.float32)
    g, beta = oracle.gdn_gates(a, b, A_log, dt_bias)
    e3 = np.exp(np.float64(ln3))
    np.testing.assert_allclose(g[0, 0], -np.log(2.0), rtol=1e-15)
    np.testing.assert_allclose(g[0, 1], -e3 * np.log(2.0), rtol=1e-15)      # the per-head decay rate scales
    np.testing.assert_allclose(g[0, 2], -np.log1p(np.exp(np.float64(lnem1))), rtol=1e-15)
    assert abs(g[0, 2] + 1.0) < 1e-7
    np.testing.assert_allclose(g[0, 3], -np.log(2.0), rtol=1e-15)           # dt_bias shifts the argument
    np.testing.assert_allclose(g[0, 4], -60.0, rtol=1e-15)                  # softplus(x) -> x
    np.testing.assert_allclose(g[0, 5], -np.exp(-60.0), rtol=1e-12)         # softplus(x) -> e^x
    np.testing.assert_allclose(beta[0, :3], [0.5, 0.75, 0.25], rtol=1e-7)
    np.testing.assert_allclose(beta[0, 3], 1.0 - np.exp(-30.0), rtol=1e-15)
    np.testing.assert_allclose(beta[0, 4], np.exp(-30.0), rtol=1e-12)
    assert np.all(g < 0) and np.all((beta > 0) & (beta < 1))


def test_gdn_gates_identities(oracle_lib):
    """softplus(x) - softplus(-x) = x, sigmoid(x) + sigmoid(-x) = 1 and
    softplus' = sigmoid: the g and beta paths checked against each other, per
    head, on random values."""
    rng = np.random.default_rng(21)
    m, heads = 64, 48
    x = rng.normal(0, 6, (m, heads)).astype(np.float32)
    A_log = rng.normal(0, 1, heads).astype(np.float32)
    zero = np.zeros(heads, np.float32)
    g_p, s_p = oracle.gdn_gates(x, x, A_log, zero)
    g_n, s_n = oracle.gdn_gates(-x, -x, A_log, zero)
    rate = np.exp(A_log.astype(np.float64))
    np.testing.assert_allclose((g_n - g_p) / rate, x.astype(np.float64), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s_p + s_n, 1.0, rtol=1e-15)
    # dt_bias enters as a shift of a: g(a, dt) = g(a + dt, 0)
    dt = rng.normal(0, 1, heads).astype(np.float32)
    y = (x.astype(np.float64) + dt).astype(np.float32)
    exact = (x.astype(np.float64) + dt) == y.astype(np.float64)
    g_dt, _ = oracle.gdn_gates(x, x, A_log, dt)
    g_y, _ = oracle.gdn_gates(y, y, A_log, zero)
    np.testing.assert_array_equal(g_dt[exact], g_y[exact])
    # central difference of -g / rate (softplus) equals beta (sigmoid)
    h = np.float32(2.0 ** -8)
    lo, hi = (x - h).astype(np.float32), (x + h).astype(np.float32)
    g_lo, _ = oracle.gdn_gates(lo, lo, np.zeros(heads, np.float32), zero)
    g_hi, _ = oracle.gdn_gates(hi, hi, np.zeros(heads, np.float32), zero)
    deriv = -(g_hi - g_lo) / (hi.astype(np.float64) - lo.astype(np.float64))
    np.testing.assert_allclose(deriv, s_p, atol=2e-6)


# --------------------------------------------------------------------------- FP8 KV cache
def _e4m3_value(code: int) -> float:
    """E4M3 (fn) value of a byte, from the format's definition: bias 7, three
    mantissa bits, exponent field 0 subnormal, 0x7f/0xff NaN."""
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 15, code & 7
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return sign * mag


def test_fp8_codes_round_trip_and_ties(oracle_lib):
    """Every finite E4M3 byte survives value -> byte; the midpoint of two
    neighbouring values rounds to the even mantissa; beyond 448 saturates
    ("calibrated FP8 KV-cache", abstract; Glonce "How to use it")."""
    codes = [c for c in range(256) if c & 0x7F != 0x7F]
    vals = np.array([_e4m3_value(c) for c in codes], np.float32)
    vals[codes.index(0x80)] = np.float32(-0.0)
    np.testing.assert_array_equal(oracle.fp8_quantize(vals, 1.0), np.array(codes, np.uint8))
    pos = [c for c in range(0x7F)]
    mids = np.array([(_e4m3_value(c) + _e4m3_value(c + 1)) / 2 for c in pos[:-1]], np.float32)
    got = oracle.fp8_quantize(mids, 1.0)
    want = np.array([c if c % 2 == 0 else c + 1 for c in pos[:-1]], np.uint8)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(oracle.fp8_quantize(-mids, 1.0), want | 0x80)
    big = np.array([448.0, 464.0, 479.9, 480.0, 1e30, np.inf], np.float32)
    np.testing.assert_array_equal(oracle.fp8_quantize(big, 1.0), np.full(6, 0x7E, np.uint8))
    np.testing.assert_array_equal(oracle.fp8_quantize(-big, 1.0), np.full(6, 0xFE, np.uint8))


def test_fp8_matches_torch_float8_in_range(oracle_lib):
    """Inside +-448 the bytes equal PyTorch's float8_e4m3fn cast (an independent
    round-to-nearest-even implementation), subnormals included."""
    rng = np.random.default_rng(31)
    x = (rng.standard_normal(200_000) * np.exp2(rng.uniform(-14, 8.7, 200_000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.fp8_quantize(x, 1.0), want)


def test_fp8_scale_is_a_divisor_and_bounds_the_error(oracle_lib):
    """s = amax / 448 maps the largest magnitude onto 448; values are divided
    by s (quantize(x, 2s) == quantize(x / 2, s)); read back as byte * s the
    error is at most half an E4M3 step."""
    rng = np.random.default_rng(32)
    x = (rng.standard_normal((256, 512)) * 3.0).astype(np.float32)
    x[17, 300] = -41.5
    amax = np.float32(np.abs(x).max())
    s = oracle.fp8_scale_from_amax(amax)
    assert s == np.float32(amax / np.float32(448.0))
    assert oracle.fp8_scale_from_amax(0.0) == 1.0 and oracle.fp8_scale_from_amax(448.0) == 1.0
    q = oracle.fp8_quantize(x, s)
    assert q[17, 300] == 0xFE
    np.testing.assert_array_equal(oracle.fp8_quantize(x, np.float32(2.0) * s), oracle.fp8_quantize(x / 2, s))
    back = np.vectorize(_e4m3_value)(q.astype(np.int64)) * np.float64(s)
    err = np.abs(back - x.astype(np.float64))
    bound = 2.0 ** -4 * np.abs(x) * (1 + 2.0 ** -20) + 2.0 ** -10 * np.float64(s)
    assert np.all(err <= bound)
    assert np.all(np.sign(back[np.abs(back) > 0]) == np.sign(x[np.abs(back) > 0]))
