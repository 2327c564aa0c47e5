"""Pins for the float64 oracle, checked against things other than itself.

Every check below is a closed form, a hand-derived worked value, a library
routine (torch's float64 scaled-dot-product attention, torch's bfloat16 and
float8_e4m3fn casts) or an invariant, chosen so that a plausible mistake in
the oracle (a dropped term, a wrong sign, index or axis, a transposed
operand, a wrong rounding rule) fails at least one of them.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import inputs as I

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------- bf16 ----

def test_bf16_round_matches_torch_cast_on_float32_values():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-20, 20, 20000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_ties_to_even():
    # ulp(1) in bf16 is 2**-7; 1 + 2**-8 is a tie between 1 and 1 + 2**-7.
    assert O.bf16_round(1 + 2.0 ** -8) == 1.0
    # 1 + 1.5 * 2**-7 ties between 1 + 2**-7 (odd) and 1 + 2**-6 (even).
    assert O.bf16_round(1 + 1.5 * 2.0 ** -7) == 1 + 2.0 ** -6
    assert O.bf16_round(-(1 + 2.0 ** -8)) == -1.0


def test_bf16_ulp_distance():
    a = np.array([1.0, 1.0, -1.0, 0.0])
    b = np.array([1.0 + 2.0 ** -7, 1.0 + 2.0 ** -6, -1.0 - 2.0 ** -7, -0.0])
    assert list(O.bf16_ulp_distance(a, b)) == [1, 2, 1, 0]


# -------------------------------------------------------------- RMSNorm ----

def test_rmsnorm_hand_case():
    x = np.tile([3.0, 4.0], 64)            # mean(x^2) = 12.5
    y = O.rmsnorm(x, eps=1e-6)
    r = math.sqrt(12.5 + 1e-6)
    assert np.allclose(y[:2], [3 / r, 4 / r], rtol=0, atol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 128))
    y = O.rmsnorm(x, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-14)
    assert np.allclose(O.rmsnorm(37.5 * x, eps=0.0), y, atol=1e-13)


def test_rmsnorm_weight_is_channelwise():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 128))
    w = rng.uniform(0.5, 2, 128)
    assert np.allclose(O.rmsnorm(x, w), O.rmsnorm(x) * w[None, :], atol=1e-14)


# --------------------------------------------------------- positions ----

def test_token_positions_small_grid():
    rows, cols = O.token_positions(2, 2, 3, ref_h=2, ref_w=2, ref_row_offset=2)
    assert list(rows) == [0, 0, 0, 0, 0, 1, 1, 1, 2, 2, 3, 3]
    assert list(cols) == [0, 0, 0, 1, 2, 0, 1, 2, 0, 1, 0, 1]


def test_token_positions_several_reference_grids():
    # Text 1, image 1 x 2, then a 2 x 1 reference at (5, 3) and a 1 x 2 one at (7, 0).
    rows, cols = O.token_positions(1, 1, 2, ref_grids=[(2, 1, 5, 3), (1, 2, 7, 0)])
    assert list(rows) == [0, 0, 0, 5, 6, 7, 7]
    assert list(cols) == [0, 0, 1, 3, 3, 0, 1]
    # One grid at column 0 is the single-reference rule.
    r1, c1 = O.token_positions(2, 2, 3, ref_h=2, ref_w=2, ref_row_offset=2)
    r2, c2 = O.token_positions(2, 2, 3, ref_grids=[(2, 2, 2, 0)])
    assert list(r1) == list(r2) and list(c1) == list(c2)


def test_shifting_one_reference_grid_keeps_its_own_scores():
    # RoPE scores depend on position differences only: moving a whole
    # reference grid leaves the scores among its own tokens unchanged and
    # changes those against the other streams.
    rng = np.random.default_rng(12)
    n_txt, img_h, img_w = 2, 2, 3
    grids_a = [(2, 2, 2, 0), (1, 3, 4, 0)]
    grids_b = [(2, 2, 2, 0), (1, 3, 9, 5)]
    N = n_txt + img_h * img_w + 4 + 3
    q = rng.standard_normal((1, N, 1, 128))
    k = rng.standard_normal((1, N, 1, 128))
    out = []
    for g in (grids_a, grids_b):
        qp, kp = O.prologue(q, k, n_txt=n_txt, img_h=img_h, img_w=img_w, ref_grids=g)
        out.append(qp[0, :, 0] @ kp[0, :, 0].T)
    own = slice(N - 3, N)
    np.testing.assert_allclose(out[0][own, own], out[1][own, own], rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(out[0][own, :n_txt + 6] - out[1][own, :n_txt + 6])) > 1e-3


# ----------------------------------------------------------------- RoPE ----

def _unit(ch, d=128):
    x = np.zeros((1, 1, d))
    x[0, 0, ch] = 1.0
    return x


def test_rope_identity_at_origin():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 2, 128))
    assert np.array_equal(O.rope_2d(x, np.zeros(3), np.zeros(3)), x)


def test_rope_row_half_frequency_and_sign():
    # pair i=16 of the row half: omega = 10000**(-32/64) = 1e-2; pos 100 -> 1 rad
    y = O.rope_2d(_unit(32), np.array([100]), np.array([0]))
    expect = np.zeros(128)
    expect[32], expect[33] = math.cos(1.0), math.sin(1.0)
    assert np.allclose(y[0, 0], expect, atol=1e-15)


def test_rope_col_half_odd_element():
    # pair i=8 of the column half: omega = 10000**(-16/64) = 0.1; pos 25 -> 2.5 rad
    # (a, b) = (0, 1) rotates to (-sin, cos).
    y = O.rope_2d(_unit(64 + 17), np.array([7]), np.array([25]))
    expect = np.zeros(128)
    expect[80], expect[81] = -math.sin(2.5), math.cos(2.5)
    assert np.allclose(y[0, 0], expect, atol=1e-14)


def test_rope_pair0_rotates_by_position_radians():
    for pos in (1, 5, 127, 255):
        y = O.rope_2d(_unit(0), np.array([pos]), np.array([3]))
        assert math.isclose(y[0, 0, 0], math.cos(pos), abs_tol=1e-13)
        assert math.isclose(y[0, 0, 1], math.sin(pos), abs_tol=1e-13)


def test_rope_matches_complex_rotation():
    """Independent formulation: pairs as complex numbers times e^{i phi}."""
    rng = np.random.default_rng(5)
    N, H, d = 6, 3, 128
    x = rng.standard_normal((N, H, d))
    pr, pc = rng.integers(0, 300, N), rng.integers(0, 300, N)
    y = O.rope_2d(x, pr, pc)
    z = x[..., 0::2] + 1j * x[..., 1::2]                      # [N, H, 64]
    freq = np.concatenate([10000.0 ** (-np.arange(32) / 32.0)] * 2)
    pos = np.concatenate([np.repeat(pr[:, None], 32, 1), np.repeat(pc[:, None], 32, 1)], 1)
    zr = z * np.exp(1j * pos[:, None, :] * freq[None, None, :])
    assert np.allclose(y[..., 0::2], zr.real, atol=1e-12)
    assert np.allclose(y[..., 1::2], zr.imag, atol=1e-12)


def test_rope_preserves_pair_norms_and_relative_positions():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    p, pp, delta = (3, 9), (40, 2), (128, 17)
    qr = O.rope_2d(q, [p[0]], [p[1]])
    kr = O.rope_2d(k, [pp[0]], [pp[1]])
    qs = O.rope_2d(q, [p[0] + delta[0]], [p[1] + delta[1]])
    ks = O.rope_2d(k, [pp[0] + delta[0]], [pp[1] + delta[1]])
    assert math.isclose(float(np.sum(qr * kr)), float(np.sum(qs * ks)), rel_tol=1e-12, abs_tol=1e-12)
    n0 = q[..., 0::2] ** 2 + q[..., 1::2] ** 2
    n1 = qr[..., 0::2] ** 2 + qr[..., 1::2] ** 2
    assert np.allclose(n0, n1, atol=1e-13)


# ------------------------------------------------------------- prologue ----

def test_prologue_norm_then_rope_hand_case():
    """Norm first (with a non-uniform weight), RoPE second, on one token."""
    q = np.zeros((1, 1, 1, 128))
    q[..., 0], q[..., 1] = 3.0, 4.0            # mean(x^2) = 25/128
    w = np.ones(128)
    w[0] = 2.0
    qp, kp = O.prologue(q, q, n_txt=0, img_h=1, img_w=1, q_norm_w=w, eps=0.0)
    # image token 0 sits at (0, 0): no rotation.  Now move it to row 2 via a
    # 3x1 grid (token index 2 -> (2, 0)).
    q3 = np.zeros((1, 3, 1, 128))
    q3[0, 2, 0, 0], q3[0, 2, 0, 1] = 3.0, 4.0
    qp3, _ = O.prologue(q3, q3, n_txt=0, img_h=3, img_w=1, q_norm_w=w, eps=0.0)
    r = math.sqrt(25.0 / 128.0)
    a, b = 3.0 / r * 2.0, 4.0 / r             # normalised and weighted
    assert np.allclose(qp[0, 0, 0, :2], [a, b], atol=1e-12)
    c, s = math.cos(2.0), math.sin(2.0)
    assert np.allclose(qp3[0, 2, 0, :2], [a * c - b * s, a * s + b * c], atol=1e-12)
    # RoPE first then norm would give a different pair (the weight would hit
    # the rotated value): make sure the two orders really differ here.
    alt = O.rmsnorm(O.rope_2d(q3, [0, 1, 2], [0, 0, 0]), w, eps=0.0)[0, 2, 0, :2]
    assert not np.allclose(alt, qp3[0, 2, 0, :2])


def test_prologue_invariant_to_row_scaling_of_inputs():
    """RMSNorm makes the prologue blind to per-row gains (outlier rows)."""
    w = I.WORKLOADS["tiny"]
    q, k, _ = I.make_qkv(w, seed=0)
    kf = k.double().numpy()
    k8 = kf.copy()
    k8[0, 5, 1, :] *= 8.0
    _, a = O.prologue(kf, kf, n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w, eps=0.0)
    _, b = O.prologue(k8, k8, n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w, eps=0.0)
    assert np.allclose(a, b, atol=1e-12)


# ----------------------------------------------------------------- E4M3 ----

@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x30, 0.5), (0x38, 1.0), (0x39, 1.125), (0x40, 2.0), (0x77, 240.0),
    (0x7E, 448.0), (0xFE, -448.0), (0xB8, -1.0),
])
def test_e4m3_decode_closed_form(code, value):
    assert O.e4m3_decode(code) == value


def test_e4m3_decode_all_codes_against_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    mine = O.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


def test_e4m3_encode_against_torch_cast():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal(50000) * np.exp2(rng.integers(-12, 9, 50000))).astype(np.float32)
    v = np.clip(v, -448, 448)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = O.e4m3_encode(v)
    assert np.array_equal(mine, ref)                     # including -0 (0x80) for tiny negatives


def test_e4m3_ties_and_saturation():
    assert O.e4m3_encode(1.0625) == 0x38       # tie 1.0 / 1.125 -> even (1.0)
    assert O.e4m3_encode(1.1875) == 0x3A       # tie 1.125 / 1.25 -> even (1.25)
    assert O.e4m3_encode(3 * 2.0 ** -10) == 0x02   # subnormal tie 1 / 2 quanta -> 2
    assert O.e4m3_encode(464.0) == 0x7E
    assert O.e4m3_encode(1e6) == 0x7E
    assert O.e4m3_encode(-1e6) == 0xFE
    assert O.e4m3_encode(-2.0 ** -12) == 0x80      # rounds to zero, keeps the sign
    assert O.e4m3_encode(-0.0) == 0x80 and O.e4m3_encode(0.0) == 0x00


def test_e4m3_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])   # -0 (0x80) included
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)


# ------------------------------------------------------ block quantiser ----

def test_block_quant_constant_block():
    x = np.full((1, 64, 1, 128), 2.0, dtype=np.float32)
    codes, scales = O.block_quantize_e4m3(x)
    assert scales[0, 0, 0] == np.float32(2.0) / np.float32(448.0)
    assert (codes == 0x7E).all()


def test_block_quant_absmax_448_is_identity_scale():
    rng = np.random.default_rng(8)
    x = np.clip(rng.standard_normal((1, 64, 1, 128)) * 100, -448, 448).astype(np.float32)
    x[0, 3, 0, 5] = -448.0
    codes, scales = O.block_quantize_e4m3(x)
    assert scales[0, 0, 0] == 1.0
    assert np.array_equal(codes, O.e4m3_encode(x))


def test_block_quant_zero_block_and_partial_tail():
    x = np.zeros((1, 70, 2, 128), dtype=np.float32)
    x[0, 66, 1, 0] = 3.0                     # only in the 6-token tail block of head 1
    codes, scales = O.block_quantize_e4m3(x)
    assert scales.shape == (1, 2, 2)
    assert scales[0, 0, 0] == 1.0 and scales[0, 0, 1] == 1.0 and scales[0, 1, 0] == 1.0
    assert scales[0, 1, 1] == np.float32(3.0) / np.float32(448.0)
    assert codes[0, 66, 1, 0] == 0x7E and codes.sum() == 0x7E


def test_block_quant_error_bound_and_block_independence():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((2, 150, 3, 128)).astype(np.float32)
    x[:, :, 2, :] *= 1000.0                  # a loud head must not change the others
    codes, scales = O.block_quantize_e4m3(x)
    deq = O.dequantize_e4m3(codes, scales)
    s = np.repeat(scales.astype(np.float64), 64, axis=2)[:, :, :150].transpose(0, 2, 1)[..., None]
    err = np.abs(deq - x)
    # 3 mantissa bits: half-ulp relative bound 2**-4 (normal range), plus the
    # subnormal quantum 2**-10 * scale; plus the float32 rounding of x * inv.
    bound = np.abs(x) * (2.0 ** -4 + 2.0 ** -22) + s * 2.0 ** -10
    assert (err <= bound).all()
    c2, s2 = O.block_quantize_e4m3(x[:, :, :2, :])
    assert np.array_equal(c2, codes[:, :, :2, :]) and np.array_equal(s2, scales[:, :2, :])


# ------------------------------------------------------------ attention ----

def test_attention_hand_two_keys():
    q = np.array([[[[1.0]]]])                               # B=N_q=H=d=1
    k = np.array([[[[0.0]], [[math.log(3.0)]]]]).reshape(1, 2, 1, 1)
    v = np.array([1.0, 5.0]).reshape(1, 2, 1, 1)
    out, lse = O.joint_attention(np.repeat(q, 2, axis=1), k, v, 1.0, rows=[0])
    assert math.isclose(out[0, 0, 0, 0], 4.0, rel_tol=1e-14)   # 1/4*1 + 3/4*5
    assert math.isclose(lse[0, 0, 0], math.log(4.0), rel_tol=1e-14)


def test_attention_matches_torch_sdpa_float64():
    rng = np.random.default_rng(10)
    B, N, H, d = 2, 77, 3, 128
    q, k, v = (rng.standard_normal((B, N, H, d)) for _ in range(3))
    scale = 1 / math.sqrt(d)
    out, lse = O.joint_attention(q, k, v, scale)
    t = lambda a: torch.from_numpy(a).permute(0, 2, 1, 3)   # [B, H, N, d]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)
    assert np.allclose(out, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    s = torch.einsum("bhnd,bhmd->bhnm", t(q), t(k)) * scale
    assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def test_attention_invariants():
    rng = np.random.default_rng(11)
    B, N, H, d = 1, 40, 2, 128
    q, k, v = (rng.standard_normal((B, N, H, d)) for _ in range(3))
    # rows of softmax sum to 1: V of ones gives ones
    out, _ = O.joint_attention(q, k, np.ones_like(v), 0.1)
    assert np.allclose(out, 1.0, atol=1e-13)
    # Q = 0 gives the mean of V over all keys
    out, _ = O.joint_attention(np.zeros_like(q), k, v, 0.1)
    assert np.allclose(out, v.mean(axis=1, keepdims=True), atol=1e-13)
    # one key: O = V
    out, _ = O.joint_attention(q[:, :1], k[:, :1], v[:, :1], 0.1)
    assert np.allclose(out, v[:, :1], atol=1e-15)
    # permuting keys together with values leaves O unchanged
    perm = rng.permutation(N)
    o1, l1 = O.joint_attention(q, k, v, 0.1)
    o2, l2 = O.joint_attention(q, k[:, perm], v[:, perm], 0.1, rows=np.arange(N))
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)
    # one dominant logit selects its value row
    kd = k.copy()
    kd[0, 17, :, :] = q[0, 3, :, :] * 50.0
    out, _ = O.joint_attention(q, kd, v, 1.0, rows=[3])
    assert np.allclose(out[0, 0], v[0, 17], atol=1e-12)


def test_attention_sampled_rows_equal_full_rows():
    rng = np.random.default_rng(12)
    q, k, v = (rng.standard_normal((1, 50, 2, 128)) for _ in range(3))
    rows = [0, 7, 49]
    full, lf = O.joint_attention(q, k, v, 0.09)
    part, lp = O.joint_attention(q, k, v, 0.09, rows=rows)
    assert np.allclose(full[:, rows], part, rtol=0, atol=1e-14)
    assert np.allclose(lf[:, :, rows], lp, rtol=0, atol=1e-14)


# ------------------------------------------------------- input recipe ----

def test_inputs_are_seeded_and_shaped():
    w = I.WORKLOADS["tiny"]
    a = I.make_qkv(w, 0)
    b = I.make_qkv(w, 0)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert a[0].shape == (1, 288, 2, 128) and a[0].dtype == torch.bfloat16
    rows = I.sampled_rows(I.WORKLOADS["i2i_2048"], 256)
    assert len(rows) == 256 and len(set(rows.tolist())) == 256
    for t in (0, 511, 512, 512 + 16383, 512 + 16384, 33279):
        assert t in rows
    m = I.outlier_rows(I.WORKLOADS["t2i_2048"])
    assert m.sum() == round(0.01 * m.size)


# ---------------------------------------------------------------------------
# RoPE table and the fused QKV projection
# ---------------------------------------------------------------------------

def test_rope_table_closed_form_entries():
    t = O.rope_table(n_txt=3, img_h=4, img_w=5, ref_h=2, ref_w=2, ref_row_offset=4)
    assert t.shape == (3 + 20 + 4, 64, 2)
    np.testing.assert_allclose(t[..., 0] ** 2 + t[..., 1] ** 2, 1.0, atol=1e-15)
    np.testing.assert_array_equal(t[:3], np.broadcast_to([1.0, 0.0], (3, 64, 2)))   # text at (0, 0)
    tok = 3 + 2 * 5 + 3                          # image token at (row 2, col 3)
    assert t[tok, 0].tolist() == [math.cos(2.0), math.sin(2.0)]          # pair 0: pos radians
    assert t[tok, 32].tolist() == [math.cos(3.0), math.sin(3.0)]
    phi = 2.0 * math.pow(10000.0, -1.0 / 32.0)                         # pair 1 of the row half
    np.testing.assert_allclose(t[tok, 1], [math.cos(phi), math.sin(phi)], rtol=0, atol=1e-15)
    ref = 3 + 20 + 3                              # reference token (row 4 + 1, col 1)
    assert t[ref, 0].tolist() == [math.cos(5.0), math.sin(5.0)]
    assert t[ref, 32].tolist() == [math.cos(1.0), math.sin(1.0)]


def test_rope_table_is_the_rotation_rope_2d_applies():
    rows, cols = O.token_positions(2, 3, 4)
    t = O.rope_table(2, 3, 4)
    e = np.zeros((1, len(rows), 1, 128))
    e[..., 0::2] = 1.0                            # unit first element of every pair
    r = O.rope_2d(e, rows, cols)[0, :, 0]
    np.testing.assert_allclose(r[:, 0::2], t[..., 0], atol=1e-15)
    np.testing.assert_allclose(r[:, 1::2], t[..., 1], atol=1e-15)


def _qkv_case(C=256, H=2, n_txt=3, img_h=2, img_w=3, seed=5):
    rng = np.random.default_rng(seed)
    n = n_txt + img_h * img_w
    x = rng.standard_normal((2, n, C))
    w_txt = rng.standard_normal((3 * H * 128, C)) / np.sqrt(C)
    w_img = rng.standard_normal((3 * H * 128, C)) / np.sqrt(C)
    return x, w_txt, w_img, dict(n_txt=n_txt, img_h=img_h, img_w=img_w, H=H)


def test_qkv_fused_identity_weights_reduce_to_prologue():
    H, n_txt = 2, 3
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, n_txt + 6, H * 128))
    eye = np.eye(H * 128)
    w = np.concatenate([eye, eye, eye])           # Q = K = V = x
    q, k, v = O.qkv_fused(x, w, w, n_txt=n_txt, img_h=2, img_w=3, H=H)
    xh = x.reshape(1, n_txt + 6, H, 128)
    qp, kp = O.prologue(xh, xh, n_txt=n_txt, img_h=2, img_w=3)
    np.testing.assert_array_equal(v, xh)
    np.testing.assert_allclose(q, qp, rtol=0, atol=1e-14)
    np.testing.assert_allclose(k, kp, rtol=0, atol=1e-14)


def test_qkv_fused_streams_use_their_own_weights():
    x, w_txt, w_img, kw = _qkv_case()
    q0, k0, v0 = O.qkv_fused(x, w_txt, w_img, **kw)
    q1, k1, v1 = O.qkv_fused(x, w_txt, 2.0 * w_img + 1.0, **kw)        # image weights only
    n = kw["n_txt"]
    for a, b in ((q0, q1), (k0, k1), (v0, v1)):
        np.testing.assert_array_equal(a[:, :n], b[:, :n])
        assert not np.allclose(a[:, n:], b[:, n:])
    q2, _, v2 = O.qkv_fused(x, 3.0 * w_txt, w_img, eps=0.0, **kw)       # text weights only
    q0e, _, _ = O.qkv_fused(x, w_txt, w_img, eps=0.0, **kw)
    np.testing.assert_array_equal(q2[:, n:], q0e[:, n:])
    np.testing.assert_allclose(v2[:, :n], 3.0 * v0[:, :n], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(q2[:, :n], q0e[:, :n], rtol=0, atol=1e-12)  # RMSNorm (eps 0) removes the scale


def test_qkv_fused_value_brute_force_and_norm_weights():
    x, w_txt, w_img, kw = _qkv_case(C=64, H=2)
    H = kw["H"]
    q, k, v = O.qkv_fused(x, w_txt, w_img, **kw)
    b, t, h, c = 1, 5, 1, 17                      # an image token
    f = 2 * H * 128 + h * 128 + c
    want = sum(float(x[b, t, i]) * float(w_img[f, i]) for i in range(64))
    assert abs(v[b, t, h, c] - want) < 1e-12
    wq = np.linspace(0.5, 1.5, 128)
    q2, _, _ = O.qkv_fused(x, w_txt, w_img, q_norm_w=(None, wq), **kw)
    n = kw["n_txt"]
    np.testing.assert_array_equal(q2[:, :n], q[:, :n])                    # text tokens untouched
    # RoPE mixes pairs, so compare the pair norms: weights scale channel-wise
    # before rotation; with equal weights within a pair the norm scales by it.
    wq_pairs = np.repeat(np.linspace(0.5, 1.5, 64), 2)
    q3, _, _ = O.qkv_fused(x, w_txt, w_img, q_norm_w=(None, wq_pairs), **kw)
    pn = lambda a: np.sqrt(a[..., 0::2] ** 2 + a[..., 1::2] ** 2)
    np.testing.assert_allclose(pn(q3[:, n:]), pn(q[:, n:]) * wq_pairs[0::2], rtol=1e-12)


# ---------------------------------------------------------------------------
# FP8 repair budget
# ---------------------------------------------------------------------------

def test_repair_count():
    assert O.repair_count(16896, 0.005) == 85          # ceil(84.48)
    assert O.repair_count(200, 0.005) == 1
    assert O.repair_count(100, 0.0) == 0
    assert O.repair_count(10, 1.0) == 10 and O.repair_count(10, 2.0) == 10
    assert O.repair_count(1000, 0.002) == 2            # exact product: no extra token


def test_repair_select_hand_case():
    # 1 batch, 1 head, 6 tokens, d = 2.  Errors: token 0: 1 (K), 1: 4 (V),
    # 2: 0, 3: 4 (2 from K, 2 from V), 4: 9, 5: 4.
    ke = np.zeros((1, 6, 1, 2)); kd = np.zeros_like(ke)
    ve = np.zeros_like(ke); vd = np.zeros_like(ke)
    kd[0, 0, 0, 0] = 1.0                 # e = 1
    vd[0, 1, 0, 1] = 2.0                 # e = 4
    kd[0, 3, 0, :] = 1.0; vd[0, 3, 0, :] = -1.0             # e = 2 + 2 = 4
    ke[0, 4, 0, 1] = 3.0                 # e = 9
    ve[0, 5, 0, 0] = -2.0                # e = 4
    idx, err = O.repair_select(ke, ve, kd, vd, rho=0.5)   # m = 3
    np.testing.assert_allclose(err[0, 0], [1, 4, 0, 4, 9, 4], rtol=1e-12)
    # Largest: 4 (9), then the ties at 4 in token order: 1, 3 (5 is left out).
    assert idx[0, 0].tolist() == [1, 3, 4]


def test_repaired_attention_limits():
    rng = np.random.default_rng(11)
    shape = (1, 70, 2, 128)
    ke, ve, qd = (rng.standard_normal(shape) for _ in range(3))
    kd = ke + 0.05 * rng.standard_normal(shape)
    vd = ve + 0.05 * rng.standard_normal(shape)
    none = np.zeros((1, 2, 0), dtype=np.int64)
    o0, l0 = O.repaired_attention(qd, kd, vd, ke, ve, none, 0.09)
    r0, rl0 = O.joint_attention(qd, kd, vd, 0.09)
    np.testing.assert_array_equal(o0, r0)                               # no budget: plain FP8
    np.testing.assert_array_equal(l0, rl0)
    allk = np.broadcast_to(np.arange(70), (1, 2, 70))
    o1, _ = O.repaired_attention(qd, kd, vd, ke, ve, allk, 0.09)
    r1, _ = O.joint_attention(qd, ke, ve, 0.09)
    np.testing.assert_allclose(o1, r1, rtol=0, atol=1e-15)             # full budget: exact K, V
    # A partial budget on the worst tokens moves the result toward exact.
    idx, _ = O.repair_select(ke, ve, kd, vd, rho=0.3)
    oh, _ = O.repaired_attention(qd, kd, vd, ke, ve, idx, 0.09)
    assert np.linalg.norm(oh - r1) < np.linalg.norm(o0 - r1)


# -------------------------------------------------------- block sparse ----

def test_sparse_pool_block_means_of_a_ramp():
    # x[b, t, h, c] = t + 100 h: the mean of a block [a, e) is (a + e - 1) / 2.
    N, H = 11, 2
    x = np.zeros((1, N, H, 3))
    for h in range(H):
        x[0, :, h, :] = (np.arange(N) + 100 * h)[:, None]
    pooled = O.sparse_pool(x, 4)
    assert pooled.shape == (1, H, 3, 3)
    for h in range(H):
        np.testing.assert_allclose(pooled[0, h, :, 0], np.array([1.5, 5.5, 9.0]) + 100 * h)


def _hand_sparse_case():
    # Query rows all e0; key block j (2 tokens) rows ln(j + 1) e0; scale 1:
    # pooled scores ln(j + 1), so p_ij = (j + 1) / 10 for every query block.
    N, d = 8, 4
    q = np.zeros((1, N, 1, d))
    k = np.zeros((1, N, 1, d))
    q[0, :, 0, 0] = 1.0
    for j in range(4):
        k[0, 2 * j:2 * j + 2, 0, 0] = math.log(j + 1)
    return q, k


def test_sparse_probs_hand_case():
    q, k = _hand_sparse_case()
    p = O.sparse_probs(q, k, 1.0, qblock=2, kblock=2)
    assert p.shape == (1, 1, 4, 4)
    np.testing.assert_allclose(p, np.broadcast_to([0.1, 0.2, 0.3, 0.4], p.shape), rtol=1e-12)


@pytest.mark.parametrize("tau,kept", [(0.0, [0, 1, 2, 3]), (0.5, [1, 2, 3]), (1.0, [2, 3]), (2.0, [3]),
                                      (9.0, [3])])
def test_sparse_keep_hand_case(tau, kept):
    # Threshold tau / 4 against p = (0.1, 0.2, 0.3, 0.4); the top block always stays.
    q, k = _hand_sparse_case()
    keep = O.sparse_keep(O.sparse_probs(q, k, 1.0, qblock=2, kblock=2), tau)
    for i in range(4):
        assert np.nonzero(keep[0, 0, i])[0].tolist() == kept


def test_sparse_keep_ties_take_the_first_maximum():
    keep = O.sparse_keep(np.array([[0.25, 0.375, 0.375]]), 5.0)
    assert keep.tolist() == [[False, True, False]]


def test_sparse_keep_monotone_in_tau():
    rng = np.random.default_rng(3)
    p = rng.dirichlet(np.ones(37), size=(2, 3, 5))
    k0, k1, k2 = (O.sparse_keep(p, t) for t in (0.5, 1.0, 2.0))
    assert not (k1 & ~k0).any() and not (k2 & ~k1).any()
    assert O.sparse_keep(p, 0.0).all()
    top = np.argmax(p, axis=-1)
    assert np.take_along_axis(k2, top[..., None], axis=-1).all()


def _brute_block_sparse(q, k, v, keep, scale, qblock, kblock):
    # Naive loops: collect each query's keys one by one, softmax with math.exp.
    B, N, H, d = q.shape
    out = np.zeros((B, N, H, d))
    lse = np.full((B, H, N), -math.inf)
    for b in range(B):
        for h in range(H):
            for t in range(N):
                keys = [u for u in range(N) if keep[b, h, t // qblock, u // kblock]]
                if not keys:
                    continue
                s = [scale * sum(q[b, t, h, c] * k[b, u, h, c] for c in range(d)) for u in keys]
                m = max(s)
                w = [math.exp(x - m) for x in s]
                tot = sum(w)
                for c in range(d):
                    out[b, t, h, c] = sum(wi * v[b, u, h, c] for wi, u in zip(w, keys)) / tot
                lse[b, h, t] = m + math.log(tot)
    return out, lse


def test_block_sparse_attention_brute_force():
    rng = np.random.default_rng(4)
    B, N, H, d = 1, 11, 2, 3
    q, k, v = (rng.standard_normal((B, N, H, d)) for _ in range(3))
    keep = rng.random((B, H, 4, 3)) < 0.5       # query blocks of 3, key blocks of 4
    keep[0, 0, 1] = False                       # one query block with no keys
    keep[0, 1, 2] = [False, False, True]        # only the partial last key block
    got, glse = O.block_sparse_attention(q, k, v, keep, 0.7, qblock=3, kblock=4)
    ref, rlse = _brute_block_sparse(q, k, v, keep, 0.7, 3, 4)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(np.isinf(glse), np.isinf(rlse))
    fin = np.isfinite(rlse)
    np.testing.assert_allclose(glse[fin], rlse[fin], rtol=1e-12)
    assert np.all(got[0, 3:6, 0] == 0.0)


def test_block_sparse_attention_all_kept_is_joint_attention():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((2, 70, 2, 8)) for _ in range(3))
    keep = O.sparse_keep(O.sparse_probs(q, k, 0.3, qblock=32, kblock=16), 0.0)
    assert keep.all()
    got, glse = O.block_sparse_attention(q, k, v, keep, 0.3, qblock=32, kblock=16)
    ref, rlse = O.joint_attention(q, k, v, 0.3)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(glse, rlse, rtol=1e-12)
    rows = np.array([0, 31, 32, 69])
    sub, slse = O.block_sparse_attention(q, k, v, keep, 0.3, rows=rows, qblock=32, kblock=16)
    np.testing.assert_allclose(sub, ref[:, rows], rtol=1e-12, atol=1e-13)


def test_block_sparse_attention_of_constant_values_is_constant():
    rng = np.random.default_rng(6)
    q, k = (rng.standard_normal((1, 40, 1, 4)) for _ in range(2))
    v = np.ones((1, 40, 1, 4)) * 2.5
    keep = O.sparse_keep(O.sparse_probs(q, k, 0.5, qblock=16, kblock=8), 1.0)
    got, _ = O.block_sparse_attention(q, k, v, keep, 0.5, qblock=16, kblock=8)
    np.testing.assert_allclose(got, 2.5, rtol=1e-13)
