"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a closed form, a value the pages print
(tests/golden/), a library routine that computes the same definition by
another route, a special case, or brute force on a tiny input. The last block
plants plausible mistakes into the oracle (on the CPU) and checks that a pin
catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import vlm_oracle as O
from vision_language_model_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


# ---------------------------------------------------------------------------
# a0 / a13 counts: values printed on the pages
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("token_counts.json")["cases"], ids=lambda c: c["name"])
def test_token_counts_match_pages(case):
    h, w = O.patch_grid(case["height"], case["width"], case["patch"])
    assert h * w == case["patches"]
    hm, wm = O.merged_grid(h, w, case["merge"])
    assert hm * wm == case["merged"]


@pytest.mark.parametrize("case", _golden("token_counts.json")["tiled"], ids=lambda c: c["name"])
def test_tiled_token_counts_match_pages(case):
    n = O.tile_count(case["height"], case["width"], case["tile"])
    assert n == case["tiles"]
    h, w = O.patch_grid(case["tile"], case["tile"], case["patch"])
    assert n * h * w == case["tokens"]


def test_hparams_match_pages():
    g = _golden("hparams.json")
    for preset, ref in (("mistral3", O.MISTRAL3), ("pixtral12b", O.PIXTRAL12B)):
        for key in ("width", "mlp", "layers", "heads", "patch", "rope_theta", "merge"):
            assert ref[key] == g[preset][key], (preset, key)
    assert O.MISTRAL3["image_token_id"] == g["mistral3"]["image_token_id"]
    assert O.MISTRAL3["proj_out"] == g["mistral3"]["proj_out"]
    assert list(O.IMAGE_MEAN) == g["processor"]["image_mean"]
    assert list(O.IMAGE_STD) == g["processor"]["image_std"]
    assert O.LONGEST_EDGE == g["processor"]["longest_edge"]


def test_off_grid_sizes_rejected():
    with pytest.raises(ValueError):
        O.patch_grid(225, 224, 14)
    with pytest.raises(ValueError):
        O.merged_grid(15, 16, 2)
    assert O.merged_grid(15, 16, 1) == (15, 16)


def test_positions_restart_per_image():
    rows, cols, cu = O.positions([(2, 3), (1, 2)])
    assert cu.tolist() == [0, 6, 8]
    assert rows.tolist() == [0, 0, 0, 1, 1, 1, 0, 0]
    assert cols.tolist() == [0, 1, 2, 0, 1, 2, 0, 1]


# ---------------------------------------------------------------------------
# a1, a2: normalisation and patch embedding
# ---------------------------------------------------------------------------

def test_normalize_constants():
    img = np.ones((3, 2, 2))
    got = O.normalize_pixels(img)
    for c in range(3):
        assert got[c, 0, 0] == pytest.approx((1.0 - O.IMAGE_MEAN[c]) / O.IMAGE_STD[c], rel=1e-15)


@pytest.mark.parametrize("patch,hw", [(14, (28, 42)), (16, (32, 48)), (3, (9, 6))])
def test_patch_embed_equals_strided_conv2d(patch, hw):
    d = 8
    img = RNG.standard_normal((3, *hw))
    w = RNG.standard_normal((d, 3, patch, patch))
    got = O.patch_embed(img, w)
    ref = F.conv2d(torch.from_numpy(img)[None], torch.from_numpy(w), stride=patch)[0]  # [D, h, w]
    ref = ref.permute(1, 2, 0).reshape(-1, d).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_patch_embed_p1_identity_is_passthrough():
    img = RNG.standard_normal((3, 4, 5))
    w = np.eye(3).reshape(3, 3, 1, 1)
    got = O.patch_embed(img, w)
    np.testing.assert_array_equal(got, img.transpose(1, 2, 0).reshape(20, 3))


# ---------------------------------------------------------------------------
# RMSNorm
# ---------------------------------------------------------------------------

def test_rmsnorm_constant_vector_gives_sign_times_gain():
    g = RNG.standard_normal(64)
    for cval in (3.5, -0.25):
        y = O.rms_norm(np.full((1, 64), cval), g, 0.0)
        np.testing.assert_allclose(y[0], math.copysign(1.0, cval) * g, rtol=1e-14)


def test_rmsnorm_matches_torch():
    x = RNG.standard_normal((7, 1024)) * 3
    g = RNG.standard_normal(1024)
    ref = F.rms_norm(torch.from_numpy(x), (1024,), torch.from_numpy(g), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-5), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# 2D RoPE
# ---------------------------------------------------------------------------

def test_rope_frequencies_closed_form():
    om = O.rope_frequencies(1e4, 64)
    assert om[0] == 1.0
    assert om[2] == pytest.approx(10.0 ** -0.25, rel=1e-14)   # 1e4^(-4/64)
    assert om[31] == pytest.approx(1e4 ** (-62 / 64), rel=1e-14)
    # pair 1 at (row 1, col 0) turns by w_2; pair 16 at (row 0, col 1) by w_1
    ang = O.rope_angles([1, 0], [0, 1], 1e4, 64)
    assert ang[0, 1] == pytest.approx(10.0 ** -0.25, rel=1e-14)
    assert ang[1, 16] == pytest.approx(1e4 ** (-2 / 64), rel=1e-14)
    assert np.all(ang[0, 16:] == 0) and np.all(ang[1, :16] == 0)


def test_rope_is_complex_rotation():
    x = RNG.standard_normal((5, 2, 64))
    ang = O.rope_angles(np.arange(5), np.arange(5)[::-1], 1e4, 64)
    got = O.apply_rope(x, ang)
    z = (x[..., :32] + 1j * x[..., 32:]) * np.exp(1j * ang)[:, None, :]
    np.testing.assert_allclose(got[..., :32], z.real, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(got[..., 32:], z.imag, rtol=1e-13, atol=1e-13)


def test_rope_preserves_norm_and_origin_is_identity():
    x = RNG.standard_normal((16, 3, 64))
    rows, cols, _ = O.positions([(4, 4)])
    y = O.apply_rope(x, O.rope_angles(rows, cols, 1e4, 64))
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-6)
    np.testing.assert_array_equal(y[0], x[0])  # position (0, 0)


def test_rope_scores_depend_only_on_relative_position_bruteforce_4x4():
    q = RNG.standard_normal(64)
    k = RNG.standard_normal(64)
    grid = [(r, c) for r in range(4) for c in range(4)]
    seen = {}
    for r1, c1 in grid:
        for r2, c2 in grid:
            qa = O.apply_rope(q[None, None], O.rope_angles([r1], [c1], 1e4, 64))[0, 0]
            ka = O.apply_rope(k[None, None], O.rope_angles([r2], [c2], 1e4, 64))[0, 0]
            seen.setdefault((r1 - r2, c1 - c2), []).append(float(qa @ ka))
    assert len(seen) == 49
    for vals in seen.values():
        assert max(vals) - min(vals) < 1e-5 * max(1.0, max(abs(v) for v in vals))
    # different offsets give different scores in general
    assert abs(seen[(1, 0)][0] - seen[(0, 1)][0]) > 1e-6


def test_rope_row_shift_changes_only_row_half():
    x = RNG.standard_normal((1, 1, 64))
    a = O.apply_rope(x, O.rope_angles([0], [2], 1e4, 64))
    b = O.apply_rope(x, O.rope_angles([3], [2], 1e4, 64))
    pairs_changed = np.abs(a - b)[0, 0]
    changed = (pairs_changed[:32] > 0) | (pairs_changed[32:] > 0)
    assert changed[:16].all() and not changed[16:].any()


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _sdpa_blockdiag(q, k, v, cu):
    t = q.shape[0]
    mask = torch.zeros(t, t, dtype=torch.bool)
    for b in range(len(cu) - 1):
        mask[cu[b]:cu[b + 1], cu[b]:cu[b + 1]] = True
    qt, kt, vt = (torch.from_numpy(a).permute(1, 0, 2)[None] for a in (q, k, v))
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)[0]  # [H, T, dh]
    return o.permute(1, 0, 2).reshape(t, -1).numpy()


def test_attention_matches_sdpa_block_diagonal():
    cu = [0, 5, 6, 19, 40]
    q, k, v = (RNG.standard_normal((40, 3, 64)) * 2 for _ in range(3))
    np.testing.assert_allclose(O.attention(q, k, v, cu), _sdpa_blockdiag(q, k, v, cu), rtol=1e-11, atol=1e-12)
    rows = [0, 5, 18, 39]
    np.testing.assert_allclose(O.attention_rows(q, k, v, cu, rows), O.attention(q, k, v, cu)[rows], rtol=1e-12)


def test_attention_single_patch_returns_v_and_zero_q_gives_mean():
    q, k, v = (RNG.standard_normal((1, 2, 64)) for _ in range(3))
    np.testing.assert_array_equal(O.attention(q, k, v, [0, 1]), v.reshape(1, -1))
    q0 = np.zeros((9, 2, 64))
    k, v = RNG.standard_normal((9, 2, 64)), RNG.standard_normal((9, 2, 64))
    out = O.attention(q0, k, v, [0, 9])
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=0).reshape(1, -1), (9, 128)), rtol=1e-13)


# ---------------------------------------------------------------------------
# Activations and MLP
# ---------------------------------------------------------------------------

def test_activations_special_values_and_library():
    z = np.linspace(-8, 8, 101)
    assert O.silu(0.0) == 0.0 and O.gelu(0.0) == 0.0
    np.testing.assert_allclose(O.silu(z), F.silu(torch.from_numpy(z)).numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O.gelu(z), F.gelu(torch.from_numpy(z)).numpy(), rtol=1e-13, atol=1e-15)
    assert O.gelu(30.0) == pytest.approx(30.0, rel=1e-15)
    assert O.gelu(1.0) == pytest.approx(0.5 * (1 + math.erf(1 / math.sqrt(2))), rel=1e-15)


def _tiny_tower(seed=0, layers=2, width=64, mlp=128, patch=14, heads=4):
    cfg = dict(O.MISTRAL3, layers=layers, width=width, mlp=mlp, heads=heads, head_dim=width // heads)
    tw = {k: v.double().numpy() for k, v in synth.tower_weights(seed, layers, width, mlp, patch).items()}
    return cfg, tw


def test_mlp_with_zero_up_is_identity_block_on_ffn_half():
    cfg, tw = _tiny_tower(layers=1, heads=1)
    cfg["head_dim"] = 64
    lw = O.layer_weights(tw, 0)
    lw["w_up"][:] = 0.0
    lw["wo"][:] = 0.0  # attention branch off too
    x = RNG.standard_normal((6, 64))
    rows, cols, cu = O.positions([(2, 3)])
    y = O.tower_block(x, lw, O.rope_angles(rows, cols, 1e4, 64), cu, cfg)
    np.testing.assert_array_equal(y, x)


def test_block_rows_equals_full_block_on_those_rows():
    cfg, tw = _tiny_tower(layers=1, heads=1)
    cfg["head_dim"] = 64
    lw = O.layer_weights(tw, 0)
    grids = [(3, 4), (2, 2)]
    rows_, cols_, cu = O.positions(grids)
    ang = O.rope_angles(rows_, cols_, 1e4, 64)
    x = RNG.standard_normal((16, 64))
    full = O.tower_block(x, lw, ang, cu, cfg)
    sel = [0, 5, 11, 12, 15]
    np.testing.assert_allclose(O.tower_block_rows(x, lw, ang, cu, cfg, sel), full[sel], rtol=1e-12, atol=1e-12)
    kv = O.block_keys_values(x, lw, ang, cfg)
    np.testing.assert_allclose(O.tower_block_rows(x, lw, ang, cu, cfg, [3], kv=kv), full[[3]], rtol=1e-12)


# ---------------------------------------------------------------------------
# Tower-level invariants: isolation and packing
# ---------------------------------------------------------------------------

def test_tower_isolation_and_packed_equals_separate():
    cfg, tw = _tiny_tower(heads=1)
    cfg["head_dim"] = 64
    imgs = [synth.pixels_u01(0, f"iso{i}", h, w).double().numpy() for i, (h, w) in enumerate([(28, 42), (14, 14), (42, 28)])]
    packed = O.tower(imgs, tw, cfg)
    sep = np.concatenate([O.tower([im], tw, cfg) for im in imgs], axis=0)
    np.testing.assert_allclose(packed, sep, rtol=1e-12, atol=1e-12)
    pert = [im.copy() for im in imgs]
    pert[1] += 0.5
    out2 = O.tower(pert, tw, cfg)
    n0, n1 = 6, 1
    np.testing.assert_array_equal(out2[:n0], packed[:n0])
    np.testing.assert_array_equal(out2[n0 + n1:], packed[n0 + n1:])
    assert np.abs(out2[n0:n0 + n1] - packed[n0:n0 + n1]).max() > 1e-3


# ---------------------------------------------------------------------------
# Merge
# ---------------------------------------------------------------------------

def test_merge_matches_torch_unfold():
    d = 5
    grids = [(4, 6), (2, 2)]
    x = RNG.standard_normal((28, d))
    got = O.merge_unfold(x, grids, 2)
    ref, off = [], 0
    for h, w in grids:
        img = torch.from_numpy(x[off:off + h * w]).reshape(h, w, d).permute(2, 0, 1)[None]  # [1, D, h, w]
        ref.append(F.unfold(img, kernel_size=2, stride=2)[0].T.numpy())  # [L, D*4] channel-major
        off += h * w
    np.testing.assert_array_equal(got, np.concatenate(ref))


def test_merge_selector_weights_pick_the_right_patch():
    d, h, w = 3, 4, 4
    x = RNG.standard_normal((h * w, d))
    z = O.merge_unfold(x, [(h, w)], 2)
    for c in range(d):
        for dy in range(2):
            for dx in range(2):
                sel = np.zeros(4 * d)
                sel[c * 4 + dy * 2 + dx] = 1.0
                for i in range(2):
                    for j in range(2):
                        assert z[i * 2 + j] @ sel == x[(2 * i + dy) * w + (2 * j + dx), c]


# ---------------------------------------------------------------------------
# Scatter
# ---------------------------------------------------------------------------

def test_scatter_matches_masked_scatter_bit_exact():
    ids = synth.text_sequences(3, 2, 64, [[5], [7, 2]])
    n_img = int((ids == 10).sum())
    assert n_img == 14
    img = synth.randn_bf16(3, "img", (n_img, 32), 1.0)
    text = synth.text_embeddings(3, 128, 32)
    got = O.scatter(ids.numpy(), img.view(torch.int16).numpy(), text.view(torch.int16).numpy(), 10)
    mask = (ids.reshape(-1) == 10)[:, None].expand(-1, 32)
    ref = text.masked_scatter(mask, img)
    assert np.array_equal(got, ref.view(torch.int16).numpy())
    untouched = ~(ids.reshape(-1) == 10).numpy()
    assert np.array_equal(got[untouched], text.view(torch.int16).numpy()[untouched])


def test_scatter_count_mismatch_raises():
    ids = np.array([1, 10, 10, 3])
    with pytest.raises(ValueError):
        O.scatter(ids, np.zeros((3, 4), np.int16), np.zeros((4, 4), np.int16), 10)
    with pytest.raises(ValueError):
        O.scatter(ids, np.zeros((1, 4), np.int16), np.zeros((4, 4), np.int16), 10)


def test_text_placeholder_runs_count():
    ids = synth.text_sequences(0, 4, 4096, [[1536]] * 4)
    assert ((ids == 10).sum(dim=1) == 1536).all()
    # one contiguous run per sequence
    for s in range(4):
        pos = torch.nonzero(ids[s] == 10).reshape(-1)
        assert int(pos[-1] - pos[0]) == 1535


# ---------------------------------------------------------------------------
# FLOP counter: closed form of the config-2 total
# ---------------------------------------------------------------------------

def test_flop_count_closed_form():
    total = O.flops(O.MISTRAL3, [(110, 110)])
    t, d, f = 12100, 1024, 4096
    tower = 24 * (t * 2 * (4 * d * d + 3 * d * f) + 4 * t * t * d)
    assert total == pytest.approx(tower + t * 2 * 588 * d + 3025 * 2 * (4096 * d + d * 5120 + 5120 * 5120), rel=1e-15)
    assert total == pytest.approx(2.437e13, rel=2e-3)


# ---------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the pins above
# ---------------------------------------------------------------------------

def test_planted_rope_sign_error_is_caught(monkeypatch):
    def bad(x, angles):
        half = x.shape[-1] // 2
        cos, sin = np.cos(angles)[:, None, :], np.sin(angles)[:, None, :]
        a, b = x[..., :half], x[..., half:]
        return np.concatenate([a * cos + b * sin, b * cos + a * sin], axis=-1)
    monkeypatch.setattr(O, "apply_rope", bad)
    with pytest.raises(AssertionError):
        test_rope_preserves_norm_and_origin_is_identity()


def test_planted_missing_attention_scale_is_caught(monkeypatch):
    orig = O.attention

    def bad(q, k, v, cu):
        return orig(np.asarray(q) * 8.0, k, v, cu)
    monkeypatch.setattr(O, "attention", bad)
    with pytest.raises(AssertionError):
        test_attention_matches_sdpa_block_diagonal()


def test_planted_merge_order_swap_is_caught(monkeypatch):
    def bad(x, grids, merge):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[1]
        out, off = [], 0
        for h, w in grids:
            hm, wm = h // merge, w // merge
            img = x[off:off + h * w].reshape(hm, merge, wm, merge, d)
            out.append(img.transpose(0, 2, 4, 3, 1).reshape(hm * wm, d * merge * merge))  # dx, dy swapped
            off += h * w
        return np.concatenate(out, axis=0)
    monkeypatch.setattr(O, "merge_unfold", bad)
    with pytest.raises(AssertionError):
        test_merge_matches_torch_unfold()


def test_planted_rope_frequency_split_swap_is_caught(monkeypatch):
    orig = O.rope_angles

    def bad(rows, cols, theta, head_dim):
        return orig(cols, rows, theta, head_dim)
    monkeypatch.setattr(O, "rope_angles", bad)
    with pytest.raises(AssertionError):
        test_rope_frequencies_closed_form()


# ---------------------------------------------------------------------------
# Front end: resize onto the grid, tiling, placeholder expansion
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("hw,expect", [((1540, 1540), (1540, 1540)), ((3080, 1540), (1540, 784)),
                                       ((100, 50), (112, 56)), ((2000, 1000), (1540, 784)), ((27, 3000), (28, 1540))])
def test_resized_hw_closed_form(hw, expect):
    assert O.resized_hw(*hw, 1540, 28) == expect
    h, w = O.resized_hw(*hw, 1540, 28)
    assert h % 28 == 0 and w % 28 == 0 and max(h, w) <= 1540


def test_resized_hw_rejects_longest_edge_off_the_grid():
    """With longest_edge not a multiple of the grid, rounding a side up could
    carry it past longest_edge: rejected instead."""
    with pytest.raises(ValueError):
        O.resized_hw(2000, 1000, 1000, 28)
    assert O.resized_hw(2000, 1000, 1008, 28) == (1008, 504)


@pytest.mark.parametrize("src,dst", [((13, 17), (28, 56)), ((64, 48), (28, 28)), ((5, 5), (5, 5))])
def test_resize_bilinear_matches_torch_interpolate(src, dst):
    img = RNG.random((3, *src))
    ref = F.interpolate(torch.from_numpy(img)[None], size=dst, mode="bilinear", align_corners=False,
                        antialias=False)[0].numpy()
    np.testing.assert_allclose(O.resize_bilinear(img, *dst), ref, rtol=1e-12, atol=1e-12)


def test_resize_identity_and_constant():
    img = RNG.random((3, 7, 9))
    np.testing.assert_allclose(O.resize_bilinear(img, 7, 9), img, rtol=0, atol=1e-15)
    const = np.full((3, 5, 6), 0.25)
    np.testing.assert_allclose(O.resize_bilinear(const, 28, 14), 0.25, rtol=0, atol=1e-15)


def test_tile_image_round_trip_and_count():
    img = RNG.random((3, 8, 12))
    tiles = O.tile_image(img, 4)
    assert len(tiles) == 6
    back = np.concatenate([np.concatenate(tiles[r * 3:(r + 1) * 3], axis=2) for r in range(2)], axis=1)
    np.testing.assert_array_equal(back, img)
    with pytest.raises(ValueError):
        O.tile_image(np.zeros((3, 10, 8)), 4)


def test_expand_placeholders_definition():
    ids = np.array([1, 2, 99, 3, 99, 4])
    got = O.expand_placeholders(ids, 99, [3, 1], 10)
    assert got.tolist() == [1, 2, 10, 10, 10, 3, 10, 4]
    assert O.expand_placeholders(np.array([5, 6]), 99, [], 10).tolist() == [5, 6]
    with pytest.raises(ValueError):
        O.expand_placeholders(ids, 99, [3], 10)
    # the pages' count: one 896x1344 image is 1,536 placeholders
    h, w = O.merged_grid(*O.patch_grid(896, 1344, 14), 2)
    assert int((O.expand_placeholders(np.array([7, 99, 8]), 99, [h * w], 10) == 10).sum()) == 1536


def test_pixels_from_u8_layout_and_scale():
    img = np.zeros((2, 3, 3), dtype=np.uint8)
    img[1, 2] = (255, 0, 51)   # pixel at row 1, column 2
    x = O.pixels_from_u8(img)
    assert x.shape == (3, 2, 3)
    assert x[0, 1, 2] == 1.0 and x[1, 1, 2] == 0.0 and x[2, 1, 2] == pytest.approx(0.2, abs=1e-15)
    assert np.count_nonzero(x) == 2


# ---------------------------------------------------------------------------
# FP8 (E4M3) tower GEMMs
# ---------------------------------------------------------------------------

def _e4m3_codes():
    """All finite E4M3 values from the bit layout s.eeee.mmm (bias 7, code 0x7F/0xFF are NaN)."""
    vals = []
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e, m = (code >> 3) & 0xF, code & 7
        if e == 15 and m == 7:
            continue
        vals.append(sign * (m / 8.0) * 2.0 ** -6 if e == 0 else sign * (1 + m / 8.0) * 2.0 ** (e - 7))
    return np.unique(np.array(vals))


def test_e4m3_codes_are_fixed_points_and_range():
    codes = _e4m3_codes()
    assert codes.max() == 448.0 and codes.min() == -448.0
    assert len(codes) == 253  # 254 finite codes, +0 and -0 collapse
    np.testing.assert_array_equal(O.e4m3_round(codes), codes)


def test_e4m3_midpoints_round_to_even_mantissa():
    pos = _e4m3_codes()
    pos = pos[pos >= 0]
    mids = (pos[:-1] + pos[1:]) / 2
    got = O.e4m3_round(mids)
    for lo, hi, g in zip(pos[:-1], pos[1:], got):
        # the even neighbour has an even mantissa field: its value / quantum is even
        _, e = np.frexp(lo if lo > 0 else hi)
        q = 2.0 ** (max(min(e - 1, 8), -6) - 3)
        even = lo if round(lo / q) % 2 == 0 else hi
        assert g == even, (lo, hi, g)


def test_e4m3_matches_torch_float8_and_saturates():
    rng = np.random.default_rng(8)
    mag = np.exp2(rng.uniform(-12, np.log2(460), 200000))
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3_round(x), ref)
    np.testing.assert_array_equal(O.e4m3_round([464.0001, 1e6, -1e30]), [448.0, 448.0, -448.0])
    assert np.isnan(O.e4m3_round([np.nan]))[0]


def test_quantize_weight_rows_scale_and_error_bound():
    w = RNG.standard_normal((16, 96)).astype(np.float32) * 0.02
    w[3] = 0.0
    q, s = O.quantize_weight_rows(w)
    assert s.dtype == np.float32 and s[3] == 1.0 and np.all(q[3] == 0)
    amax_idx = np.argmax(np.abs(w), axis=1)
    for n in range(16):
        if n != 3:
            assert abs(q[n, amax_idx[n]]) == 448.0
    rec = q * s[:, None].astype(np.float64)
    normal = np.abs(w) >= 2.0 ** -6 * s[:, None]
    assert np.all(np.abs(rec - w)[normal] <= np.abs(w)[normal] * 2.0 ** -4 * (1 + 1e-6))


def test_fp8_linear_exact_on_representable_inputs():
    """With activations on the scaled E4M3 grid and a power-of-two scale the
    activation quantisation is exact, so fp8_linear equals a plain matmul with
    the dequantised weights."""
    codes = _e4m3_codes()
    a = RNG.choice(codes[np.abs(codes) <= 64], size=(5, 32)) * 0.25
    w = RNG.standard_normal((7, 32)) * 0.05
    q_w, s_w = O.quantize_weight_rows(w)
    got = O.fp8_linear(a, q_w, s_w, 0.25)
    ref = (a / 0.25) @ q_w.T * (np.float32(0.25) * s_w.astype(np.float32)).astype(np.float64)[None, :]
    np.testing.assert_allclose(got, ref, rtol=1e-15, atol=0)
    np.testing.assert_allclose(got, a @ (q_w * s_w[:, None].astype(np.float64)).T, rtol=1e-12, atol=1e-15)


def test_tower_block_fp8_close_to_bf16_block():
    """The E4M3 block stays within E4M3's quantisation error of the exact block
    and differs from it (the quantisation is really applied)."""
    t, d, f = 24, 64, 128
    cfg = dict(O.MISTRAL3, width=d, heads=1, mlp=f)
    lw = {n: RNG.standard_normal(sh) * 0.05 for n, sh in
          (("wq", (d, d)), ("wk", (d, d)), ("wv", (d, d)), ("wo", (d, d)), ("w_gate", (f, d)), ("w_up", (f, d)),
           ("w_down", (d, f)))}
    lw["g_attn"] = 1 + 0.02 * RNG.standard_normal(d)
    lw["g_ffn"] = 1 + 0.02 * RNG.standard_normal(d)
    x = RNG.standard_normal((t, d))
    rows, cols, cu = O.positions([(4, 6)])
    ang = O.rope_angles(rows, cols, 1e4, d)
    exact = O.tower_block(x, lw, ang, cu, cfg)
    fp8 = O.tower_block_fp8(x, O.quantize_layer(lw), (8 / 448, 4 / 448, 8 / 448, 8 / 448), ang, cu, cfg)
    err = np.abs(fp8 - exact).max() / np.abs(exact).max()
    assert 1e-4 < err < 5e-2, err


def test_planted_fp8_missing_weight_scale_is_caught(monkeypatch):
    def bad(a, q_w, s_w, s_a):
        inv = np.float32(1.0 / np.float64(np.float32(s_a)))
        q_a = O.e4m3_round(np.asarray(a, dtype=np.float32) * inv)
        return (q_a @ np.asarray(q_w, dtype=np.float64).T) * np.float64(s_a)  # per-row weight scale dropped
    monkeypatch.setattr(O, "fp8_linear", bad)
    with pytest.raises(AssertionError):
        test_fp8_linear_exact_on_representable_inputs()


def test_planted_e4m3_truncation_is_caught(monkeypatch):
    def bad(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        _, e = np.frexp(a)
        q = np.ldexp(1.0, (np.clip(e - 1, -6, 8) - 3).astype(np.int64))
        return np.copysign(np.minimum(np.floor(a / q) * q, 448.0), x)  # rounds toward zero
    monkeypatch.setattr(O, "e4m3_round", bad)
    with pytest.raises(AssertionError):
        test_e4m3_matches_torch_float8_and_saturates()


@pytest.mark.parametrize("after", [False, True])
def test_projector_both_norm_orders_match_torch_composition(after):
    """The projector in either reading of the norm's place equals the same
    steps written with torch (rms_norm, unfold, linear, exact GELU)."""
    d, e = 8, 12
    grids = [(4, 6), (2, 2)]
    x = RNG.standard_normal((28, d))
    pw = {"g_proj": 1 + 0.1 * RNG.standard_normal(d), "w_merge": RNG.standard_normal((d, 4 * d)) * 0.3,
          "w1": RNG.standard_normal((e, d)) * 0.3, "w2": RNG.standard_normal((e, e)) * 0.3}
    cfg = dict(O.MISTRAL3, eps=1e-5, merge=2, norm_after_merge=after)
    got = O.projector(x, grids, pw, cfg)
    t = {k: torch.from_numpy(v) for k, v in pw.items()}
    xt = torch.from_numpy(x)
    if not after:
        xt = F.rms_norm(xt, (d,), t["g_proj"], eps=1e-5)
    zs, off = [], 0
    for h, w in grids:
        img = xt[off:off + h * w].reshape(h, w, d).permute(2, 0, 1)[None]
        zs.append(F.unfold(img, kernel_size=2, stride=2)[0].T)
        off += h * w
    y = torch.cat(zs) @ t["w_merge"].T
    if after:
        y = F.rms_norm(y, (d,), t["g_proj"], eps=1e-5)
    ref = F.gelu(y @ t["w1"].T, approximate="none") @ t["w2"].T
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)
    other = O.projector(x, grids, pw, dict(cfg, norm_after_merge=not after))
    assert np.abs(other - got).max() > 1e-3  # the two readings really differ
    # with merge 1 the flag changes nothing
    cfg1 = dict(cfg, merge=1)
    np.testing.assert_array_equal(O.projector(x, [(28, 1)], pw, cfg1), O.projector(x, [(28, 1)], pw, dict(cfg1, norm_after_merge=not after)))


def test_tower_block_fp8_scales_feed_the_right_gemms():
    """Each static scale belongs to one GEMM input: a tiny scale saturates that
    input to +-448 s, which all but removes that GEMM's contribution. With the
    attention-output scale tiny the block equals the exact block without its
    O projection (Wo = 0); with the hidden-state scale tiny, without its MLP
    (W_down = 0); with either norm-output scale tiny the matching GEMMs see
    inputs of size 448 s and their outputs shrink the same way."""
    t, d, f = 12, 64, 128
    cfg = dict(O.MISTRAL3, width=d, heads=1, mlp=f)
    rng = np.random.default_rng(21)
    lw = {n: rng.standard_normal(sh) * 0.05 for n, sh in
          (("wq", (d, d)), ("wk", (d, d)), ("wv", (d, d)), ("wo", (d, d)), ("w_gate", (f, d)), ("w_up", (f, d)),
           ("w_down", (d, f)))}
    lw["g_attn"] = np.ones(d)
    lw["g_ffn"] = np.ones(d)
    x = rng.standard_normal((t, d))
    rows, cols, cu = O.positions([(3, 4)])
    ang = O.rope_angles(rows, cols, 1e4, d)
    lq = O.quantize_layer(lw)
    ok = (8 / 448, 4 / 448, 8 / 448, 16 / 448)
    tiny = 1e-9
    no_o = O.tower_block(x, dict(lw, wo=np.zeros((d, d))), ang, cu, cfg)
    no_mlp = O.tower_block(x, dict(lw, w_down=np.zeros((d, f))), ang, cu, cfg)
    exact = O.tower_block(x, lw, ang, cu, cfg)

    def rel(a, b):
        return np.abs(a - b).max() / np.abs(b).max()

    # attention output crushed: the O projection adds ~0, the MLP then sees x (not x + attention)
    got = O.tower_block_fp8(x, lq, (ok[0], tiny, ok[2], ok[3]), ang, cu, cfg)
    xo = x.copy()
    ref = xo + (O.silu(O.rms_norm(xo, lw["g_ffn"], 1e-5) @ lw["w_gate"].T) *
                (O.rms_norm(xo, lw["g_ffn"], 1e-5) @ lw["w_up"].T)) @ lw["w_down"].T
    assert rel(got, ref) < 5e-2 and rel(got, exact) > rel(got, ref)
    # hidden state crushed: the block is x + attention only
    got = O.tower_block_fp8(x, lq, (ok[0], ok[1], ok[2], tiny), ang, cu, cfg)
    assert rel(got, no_mlp) < 5e-2 and rel(got, exact) > rel(got, no_mlp)
    # MLP-norm output crushed: gate and up see ~0, so the MLP adds ~0 as well
    got = O.tower_block_fp8(x, lq, (ok[0], ok[1], tiny, ok[3]), ang, cu, cfg)
    assert rel(got, no_mlp) < 5e-2
    # attention-norm output crushed: q, k, v ~0, so attention (and the O projection) add ~0
    got = O.tower_block_fp8(x, lq, (tiny, ok[1], ok[2], ok[3]), ang, cu, cfg)
    assert rel(got, ref) < 5e-2
    assert no_o.shape == got.shape


# ---------------------------------------------------------------------------
# NVFP4 (E2M1 values, E4M3 scale per 16, fp32 global scale)
# ---------------------------------------------------------------------------

def _e2m1_codes():
    """The 16 E2M1 codes decoded from the bit layout s.ee.m (bias 1; e = 0 is subnormal: m * 0.5)."""
    out = []
    for code in range(16):
        sign = -1.0 if code & 8 else 1.0
        e, m = (code >> 1) & 3, code & 1
        out.append((code, sign * (0.5 * m if e == 0 else (1 + m / 2.0) * 2.0 ** (e - 1))))
    return out


def _e2m1_brute(x):
    """Nearest code by exhaustive search; a tie goes to the code whose mantissa bit is 0."""
    res = np.empty(len(x))
    codes = _e2m1_codes()
    for i, v in enumerate(x):
        if v > 6.0 or v < -6.0:
            res[i] = math.copysign(6.0, v)
            continue
        best = min(abs(v - c) for _, c in codes)
        cands = [(code, c) for code, c in codes if abs(v - c) == best]
        even = [c for code, c in cands if code & 1 == 0]
        res[i] = even[0] if even else cands[0][1]
    return res


def test_e2m1_grid_fixed_points_and_range():
    vals = np.unique([c for _, c in _e2m1_codes()])
    np.testing.assert_array_equal(vals, [-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(O.e2m1_round(vals), vals)


def test_e2m1_round_matches_brute_force_and_ties_to_even():
    rng = np.random.default_rng(41)
    grid = np.unique([abs(c) for _, c in _e2m1_codes()])
    mids = (grid[:-1] + grid[1:]) / 2
    x = np.concatenate([rng.uniform(-7.5, 7.5, 20000), mids, -mids, [6.0, 6.5, 1e9, -1e9, 0.0]])
    np.testing.assert_array_equal(O.e2m1_round(x), _e2m1_brute(x))
    # the ties, spelled out: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    np.testing.assert_array_equal(O.e2m1_round(mids), [0, 1, 1, 2, 2, 4, 4])
    assert np.isnan(O.e2m1_round([np.nan]))[0]


def _nvfp4_representable(rows, k, rng, s_g):
    """Codes on the grid, a +-6 in every block, power-of-two block scales: x = q s_b s_g exactly."""
    q = rng.choice([c for _, c in _e2m1_codes()], size=(rows, k))
    q[:, ::16] = rng.choice([-6.0, 6.0], size=(rows, k // 16))
    s_b = np.exp2(rng.integers(-6, 8, size=(rows, k // 16))).astype(np.float64)
    return q * np.repeat(s_b, 16, axis=1) * s_g, q, s_b


def test_quantize_nvfp4_exact_on_representable_input():
    rng = np.random.default_rng(42)
    s_g = 2.0 ** -5
    x, q, s_b = _nvfp4_representable(6, 96, rng, s_g)
    got_q, got_s = O.quantize_nvfp4(x, s_g)
    np.testing.assert_array_equal(got_s, s_b)
    np.testing.assert_array_equal(got_q, q)
    np.testing.assert_array_equal(O.dequantize_nvfp4(got_q, got_s, s_g), x)


def test_quantize_nvfp4_zero_block_and_error_bound():
    rng = np.random.default_rng(43)
    x = (rng.standard_normal((40, 128)) * np.exp2(rng.uniform(-3, 3, (40, 1)))).astype(np.float32)
    x[5, 16:32] = 0.0
    s_g = O.nvfp4_global_scale(x)
    q, s_b = O.quantize_nvfp4(x, s_g)
    assert s_b[5, 1] == 0 and np.all(q[5, 16:32] == 0) and np.all(np.isfinite(q))
    # the block holding the tensor's largest magnitude takes the largest scale
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert s_b[r, c // 16] == 448.0
    # every nonzero block's largest value lands on +-6
    blocks = np.abs(x).reshape(40, 8, 16)
    top = np.argmax(blocks, axis=2)
    qb = np.abs(q).reshape(40, 8, 16)
    live = s_b > 2.0 ** -6   # normal E4M3 scales (relative step 1/16)
    assert np.all(np.take_along_axis(qb, top[:, :, None], 2)[:, :, 0][live] == 6.0)
    # elementwise: within half an E2M1 step of x / s (s = s_b s_g), where the block scale is normal
    s = np.repeat(s_b * np.float64(s_g), 16, axis=1)
    y = x / np.where(s > 0, s, 1)
    err = np.abs(O.dequantize_nvfp4(q, s_b, s_g) - x)
    bound = s * np.maximum(0.25, np.abs(y) / 4) * (1 + 1e-6)
    ok = np.repeat(live, 16, axis=1)
    assert np.all(err[ok] <= bound[ok])


def test_nvfp4_linear_exact_against_fractions():
    """Brute force with exact rationals on a small case."""
    from fractions import Fraction
    rng = np.random.default_rng(44)
    xa, qa, sa = _nvfp4_representable(3, 64, rng, 2.0 ** -4)
    xw, qw, sw = _nvfp4_representable(4, 64, rng, 2.0 ** -7)
    got = O.nvfp4_linear(qa, sa, 2.0 ** -4, qw, sw, 2.0 ** -7)
    for i in range(3):
        for j in range(4):
            acc = sum(Fraction(qa[i, k]) * Fraction(sa[i, k // 16]) * Fraction(qw[j, k]) * Fraction(sw[j, k // 16])
                      for k in range(64))
            assert Fraction(got[i, j]) == acc * Fraction(2.0 ** -4) * Fraction(2.0 ** -7)
    np.testing.assert_array_equal(got, xa @ xw.T)


def test_planted_e2m1_round_half_up_is_caught(monkeypatch):
    def bad(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        _, e = np.frexp(a)
        quantum = np.ldexp(1.0, (np.clip(e - 1, 0, 2) - 1).astype(np.int64))
        return np.copysign(np.minimum(np.floor(a / quantum + 0.5) * quantum, 6.0), x)
    monkeypatch.setattr(O, "e2m1_round", bad)
    with pytest.raises(AssertionError):
        test_e2m1_round_matches_brute_force_and_ties_to_even()


def test_planted_nvfp4_block_of_32_is_caught(monkeypatch):
    def bad(x, s_global):
        x = np.asarray(x, dtype=np.float32)
        r_, k_ = x.shape
        # one scale per 32 values: each pair of blocks shares the larger scale
        blocks = np.abs(x).reshape(r_, k_ // 32, 32).max(axis=2)
        s32 = O.e4m3_round((blocks / np.float32(6 * np.float32(s_global))).astype(np.float32))
        s_b = np.repeat(s32, 2, axis=1)
        recip = np.where(s_b > 0, 1.0 / np.where(s_b > 0, s_b * np.float64(s_global), 1.0), 0.0)
        return O.e2m1_round(x * np.repeat(recip, 16, axis=1)), s_b
    monkeypatch.setattr(O, "quantize_nvfp4", bad)
    with pytest.raises(AssertionError):
        test_quantize_nvfp4_exact_on_representable_input()


def test_planted_nvfp4_missing_global_scale_is_caught(monkeypatch):
    def bad(q_a, s_a, g_a, q_w, s_w, g_w):
        a = np.asarray(q_a) * np.repeat(s_a, 16, axis=1)
        w = np.asarray(q_w) * np.repeat(s_w, 16, axis=1)
        return (a @ w.T) * np.float64(g_a)  # the weights' global scale dropped
    monkeypatch.setattr(O, "nvfp4_linear", bad)
    with pytest.raises(AssertionError):
        test_nvfp4_linear_exact_against_fractions()


def _small_layer(rng, d=64, f=128, gains_one=False):
    lw = {n: rng.standard_normal(sh) * 0.05 for n, sh in
          (("wq", (d, d)), ("wk", (d, d)), ("wv", (d, d)), ("wo", (d, d)), ("w_gate", (f, d)), ("w_up", (f, d)),
           ("w_down", (d, f)))}
    lw["g_attn"] = np.ones(d) if gains_one else 1 + 0.02 * rng.standard_normal(d)
    lw["g_ffn"] = np.ones(d) if gains_one else 1 + 0.02 * rng.standard_normal(d)
    return lw


NVFP4_ACT = (8 / 2688, 4 / 2688, 8 / 2688, 16 / 2688)


def test_quantize_layer_nvfp4_one_global_scale_per_executed_gemm():
    rng = np.random.default_rng(71)
    lw = _small_layer(rng)
    lq = O.quantize_layer_nvfp4(lw)
    qkv = np.concatenate([lw["wq"], lw["wk"], lw["wv"]]).astype(np.float32)
    q, sb, g = lq["qkv"]
    assert g == O.nvfp4_global_scale(qkv) and q.shape == qkv.shape and sb.shape == (192, 4)
    # the fused tensor's largest block takes scale 448, and every value is within half an E2M1 step
    # of its block's grid (scale s = s_b s_g per block of 16)
    assert sb.max() == 448.0
    s_full = np.repeat(sb * np.float64(g), 16, axis=1)
    err = np.abs(O.dequantize_nvfp4(q, sb, g) - qkv)
    assert np.all(err <= s_full * np.maximum(0.25, np.abs(qkv) / s_full / 4) * (1 + 1e-6))


def test_tower_block_nvfp4_close_to_exact_block():
    """The NVFP4 block stays within NVFP4's quantisation error of the exact block
    and differs from it (the quantisation is really applied)."""
    rng = np.random.default_rng(72)
    d = 64
    cfg = dict(O.MISTRAL3, width=d, heads=1, mlp=128)
    lw = _small_layer(rng)
    x = rng.standard_normal((24, d))
    rows, cols, cu = O.positions([(4, 6)])
    ang = O.rope_angles(rows, cols, 1e4, d)
    exact = O.tower_block(x, lw, ang, cu, cfg)
    fp4 = O.tower_block_nvfp4(x, O.quantize_layer_nvfp4(lw), NVFP4_ACT, ang, cu, cfg)
    err = np.abs(fp4 - exact).max() / np.abs(exact).max()
    assert 1e-3 < err < 0.15, err


def test_tower_block_nvfp4_scales_feed_the_right_gemms():
    """A tiny global scale saturates every block of that GEMM input to +-6 at
    scale 448, i.e. +-2688 g: the input all but vanishes. With the attention-
    output scale tiny the block equals the exact block without its O projection;
    with the hidden-state scale tiny, without its MLP; with the attention-norm
    scale tiny, q = k = v ~ 0 and the attention output vanishes as well; with the
    MLP-norm scale tiny, gate and up vanish and so does the MLP."""
    rng = np.random.default_rng(73)
    d, f = 64, 128
    cfg = dict(O.MISTRAL3, width=d, heads=1, mlp=f)
    lw = _small_layer(rng, gains_one=True)
    x = rng.standard_normal((12, d))
    rows, cols, cu = O.positions([(3, 4)])
    ang = O.rope_angles(rows, cols, 1e4, d)
    lq = O.quantize_layer_nvfp4(lw)
    no_o = O.tower_block(x, dict(lw, wo=np.zeros((d, d))), ang, cu, cfg)
    no_mlp = O.tower_block(x, dict(lw, w_down=np.zeros((d, f))), ang, cu, cfg)
    exact = O.tower_block(x, lw, ang, cu, cfg)

    def rel(a, b):
        return np.abs(a - b).max() / np.abs(b).max()

    tiny = 1e-12
    for i, ref in ((0, no_o), (1, no_o), (2, no_mlp), (3, no_mlp)):
        act = list(NVFP4_ACT)
        act[i] = tiny
        got = O.tower_block_nvfp4(x, lq, act, ang, cu, cfg)
        assert rel(got, ref) < 0.1, (i, rel(got, ref))
        assert rel(got, exact) > 3 * rel(got, ref), (i, rel(got, exact), rel(got, ref))


def test_planted_nvfp4_act_scales_swapped_is_caught(monkeypatch):
    real = O.tower_block_nvfp4

    def bad(x, lq, act, angles, cu, cfg):
        a = list(act)
        a[1], a[3] = a[3], a[1]   # the attention-output and hidden-state scales exchanged
        return real(x, lq, a, angles, cu, cfg)
    monkeypatch.setattr(O, "tower_block_nvfp4", bad)
    with pytest.raises(AssertionError):
        test_tower_block_nvfp4_scales_feed_the_right_gemms()


def _identity_nvfp4(monkeypatch):
    """Quantisation switched off: codes = the fp32 values, every scale 1."""
    monkeypatch.setattr(O, "quantize_nvfp4",
                        lambda x, g: (np.asarray(x, np.float32).astype(np.float64),
                                      np.ones((np.shape(x)[0], np.shape(x)[1] // 16))))
    monkeypatch.setattr(O, "nvfp4_global_scale", lambda w: np.float32(1.0))


def _nvfp4_tower_setup():
    cfg = dict(O.MISTRAL3, layers=2, width=64, heads=1, head_dim=64, mlp=128)
    tw = {k: v.double().numpy() for k, v in synth.tower_weights(4, 2, 64, 128, 14).items()}
    imgs = [synth.pixels_u01(4, f"nvfp4tower{i}", h, w).double().numpy()
            for i, (h, w) in enumerate([(28, 42), (14, 28)])]
    return cfg, tw, imgs


def test_tower_nvfp4_without_quantisation_is_the_tower(monkeypatch):
    """With quantisation switched off (codes = the fp32 values, unit block and
    global scales) tower_nvfp4 must be the pinned tower() -- same patch embed,
    ln_pre, blocks and positions -- up to the fp32 rounding of each GEMM input;
    with it on, it must differ by NVFP4's error and no more."""
    cfg, tw, imgs = _nvfp4_tower_setup()
    ref = O.tower(imgs, tw, cfg)
    quant = O.tower_nvfp4(imgs, tw, [NVFP4_ACT] * 2, cfg)
    err_q = np.abs(quant - ref).max() / np.abs(ref).max()
    assert 1e-3 < err_q < 0.2, err_q
    _identity_nvfp4(monkeypatch)
    got = O.tower_nvfp4(imgs, tw, [(1.0, 1.0, 1.0, 1.0)] * 2, cfg)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-5 * np.abs(ref).max())


def test_planted_nvfp4_tower_without_ln_pre_is_caught(monkeypatch):
    cfg, tw, imgs = _nvfp4_tower_setup()
    ref = O.tower(imgs, tw, cfg)
    _identity_nvfp4(monkeypatch)
    g_pre = tw["g_pre"]
    real = O.rms_norm
    monkeypatch.setattr(O, "rms_norm", lambda x, g, eps: np.asarray(x, np.float64) if g is g_pre else real(x, g, eps))
    got = O.tower_nvfp4(imgs, tw, [(1.0, 1.0, 1.0, 1.0)] * 2, cfg)
    assert np.abs(got - ref).max() > 1e-2 * np.abs(ref).max()
