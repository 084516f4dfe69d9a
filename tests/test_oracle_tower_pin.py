"""Independent pin of the oracle's tower composition.

The leaf functions of the oracle are pinned one by one elsewhere. This file
pins how they are put together: the vision tower as "Mistral 3"
(KerasFormers), API table `Mistral3VisionModel`, describes it -- a convolution
as the patch embed, an RMS pre-norm, then blocks with 2D rotary attention over
a packed sequence of images -- rebuilt here from torch primitives in that
order, by another route for every step:

* the patch embed is `F.conv2d` with kernel = stride = patch;
* `ln_pre` and the two pre-norms of every block are `F.rms_norm`;
* 2D RoPE is a complex rotation: pair (x_i, x_{i+32}) is the complex number
  x_i + j x_{i+32}, multiplied by exp(j phi_i) (`torch.polar`), with phi from
  the row index for the even frequencies and from the column index for the odd;
* attention is `F.scaled_dot_product_attention` with a block-diagonal mask;
* the MLP gate is `F.silu`, and every linear is `F.linear`;
* the projector is `F.unfold` + `F.linear` + `F.gelu`.

The oracle and this composition must agree to rounding on a 2-layer packed
batch of three images. Three plausible composition mistakes are planted into
the oracle (on the CPU) and each one must break that agreement.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import vlm_oracle as O
from vision_language_model_b200 import synth

SIZES = [(28, 42), (14, 28), (42, 28)]   # patch grids 2x3, 1x2, 3x2 at patch 14
WIDTH, HEADS, HEAD_DIM, MLP, LAYERS = 128, 2, 64, 256, 2


def _setup(seed=0):
    """Weights with strongly non-unit gains and peaked q/k, so a swapped gain
    or a mis-rotated operand moves the output far beyond rounding."""
    cfg = dict(O.MISTRAL3, layers=LAYERS, width=WIDTH, heads=HEADS, head_dim=HEAD_DIM, mlp=MLP)
    tw = {k: v.double().numpy().copy() for k, v in synth.tower_weights(seed, LAYERS, WIDTH, MLP, 14).items()}
    rng = np.random.default_rng(seed + 77)
    for name in ("g_pre", "g_attn", "g_ffn"):
        tw[name] = 1.0 + 0.5 * rng.standard_normal(tw[name].shape)
    tw["wq"] = tw["wq"] * 6.0
    tw["wk"] = tw["wk"] * 6.0
    tw["w_down"] = tw["w_down"] * 4.0
    imgs = [synth.pixels_u01(seed, f"towerpin{i}", h, w).double().numpy() for i, (h, w) in enumerate(SIZES)]
    return cfg, tw, imgs


def _torch_rope(x, rows, cols, theta):
    """x [T, H, 64]; rotation of pair (i, i+32) as a complex product."""
    half = x.shape[-1] // 2
    inv = theta ** (-torch.arange(0, x.shape[-1], 2, dtype=torch.float64) / x.shape[-1])  # 32 frequencies
    phi = torch.cat([rows[:, None] * inv[0::2][None, :], cols[:, None] * inv[1::2][None, :]], dim=1)  # [T, 32]
    z = torch.complex(x[..., :half], x[..., half:]) * torch.polar(torch.ones_like(phi), phi)[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def _torch_tower(imgs, tw, cfg):
    """The tower in the page's order, from torch primitives only."""
    p, d, heads, dh, eps = cfg["patch"], cfg["width"], cfg["heads"], cfg["head_dim"], cfg["eps"]
    t = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in tw.items()}
    mean = torch.tensor((0.48145466, 0.4578275, 0.40821073), dtype=torch.float64)[:, None, None]
    std = torch.tensor((0.26862954, 0.26130258, 0.27577711), dtype=torch.float64)[:, None, None]
    feats, rows, cols, blocks = [], [], [], []
    for im in imgs:
        x = (torch.from_numpy(im) - mean) / std
        y = F.conv2d(x[None], t["w_pe"], stride=p)[0]            # [D, h, w]
        h, w = y.shape[1:]
        feats.append(y.permute(1, 2, 0).reshape(h * w, d))
        rows.append(torch.arange(h, dtype=torch.float64).repeat_interleave(w))
        cols.append(torch.arange(w, dtype=torch.float64).repeat(h))
        blocks.append(h * w)
    x = F.rms_norm(torch.cat(feats), (d,), t["g_pre"], eps=eps)
    rows, cols = torch.cat(rows), torch.cat(cols)
    n = x.shape[0]
    mask = torch.block_diag(*[torch.ones(b, b, dtype=torch.bool) for b in blocks])
    for layer in range(cfg["layers"]):
        xn = F.rms_norm(x, (d,), t["g_attn"][layer], eps=eps)
        q = _torch_rope(F.linear(xn, t["wq"][layer]).view(n, heads, dh), rows, cols, cfg["rope_theta"])
        k = _torch_rope(F.linear(xn, t["wk"][layer]).view(n, heads, dh), rows, cols, cfg["rope_theta"])
        v = F.linear(xn, t["wv"][layer]).view(n, heads, dh)
        o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1), attn_mask=mask)
        x = x + F.linear(o.transpose(0, 1).reshape(n, heads * dh), t["wo"][layer])
        xn = F.rms_norm(x, (d,), t["g_ffn"][layer], eps=eps)
        x = x + F.linear(F.silu(F.linear(xn, t["w_gate"][layer])) * F.linear(xn, t["w_up"][layer]), t["w_down"][layer])
    return x.numpy()


def _torch_projector(x, grids, pw, cfg):
    d, m, eps = cfg["width"], cfg["merge"], cfg["eps"]
    t = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in pw.items()}
    xn = F.rms_norm(torch.from_numpy(x), (d,), t["g_proj"], eps=eps)
    zs, off = [], 0
    for h, w in grids:
        zs.append(F.unfold(xn[off:off + h * w].reshape(h, w, d).permute(2, 0, 1)[None], kernel_size=m, stride=m)[0].T)
        off += h * w
    y = F.linear(torch.cat(zs), t["w_merge"])
    return F.linear(F.gelu(F.linear(y, t["w1"]), approximate="none"), t["w2"]).numpy()


def _close(a, b):
    return np.abs(a - b).max() <= 1e-12 * max(1.0, np.abs(b).max())


def test_tower_equals_torch_composition():
    cfg, tw, imgs = _setup()
    got = O.tower(imgs, tw, cfg)
    ref = _torch_tower(imgs, tw, cfg)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.abs(ref).max() > 1.0  # the blocks did real work


def test_encode_merge_project_equals_torch_composition():
    """Tower then projector (per-patch RMSNorm, 2x2 unfold, merge linear,
    W1, GELU, W2) on grids that merge evenly: 2x4, 2x2 and 4x2 patches."""
    cfg, tw, _ = _setup(seed=3)
    sizes = [(28, 56), (28, 28), (56, 28)]
    pw = {k: v.double().numpy() for k, v in synth.projector_weights(3, WIDTH, 2, 96).items()}
    imgs = [synth.pixels_u01(3, f"empin{i}", h, w).double().numpy() for i, (h, w) in enumerate(sizes)]
    grids = [(h // 14, w // 14) for h, w in sizes]
    xt, y = O.encode_merge_project(imgs, tw, pw, cfg)
    ref_t = _torch_tower(imgs, tw, cfg)
    np.testing.assert_allclose(xt, ref_t, rtol=1e-12, atol=1e-12 * np.abs(ref_t).max())
    ref_y = _torch_projector(ref_t, grids, pw, cfg)
    np.testing.assert_allclose(y, ref_y, rtol=1e-11, atol=1e-12 * np.abs(ref_y).max())
    assert y.shape == (2 + 1 + 2, 96)


def test_torch_rope_matches_pinned_pairing_on_one_vector():
    """The complex rotation above is the pairing the pages' reading fixes:
    position (r, c) = (1, 0) turns pair 0 by 1 rad (w_0 = 1) and pair 16
    (the first column frequency, w_1) not at all."""
    x = torch.zeros(1, 1, 64, dtype=torch.float64)
    x[0, 0, 0] = 1.0
    x[0, 0, 16] = 1.0
    y = _torch_rope(x, torch.tensor([1.0], dtype=torch.float64), torch.tensor([0.0], dtype=torch.float64), 1e4)
    assert y[0, 0, 0].item() == pytest.approx(math.cos(1.0), abs=1e-15)
    assert y[0, 0, 32].item() == pytest.approx(math.sin(1.0), abs=1e-15)
    assert y[0, 0, 16].item() == 1.0 and y[0, 0, 48].item() == 0.0


# ---------------------------------------------------------------------------
# Planted composition mistakes: each must break agreement with the torch tower
# ---------------------------------------------------------------------------

def _oracle_block_mutant(kind):
    """The oracle's block with one composition mistake planted:
    "swap_gains" uses g_ffn before attention and g_attn before the MLP,
    "rope_on_v" rotates v as well as q and k, "post_norm" normalises after
    each residual add instead of before each branch."""
    def attn_branch(h, lw, angles, cu_seqlens, cfg):
        t_total, heads, dh = h.shape[0], cfg["heads"], cfg["head_dim"]
        q = O.apply_rope((h @ lw["wq"].T).reshape(t_total, heads, dh), angles)
        k = O.apply_rope((h @ lw["wk"].T).reshape(t_total, heads, dh), angles)
        v = (h @ lw["wv"].T).reshape(t_total, heads, dh)
        if kind == "rope_on_v":
            v = O.apply_rope(v, angles)
        return O.attention(q, k, v, cu_seqlens) @ lw["wo"].T

    def mlp_branch(h, lw):
        return (O.silu(h @ lw["w_gate"].T) * (h @ lw["w_up"].T)) @ lw["w_down"].T

    def block(x, lw, angles, cu_seqlens, cfg):
        eps = cfg["eps"]
        g_attn, g_ffn = (lw["g_ffn"], lw["g_attn"]) if kind == "swap_gains" else (lw["g_attn"], lw["g_ffn"])
        if kind == "post_norm":
            x = O.rms_norm(x + attn_branch(x, lw, angles, cu_seqlens, cfg), g_attn, eps)
            return O.rms_norm(x + mlp_branch(x, lw), g_ffn, eps)
        x = x + attn_branch(O.rms_norm(x, g_attn, eps), lw, angles, cu_seqlens, cfg)
        return x + mlp_branch(O.rms_norm(x, g_ffn, eps), lw)
    return block


@pytest.mark.parametrize("kind", ["swap_gains", "rope_on_v", "post_norm"])
def test_planted_block_composition_mistake_is_caught(monkeypatch, kind):
    cfg, tw, imgs = _setup()
    ref = _torch_tower(imgs, tw, cfg)
    monkeypatch.setattr(O, "tower_block", _oracle_block_mutant(kind))
    assert not _close(O.tower(imgs, tw, cfg), ref)


def test_planted_dropped_ln_pre_is_caught(monkeypatch):
    cfg, tw, imgs = _setup()
    ref = _torch_tower(imgs, tw, cfg)
    g_pre = tw["g_pre"]
    real = O.rms_norm
    monkeypatch.setattr(O, "rms_norm", lambda x, gain, eps: np.asarray(x, np.float64) if gain is g_pre else real(x, gain, eps))
    assert not _close(O.tower(imgs, tw, cfg), ref)


def test_mutant_without_mistake_agrees():
    """The mutant scaffold itself is faithful when nothing is planted, so the
    failures above come from the planted mistakes alone."""
    cfg, tw, imgs = _setup()
    ref = _torch_tower(imgs, tw, cfg)
    saved = O.tower_block
    try:
        O.tower_block = _oracle_block_mutant("none")
        assert _close(O.tower(imgs, tw, cfg), ref)
    finally:
        O.tower_block = saved
