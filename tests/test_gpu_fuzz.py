"""Seeded random batches through the bf16, E4M3 and NVFP4 towers against the oracle.

Each case draws 1-5 images with sides 28 * U{1..15} pixels (ragged attention
blocks, ragged 128-row query tiles, GEMM row counts off every tile size and
NVFP4 scale groups of every fill), runs one tower layer plus the projector,
and compares every row with the oracle: the bf16 and E4M3 paths at the usual
2e-2 / 0.999 (the E4M3 one against the oracle's E4M3 tower), the NVFP4 path at the end-to-end bounds measured from the oracle's own
sensitivity (tests/test_gpu_nvfp4_tower.py). The NVFP4 case also checks that
the last image's rows equal its rows when it runs alone (bit-identical).
Every pipeline also writes its embeddings into a token sequence with the
scatter fused into the projector's last linear (ImagePipeline.embed_into),
which must equal vlm_merge_project + vlm_scatter bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import compare, pixels_to_device, to_oracle, tower_to_device
from tests.test_gpu_nvfp4_tower import E2E_MAX_REL, E2E_MIN_COS
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu


def _check_fused(pipe, pix, emb, seed, token):
    """embed_into == scatter(merge_project) on random placeholder positions."""
    rng = np.random.default_rng(2000 + seed)
    Tm = emb.shape[0]
    n = Tm + int(rng.integers(1, 300))
    ids = rng.integers(token + 1, token + 5000, size=n)
    ids[np.sort(rng.choice(n, size=Tm, replace=False))] = token
    ids = torch.from_numpy(ids.astype(np.int64)).cuda()
    g = torch.Generator().manual_seed(3000 + seed)
    text = torch.randn(n, emb.shape[1], generator=g).to(torch.bfloat16).cuda()
    sep = text.clone()
    vlm.scatter(ids, emb, sep, image_token_id=token)
    pipe.embed_into(pix, ids, text)
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(text, sep)


def _sizes(seed):
    rng = np.random.default_rng(1000 + seed)
    return [(28 * int(rng.integers(1, 16)), 28 * int(rng.integers(1, 16))) for _ in range(int(rng.integers(1, 6)))]


@pytest.mark.parametrize("seed", range(12))
def test_random_batches_bf16_fp8_nvfp4_vs_oracle(seed):
    sizes = _sizes(seed)
    layers = 1
    cfg = vlm.preset("mistral3", layers=layers)
    tw = synth.tower_weights(seed, layers, cfg.width, cfg.mlp, cfg.patch)
    pw = synth.projector_weights(seed, cfg.width, cfg.merge, cfg.proj_out)
    imgs = synth.images(seed, sizes)
    twd, pwd, pix = tower_to_device(tw), tower_to_device(pw), pixels_to_device(imgs)
    ocfg = dict(O.MISTRAL3, layers=layers)
    imgs64 = [im.double().numpy() for im in imgs]
    grids = [O.patch_grid(h, w, 14) for h, w in sizes]

    pipe = vlm.ImagePipeline(cfg, twd, pwd, sizes)
    emb = pipe(pix)
    assert vlm.status_sync(pipe.status) == vlm.OK
    x_ref, y_ref = O.encode_merge_project(imgs64, to_oracle(tw), to_oracle(pw), ocfg)
    compare(pipe.tower_out, x_ref, what=f"bf16 tower {sizes}")
    compare(emb, y_ref, what=f"bf16 projector {sizes}")
    _check_fused(pipe, pix, emb, seed, cfg.image_token_id)

    act8 = synth.fp8_act_scales(layers)
    pipe8 = vlm.ImagePipeline(cfg, twd, pwd, sizes, fp8_act_scales=act8)
    emb8 = pipe8(pix)
    assert vlm.status_sync(pipe8.status) == vlm.OK
    x8 = O.tower_fp8(imgs64, to_oracle(tw), act8, ocfg)
    compare(pipe8.tower_out, x8, what=f"fp8 tower {sizes}")
    compare(emb8, O.projector(x8, grids, to_oracle(pw), ocfg), what=f"fp8 projector {sizes}")
    _check_fused(pipe8, pix, emb8, seed, cfg.image_token_id)

    act = synth.nvfp4_act_scales(layers)
    pipe4 = vlm.ImagePipeline(cfg, twd, pwd, sizes, nvfp4_act_scales=act)
    emb4 = pipe4(pix)
    assert vlm.status_sync(pipe4.status) == vlm.OK
    x4 = O.tower_nvfp4(imgs64, to_oracle(tw), act, ocfg)
    compare(pipe4.tower_out, x4, max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS, what=f"nvfp4 tower {sizes}")
    compare(emb4, O.projector(x4, grids, to_oracle(pw), ocfg), max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS,
            what=f"nvfp4 projector {sizes}")
    _check_fused(pipe4, pix, emb4, seed, cfg.image_token_id)
    if len(sizes) > 1:
        last = sizes[-1:]
        alone = vlm.ImagePipeline(cfg, twd, pwd, last, nvfp4_act_scales=act)
        alone(pixels_to_device(imgs[-1:]))
        assert vlm.status_sync(alone.status) == vlm.OK
        t_last = grids[-1][0] * grids[-1][1]
        assert torch.equal(pipe4.tower_out[-t_last:], alone.tower_out)
