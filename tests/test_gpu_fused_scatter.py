"""vlm_merge_project_scatter: the projector with the masked scatter fused into
its last linear ("Mistral 3", Mistral3Model: the image features replace the
image_token_id rows of the token embeddings). Its rows must equal, bit for
bit, those of vlm_merge_project followed by vlm_scatter, the other rows must be
untouched, and the image rows must match the oracle; a placeholder count that
differs from the number of merged tokens writes nothing.
"""
import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import compare, guarded_copy, pixels_to_device, to_oracle, tower_to_device
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu


def _ids(n_text, n_img, seed, token):
    """n_text text ids (never the placeholder) and n_img placeholders at random positions."""
    rng = np.random.default_rng(seed)
    ids = rng.integers(token + 1, token + 30000, size=n_text + n_img)
    ids[np.sort(rng.choice(n_text + n_img, size=n_img, replace=False))] = token
    return torch.from_numpy(ids.astype(np.int64)).cuda()


def _setup(preset, sizes, seed, layers=1, **over):
    cfg = vlm.preset(preset, layers=layers, **over)
    tw = synth.tower_weights(seed, layers, cfg.width, cfg.mlp, cfg.patch)
    pw = synth.projector_weights(seed, cfg.width, cfg.merge, cfg.proj_out)
    imgs = synth.images(seed, sizes)
    pipe = vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), sizes)
    return cfg, tw, pw, imgs, pipe


def _text(n, e, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(n, e, generator=g).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("preset,sizes,over", [
    ("mistral3", [(224, 336), (112, 112), (196, 84)], {}),   # three images, placeholders scattered
    ("pixtral12b", [(64, 96), (32, 32)], {}),                # no merge
    ("mistral3", [(28, 28)], {"proj_out": 768}),             # one merged token, another width
])
def test_fused_equals_merge_project_then_scatter_and_oracle(preset, sizes, over):
    cfg, tw, pw, imgs, pipe = _setup(preset, sizes, seed=5, **over)
    pix = pixels_to_device(imgs)
    Tm = vlm.num_merged(cfg, sizes)
    ids = _ids(2 * Tm + 17, Tm, seed=6, token=cfg.image_token_id)
    text0 = _text(ids.numel(), cfg.proj_out, seed=7)
    sep = text0.clone()
    vlm.scatter(ids, pipe(pix).clone(), sep, image_token_id=cfg.image_token_id)
    assert vlm.status_sync(pipe.status) == vlm.OK
    fused = guarded_copy(text0)
    pipe.embed_into(pix, ids, fused)
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(fused, sep)
    mask = ids == cfg.image_token_id
    assert torch.equal(fused[~mask], text0[~mask])
    ocfg = dict(O.MISTRAL3 if cfg.merge == 2 else O.PIXTRAL12B)
    ocfg.update(layers=cfg.layers, patch=cfg.patch, merge=cfg.merge)
    _, y_ref = O.encode_merge_project([im.double().numpy() for im in imgs], to_oracle(tw), to_oracle(pw), ocfg)
    compare(fused[mask], y_ref, what="fused image rows")


@pytest.mark.parametrize("delta", [-1, 1])
def test_fused_count_mismatch_writes_nothing(delta):
    sizes = [(112, 168)]
    cfg, _, _, imgs, pipe = _setup("mistral3", sizes, seed=8)
    Tm = vlm.num_merged(cfg, sizes)
    ids = _ids(40, Tm + delta, seed=9, token=cfg.image_token_id)
    text0 = _text(ids.numel(), cfg.proj_out, seed=10)
    fused = guarded_copy(text0)
    pipe.embed_into(pixels_to_device(imgs), ids, fused)
    assert vlm.status_sync(pipe.status) == vlm.ERR_COUNT_MISMATCH
    assert torch.equal(fused, text0)


def test_fused_full_size_1540_equals_separate():
    """The headline image (3,025 merged tokens) among 4,096 ids, one tower layer."""
    sizes = [(1540, 1540)]
    cfg, _, _, imgs, pipe = _setup("mistral3", sizes, seed=11)
    pix = pixels_to_device(imgs)
    ids = _ids(4096 - 3025, 3025, seed=12, token=cfg.image_token_id)
    text0 = _text(4096, cfg.proj_out, seed=13)
    sep = text0.clone()
    vlm.scatter(ids, pipe(pix).clone(), sep, image_token_id=cfg.image_token_id)
    fused = text0.clone()
    pipe.embed_into(pix, ids, fused)
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(fused, sep)


def test_fused_above_one_cta_id_limit():
    """40,000 ids, above the one-CTA kernel's 4,096: the placeholder rows come
    from the count, scan and positions kernels; same rows, and a count
    mismatch still writes nothing."""
    sizes = [(224, 224), (84, 112)]
    cfg, _, _, imgs, pipe = _setup("mistral3", sizes, seed=14)
    pix = pixels_to_device(imgs)
    Tm = vlm.num_merged(cfg, sizes)
    ids = _ids(40000 - Tm, Tm, seed=15, token=cfg.image_token_id)
    text0 = _text(ids.numel(), cfg.proj_out, seed=16)
    sep = text0.clone()
    vlm.scatter(ids, pipe(pix).clone(), sep, image_token_id=cfg.image_token_id)
    fused = text0.clone()
    pipe.embed_into(pix, ids, fused)
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(fused, sep)
    bad = ids.clone()
    bad[torch.nonzero(bad == cfg.image_token_id)[0]] = cfg.image_token_id + 1   # one placeholder too few
    fused = text0.clone()
    pipe.embed_into(pix, bad, fused)
    assert vlm.status_sync(pipe.status) == vlm.ERR_COUNT_MISMATCH
    assert torch.equal(fused, text0)
