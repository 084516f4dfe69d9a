"""Parity of the image front end (vlm_preprocess: resize onto the patch grid,
Pixtral tiling) and of the device placeholder expansion with the CPU oracle.

Resize: fp32 on the GPU against the fp64 oracle. The sample position's
integer part and fraction come from an exact integer division on the GPU, so
the only differences are fp32 rounding of the fraction and of the 4-tap
blend on values <= 255: the bound 4e-6 (on values in [0, 1]) is about 30
units of fp32 rounding at 1.0. Expansion is integer work: bit-exact.
"""
import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import compare, to_np, to_oracle, tower_to_device, guarded_copy
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu

RESIZE_ATOL = 4e-6


def _oracle_front(photos, out_hw, tile=0):
    parts = []
    for ph, (oh, ow) in zip(photos, out_hw):
        img = O.resize_bilinear(O.pixels_from_u8(ph.numpy()), oh, ow)
        if tile:
            parts += [t.reshape(-1) for t in O.tile_image(img, tile)]
        else:
            parts.append(img.reshape(-1))
    return np.concatenate(parts)


def _gpu_front(photos, out_hw, tile=0):
    src = torch.cat([p.reshape(-1) for p in photos]).cuda()
    src_hw = [tuple(p.shape[:2]) for p in photos]
    out = vlm.preprocess(src, src_hw, out_hw, tile=tile)
    torch.cuda.synchronize()
    return to_np(out)


@pytest.mark.parametrize("src,dst", [
    ((61, 83), (28, 56)),       # downscale, ragged
    ((50, 70), (56, 84)),       # upscale
    ((84, 112), (84, 112)),     # identity size: exact copy of u8 / 255
    ((1, 1), (28, 28)),         # single source pixel
    ((1000, 7), (28, 4)),       # extreme aspect
    ((5, 17000), (28, 56)),     # source rows too long to stage in shared memory
    ((2, 65536), (4, 16384)),   # (2 out_w + 1) * W above 2^31: 64-bit coordinates
])
def test_resize_matches_oracle(src, dst):
    ph = synth.photo_u8(1, f"resize{src}", *src)
    got = _gpu_front([ph], [dst])
    ref = _oracle_front([ph], [dst])
    np.testing.assert_allclose(got, ref, rtol=0, atol=RESIZE_ATOL)


def test_resize_identity_is_u8_over_255():
    """Same size in and out: every tap weight is 0 or 1, so the output is the
    u8 value times fp32(1/255), two fp32 roundings of u8/255: within 2^-23."""
    ph = synth.photo_u8(2, "ident", 56, 84)
    got = _gpu_front([ph], [(56, 84)])
    ref = (ph.permute(2, 0, 1).reshape(-1).double() / 255.0).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=2.0 ** -23)


def test_resize_batch_of_photos_to_processor_sizes():
    """Several photos at once, each to vlm_resize_target's size (longest edge
    1540, 28-pixel grid); more photos than one launch chunk holds."""
    rng = np.random.default_rng(3)
    srcs = [(int(rng.integers(20, 700)), int(rng.integers(20, 700))) for _ in range(37)]
    photos = [synth.photo_u8(3, f"b{i}", h, w) for i, (h, w) in enumerate(srcs)]
    out_hw = [vlm.resize_target(h, w, 1540, 28) for h, w in srcs]
    assert out_hw == [O.resized_hw(h, w, 1540, 28) for h, w in srcs]
    got = _gpu_front(photos, out_hw)
    np.testing.assert_allclose(got, _oracle_front(photos, out_hw), rtol=0, atol=RESIZE_ATOL)


def test_resize_full_size_photo():
    """A 4032x3024 camera frame to the processor size 1176x1540 (whole output)."""
    ph = synth.photo_u8(4, "camera", 3024, 4032)
    out_hw = [vlm.resize_target(3024, 4032, 1540, 28)]
    assert out_hw == [(1176, 1540)]
    got = _gpu_front([ph], out_hw)
    np.testing.assert_allclose(got, _oracle_front([ph], out_hw), rtol=0, atol=RESIZE_ATOL)


def test_pixtral_tiling():
    """Resize to whole 1024-pixel tiles and cut into tiles in the same pass."""
    photos = [synth.photo_u8(5, "tile_a", 1500, 2100), synth.photo_u8(5, "tile_b", 700, 900)]
    out_hw = [(1024, 2048), (1024, 1024)]
    got = _gpu_front(photos, out_hw, tile=1024)
    assert got.size == 3 * 3 * 1024 * 1024
    np.testing.assert_allclose(got, _oracle_front(photos, out_hw, tile=1024), rtol=0, atol=RESIZE_ATOL)
    assert vlm.tiled_hw(out_hw, 1024) == [(1024, 1024)] * 3


def test_photo_through_front_end_and_tower():
    """u8 photo -> vlm_preprocess -> vlm_encode -> vlm_merge_project against the
    oracle taking the same steps (2 layers)."""
    cfg = vlm.preset("mistral3", layers=2)
    tw = synth.tower_weights(6, 2, cfg.width, cfg.mlp, cfg.patch)
    pw = synth.projector_weights(6, cfg.width, cfg.merge, cfg.proj_out)
    ph = synth.photo_u8(6, "e2e", 333, 250)
    out_hw = [vlm.resize_target(333, 250, 1540, 28)]
    pix = vlm.preprocess(ph.reshape(-1).cuda(), [(333, 250)], out_hw)
    pipe = vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), out_hw)
    emb = pipe(pix)
    assert vlm.status_sync(pipe.status) == vlm.OK
    ocfg = dict(O.MISTRAL3, layers=2)
    img = O.resize_bilinear(O.pixels_from_u8(ph.numpy()), *out_hw[0])
    _, ref = O.encode_merge_project([img], to_oracle(tw), to_oracle(pw), ocfg)
    compare(emb, ref, what="photo pipeline")


# ---------------------------------------------------------------------------
# Placeholder expansion
# ---------------------------------------------------------------------------
MARKER = 7


def _ids_with_markers(rng, n_text, n_images):
    ids = rng.integers(11, 32000, n_text).astype(np.int64)
    where = np.sort(rng.choice(n_text + n_images, n_images, replace=False))
    out = np.empty(n_text + n_images, dtype=np.int64)
    mask = np.zeros(n_text + n_images, dtype=bool)
    mask[where] = True
    out[mask] = MARKER
    out[~mask] = ids
    return out


@pytest.mark.parametrize("n_text,counts", [
    (10, [3]),
    (0, [5, 0, 2]),                       # markers only, one empty image
    (300, []),                            # no images: plain copy
    (1000, [1540, 256, 1]),
    (100000, [1536] * 70),                # many chunks, many images
])
def test_expand_matches_oracle(n_text, counts):
    rng = np.random.default_rng(len(counts) * 1000 + n_text)
    ids = _ids_with_markers(rng, n_text, len(counts))
    got = vlm.expand_placeholders(torch.from_numpy(ids).cuda(), MARKER, counts, image_token_id=10)
    torch.cuda.synchronize()
    ref = O.expand_placeholders(ids, MARKER, counts, 10)
    np.testing.assert_array_equal(got.cpu().numpy(), ref)


def test_expand_edges_markers_first_last_adjacent():
    ids = np.array([MARKER, MARKER, 5, 6, MARKER] + [9] * 600 + [MARKER], dtype=np.int64)
    counts = [4, 1, 300, 2]
    got = vlm.expand_placeholders(torch.from_numpy(ids).cuda(), MARKER, counts)
    np.testing.assert_array_equal(got.cpu().numpy(), O.expand_placeholders(ids, MARKER, counts, 10))


def test_expand_count_mismatch_writes_nothing():
    ids = torch.tensor([1, MARKER, 2, MARKER], dtype=torch.int64, device="cuda")
    status = vlm.new_status()
    out = torch.full((64,), -1, dtype=torch.int64, device="cuda")
    vlm.expand_placeholders(ids, MARKER, [3, 4, 5], out=out, status=status)
    assert vlm.status_sync(status) == vlm.ERR_COUNT_MISMATCH
    assert (out == -1).all()


def test_expand_then_scatter_equals_oracle():
    """Expansion feeding the masked scatter: placeholders land where the
    oracle's scatter puts the image rows."""
    rng = np.random.default_rng(11)
    counts = [12, 30]
    ids = _ids_with_markers(rng, 50, 2)
    exp = vlm.expand_placeholders(torch.from_numpy(ids).cuda(), MARKER, counts)
    n = exp.numel()
    text = guarded_copy(synth.text_embeddings(11, n, 256))
    img = synth.text_embeddings(12, sum(counts), 256).cuda()
    ref = O.scatter(O.expand_placeholders(ids, MARKER, counts, 10), to_np(img), to_np(text), 10)
    vlm.scatter(exp, img, text, image_token_id=10)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(text), ref)
