"""Parity of the FP8 (E4M3) tower path with the oracle: weight quantisation
bit-exact, the E4M3 GEMM epilogues, the E4M3 RMSNorm output, and the whole
FP8 tower against the oracle's FP8 tower on the same quantised weights.

Quantisation codes are integers decided in fp32 on both sides; values that
land within fp32 rounding of a midpoint may round differently, so code
comparisons allow a few differences of one code step (never more).
"""
import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import compare, pixels_to_device, to_np, to_oracle, tower_to_device, guarded
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(77)


def _codes_to_np(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


def _e4m3_tensor(values: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(values, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).cuda()


def _assert_codes_close(got, want, max_frac=1e-4):
    """Equal E4M3 values except for a few one-step differences."""
    got, want = np.asarray(got).ravel(), np.asarray(want).ravel()
    diff = got != want
    if diff.any():
        grid = O.e4m3_round(np.concatenate([got[diff], want[diff]]))
        np.testing.assert_array_equal(grid, np.concatenate([got[diff], want[diff]]))  # both on the grid
        step = np.abs(got[diff] - want[diff]) / np.maximum(np.abs(want[diff]), 2.0 ** -9)
        assert np.all(step <= 0.126 + 1e-9), step.max()
    assert diff.mean() <= max_frac, diff.mean()


def test_pack_tower_fp8_quantisation_bit_exact():
    cfg = vlm.preset("mistral3", layers=2, width=256, heads=4, mlp=512)
    tw = synth.tower_weights(5, 2, cfg.width, cfg.mlp, cfg.patch)
    act = synth.fp8_act_scales(2)
    packed = vlm.pack_tower_fp8(cfg, tower_to_device(tw), act)
    torch.cuda.synchronize()
    D, F = cfg.width, cfg.mlp
    kp = -(-3 * cfg.patch ** 2 // 64) * 64
    al = lambda v: -(-v // 256) * 256
    layer0 = al(D * kp * 2) + al(D * 4)
    off, offs = 0, {}
    for name, nbytes in (("wqkv", 3 * D * D), ("wo", D * D), ("wgu", 2 * F * D), ("wdown", D * F),
                         ("cs_qkv", 3 * D * 4), ("cs_o", D * 4), ("cs_gu", 2 * F * 4), ("cs_down", D * 4),
                         ("g_attn", D * 4), ("g_ffn", D * 4)):
        offs[name] = off
        off = al(off + nbytes)
    stride = off
    for layer in range(2):
        base = layer0 + layer * stride
        lw = O.layer_weights(to_oracle(tw), layer)
        gate_up = np.empty((2 * F, D))
        for j in range(F // 16):
            gate_up[32 * j:32 * j + 16] = lw["w_gate"][16 * j:16 * j + 16]
            gate_up[32 * j + 16:32 * j + 32] = lw["w_up"][16 * j:16 * j + 16]
        for name, w, rows, cols, a in (("wqkv", np.concatenate([lw["wq"], lw["wk"], lw["wv"]]), 3 * D, D, act[layer][0]),
                                       ("wo", lw["wo"], D, D, act[layer][1]), ("wgu", gate_up, 2 * F, D, act[layer][2]),
                                       ("wdown", lw["w_down"], D, F, act[layer][3])):
            q_ref, s_ref = O.quantize_weight_rows(w)
            q_gpu = _codes_to_np(packed[base + offs[name]:base + offs[name] + rows * cols]).reshape(rows, cols)
            np.testing.assert_array_equal(q_gpu, q_ref)
            cs_name = {"wqkv": "cs_qkv", "wo": "cs_o", "wgu": "cs_gu", "wdown": "cs_down"}[name]
            cs_gpu = packed[base + offs[cs_name]:base + offs[cs_name] + rows * 4].view(torch.float32).cpu().numpy()
            np.testing.assert_array_equal(cs_gpu, (np.float32(a) * s_ref).astype(np.float32))


@pytest.mark.parametrize("M,N,K", [(300, 512, 384), (1000, 256, 1024)])
def test_gemm_fp8_bf16_and_resid_epilogues(M, N, K):
    codes = O.e4m3_round(RNG.standard_normal((M + N) * K) * 40).reshape(M + N, K)
    a, b = codes[:M], codes[M:]
    cs = (RNG.uniform(0.5, 2.0, N) * 1e-3).astype(np.float32)
    ref = (a @ b.T) * cs.astype(np.float64)[None, :]
    out = guarded((M, N), dtype=torch.bfloat16)
    csd = torch.from_numpy(cs).cuda()
    vlm.gemm_fp8(vlm.EPI_BF16, _e4m3_tensor(a), _e4m3_tensor(b), csd, out)
    torch.cuda.synchronize()
    compare(out, ref, max_rel=8e-3, min_cos=0.99999, what="fp8 gemm bf16")
    x0 = RNG.standard_normal((M, N)).astype(np.float32)
    x = torch.from_numpy(x0).cuda()
    vlm.gemm_fp8(vlm.EPI_RESID, _e4m3_tensor(a), _e4m3_tensor(b), csd, x)
    torch.cuda.synchronize()
    # the tensor core's fp32 accumulation order differs from numpy's: bound relative to the sums' scale
    np.testing.assert_allclose(to_np(x), x0 + ref, rtol=0, atol=3e-4 * np.abs(ref).max())


def test_gemm_fp8_swiglu_e4m3_output():
    M, N, K, out_scale = 260, 512, 256, 448.0 / 16.0
    codes = O.e4m3_round(RNG.standard_normal((M + N) * K) * 30).reshape(M + N, K)
    a, b = codes[:M], codes[M:]
    cs = np.full(N, 2e-3, dtype=np.float32)
    acc = (a @ b.T) * cs.astype(np.float64)[None, :]
    gate = np.concatenate([acc[:, 32 * j:32 * j + 16] for j in range(N // 32)], axis=1)
    up = np.concatenate([acc[:, 32 * j + 16:32 * j + 32] for j in range(N // 32)], axis=1)
    ref = O.e4m3_round(np.float32(O.silu(gate) * up) * np.float32(out_scale))
    out = guarded((M, N // 2), dtype=torch.uint8)
    vlm.gemm_fp8(vlm.EPI_SWIGLU, _e4m3_tensor(a), _e4m3_tensor(b), torch.from_numpy(cs).cuda(), out,
                 out_scale=out_scale)
    torch.cuda.synchronize()
    # SiLU runs on MUFU ex2/rcp (about 2 ulp): allow one-step code differences on 1% of values
    _assert_codes_close(_codes_to_np(out), ref, max_frac=1e-2)


def test_rmsnorm_fp8_codes():
    rows, width, scale = 777, 1024, 448.0 / 8.0
    x0 = (RNG.standard_normal((rows, width)) * 3).astype(np.float32)
    g = (1 + 0.02 * RNG.standard_normal(width)).astype(np.float32)
    out = vlm.rmsnorm_fp8(torch.from_numpy(x0).cuda(), torch.from_numpy(g).cuda(), scale)
    torch.cuda.synchronize()
    ref = O.e4m3_round(np.float32(O.rms_norm(x0.astype(np.float64), g.astype(np.float64), 1e-5)) * np.float32(scale))
    _assert_codes_close(_codes_to_np(out), ref, max_frac=1e-3)


def _fp8_setup(sizes, layers=2, seed=6):
    cfg = vlm.preset("mistral3", layers=layers)
    tw = synth.tower_weights(seed, layers, cfg.width, cfg.mlp, cfg.patch)
    pw = synth.projector_weights(seed, cfg.width, cfg.merge, cfg.proj_out)
    act = synth.fp8_act_scales(layers)
    return cfg, tw, pw, act, synth.images(seed, sizes)


def test_encode_fp8_matches_oracle_fp8_tower():
    sizes = [(224, 224), (112, 168)]
    cfg, tw, pw, act, imgs = _fp8_setup(sizes)
    pipe = vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), sizes, fp8_act_scales=act)
    emb = pipe(pixels_to_device(imgs))
    assert vlm.status_sync(pipe.status) == vlm.OK
    ocfg = dict(O.MISTRAL3, layers=2)
    imgs64 = [im.double().numpy() for im in imgs]
    x_ref = O.tower_fp8(imgs64, to_oracle(tw), act, ocfg)
    compare(pipe.tower_out, x_ref, what="fp8 tower")
    grids = [O.patch_grid(h, w, 14) for h, w in sizes]
    compare(emb, O.projector(x_ref, grids, to_oracle(pw), ocfg), what="fp8 tower + projector")
    # and the quantisation is really there: the bf16 oracle differs by more than the bf16 path's error
    x_bf16 = O.tower(imgs64, to_oracle(tw), ocfg)
    rel = np.abs(to_np(pipe.tower_out) - x_bf16).max() / np.abs(x_bf16).max()
    assert rel > 1e-3, rel


def test_encode_fp8_isolation_and_determinism_full_size():
    """24 layers on two images: each image's rows equal its rows when run alone
    (bit-identical), and two runs agree bit for bit."""
    sizes = [(1540, 1540), (448, 672)]
    cfg, tw, pw, act, imgs = _fp8_setup(sizes, layers=24, seed=8)
    twd, pwd = tower_to_device(tw), tower_to_device(pw)
    pipe = vlm.ImagePipeline(cfg, twd, pwd, sizes, fp8_act_scales=act)
    pix = pixels_to_device(imgs)
    pipe(pix)
    first = pipe.tower_out.clone()
    pipe(pix)
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(first, pipe.tower_out)
    assert torch.isfinite(first.float()).all()
    alone = vlm.ImagePipeline(cfg, twd, pwd, sizes[1:], fp8_act_scales=act)
    alone(pixels_to_device(imgs[1:]))
    assert vlm.status_sync(alone.status) == vlm.OK
    assert torch.equal(first[12100:], alone.tower_out)
