"""The NVFP4 tower (vlm_encode_nvfp4) against the oracle.

Every GEMM input is quantised to NVFP4 from fp32 inside the kernel that
produces it: the RMSNorm, the attention epilogue and the SwiGLU epilogue of
the gate/up GEMM; QKV takes RoPE in its epilogue. Each producer is compared
with the oracle's quantiser applied to the oracle's fp32 values, then the
whole tower with `tower_nvfp4` ("Mistral 3", `Mistral3VisionModel`, with the
NVFP4 weights of the vllm.cpp issue, "Why this one is smaller than it looks").

Codes and scales: the GPU computes the quantiser's input in fp32 with its own
rounding order (rsqrt, exponentials, fp32 accumulation), so a value that sits
on a rounding boundary may land one step away from the oracle's; such codes
must stay a small fraction (the bound is stated per test) and the decoded
values must match everywhere else.
"""
import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import compare, pixels_to_device, to_np, to_oracle, tower_to_device
from tests.test_gpu_nvfp4 import _MAGS, _dev_scalar, _operand, _unpack_codes, _unpack_sf
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(91)


def _decoded(q, sf, rows, k):
    """(codes as E2M1 values [rows, k], block scales [rows, k/16]) of a GPU NVFP4 tensor."""
    return _unpack_codes(q)[:rows], _unpack_sf(sf, rows, k)


def _assert_nvfp4_close(q, sf, x32, sg, max_frac, what):
    """GPU codes / scales against O.quantize_nvfp4(x32, sg): at most max_frac of
    the block scales and of the codes differ, each by one step at most."""
    rows, k = x32.shape
    q_got, s_got = _decoded(q, sf, rows, k)
    q_ref, s_ref = O.quantize_nvfp4(x32, sg)
    s_bad = s_got != s_ref
    assert s_bad.mean() <= max_frac, f"{what}: {s_bad.mean():.2e} of block scales differ"
    # where the block scale agrees, a code may move by one E2M1 step only
    same = np.repeat(~s_bad, 16, axis=1)
    c_bad = (q_got != q_ref) & same
    assert c_bad.mean() <= max_frac, f"{what}: {c_bad.mean():.2e} of codes differ"
    step = np.abs(np.searchsorted(_MAGS, np.abs(q_got)) - np.searchsorted(_MAGS, np.abs(q_ref)))
    assert np.all(step[c_bad] <= 1) and np.all(np.sign(q_got[c_bad]) * np.sign(q_ref[c_bad]) >= 0), what
    # and the decoded tensor is the oracle's to NVFP4 accuracy
    got = O.dequantize_nvfp4(q_got, s_got, sg)
    ref = O.dequantize_nvfp4(q_ref, s_ref, sg)
    assert np.abs(got - ref).max() <= 0.5 * np.abs(ref).max(), what
    return float(c_bad.mean())


def test_rmsnorm_nvfp4_codes():
    rows, width, sg = 777, 1024, 8.0 / 2688.0
    x0 = (RNG.standard_normal((rows, width)) * 3).astype(np.float32)
    x0[5] *= 1e-3                                      # a row of small values
    g = (1 + 0.3 * RNG.standard_normal(width)).astype(np.float32)
    q, sf = vlm.rmsnorm_nvfp4(torch.from_numpy(x0).cuda(), torch.from_numpy(g).cuda(), sg)
    torch.cuda.synchronize()
    ref = np.float32(O.rms_norm(x0.astype(np.float64), g.astype(np.float64), 1e-5))
    _assert_nvfp4_close(q, sf, ref, sg, 2e-3, "rmsnorm nvfp4")
    # the padding rows of the last 128-row group keep scale 0
    assert np.all(_unpack_sf(sf, 896, width)[rows:] == 0)


def test_rmsnorm_nvfp4_with_ln_pre_writes_back():
    rows, width, sg = 300, 1024, 8.0 / 2688.0
    x0 = (RNG.standard_normal((rows, width)) * 2).astype(np.float32)
    g0 = (1 + 0.1 * RNG.standard_normal(width)).astype(np.float32)
    g1 = (1 + 0.1 * RNG.standard_normal(width)).astype(np.float32)
    x = torch.from_numpy(x0).cuda()
    q, sf = vlm.rmsnorm_nvfp4(x, torch.from_numpy(g1).cuda(), sg, g0=torch.from_numpy(g0).cuda())
    torch.cuda.synchronize()
    y = O.rms_norm(x0.astype(np.float64), g0.astype(np.float64), 1e-5)
    np.testing.assert_allclose(to_np(x), y, rtol=2e-6, atol=2e-6)
    _assert_nvfp4_close(q, sf, np.float32(O.rms_norm(y, g1.astype(np.float64), 1e-5)), sg, 2e-3, "ln_pre + norm")


@pytest.mark.parametrize("lens", [[300, 77], [128], [1, 255, 0, 129]])
def test_attention_nvfp4_codes(lens):
    heads, sg = 2, 4.0 / 2688.0
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    qkv = torch.from_numpy(RNG.standard_normal((T, 3 * heads * 64)) * 1.5).to(torch.bfloat16)
    q, sf = vlm.attention_nvfp4(qkv.cuda(), cu.tolist(), heads, sg)
    torch.cuda.synchronize()
    x = qkv.double().numpy().reshape(T, 3, heads, 64)
    ref = O.attention(x[:, 0], x[:, 1], x[:, 2], cu).reshape(T, heads * 64)
    # P is rounded to bf16 on the GPU, so the output carries a relative error
    # eps of about 2^-10..2^-9; an E4M3 block scale moves when the block's amax
    # lies within eps of a rounding boundary, and those sit 2^-4..2^-3 apart
    # (relative), so up to about 16..30 eps = 1.5..6 % of scales may move
    _assert_nvfp4_close(q, sf, np.float32(ref), sg, 4e-2, f"attention nvfp4 {lens}")


def _interleave_gate_up(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """Rows 32j..32j+15 from gate rows 16j.., 32j+16..32j+31 from up rows 16j.."""
    f = gate.shape[0]
    out = np.empty((2 * f,) + gate.shape[1:], gate.dtype)
    for j in range(f // 16):
        out[32 * j:32 * j + 16] = gate[16 * j:16 * j + 16]
        out[32 * j + 16:32 * j + 32] = up[16 * j:16 * j + 16]
    return out


def _random_nvfp4(rows, k, exps=(-3, 2)):
    q = RNG.choice(np.concatenate([_MAGS, -_MAGS[1:]]), size=(rows, k))
    s = np.exp2(RNG.integers(exps[0], exps[1], size=(rows, k // 16))) * RNG.choice([1.0, 1.25, 1.5], (rows, k // 16))
    return q, s


@pytest.mark.parametrize("M", [300, 12100])
def test_gemm_nvfp4_swiglu_nvfp4_output(M):
    """The gate/up GEMM's SwiGLU epilogue quantises silu(gate) * up (fp32) to NVFP4."""
    K, F = 512, 512
    ga, gb, sg = np.float32(0.37), np.float32(0.011), np.float32(16.0 / 2688.0)
    qa, sa = _random_nvfp4(M, K)
    qg, sgate = _random_nvfp4(F, K)
    qu, sup = _random_nvfp4(F, K)
    qb, sb = _interleave_gate_up(qg, qu), _interleave_gate_up(sgate, sup)
    hq, hsf = vlm.gemm_nvfp4_swiglu(_operand(qa, sa, ga, K), _operand(qb, sb, gb, K), float(sg))
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 512 else np.sort(np.concatenate([RNG.choice(M, 200, replace=False), [0, M - 1]]))
    gate = O.nvfp4_linear(qa[rows], sa[rows], ga, qg, sgate, gb)
    up = O.nvfp4_linear(qa[rows], sa[rows], ga, qu, sup, gb)
    h = np.float32(O.silu(gate) * up)
    hq_np, hsf_np = hq.cpu(), _unpack_sf(hsf, M, F)[rows]
    q_got = _unpack_codes(hq_np)[rows]
    q_ref, s_ref = O.quantize_nvfp4(h, sg)
    s_bad = hsf_np != s_ref
    assert s_bad.mean() <= 1e-2, s_bad.mean()
    c_bad = (q_got != q_ref) & np.repeat(~s_bad, 16, axis=1)
    assert c_bad.mean() <= 1e-2, c_bad.mean()
    if M % 128:
        assert np.all(_unpack_sf(hsf, (M + 127) // 128 * 128, F)[M:] == 0)


def test_gemm_nvfp4_rope_epilogue():
    """QKV with RoPE in the epilogue: three 256-column blocks (4 heads), the
    first two rotated by the rows' (row, col) positions."""
    h, w, D = 23, 17, 256
    M, K = h * w, 512
    ga, gb = np.float32(0.21), np.float32(0.05)
    qa, sa = _random_nvfp4(M, K)
    qb, sb = _random_nvfp4(3 * D, K)
    rows, cols, _ = O.positions([(h, w)])
    pos = torch.from_numpy((rows << 16 | cols).astype(np.int32)).cuda()
    tab = vlm.rope_table(1e4, 64, max(h, w))
    out = torch.empty((M, 3 * D), dtype=torch.bfloat16, device="cuda")
    vlm.gemm_nvfp4_rope(_operand(qa, sa, ga, K), _operand(qb, sb, gb, K), out, pos, tab, 2 * D)
    torch.cuda.synchronize()
    acc = O.nvfp4_linear(qa, sa, ga, qb, sb, gb)
    ang = O.rope_angles(rows, cols, 1e4, 64)
    qr = O.apply_rope(acc[:, :D].reshape(M, 4, 64), ang).reshape(M, D)
    kr = O.apply_rope(acc[:, D:2 * D].reshape(M, 4, 64), ang).reshape(M, D)
    compare(out, np.concatenate([qr, kr, acc[:, 2 * D:]], axis=1), max_rel=1e-2, min_cos=0.9999,
            what="nvfp4 qkv rope")


def _nvfp4_setup(sizes, layers=2, seed=6):
    cfg = vlm.preset("mistral3", layers=layers)
    tw = synth.tower_weights(seed, layers, cfg.width, cfg.mlp, cfg.patch)
    pw = synth.projector_weights(seed, cfg.width, cfg.merge, cfg.proj_out)
    return cfg, tw, pw, synth.nvfp4_act_scales(layers), synth.images(seed, sizes)


def _gpu_weights_nvfp4(tw_dev, layer, D, F):
    """One layer's four GEMM weights quantised by the library's quantiser in the
    executed row orders ([Wq; Wk; Wv], Wo, gate / up interleaved by 16, W_down)."""
    def quant(w):
        g = vlm.amax_scale(w)
        q, sf = vlm.quant_nvfp4(w, g)
        return q, sf, g
    gate, up = tw_dev["w_gate"][layer], tw_dev["w_up"][layer]
    gu = torch.empty((2 * F, D), dtype=gate.dtype, device=gate.device)
    gu.view(F // 16, 2, 16, D)[:, 0] = gate.view(F // 16, 16, D)
    gu.view(F // 16, 2, 16, D)[:, 1] = up.view(F // 16, 16, D)
    return {"qkv": quant(torch.cat([tw_dev["wq"][layer], tw_dev["wk"][layer], tw_dev["wv"][layer]])),
            "o": quant(tw_dev["wo"][layer].contiguous()), "gate_up": quant(gu),
            "down": quant(tw_dev["w_down"][layer].contiguous())}


def _codes(q, sf, rows, k):
    return _unpack_codes(q)[:rows], _unpack_sf(sf, rows, k)


def test_encode_nvfp4_stepwise_against_oracle():
    """The NVFP4 tower as a chain of the library's kernels, each step checked
    against the oracle applied to the GPU's own previous state (every rounding
    decision is then the same input on both sides up to fp32 rounding):
    RMSNorm and attention codes within their flip bounds, the GEMMs on the
    GPU's codes to fp32 accumulation, the weight codes bit-exact. The chain runs
    the same kernels in the same order as vlm_encode_nvfp4, whose output must
    then equal the chain's bit for bit: this pins the encoder's wiring (which
    scale feeds which producer, the gate / up order) that no end-to-end
    tolerance can see, since NVFP4 re-rounds under any rounding-level change."""
    sizes = [(224, 224), (112, 168)]
    layers = 2
    cfg, tw, pw, act, imgs = _nvfp4_setup(sizes, layers=layers)
    D, F, H = cfg.width, cfg.mlp, cfg.heads
    twd = tower_to_device(tw)
    pix = pixels_to_device(imgs)
    packed = vlm.pack_tower_nvfp4(cfg, twd, act)
    enc = vlm.encode_nvfp4(cfg, pix, sizes, packed, act)
    torch.cuda.synchronize()

    ocfg = dict(O.MISTRAL3, layers=layers)
    tw64 = to_oracle(tw)
    grids = [O.patch_grid(h, w, 14) for h, w in sizes]
    rows, cols, cu = O.positions(grids)
    T = len(rows)
    pos = torch.from_numpy((rows << 16 | cols).astype(np.int32)).cuda()
    tab = vlm.rope_table(cfg.rope_theta, 64, max(max(g) for g in grids))
    ang = O.rope_angles(rows, cols, cfg.rope_theta, 64)

    x = vlm.patch_embed(cfg, pix, sizes, packed)
    torch.cuda.synchronize()
    x_pe = np.concatenate([O.patch_embed(O.normalize_pixels(im.double().numpy()), tw64["w_pe"]) for im in imgs])
    compare(x, x_pe, max_rel=1e-2, min_cos=0.99999, what="patch embed")
    for layer in range(layers):
        a = [float(np.float32(v)) for v in act[layer]]
        a_dev = [_dev_scalar(v) for v in a]
        w = _gpu_weights_nvfp4(twd, layer, D, F)
        lq = O.quantize_layer_nvfp4(O.layer_weights(tw64, layer))
        for name, k in (("qkv", D), ("o", D), ("down", F)):          # weights bit-exact
            qg, sg_ = _codes(w[name][0], w[name][1], lq[name][0].shape[0], k)
            np.testing.assert_array_equal(qg, lq[name][0])
            np.testing.assert_array_equal(sg_, lq[name][1])
            assert w[name][2].item() == float(lq[name][2])
        qg, sg_ = _codes(w["gate_up"][0], w["gate_up"][1], 2 * F, D)
        back = np.concatenate([np.arange(F).reshape(-1, 16) // 16 * 32 + np.arange(16),
                               np.arange(F).reshape(-1, 16) // 16 * 32 + 16 + np.arange(16)]).reshape(-1)
        np.testing.assert_array_equal(qg[back], lq["gate_up"][0])
        np.testing.assert_array_equal(sg_[back], lq["gate_up"][1])

        # attention norm (ln_pre folded into the first)
        x_before = to_np(x).astype(np.float64)
        q1, s1 = vlm.rmsnorm_nvfp4(x, twd["g_attn"][layer].contiguous(), a[0],
                                   g0=twd["g_pre"] if layer == 0 else None)
        torch.cuda.synchronize()
        if layer == 0:
            x_before = O.rms_norm(x_before, tw64["g_pre"], cfg.eps)
            np.testing.assert_allclose(to_np(x), x_before, rtol=0, atol=2e-6 * np.abs(x_before).max())
        x_cur = to_np(x).astype(np.float64)
        _assert_nvfp4_close(q1, s1, np.float32(O.rms_norm(x_cur, tw64["g_attn"][layer], cfg.eps)), a[0], 2e-3,
                            f"layer {layer} attention norm")
        # QKV + RoPE on the GPU's codes
        qkv = torch.empty((T, 3 * D), dtype=torch.bfloat16, device="cuda")
        vlm.gemm_nvfp4_rope((q1, s1, a_dev[0]), w["qkv"], qkv, pos, tab, 2 * D)
        torch.cuda.synchronize()
        c1, b1 = _codes(q1, s1, T, D)
        y = O.nvfp4_linear(c1, b1, a[0], *lq["qkv"])
        ref = np.concatenate([O.apply_rope(y[:, :D].reshape(T, H, 64), ang).reshape(T, D),
                              O.apply_rope(y[:, D:2 * D].reshape(T, H, 64), ang).reshape(T, D), y[:, 2 * D:]], axis=1)
        compare(qkv, ref, max_rel=1e-2, min_cos=0.9999, what=f"layer {layer} qkv")
        # attention on the GPU's q, k, v
        aq, asf = vlm.attention_nvfp4(qkv, cu.tolist(), H, a[1])
        torch.cuda.synchronize()
        v3 = qkv.double().cpu().numpy().reshape(T, 3, H, 64)
        _assert_nvfp4_close(aq, asf, np.float32(O.attention(v3[:, 0], v3[:, 1], v3[:, 2], cu).reshape(T, D)), a[1],
                            4e-2, f"layer {layer} attention")
        # O projection into the residual on the GPU's codes
        vlm.gemm_nvfp4(vlm.EPI_RESID, (aq, asf, a_dev[1]), w["o"], x)
        torch.cuda.synchronize()
        ca, ba = _codes(aq, asf, T, D)
        x_ref = x_cur + O.nvfp4_linear(ca, ba, a[1], *lq["o"])
        np.testing.assert_allclose(to_np(x), x_ref, rtol=0, atol=2e-5 * np.abs(x_ref).max())
        # MLP norm
        x_cur = to_np(x).astype(np.float64)
        q2, s2 = vlm.rmsnorm_nvfp4(x, twd["g_ffn"][layer].contiguous(), a[2])
        torch.cuda.synchronize()
        _assert_nvfp4_close(q2, s2, np.float32(O.rms_norm(x_cur, tw64["g_ffn"][layer], cfg.eps)), a[2], 2e-3,
                            f"layer {layer} MLP norm")
        # gate / up with SwiGLU and the hidden state's quantisation on the GPU's codes
        hq, hsf = vlm.gemm_nvfp4_swiglu((q2, s2, a_dev[2]), w["gate_up"], a[3])
        torch.cuda.synchronize()
        c2, b2 = _codes(q2, s2, T, D)
        gu = O.nvfp4_linear(c2, b2, a[2], *lq["gate_up"])
        _assert_nvfp4_close(hq, hsf, np.float32(O.silu(gu[:, :F]) * gu[:, F:]), a[3], 1e-2, f"layer {layer} hidden")
        # down projection into the residual on the GPU's codes
        vlm.gemm_nvfp4(vlm.EPI_RESID, (hq, hsf, a_dev[3]), w["down"], x)
        torch.cuda.synchronize()
        ch, bh = _codes(hq, hsf, T, F)
        x_ref = x_cur + O.nvfp4_linear(ch, bh, a[3], *lq["down"])
        np.testing.assert_allclose(to_np(x), x_ref, rtol=0, atol=2e-5 * np.abs(x_ref).max())
    # the encoder ran exactly this chain
    assert torch.equal(x.to(torch.bfloat16), enc), "vlm_encode_nvfp4 differs from the kernel chain"
    # and it is NVFP4: the bf16 oracle tower is further away than bf16 rounding
    x_bf16 = O.tower([im.double().numpy() for im in imgs], tw64, ocfg)
    assert np.abs(to_np(enc) - x_bf16).max() / np.abs(x_bf16).max() > 3e-3


# NVFP4 end to end: a rounding-level change of any GEMM input re-rounds a share
# of the codes downstream (attention spreads a change over its whole block),
# and each re-rounded value moves by up to a third of its block's maximum. The
# oracle against itself with its activations perturbed by 1e-5..1e-3 (relative)
# before every quantisation differs by 5.2e-2..6.2e-2 (max relative) and a
# minimum row cosine of 0.9976..0.998 on these workloads (2 layers), so the
# end-to-end bound is twice that: max relative 0.1, row cosine >= 0.995. The
# stepwise test above is where exactness is checked.
E2E_MAX_REL, E2E_MIN_COS = 0.1, 0.995


def test_encode_nvfp4_matches_oracle_nvfp4_tower():
    sizes = [(224, 224), (112, 168)]
    cfg, tw, pw, act, imgs = _nvfp4_setup(sizes)
    pipe = vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), sizes, nvfp4_act_scales=act)
    emb = pipe(pixels_to_device(imgs))
    assert vlm.status_sync(pipe.status) == vlm.OK
    ocfg = dict(O.MISTRAL3, layers=2)
    imgs64 = [im.double().numpy() for im in imgs]
    x_ref = O.tower_nvfp4(imgs64, to_oracle(tw), act, ocfg)
    compare(pipe.tower_out, x_ref, max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS, what="nvfp4 tower")
    grids = [O.patch_grid(h, w, 14) for h, w in sizes]
    compare(emb, O.projector(x_ref, grids, to_oracle(pw), ocfg), max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS,
            what="nvfp4 tower + projector")


def test_encode_nvfp4_1540_two_layers_every_row_vs_oracle():
    """One 1540x1540 image ("Mistral 3", `Mistral3Model`, image_size 1540):
    12,100 patches in one attention block, every row against the oracle."""
    sizes = [(1540, 1540)]
    cfg, tw, pw, act, imgs = _nvfp4_setup(sizes, seed=9)
    pipe = vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), sizes, nvfp4_act_scales=act)
    emb = pipe(pixels_to_device(imgs))
    assert vlm.status_sync(pipe.status) == vlm.OK
    ocfg = dict(O.MISTRAL3, layers=2)
    x_ref = O.tower_nvfp4([im.double().numpy() for im in imgs], to_oracle(tw), act, ocfg)
    compare(pipe.tower_out, x_ref, max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS, what="nvfp4 1540 tower")
    compare(emb, O.projector(x_ref, [(110, 110)], to_oracle(pw), ocfg), max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS,
            what="nvfp4 1540 projector")


def test_encode_nvfp4_isolation_and_determinism_full_size():
    """24 layers on two images: each image's rows equal its rows when run alone
    (bit-identical), two runs agree bit for bit, and the output is finite."""
    sizes = [(1540, 1540), (448, 672)]
    cfg, tw, pw, act, imgs = _nvfp4_setup(sizes, layers=24, seed=8)
    twd, pwd = tower_to_device(tw), tower_to_device(pw)
    pipe = vlm.ImagePipeline(cfg, twd, pwd, sizes, nvfp4_act_scales=act)
    pix = pixels_to_device(imgs)
    pipe(pix)
    first = pipe.tower_out.clone()
    pipe(pix)
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(first, pipe.tower_out)
    assert torch.isfinite(first.float()).all()
    alone = vlm.ImagePipeline(cfg, twd, pwd, sizes[1:], nvfp4_act_scales=act)
    alone(pixels_to_device(imgs[1:]))
    assert vlm.status_sync(alone.status) == vlm.OK
    assert torch.equal(first[12100:], alone.tower_out)


def test_encode_nvfp4_rejects_bad_inputs():
    cfg, tw, pw, act, imgs = _nvfp4_setup([(112, 112)], layers=1)
    twd = tower_to_device(tw)
    with pytest.raises(vlm.VlmError):
        vlm.pack_tower_nvfp4(cfg, twd, [[1.0, 0.0, 1.0, 1.0]])       # a scale that is not > 0
    packed = vlm.pack_tower_nvfp4(cfg, twd, act)
    pix = pixels_to_device(imgs)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(vlm.VlmError):
        vlm.encode_nvfp4(cfg, pix, [(112, 112)], packed, act, workspace=small)


def test_encode_nvfp4_zero_layers_is_the_bf16_encoder():
    """Without blocks the NVFP4 encoder is patch embed + ln_pre, as the bf16 one."""
    sizes = [(224, 224), (112, 168)]
    cfg, tw, pw, act, imgs = _nvfp4_setup(sizes, layers=0)
    twd, pix = tower_to_device(tw), pixels_to_device(imgs)
    a = vlm.encode_nvfp4(cfg, pix, sizes, vlm.pack_tower_nvfp4(cfg, twd, act), act)
    b = vlm.encode(cfg, pix, sizes, vlm.pack_tower(cfg, twd))
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_encode_nvfp4_tiny_batch_vs_oracle():
    """28 patches: every GEMM's rows are a fraction of one 128-row scale group
    (the padding rows' scales stay 0) and of one 256-row tile."""
    sizes = [(28, 28), (56, 84)]
    cfg, tw, pw, act, imgs = _nvfp4_setup(sizes, layers=2, seed=11)
    pipe = vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), sizes, nvfp4_act_scales=act)
    emb = pipe(pixels_to_device(imgs))
    assert vlm.status_sync(pipe.status) == vlm.OK
    ocfg = dict(O.MISTRAL3, layers=2)
    x_ref = O.tower_nvfp4([im.double().numpy() for im in imgs], to_oracle(tw), act, ocfg)
    compare(pipe.tower_out, x_ref, max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS, what="nvfp4 tiny tower")
    grids = [O.patch_grid(h, w, 14) for h, w in sizes]
    compare(emb, O.projector(x_ref, grids, to_oracle(pw), ocfg), max_rel=E2E_MAX_REL, min_cos=E2E_MIN_COS,
            what="nvfp4 tiny projector")
