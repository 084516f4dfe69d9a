"""Per-kernel parity of the sm_100a kernels against the CPU oracle.

Every call goes through the C-ABI (include/vlm_kernels.h, include/vlm.h).
Inputs are seeded; sizes span several tiles and end in a ragged tail; the
full-size cases use the shapes of a 1540x1540 image (12,100 patches) and are
checked on sampled rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import compare, to_np, guarded, guarded_copy
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu


def _randn(seed, name, shape, std=1.0):
    return synth.randn_bf16(seed, name, shape, std).cuda()


# ---------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (300, 256, 640), (1000, 1024, 1024), (129, 3072, 128),
                                   (4097, 512, 4096)])
def test_gemm_bf16_store(M, N, K):
    a = _randn(1, "a", (M, K))
    b = _randn(1, "b", (N, K), 0.05)
    c = guarded((M, N), dtype=torch.bfloat16)
    vlm.gemm(vlm.EPI_BF16, a, b, c)
    ref = to_np(a) @ to_np(b).T
    compare(c, ref, max_rel=1e-2, min_cos=0.9999, what="gemm bf16")


@pytest.mark.parametrize("M,N,K", [(333, 1024, 640), (130, 128, 64)])
def test_gemm_f32_and_resid(M, N, K):
    a = _randn(2, "a", (M, K))
    b = _randn(2, "b", (N, K), 0.05)
    c = guarded((M, N), dtype=torch.float32)
    vlm.gemm(vlm.EPI_F32, a, b, c)
    ref = to_np(a) @ to_np(b).T
    compare(c, ref, max_rel=1e-5, min_cos=0.999999, what="gemm f32")
    base = torch.randn((M, N), generator=synth.generator(2, "resid"), dtype=torch.float32).cuda()
    c2 = base.clone()
    cb = guarded((M, N), dtype=torch.bfloat16)
    vlm.gemm(vlm.EPI_RESID, a, b, c2, out_bf16=cb)
    ref2 = to_np(base) + ref
    compare(c2, ref2, max_rel=1e-5, min_cos=0.999999, what="gemm resid")
    compare(cb, ref2, max_rel=1e-2, min_cos=0.9999, what="gemm resid bf16 copy")


def _interleave(gate, up):
    f, d = gate.shape
    g = gate.reshape(f // 16, 16, d)
    u = up.reshape(f // 16, 16, d)
    return torch.stack([g, u], dim=1).reshape(2 * f, d).contiguous()


@pytest.mark.parametrize("M,F,K", [(513, 256, 256), (200, 4096, 1024)])
def test_gemm_swiglu(M, F, K):
    a = _randn(3, "a", (M, K))
    wg = _randn(3, "wg", (F, K), 0.05)
    wu = _randn(3, "wu", (F, K), 0.05)
    c = guarded((M, F), dtype=torch.bfloat16)
    vlm.gemm(vlm.EPI_SWIGLU, a, _interleave(wg, wu), c)
    an = to_np(a)
    ref = O.silu(an @ to_np(wg).T) * (an @ to_np(wu).T)
    compare(c, ref, what="gemm swiglu")


def test_gemm_gelu():
    a = _randn(4, "a", (700, 512))
    b = _randn(4, "b", (1280, 512), 0.08)
    c = guarded((700, 1280), dtype=torch.bfloat16)
    vlm.gemm(vlm.EPI_GELU, a, b, c)
    compare(c, O.gelu(to_np(a) @ to_np(b).T), what="gemm gelu")


@pytest.mark.parametrize("h,w", [(7, 9), (110, 110)])
def test_gemm_qkv_rope(h, w):
    D = 1024
    M = h * w
    a = _randn(5, "a", (M, D))
    b = _randn(5, "b", (3 * D, D), 0.05)
    rows, cols, _ = O.positions([(h, w)])
    pos = torch.from_numpy((rows << 16 | cols).astype(np.int32)).cuda()
    tab = vlm.rope_table(1e4, 64, max(h, w))
    c = guarded((M, 3 * D), dtype=torch.bfloat16)
    vlm.gemm(vlm.EPI_ROPE, a, b, c, pos=pos, rope_table=tab, rope_cols=2 * D)
    acc = to_np(a) @ to_np(b).T
    ang = O.rope_angles(rows, cols, 1e4, 64)
    q = O.apply_rope(acc[:, :D].reshape(M, 16, 64), ang).reshape(M, D)
    k = O.apply_rope(acc[:, D:2 * D].reshape(M, 16, 64), ang).reshape(M, D)
    ref = np.concatenate([q, k, acc[:, 2 * D:]], axis=1)
    compare(c, ref, max_rel=1e-2, min_cos=0.9999, what="gemm qkv rope")


def test_rope_table_values():
    tab = to_np(vlm.rope_table(1e4, 64, 50))
    ang = O.rope_angles(np.arange(50), np.zeros(50), 1e4, 64)[:, :16]
    np.testing.assert_allclose(tab[:, :16, 0], np.cos(ang), atol=2e-7)
    np.testing.assert_allclose(tab[:, :16, 1], np.sin(ang), atol=2e-7)
    angc = O.rope_angles(np.zeros(50), np.arange(50), 1e4, 64)[:, 16:]
    np.testing.assert_allclose(tab[:, 16:, 0], np.cos(angc), atol=2e-7)


def test_gemm_full_size_sampled():
    """The QKV projection of a 1540x1540 image: [12100, 1024] x [3072, 1024]^T."""
    M, N, K = 12100, 3072, 1024
    a = _randn(6, "a", (M, K))
    b = _randn(6, "b", (N, K), 0.05)
    c = guarded((M, N), dtype=torch.bfloat16)
    vlm.gemm(vlm.EPI_BF16, a, b, c)
    rows = np.random.default_rng(0).choice(M, 64, replace=False)
    rows = np.concatenate([rows, [0, 127, 128, M - 1]])
    ref = to_np(a[rows]) @ to_np(b).T
    compare(c[rows], ref, max_rel=1e-2, min_cos=0.9999, what="gemm full size")


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _qkv(seed, T, heads=16, q_scale=1.0):
    q = synth.randn_bf16(seed, "q", (T, heads, 64), q_scale)
    k = synth.randn_bf16(seed, "k", (T, heads, 64), 1.0)
    v = synth.randn_bf16(seed, "v", (T, heads, 64), 1.0)
    qkv = torch.cat([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], dim=1).cuda().contiguous()
    return qkv, q.double().numpy(), k.double().numpy(), v.double().numpy()


@pytest.mark.parametrize("cu", [[0, 1], [0, 1, 65, 200, 457], [0, 128, 256], [0, 300], [0, 64, 64, 191]])
@pytest.mark.parametrize("q_scale", [1.0, 0.3, 6.0])
def test_attention_blocks(cu, q_scale):
    T = cu[-1]
    qkv, q, k, v = _qkv(7, T, q_scale=q_scale)
    out = vlm.attention(qkv, cu, 16)
    compare(out, O.attention(q, k, v, cu), what=f"attention {cu}")


def test_attention_single_patch_is_v():
    qkv, q, k, v = _qkv(8, 1)
    out = vlm.attention(qkv, [0, 1], 16)
    # one key: probability exactly 1, so the output is v itself
    np.testing.assert_array_equal(to_np(out), v.reshape(1, -1))


def test_attention_full_size_sampled():
    """One 1540x1540 image: a single block of 12,100 patches, 16 heads."""
    T = 12100
    qkv, q, k, v = _qkv(9, T)
    out = vlm.attention(qkv, [0, T], 16)
    rows = np.concatenate([np.random.default_rng(1).choice(T, 24, replace=False), [0, T - 1]])
    compare(out[rows], O.attention_rows(q, k, v, [0, T], rows), what="attention full size")


def test_attention_pixtral_tiles_sampled():
    """16 tiles of 4,096 patches (a 4096x4096 Pixtral image)."""
    cu = [4096 * i for i in range(17)]
    T = cu[-1]
    qkv, q, k, v = _qkv(10, T, q_scale=0.5)
    out = vlm.attention(qkv, cu, 16)
    rows = np.concatenate([np.random.default_rng(2).choice(T, 24, replace=False), [4095, 4096, T - 1]])
    compare(out[rows], O.attention_rows(q, k, v, cu, rows), what="attention tiles")


# ---------------------------------------------------------------------------
# RMSNorm
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rows", [1, 1000, 12100])
def test_rmsnorm(rows):
    x = torch.randn((rows, 1024), generator=synth.generator(11, "x"), dtype=torch.float32) * 3
    g0 = synth.gain(11, "g0", (1024,))
    g1 = synth.gain(11, "g1", (1024,))
    xd = guarded_copy(x)
    out = vlm.rmsnorm(xd, g1.cuda())
    compare(out, O.rms_norm(x.double().numpy(), g1.double().numpy(), 1e-5), max_rel=8e-3, min_cos=0.9999,
            what="rmsnorm")
    xd2 = guarded_copy(x)
    out2 = vlm.rmsnorm(xd2, g1.cuda(), g0=g0.cuda())
    y = O.rms_norm(x.double().numpy(), g0.double().numpy(), 1e-5)
    compare(xd2, y, max_rel=1e-5, min_cos=0.999999, what="rmsnorm in-place")
    compare(out2, O.rms_norm(y, g1.double().numpy(), 1e-5), max_rel=8e-3, min_cos=0.9999, what="rmsnorm twice")


# ---------------------------------------------------------------------------
# Scatter (bit-exact)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n_seq,seq_len,runs,width", [
    (4, 4096, [[1536]] * 4, 5120), (1, 300, [[3, 50, 7]], 64), (2, 1, [[1], []], 16), (3, 257, [[0], [256], [1]], 128),
    (8, 4096, [[1536]] * 8, 256),                 # 32,768 ids: the largest single-launch scatter
    (2, 20000, [[5000, 3000], [7000]], 64),       # 40,000 ids: the multi-kernel path
])
def test_scatter_bit_exact(n_seq, seq_len, runs, width):
    ids = synth.text_sequences(12, n_seq, seq_len, runs)
    n_img = int((ids == 10).sum())
    img = synth.randn_bf16(12, "img", (n_img, width), 1.0)
    text = synth.text_embeddings(12, n_seq * seq_len, width)
    ref = O.scatter(ids.numpy(), img.view(torch.int16).numpy(), text.view(torch.int16).numpy(), 10)
    t_gpu = guarded_copy(text)
    status = vlm.new_status()
    vlm.scatter(ids.reshape(-1).cuda(), img.cuda(), t_gpu, 10, status=status)
    assert vlm.status_sync(status) == vlm.OK
    assert np.array_equal(t_gpu.view(torch.int16).cpu().numpy(), ref)


@pytest.mark.parametrize("seq_len,run,n_img", [(500, 40, 39), (500, 40, 41), (100, 10, 600), (40000, 900, 899)],
                         ids=["fewer_rows", "more_rows", "more_rows_than_ids", "multi_kernel"])
def test_scatter_count_mismatch_writes_nothing(seq_len, run, n_img):
    ids = synth.text_sequences(13, 1, seq_len, [[run]])
    img = synth.randn_bf16(13, "img", (n_img, 256), 1.0)
    text = synth.text_embeddings(13, seq_len, 256)
    t_gpu = guarded_copy(text)
    status = vlm.new_status()
    vlm.scatter(ids.reshape(-1).cuda(), img.cuda(), t_gpu, 10, status=status)
    assert vlm.status_sync(status) == vlm.ERR_COUNT_MISMATCH
    assert torch.equal(t_gpu.cpu().view(torch.int16), text.view(torch.int16))


# ---------------------------------------------------------------------------
# Failure detection: a barrier wait that runs out reports, it does not hang
# ---------------------------------------------------------------------------

def test_bounded_wait_times_out_into_status_and_context_survives():
    status = vlm.new_status()
    vlm.selftest_wait_timeout(2_000_000, status)  # ~1 ms of SM clocks
    assert vlm.status_sync(status) == vlm.ERR_TIMEOUT
    # the context is still usable: a normal call after it succeeds
    qkv, q, k, v = _qkv(8, 1)
    out = vlm.attention(qkv, [0, 1], 16)
    np.testing.assert_array_equal(to_np(out), v.reshape(1, -1))


def test_attention_last_wave_rows_single_block():
    """16 heads x 95 query tiles = 1,520 CTAs: rows of the CTAs of the partial
    last wave (head 15, query tiles 55..94) and rows outside it, with peaked
    scores."""
    T = 12100
    qkv, q, k, v = _qkv(12, T, q_scale=2.0)
    out = vlm.attention(qkv, [0, T], 16)
    rng = np.random.default_rng(3)
    rows = np.concatenate([rng.choice(np.arange(55 * 128, T), 20, replace=False), rng.choice(55 * 128, 6), [T - 1]])
    compare(out[rows], O.attention_rows(q, k, v, [0, T], rows), what="attention last wave")


def test_attention_many_small_blocks_last_wave():
    """300 blocks of 131 keys (2 key tiles each, the second one almost all
    masked): rows of the last blocks (in the last wave) and others."""
    cu = [131 * i for i in range(301)]
    T = cu[-1]
    qkv, q, k, v = _qkv(13, T, q_scale=2.0)
    out = vlm.attention(qkv, cu, 16)
    rng = np.random.default_rng(4)
    rows = np.concatenate([rng.choice(np.arange(236 * 131, T), 24, replace=False), rng.choice(236 * 131, 6),
                           [T - 1, 236 * 131, 299 * 131 + 128]])
    compare(out[rows], O.attention_rows(q, k, v, cu, rows), what="attention small blocks")
