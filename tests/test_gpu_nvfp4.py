"""Parity of the NVFP4 operands and the block-scaled GEMM with the oracle:
quantisation codes and block scales bit-exact, the global scale exact, and
the GEMM against the oracle's exact blocked sums (bit-exact where every
partial sum is representable in fp32, else within fp32 accumulation error).

The packing helpers below (E2M1 codes into bytes, block scales into their
512-byte atoms) are written here from the format's definition, independently
of the library, so a layout mistake on either side fails a comparison.
"""
import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import compare, to_np, guarded, guarded_zeros
from vision_language_model_b200 import vlm

pytestmark = pytest.mark.gpu

_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _codes_from_values(q: np.ndarray) -> np.ndarray:
    """E2M1 values -> 4-bit codes s.ee.m (magnitude index in the low 3 bits)."""
    mag = np.searchsorted(_MAGS, np.abs(q))
    assert np.all(_MAGS[mag] == np.abs(q)), "value off the E2M1 grid"
    return (mag | (np.signbit(q) & (q != 0)) * 8).astype(np.uint8)


def _pack_codes(q: np.ndarray) -> torch.Tensor:
    c = _codes_from_values(q)
    return torch.from_numpy((c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)).cuda()


def _unpack_codes(b: torch.Tensor) -> np.ndarray:
    b = b.cpu().numpy()
    c = np.empty((b.shape[0], 2 * b.shape[1]), np.uint8)
    c[:, 0::2], c[:, 1::2] = b & 15, b >> 4
    v = _MAGS[c & 7]
    return np.where(c & 8, -v, v)


def _sf_index(rows: int, k: int) -> np.ndarray:
    """Byte offset of every (row, block) scale in the atom layout."""
    r = np.arange(rows)[:, None]
    j = np.arange(k // 16)[None, :]
    atom = (r // 128) * (k // 64) + j // 4
    return atom * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + j % 4


def _pack_sf(s: np.ndarray, k: int) -> torch.Tensor:
    rows = s.shape[0]
    buf = np.zeros(vlm.nvfp4_sf_bytes(rows, k), np.uint8)
    codes = torch.from_numpy(s.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.all(torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy() == s)
    buf[_sf_index(rows, k)] = codes
    return torch.from_numpy(buf).cuda()


def _unpack_sf(sf: torch.Tensor, rows: int, k: int) -> np.ndarray:
    b = sf.cpu()
    return b[torch.from_numpy(_sf_index(rows, k))].view(torch.float8_e4m3fn).double().numpy()


def _dev_scalar(v) -> torch.Tensor:
    return torch.tensor([float(np.float32(v))], dtype=torch.float32, device="cuda")


def _operand(q, s, g, k):
    return _pack_codes(q), _pack_sf(s, k), _dev_scalar(g)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quant_nvfp4_codes_and_scales_bit_exact(dtype):
    rng = np.random.default_rng(61)
    rows, k = 300, 1024
    x = rng.standard_normal((rows, k)) * np.exp2(rng.uniform(-4, 4, (rows, 1)))
    x[7, 32:48] = 0.0                        # an all-zero block
    x[9, :16] = 1e-30                        # a block whose scale underflows to 0
    xt = torch.from_numpy(x).to(dtype)
    x32 = xt.float().numpy()                 # the exact values the kernel reads
    for sg in (O.nvfp4_global_scale(x32), np.float32(O.nvfp4_global_scale(x32) / 64)):  # the second saturates
        q, sf = vlm.quant_nvfp4(xt.cuda(), _dev_scalar(sg))
        torch.cuda.synchronize()
        q_ref, s_ref = O.quantize_nvfp4(x32, sg)
        np.testing.assert_array_equal(_unpack_sf(sf, rows, k), s_ref)
        np.testing.assert_array_equal(_unpack_codes(q), q_ref)
        # the 84 pad rows of the last 128-row group carry scale 0
        pad = _unpack_sf(sf, 384, k)[rows:]
        assert np.all(pad == 0)


def test_amax_scale_matches_oracle_global_scale():
    rng = np.random.default_rng(62)
    for dtype in (torch.bfloat16, torch.float32):
        x = torch.from_numpy(rng.standard_normal((777, 333)) * 3).to(dtype)
        got = vlm.amax_scale(x.cuda())
        torch.cuda.synchronize()
        assert got.item() == float(O.nvfp4_global_scale(x.float().numpy()))


def _random_operand(rng, rows, k, exps=(-6, 7)):
    q = rng.choice([c for c in np.concatenate([_MAGS, -_MAGS[1:]])], size=(rows, k))
    s = np.exp2(rng.integers(exps[0], exps[1], size=(rows, k // 16))).astype(np.float64)
    s *= rng.choice([1.0, 1.25, 1.5, 1.75], size=s.shape)  # E4M3 mantissas
    return q, s


def test_gemm_nvfp4_exact_when_partial_sums_are_representable():
    """Power-of-two scales in a narrow range keep every partial sum a multiple
    of 2^-6 below 2^18: fp32 accumulation is exact in any order, so the GEMM
    must reproduce the exact blocked sum bit for bit. Scales differ from block
    to block, so a scale taken from the wrong row or block shows."""
    rng = np.random.default_rng(63)
    M, N, K = 300, 256, 256
    qa, _ = _random_operand(rng, M, K)
    qb, _ = _random_operand(rng, N, K)
    sa = np.exp2(rng.integers(-2, 3, size=(M, K // 16))).astype(np.float64)
    sb = np.exp2(rng.integers(-2, 3, size=(N, K // 16))).astype(np.float64)
    ref = O.nvfp4_linear(qa, sa, 1.0, qb, sb, 1.0)
    out = guarded_zeros((M, N), dtype=torch.float32)
    st = vlm.new_status()
    vlm.gemm_nvfp4(vlm.EPI_RESID, _operand(qa, sa, 1.0, K), _operand(qb, sb, 1.0, K), out, status=st)
    torch.cuda.synchronize()
    assert vlm.status_sync(st) == vlm.OK
    np.testing.assert_array_equal(to_np(out), ref)


@pytest.mark.parametrize("M,N,K", [(300, 256, 512), (1000, 384, 1024), (77, 128, 256), (1, 128, 256),
                                   (129, 256, 768), (640, 1024, 4096)])
def test_gemm_nvfp4_bf16_and_resid_epilogues(M, N, K):
    rng = np.random.default_rng(M + N + K)
    qa, sa = _random_operand(rng, M, K)
    qb, sb = _random_operand(rng, N, K)
    ga, gb = np.float32(2.0 ** -3 * 1.3), np.float32(2.0 ** -9 * 0.7)
    ref = O.nvfp4_linear(qa, sa, ga, qb, sb, gb)
    a, b = _operand(qa, sa, ga, K), _operand(qb, sb, gb, K)
    st = vlm.new_status()
    out = guarded((M, N), dtype=torch.bfloat16)
    vlm.gemm_nvfp4(vlm.EPI_BF16, a, b, out, status=st)
    torch.cuda.synchronize()
    assert vlm.status_sync(st) == vlm.OK
    compare(out, ref, max_rel=8e-3, min_cos=0.99999, what="nvfp4 gemm bf16")
    x0 = rng.standard_normal((M, N)).astype(np.float32)
    x = torch.from_numpy(x0).cuda()
    vlm.gemm_nvfp4(vlm.EPI_RESID, a, b, x, status=st)
    torch.cuda.synchronize()
    # fp32 accumulation in the tensor core's order: bound relative to the sums' scale
    np.testing.assert_allclose(to_np(x), x0 + ref, rtol=0, atol=2e-5 * np.abs(ref).max())


@pytest.mark.parametrize("N,K", [(3072, 1024), (1024, 1024), (8192, 1024), (1024, 4096)])
def test_tower_shapes_quantise_and_multiply_on_sampled_rows(N, K):
    """The tower's four GEMM shapes on 12,100 rows (one 1540x1540 image): bf16
    activations and weights quantised on the GPU (global scales from the data
    for the weights, a static one for the activations), product checked on a
    sample of rows against the oracle quantising the same inputs itself."""
    rng = np.random.default_rng(N + K)
    M = 12100
    x = torch.from_numpy(rng.standard_normal((M, K)) * 2).to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((N, K)) * 0.02).to(torch.bfloat16)
    sg_a = np.float32(12.0 / 2688.0)
    xd, wd = x.cuda(), w.cuda()
    ga = _dev_scalar(sg_a)
    gw = vlm.amax_scale(wd)
    qa, sfa = vlm.quant_nvfp4(xd, ga)
    qw, sfw = vlm.quant_nvfp4(wd, gw)
    out = guarded((M, N), dtype=torch.bfloat16)
    st = vlm.new_status()
    vlm.gemm_nvfp4(vlm.EPI_BF16, (qa, sfa, ga), (qw, sfw, gw), out, status=st)
    torch.cuda.synchronize()
    assert vlm.status_sync(st) == vlm.OK
    rows = np.sort(np.concatenate([rng.choice(M, 48, replace=False), [0, 255, 256, 12031, M - 1]]))
    x32, w32 = x.float().numpy(), w.float().numpy()
    sg_w = O.nvfp4_global_scale(w32)
    assert gw.item() == float(sg_w)
    q_w, s_w = O.quantize_nvfp4(w32, sg_w)
    q_x, s_x = O.quantize_nvfp4(x32[rows], sg_a)
    ref = O.nvfp4_linear(q_x, s_x, sg_a, q_w, s_w, sg_w)
    compare(out[torch.from_numpy(rows).cuda()], ref, max_rel=8e-3, min_cos=0.99999, what=f"nvfp4 {N}x{K}")
    # and the NVFP4 product stays close to the unquantised one
    exact = x32[rows].astype(np.float64) @ w32.astype(np.float64).T
    rel = np.abs(ref - exact).max() / np.abs(exact).max()
    assert 1e-3 < rel < 0.25, rel


def _pow2_operand(rng, rows, k):
    q = rng.choice(np.concatenate([_MAGS, -_MAGS[1:]]), size=(rows, k))
    s = np.exp2(rng.integers(-2, 1, size=(rows, k // 16))).astype(np.float64)
    return q, s


@pytest.mark.parametrize("N,K", [(1024, 4096), (8192, 1024)])
def test_gemm_nvfp4_exact_and_repeatable_at_tower_shapes(N, K):
    """The tower's row count with a long K loop (16 stages of 256 values per
    tile) and with many tiles: block scales in {1/4, 1/2, 1} keep every term a
    multiple of 2^-6 of magnitude <= 36, so every partial sum over K <= 4096 is
    exact in fp32 and sampled rows must equal the oracle bit for bit. A block
    scale read from tensor memory before its copy has landed, or from another
    stage's scale slot, breaks that; 20 further launches must agree bit for bit
    with the first."""
    rng = np.random.default_rng(N + 3 * K)
    M = 12100
    qa, sa = _pow2_operand(rng, M, K)
    qb, sb = _pow2_operand(rng, N, K)
    a, b = _operand(qa, sa, 1.0, K), _operand(qb, sb, 1.0, K)
    out = guarded_zeros((M, N), dtype=torch.float32)
    st = vlm.new_status()
    vlm.gemm_nvfp4(vlm.EPI_RESID, a, b, out, status=st)
    torch.cuda.synchronize()
    assert vlm.status_sync(st) == vlm.OK
    rows = np.sort(np.concatenate([rng.choice(M, 60, replace=False), [0, 127, 128, 255, 256, 12031, M - 1]]))
    ref = O.nvfp4_linear(qa[rows], sa[rows], 1.0, qb, sb, 1.0)
    np.testing.assert_array_equal(to_np(out[torch.from_numpy(rows).cuda()]), ref)
    first = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    vlm.gemm_nvfp4(vlm.EPI_BF16, a, b, first, status=st)
    again = torch.empty_like(first)
    for _ in range(20):
        vlm.gemm_nvfp4(vlm.EPI_BF16, a, b, again, status=st)
        assert torch.equal(again, first)
    assert vlm.status_sync(st) == vlm.OK
