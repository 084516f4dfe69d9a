"""Host-side checks of the C-ABI library (no GPU needed).

The library must load, export every function that include/*.h declares, and
reject bad arguments on the host before launching anything.
"""
import ctypes
import os
import re

import pytest

from vision_language_model_b200 import vlm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"VLM_API\s+[\w\s\*]+?\b(vlm_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(vlm.lib_path()):
        from vision_language_model_b200 import build
        build.build()
    return vlm.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"vlm_encode", "vlm_merge_project", "vlm_scatter", "vlm_gemm", "vlm_attention"} <= names
    for n in sorted(names):
        assert hasattr(L, n), n


def test_presets_match_pages(L):
    m = vlm.preset("mistral3")
    assert (m.layers, m.width, m.heads, m.head_dim, m.mlp, m.patch, m.merge, m.proj_out, m.image_token_id) == \
        (24, 1024, 16, 64, 4096, 14, 2, 5120, 10)
    assert m.rope_theta == 10000.0 and abs(m.eps - 1e-5) < 1e-12
    p = vlm.preset("pixtral12b")
    assert (p.patch, p.merge) == (16, 1)


def test_patch_and_merged_counts(L):
    m = vlm.preset("mistral3")
    assert vlm.num_patches(m, [(1540, 1540)]) == 12100
    assert vlm.num_merged(m, [(1540, 1540)]) == 3025
    assert vlm.num_patches(m, [(896, 1344)] * 4) == 4 * 6144
    assert vlm.num_merged(m, [(896, 1344)] * 4) == 4 * 1536
    p = vlm.preset("pixtral12b")
    assert vlm.num_patches(p, [(1024, 1024)] * 16) == 65536
    assert vlm.num_merged(p, [(1024, 1024)] * 16) == 65536


@pytest.mark.parametrize("hw", [[(225, 224)], [(14 * 3, 28)], []])
def test_bad_shapes_rejected_on_host(L, hw):
    m = vlm.preset("mistral3")
    with pytest.raises(vlm.VlmError) as e:
        vlm.num_patches(m, hw)
    assert e.value.rc == vlm.ERR_BAD_SHAPE


def test_norm_after_merge_flag_checked(L):
    c = vlm.preset("mistral3")
    assert c.norm_after_merge == 0
    c.norm_after_merge = 2
    hw = (ctypes.c_int32 * 2)(224, 224)
    assert L.vlm_num_patches(ctypes.byref(c), hw, 1) == vlm.ERR_INVALID_ARG


def test_negative_sm_budget_rejected(L):
    cfg = vlm.preset("mistral3", sm_budget=-1)
    arr = (ctypes.c_int32 * 2)(224, 224)
    assert L.vlm_num_patches(ctypes.byref(cfg), arr, 1) == vlm.ERR_INVALID_ARG
    cfg.sm_budget = 64
    assert L.vlm_num_patches(ctypes.byref(cfg), arr, 1) == 256


def test_unsupported_config_rejected(L):
    with pytest.raises(vlm.VlmError) as e:
        vlm.num_patches(vlm.preset("mistral3", head_dim=128, heads=8), [(28, 28)])
    assert e.value.rc == vlm.ERR_UNSUPPORTED
    assert L.vlm_tower_packed_bytes(ctypes.byref(vlm.preset("mistral3", width=1000))) == 0


def test_workspace_sizes_cover_buffers(L):
    m = vlm.preset("mistral3")
    ws = vlm.encode_workspace_size(m, [(1540, 1540)])
    T, D, F = 12100, 1024, 4096
    assert ws >= T * D * 4 + T * D * 2 * 2 + T * 3 * D * 2 + T * F * 2
    assert vlm.merge_project_workspace_size(m, [(1540, 1540)]) >= 3025 * 5120 * 2
    assert vlm.scatter_workspace_size(16384) >= 16384 * 8


def test_scatter_argument_errors_return_before_launch(L):
    null = None
    # row_bytes not a multiple of 16
    rc = L.vlm_scatter(null, 4, 10, null, 0, null, 10, null, 0, null, null)
    assert rc == vlm.ERR_INVALID_ARG
    # empty id list with image rows
    rc = L.vlm_scatter(null, 0, 10, null, 3, null, 16, null, 0, null, null)
    assert rc == vlm.ERR_BAD_SHAPE
    # null pointers
    rc = L.vlm_scatter(null, 4, 10, null, 1, null, 16, null, 1 << 20, null, null)
    assert rc == vlm.ERR_INVALID_ARG


def test_status_strings(L):
    assert vlm.status_string(vlm.ERR_COUNT_MISMATCH) == "VLM_ERR_COUNT_MISMATCH"
    assert vlm.status_string(vlm.ERR_TIMEOUT) == "VLM_ERR_TIMEOUT"
    assert vlm.status_string(123) == "VLM_ERR_UNKNOWN"


def test_gemm_shape_checks_return_before_launch(L):
    fake = ctypes.c_void_p(256)
    st = None
    assert L.vlm_gemm(0, fake, fake, 128, 100, 64, fake, None, None, None, 0, st, None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm(0, fake, fake, 128, 128, 60, fake, None, None, None, 0, st, None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm(3, fake, fake, 128, 384, 64, fake, None, None, None, 0, st, None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm(0, None, fake, 128, 128, 64, fake, None, None, None, 0, st, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_gemm(0, fake, fake, 0, 128, 64, fake, None, None, None, 0, st, None) == vlm.ERR_BAD_SHAPE
    # epilogue codes outside the public set (6 is the projector's internal row-scattered store)
    for epi in (-1, 6, 7):
        assert L.vlm_gemm(epi, fake, fake, 128, 256, 64, fake, None, None, None, 0, st, None) == vlm.ERR_INVALID_ARG


def test_package_import_does_not_load_library():
    import importlib
    import sys
    for k in [k for k in sys.modules if k.startswith("vision_language_model_b200")]:
        sys.modules.pop(k)
    pkg = importlib.import_module("vision_language_model_b200")
    assert not hasattr(pkg, "_lib")


def test_resize_target_matches_oracle_sweep(L):
    """vlm_resize_target (host only) against the oracle's resized_hw, exactly."""
    from oracle import vlm_oracle as O
    import numpy as np
    rng = np.random.default_rng(7)
    sizes = [(1540, 1540), (4032, 3024), (3024, 4032), (1, 1), (27, 3000), (1541, 1540), (200, 100)]
    sizes += [tuple(int(v) for v in rng.integers(1, 9000, 2)) for _ in range(300)]
    for (h, w) in sizes:
        for edge, grid in ((1540, 28), (1540, 14), (4096, 1024), (1024, 16)):
            assert vlm.resize_target(h, w, edge, grid) == O.resized_hw(h, w, edge, grid), (h, w, edge, grid)


def test_front_end_argument_errors_return_before_launch(L):
    fake = ctypes.c_void_p(256)  # never dereferenced: every case fails validation first
    src = (ctypes.c_int32 * 2)(100, 100)
    bad_w = (ctypes.c_int32 * 2)(28, 30)       # width not a multiple of 4
    off_tile = (ctypes.c_int32 * 2)(1024, 1000)  # not a whole number of tiles
    assert L.vlm_preprocess(fake, src, 1, bad_w, 0, fake, None) == vlm.ERR_BAD_SHAPE
    assert L.vlm_preprocess(fake, src, 1, off_tile, 1024, fake, None) == vlm.ERR_BAD_SHAPE
    assert L.vlm_preprocess(fake, src, 0, src, 0, fake, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_preprocess(fake, src, 1, src, 6, fake, None) == vlm.ERR_BAD_SHAPE  # tile % 4
    assert L.vlm_preprocess(fake, src, 1, src, 0, ctypes.c_void_p(260), None) == vlm.ERR_INVALID_ARG  # unaligned
    oh, ow = ctypes.c_int32(), ctypes.c_int32()
    assert L.vlm_resize_target(0, 5, 1540, 28, ctypes.byref(oh), ctypes.byref(ow)) == vlm.ERR_INVALID_ARG
    # a longest_edge off the grid: rounding up could exceed it, so it is refused
    assert L.vlm_resize_target(2000, 1000, 1000, 28, ctypes.byref(oh), ctypes.byref(ow)) == vlm.ERR_BAD_SHAPE
    assert L.vlm_resize_target(2000, 1000, 1008, 28, ctypes.byref(oh), ctypes.byref(ow)) == vlm.OK
    assert (oh.value, ow.value) == (1008, 504)
    # placeholder expansion: output too small, and more images than ids
    counts = (ctypes.c_int64 * 2)(100, 200)
    n_out = ctypes.c_int64()
    ws = ctypes.c_void_p(1 << 20)
    assert L.vlm_expand_placeholders(fake, 10, 99, counts, 2, 10, fake, 100, ctypes.byref(n_out), ws, 1 << 20, fake,
                                     None) == vlm.ERR_WORKSPACE
    assert n_out.value == 0
    zero = (ctypes.c_int64 * 2)(0, 0)
    assert L.vlm_expand_placeholders(fake, 1, 99, zero, 2, 10, fake, 100, ctypes.byref(n_out), ws, 1 << 20, fake,
                                     None) == vlm.ERR_BAD_SHAPE
    assert L.vlm_expand_placeholders(fake, 0, 99, zero, 0, 10, fake, 0, ctypes.byref(n_out), ws, 0, fake,
                                     None) == vlm.OK and n_out.value == 0


def test_fp8_argument_errors_return_before_launch(L):
    fake = ctypes.c_void_p(256)  # never dereferenced: every case fails validation first
    cs = ctypes.c_void_p(512)
    st = ctypes.c_void_p(1024)
    # K % 128, N % 256, null colscale, unaligned operand, BF16-only epilogue set
    assert L.vlm_gemm_fp8(vlm.EPI_BF16, fake, fake, cs, 1.0, 256, 256, 64, fake, None, None, None, 0, st,
                          None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm_fp8(vlm.EPI_BF16, fake, fake, cs, 1.0, 256, 128, 128, fake, None, None, None, 0, st,
                          None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm_fp8(vlm.EPI_BF16, fake, fake, None, 1.0, 256, 256, 128, fake, None, None, None, 0, st,
                          None) == vlm.ERR_INVALID_ARG
    assert L.vlm_gemm_fp8(vlm.EPI_BF16, ctypes.c_void_p(264), fake, cs, 1.0, 256, 256, 128, fake, None, None, None,
                          0, st, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_gemm_fp8(vlm.EPI_GELU, fake, fake, cs, 1.0, 256, 256, 128, fake, None, None, None, 0, st,
                          None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_rmsnorm_fp8(fake, None, fake, fake, 4, 1024, 1e-5, 0.0, None) == vlm.ERR_INVALID_ARG
    cfg = vlm.preset("mistral3", layers=2)
    tw = vlm.TowerWeights(**{k: 256 for k, _ in vlm.TowerWeights._fields_})
    good = (ctypes.c_float * 8)(*([0.02] * 8))
    for bad_vals in ([0.02] * 7 + [0.0], [0.02] * 7 + [-1.0], [0.02] * 7 + [float("nan")], [0.02] * 7 + [float("inf")]):
        bad = (ctypes.c_float * 8)(*bad_vals)
        assert L.vlm_pack_tower_fp8(ctypes.byref(cfg), ctypes.byref(tw), bad, fake, 1 << 40, None) == \
            vlm.ERR_INVALID_ARG
    assert L.vlm_pack_tower_fp8(ctypes.byref(cfg), ctypes.byref(tw), None, fake, 1 << 40, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_pack_tower_fp8(ctypes.byref(cfg), ctypes.byref(tw), good, fake, 16, None) == vlm.ERR_WORKSPACE
    hw = (ctypes.c_int32 * 2)(224, 224)
    assert L.vlm_encode_fp8(ctypes.byref(cfg), fake, hw, 1, fake, None, fake, fake, 1 << 40, st, None) == \
        vlm.ERR_INVALID_ARG
    fp8_bytes = L.vlm_tower_fp8_packed_bytes(ctypes.byref(cfg))
    assert 0 < fp8_bytes < L.vlm_tower_packed_bytes(ctypes.byref(cfg))


def test_nvfp4_scale_sizes_and_argument_errors_return_before_launch(L):
    # one 512-byte atom per 128 rows x 64 values of K
    assert L.vlm_nvfp4_sf_bytes(1, 64) == 512
    assert L.vlm_nvfp4_sf_bytes(128, 1024) == 16 * 512
    assert L.vlm_nvfp4_sf_bytes(129, 1024) == 32 * 512
    assert L.vlm_nvfp4_sf_bytes(12100, 4096) == 95 * 64 * 512
    for rows, k in ((0, 64), (5, 0), (5, 48), (-1, 64)):
        assert L.vlm_nvfp4_sf_bytes(rows, k) == 0
    fake = ctypes.c_void_p(256)  # never dereferenced: every case fails validation first
    st = ctypes.c_void_p(1024)
    # K % 256, N % 128, a null scale pointer, an unaligned operand, an unsupported epilogue
    assert L.vlm_gemm_nvfp4(vlm.EPI_BF16, fake, fake, fake, fake, fake, fake, 256, 128, 128, fake, st,
                            None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm_nvfp4(vlm.EPI_BF16, fake, fake, fake, fake, fake, fake, 256, 192, 256, fake, st,
                            None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm_nvfp4(vlm.EPI_BF16, fake, None, fake, fake, fake, fake, 256, 128, 256, fake, st,
                            None) == vlm.ERR_INVALID_ARG
    assert L.vlm_gemm_nvfp4(vlm.EPI_BF16, fake, fake, fake, ctypes.c_void_p(264), fake, fake, 256, 128, 256, fake,
                            st, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_gemm_nvfp4(vlm.EPI_SWIGLU, fake, fake, fake, fake, fake, fake, 256, 128, 256, fake, st,
                            None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_gemm_nvfp4(vlm.EPI_BF16, fake, fake, fake, fake, fake, fake, 0, 128, 256, fake, st,
                            None) == vlm.ERR_BAD_SHAPE
    # quantiser: K % 64, bad dtype, null global scale, unaligned input
    assert L.vlm_quant_nvfp4(fake, vlm.DTYPE_BF16, 4, 96, fake, fake, fake, None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_quant_nvfp4(fake, 7, 4, 128, fake, fake, fake, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_quant_nvfp4(fake, vlm.DTYPE_F32, 4, 128, None, fake, fake, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_quant_nvfp4(ctypes.c_void_p(260), vlm.DTYPE_F32, 4, 128, fake, fake, fake, None) == \
        vlm.ERR_INVALID_ARG
    assert L.vlm_amax_scale(fake, vlm.DTYPE_BF16, 10, 0.0, fake, None) == vlm.ERR_BAD_SHAPE
    assert L.vlm_amax_scale(None, vlm.DTYPE_BF16, 10, 2688.0, fake, None) == vlm.ERR_INVALID_ARG


def test_nvfp4_tower_entry_points_reject_bad_arguments_before_launch(L):
    """Every case fails validation before any CUDA call (the fake pointers are never dereferenced)."""
    fake, st = ctypes.c_void_p(256), ctypes.c_void_p(1024)
    gx = L.vlm_gemm_nvfp4_ex
    args = lambda epi, n, c_sf=fake, sg=1.0, pos=fake, rope=fake, rc=256: (
        epi, fake, fake, fake, fake, fake, fake, 256, n, 256, fake, c_sf, sg, pos, rope, rc, st, None)
    assert gx(*args(vlm.EPI_ROPE, 512, pos=None)) == vlm.ERR_INVALID_ARG          # RoPE without positions
    assert gx(*args(vlm.EPI_ROPE, 512, rc=32)) == vlm.ERR_INVALID_ARG             # rope_cols not whole heads
    assert gx(*args(vlm.EPI_ROPE, 384)) == vlm.ERR_UNSUPPORTED                    # RoPE needs N % 256 == 0
    assert gx(*args(vlm.EPI_SWIGLU, 384)) == vlm.ERR_UNSUPPORTED
    assert gx(*args(vlm.EPI_SWIGLU, 512, c_sf=None)) == vlm.ERR_INVALID_ARG       # no hidden-state scales
    assert gx(*args(vlm.EPI_SWIGLU, 512, sg=0.0)) == vlm.ERR_INVALID_ARG          # global scale not > 0
    assert gx(*args(vlm.EPI_SWIGLU, 512, c_sf=ctypes.c_void_p(258))) == vlm.ERR_INVALID_ARG
    assert gx(*args(vlm.EPI_GELU, 512)) == vlm.ERR_UNSUPPORTED
    # RMSNorm to NVFP4: scale, scale buffer, width
    assert L.vlm_rmsnorm_nvfp4(fake, None, fake, fake, fake, 8, 1024, 1e-5, 0.0, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_rmsnorm_nvfp4(fake, None, fake, fake, None, 8, 1024, 1e-5, 1.0, None) == vlm.ERR_INVALID_ARG
    assert L.vlm_rmsnorm_nvfp4(fake, None, fake, fake, fake, 8, 100, 1e-5, 1.0, None) == vlm.ERR_UNSUPPORTED
    assert L.vlm_rmsnorm_nvfp4(fake, None, fake, fake, fake, 0, 1024, 1e-5, 1.0, None) == vlm.OK
    # attention to NVFP4: scale buffer, scale, alignment of the codes
    cu = (ctypes.c_int32 * 2)(0, 128)
    att = L.vlm_attention_nvfp4
    assert att(fake, 128, 2, 64, cu, 1, fake, None, 1.0, fake, 4096, st, None) == vlm.ERR_INVALID_ARG
    assert att(fake, 128, 2, 64, cu, 1, fake, fake, -1.0, fake, 4096, st, None) == vlm.ERR_INVALID_ARG
    assert att(fake, 128, 2, 64, cu, 1, ctypes.c_void_p(264), fake, 1.0, fake, 4096, st, None) == vlm.ERR_INVALID_ARG
    # packing and encoding
    cfg = vlm.preset("mistral3", layers=1)
    tw = vlm.TowerWeights(*([fake.value] * len(vlm.TowerWeights._fields_)))
    good = (ctypes.c_float * 4)(1.0, 1.0, 1.0, 1.0)
    bad = (ctypes.c_float * 4)(1.0, 0.0, 1.0, 1.0)
    need = L.vlm_tower_nvfp4_packed_bytes(ctypes.byref(cfg))
    assert need > 0
    pk = L.vlm_pack_tower_nvfp4
    assert pk(ctypes.byref(cfg), ctypes.byref(tw), bad, fake, need, None) == vlm.ERR_INVALID_ARG
    assert pk(ctypes.byref(cfg), None, good, fake, need, None) == vlm.ERR_INVALID_ARG
    assert pk(ctypes.byref(cfg), ctypes.byref(tw), good, ctypes.c_void_p(272), need, None) == vlm.ERR_INVALID_ARG
    assert pk(ctypes.byref(cfg), ctypes.byref(tw), good, fake, need - 1, None) == vlm.ERR_WORKSPACE
    hw = (ctypes.c_int32 * 2)(224, 224)
    ws = L.vlm_encode_nvfp4_workspace_size(ctypes.byref(cfg), hw, 1)
    assert ws > L.vlm_encode_workspace_size(ctypes.byref(cfg), hw, 1)   # plus the inputs' block scales
    enc = L.vlm_encode_nvfp4
    assert enc(ctypes.byref(cfg), None, hw, 1, fake, good, fake, fake, ws, st, None) == vlm.ERR_INVALID_ARG
    assert enc(ctypes.byref(cfg), fake, hw, 1, fake, good, fake, ctypes.c_void_p(272), ws, st, None) == \
        vlm.ERR_INVALID_ARG
    assert enc(ctypes.byref(cfg), fake, hw, 1, fake, good, fake, fake, ws - 1, st, None) == vlm.ERR_WORKSPACE
    assert enc(ctypes.byref(cfg), fake, hw, 1, fake, bad, fake, fake, ws, st, None) == vlm.ERR_INVALID_ARG
    # the patch embed alone
    pe = L.vlm_patch_embed
    ws_pe = L.vlm_encode_workspace_size(ctypes.byref(cfg), hw, 1)
    assert pe(ctypes.byref(cfg), fake, hw, 1, fake, None, fake, ws_pe, st, None) == vlm.ERR_INVALID_ARG
    assert pe(ctypes.byref(cfg), fake, hw, 1, fake, fake, ctypes.c_void_p(272), ws_pe, st, None) == vlm.ERR_INVALID_ARG
    assert pe(ctypes.byref(cfg), fake, hw, 1, fake, fake, fake, ws_pe - 1, st, None) == vlm.ERR_WORKSPACE


def test_gemm_tile_counts_that_overflow_32_bits_are_rejected(L):
    """Tile indices and scale-atom rows are 32-bit in the kernels: shapes whose
    counts would not fit are refused on the host before any launch."""
    fake = ctypes.c_void_p(256)
    st = ctypes.c_void_p(1024)
    big_m = (1 << 31) - 1
    assert L.vlm_gemm(vlm.EPI_BF16, fake, fake, big_m, 65535 * 256, 64, fake, None, None, None, 0, st,
                      None) == vlm.ERR_BAD_SHAPE
    assert L.vlm_gemm_fp8(vlm.EPI_BF16, fake, fake, fake, 1.0, big_m, 65535 * 256, 128, fake, None, None, None, 0,
                          st, None) == vlm.ERR_BAD_SHAPE
    # NVFP4: 16.8M row groups x 16,384 scale atoms per row group
    assert L.vlm_gemm_nvfp4(vlm.EPI_BF16, fake, fake, fake, fake, fake, fake, big_m, 128, 1 << 20, fake, st,
                            None) == vlm.ERR_BAD_SHAPE


def test_release_library_has_no_debug_checks(L):
    """The release build compiles every index check out: it says so, reads no
    device record, and refuses the deliberate-failure self-test before any
    launch (a non-null pointer it never dereferences)."""
    assert L.vlm_debug_build() == 0
    code = ctypes.c_int32(77)
    assert L.vlm_debug_checks(ctypes.byref(code)) == vlm.ERR_UNSUPPORTED and code.value == 0
    assert L.vlm_debug_selftest_bounds(ctypes.c_void_p(256), 4, None) == vlm.ERR_UNSUPPORTED


def test_debug_library_loads_and_exports_every_symbol():
    """The index-checked build (-DVLM_DEBUG) sits beside the release library,
    exports the same C ABI and identifies itself (no CUDA call needed)."""
    path = vlm.DEBUG_LIB_PATH
    if not os.path.exists(path):
        from vision_language_model_b200 import build
        build.build(debug=True)
    D = ctypes.CDLL(path, mode=ctypes.RTLD_LOCAL)
    for n in sorted(_declared()):
        assert hasattr(D, n), n
    D.vlm_debug_build.restype = ctypes.c_int
    assert D.vlm_debug_build() == 1
    D.vlm_debug_checks.restype = ctypes.c_int
    assert D.vlm_debug_checks(None) == vlm.ERR_INVALID_ARG


def test_merge_project_scatter_rejects_bad_arguments_before_launch(L):
    """Every case fails validation before any CUDA call (the fake pointers are never dereferenced)."""
    fake, st = ctypes.c_void_p(256), ctypes.c_void_p(1024)
    cfg = vlm.preset("mistral3", layers=1)
    hw = (ctypes.c_int32 * 2)(224, 224)
    n = 300
    ws = L.vlm_merge_project_scatter_workspace_size(ctypes.byref(cfg), hw, 1, n)
    assert ws >= L.vlm_merge_project_workspace_size(ctypes.byref(cfg), hw, 1) + L.vlm_scatter_workspace_size(n)
    assert L.vlm_merge_project_scatter_workspace_size(ctypes.byref(cfg), hw, 1, 0) == 0
    base = [ctypes.byref(cfg), fake, hw, 1, fake, fake, n, fake, fake, ws, st, None]

    def call(i=None, v=None):
        a = list(base)
        if i is not None:
            a[i] = v
        return L.vlm_merge_project_scatter(*a)

    for i in (1, 4, 5, 7, 8, 10):                          # tower_out, projector, ids, text, workspace, status
        assert call(i, None) == vlm.ERR_INVALID_ARG, i
    assert call(6, 0) == vlm.ERR_BAD_SHAPE                 # no ids
    assert call(8, ctypes.c_void_p(384)) == vlm.ERR_INVALID_ARG   # workspace not 256-byte aligned
    assert call(7, ctypes.c_void_p(264)) == vlm.ERR_INVALID_ARG   # text rows not 16-byte aligned
    assert call(9, ws - 1) == vlm.ERR_WORKSPACE
    assert call(2, (ctypes.c_int32 * 2)(225, 224)) != vlm.OK      # not on the merged-patch grid


def test_merge_project_scatter_wrapper_checks_dtypes_and_shapes():
    """The binding rejects a wrong id dtype or token-table shape before calling the library."""
    import torch
    cfg = vlm.preset("mistral3", layers=1)
    tower_out = torch.zeros(256, cfg.width, dtype=torch.bfloat16)
    proj = torch.zeros(16, dtype=torch.uint8)
    ids = torch.full((100,), cfg.image_token_id, dtype=torch.int64)
    good_text = torch.zeros(100, cfg.proj_out, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        vlm.merge_project_scatter(cfg, tower_out, [(224, 224)], proj, ids.to(torch.int32), good_text)
    for bad in (torch.zeros(99, cfg.proj_out, dtype=torch.bfloat16), torch.zeros(100, 1024, dtype=torch.bfloat16),
                torch.zeros(100, cfg.proj_out, dtype=torch.float32)):
        with pytest.raises(ValueError):
            vlm.merge_project_scatter(cfg, tower_out, [(224, 224)], proj, ids, bad)
