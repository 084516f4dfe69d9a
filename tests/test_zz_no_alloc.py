"""vlm_scatter_noalloc: the masked scatter for callers that cannot allocate.

Serving engines that give all free device memory to their own pools, and
plugin hosts that pass an operator only its inputs and outputs, cannot lend
vlm_scatter a workspace. vlm_scatter_noalloc keeps that scratch in a fixed
array inside the library instead. These tests call it through the C ABI and
check its result, bit for bit (the scatter is a pure copy), against the CPU
oracle's scatter and against vlm_scatter's, on two calls in a row: the second
call is smaller than the first, so positions left over from the first call
would show up as wrong rows.

This file is collected last on purpose, so a run that stops at its first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import vlm_oracle as O
from tests.gpu_util import guarded, guarded_copy, guarded_zeros
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu

MAX_TOKENS = 262144  # VLM_SCATTER_NOALLOC_MAX_TOKENS in include/vlm.h


def _noalloc():
    fn = vlm.lib().vlm_scatter_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                   ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    return fn


def _call(ids, img, text, status):
    row_bytes = text[0].numel() * text.element_size()
    return _noalloc()(ids.data_ptr(), ids.numel(), 10, img.data_ptr(), img.shape[0], text.data_ptr(), row_bytes,
                      status.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("case", [
    [(4, 4096, [[1536]] * 4, 5120, 21), (2, 1000, [[7, 300], [1]], 5120, 22)],
    [(1, 65536, [[4096, 4096]], 256, 23), (3, 129, [[1], [0], [128]], 256, 24)],
])
def test_noalloc_matches_workspace_scatter_on_two_calls(case):
    for n_seq, seq_len, runs, width, seed in case:
        ids = synth.text_sequences(seed, n_seq, seq_len, runs).reshape(-1).cuda()
        n_img = int((ids == 10).sum())
        img = synth.randn_bf16(seed, "img", (n_img, width), 1.0).cuda()
        text = synth.text_embeddings(seed, ids.numel(), width).cuda()
        ref = guarded_copy(text)
        st_ref = vlm.new_status()
        vlm.scatter(ids, img, ref, 10, status=st_ref)
        got = guarded_copy(text)
        st = vlm.new_status()
        assert _call(ids, img, got, st) == vlm.OK
        assert vlm.status_sync(st) == vlm.OK and vlm.status_sync(st_ref) == vlm.OK
        expect = O.scatter(ids.cpu().numpy(), img.cpu().view(torch.int16).numpy(),
                           text.cpu().view(torch.int16).numpy(), 10)
        np.testing.assert_array_equal(got.cpu().view(torch.int16).numpy(), expect)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_noalloc_count_mismatch_writes_nothing():
    ids = synth.text_sequences(25, 1, 512, [[40]]).reshape(-1).cuda()
    img = synth.randn_bf16(25, "img", (41, 128), 1.0).cuda()
    text = synth.text_embeddings(25, 512, 128).cuda()
    before = text.clone()
    st = vlm.new_status()
    assert _call(ids, img, text, st) == vlm.OK
    assert vlm.status_sync(st) == vlm.ERR_COUNT_MISMATCH
    assert torch.equal(text.view(torch.int16), before.view(torch.int16))


def test_noalloc_rejects_more_ids_than_its_scratch_holds():
    ids = torch.full((MAX_TOKENS + 1,), 11, dtype=torch.int64, device="cuda")
    img = guarded((0, 8), dtype=torch.bfloat16)
    text = guarded_zeros((MAX_TOKENS + 1, 8), dtype=torch.bfloat16)
    st = vlm.new_status()
    assert _call(ids, img, text, st) == vlm.ERR_BAD_SHAPE
    ids = ids[:MAX_TOKENS]
    assert _call(ids, img, text[:MAX_TOKENS], st) == vlm.OK
    assert vlm.status_sync(st) == vlm.OK
