"""moe_permute_noalloc: the permutation entry point for callers that cannot
allocate device memory (a runtime with its own fixed memory pool, a serving
process that must not block in the driver's allocator). Its scratch is a fixed
array inside the library; these tests check that it returns exactly what
moe_permute returns, on two calls in a row, and that oversized problems are
refused before anything runs.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import tqp_oracle as O
import quantized_base_lora_moe_b200 as Q


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = Q.lib()
    assert L.moe_permute_noalloc_max_bytes() >= 1 << 20
    # T > 16384 or E > 512: refused on the host (TQP_ERR_UNSUPPORTED) before any launch
    assert L.moe_permute_noalloc(ctypes.c_void_p(16), 16385, 8, 2, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                 ctypes.c_void_p(16), None, None) == -2
    assert L.moe_permute_noalloc(ctypes.c_void_p(16), 64, 513, 2, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                 ctypes.c_void_p(16), None, None) == -2
    assert L.moe_permute_noalloc(None, 64, 8, 9, ctypes.c_void_p(16), None, None, None, None) == -1


def _permute_both(ids_np, E):
    T, k = ids_np.shape
    ids = torch.from_numpy(ids_np).cuda()
    out = []
    for fn in (Q.moe_permute, Q.moe_permute_noalloc):
        offsets = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
        perm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        inv = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        st = Q.Status()
        fn(ids, E, offsets, perm, inv, status=st)
        torch.cuda.synchronize()
        assert st.read() == 0
        out.append((offsets.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy()))
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("T,E,k,skew", [(8192, 460, 12, False), (16384, 460, 12, True), (300, 23, 5, False)])
def test_noalloc_matches_moe_permute_on_two_calls_in_a_row(T, E, k, skew):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    bias = synth.zipf_bias(E, 1.1) if skew else None
    for call in range(2):          # the second call runs on the first call's leftover scratch
        ids = O.topk(synth.make_logits(T, E, seed=100 * call + T, bias=bias), k).astype(np.int32)
        (a_off, a_perm, a_inv), (b_off, b_perm, b_inv) = _permute_both(ids, E)
        assert np.array_equal(a_off, b_off)
        assert np.array_equal(a_perm, b_perm)
        assert np.array_equal(a_inv, b_inv)
