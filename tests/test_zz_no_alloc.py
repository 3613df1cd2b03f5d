"""moe_permute_noalloc: the permutation entry point for callers that cannot
allocate device memory (a runtime with its own fixed memory pool, a serving
process that must not block in the driver's allocator). Its scratch is a fixed
array inside the library; these tests check that it returns exactly what the
oracle's permutation and moe_permute return, on two calls in a row, that the
second call takes no device memory, and that oversized problems and bad
arguments are refused before anything runs.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import tqp_oracle as O
import quantized_base_lora_moe_b200 as Q


def test_binding_refuses_wrong_dtypes_and_short_outputs():
    """Checked in the binding before any pointer reaches the library (no GPU needed)."""
    ids64 = torch.zeros(4, 2, dtype=torch.int64)
    ok = lambda n: torch.zeros(n, dtype=torch.int32)
    for fn in (Q.moe_permute, Q.moe_permute_noalloc):
        with pytest.raises(ValueError):
            fn(ids64, 8, ok(9), ok(8), ok(8))                        # int64 ids
        with pytest.raises(ValueError):
            fn(ids64.to(torch.int32), 8, ok(9), ok(7), ok(8))        # perm_token too short
        with pytest.raises(ValueError):
            fn(ids64.to(torch.int32), 8, ok(8), ok(8), ok(8))        # offsets too short
        with pytest.raises(ValueError):
            fn(ids64.to(torch.int32).t(), 8, ok(9), ok(8), ok(8))    # not contiguous


@pytest.mark.gpu
def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = Q.lib()
    assert L.moe_permute_noalloc_max_bytes() >= 1 << 20
    # real (small) device buffers: the size checks refuse these calls on the host
    # before anything is enqueued, whatever the buffers hold
    buf = torch.zeros(64, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())
    assert L.moe_permute_noalloc(p, 16385, 8, 2, p, p, p, None, None) == -2      # T > 16384
    assert L.moe_permute_noalloc(p, 16, 513, 2, p, p, p, None, None) == -2       # E > 512
    assert L.moe_permute_noalloc(p, 16, 8, 9, p, p, p, None, None) == -1         # k > E
    torch.cuda.synchronize()
    assert torch.count_nonzero(buf).item() == 0                                  # nothing ran


class _Out:
    """Output buffers and status word, allocated before any measurement."""

    def __init__(self, T, k, E):
        self.offsets = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
        self.perm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        self.inv = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        self.st = Q.Status()

    def run(self, fn, ids, E):
        fn(ids, E, self.offsets, self.perm, self.inv, status=self.st)
        torch.cuda.synchronize()
        assert self.st.read() == 0
        return self.offsets.cpu().numpy(), self.perm.cpu().numpy(), self.inv.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("T,E,k,skew", [(8192, 460, 12, False), (16384, 460, 12, True), (300, 23, 5, False)])
def test_noalloc_matches_oracle_and_moe_permute_on_two_calls_in_a_row(T, E, k, skew):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    bias = synth.zipf_bias(E, 1.1) if skew else None
    for call in range(2):          # the second call runs on the first call's leftover scratch
        ids_np = O.topk(synth.make_logits(T, E, seed=100 * call + T, bias=bias), k).astype(np.int32)
        ids = torch.from_numpy(ids_np).cuda()
        ref = _Out(T, k, E).run(Q.moe_permute, ids, E)
        out = _Out(T, k, E)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        got = out.run(Q.moe_permute_noalloc, ids, E)
        free1 = torch.cuda.mem_get_info()[0]
        if call == 1:              # module loaded and address cached: the call takes no device memory
            assert free1 >= free0, (free0, free1)
        o_off, o_perm, o_inv = O.permute(ids_np, E)
        assert np.array_equal(got[0], o_off) and np.array_equal(got[1], o_perm) and np.array_equal(got[2], o_inv)
        for a, b in zip(got, ref):
            assert np.array_equal(a, b)
