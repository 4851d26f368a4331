"""moe_permute_noalloc -- the allocation-free permute -- against moe_permute.

Some callers cannot let a library allocate device memory (a serving runtime that has
reserved all of it up front, or a latency-bound loop that cannot take cudaMalloc's device
synchronization); moe_permute_noalloc keeps its scratch in a fixed array instead. This
file is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test. It calls the entry point through the C ABI (ctypes)
with buffers the test allocates, and compares with moe_permute bit for bit on two calls
in a row, so that what the first call leaves in the shared scratch cannot leak into the
second.
"""
import ctypes

import numpy as np
import pytest
import torch

from mxfp4_block_scaled_moe_b200 import inputs

pytestmark = pytest.mark.gpu


def _noalloc(L, idx, E):
    T, k = idx.shape
    off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    pt = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    ps = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    rc = L.moe_permute_noalloc(ctypes.c_void_p(idx.data_ptr()), T, E, k, ctypes.c_void_p(off.data_ptr()),
                               ctypes.c_void_p(pt.data_ptr()), ctypes.c_void_p(ps.data_ptr()),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, L.mxmoe_last_error()
    return off, pt, ps


def _routing(T, E, k, skew, seed):
    rng = np.random.default_rng(seed)
    p = np.arange(1, E + 1, dtype=np.float64) ** -skew
    p /= p.sum()
    keys = rng.random((T, E)) ** (1.0 / p)[None, :]
    return torch.from_numpy(np.argsort(-keys, axis=1)[:, :k].astype(np.int32)).cuda()


@pytest.mark.parametrize("first,second", [((16384, 128, 4, 1.1), (8, 32, 4, 0.0)),
                                          ((3, 23, 4, 0.0), (4096, 128, 4, 0.0)),
                                          ((65536, 256, 4, 0.5), (65536, 256, 4, 0.0))])
def test_noalloc_permute_matches_moe_permute_twice(first, second):
    from mxfp4_block_scaled_moe_b200 import binding as B
    L = B.lib()
    for n, (T, E, k, skew) in enumerate((first, second)):
        idx = _routing(T, E, k, skew, seed=T + E + n)
        ref = B.moe_permute(idx, E)
        got = _noalloc(L, idx, E)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    from mxfp4_block_scaled_moe_b200 import binding as B
    L = B.lib()
    idx = torch.zeros((65537, 4), dtype=torch.int32, device="cuda")   # 262148 pairs > 262144
    rc = L.moe_permute_noalloc(ctypes.c_void_p(idx.data_ptr()), 65537, 8, 4, None, None, None, None)
    assert rc == B.EUNSUPPORTED
    assert b"262144" in L.mxmoe_last_error()


def test_noalloc_permute_drops_an_out_of_range_expert_id():
    """A pair whose expert id lies outside [0, E) is left out: offsets[E] counts the other
    T*k - 1 pairs, which are grouped exactly as moe_permute groups them; the positions from
    offsets[E] on stay unwritten, and the device error word stays clear (moe_permute itself
    reports the same input as MXMOE_EDEVICE)."""
    from mxfp4_block_scaled_moe_b200 import binding as B
    L = B.lib()
    T, E, k = 300, 32, 4
    idx = _routing(T, E, k, 0.3, seed=5)
    idx[123, 2] = E                      # one id past the last expert
    B.mxmoe_check()                      # start from a clear error word
    off, pt, ps = _noalloc(L, idx, E)
    assert L.mxmoe_check(None) == 0
    n = T * k - 1
    assert int(off[E]) == n
    assert torch.all(pt[n:] == -1) and torch.all(ps[n:] == -1)
    ref = B.moe_permute(idx, E)
    with pytest.raises(B.MxmoeError) as ei:
        B.mxmoe_check()
    assert ei.value.rc == B.EDEVICE
    assert torch.equal(off, ref[0])
    assert torch.equal(pt[:n], ref[1][:n]) and torch.equal(ps[:n], ref[2][:n])
