"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device
memory (a plugin whose host runtime owns all allocations, a server whose pool
is fully reserved, a path that cannot afford cudaMalloc's synchronisation).

It keeps its scratch in a fixed array inside libmoe instead of a caller
workspace. Its results must equal moe_dispatch's, call after call, since all
calls reuse the same array. This file is collected last so that a failure
here does not stop the rest of the suite under -x.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


def _routing(T, E, K, skew, seed):
    rng = np.random.default_rng(seed)
    idx, _, _ = oracle.select_topk(rng.normal(size=(T, E)), -skew * np.log(np.arange(E) + 1.0), K)
    return idx


def _buffers(T, E, K):
    i32 = lambda n: torch.full((n,), -7, dtype=torch.int32, device="cuda")
    return i32(E), i32(E + 1), i32(T * K), i32(T * K)


def test_noalloc_dispatch_matches_dispatch_on_two_calls_in_a_row(M):
    # two different batches back to back: the second call reuses the scratch
    # array the first one filled
    for call, (T, E, K, skew) in enumerate([(3000, 128, 8, 1.0), (777, 256, 8, 0.5)]):
        idx = torch.from_numpy(_routing(T, E, K, skew, seed=100 + call)).cuda()
        d = M.make_desc(T, 128, E, K, 128, 0, M.MOE_BF16)
        ref = _buffers(T, E, K)
        M.moe_dispatch(d, idx, *ref, M.alloc_workspace(d))
        got = _buffers(T, E, K)
        M.moe_dispatch_noalloc(d, idx, *got)
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "perm", "inv"), got, ref):
            assert torch.equal(a, b), (call, name)


def test_noalloc_dispatch_rejects_batches_beyond_its_array(M):
    T, E, K = 8193, 128, 8                      # T*K = 65544 > 65536
    d = M.make_desc(T, 128, E, K, 128, 0, M.MOE_BF16)
    idx = torch.zeros((T, K), dtype=torch.int32, device="cuda")
    with pytest.raises(M.MoEError) as ei:
        M.moe_dispatch_noalloc(d, idx, *_buffers(T, E, K))
    assert ei.value.status == 2                 # MOE_ERR_UNSUPPORTED, nothing launched
