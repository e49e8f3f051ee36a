"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device
memory (a plugin whose host runtime owns all allocations, a server whose pool
is fully reserved, a path that cannot afford cudaMalloc's synchronisation).

It keeps its scratch in a fixed array inside libmoe instead of a caller
workspace. Its results must equal the oracle's dispatch and moe_dispatch's,
call after call, since all calls reuse the same array. The batches cover the
one-chunk decode sizes (where moe_dispatch takes its one-CTA kernel and this
entry point the chunked kernels), a batch of exactly one chunk, several
chunks and the empty batch. This file is collected last so that a failure
here does not stop the rest of the suite under -x.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

BATCHES = [(1, 128, 8, 1.0), (16, 256, 8, 1.3), (256, 128, 8, 0.5), (3000, 128, 8, 1.0),
           (777, 256, 8, 0.5), (5, 4, 4, 0.0), (8192, 512, 8, 0.2)]


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


def test_noalloc_dispatch_matches_oracle_and_dispatch_on_calls_in_a_row(M):
    # different batches back to back: each call reuses the scratch array the
    # previous one filled
    for call, (T, E, K, skew) in enumerate(BATCHES + BATCHES[:2]):
        idx_np = _routing(T, E, K, skew, seed=100 + call)
        idx = torch.from_numpy(idx_np).cuda()
        d = M.make_desc(T, 128, E, K, 128, 0, M.MOE_BF16)
        got = _buffers(T, E, K)
        M.moe_dispatch_noalloc(d, idx, *got)
        ref = _buffers(T, E, K)
        M.moe_dispatch(d, idx, *ref, M.alloc_workspace(d))
        torch.cuda.synchronize()
        want = oracle.dispatch(idx_np, E)
        for name, a, b, w in zip(("counts", "offsets", "perm", "inv"), got, ref, want):
            assert (a.cpu().numpy() == w).all(), (call, T, name, "oracle")
            assert torch.equal(a, b), (call, T, name, "moe_dispatch")


def test_noalloc_dispatch_empty_batch(M):
    d = M.make_desc(0, 128, 8, 2, 128, 0, M.MOE_BF16)
    counts, offsets = _buffers(0, 8, 2)[:2]
    M.moe_dispatch_noalloc(d, None, counts, offsets, None, None)
    torch.cuda.synchronize()
    assert (counts.cpu().numpy() == 0).all() and (offsets.cpu().numpy() == 0).all()


def test_noalloc_dispatch_rejects_batches_beyond_its_array(M):
    T, E, K = 8193, 128, 8                      # T*K = 65544 > 65536
    d = M.make_desc(T, 128, E, K, 128, 0, M.MOE_BF16)
    idx = torch.zeros((T, K), dtype=torch.int32, device="cuda")
    with pytest.raises(M.MoEError) as ei:
        M.moe_dispatch_noalloc(d, idx, *_buffers(T, E, K))
    assert ei.value.status == 2                 # MOE_ERR_UNSUPPORTED, nothing launched
