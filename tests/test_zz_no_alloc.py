"""moe_permute_noalloc, the permutation entry point for callers that cannot
allocate device memory at call time (a fixed start-up memory budget, a host
caching allocator that owns the device, or a path that must not risk the
synchronisation of cudaMalloc/cudaFree): its scratch lives in a static device
array.  Its results must equal those of moe_permute, which allocates its
scratch, on consecutive calls (the array keeps the previous call's contents).
This file is collected last so that a failure here never hides another test."""
import numpy as np
import pytest
import torch

from bit_quantized_mixture_b200 import moe
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _ids(T, k, E, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)).to(DEV)


def test_noalloc_permutation_equals_allocating_one_on_consecutive_calls():
    # a large call, then a small one that reuses the shared scratch array
    for T, k, E, seed in ((4096, 10, 512, 1), (37, 4, 16, 2)):
        ids = _ids(T, k, E, seed)
        ref = moe.permute(ids, E)
        got = moe.permute_noalloc(ids, E)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g)          # integer outputs: bit-exact
        # and directly against the oracle's permutation
        for o, g in zip(O.permute(ids.cpu().numpy(), E), got):
            assert np.array_equal(o, g.cpu().numpy())


def test_noalloc_rejects_sizes_beyond_its_scratch():
    ids = torch.zeros((1, 1), dtype=torch.int32, device=DEV)
    L = moe.lib()
    out = [torch.empty(2048, dtype=torch.int32, device=DEV) for _ in range(4)]
    s = L.moe_permute_noalloc(ids.data_ptr(), 262145, 1, 16, *[o.data_ptr() for o in out], None)
    assert s == moe.MOE_ERR_INVALID_ARG
    assert b"262144" in L.moe_last_error(None)
    s = L.moe_permute_noalloc(ids.data_ptr(), 1, 1, 1025, *[o.data_ptr() for o in out], None)
    assert s == moe.MOE_ERR_INVALID_ARG
