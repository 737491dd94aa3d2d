"""The allocation-free momentum entry point (signmuon_momentum_norm_noalloc).

Some callers cannot allocate device memory around the optimizer step (their
runtime's allocator owns the whole device, or cudaMalloc's device
synchronisation is not acceptable in their loop).  For them the library
offers a variant of the momentum + Frobenius-norm call whose scratch lives in
a fixed 1 MiB device array inside the library.  This test checks, through the
C ABI, that two calls in a row give exactly what the workspace-based entry
point gives on the same inputs, and that requests beyond the array's limits
are refused.  It lives in its own file so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from sign_muon_optimizer_momentum_b200 import _lib as L
from sign_muon_optimizer_momentum_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _inputs(shapes, M, seed, dtype):
    grads = [syn.gaussian(s, 2.0, "cpu", "za_g", seed, i, m, dtype=dtype).cuda()
             for i, s in enumerate(shapes) for m in range(M)]
    moms = [syn.gaussian(s, 1.0, "cpu", "za_m", seed, i, m).cuda() for i, s in enumerate(shapes) for m in range(M)]
    return grads, moms


def _buffers(shapes, M):
    xs = [torch.zeros((r, L.signmuon_x_ld(c)), dtype=torch.bfloat16, device="cuda") for r, c in shapes
          for _ in range(M)]
    inv = torch.zeros(len(shapes) * M, dtype=torch.float32, device="cuda")
    return xs, inv


def _ptrs(ts):
    return [t.data_ptr() for t in ts]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_workspace_entry_point_twice(cuda_lib, dtype):
    shapes, M, beta = [(256, 256), (64, 147), (300, 1000), (1, 1)], 3, 0.9
    code = L.SIGNMUON_BF16 if dtype == torch.bfloat16 else L.SIGNMUON_F32
    stream = torch.cuda.current_stream().cuda_stream
    grads, moms = _inputs(shapes, M, 1, dtype)
    moms_ref = [m.clone() for m in moms]
    x_ref, inv_ref = _buffers(shapes, M)
    x_new, inv_new = _buffers(shapes, M)
    ws = torch.zeros(L.signmuon_momentum_workspace_bytes(shapes, M), dtype=torch.uint8, device="cuda")
    for call in range(2):   # two calls in a row: the shared scratch is reused
        L.signmuon_momentum_norm(shapes, M, code, _ptrs(grads), _ptrs(moms_ref), beta, _ptrs(x_ref),
                                 inv_ref.data_ptr(), ws.data_ptr(), ws.numel(), stream)
        L.signmuon_momentum_norm_noalloc(shapes, M, code, _ptrs(grads), _ptrs(moms), beta, _ptrs(x_new),
                                         inv_new.data_ptr(), stream)
        torch.cuda.synchronize()
        # The momentum arithmetic is exact in both, so results are identical.
        for a, b in zip(moms, moms_ref):
            assert torch.equal(a, b), call
        for a, b in zip(x_new, x_ref):
            assert torch.equal(a, b), call
        assert torch.equal(inv_new, inv_ref), call
        assert np.all(np.isfinite(inv_new.cpu().numpy()))


def test_noalloc_refuses_requests_beyond_its_scratch(cuda_lib):
    fake = 1 << 20
    too_many_units = [(1, 8)] * 1171
    with pytest.raises(L.SignMuonError) as e:
        L.signmuon_momentum_norm_noalloc(too_many_units, 1, 0, [fake] * 1171, [fake] * 1171, 0.9,
                                         [fake] * 1171, fake)
    assert e.value.status == L.SIGNMUON_ERR_WORKSPACE
    too_many_elems = [(65536, 16385)]     # 262160 blocks of 4096 elements; the limit is 245760
    with pytest.raises(L.SignMuonError) as e:
        L.signmuon_momentum_norm_noalloc(too_many_elems, 1, 0, [fake], [fake], 0.9, [fake], fake)
    assert e.value.status == L.SIGNMUON_ERR_WORKSPACE
