"""bfmoe_route_static: routing for callers that cannot allocate device memory.

Some callers (a plugin inside a framework that owns every allocation, a
real-time loop where allocation is forbidden) can pass their inputs and
outputs but cannot hand the library a workspace.  bfmoe_route_static keeps
its scratch in a fixed array inside the library.  These tests call it
through the C ABI and check its results against bfmoe_route, which takes a
caller-provided workspace, on two calls in a row (the second call must not
see the first call's leftover scratch).  This file is collected last so a
failure here does not hide the other tests' results.
"""
import numpy as np
import pytest

import oracle
import ternary_moe_butterfly_b200 as bf

FAKE = 1 << 20  # aligned non-null address, never dereferenced


def test_rejects_too_many_experts_on_the_host():
    # the scratch array holds the histogram of up to 510 experts
    assert bf.bfmoe_route_static(FAKE, 64, 511, 2, FAKE, FAKE, FAKE, FAKE, None) == bf.ERR_UNSUPPORTED
    assert bf.bfmoe_route_static(FAKE, 64, 8, 9, FAKE, FAKE, FAKE, FAKE, None) == bf.ERR_INVALID_ARG
    assert bf.bfmoe_route_static(None, 64, 8, 2, FAKE, FAKE, FAKE, FAKE, None) == bf.ERR_INVALID_ARG


@pytest.mark.gpu
def test_static_route_matches_workspace_route_twice():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ternary_moe_butterfly_b200 import build
    build.build()
    stream = torch.cuda.current_stream()
    for call, (T, N, k, seed) in enumerate([(4096, 64, 2, 31), (1000, 256, 4, 32)]):
        rng = np.random.default_rng(seed)
        lg_np = rng.standard_normal((T, N)).astype(np.float32)
        lg_np[:: 7] = np.round(lg_np[:: 7])  # ties
        lg = torch.from_numpy(lg_np).cuda()
        out = {name: torch.full(shape, -7, dtype=dt, device="cuda") for name, shape, dt in
               [("idx", (T, k), torch.int32), ("gates", (T, k), torch.float32), ("perm", (T * k,), torch.int32),
                ("offsets", (N + 1,), torch.int32)]}
        code = bf.bfmoe_route_static(lg.data_ptr(), T, N, k, out["idx"].data_ptr(), out["gates"].data_ptr(),
                                     out["perm"].data_ptr(), out["offsets"].data_ptr(), stream.cuda_stream)
        assert code == bf.OK, (call, bf.status_string(code))
        idx, gates, perm, offsets, ws = bf.route(lg, k)
        assert bf.sync_status(ws) == bf.OK
        torch.cuda.synchronize()
        assert torch.equal(out["idx"], idx), call
        assert torch.equal(out["perm"], perm), call
        assert torch.equal(out["offsets"], offsets), call
        np.testing.assert_allclose(out["gates"].cpu().numpy(), gates.cpu().numpy(), rtol=1e-6, atol=1e-7)
        # and both agree with the oracle
        ridx, rg, rperm, roff = oracle.route(lg_np, k)
        np.testing.assert_array_equal(out["perm"].cpu().numpy(), rperm)
        np.testing.assert_array_equal(out["idx"].cpu().numpy(), ridx)
