"""twell_pack_noalloc, the allocation-free variant of twell_pack, against twell_pack.

Callers that may not allocate device memory (a plug-in inside a host whose
allocator owns the device, or a latency-critical loop that cannot afford an
allocation's synchronisation) use this entry point; it keeps its scratch in a
fixed array inside the library. This file is collected last so that a failure
here leaves every other test already run.
"""

import ctypes

import numpy as np
import pytest

from synthetic import Workload, make_inputs
from twell_testlib import assert_pack_equal, state_to_numpy, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tw():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import activation_sparse_ffn_gemm_b200 as tw

    tw.lib()
    return tw


def _inputs(seed):
    # lognormal token scale: some tiles overflow K, so the scratch is written and read back
    w = Workload("noalloc", 700, 256, 4096, 128, 8, 0.04, row_scale="lognormal", seed=seed)
    inp = make_inputs(w)
    return {k: to_dev(v) for k, v in inp.items() if k != "meta"}


def test_noalloc_pack_matches_workspace_pack_twice(tw):
    assert 700 * 4096 * 2 <= tw.NOALLOC_SCRATCH_BYTES
    for seed in (31, 32):  # two calls in a row, different data
        D = _inputs(seed)
        ref, z_ref = tw.pack(D["X"], D["W_g"], D["b_g"], T_n=128, K=8, z_debug=True)
        new, z_new = tw.pack_noalloc(D["X"], D["W_g"], D["b_g"], T_n=128, K=8, z_debug=True)
        torch.cuda.synchronize()
        p_ref, p_new = state_to_numpy(ref), state_to_numpy(new)
        assert p_ref["n_ovf"] > 0, "the case must exercise the spilled slices"
        assert_pack_equal(p_new, p_ref)
        assert torch.equal(z_new, z_ref)
        assert new.read_status() == 0 and ref.read_status() == 0


def test_noalloc_rejects_oversize_shape(tw):
    M, d, f = 2048, 128, 8192  # M * d_ff * 2 = 32 MiB > 16 MiB of scratch
    X = torch.zeros((M, d), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((f, d), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(f, dtype=torch.bfloat16, device="cuda")
    st = tw.HybridState(M, f, 128, 8, M, "cuda", with_u=False)
    code = tw.lib().twell_pack_noalloc(ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                                       ctypes.c_void_p(b.data_ptr()), d, ctypes.byref(st.c), None, None)
    assert code == 6  # TWELL_EWORKSPACE
