"""The allocation-free LUT-gradient call (sk_linear_bwd_lut_noalloc).

It exists for callers that cannot allocate device memory when they need the
gradient (for instance a plugin inside another framework's executor that owns
every device allocation).  It must give the same result as the workspace-taking
sk_linear_bwd_lut, within the LUT-gradient tolerance of the other parity
tests, on consecutive calls that share its one scratch array.  This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def _noalloc(sk, packed, bits, gpr, n, d, X, dY, T, out, accumulate=0, task=None, ntask=1):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sk.lib.sk_linear_bwd_lut_noalloc(sk._ptr(packed), bits, gpr, n, d, sk._ptr(X), sk._ptr(dY), T,
                                            sk._ptr(task), ntask, sk._ptr(out), accumulate, stream)


def test_noalloc_matches_workspace_call_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from compressive_fine_tuning_b200 import sk, synth
    from tests import gpu_cases as gc

    # two different layers back to back: the second call reuses the scratch
    # array the first one filled, so stale partial sums would show up here
    cases = [((1024, 2048, 4, 8), 256, 11), ((512, 1376, 3, 1), 300, 12), ((1024, 2048, 4, 8), 256, 13)]
    for (n, d, bits, gpr), T, seed in cases:
        c = synth.layer_case(seed, n=n, d=d, bits=bits, gpr=gpr, T=T)
        packed, lut, X, dY, _ = gc.dev_case(c)
        assert sk.workspace_bytes(sk.SK_OP_BWD_LUT, n, d, bits, gpr, T, 1) > 0   # the scratch-using path
        ref = sk.linear_bwd_lut(packed, bits, gpr, X, dY)                       # workspace entry point
        got = torch.full_like(ref, float("nan"))
        assert _noalloc(sk, packed, bits, gpr, n, d, X, dY, T, got) == 0, sk.lib.sk_last_error()
        torch.cuda.synchronize()
        gc.check_dlut(got.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "allocation-free dlut")
        again = torch.full_like(ref, float("nan"))
        assert _noalloc(sk, packed, bits, gpr, n, d, X, dY, T, again) == 0
        torch.cuda.synchronize()
        assert torch.equal(again, got)                                           # deterministic, no leftovers
    assert sk.device_check() == 0


def test_noalloc_rejects_layers_beyond_its_scratch():
    from compressive_fine_tuning_b200 import sk
    # a 70B-sized gate projection needs more partial-bin scratch than the fixed array
    n, d, bits, gpr, T = 28672, 8192, 4, 4, 4096
    need = sk.workspace_bytes(sk.SK_OP_BWD_LUT, n, d, bits, gpr, T, 1)
    assert need > (32 << 20)
    fake = [ctypes.c_void_p(a) for a in (0x10000000, 0x20000000, 0x40000000, 0x80000000)]
    st = sk.lib.sk_linear_bwd_lut_noalloc(fake[0], bits, gpr, n, d, fake[1], fake[2], T, None, 1, fake[3], 0, None)
    assert st == 1  # SK_ERR_INVALID_ARG, nothing launched
    assert b"scratch" in sk.lib.sk_last_error()
