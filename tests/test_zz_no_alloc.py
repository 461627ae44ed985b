"""The allocation-free LUT-gradient call (sk_linear_bwd_lut_noalloc).

It exists for callers that cannot allocate device memory when they need the
gradient (for instance a plugin inside another framework's executor that owns
every device allocation, or a loop that has reserved its whole memory budget up
front).  It must give the same result as the workspace-taking
sk_linear_bwd_lut, and the oracle's, within the LUT-gradient tolerance of the
other parity tests, on consecutive calls that share its one scratch array.
This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
(The host-side rejection of layers too large for the array is tested without a
device in tests/test_abi_host.py.)
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _default_paths(monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # the kernel choice must be the library's own
    monkeypatch.delenv("SK_BWD_PATH", raising=False)


def _noalloc(sk, packed, bits, gpr, n, d, X, dY, T, out, accumulate=0, task=None, ntask=1):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sk.lib.sk_linear_bwd_lut_noalloc(sk._ptr(packed), bits, gpr, n, d, sk._ptr(X), sk._ptr(dY), T,
                                            sk._ptr(task), ntask, sk._ptr(out), accumulate, stream)


def test_noalloc_matches_workspace_call_on_consecutive_calls():
    import oracle
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
        gc.check_dlut(got.cpu().numpy()[0], oracle.backward_lut(c.x, c.dy, c.idx, gpr, 1 << bits),
                      "allocation-free dlut vs oracle")
        again = torch.full_like(ref, float("nan"))
        assert _noalloc(sk, packed, bits, gpr, n, d, X, dY, T, again) == 0
        torch.cuda.synchronize()
        assert torch.equal(again, got)                                           # deterministic, no leftovers
    assert sk.device_check() == 0


@pytest.mark.parametrize("kind", ["accumulate", "multitask", "few_tokens", "empty"])
def test_noalloc_other_paths_match_oracle(kind):
    """accumulate = 1 onto a non-zero gradient (tensor-core path), eight LUT
    sets with task ids, a batch below the tensor-core threshold, and an empty
    batch; each compared with the oracle, twice in a row."""
    import oracle
    from compressive_fine_tuning_b200 import sk, synth
    from tests import gpu_cases as gc

    n, d, bits, gpr = 512, 2048, 4, 4
    T = {"accumulate": 256, "multitask": 200, "few_tokens": 32, "empty": 0}[kind]
    ntask = 8 if kind == "multitask" else 1
    c = synth.layer_case(21 + T, n=n, d=d, bits=bits, gpr=gpr, T=max(T, 1), ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    X, dY = X[:T], dY[:T]
    if task is not None:
        task = task[:T].contiguous()
    ref = oracle.backward_lut(c.x[:T], c.dy[:T], c.idx, gpr, 1 << bits,
                              task=None if c.task is None else c.task[:T], ntask=ntask)
    ref = ref.reshape(ntask, n, gpr, 1 << bits)
    start = np.full(ref.shape, 0.125) if kind in ("accumulate", "empty") else np.zeros(ref.shape)
    acc = 1 if kind in ("accumulate", "empty") else 0
    for _ in range(2):
        out = torch.from_numpy(start.astype(np.float32)).cuda() if acc else torch.full(ref.shape, float("nan"),
                                                                                      device="cuda")
        st = _noalloc(sk, packed, bits, gpr, n, d, X, dY, T, out, accumulate=acc, task=task, ntask=ntask)
        assert st == 0, sk.lib.sk_last_error()
        torch.cuda.synchronize()
        want = ref + (start if acc else 0.0)
        if T == 0:
            assert np.array_equal(out.cpu().numpy(), want.astype(np.float32))
        else:
            gc.check_dlut(out.cpu().numpy(), want, f"allocation-free dlut ({kind})")
    assert sk.device_check() == 0
