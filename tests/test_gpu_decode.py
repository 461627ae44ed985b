"""Parity of the decode forward kernel (4-bit, one LUT set, 1 <= T <= 16) with the oracle.

The decode kernel splits the rows over the CTAs (several 16-row tiles per CTA
once the layer has more tiles than the GPU has SMs), streams the columns in
stages of 512 to 2048 columns, and permutes the K order inside every MMA
step.  The shapes
below make each of those visible: ragged last row tiles, a partial last stage,
groups that straddle stages, 32-column groups, CTAs whose warps span two row
tiles, and token counts on both sides of the 8-token MMA tile.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from compressive_fine_tuning_b200 import synth  # noqa: E402
from tests import gpu_cases as gc  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from compressive_fine_tuning_b200 import sk  # noqa: F401
    yield
    torch.cuda.synchronize()


DECODE_SHAPES = [
    (256, 512, 1),      # the tiny configuration, one stage
    (4104, 4096, 8),    # 257 row tiles: two per CTA, ragged last tile
    (2376, 2816, 2),    # 1408-column groups straddling stages, partial last stage
    (96, 512, 16),      # 32-column groups, many per stage
    (264, 256, 1),      # narrowest width the kernel takes, one 256-column block
]


@pytest.mark.parametrize("shape", DECODE_SHAPES)
@pytest.mark.parametrize("T", [1, 2, 5, 8, 9, 16])
def test_decode_forward(monkeypatch, shape, T):
    from compressive_fine_tuning_b200 import sk
    monkeypatch.setenv("SK_FWD_PATH", "dq")
    n, d, gpr = shape
    c = synth.layer_case(31000 + n + T, n=n, d=d, bits=4, gpr=gpr, T=T)
    packed, lut, X, dY, task = gc.dev_case(c)
    Y = sk.linear_fwd(packed, lut, 4, X, task)
    gc.check_fwd(c, Y)
    assert sk.device_check() == 0


@pytest.mark.parametrize("n,d", [(11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("T", [1, 16])
def test_decode_forward_7b_shapes(monkeypatch, n, d, T):
    """The gate/up shape puts four or five row tiles in every CTA, so a warp's
    items span two row tiles; the down shape ends on a 256-column stage."""
    from compressive_fine_tuning_b200 import sk
    monkeypatch.setenv("SK_FWD_PATH", "dq")
    c = synth.layer_case(32000 + n + T, n=n, d=d, bits=4, gpr=8, T=T)
    packed, lut, X, dY, task = gc.dev_case(c)
    Y = sk.linear_fwd(packed, lut, 4, X, task)
    gc.check_fwd(c, Y)
    assert sk.device_check() == 0


@pytest.mark.parametrize("T", [1, 16])
def test_decode_matches_tensor_core_path_and_is_deterministic(monkeypatch, T):
    """Each kernel meets the oracle on every element; the two (the same bf16
    weights, fp32 sums in different orders) agree to a few bf16 ulps, and the
    decode kernel repeats itself bit for bit."""
    from compressive_fine_tuning_b200 import sk
    c = synth.layer_case(33000 + T, n=4096, d=4096, bits=4, gpr=8, T=T)
    packed, lut, X, dY, task = gc.dev_case(c)
    monkeypatch.setenv("SK_FWD_PATH", "dq")
    y1 = sk.linear_fwd(packed, lut, 4, X, task)
    y2 = sk.linear_fwd(packed, lut, 4, X, task)
    assert torch.equal(y1, y2)
    monkeypatch.setenv("SK_FWD_PATH", "tc")
    y3 = sk.linear_fwd(packed, lut, 4, X, task)
    gc.check_fwd(c, y1)
    gc.check_fwd(c, y3)
    a, b = y1.float(), y3.float()
    assert torch.allclose(a, b, rtol=2 ** -6, atol=1e-3 * b.abs().max().item())


def test_decode_identity_is_exact(monkeypatch):
    """idx = I with the {0, 1} LUT (SpaLLM section 2.4): Y == X bit for bit."""
    from compressive_fine_tuning_b200 import sk
    monkeypatch.setenv("SK_FWD_PATH", "dq")
    n = d = 512
    idx = np.zeros((n, d), dtype=np.uint8)
    idx[np.arange(n), np.arange(n)] = 1
    lut = np.zeros((1, n, 1, 16), dtype=np.float16)
    lut[..., 1] = 1.0
    lut[..., 2:] = np.float16(np.nan)   # never read
    rng = synth.rng_for(34000)
    x = synth.make_bf16(rng, (7, d), 1.0)
    packed = sk.pack(torch.from_numpy(idx).cuda(), 4)
    X = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    Y = sk.linear_fwd(packed, torch.from_numpy(lut).cuda(), 4, X, None)
    np.testing.assert_array_equal(Y.view(torch.int16).cpu().numpy().view(np.uint16), x)


@pytest.mark.parametrize("tau", [0, 5, 7])
def test_decode_single_token_multitask(tau):
    """One token with a task id picks its LUT set on the device (SpaLLM section
    2.3); the routed path is not needed for a single token."""
    from compressive_fine_tuning_b200 import sk
    c = synth.layer_case(35000 + tau, n=1024, d=2048, bits=4, gpr=4, T=1, ntask=8, with_task=True)
    c.task[:] = tau
    packed, lut, X, dY, task = gc.dev_case(c)
    sk.device_check(clear=True)
    Y = sk.linear_fwd(packed, lut, 4, X, task)
    gc.check_fwd(c, Y)
    assert sk.device_check() == 0


def test_decode_single_token_bad_task_zeroes_and_flags():
    from compressive_fine_tuning_b200 import sk
    c = synth.layer_case(35100, n=512, d=1024, bits=4, gpr=2, T=1, ntask=4, with_task=True)
    packed, lut, X, dY, task = gc.dev_case(c)
    task.fill_(9)
    sk.device_check(clear=True)
    Y = sk.linear_fwd(packed, lut, 4, X, task)
    assert sk.device_check(clear=True) & sk.SK_CHECK_TASK_RANGE
    assert not Y.float().abs().any()


# ---------------------------------------------------------------------------
# several layers in one call (sk_linear_fwd_group)
# ---------------------------------------------------------------------------

def _shared_x(c, src):
    """The case `c` with the activations of `src` (layers that read one input)."""
    return synth.LayerCase(c.n, c.d, c.bits, c.gpr, src.T, c.ntask, c.idx, c.lut, src.x_bits, c.dy_bits, src.task)


@pytest.mark.parametrize("T", [1, 5, 9, 16])
def test_decode_group_matches_oracle(T):
    """Mixed widths, ragged row tiles, groups that straddle stages, 32-column
    groups and two layers that share one input, in one launch: every layer's
    Y against the oracle."""
    from compressive_fine_tuning_b200 import sk
    shapes = [(264, 256, 1), (2376, 2816, 2), (96, 512, 16), (4104, 4096, 8), (1032, 4096, 8)]
    cases = [synth.layer_case(36000 + 10 * i + T, n=n, d=d, bits=4, gpr=g, T=T) for i, (n, d, g) in enumerate(shapes)]
    cases[4] = _shared_x(cases[4], cases[3])
    dev = [gc.dev_case(c) for c in cases]
    Xs = [dv[2] for dv in dev]
    Xs[4] = Xs[3]
    ys = sk.linear_fwd_group([(dv[0], dv[1], x) for dv, x in zip(dev, Xs)], 4)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        gc.check_fwd(c, y)
    assert sk.device_check() == 0
    # the same call twice gives the same bits
    ys2 = sk.linear_fwd_group([(dv[0], dv[1], x) for dv, x in zip(dev, Xs)], 4)
    assert all(torch.equal(a, b) for a, b in zip(ys, ys2))


@pytest.mark.parametrize("T", [1, 16])
def test_decode_group_llama7b_block_sampled(T):
    """The seven LLaMA-2-7B projections (4-bit, 8 groups per row) as one group,
    q/k/v and gate/up each sharing an input: 96 sampled rows per layer."""
    from compressive_fine_tuning_b200 import sk
    cases = [synth.layer_case(37000 + 10 * i + T, n=n, d=d, bits=4, gpr=8, T=T)
             for i, (n, d) in enumerate(synth.LLAMA2_7B)]
    for i, src in ((1, 0), (2, 0), (5, 4)):
        cases[i] = _shared_x(cases[i], cases[src])
    dev = [gc.dev_case(c) for c in cases]
    xs = [dev[{1: 0, 2: 0, 5: 4}.get(i, i)][2] for i in range(7)]
    ys = sk.linear_fwd_group([(dv[0], dv[1], x) for dv, x in zip(dev, xs)], 4)
    torch.cuda.synchronize()
    assert sk.device_check() == 0
    for i, (c, y) in enumerate(zip(cases, ys)):
        rows = np.sort(synth.rng_for(37100 + i).choice(c.n, size=96, replace=False))
        gc.check_fwd(c, y, rows=rows)


def test_decode_group_single_token_multitask():
    """One token with a task id over a group: every layer uses that set."""
    from compressive_fine_tuning_b200 import sk
    cases = [synth.layer_case(38000 + i, n=n, d=d, bits=4, gpr=4, T=1, ntask=8, with_task=True)
             for i, (n, d) in enumerate([(1024, 2048), (512, 4096), (2048, 1024)])]
    for c in cases:
        c.task[:] = 6
    dev = [gc.dev_case(c) for c in cases]
    ys = sk.linear_fwd_group([(dv[0], dv[1], dv[2]) for dv in dev], 4, task=dev[0][4])
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        gc.check_fwd(c, y)
    assert sk.device_check() == 0


def test_group_outside_the_decode_kernel_runs_per_layer():
    """2-bit layers at 64 tokens are not decode work: the group call runs the
    layers one by one on their own kernels, with the same results."""
    from compressive_fine_tuning_b200 import sk
    cases = [synth.layer_case(39000 + i, n=n, d=d, bits=2, gpr=2, T=64) for i, (n, d) in enumerate([(256, 512), (136, 1024)])]
    dev = [gc.dev_case(c) for c in cases]
    ys = sk.linear_fwd_group([(dv[0], dv[1], dv[2]) for dv in dev], 2)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        gc.check_fwd(c, y)
