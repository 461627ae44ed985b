"""Parity with the oracle at the workloads' own sizes.

The kernels take size-dependent paths (tile counts, K loops over thousands of
tokens, 3-bit rows of 5120 and 13824 columns, routed grids of 28672 rows with
eight LUT sets), so every layer shape of each workload runs here at its full
size, in the launch configuration the benchmark times, and is compared with the
oracle on outputs it can compute cheaply:

* Y on 96 sampled rows for every token (the oracle needs only those rows of the
  index map and LUTs);
* dX on 64 sampled tokens for every column (the oracle needs only those rows
  of dY);
* the LUT gradient on 96 sampled rows (the oracle bins dY[:, rows]^T X).

Workloads ("SpaLLM: Unified Compressive Adaptation of LLMs with Sketching",
section 2.2 Eq. 1 with groups per row, section 2.3 multiple LUT sets, on
LLaMA-shaped layers):
* 7B fine-tune step: 2-bit, 8 groups per row, T = 8192: Y, dX, dLUT;
* 13B forward and backward: 3-bit, one group per row, T = 4096: Y, dX, dLUT;
* 70B multi-task serving: 4-bit, 4 groups per row, 8 LUT sets with uniform
  task ids: decode at 1 and 64 tokens and prefill at 4096 tokens.

Tolerances are those of the other parity tests (tests/gpu_cases.py).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from compressive_fine_tuning_b200 import synth  # noqa: E402
from tests import gpu_cases as gc  # noqa: E402

pytestmark = pytest.mark.gpu

N_ROWS = 96
N_TOKENS = 64


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from compressive_fine_tuning_b200 import sk  # noqa: F401  (fails loudly if the library is missing)
    yield
    torch.cuda.synchronize()


@pytest.fixture(autouse=True)
def _default_paths(monkeypatch):
    # the library's own kernel choice, as in the benchmark
    monkeypatch.delenv("SK_FWD_PATH", raising=False)
    monkeypatch.delenv("SK_BWD_PATH", raising=False)


def _sk():
    from compressive_fine_tuning_b200 import sk
    return sk


def _sample(seed, total, k):
    return np.sort(synth.rng_for(seed).choice(total, size=min(k, total), replace=False))


def _check_y_rows(c, x, task, Y, rows):
    idx, lut = c.idx[rows], c.lut[:, rows]
    ref = oracle.forward(x, idx, lut, task)
    bound = oracle.forward(np.abs(x), idx, np.abs(lut.astype(np.float64)), task)
    gc.check_rows(gc.bf16_to_f64(Y)[:, rows], ref, bound, "Y (sampled rows)")


def _check_dx_tokens(c, dX, toks):
    dy = c.dy[toks]
    ref = oracle.backward_input(dy, c.idx, c.lut)
    bound = oracle.backward_input(np.abs(dy), c.idx, np.abs(c.lut.astype(np.float64)))
    gc.check_rows(gc.bf16_to_f64(dX[torch.from_numpy(toks).cuda()]), ref, bound, "dX (sampled tokens)")


def _check_dlut_rows(c, x, dl, rows):
    ref = oracle.backward_lut(x, c.dy[:, rows], c.idx[rows], c.gpr, c.k)
    gc.check_dlut(dl[0, torch.from_numpy(rows).cuda()].cpu().numpy(), ref, "dlut (sampled rows)")


def _train_layer(shapes, layer, bits, gpr, T, seed):
    """Y, dX and the LUT gradient of one full-size layer against the oracle."""
    sk = _sk()
    n, d = shapes[layer]
    c = synth.layer_case(seed, n=n, d=d, bits=bits, gpr=gpr, T=T)
    packed, lut, X, dY, _ = gc.dev_case(c)
    Y = sk.linear_fwd(packed, lut, bits, X)
    dX = sk.linear_bwd_input(packed, lut, bits, d, dY)
    dl = sk.linear_bwd_lut(packed, bits, gpr, X, dY)
    torch.cuda.synchronize()
    assert sk.device_check() == 0
    del packed, lut, X, dY
    x = c.x
    rows = _sample(seed + 1, n, N_ROWS)
    _check_y_rows(c, x, None, Y, rows)
    _check_dlut_rows(c, x, dl, rows)
    del x
    _check_dx_tokens(c, dX, _sample(seed + 2, T, N_TOKENS))


@pytest.mark.parametrize("layer", range(7), ids=synth.LAYER_NAMES)
def test_llama7b_finetune_full_size(layer):
    """7B-shaped fine-tune step: 2-bit, 8 groups per row, 8192 tokens."""
    _train_layer(synth.LLAMA2_7B, layer, bits=2, gpr=8, T=8192, seed=31_000 + 10 * layer)


@pytest.mark.parametrize("layer", range(7), ids=synth.LAYER_NAMES)
def test_llama13b_train_full_size(layer):
    """13B-shaped forward and backward: 3-bit (32 indices per three words), one
    group per row (5120- and 13824-column groups), 4096 tokens."""
    _train_layer(synth.LLAMA2_13B, layer, bits=3, gpr=1, T=4096, seed=32_000 + 10 * layer)


@pytest.mark.parametrize("layer", range(7), ids=synth.LAYER_NAMES)
def test_llama70b_multitask_serving_full_size(layer):
    """70B-shaped multi-task serving: 4-bit, 4 groups per row, 8 LUT sets
    sharing one index map, uniform task ids; decode at 1 and 64 tokens and
    prefill at 4096 tokens, each token with its own set."""
    sk = _sk()
    n, d = synth.LLAMA3_70B[layer]
    seed = 33_000 + 10 * layer
    c = synth.layer_case(seed, n=n, d=d, bits=4, gpr=4, T=4096, ntask=8)
    packed, lut, X, _, task = gc.dev_case(c)
    x_all = c.x
    rows = _sample(seed + 1, n, N_ROWS)
    for T in (1, 64, 4096):
        Y = sk.linear_fwd(packed, lut, 4, X[:T].contiguous(), task[:T].contiguous())
        torch.cuda.synchronize()
        assert sk.device_check() == 0
        _check_y_rows(c, x_all[:T], c.task[:T], Y, rows)
