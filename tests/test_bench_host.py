"""Host-side pieces of bench.py: the algorithmic units behind every reported
rate, the kernel attribution and the traffic records (no GPU needed)."""
import json
import os

import pytest

import bench
from compressive_fine_tuning_b200 import synth

W = bench.WORKLOADS


def test_decode_bytes_match_the_layer_shapes():
    """Algorithmic bytes of a 4-bit, GPR-8 decode launch: n d / 2 of indices,
    n * 8 * 16 * 2 of LUTs, (n + d) * 2 * T of activations.  Summed over the
    seven 7B layers at T = 1: 101 187 584 index bytes and 10 878 976 LUT bytes."""
    assert bench.launch_bytes(4096, 4096, 4, 8, 1) == 8_388_608 + 1_048_576 + 16_384
    idx = sum(n * d // 2 for n, d in synth.LLAMA2_7B)
    lut = sum(n * 8 * 16 * 2 for n, d in synth.LLAMA2_7B)
    assert idx == 101_187_584 and lut == 10_878_976
    total = sum(bench.launch_bytes(n, d, 4, 8, 1) for n, d in synth.LLAMA2_7B)
    assert total == idx + lut + sum((n + d) * 2 for n, d in synth.LLAMA2_7B)


def test_training_flops_are_three_products():
    T = 8192
    step = sum(bench.launch_flops(n, d, T, op) for n, d in synth.LLAMA2_7B for op in ("fwd", "dx", "dlut"))
    assert step == 6 * T * sum(n * d for n, d in synth.LLAMA2_7B)
    assert abs(step - 9.95e12) < 0.01e12


@pytest.mark.parametrize("op,T,workload,name", [
    ("fwd", 1, "decode7b", "decode_group_kernel"),
    ("fwd", 16, "decode7b", "decode_group_kernel"),
    ("fwd", 8192, "finetune7b", "fwd_tc_pair_kernel"),
    ("fwd", 128, "finetune7b", "fwd_tc_kernel"),
    ("dx", 8192, "finetune7b", "dx_tc_pair_kernel"),
    ("dx", 8192, "finetune7b_mt", "dx_tc_pair_kernel (routed)"),
    ("dlut", 8192, "finetune7b_mt", "dlut_tc_pair_kernel (routed)"),
    ("fwd", 1, "serve70b_decode", "decode_group_kernel"),
    ("fwd", 64, "serve70b_decode", "fwd_tc_kernel (routed)"),
    ("fwd", 4096, "serve70b_prefill", "fwd_tc_pair_kernel (routed)"),
])
def test_kernel_attribution(op, T, workload, name, monkeypatch):
    monkeypatch.delenv("SK_FWD_PATH", raising=False)
    monkeypatch.delenv("SK_TC_PAIR", raising=False)
    monkeypatch.delenv("SK_DX_PAIR", raising=False)
    monkeypatch.delenv("SK_DLUT_PAIR", raising=False)
    assert bench.kernel_name(op, T, W[workload]) == name


def test_kernel_attribution_single_cta_forward(monkeypatch):
    monkeypatch.delenv("SK_FWD_PATH", raising=False)
    monkeypatch.setenv("SK_TC_PAIR", "0")
    assert bench.kernel_name("fwd", 8192, W["finetune7b"]) == "fwd_tc_kernel"
    assert bench.kernel_name("fwd", 4096, W["serve70b_prefill"]) == "fwd_tc_kernel (routed)"
    monkeypatch.setenv("SK_DX_PAIR", "0")
    assert bench.kernel_name("dx", 8192, W["finetune7b"]) == "dx_tc_kernel"
    monkeypatch.setenv("SK_DLUT_PAIR", "0")
    assert bench.kernel_name("dlut", 8192, W["finetune7b"]) == "dlut_tc_kernel"


def test_sketch_factor_launch_count():
    """The inverse factor of a 4096-wide Gram matrix: 2 (damping, reversal) +
    Cholesky (64 diagonal blocks, 63 panels, 32 strip and 31 trailing updates)
    + identity + inverse (64 block rows, 32 strip and 31 trailing updates) + 2
    (reversal, norms) = 322 launches, as the ncu launch list of the stage shows."""
    assert bench.sketch_factor_launches(4096) == 2 + (64 + 63 + 32 + 31) + 1 + (64 + 32 + 31) + 2 == 322


def test_traffic_records_are_well_formed():
    """Every record names a workload and its kernel's sources; it reads back
    exactly when the sources are unchanged since the capture, else as null."""
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    recs = json.load(open(path))
    for key, rec in recs.items():
        kernel, workload = key.split("@")
        assert workload in W, key
        assert rec["dram_bytes"] > 0 and rec["algorithmic_units"] > 0 and rec["source"]
        got = bench.traffic_per_launch(kernel, workload, rec["algorithmic_units"])
        assert got in (rec["dram_bytes"], None), key


def test_stale_traffic_reads_as_null(monkeypatch, tmp_path):
    recs = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    key = next(iter(recs))
    recs[key]["source_sha256"] = "0" * 64
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(recs))
    csrc = tmp_path / "compressive_fine_tuning_b200"
    csrc.symlink_to(os.path.join(bench.ROOT, "compressive_fine_tuning_b200"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    kernel, workload = key.split("@")
    assert bench.traffic_per_launch(kernel, workload, recs[key]["algorithmic_units"]) is None


def test_every_batch_reads_its_own_weight_copy():
    """Decode: the T=1 and T=16 batches of a step, and consecutive steps, read
    distinct copies; a copy returns only after all the others, which together
    hold more than 3x L2 of index bytes."""
    w = W["decode7b"]
    weight_bytes = sum(n * d * w["bits"] // 8 for n, d in synth.LLAMA2_7B)
    copies = max(2, int(-(-3 * bench.L2_BYTES // weight_bytes)) + 1)
    nb = len(w["batches"])
    seq = [bench.weight_copy(s, bi, nb, copies) for s in range(12) for bi in range(nb)]
    for i in range(len(seq)):
        window = seq[i:i + copies]
        assert len(set(window)) == len(window)
    assert (copies - 1) * weight_bytes > 3 * bench.L2_BYTES
