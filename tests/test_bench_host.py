"""Host-side logic of bench.py, on CPU: the mirror of the library's kernel
selection, the DRAM-traffic table and the code hashes that key it, and the
units and descriptions a bench line is built from."""
import types

import pytest

import bench
from rwkv_linear_rnn_b200 import workloads


@pytest.mark.parametrize("op", ["fwd", "bwd"])
@pytest.mark.parametrize("gate", [False, True])
def test_auto_kernel_on_the_workload_shapes(op, gate):
    """The 1.5B-shaped layer (512 chains) occupies 60 % or more of the 148 x 4
    warp schedulers: chain kernels.  The 169M-shaped layer (192
    chains) and the long sequence (80 chains) do not."""
    assert bench.auto_kernel(op, 8, 2048, gate) == "chain"
    assert bench.auto_kernel(op, 8, 768, gate) in ("tile", "segment")
    assert bench.auto_kernel(op, 1, 2560, gate) == "segment"


def test_auto_kernel_chain_threshold():
    """From 60 % of the 148 x 4 warp schedulers up (356 chains), in one wave
    or several, the chain kernels run; below it, the time-parallel ones."""
    slots = 4 * 148
    lo = (3 * slots + 4) // 5  # the fewest chains with chains * 5 >= 3 * slots
    assert lo == 356
    assert bench.auto_kernel("fwd", lo, 32, False) == "chain"
    assert bench.auto_kernel("fwd", lo - 1, 32, False) != "chain"
    assert bench.auto_kernel("fwd", slots, 32, False) == "chain"
    assert bench.auto_kernel("bwd", 3 * slots + 7, 32, True) == "chain"
    # a ragged channel tile counts as a chain
    assert bench.auto_kernel("bwd", 1, 32 * lo - 31, False) == "chain"


def test_every_selectable_kernel_has_sources():
    for plan in (bench.FWD_PLAN, bench.BWD_PLAN):
        for sel, (kernel, launches) in plan.items():
            assert sel in bench.KERNEL_IDS
            assert launches >= 1
            if kernel in ("fwd_clu_kernel",):
                continue  # selectable, never the bench's dominant kernel
            assert kernel in bench.KERNEL_SOURCES, kernel
            assert len(bench.kernel_hash(kernel)) == 16


def test_code_hash_ignores_comments_and_blank_lines():
    a = "int f() {  // one\n  return 1; /* two\n three */\n}\n\n"
    b = "int f() {\n  return 1;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(b) != bench._code_only(b.replace("1", "2"))


def test_traffic_table_is_keyed_by_the_current_code():
    """Every recorded traffic figure is positive and at most the DRAM bytes
    a launch could plausibly move; a lookup answers only for the kernel's
    current code hash, and an unknown workload gets None."""
    for (wl, kernel, gated, h), val in bench.TRAFFIC.items():
        assert val > 0
        assert len(h) == 16
        if h == bench.kernel_hash(kernel):
            assert bench.traffic_for(wl, kernel, gated) == val
    assert bench.traffic_for("no_such_workload", "fwd_chain_kernel", False) is None


def test_units_and_modes_of_the_workloads():
    c3 = workloads.WORKLOADS["rwkv1b5_bf16"]
    assert bench.workload_mode("rwkv1b5_bf16") == "fwdbwd"
    assert bench.units_per_step(c3) == 8 * 4096 * 2048
    assert bench.workload_mode("longctx") == "fwd"
    assert bench.workload_mode("decode14b") == "step"
    dec = workloads.WORKLOADS["decode14b"]
    assert bench.units_per_step(dec) == dec.B * dec.C * dec.steps
    assert "fwd+bwd" in bench.metric_name("fwdbwd", False)
    assert "gated" in bench.metric_name("fwdbwd", True)
    assert "decode-step" in bench.metric_name("step", False)


def test_config_names_the_workload_and_its_sizes():
    args = types.SimpleNamespace(gate=False)
    cfg = bench.make_config(args, workloads.WORKLOADS["rwkv1b5_bf16"], 1)
    assert cfg["workload"] == "rwkv1b5_bf16"
    assert (cfg["B"], cfg["T"], cfg["C"]) == (8, 4096, 2048)
    assert cfg["io_dtype"] == "bf16"
    assert "flushed" in cfg["l2"]
    assert cfg["parallelism"] == "single GPU"
    cfg2 = bench.make_config(types.SimpleNamespace(gate=True), workloads.WORKLOADS["rwkv169m"], 2)
    assert cfg2["gate"] is True and cfg2["parallelism"] == "replicas x2"


def test_peak_falls_back_without_measurements(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == (6650.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6443.2}')
    assert bench.peaks() == (6443.2, "measured")
