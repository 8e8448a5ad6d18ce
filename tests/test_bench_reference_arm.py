"""bench.py's reference arm (CPU): the fp64 oracle timed on a bounded sample of
the step's dominant part, reported on the native arm's metric, unit and step
config, with no host-device bytes and no GPU launches; ranks other than 0
do no work."""
import argparse
import json

import bench


def test_reference_arm_line_matches_the_native_contract():
    args = argparse.Namespace(steps=1, warmup=1, cpu_seconds=0.3)
    line = bench.run_reference(args, 0, 1)
    json.dumps(line)                                     # one JSON line
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["config"] == bench.step_config(1)        # the same workload as the native arm
    assert line["steps"] == 1 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["ms_per_step"] > 0
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1 and cpu["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert line["gpu_launches"] == 0


def test_reference_arm_other_ranks_do_no_work():
    args = argparse.Namespace(steps=1, warmup=1, cpu_seconds=0.3)
    assert bench.run_reference(args, 1, 2) is None
