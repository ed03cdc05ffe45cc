"""bench.py's reference arm (the fp64 oracle timed on the host cores) prints
one JSON line with the keys of the GPU arm's line plus ``impl``,
``cpu_baseline`` and a zero-copy ``e2e``; run here on small workloads (the
tiny causal layer, and a varlen batch with a resident prefix that is not a
multiple of the block, a decode row and an empty sequence)."""
import argparse
import json

import bench
from block_sparse_long_blockmean_b200 import synth
from tests import harness as H

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
        "cpu_baseline", "e2e"}


def _args(workload):
    return argparse.Namespace(workload=workload, drop=None, warmup=1, steps=2, gpus=1,
                              group_masks=False, out_fp8=False)


def _line(capsys):
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1, out
    return json.loads(out[0])


def _check(line, steps):
    assert KEYS <= set(line), KEYS - set(line)
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "ms/layer" and line["higher_is_better"] is False
    assert line["steps"] == steps and line["value"] > 0 and line["value"] == line["ms_per_step"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_line_on_the_tiny_layer(capsys):
    bench.reference_arm(_args(1))
    line = _line(capsys)
    _check(line, 2)
    assert line["config"]["seq_len"] == 1024 and line["config"]["num_q_heads"] == 4


def test_reference_line_on_a_varlen_batch(monkeypatch, capsys):
    shape = H.small_shape([300, 1, 0, 200], [300 + 77, 500, 40, 200], Hq=4, Hkv=2, d=16, B=16,
                          seed=31, drop=0.6)
    monkeypatch.setattr(synth, "workload", lambda cid, dtype=None: shape)
    monkeypatch.setitem(synth.WORKLOAD_NAMES, 99, "small varlen test batch")
    bench.reference_arm(_args(99))
    line = _line(capsys)
    _check(line, 2)
    cfg = line["config"]
    assert cfg["global_batch"] == 4 and cfg["seq_lens"] == [300, 1, 0, 200]
    assert cfg["prefix_lens"] == [77, 499, 40, 0] and cfg["total_tokens"] == 501
    assert "all 4 sequence(s)" in line["cpu_baseline"]["sample"]
