"""The roofline's DRAM traffic comes from a committed ncu record keyed to the attention
kernel's device code: it is reported for that exact code and dropped (None) as soon as
the kernel text changes; host code after the kernel does not affect it."""
import os
import shutil

import bench

SRC = os.path.join(bench.ROOT, "streaming_flow_matching_b200", "csrc", "attn_tc.cu")
TABLE = os.path.join(bench.ROOT, "profiles", "traffic.json")


def _copy(tmp_path, edit=None):
    d = tmp_path / "attn_tc.cu"
    shutil.copy(SRC, d)
    if edit:
        text = d.read_bytes()
        d.write_bytes(edit(text))
    return str(d)


def test_record_matches_the_committed_kernel():
    assert bench.traffic_for(SRC, TABLE) is not None


def test_host_code_edits_keep_the_record(tmp_path):
    p = _copy(tmp_path, lambda t: t + b"\n// host-side note\n")
    assert bench.traffic_for(p, TABLE) == bench.traffic_for(SRC, TABLE)


def test_kernel_edits_drop_the_record(tmp_path):
    end = open(SRC, "rb").read().find(bench.KERNEL_END)
    assert end > 0
    p = _copy(tmp_path, lambda t: t[:end] + b"// changed\n" + t[end:])
    assert bench.traffic_for(p, TABLE) is None
