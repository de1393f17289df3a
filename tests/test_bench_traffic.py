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


def test_roofline_work_counts_at_640x368():
    # the numerators of the bench's roofline fractions, against hand counts:
    # attention 4 N (S_c + N) H D per layer launch, GEMMs 2 M K N, append K+V read + write
    import sfm_synth as S
    w = S.V02
    fl = bench.flop_counts(w, [57600])
    assert fl["attention_per_launch"] == 4 * 924 * (57600 + 924) * 24 * 128 == 664488050688
    assert fl["gemm_per_layer"] == 2 * 924 * 3072 * (9216 + 3072 + 12288 + 12288)
    assert abs(fl["per_euler_step"] / 1e12 - 24.47) < 0.01
    assert bench.append_bytes(w) == 2 * 2 * 28 * 1200 * 3072 * 2 == 825753600
    # a ragged batch counts every session's own cache
    fl2 = bench.flop_counts(w, [57600, 1200])
    assert fl2["attention_per_launch"] == fl["attention_per_launch"] + 4 * 924 * (1200 + 924) * 3072
    assert fl2["gemm_per_layer"] == 2 * fl["gemm_per_layer"]
