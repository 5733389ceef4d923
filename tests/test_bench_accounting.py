"""The benchmark's accounting against the figures it is defined by: the scan's algorithmic
bytes (q, k, v, g read and o written at 2 bytes, beta at 2: 1282 B per token and head,
20,512 B per token at H = 16, plus the fp32 final state) and the conv's multiply-adds
(taps x channels x tokens per segment, for q, k and v)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from linear_attention_sequence_mshortconv_b200 import inputs as W  # noqa: E402


def test_scan_bytes_of_the_video_clip():
    w = W.VIDEO_CLIP
    assert w.B * w.T == 32768 and w.H == 16 and w.D == 128
    state = 16 * 128 * 128 * 4
    assert bench.algorithmic_bytes(w) == 32768 * 20512 + state


def test_conv_multiply_adds_of_the_fused_stream():
    w = W.FUSED_MIXED
    C = w.H * w.D
    # text 512 tokens x Kt taps, image 64 x 64 x 9, video 21 x 32 x 48 x 27, for 3 tensors
    want = 3 * C * (512 * w.Kt + 64 * 64 * 9 + 21 * 32 * 48 * 27)
    assert bench.conv_fmas(w) == want


def test_tiny_fp32_bytes_use_four_byte_elements():
    w = W.TINY_FP32
    assert bench.algorithmic_bytes(w) == w.B * w.T * w.H * (5 * w.D * 4 + 4) + w.B * w.H * w.D * w.D * 4


def test_traffic_record_is_dropped_once_the_kernel_source_changes(tmp_path, monkeypatch):
    """A committed DRAM figure is reported only while the hash of the source it was taken
    on matches the file as it is; after any edit the bench reports null."""
    import hashlib
    import json

    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"wl": {"source": "kernel.cu", "source_sha256": hashlib.sha256(src.read_bytes()).hexdigest(),
                  "dram_bytes_per_step": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("wl") == 123
    assert bench.traffic_record("other") is None
    src.write_text("// version 2\n")
    assert bench.traffic_record("wl") is None


def test_committed_traffic_records_are_consistent():
    """Each committed record names a workload, its total is read + write, and it is not
    below the workload's algorithmic bytes (ncu saw at least the bytes the call must move,
    less what is still in L2 when the last launch ends)."""
    import json

    recs = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for name, rec in recs.items():
        assert name in W.BY_NAME, name
        assert rec["dram_bytes_per_step"] == rec["dram_read_bytes"] + rec["dram_write_bytes"], name
        assert rec["dram_bytes_per_step"] >= bench.algorithmic_bytes(W.BY_NAME[name]) * 0.9, name
