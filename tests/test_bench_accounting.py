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
