"""Algorithmic byte accounting of the benchmark (the numerators of every GB/s and roofline
fraction it reports), against closed forms of the block layout: K q6_0 rows of 208 B, V
q5_0 rows of 176 B and q8_0 ring rows of 272 B at head_dim 256, fp32 inputs."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_row_bytes():
    assert (bench.ROW_K, bench.ROW_V, bench.ROW_T) == (8 * 26, 8 * 22, 8 * 34)


def test_decode_bytes_config_d():
    # 32,768 positions, 2,048 of them in the ring: 4 KV heads x (30,720 x 384 + 2,048 x 544)
    # plus q and out (24 heads x 256 fp32 each)
    assert bench.decode_bytes(32768) == 4 * (30720 * 384 + 2048 * 544) + 2 * 24 * 256 * 4
    # within the window every row is a ring row
    assert bench.decode_bytes(1024) == 4 * 1024 * 544 + 2 * 24 * 256 * 4


def test_append_bytes_steady_state():
    # a 1,024-position append once the ring is full: per position and KV head, fp32 K and V
    # (2,048 B), a ring write and an evicted ring read (2 x 544 B) and a low-bit row (384 B)
    per_pos = bench.append_bytes(8192, 1024) / 1024
    assert per_pos == 4 * (2048 + 544 + 544 + 384) == 14080


def test_append_bytes_filling_and_bulk():
    # while the ring fills nothing is evicted and no low-bit row is written
    assert bench.append_bytes(0, 1024) == 4 * 1024 * (2048 + 544)
    # an 8,192-position append into a full ring: 2,048 positions end in the ring (and evict
    # 2,048), 6,144 enter and leave; every position ends with a low-bit row
    assert bench.append_bytes(65536, 8192) == 4 * (8192 * 2048 + 2048 * 544 * 2 + 8192 * 384)
    # no ring
    assert bench.append_bytes(0, 100, W=0) == 4 * 100 * (2048 + 384)
