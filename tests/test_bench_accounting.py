"""Algorithmic byte and FLOP accounting of the benchmark (the numerators of every GB/s,
TFLOP/s and roofline fraction it reports), against closed forms of the block layout: K q6_0
rows of 208 B, V q5_0 rows of 176 B and q8_0 ring rows of 272 B at head_dim 256, fp32
inputs; and the causal prefill FLOP count of the full-length workload."""
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


def test_headline_step_accounting():
    a = bench.step_accounting()
    # 64 decode steps x 16 layers at 262,081 .. 262,144: 4 KV heads x ((n - 2048) x 384 + 2048 x 544) + q, out
    want = 16 * sum(4 * ((n - 2048) * 384 + 2048 * 544) + 2 * 24 * 256 * 4 for n in range(262081, 262145))
    assert a["decode_bytes"] == want
    # one decode at 262,080 reads ~404 MB (399.5 MB of low-bit rows + 4.46 MB of ring rows)
    assert abs(bench.decode_bytes(262080) - 403.9e6) < 0.1e6
    # the fill: 257,984 positions per layer; the first 2,048 only touch the ring, every later
    # position is written once to the low-bit store; 2,048 stay in the ring at the end
    per_layer = 4 * (257984 * 2048 + (257984 - 2048) * 384 + 2048 * 544 + (32 - 1) * 2048 * 544 * 2)
    assert a["fill_bytes"] == 16 * per_layer
    assert a["fill_positions"] == 16 * 257984
    # launches: 32 fill appends + the chunk append + the prefill's three (tile images, staged
    # kernel, split merge) per layer; each decode step appends once and launches the ring
    # pass, the low-bit pass and the merge per layer
    assert a["launches"] == 16 * 36 + 16 * 64 * 4


def test_prefill_flop_count():
    # row i of the 4,096-row chunk attends to 257,984 + i + 1 keys: sum = C n + C (C + 1) / 2
    keys = 4096 * 257984 + 4096 * 4097 // 2
    assert bench.prefill_flops(257984, 4096) == keys * 24 * 4 * 256
    assert abs(bench.prefill_flops(257984, 4096) - 2.62e13) < 0.01e13      # per layer
    assert bench.prefill_flops(0, 1) == 24 * 4 * 256


def test_end_to_end_copy_volumes():
    # every fill append's K and V, the chunk's K, V and queries, the decode steps' K, V, q
    assert bench.hi_h2d() == 16 * 4 * (257984 * 2 * 4 * 256 + 4096 * (2 * 4 * 256 + 24 * 256) + 64 * (2 * 4 * 256 + 24 * 256))
    assert bench.hi_d2h() == 16 * 4 * (4096 + 64) * 24 * 256
