"""Host-side pieces of bench.py that need no GPU: the algorithmic byte counts
behind every GB/s figure and the launch count it reports."""
import bench


def test_packed_bytes_match_formats():
    # base-3: ceil(G/5) code bytes + 2 scale bytes per group
    assert bench.packed_bytes(3584, 1024, 64) == 3584 * 16 * (13 + 2)
    assert bench.packed_bytes(1024, 3584, 128) == 1024 * 28 * (26 + 2)
    # 2-bit: G/4 code bytes + 2 scale bytes per group
    assert bench.packed2_bytes(3584, 1024, 64) == 3584 * 16 * (16 + 2)
    assert bench.packed2_bytes(172032, 1024, 128) == 172032 * 8 * (32 + 2)
    # the page's payload rates: 1.875 and 1.75 bits per weight
    assert bench.packed_bytes(3584, 1024, 64) * 8 / (3584 * 1024) == 1.875
    assert bench.packed_bytes(3584, 1024, 128) * 8 / (3584 * 1024) == 1.75


def test_count_launches_nested():
    res = {"stream": {"launches": 48, "us": 1.0},
           "pack": {"G64": {"launches": 24}, "G128": {"launches": 24}},
           "ternary2": {"pack": {"G64": {"launches": 6}}, "decode_stack": {"launches": 864,
                                                                          "launches_per_step": 288}},
           "note": "launches", "other": [1, 2]}
    assert bench.count_launches(res) == 48 + 24 + 24 + 6 + 864
