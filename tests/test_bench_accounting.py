"""The bench's partition byte count, worked by hand for the mid workload."""
import importlib.util
import os

from synthetic import workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_partition_bytes_mid_by_hand():
    # mid: 24 heads x 8192 rows, d = 128 (256 B per bf16 row), 32 fp32 key
    # coordinates (128 B per row), T = 10 iterations.  Per row:
    #   RMS + 10 query assignments 11 x 256; projection 256 + 128;
    #   10 key assignments 10 x 128; three permuted copies 3 x 512;
    #   two group-mean passes 2 x 256
    #   2816 + 384 + 1280 + 1536 + 512            -> 6528 B per row
    wl = workload("mid")
    per_row = 11 * 256 + 256 + 128 + 10 * 128 + 3 * 512 + 2 * 256
    assert per_row == 6528
    assert _bench().partition_bytes(wl) == per_row * 8192 * 24


def _fake_tree(tmp_path, source: bytes, profile: str):
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "free_block_sparse_means_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k_attend_tc.cu").write_bytes(source)
    (tmp_path / "profiles" / "k_attend_tc_hunyuan.md").write_text(profile)


def test_profiled_traffic_scales_by_heads_and_checks_the_source(tmp_path):
    import hashlib
    b = _bench()
    src = b"// kernel source\n"
    sha = hashlib.sha256(src).hexdigest()[:16]
    prof = ("# capture\n\n    kernel_source_sha256_16: %s\n    workload: hunyuan\n"
            "    heads_captured: 2\n    traffic_bytes_per_launch: 1000\n" % sha)
    _fake_tree(tmp_path, src, prof)
    b.ROOT = str(tmp_path)
    # 2 of 24 heads captured: the full launch moves 12 x the bytes
    assert b.profiled_traffic("hunyuan", 24) == 12000
    assert b.profiled_traffic("hunyuan", 2) == 1000
    # another workload has no capture
    assert b.profiled_traffic("wan", 40) is None
    # a changed kernel source voids the figure
    (tmp_path / "free_block_sparse_means_b200" / "csrc" / "k_attend_tc.cu").write_bytes(
        src + b"// edited\n")
    assert b.profiled_traffic("hunyuan", 24) is None
