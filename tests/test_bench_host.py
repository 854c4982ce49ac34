"""Host-side accounting of the benchmark, on CPU: a captured DRAM-traffic record
is reported only while its kernel sources are unchanged, and the per-call
algorithmic bytes of the indexer loss match the count in its profile summary."""
import hashlib
import os

import bench
from sparse_long_context_04_b200 import workloads as W


def test_captured_traffic_follows_the_sources(tmp_path):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    rec = tmp_path / "traffic.txt"

    def write_record(body_sha):
        rec.write_text(f"# comment\nsources={src}\nsha256={body_sha}\ntraffic_bytes_per_launch=12345\n")

    write_record(hashlib.sha256(src.read_bytes()).hexdigest())
    assert bench.captured_traffic(str(rec)) == 12345
    src.write_text("// kernel v2\n")                       # the kernel changed since the capture
    assert bench.captured_traffic(str(rec)) is None
    assert bench.captured_traffic(str(tmp_path / "missing.txt")) is None


def test_committed_traffic_records_name_existing_sources():
    for name in ("indexer_fp8_traffic.txt", "indexer_kl_traffic.txt"):
        path = os.path.join(bench.ROOT, "profiles", name)
        kv = dict(line.split("=", 1) for line in open(path).read().splitlines()
                  if line and not line.startswith("#") and "=" in line)
        for f in kv["sources"].split():
            assert os.path.exists(os.path.join(bench.ROOT, f)), f
        assert int(kv["traffic_bytes_per_launch"]) > 0


def test_indexer_loss_bytes_match_the_profile_count():
    # 16 rows x 2048 valid slots: 1152 + 4 B per slot, 147,456 + 512 + 4 B per row,
    # 8 B per slot for the index and the gradient
    s = W.PAGED_DECODE_128K
    out = bench.indexer_kl_summary(28.9, 16, s, 16 * 2048, 6559.0, "measured")
    assert out["algorithmic_bytes_per_call"] == 40_509_504
    assert abs(out["frac"] - out["achieved"] / 6559.0) < 1e-12
    assert out["bound"] == "hbm" and out["unit"] == "GB/s"


def test_attention_backward_bytes_by_hand():
    # 32768 slots x (1152 + 2 x 2304) + 16 rows x 128 heads x (1152 + 2 x 1024 + 4)
    # + dq read and written 16 x 128 x 576 x 8 + the selection 16 x 2048 x 4
    s = W.PAGED_DECODE_128K
    out = bench.attn_backward_summary(50.0, 16, s, 16 * 2048, 6559.0, "measured")
    assert out["algorithmic_bytes_per_call"] == 188_743_680 + 6_561_792 + 9_437_184 + 131_072
