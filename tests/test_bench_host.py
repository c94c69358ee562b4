"""Host-side bench logic that needs no GPU: the traffic figure read from the
committed ncu summary is attached only to the launch it was captured on."""
import bench


def test_traffic_needs_matching_source_digest():
    assert bench.profiled_traffic("0" * 16) is None


def test_traffic_needs_matching_algorithmic_bytes():
    d = bench.kernel_source_digest()
    t = bench.profiled_traffic(d)
    if t is None:
        return  # summary predates the current source; nothing to attach
    vals = {}
    for line in open(bench.os.path.join(bench.ROOT, "profiles", "gemv_decode_stream_traffic.md")):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    alg = int(vals["algorithmic_bytes_per_launch"])
    assert bench.profiled_traffic(d, alg) == t
    assert bench.profiled_traffic(d, alg + 1) is None
    # the tau = 6 stream moves fewer bytes and must not borrow the tau = 3 capture
    assert bench.profiled_traffic(d, 800191364) is None


def test_algorithmic_bytes_counts_every_stream():
    # 32 x 64 bulk at 4.625 bits per weight (4-bit code, FP16 scale and 4-bit
    # zero point per 32) = 1184 B; one BF16 outlier column of 32 rows = 64 B;
    # its int32 index = 4 B; x = 64 BF16 = 128 B; y = 32 FP32 = 128 B.
    assert bench.algorithmic_bytes(32, 64, 1) == 1184 + 64 + 4 + 128 + 128
