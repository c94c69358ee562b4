"""Host-side bench logic that needs no GPU: the traffic figure read from the
committed ncu summaries is attached only to the launch it was captured on,
and the algorithmic byte counts of every row are what their formulas say."""
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


def test_compacted_traffic_summary_is_matched_by_its_own_bytes():
    d = bench.kernel_source_digest()
    per_file = {}
    for name in bench.TRAFFIC_PROFILES:
        vals = {}
        for line in open(bench.os.path.join(bench.ROOT, "profiles", name)):
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
        per_file[name] = vals
    for name, vals in per_file.items():
        if vals.get("kernel_source_sha256_16") != d:
            continue  # captured on an older source: nothing to attach
        alg = int(vals["algorithmic_bytes_per_launch"])
        assert bench.profiled_traffic(d, alg) == float(vals["dram_bytes_per_launch"]), name


def test_compacted_bytes_count_the_bulk_columns_only():
    # n = 32, k = 96, 40 outlier columns -> k_bulk = 64: bulk 32 x 64 at
    # 4.625 bits = 1184 B; the bulk column list 64 x 4 = 256 B; 40 BF16 outlier
    # columns of 32 rows = 2560 B; their indices 160 B; x = 96 BF16 = 192 B;
    # y = 32 FP32 = 128 B
    assert bench.algorithmic_bytes_compact(32, 96, 64, 40) == 1184 + 256 + 2560 + 160 + 192 + 128

    class Lay:
        n, k, n_outliers, k_bulk, compact = 32, 96, 40, 64, True

    assert bench.layer_bytes(Lay()) == bench.algorithmic_bytes_compact(32, 96, 64, 40)
    Lay.compact = False
    assert bench.layer_bytes(Lay()) == bench.algorithmic_bytes(32, 96, 40)


def test_embedding_bytes():
    # two rows of a 64-column table with 3 outlier columns, BF16 out: per row
    # 64 * 4.625 / 8 = 37 B of codes, scales and zeros, 6 B of outliers, a
    # 4-byte id and 128 B written; plus the 3 indices once
    assert bench.embed_bytes(64, 3, 2) == 2 * (32 + 4 + 1 + 6 + 4 + 128) + 12
