"""Host-side bench logic that needs no GPU: the traffic figure read from the
committed ncu summaries is attached only to the launch it was captured on,
and the algorithmic byte counts of every row are what their formulas say."""
import bench
from outlier_split_bit_b200 import workload as wl


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


def test_summary_is_last_and_short():
    """The line's last key digests the rows a reader needs; the driver keeps
    only the tail of a long line, so the digest stays under 1400 characters
    with every row present."""
    import json
    line = {"us_per_step": 324.1, "roofline": {"frac": 0.9562}, "e2e": {"value": 6118.7}}
    per = [{"matrix": s.name, "bytes": 9_000_000 + i, "frac": 0.543} for i, s in enumerate(wl.LAYER_1P5B)]
    sweep = [{"matrix": s.name, "m": m, "frac": 0.123} for s in wl.LAYER_4B for m in wl.BATCH_SWEEP]
    extra = {
        "decode_stream_tau6": {"us_per_step": 197.31, "frac": 0.6212},
        "decode_stream_dependent_chain": {"us_per_step": 548.22, "frac": 0.6212, "us_per_launch": 548.22},
        "decode_stream_dependent_launches": {"us_per_step": 1148.22, "frac": 0.2712, "us_per_launch": 5.858},
        "decode_stream_stages_chain": {"us_per_step": 1250.24, "frac": 0.2479, "us_per_launch": 1250.24},
        "decode_stream_stages_launches": {"us_per_step": 1106.35, "frac": 0.2801, "us_per_launch": 9.878},
        "embed_rows_row_table_131072x3072_bf16": [{"frac_single_flushed": 0.224}],
        "per_matrix_1p5b": per, "batch_sweep_4b": sweep,
        "lm_head_131072x3072": [{"frac_t_columns": f, "frac": 0.801} for f in wl.LM_HEAD_FRACTIONS],
        "lm_head_batch_131072x3072": [{"m": m, "frac": 0.371} for m in (1, 16, 32)],
        "single_512x512": [{"tau": t, "us_back_to_back": 3.12, "oracle_us_1thread": 912.3} for t in (3.0, 6.0)],
        "trdc_container_4_layers": {"load_gbs": 1.84},
        "kv_attention_decode_8192": [{"us_back_to_back": 16.72}, {"us_back_to_back": 26.45}],
        "embed_rows_131072x3072_bf16": [{"frac_single_flushed": 0.16}],
    }
    cpu = {"cores": 224, "matvec_gbs_1thread": 0.1396, "matvec_gbs_all_cores": 12.3456,
           "pack_mweights_per_s_1thread": 30.84, "pack_mweights_per_s_all_cores": 1575.53}
    s = bench.summary_of(line, extra, cpu)
    text = json.dumps({"summary": s})
    assert len(text) < 1400, len(text)
    assert set(s["ge8MB_m1_frac"]) >= {"1p5b_gate", "4b_gate", "4b_up", "4b_down", "lm_head_t0.1"}
    assert s["tc_frac"]["4b_gate_m16"] == 0.123 and s["tc_frac"]["lm_head_m32"] == 0.371
    assert s["chain"]["frac"] == 0.621 and s["chain_196_launches"]["us"] == 1148.22
    assert s["stream_tau6"]["frac"] == 0.621
    assert s["stages_chain"]["us"] == 1250.24 and s["stages_112_launches"]["frac"] == 0.28
    assert s["cpu"]["matvec_gbs"] == [0.1396, 12.3456]


def test_decoder_stages_group_shared_inputs():
    names = [s.name for _ in range(3) for s in wl.LAYER_1P5B]
    st = bench.decoder_stages(names)
    # q, k, v | o | gate, up | down, four stages per layer, nondecreasing
    assert st[:7] == [0, 0, 0, 1, 2, 2, 3]
    assert st[7:14] == [4, 4, 4, 5, 6, 6, 7]
    assert st == sorted(st) and len(set(st)) == 12

