"""Host-side measurement logic of bench.py (no GPU): the algorithmic byte
counts the rooflines divide by, and the kernel-source hash that keeps a
committed DRAM-traffic capture tied to the sources it was taken on."""
import bench
from block_scaled_precision_05_b200 import _native as nat


def test_quantize_algorithmic_bytes():
    # 2 B read + 0.5 B codes per element, one scale byte per 16 on padded rows
    assert bench.quant_bytes(32760, 1536, "nvfp4") == 32760 * 1536 * 2 + 32760 * 768 + 32768 * 96
    assert bench.quant_bytes(16, 5120, "nvfp4", "8x4") == 16 * 5120 * 2 + 16 * 2560 + 16 * 320
    assert bench.quant_bytes(1, 5120, "nvfp4") == 5120 * 2 + 2560 + 128 * 320
    # MXFP8: 2 B read + 1 B elements, one scale byte per 32
    assert bench.quant_bytes(32760, 5120, "mxfp8") == 32760 * 5120 * 3 + 32768 * 160
    # the scale term is exactly the library's scale-buffer size
    for M, K in ((1, 64), (130, 80), (32760, 1536), (7, 13824)):
        assert bench.quant_bytes(M, K, "nvfp4") - 2 * M * K - M * K // 2 == nat.lib().bsp_nvfp4_sf_bytes(M, K)


def test_source_hash_ignores_comments_and_layout():
    a = 'int f(int x) {\n  // a comment\n  return x + 1; /* block\n comment */\n}\nconst char* s = "// kept";\n'
    b = 'int f(int x) { return x + 1; }\nconst char* s = "// kept";'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only('x = "a /* b */ c";') == 'x = "a /* b */ c";'
    assert bench._code_only("int a = 1;") != bench._code_only("int a = 2;")
    h = bench.source_hash()
    assert len(h) == 16 and h == bench.source_hash()


def test_traffic_entries_are_keyed_to_their_kernels_sources():
    import json
    import os
    assert bench.kernel_source_hash("nvfp4_gemm") == bench.kernel_source_hash("mxfp8_gemm")
    assert bench.kernel_source_hash("nvfp4_gemm") != bench.kernel_source_hash("nvfp4_quantize")
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    for workload, entries in t.items():
        if workload.startswith("_"):
            continue
        for kernel, e in entries.items():
            assert tuple(e["sources"]) == bench.KERNEL_SOURCES[kernel]
            assert abs(e["read"] + e["write"] - e["dram_bytes_per_launch"]) <= 1  # each averaged, then truncated
