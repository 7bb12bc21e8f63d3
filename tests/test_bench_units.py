"""The bench's algorithmic units for the 70B MLP layer (28672×8192, 2:4, r = 256,
top-k at 5 %), checked term by term against counts worked out by hand from the
layouts (bf16 values, 4-bit 2:4 metadata per group, int32 CSR columns, bf16
values and int32 row pointers)."""
import bench


def test_decode_bytes_terms():
    m, n, r = 28672, 8192, 256
    values = m * n // 2 * 2                 # kept half, bf16: 234,881,024
    meta = m * (n // 4) // 2                # 4 bits per group: 29,360,128
    factors = (m + n) * r * 2               # U and V, bf16: 18,874,368
    xy = (n + m) * 2                        # x and y of one token: 73,728
    assert (values, meta, factors, xy) == (234_881_024, 29_360_128, 18_874_368, 73_728)
    assert bench.decode_bytes() == values + meta + factors + xy == 283_189_248


def test_prefill_flops():
    # 2·T·(nnz + r·(m + n)) with nnz = m·n/2 and T = 4096 tokens
    assert bench.prefill_flops() == 2 * 4096 * (117_440_512 + 256 * 36_864) == 1_039_382_085_632


def test_split_bytes():
    k = 11_744_051                          # floor(0.05 · 28672 · 8192)
    rw = 2 * 28672 * 8192 * 2               # read W + write R, bf16
    assert bench.split_topk_bytes() == rw + k * (4 + 2) + 28673 * 4 == 1_010_103_094
    assert bench.split_24_bytes() == rw + 117_440_512 * 2 + 28672 * 2048 == 1_233_125_376


def test_decode_traffic_comes_from_the_profile_of_the_current_source(tmp_path, monkeypatch):
    """roofline.traffic is read from the committed ncu summary, and only while
    the kernel source is the one the capture was taken on."""
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    prof = tmp_path / "p.md"
    prof.write_text(f"x\ndram_bytes_per_launch: 286874880\nsource_digest: `{bench.source_digest(str(src))}`\n")
    monkeypatch.setattr(bench, "DECODE_PROFILE", str(prof))
    monkeypatch.setattr(bench, "DECODE_SOURCE", str(src))
    assert bench.decode_traffic() == 286_874_880
    src.write_text("kernel v2")
    assert bench.decode_traffic() is None
    monkeypatch.setattr(bench, "DECODE_PROFILE", str(tmp_path / "missing.md"))
    assert bench.decode_traffic() is None


def test_workload_units():
    # 4096² CSR at 2 %: 335,544 bf16 values + 16-bit columns, 4097 row pointers,
    # U and V of rank 128, one token in and out
    assert bench.csr_apply_bytes(335_544, 4096, 4096, 128, 1, 2) == \
        335_544 * 4 + 4097 * 4 + 8192 * 128 * 2 + 8192 * 2 == 3_472_100
    # 11008×4096 2:4, r = 64, batch 16
    assert bench.nm24_apply_bytes(11008, 4096, 64, 16) == \
        11008 * 2048 * 2 + 11008 * 1024 // 2 + 15104 * 64 * 2 + 16 * 15104 * 2
    # 2048 tokens of the same layer: 2·T·(nnz + r(m + n)) = 96.3 GFLOP
    assert bench.apply_flops(11008 * 2048, 11008, 4096, 64, 2048) == 96_301_219_840
    # 1024² f32 top-k split without a residual: read W, S (int32 col + f32 value), row pointers
    assert bench.topk_split_bytes(1024, 1024, 52_428, 4, 4) - 1024 * 1024 * 4 == \
        1024 * 1024 * 4 + 52_428 * 8 + 1025 * 4
    assert bench.nm24_split_bytes(11008, 4096, 2, 2) == \
        2 * 11008 * 4096 * 2 + 11008 * 2048 * 2 + 11008 * 1024
