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


def test_decode_traffic_is_close_to_the_algorithmic_bytes():
    # DRAM bytes of one launch from the ncu capture: within 2 % of the algorithmic
    # count, i.e. no operand is read twice
    assert abs(bench.DECODE_TRAFFIC_BYTES / bench.decode_bytes() - 1) < 0.02
