"""CPU checks of bench.py's algorithmic accounting (the numerators of the
reported TFLOP/s and GB/s), written out from the scope table's rules:
GEMM flops = 2*M*N*K per GEMM; a dual quantize of a bf16 tensor moves
2 bytes in and 2 bytes out per element plus the 96-byte ring.
"""

import bench


def test_gemm_flops_of_the_linear_step():
    M, H, F = 8192, 1536, 4096
    # per linear: forward M x N x H, dX M x H x N, dW N x H x M -- three GEMMs of 2*M*N*H flops
    want = sum(3 * 2 * M * n * H for n in (H, F))
    assert bench.gemm_flops(M) == want == 425_201_762_304


def test_quantize_bytes_of_the_linear_step():
    M, H, F = 8192, 1536, 4096
    per_call = lambda elems: elems * (2 + 2) + 96  # noqa: E731  bf16 in, two FP8 copies out, the ring
    want = 0
    for n in (H, F):
        want += per_call(M * H) + per_call(n * H) + per_call(M * n)  # X, W, G
    assert bench.quant_bytes(M) == want


def test_workload_config_names_the_step():
    cfg = bench.workload_config(8192, 1)
    assert cfg["M"] == 8192 and cfg["linears"] == [[1536, 1536], [4096, 1536]]
    assert "replicas x1" == cfg["parallelism"]
