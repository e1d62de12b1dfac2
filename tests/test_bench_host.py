"""Host-side logic of bench.py that decides what a number means: the replica
sets that keep every timed step streaming from HBM, and the source digest that
decides whether a recorded DRAM traffic figure still describes the kernel."""
import bench
from bit_quantized_linear_svdq_b200 import synthetic


def test_replica_sets_exceed_twice_l2_for_every_bench_workload():
    for name in synthetic.CONFIGS:
        if name.startswith("tiny"):
            continue                      # parity-only case, never a bench line
        ck = synthetic.load(name)
        ns = bench.n_sets(ck)
        assert ns >= 8
        assert ns * bench.set_bytes(ck) >= 2 * bench.L2_BYTES, name
        assert "> 126 MB L2" in bench.config_of(ck)["l2"]


def test_tiny_workload_says_it_fits_in_l2():
    ck = synthetic.load("tiny_16x256x256_r32")
    assert "fits in the 126 MB L2" in bench.config_of(ck)["l2"]


def test_source_digest_follows_device_headers_only(tmp_path):
    (tmp_path / "k.cu").write_text('#include "a.cuh"\n#include "decl.h"\nkernel body\n')
    (tmp_path / "a.cuh").write_text('#include "b.cuh"\ndevice helper\n')
    (tmp_path / "b.cuh").write_text("inner helper\n")
    (tmp_path / "decl.h").write_text("host declarations\n")
    d0 = bench.source_digest(str(tmp_path / "k.cu"))
    (tmp_path / "decl.h").write_text("host declarations, one more\n")
    assert bench.source_digest(str(tmp_path / "k.cu")) == d0
    (tmp_path / "b.cuh").write_text("inner helper, changed\n")
    d1 = bench.source_digest(str(tmp_path / "k.cu"))
    assert d1 != d0
    (tmp_path / "k.cu").write_text('#include "a.cuh"\n#include "decl.h"\nkernel body, changed\n')
    assert bench.source_digest(str(tmp_path / "k.cu")) != d1



def test_gemm_roofline_bound_follows_rows():
    """Few rows read the weights (HBM-bound); the headline shape is a dense
    contraction (tensor-bound); the crossover sits between M = 256 and 1024
    at K = N = 4096 with the measured peaks (6553 GB/s, 8120 TFLOP/s)."""
    hbm, fp4 = 6553.0, 8120.0
    assert bench.gemm_roofline_bound(1, 4096, 4096, 32, hbm, fp4) == "hbm"
    assert bench.gemm_roofline_bound(16, 4096, 4096, 32, hbm, fp4) == "hbm"
    assert bench.gemm_roofline_bound(256, 4096, 4096, 32, hbm, fp4) == "hbm"
    assert bench.gemm_roofline_bound(1024, 4096, 4096, 32, hbm, fp4) == "tensor"
    assert bench.gemm_roofline_bound(4096, 3072, 3072, 32, hbm, fp4) == "tensor"
