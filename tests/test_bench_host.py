"""Host-side pieces of bench.py that the JSON line's claims rest on (CPU only):
the kernel-launch count per forward and the config object shared by both arms."""
import bench
from block_sparse_linear_router_b200.inputs import WORKLOADS
from oracle import sla2_oracle as O


def test_launches_per_forward_follow_the_launch_sequence():
    # pool, column means, projections, logits, top-k, linear state, reduce, sparse,
    # selected-state product, epilogue
    w = WORKLOADS["wan1.3b"]
    assert bench.launches_per_forward(w, O.topk_count(w.nk, w.topk_frac)) == 10
    # every key block kept: no selected-state product
    assert bench.launches_per_forward(w, w.nk) == 9


def test_config_names_the_workload_and_is_truthful_about_l2():
    for name, w in WORKLOADS.items():
        k = O.topk_count(w.nk, w.topk_frac)
        c = bench.bench_config(w, k, 2)
        assert c["workload"].startswith(f"{name} B={w.B} H={w.H} N={w.N} d={w.d}")
        assert f"(k={k} of {w.nk})" in c["workload"]
        assert c["parallelism"] == "replicas x2"
        qkv = 3 * 2 * w.B * w.H * w.N * w.d
        assert ("> 126 MB L2" in c["l2"]) == (qkv / 1e6 > 126)
