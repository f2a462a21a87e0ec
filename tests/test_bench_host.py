"""bench.py's host-side pieces on the CPU: the workloads' host lists (head 0
first, one list per head for the per-head tile patterns), the config block of
the JSON line, argument checks, and the kernel-source hash that ties a
committed DRAM-traffic figure to the code it was measured on."""

import json
import os

import numpy as np
import pytest

import bench
from workloads import WORKLOADS


def test_host_lists_radial_and_generic():
    rp, ci, nl = bench.host_lists(WORKLOADS["tiny"])
    assert nl == 1 and rp.size == WORKLOADS["tiny"].nqb + 1 and rp[-1] == ci.size == 220
    w = WORKLOADS["generic"]
    rp, ci, nl = bench.host_lists(w)
    assert nl == w.heads and rp.size == w.heads * w.nqb + 1 and rp[-1] == ci.size
    assert np.all(np.diff(rp) >= 1)              # every row keeps its diagonal tile


def test_workload_config_names_the_workload():
    c = bench.workload_config(WORKLOADS["wan"], nnz=31248)
    assert c["workload"].startswith("wan:") and "21x1560" in c["workload"]
    assert c["nnz_blocks_per_head"] == 31248 and c["seq_len"] == 32760
    g = bench.workload_config(WORKLOADS["generic"], nnz=287806)
    assert g["workload"].startswith("generic:") and g["nnz_blocks_all_heads"] == 287806
    json.dumps(c), json.dumps(g)


@pytest.mark.parametrize("argv", [["--warmup", "2"], ["--workload", "generic", "--pass", "bwd"],
                                  ["--impl", "reference", "--pass", "module"]])
def test_argument_checks(argv):
    with pytest.raises(SystemExit) as e:
        bench.main(argv)
    assert e.value.code == 2


def test_traffic_figure_follows_the_kernel_source_hash():
    """A committed capture's DRAM bytes are reported only while the kernel
    source it was taken on is unchanged (comments aside); otherwise null."""
    for which, name in (("fwd", "attn_fwd_pair_sm100_wan_traffic.json"),
                        ("bwd", "attn_bwd_sm100_wan_traffic.json")):
        with open(os.path.join(bench.ROOT, "profiles", name)) as f:
            d = json.load(f)
        same = d["kernel_source_hash"] == bench.kernel_source_hash(which)
        assert bench.load_traffic("wan", which) == (d["dram_bytes_per_launch"] if same else None)
    assert bench.load_traffic("generic") is None   # no capture for that workload


def test_source_hash_ignores_comments():
    code = "int f(int x) {\n  return x + 1;  // one\n}\n"
    assert bench._code_only(code) == bench._code_only("/* doc */\n" + code.replace("one", "two"))
    assert bench._code_only(code) != bench._code_only(code.replace("+ 1", "+ 2"))


def test_computed_flops_counts_valid_rows_and_columns():
    """4 * D * (valid rows x valid columns) over every listed block, per head
    and batch item, against a per-token loop (ragged last block included)."""
    import block_sparse_attention_radial_b200 as bsa

    n, blk, D, B, H = 300, 64, 32, 2, 3
    nqb = -(-n // blk)
    rng = np.random.default_rng(3)
    for L in (1, H):
        m = rng.random((L * nqb, nqb)) < 0.5
        rp = np.zeros(L * nqb + 1, dtype=np.int64)
        rp[1:] = np.cumsum(m.sum(axis=1))
        ci = np.nonzero(m)[1]
        pairs = 0
        for r in range(L * nqb):
            qb = r % nqb
            for kb in ci[rp[r]:rp[r + 1]]:
                pairs += sum(1 for i in range(qb * blk, min(n, qb * blk + blk))
                             for j in range(kb * blk, min(n, kb * blk + blk)))
        per_list_heads = H if L == 1 else 1
        assert bsa.computed_flops(rp, ci, n, blk, D, B, H, L) == 4 * D * B * per_list_heads * pairs


def test_per_config_names_cover_the_metric_range():
    # the default run records the other forward configurations beside wan
    names = bench.PER_CONFIG
    assert set(names) == {"hunyuan", "long4x", "generic"}
    for name in names:
        w = WORKLOADS[name]
        assert w.n >= 32 * 1024 and w.block == 128 and w.head_dim == 128
    assert max(WORKLOADS[n].n for n in names) == 84 * 1560


def test_gemm_shapes_are_the_module_products():
    rows, C = 21 * 1560, 40 * 128
    s = bench.GEMM_SHAPES
    assert s["qkv"][:3] == (rows, 3 * C, C) and s["out"][:3] == (rows, C, C)
    assert s["dw_qkv"][:3] == (3 * C, C, rows) and s["dx"][:3] == (rows, C, 3 * C)
    assert all(m % 8 == 0 or not amn for m, n, k, amn, bmn in s.values())
