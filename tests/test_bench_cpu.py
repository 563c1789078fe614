"""The bench's host-side measurement logic on CPU: the roofline arithmetic,
the algorithmic bytes per token-head from the tensors each pass touches,
and the traffic figures reported only while the kernel sources are the
ones they were captured on."""
import json
import os
import shutil

import bench

TH_BYTES = 2 * 128   # one bf16 row of 128 values per token-head


def test_bytes_per_token_head_from_the_tensors_touched():
    # each attention pass reads three [.., 128] bf16 tensors and writes one
    for name in ("tc_fwd", "tc_dq", "tc_dv", "tc_dk"):
        assert bench.BYTES_PER_TH[name] == 4 * TH_BYTES
    assert bench.BYTES_PER_TH["simt_dkdv"] == 6 * TH_BYTES     # q, k, v, dO in; dk, dv out
    # forward: q, k, v in, o out; backward: q, k, v, dO in, dq, dk, dv out
    assert bench.FWD_BWD_MIN_BYTES == (4 + 7) * TH_BYTES
    assert bench.FMAP_BYTES_PER_TH["feature_map"] == 4 * TH_BYTES        # q, k in; phi_q, phi_k out
    assert bench.FMAP_BYTES_PER_TH["feature_map_grad"] == 6 * TH_BYTES   # q, k, dphi_q, dphi_k; dq, dk


def test_hbm_roofline_arithmetic():
    pk = {"hbm_gbs": 6500.0, "source": "measured"}
    rec = {"launches": 4, "ms": 2.0}                     # 0.5 ms per launch
    r = bench.hbm_roofline("feature_map_grad", rec, 1536, 2_097_152, pk, traffic=123.0)
    alg = 1536 * 2_097_152
    assert r["alg_bytes_per_launch"] == alg
    assert r["avg_launch_ms"] == 0.5
    assert abs(r["achieved"] - alg / 0.5e-3 / 1e9) < 0.1
    assert abs(r["frac"] - r["achieved"] / 6500.0) < 1e-4
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 123.0


def test_traffic_only_for_the_captured_sources(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(bench.ROOT, "causal_linear_attention_fwd_b200", "csrc"),
                    root / "causal_linear_attention_fwd_b200" / "csrc")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    h = bench.kernel_source_hash("tc")
    rec = {"source_hashes": {"tc": h},
           "kernels": {"tc_fwd": {"dram_bytes_per_token_head": 1013.0}}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_for("tc_fwd", 1000) == 1013.0 * 1000
    assert bench.traffic_for("tc_dq", 1000) is None                  # not captured
    csrc = root / "causal_linear_attention_fwd_b200" / "csrc"
    # a change outside the tensor-core kernels' sources leaves the figures
    f = csrc / "la2_fmap.cuh"
    f.write_text(f.read_text() + "\n")
    assert bench.kernel_source_hash("tc") == h
    assert bench.traffic_for("tc_fwd", 1000) == 1013.0 * 1000
    # any change to the tensor-core kernels' sources retires them
    f = csrc / "la2_tc.cuh"
    f.write_text(f.read_text() + "\n")
    assert bench.kernel_source_hash("tc") != h
    assert bench.traffic_for("tc_fwd", 1000) is None


def test_source_groups_name_existing_files():
    csrc = os.path.join(bench.ROOT, "causal_linear_attention_fwd_b200", "csrc")
    for group, files in bench.SOURCE_GROUPS.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (group, f)
    assert bench.group_of("tc_dv") == "tc" and bench.group_of("decode_step") == "decode"
    assert bench.group_of("feature_map_grad") == "fmap"
