"""Host-side logic of bench.py (no GPU): the DRAM-traffic figure is attached
only while the profiled kernel's code is the one it was measured on."""
import json
import os
import shutil

import bench


def _copy_tree(tmp_path):
    root = tmp_path / "r"
    shutil.copytree(os.path.join(bench.ROOT, "compressed_domain_attention_tq_b200", "csrc"),
                    root / "compressed_domain_attention_tq_b200" / "csrc")
    (root / "profiles").mkdir()
    return root


def test_source_hash_ignores_comments_and_layout(tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    before = bench.kernel_source_hash("decode")
    src = root / "compressed_domain_attention_tq_b200" / "csrc" / "decode_mma.cu"
    text = src.read_text()
    src.write_text("// a note\n" + text.replace("\n", "\n\n", 3) + "\n/* trailing */\n")
    assert bench.kernel_source_hash("decode") == before
    src.write_text(text.replace("kWaitCycles = 4000000000LL", "kWaitCycles = 4000000001LL"))
    assert bench.kernel_source_hash("decode") != before


def test_traffic_attached_only_for_matching_code_and_workload(tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    entry = {"source_hash": bench.kernel_source_hash("decode"), "workload_name": "w128",
             "dram_bytes_per_launch": 123}
    (root / "profiles" / "traffic.json").write_text(json.dumps({"decode": entry}))
    assert bench.ncu_traffic("decode", "w128") == 123
    assert bench.ncu_traffic("decode", "other") is None
    assert bench.ncu_traffic("quantize_bulk", "w128") is None
    src = root / "compressed_domain_attention_tq_b200" / "csrc" / "tq_api.cu"
    src.write_text(src.read_text().replace("per_item_cost = mma ? 384 : 256",
                                           "per_item_cost = mma ? 385 : 256"))
    assert bench.ncu_traffic("decode", "w128") is None
