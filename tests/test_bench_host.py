"""Host-side pieces of bench.py: the source hash that ties profile figures to code, and the
lookup of committed DRAM traffic (no GPU)."""
import json

import bench


def _tree(tmp_path, src):
    d = tmp_path / "decode_persistent_block_b200" / "csrc"
    d.mkdir(parents=True)
    (d / "k.cu").write_text(src)
    return tmp_path


def test_source_hash_ignores_comments_and_whitespace_but_not_code(tmp_path, monkeypatch):
    hashes = []
    for i, src in enumerate(["int f(int a) { return a + 1; }\n",
                             "// header\nint f(int a) {  /* add one */\n    return a + 1;  // done\n}\n",
                             "int f(int a) { return a + 2; }\n"]):
        monkeypatch.setattr(bench, "ROOT", str(_tree(tmp_path / str(i), src)))
        hashes.append(bench.kernel_source_hash())
    assert hashes[0] == hashes[1] != hashes[2]


def test_committed_traffic_needs_the_current_source_hash(tmp_path, monkeypatch):
    root = _tree(tmp_path, "int g;\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    (root / "profiles").mkdir()
    entry = {"kernel_hash": bench.kernel_source_hash(), "dram_bytes_per_launch": 1234}
    (root / "profiles" / "traffic.json").write_text(json.dumps({"megakernel:llama1b": entry}))
    assert bench.committed_traffic("llama1b", "megakernel") == 1234
    assert bench.committed_traffic("llama3b", "megakernel") is None
    (root / "decode_persistent_block_b200" / "csrc" / "k.cu").write_text("int g2;\n")
    assert bench.committed_traffic("llama1b", "megakernel") is None

