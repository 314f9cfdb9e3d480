"""The benchmark's byte model against the page's KV-bytes example and small
hand counts."""
from conftest import read_golden
from paged_kv_cache_367_b200 import roofline


def test_kv_bytes_per_token_matches_the_page():
    g = read_golden("kv_bytes_per_token.txt")
    per_tok = roofline.kv_bytes_per_token(g["num_layers"], g["num_kv_heads"], g["head_dim"],
                                          g["elem_bytes"])
    assert per_tok == g["formula_bytes_per_token"]
    assert per_tok * g["context_tokens"] == g["formula_context_bytes"]
    # The page's printed totals are exactly twice the formula's product.
    assert g["page_printed_bytes_per_token"] == 2 * per_tok
    ctx_gib = g["page_printed_bytes_per_token"] * g["context_tokens"] / 1024**3
    assert abs(ctx_gib / g["page_printed_context_gb"] - 1) < 0.05   # the page rounds


def test_decode_bytes_hand_count():
    # 2 sequences of 5 and 16 tokens, Hq 4, Hkv 2, D 8, bs 4, bf16 Q, fp8 KV
    b = roofline.decode_bytes([5, 16], 4, 2, 8, 4, 2, 1)
    kv = 2 * 21 * 2 * 8 * 1
    qo = 2 * 2 * 4 * 8 * 2
    bt = 4 * (2 + 4)
    assert b == kv + qo + bt + 4 * 2


def test_shared_prefix_counts_prefix_once():
    a = roofline.decode_bytes([1024 + 10, 1024 + 20, 1024 + 30], 8, 2, 16, 16, 2, 1,
                              shared_prefix_tokens=1024)
    b = roofline.decode_bytes([1024 + 10, 1024 + 20, 1024 + 30], 8, 2, 16, 16, 2, 1)
    assert b - a == 2 * 1024 * 2 * 2 * 16 * 1


def test_append_bytes():
    assert roofline.append_bytes(64, 40, 128, 2, 2) == 2 * 64 * 40 * 128 * 4 + 8 * 64


def test_profiled_traffic_ignores_comment_edits_but_not_code_edits(tmp_path, monkeypatch):
    # The DRAM bytes of a committed ncu summary stay valid across a comment edit
    # of the decode sources and are dropped (null) once the code changes.
    import shutil
    import bench
    root = tmp_path / "repo"
    shutil.copytree(bench.ROOT + "/paged_kv_cache_367_b200/csrc", root / "paged_kv_cache_367_b200/csrc")
    shutil.copytree(bench.ROOT + "/include", root / "include")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.source_sha()
    (root / "profiles/ncu_decode_w.md").write_text(
        f"source_sha: {sha}\ntraffic_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic("w") == 1234.0
    src = root / "paged_kv_cache_367_b200/csrc/decode_tc.cu"
    text = src.read_text()
    src.write_text("// a new comment line\n" + text.replace("\n", "  \n", 3) + "/* and a block */\n")
    assert bench.source_sha() == sha and bench.profiled_traffic("w") == 1234.0
    src.write_text(text + "\nstatic int pkv_extra_symbol = 1;\n")
    assert bench.source_sha() != sha and bench.profiled_traffic("w") is None
