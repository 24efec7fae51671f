"""Host logic of bench.py that needs no GPU: the code hash that keys the stored ncu
traffic of a kernel to its source (an edit of comments alone keeps the counters, an
edit of code drops them)."""
import bench


def test_code_text_drops_comments_and_keeps_literals():
    src = ('int a = 1; // trailing\n'
           '/* block\n   comment */ int b = 2;\n'
           'const char *s = "x//y /* z */";\n'
           "char q = '\"'; // after a quote character\n"
           '\n   \n'
           'asm("{\\n\\t.reg .b32 rx; // inside the string\\n}");\n')
    t = bench.code_text(src)
    assert "trailing" not in t and "block" not in t and "after a quote" not in t
    assert '"x//y /* z */"' in t
    assert "// inside the string" in t
    assert "int a = 1;" in t and "int b = 2;" in t and "char q = '\"';" in t
    assert "\n\n" not in t


def test_file_hash_ignores_comment_edits_only(tmp_path):
    f = tmp_path / "k.cu"
    f.write_text("// v1\n__global__ void k(int *p) { p[0] = 1; }  // store\n")
    h0 = bench.file_hash([str(f)])
    f.write_text("// v2: reworded\n\n__global__ void k(int *p) { p[0] = 1; }  /* the store */\n")
    assert bench.file_hash([str(f)]) == h0
    f.write_text("// v2: reworded\n__global__ void k(int *p) { p[0] = 2; }\n")
    assert bench.file_hash([str(f)]) != h0


def test_traffic_lookup_follows_the_source_hash(tmp_path, monkeypatch):
    import json
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    entry = {"bytes_per_launch": 1234, "source_hash": bench.file_hash([str(src)]), "capture": "test"}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"kern:wl": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "kern", [str(src)])
    assert bench.kernel_traffic("kern", "wl") == 1234
    assert bench.kernel_traffic("kern", "other") is None
    src.write_text("// a comment\n__global__ void k() {}\n")
    assert bench.kernel_traffic("kern", "wl") == 1234
    src.write_text("__global__ void k() { __syncthreads(); }\n")
    assert bench.kernel_traffic("kern", "wl") is None
