"""The traffic record's source key: comments and blank lines do not change it,
code does (host logic of bench.py, CPU only)."""
import bench


def test_source_hash_ignores_comments_only(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("// header\n__global__ void k(int *p) {\n    p[0] = 1;  // store\n}\n")
    b = tmp_path / "b.cu"
    b.write_text("/* a block\n   comment */\n__global__ void k(int *p) {\n\n    p[0] = 1;\n}\n// tail\n")
    c = tmp_path / "c.cu"
    c.write_text("__global__ void k(int *p) {\n    p[0] = 2;\n}\n")
    assert bench.source_hash(str(a)) == bench.source_hash(str(b))
    assert bench.source_hash(str(a)) != bench.source_hash(str(c))

