"""Host logic behind the benchmark's DRAM traffic records (no GPU).

A record in profiles/dram_traffic.json holds the bytes one ncu capture measured
for a kernel, keyed by a hash of the code that capture ran; bench.py reports
the record only while the kernel's code still hashes the same.  Comments and
blank lines are not code: editing them must keep a record valid, editing code
must not.
"""
import bench


SRC = """// header comment
__global__ void k(float* x) {   // trailing comment
  /* block
     comment */ x[0] = 1.f;

  x[1] = 2.f;  /* inline */
}
"""


def test_code_only_drops_comments_and_blank_lines():
    assert bench._code_only(SRC) == "__global__ void k(float* x) {\n   x[0] = 1.f;\n  x[1] = 2.f;\n}"


def test_comment_edit_keeps_the_code_equal():
    edited = SRC.replace("// trailing comment", "// another remark").replace("block\n     comment", "rewritten")
    assert bench._code_only(edited) == bench._code_only(SRC)


def test_code_edit_changes_it():
    assert bench._code_only(SRC.replace("2.f", "3.f")) != bench._code_only(SRC)


def test_source_hash_is_stable_and_per_kernel():
    a = bench.kernel_source_sha("attn_fwd_kernel")
    assert a == bench.kernel_source_sha("attn_fwd_kernel") and len(a) == 16
    assert a != bench.kernel_source_sha("pool_kernel")
