"""Host-side rules of bench.py (CPU): the source hash behind the ncu traffic
figure ignores comments and blank space but not code, and the whole-job
throughput is all ranks' work over the slowest rank's time."""
import bench


def test_code_only_hash_ignores_comments_not_code():
    a = "int f(int x) {  // doubles x\n  return 2 * x;  /* twice */\n}\n"
    b = "// a comment line\nint f(int x) {\n\n  return 2 * x;\n}\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_aggregate_uses_the_slowest_rank():
    value, ms_per_step = bench.aggregate([90.0, 120.0, 100.0], [1e12] * 3, 10)
    assert ms_per_step == 12.0
    assert value == 3e12 / 0.120
