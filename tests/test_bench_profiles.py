"""bench.py's reading of the committed ncu summaries: the code digest ignores
comments and white space but not code, and a summary whose digest no longer
matches its source yields no traffic figure."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_code_digest_ignores_comments_but_not_code(tmp_path):
    bench = _bench()
    a = tmp_path / "a.cu"
    a.write_text("int f(int x) {\n  return x + 1;  // one more\n}\n/* block\n comment */\n")
    b = tmp_path / "b.cu"
    b.write_text("// a header\nint f(int x) { return x + 1; }\n")
    c = tmp_path / "c.cu"
    c.write_text("int f(int x) { return x + 2; }\n")
    assert bench.code_digest(str(a)) == bench.code_digest(str(b))
    assert bench.code_digest(str(a)) != bench.code_digest(str(c))


def test_committed_summaries_match_their_sources():
    """Every summary the bench reads belongs to the current kernel code (else
    its traffic would be reported as null)."""
    bench = _bench()
    for kernel, workload in [("kahan_sgd_vec", "kahan_sgd"), ("sr_round_vec", "sr_round"),
                             ("step_fused", "product3m_fp8"), ("step_fused", "product3m_fp8_ge5m2"),
                             ("step_fused", "product3m_e5m2"), ("step_fused", "text500k_bf16"),
                             ("step_fused", "keyword8m6_bf16"), ("topk_screen_tc", "topk5_3m_fp8")]:
        tr = bench.profiled_traffic(kernel, workload)
        assert tr is not None, f"profiles/{kernel}_{workload}.md does not match its source"
        assert tr["bytes"] > 0 and tr["labels"] > 0


def test_stale_summary_gives_no_traffic(tmp_path, monkeypatch):
    bench = _bench()
    src = tmp_path / "k.cu"
    src.write_text("int k() { return 1; }\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k_w.md").write_text(f"- source: k.cu {bench.code_digest(str(src))}\n- labels per launch: 10\n"
                                 "- dram bytes per launch: 1000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k", "w") == {"bytes": 1000.0, "labels": 10}
    src.write_text("int k() { return 2; }\n")                 # the kernel changed since the capture
    assert bench.profiled_traffic("k", "w") is None
