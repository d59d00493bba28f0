"""Host-side pieces of bench.py that need no GPU."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_code_tokens_drops_comments_and_layout_only():
    a = "int f(int x) {  // twice\n  return x * 2; /* doubled */\n}\n"
    b = "int f(int x)\n{\n    return x * 2;\n}"
    assert bench.code_tokens(a) == bench.code_tokens(b)
    assert bench.code_tokens(a) != bench.code_tokens(a.replace("2;", "3;"))


def test_code_tokens_keeps_literals():
    s = 'asm("mov.u32 %0, 1; // not a comment" : "=r"(x)); char c = \'"\';'
    t = bench.code_tokens(s)
    assert "// not a comment" in t
    assert "'\"'" in t
    assert bench.code_tokens('p = "a\\"//b";') == 'p = "a\\"//b";'


def test_recorded_traffic_follows_kernel_code():
    """The committed decode traffic record is used only while its recorded
    digest matches the kernel code in the tree."""
    import json
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    bytes_, src = bench.decode_traffic([2, 4])
    if rec["source_digest"] == bench.source_digest():
        per = rec["bytes_per_launch"]
        assert bytes_ == (per["2bit"] + per["4bit"]) // 2
    else:
        assert bytes_ is None and "changed" in src


def test_traffic_record_missing_or_other_kernel(tmp_path):
    import json
    assert bench.decode_traffic([2], path=str(tmp_path / "absent.json"))[0] is None
    p = tmp_path / "t.json"
    p.write_text(json.dumps({"source_digest": bench.source_digest(), "bytes_per_launch": {"2bit": 10, "4bit": 30}}))
    assert bench.decode_traffic([2, 4, 4], path=str(p)) == (23, "profiles/decode_traffic.json")
    assert bench.decode_traffic([8], path=str(p))[0] is None
    p.write_text(json.dumps({"source_digest": "0" * 16, "bytes_per_launch": {"2bit": 10}}))
    assert bench.decode_traffic([2], path=str(p))[0] is None


def test_host_cores_respects_quota_and_cap(tmp_path):
    f = tmp_path / "cpu.max"
    avail = len(os.sched_getaffinity(0))
    f.write_text("max 100000\n")
    assert bench.host_cores(cap=1000, cpu_max=str(f)) == avail
    f.write_text("150000 100000\n")  # 1.5 CPUs of quota -> 2 threads
    assert bench.host_cores(cap=1000, cpu_max=str(f)) == min(avail, 2)
    assert bench.host_cores(cap=1, cpu_max=str(tmp_path / "absent")) == 1
