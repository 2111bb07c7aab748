"""bench.py host logic without a GPU: the DRAM traffic a bench line carries
comes from a committed ncu summary only while the kernel sources it was
captured from are unchanged."""
import importlib.util
import os
import shutil

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_every_profiled_line_is_consistent():
    # each summary the bench reads exists and names a traffic figure and a
    # source hash; the lookup returns that figure exactly when the hash of the
    # listed sources is the one recorded, and null otherwise
    b = _bench()
    for key, (prof, sources) in b.PROFILE_TRAFFIC.items():
        assert os.path.exists(prof), prof
        assert all(os.path.exists(s) for s in sources), key
        fields = {}
        for line in open(prof):
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip()
        assert int(fields["dram_bytes_per_launch_full_size"]) > 0, key
        recorded = fields["kernel_source_sha256_16"]
        t = b.profiled_traffic(key)
        if recorded == b.source_sha(sources):
            assert t == float(fields["dram_bytes_per_launch_full_size"]), key
        else:
            assert t is None, key


def test_traffic_is_dropped_when_a_source_changes(tmp_path):
    b = _bench()
    _, sources = b.PROFILE_TRAFFIC["decode"]
    copies = []
    for s in sources:
        d = tmp_path / os.path.basename(s)
        shutil.copy(s, d)
        copies.append(str(d))
    prof = tmp_path / "summary.md"
    prof.write_text("# a summary\n\n- dram_bytes_per_launch_full_size: 12345\n"
                    f"- kernel_source_sha256_16: {b.source_sha(copies)}\n")
    b.PROFILE_TRAFFIC["decode"] = (str(prof), copies)
    assert b.profiled_traffic("decode") == 12345.0
    with open(copies[0], "a") as f:
        f.write("\n// edited\n")
    assert b.profiled_traffic("decode") is None


def test_unknown_or_missing_profile_gives_none(tmp_path):
    b = _bench()
    assert b.profiled_traffic("no-such-path") is None
    b.PROFILE_TRAFFIC["decode"] = (str(tmp_path / "missing.md"), b.PROFILE_TRAFFIC["decode"][1])
    assert b.profiled_traffic("decode") is None
