"""The recorded DRAM traffic that bench.py puts in its roofline lines: a record is keyed to a
hash of its kernel's code with comments and whitespace removed, so an edit to the code (not to
its comments) turns the figure into null instead of reporting a stale capture."""
import json

import bench
from sparse_attention_flux_b200 import record_traffic as rt

KERNEL = """// a kernel
__global__ void k(int* x) {  /* body */
  x[0] = 1;   // store
}
"""


def _write(tmp_path, name, text):
    p = tmp_path / name
    p.write_text(text)
    return str(p)


def test_code_of_drops_comments_and_whitespace():
    assert rt.code_of("a /* x\n y */ b // z\n  c\td") == "abcd"
    assert rt.code_of(KERNEL) == "__global__voidk(int*x){x[0]=1;}"


def test_hash_ignores_comments_and_layout_but_not_code(tmp_path):
    base = rt.sources_sha256([_write(tmp_path, "a.cu", KERNEL)])
    relaid = KERNEL.replace("// store", "// the only store").replace("  x[0]", "\n\n    x[0]")
    assert rt.sources_sha256([_write(tmp_path, "b.cu", relaid)]) == base
    edited = KERNEL.replace("x[0] = 1", "x[0] = 2")
    assert rt.sources_sha256([_write(tmp_path, "c.cu", edited)]) != base


def test_bench_reports_a_record_only_while_its_code_is_unchanged(tmp_path, monkeypatch):
    src = _write(tmp_path, "k.cu", KERNEL)
    (tmp_path / "profiles").mkdir()
    rec = {"kern": {"bytes_per_launch": 1234, "sources": [src],
                    "sources_sha256": rt.sources_sha256([src])}}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("kern") == 1234
    assert bench.recorded_traffic("other") is None
    with open(src, "a") as f:
        f.write("// a comment only\n")
    assert bench.recorded_traffic("kern") == 1234
    with open(src, "a") as f:
        f.write("__device__ int y;\n")
    assert bench.recorded_traffic("kern") is None


def test_committed_records_are_consistent():
    with open(rt.RECORD) as f:
        rec = json.load(f)
    assert {"prefill_fa_T65536", "prefill_sa_T65536", "decode_fa_B16_S131072"} <= set(rec)
    for key, r in rec.items():
        assert r["bytes_per_launch"] == int(round((r["dram_bytes_read"] + r["dram_bytes_write"]) *
                                                  r["scale"])), key
        assert r["sources"] and len(r["sources_sha256"]) == 64, key
        assert r["capture"].startswith("profiles/"), key
