"""Host logic of bench.py's recorded DRAM traffic: a line of
profiles/dram_traffic.txt counts only while the sources of its kernel family
hash as at the capture."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_recorded_lines_count_only_while_current():
    """Every committed line names a known kernel family, a 12-digit source
    hash and a positive byte count; the bench uses exactly the lines whose
    family still hashes as at the capture (a stale line reads as null)."""
    got = bench.recorded_traffic()
    lines = [ln.split() for ln in open(os.path.join(ROOT, "profiles", "dram_traffic.txt"))
             if ln.strip() and not ln.startswith("#")]
    assert lines
    current = set()
    for p in lines:
        fam = bench.family_of(p[0])
        assert fam is not None, p[0]
        assert len(p[1]) == 12 and all(c in "0123456789abcdef" for c in p[1]), p
        assert float(p[3]) > 0, p
        if p[1] == bench.family_hash(fam):
            current.add(p[0])
    assert set(got) == current


def test_families_and_stale_lines(tmp_path):
    assert bench.family_of("prefill_paged_chunks8") == "prefill"
    assert bench.family_of("decode_fp8_decode64") == "decode_fp8"
    assert bench.family_of("decode_decode64") == "decode"
    assert bench.family_of("fp8_prepare_gqa4k") == "fp8_prepare"
    assert bench.family_of("bwd_gqa4k") == "bwd"
    assert bench.family_of("something_else") is None
    good = bench.family_hash("decode")
    f = tmp_path / "t.txt"
    f.write_text("# header\n"
                 f"decode_decode64 {good} decode64 123\n"
                 "bwd_gqa4k 000000000000 gqa4k 456\n"
                 "unknown_key 111111111111 x 7\n")
    assert bench.recorded_traffic(str(f)) == {"decode_decode64": 123.0}
