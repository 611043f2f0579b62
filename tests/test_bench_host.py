"""Host-side logic of bench.py (no GPU): the ncu traffic records are used only while the
profiled kernel source is unchanged, and both arms describe the same workload."""
import hashlib
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_records_follow_the_source_hash():
    """The committed summaries carry the hash of the source they were captured on: while it
    matches, every recorded workload is returned; once it differs, none is."""
    import re
    for profile, source, names in (("attn_tc_kernel_decode_prefill_hca.md", "attn.cuh", ("flash64k_kv8", "pro1m_kv8")),
                                   ("attn_t_kernel_decode.md", "attn_t.cuh", ("flash64k", "pro1m")),
                                   ("index_tc_kernel_e4m3_decode.md", "index.cuh", ("flash64k", "pro1m")),
                                   ("index_tc_kernel_mxfp4_decode.md", "index.cuh", ("flash64k", "pro1m"))):
        text = open(os.path.join(ROOT, "profiles", profile)).read()
        rec = re.search(r"source_sha256_prefix=([0-9a-f]+)", text).group(1)
        src = open(os.path.join(ROOT, "long_context_compressed_b200", "csrc", source), "rb").read()
        current = hashlib.sha256(src).hexdigest()[:16] == rec
        for n in names:
            v = bench.profiled_traffic(profile, source, n)
            assert (isinstance(v, int) and v > 0) if current else v is None, (profile, n)
        assert bench.profiled_traffic(profile, source, "no_such_workload") is None


def test_traffic_is_null_once_the_source_changes(tmp_path, monkeypatch):
    """A traffic record keyed on a source's hash is used while that source is unchanged, and
    not once the source differs by one byte."""
    (tmp_path / "profiles").mkdir()
    (tmp_path / "long_context_compressed_b200" / "csrc").mkdir(parents=True)
    src = open(os.path.join(ROOT, "long_context_compressed_b200", "csrc", "attn.cuh"), "rb").read()
    h = hashlib.sha256(src).hexdigest()[:16]
    (tmp_path / "profiles" / "p.md").write_text(f"# x\ntraffic_bytes_per_launch: source_sha256_prefix={h} "
                                                f"flash64k=123456 pro1m=789\n")
    (tmp_path / "long_context_compressed_b200" / "csrc" / "attn.cuh").write_bytes(src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("p.md", "attn.cuh", "flash64k") == 123456
    assert bench.profiled_traffic("p.md", "attn.cuh", "pro1m") == 789
    (tmp_path / "long_context_compressed_b200" / "csrc" / "attn.cuh").write_bytes(src + b" ")
    assert bench.profiled_traffic("p.md", "attn.cuh", "flash64k") is None


def test_both_arms_share_the_workload_text():
    from long_context_compressed_b200 import synth
    wl = synth.WORKLOADS["flash64k"]
    t = bench.workload_text(wl, "e4m3", True)
    assert "flash64k" in t and "top-512" in t and "HCA layer" in t
    assert ("Hadamard" in t) == bench.INDEX_ROTATION
