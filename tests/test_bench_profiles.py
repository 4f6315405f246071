"""bench.py's use of the committed ncu summaries (host only, no GPU)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_source_digest_ignores_comment_lines_only(tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("// header\n__global__ void k(int* x) {\n  x[0] = 1;  // one\n}\n")
    d0 = bench.source_digest(str(src))
    src.write_text("// header, reworded\n\n__global__ void k(int* x) {\n  // a note\n  x[0] = 1;  // one\n}\n")
    assert bench.source_digest(str(src)) == d0
    src.write_text("// header\n__global__ void k(int* x) {\n  x[0] = 2;  // one\n}\n")
    assert bench.source_digest(str(src)) != d0
    src.write_text("// header\n__global__ void k(int* x) {\n  x[0] = 1;  // two\n}\n")
    assert bench.source_digest(str(src)) != d0  # trailing comments count


def test_committed_profiles_match_their_kernels():
    """Every committed digest names an existing source and a variant the
    bench reports; its traffic is used only for that variant, and only while
    the kernel source matches (else None)."""
    for wl in ("llama2_7b", "mistral_7b_gqa", "llama2_70b_beam"):
        with open(os.path.join(ROOT, "profiles", f"pa_decode_{wl}.json")) as f:
            prof = json.load(f)
        assert prof["variant"] in ("cuda_cores", "tensor_cores", "shared_prefix")
        assert os.path.exists(os.path.join(ROOT, prof["source"]))
        assert 0 < prof["traffic_over_algorithmic"] < 2
        t = bench.profiled_traffic(wl, prof["variant"], 1e9)
        fresh = bench.source_digest(os.path.join(ROOT, prof["source"])) == prof["source_sha256_16"]
        assert t == (int(round(prof["traffic_over_algorithmic"] * 1e9)) if fresh else None)
        assert bench.profiled_traffic(wl, "no_such_variant", 1e9) is None
