"""The committed ncu summaries the bench reads its DRAM traffic from
(profiles/pa_decode_<workload>.json): each names a workload and a decode
variant the bench knows, a kernel source that exists, and a traffic ratio
that is its captured DRAM bytes over the captured step's algorithmic bytes.
(Whether the source digest still matches is the bench's business: it then
reports no traffic.)"""
import glob
import json
import os

import pytest

import bench
from paged_kv_cache_458_b200 import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "pa_decode_*.json")))


def test_every_workload_has_a_profile():
    names = {os.path.basename(p)[len("pa_decode_"):-len(".json")] for p in PROFILES}
    assert set(gen.WORKLOADS) - {"tiny"} <= names


@pytest.mark.parametrize("path", PROFILES, ids=lambda p: os.path.basename(p))
def test_profile_is_consistent(path):
    with open(path) as f:
        prof = json.load(f)
    assert prof["workload"] in gen.WORKLOADS
    assert prof["variant"] in ("cuda_cores", "tensor_cores", "shared_prefix")
    assert os.path.isfile(os.path.join(ROOT, prof["source"]))
    assert len(prof["source_sha256_16"]) == 16
    assert prof["dram_bytes_captured"] == prof["dram_bytes_read"] + prof["dram_bytes_write"]
    ratio = prof["dram_bytes_captured"] / prof["algorithmic_bytes_captured"]
    assert abs(ratio - prof["traffic_over_algorithmic"]) < 1e-3
    # the bench applies the ratio when the digest matches, and only then
    digest_ok = prof["source_sha256_16"] == bench.source_digest(os.path.join(ROOT, prof["source"]))
    got = bench.profiled_traffic(prof["workload"], prof["variant"], 1e9)
    assert (got is not None) == digest_ok
    assert bench.profiled_traffic(prof["workload"], "no_such_variant", 1e9) is None
