"""Every committed profile summary and traffic line names the digest of the kernel sources
it was captured on (bench.source_digest); a kernel change without a new capture leaves a
stale figure behind, which this host test reports."""
import glob
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_profile_summaries_match_the_current_kernel_sources():
    seen = 0
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.txt"))):
        for m in re.finditer(r'source_digest\("(\w+)"\)\): (\w+)', open(path).read()):
            seen += 1
            assert bench.source_digest(m.group(1)) == m.group(2), (os.path.basename(path), m.group(1))
    assert seen >= 6


def test_traffic_lines_match_the_current_kernel_sources():
    n = 0
    for ln in open(os.path.join(ROOT, "profiles", "traffic.txt")):
        if ln.startswith("#") or not ln.strip():
            continue
        kernel, workload, digest, value = ln.split()[:4]
        assert bench.source_digest(kernel) == digest, kernel
        assert bench.recorded_traffic(kernel, workload) == float(value)
        n += 1
    assert n >= 4
