"""Host logic of bench.py that needs no GPU: the device-code hash that keeps a recorded DRAM
traffic figure tied to the kernel source it was captured on, and the lookup of that figure."""
import os
import re

import bench

KERNEL_SRC = """// kernel file
__global__ void k(int* p) {  // one thread
    p[0] = 1;  /* store */
}
"""


def test_device_hash_ignores_comments_and_whitespace():
    a = bench.device_source_sha("", text=KERNEL_SRC)
    b = bench.device_source_sha("", text=KERNEL_SRC.replace("// one thread", "// a different comment")
                                .replace("    p[0]", "\tp[0]").replace("/* store */", ""))
    assert a == b


def test_device_hash_changes_with_the_code():
    a = bench.device_source_sha("", text=KERNEL_SRC)
    assert bench.device_source_sha("", text=KERNEL_SRC.replace("p[0] = 1", "p[0] = 2")) != a


def test_device_hash_ignores_the_host_side():
    host = "\n" + bench.HOST_SIDE_MARKER + "\nint launch() { return 0; }\n"
    a = bench.device_source_sha("", text=KERNEL_SRC + host)
    b = bench.device_source_sha("", text=KERNEL_SRC + host.replace("return 0", "return 1"))
    assert a == b == bench.device_source_sha("", text=KERNEL_SRC)


def _write_profile(root, key, source, nbytes, sha):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "k.md"), "w") as f:
        f.write("# summary\n\ntraffic[%s]: bytes=%d source=%s device_sha=%s\n" % (key, nbytes, source, sha))


def test_traffic_figure_only_for_the_captured_source(tmp_path, monkeypatch):
    root = str(tmp_path)
    src = os.path.join(root, "k.cu")
    with open(src, "w") as f:
        f.write(KERNEL_SRC)
    monkeypatch.setattr(bench, "ROOT", root)
    _write_profile(root, "kern_w", "k.cu", 1234, bench.device_source_sha(src))
    assert bench.profile_traffic("kern_w") == 1234.0
    assert bench.profile_traffic("other_kernel") is None
    with open(src, "a") as f:  # a comment: still the captured code
        f.write("// note\n")
    assert bench.profile_traffic("kern_w") == 1234.0
    with open(src, "w") as f:  # changed code: the figure no longer applies
        f.write(KERNEL_SRC.replace("p[0] = 1", "p[0] = 3"))
    assert bench.profile_traffic("kern_w") is None


def test_committed_traffic_lines_parse_and_name_kernel_sources():
    here = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pat = re.compile(r"^traffic\[(\w+)\]: bytes=(\d+) source=(\S+) device_sha=([0-9a-f]{16})$")
    found = 0
    for name in sorted(os.listdir(os.path.join(here, "profiles"))):
        for line in open(os.path.join(here, "profiles", name)):
            if line.startswith("traffic["):
                m = pat.match(line.strip())
                assert m, "%s: malformed traffic line %r" % (name, line)
                assert int(m.group(2)) > 0
                assert os.path.exists(os.path.join(here, m.group(3))), m.group(3)
                found += 1
    assert found >= 1


def test_nvml_index_follows_visible_devices(monkeypatch):
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    assert bench.nvml_index(3) == 3
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "4,6")
    assert bench.nvml_index(0) == 4 and bench.nvml_index(1) == 6
    assert bench.nvml_index(5) == 5  # beyond the list: the ordinal
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-00000000-0000-0000-0000-000000000000")
    assert bench.nvml_index(0) == 0  # a UUID NVML cannot resolve here: the ordinal
