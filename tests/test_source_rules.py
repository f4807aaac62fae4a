"""Guards on the CUDA sources, checked on the CPU:
- no TMA or bulk load with cluster multicast (the library's loads read this
  GPU's own memory; multicast is kept out so that nothing multi-GPU can reach
  such a load);
- none of the batched-copy runtime/driver calls (issue one async copy per
  buffer instead);
- every kernel wait on an mbarrier goes through the bounded helper."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixture_experts_layer_44_b200", "csrc")


def _sources():
    out = {}
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name), encoding="utf-8") as f:
                out[name] = f.read()
    with open(os.path.join(ROOT, "include", "moe_b200.h"), encoding="utf-8") as f:
        out["moe_b200.h"] = f.read()
    return out


def test_no_multicast_loads():
    pat = re.compile(r"multicast" + "::" + "cluster")
    for name, src in _sources().items():
        assert not pat.search(src), name


def test_no_batched_copy_calls():
    names = ["Memcpy" + "Batch" + "Async", "Memcpy3D" + "Batch" + "Async"]
    for name, src in _sources().items():
        for n in names:
            assert n not in src, (name, n)


def test_mbarrier_waits_are_bounded():
    # the only raw try_wait loop is the bounded helper in sm100_ptx.cuh
    for name, src in _sources().items():
        if name == "sm100_ptx.cuh":
            continue
        assert "mbarrier.try_wait" not in src, name
        assert not re.search(r"while\s*\(\s*!\s*moe::mbar_try_wait", src), name
