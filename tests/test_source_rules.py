"""Static rules on the CUDA sources and the benchmark, checked on the CPU:
- no TMA or bulk load with cluster multicast (the library runs unchanged on
  several GPUs, where a multicast load could read another GPU's memory);
- no batched memcpy calls (named here only in pieces): copies are issued one
  by one or gathered by a kernel;
- no deliberate device faults: no trap instruction, no device-side assert
  (failures are reported through status words and the fault flags)."""
import glob
import os
import re

from conftest import ROOT

SOURCES = sorted(glob.glob(os.path.join(ROOT, "decode_packed_bit_b200", "csrc", "*.cu")) +
                 glob.glob(os.path.join(ROOT, "decode_packed_bit_b200", "csrc", "*.cuh")) +
                 [os.path.join(ROOT, "include", "lowbit.h"), os.path.join(ROOT, "bench.py")])


def _text(p):
    with open(p, encoding="utf-8") as f:
        return f.read()


def test_sources_found():
    assert len(SOURCES) >= 10


def test_no_multicast_loads():
    for p in SOURCES:
        assert "multicast::cluster" not in _text(p), p


def test_no_batched_memcpy():
    banned = ["cuda" + "Memcpy" + "BatchAsync", "cuda" + "Memcpy3D" + "BatchAsync",
              "cu" + "Memcpy" + "BatchAsync", "cu" + "Memcpy3D" + "BatchAsync"]
    for p in SOURCES:
        t = _text(p)
        for name in banned:
            assert name not in t, (p, name)


def test_no_deliberate_device_faults():
    for p in SOURCES:
        t = _text(p)
        assert "__trap" not in t, p
        assert not re.search(r"\btrap;", t), p
        if p.endswith((".cu", ".cuh")):
            assert not re.search(r"(?<![_\w])assert\s*\(", t), p
